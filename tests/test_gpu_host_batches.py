"""moe_layer_forward_host_batches: several batches from and to host memory, with the
copies of neighbouring batches overlapping the layer, must give each batch exactly the
output of moe_layer_forward on the same inputs (the same kernels run on the same data)."""
import pytest
import torch

from mixture_experts_ffn_08_b200 import binding as B
from mixture_experts_ffn_08_b200 import inputs, workloads as W
from tests import parity as P

pytestmark = pytest.mark.gpu

CASES = {
    # shared expert on the side stream (decode-sized batch), bf16
    "dsv3_small": W.DSV3_PREFILL.with_(name="dsv3_small", T=200, H=512, I=256, E=32, I_shared=256),
    "mixtral_small": W.MIXTRAL_PREFILL.with_(name="mixtral_small", T=1000, H=512, I=384),
    "skewed_fp8_small": W.SKEWED_FP8.with_(name="skewed_fp8_small", T=600, H=512, I=384, E=16, K=4),
}


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("n_batches", [1, 2, 5])
def test_batches_match_the_device_entry_point(name, n_batches):
    wl = CASES[name]
    fp8 = wl.dtype == W.DTYPE_FP8
    d = inputs.make_inputs(wl, seed=0, device="cuda")
    a = P.device_inputs_ptrs(d, wl)
    # a different activation batch per step (the weights are the layer's)
    xs = [inputs.make_inputs(wl, seed=10 + b, device="cuda", weights=False) for b in range(n_batches)]
    ref = []
    for xb in xs:
        run = dict(d)
        run.update({k: xb[k] for k in (("x_q", "x_scale") if fp8 else ("x",))})
        ref.append(P.run_layer(wl, run)["out"].cpu())
    p = B.params(wl)
    ws = P.alloc_ws(p)
    x_host = [(xb["x_q"] if fp8 else xb["x"]).cpu().pin_memory() for xb in xs]
    s_host = [xb["x_scale"].cpu().pin_memory() for xb in xs] if fp8 else None
    out_host = [torch.empty((wl.T, wl.H), dtype=torch.bfloat16).pin_memory() for _ in xs]
    for _ in range(2):  # twice: the second call reuses the staging slots and events
        for o in out_host:
            o.fill_(float("nan"))
        B.check(B.moe_layer_forward_host_batches(p, x_host, s_host, a["w_r"], a["bias"], a["w_gate"], a["w_up"],
                                                 a["w_down"], a["w_gate_scale"], a["w_up_scale"], a["w_down_scale"],
                                                 a["ws_gate"], a["ws_up"], a["ws_down"], out_host, ws, ws.numel()),
                "moe_layer_forward_host_batches")
        torch.cuda.synchronize()
        assert B.moe_get_device_status(ws) == 0
        for b in range(n_batches):
            assert torch.equal(out_host[b], ref[b]), f"batch {b}"


def test_zero_batches_is_a_no_op():
    wl = CASES["mixtral_small"]
    p = B.params(wl)
    ws = P.alloc_ws(p)
    assert B.moe_layer_forward_host_batches(p, [], None, None, None, None, None, None, None, None, None, None,
                                            None, None, [], ws, ws.numel()) == B.MOE_OK
