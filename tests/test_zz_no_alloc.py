"""moe_permute_noalloc: the dispatch stage for callers that cannot hand the library any
device memory (a plug-in whose host framework owns all device memory, a serving loop
that may not call cudaMalloc between launches).  It keeps its scratch in a fixed device
array inside the library, so these tests check that two calls in a row through the C
ABI give exactly what the workspace-based moe_permute gives, that a call too large for
that array is refused, and that bad expert ids are still reported.

This file is collected last so that a run stopping at its first failure has run every
other test; it also passes on its own in a fresh process."""
import numpy as np
import pytest
import torch

from mixture_experts_ffn_08_b200 import binding as B
from mixture_experts_ffn_08_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _ids(wl, seed):
    rng = np.random.default_rng(seed)
    return np.stack([rng.choice(wl.E, wl.K, replace=False) for _ in range(wl.T)]).astype(np.int32)


def _outputs(wl):
    rows = B.moe_max_padded_rows(B.params(wl))
    return dict(counts=torch.empty(wl.E, dtype=torch.int32, device="cuda"),
                offs=torch.empty(wl.E + 1, dtype=torch.int32, device="cuda"),
                rop=torch.empty(wl.T * wl.K, dtype=torch.int32, device="cuda"),
                por=torch.full((rows,), -7, dtype=torch.int32, device="cuda"),
                xp=torch.full((rows, wl.H), 3.0, dtype=torch.bfloat16, device="cuda"))


def _with_workspace(wl, ids, x):
    p = B.params(wl)
    ws = torch.empty(B.moe_workspace_size(p), dtype=torch.uint8, device="cuda")
    B.check(B.moe_clear_device_status(ws))
    o = _outputs(wl)
    B.check(B.moe_permute(p, ids, x, None, o["counts"], o["offs"], o["rop"], o["por"], o["xp"], None,
                          ws, ws.numel()))
    return o


def _without_workspace(wl, ids, x, status=None):
    o = _outputs(wl)
    B.check(B.moe_permute_noalloc(B.params(wl), ids, x, None, o["counts"], o["offs"], o["rop"],
                                  o["por"], o["xp"], None, status), "moe_permute_noalloc")
    return o


def _same(a, b, E):
    torch.cuda.synchronize()
    assert torch.equal(a["counts"], b["counts"])
    assert torch.equal(a["offs"], b["offs"])
    assert torch.equal(a["rop"], b["rop"])
    total = int(a["offs"][E].item())
    assert torch.equal(a["por"][:total], b["por"][:total])
    assert torch.equal(a["xp"][:total], b["xp"][:total])


def test_two_calls_in_a_row_match_the_workspace_entry_point():
    cases = [(W.Workload("na", T=3000, H=256, I=128, E=64, K=6), 0),
             (W.Workload("nb", T=700, H=512, I=128, E=256, K=8), 1)]
    inputs = [(wl, torch.as_tensor(_ids(wl, seed), device="cuda"),
               torch.randn((wl.T, wl.H), device="cuda").to(torch.bfloat16)) for wl, seed in cases]
    # two calls in a row: the second reuses the array the first one left behind
    got = [_without_workspace(wl, ids, x) for wl, ids, x in inputs]
    for (wl, ids, x), o in zip(inputs, got):
        _same(o, _with_workspace(wl, ids, x), wl.E)
        assert int(o["counts"].sum().item()) == wl.T * wl.K


def test_too_large_for_the_fixed_scratch_is_refused():
    wl = W.Workload("big", T=70000, H=128, I=128, E=1024, K=8)   # 2188 chunks x 1024 experts
    ids = torch.zeros((wl.T, wl.K), dtype=torch.int32, device="cuda")
    x = torch.zeros((wl.T, wl.H), dtype=torch.bfloat16, device="cuda")
    rc = B.moe_permute_noalloc(B.params(wl), ids, x, None, ids, ids, ids, ids, x, None, None)
    assert rc == 2
    torch.cuda.synchronize()


def test_bad_ids_reported_through_caller_status_word():
    wl = W.Workload("bad", T=100, H=128, I=128, E=8, K=2)
    ids_np = _ids(wl, 4)
    ids_np[3, 1] = 9
    ids = torch.as_tensor(ids_np, device="cuda")
    x = torch.randn((wl.T, wl.H), device="cuda").to(torch.bfloat16)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o = _without_workspace(wl, ids, x, status)
    torch.cuda.synchronize()
    assert int(status.item()) & B.MOE_DEV_BAD_EXPERT_ID
    assert int(o["rop"][3 * 2 + 1].item()) == -1
    _same(o, _with_workspace(wl, ids, x), wl.E)
