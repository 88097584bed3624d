"""Failure path without a GPU fault: a kernel that waits on an mbarrier nothing completes
gives up after its limit, reports MOE_DEV_TIMEOUT through the workspace status word, and
leaves the context usable for the next layer call."""
import time

import numpy as np
import pytest
import torch

from mixture_experts_ffn_08_b200 import binding as B
from mixture_experts_ffn_08_b200 import inputs, workloads as W
from oracle import moe_oracle as o
from tests import parity as P

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_reports_timeout():
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    B.check(B.moe_selftest_bounded_wait(ws, 50))
    status = B.moe_get_device_status(ws)   # synchronises
    dt = time.perf_counter() - t0
    assert status & B.MOE_DEV_TIMEOUT
    assert 0.04 <= dt < 1.5


def test_context_stays_usable_after_a_timeout():
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    B.check(B.moe_selftest_bounded_wait(ws, 20))
    assert B.moe_get_device_status(ws) & B.MOE_DEV_TIMEOUT
    wl = W.TINY
    d = inputs.make_inputs(wl, seed=9, device="cuda")
    res = P.run_layer(wl, d)
    assert B.moe_get_device_status(res["ws"]) == 0
    x = P.x_f64(d, wl)
    s = o.scores(o.router_logits(x, P.f64(d["w_r"])), wl.score_fn)
    gpu_ids = res["ids"].cpu().numpy()
    _, w_or = P.check_routing(gpu_ids, res["w"].cpu().numpy(), s, None, wl)
    ref = o.forward_given_routing(x, gpu_ids, w_or, P.expert_weights_fn(d, wl), wl.E, None, h_format="bf16")
    P.check_close(P.f64(res["out"]), ref, P.BF16_MAX_TOL, "after timeout")


def test_selftest_rejects_bad_limits():
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    assert B.moe_selftest_bounded_wait(ws, 0) == 1
    assert B.moe_selftest_bounded_wait(ws, 5000) == 1
