"""Failure detection on the GPU without a fault: bounded waits give up, report, and leave the context usable.

1. A kernel waits (the pipelined kernels' bounded wait) on an mbarrier that nothing completes: after
   the limit the error word carries MOE_DEVERR_TIMEOUT, the call returns and the GPU keeps working.
2. The whole layer runs with every wait limited to 1 ns: the waits that do not complete at once give
   up, every role of every CTA stops (copies and MMAs already issued are drained first, TMEM is freed),
   and the error word reports the timeout. The output of such a call is undefined and is not checked;
   the next call with the normal limit must be correct.
"""
import time

import numpy as np
import pytest
import torch

import synth
from mixture_experts_routed_04_b200 import binding as b
from test_parity_gpu import P_of, W_of, check_close, device_inputs, f64, reference, run_forward

pytestmark = pytest.mark.gpu


def test_wait_on_a_barrier_nothing_completes_times_out():
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    t0 = time.time()
    b.wait_selftest(ws, 2_000_000)  # 2 ms
    torch.cuda.synchronize()
    assert time.time() - t0 < 30
    assert b.get_error(ws) & b.DEVERR_TIMEOUT
    b.clear_error(ws)
    assert b.get_error(ws) == 0
    # the context is usable afterwards
    x = torch.arange(1024, device="cuda", dtype=torch.float32)
    assert float(x.sum().item()) == 1023 * 1024 / 2


@pytest.mark.parametrize("variant,tile", [(b.VARIANT_TENSOR, b.TILE_ONE), (b.VARIANT_TENSOR, b.TILE_PAIR),
                                          (b.VARIANT_STREAM, b.TILE_AUTO)])
def test_layer_with_tiny_wait_limit_reports_and_recovers(variant, tile):
    cfg = synth.CONFIGS["tiny"]
    d = device_inputs(cfg)
    p = P_of(cfg, variant, True, tile_ctas=tile)
    ws = b.workspace(p, b.WS_FORWARD)
    out = torch.empty(cfg.T, cfg.d, dtype=torch.float32, device="cuda")
    b.set_wait_limit_ns(1)
    try:
        for _ in range(3):
            b.forward(p, d["x"], d["logits"], W_of(d, True), out, ws)
        torch.cuda.synchronize()
    finally:
        b.set_wait_limit_ns(0)  # back to the default (1 s)
    err = b.get_error(ws)
    assert err & ~(b.DEVERR_TIMEOUT) == 0, f"unexpected error bits {err:#x}"
    got, _ = run_forward(cfg, d, variant, tile_ctas=tile)  # asserts a clean error word itself
    ref, _ = reference(cfg)
    check_close(f64(got), ref, "layer after a run with 1 ns waits")
