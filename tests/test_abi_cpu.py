"""The C-ABI library without a GPU: it builds for sm_100a, loads, exports every
declared entry point, and its host-side logic (parameter checks, capacity,
buffer sizes) behaves as documented. No compute call is made here."""
import ctypes
import os
import re

import pytest

import oracle
from mixture_experts_routed_04_b200 import binding as b
from mixture_experts_routed_04_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build()
    return b.lib()


def _declared():
    with open(os.path.join(ROOT, "include", "moe.h")) as fh:
        return set(re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", fh.read()))


def test_exports_every_declared_symbol(lib):
    declared = _declared()
    assert len(declared) >= 14
    assert declared == set(b.EXPORTS)
    for name in declared:
        assert hasattr(lib, name), name
    assert lib.moe_version() >= 100


def test_status_strings(lib):
    for code, text in b.STATUS.items():
        assert lib.moe_status_string(code).decode() == text


def test_capacity_matches_oracle_rule(lib):
    with open(os.path.join(ROOT, "tests", "golden", "capacity_cases.txt")) as fh:
        rows = [ln.split() for ln in fh if ln.strip() and not ln.startswith("#")]
    for T, k, E, cf, _ in rows:
        T, k, E, cf = int(T), int(k), int(E), float(cf)
        p = b.params(T, 64, 64, E, k, capacity_factor=cf)
        assert b.capacity(p) == oracle.capacity(T, k, E, cf)


def test_max_rows_and_workspace(lib):
    p = b.params(4096, 2048, 768, 128, 8)
    assert b.max_rows(p) == 4096 * 8
    capped = b.params(8192, 1024, 2048, 128, 2, capacity_factor=1.5)
    assert b.max_rows(capped) == min(8192 * 2, 128 * 192)
    shared = b.params(32, 4096, 1536, 256, 8, has_shared=1, d_ff_shared=1536)
    assert b.max_rows(shared) == 32 * 8 + 32
    for which in range(6):
        assert b.workspace_size(p, which) >= 256
    assert b.workspace_size(p, b.WS_FORWARD) > b.workspace_size(p, b.WS_EXPERT_FFN)


@pytest.mark.parametrize("bad", [
    dict(k=9), dict(k=3, E=2), dict(E=257), dict(d_model=100), dict(d_ff=32), dict(T=-1),
    dict(capacity_factor=-1.0), dict(capacity_factor=float("nan")), dict(variant=7), dict(weight_format=5),
    dict(tile_ctas=3), dict(tile_ctas=-1)])
def test_invalid_params_rejected_on_host(lib, bad):
    kw = dict(T=16, d_model=128, d_ff=256, E=8, k=2)
    kw.update(bad)
    p = b.params(**kw)
    assert b.workspace_size(p, b.WS_FORWARD) == 0
    st = lib.moe_route(ctypes.byref(p), None, None, None, None, 0, None)
    assert st == 1  # MOE_ERR_INVALID_ARG, before any launch


def test_tile_shape_choice(lib):
    """MOE_TILE_AUTO is one SM per tile; SM pairs only on request, and only for bf16 weights."""
    prompt = dict(T=4096, d_model=2048, d_ff=768, E=128, k=8)
    assert b.tile_ctas(b.params(**prompt)) == b.TILE_ONE
    assert b.tile_ctas(b.params(**prompt, tile_ctas=b.TILE_ONE)) == b.TILE_ONE
    assert b.tile_ctas(b.params(**prompt, tile_ctas=b.TILE_PAIR)) == b.TILE_PAIR
    assert b.tile_ctas(b.params(8192, 1024, 2048, 128, 2, capacity_factor=1.5)) == b.TILE_ONE
    assert b.tile_ctas(b.params(1, 4096, 1536, 256, 8, has_shared=1, d_ff_shared=1536)) == b.TILE_ONE
    assert b.tile_ctas(b.params(64, 128, 256, 8, 2, tile_ctas=b.TILE_PAIR)) == b.TILE_PAIR
    # the Q4G32 GEMMs keep one SM per tile even when pairs are asked for
    q4 = b.params(32768, 2048, 768, 128, 8, weight_format=b.WEIGHTS_Q4G32, tile_ctas=b.TILE_PAIR)
    assert b.tile_ctas(q4) == b.TILE_ONE


def test_empty_batch_is_valid_and_launches_nothing(lib):
    # T = 0: a rank with no tokens. Sizes are defined, the capacity is 0 and no kernel is launched.
    p = b.params(0, 128, 256, 8, 2, capacity_factor=1.5)
    assert b.workspace_size(p, b.WS_FORWARD) >= 256
    assert b.capacity(p) == 0
    for which in range(6):
        n = ctypes.c_int(-1)
        assert lib.moe_launch_count(ctypes.byref(p), which, ctypes.byref(n)) == 0
        assert n.value == 0


def test_unsupported_and_missing_buffers(lib):
    p = b.params(8, 128, 256, 8, 2, has_shared=1, d_ff_shared=128)
    assert lib.moe_route(ctypes.byref(p), None, None, None, None, 0, None) == 3  # UNSUPPORTED
    ok = b.params(8, 128, 256, 8, 2)
    # null workspace / buffers: rejected before any CUDA call
    assert lib.moe_route(ctypes.byref(ok), None, None, None, None, 0, None) == 1
    assert lib.moe_forward(ctypes.byref(ok), None, None, None, None, None, None, 0, None) == 1
    assert lib.moe_forward_host_async(ctypes.byref(ok), None, None, None, None, None, 0, None) == 1
    assert lib.moe_forward_host_async(ctypes.byref(p), None, None, None, None, None, 0, None) == 3
    # the wait self-test validates its arguments before any launch
    assert lib.moe_wait_selftest(None, 1000, None) == 1
    assert lib.moe_wait_selftest(ctypes.c_void_p(16), 0, None) == 1
    assert lib.moe_wait_selftest(ctypes.c_void_p(16), 20_000_000_000, None) == 1
    # the no-allocation permutation checks its parameters and pointers first
    assert lib.moe_permute_noalloc(ctypes.byref(ok), None, None, None, None, None, None, None, None, None) == 1


def test_product_path_never_touches_the_oracle():
    pkg = os.path.join(ROOT, "mixture_experts_routed_04_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                with open(os.path.join(dirpath, fn)) as fh:
                    src = fh.read()
                assert not re.search(r"\boracle\b", src), fn
    with open(os.path.join(ROOT, "oracle", "__init__.py")) as fh:
        assert "mixture_experts_routed_04_b200" not in fh.read()


def test_backward_host_checks(lib):
    """moe_expert_ffn_backward refuses Q4G32 weights and a bf16 W_down (it multiplies the fp16
    copy) before touching any pointer; its workspace grows with the padded row space."""
    p = b.params(T=64, d_model=128, d_ff=256, E=8, k=2, weight_format=b.WEIGHTS_Q4G32)
    st = lib.moe_expert_ffn_backward(ctypes.byref(p), None, None, None, None, None, None, None, None, None, None,
                                     None, 0, None)
    assert st == 3  # MOE_ERR_UNSUPPORTED
    p = b.params(T=64, d_model=128, d_ff=256, E=8, k=2, down_dtype=b.DOWN_BF16)
    st = lib.moe_expert_ffn_backward(ctypes.byref(p), None, None, None, None, None, None, None, None, None, None,
                                     None, 0, None)
    assert st == 3
    small = b.workspace_size(b.params(T=64, d_model=128, d_ff=256, E=8, k=2, down_dtype=b.DOWN_F16), b.WS_BACKWARD)
    large = b.workspace_size(b.params(T=640, d_model=128, d_ff=256, E=8, k=2, down_dtype=b.DOWN_F16), b.WS_BACKWARD)
    assert 0 < small < large


def test_variant_table_is_finite_and_monotone(lib):
    """The measured table of the default variant choice: finite, tile bounds increasing,
    streamed expert sizes shrinking as more tiles are available, and every entry sensible."""
    import math
    table = b.variant_table()
    assert 1 <= len(table) <= 16
    bounds = [t for t, _ in table]
    rows = [r for _, r in table]
    assert all(math.isfinite(t) and 0.0 < t < 64.0 for t in bounds)
    assert all(1 <= r <= 64 for r in rows)
    assert all(a < c for a, c in zip(bounds, bounds[1:]))
    assert all(a >= c for a, c in zip(rows, rows[1:]))


def test_default_variant_follows_the_table(lib):
    """Single-token decode (8 routed experts + the shared one: 108 gate/up tiles on 148 SMs, or
    whatever the host's default count) streams; eight tokens (up to 65 experts) take the tiles.
    The streaming kernels replace the two tile GEMMs and the combine in moe_forward's count."""
    def launches(T):
        p = b.params(T=T, d_model=4096, d_ff=1536, E=256, k=8, has_shared=1, d_ff_shared=1536)
        return b.launch_count(p, b.WS_FORWARD), b.launch_count(b.params(
            T=T, d_model=4096, d_ff=1536, E=256, k=8, has_shared=1, d_ff_shared=1536,
            variant=b.VARIANT_TENSOR), b.WS_FORWARD)
    auto1, tiles1 = launches(1)
    auto8, tiles8 = launches(8)
    # T=1: the two tile GEMMs give way to the streaming gate/up and down (the down kernel
    # sums the gate/up's K-split partials itself and, every expert streaming, does the combine)
    assert auto1 == tiles1 - 1
    assert auto8 == tiles8  # T=8: every expert on the tiles
    # the single-token layer: the front kernel (routing, permutation, schedule and, for at most
    # 96 KB of rows, the gather) and the two streaming kernels
    assert auto1 == 3
    assert auto8 == 5  # front, gather, two tile GEMMs, combine


def test_streaming_reduce_folds_into_down_when_h_fits(lib):
    """The K-split gate/up partials are summed by the streaming down kernel while its h buffer
    (8 rows of d_ff fp16) fits beside its stages, else by a separate reduce launch."""
    def launches(f):
        p = b.params(T=3, d_model=256, d_ff=f, E=4, k=2, variant=b.VARIANT_STREAM)
        return b.launch_count(p, b.WS_EXPERT_FFN)
    # schedule + gather + streaming gate/up + down, (+ reduce)
    assert launches(2112) == 4
    assert launches(2176) == 5


def test_forward_permutation_forms_its_scan_in_the_scatter(lib):
    """Above the front kernel's batch size, moe_forward's scatter blocks form the permutation's
    scan themselves (no scan launch) while the per-block counts fit their shared memory and one
    thread per expert fits a block; moe_permute keeps its three launches."""
    def fwd(T, E=128, k=8):
        return b.launch_count(b.params(T=T, d_model=2048, d_ff=768, E=E, k=k), b.WS_FORWARD)
    # routing, count, scatter (with the scan and the schedule), gather, gate/up, down, combine
    assert fwd(4096) == 7
    assert fwd(32768) == 7  # 128 blocks of 2048 pairs x 128 experts: 64 KB of counts
    assert fwd(1024, E=256, k=8) == 7  # 256 experts, no shared one: a thread each
    p = b.params(T=4096, d_model=2048, d_ff=768, E=256, k=8, has_shared=1, d_ff_shared=768)
    assert b.launch_count(p, b.WS_FORWARD) == 8  # 257 experts: the scan kernel runs
    assert b.launch_count(b.params(T=4096, d_model=2048, d_ff=768, E=128, k=8), b.WS_PERMUTE) == 3
    # 128 blocks of 2048 pairs x 256 experts: 128 KB of counts, above the 96 KB the blocks copy
    assert fwd(32768, E=256, k=8) == 8
