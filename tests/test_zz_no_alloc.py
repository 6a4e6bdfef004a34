"""moe_permute_noalloc: the permutation with its scratch in a fixed device array.

Some callers cannot call cudaMalloc at the point where they permute — an engine
that has handed all free device memory to its own budget at load time and must
not allocate later, or a plugin running inside another framework's stream with
no allocator of its own. This entry point serves them: they pass only inputs
and outputs. It is checked here against moe_permute (which takes a caller
workspace) through the C ABI, on two calls in a row of different sizes, so a
call that saw the previous call's leftovers in the shared array would fail.
The outputs are integers: they must match exactly.

The file name sorts last, so a run that stops at the first failure has already
run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth
from mixture_experts_routed_04_b200 import binding as b

pytestmark = pytest.mark.gpu


def _buffers(cfg, rows):
    i32 = dict(dtype=torch.int32, device="cuda")
    Et = cfg.E + int(cfg.has_shared)
    return [torch.full((Et,), -5, **i32), torch.full((Et,), -5, **i32), torch.full((Et + 1,), -5, **i32),
            torch.full((rows,), -5, **i32), torch.full((rows,), -5, **i32), torch.full((cfg.T * cfg.k,), -5, **i32)]


def _compare_with_workspace_version(cfg):
    p = b.params_for(cfg)
    rows = b.max_rows(p)
    logits = torch.from_numpy(synth.logits(cfg)).cuda()
    idx = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device="cuda")
    w = torch.empty(cfg.T, cfg.k, dtype=torch.float32, device="cuda")
    b.route(p, logits, idx, w, b.workspace(p, b.WS_ROUTE))

    want = _buffers(cfg, rows)
    ws = b.workspace(p, b.WS_PERMUTE)
    b.permute(p, idx, *want, ws)

    got = _buffers(cfg, rows)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    b.permute_noalloc(p, idx, *got, err_word=err)
    torch.cuda.synchronize()

    assert b.get_error(ws) == 0 and int(err.item()) == 0
    n = int(want[2][-1].item())
    for name, a, c in zip(("counts", "kept", "offsets"), want[:3], got[:3]):
        assert torch.equal(a, c), name
    assert torch.equal(want[3][:n], got[3][:n]), "sorted_token"
    assert torch.equal(want[4][:n], got[4][:n]), "sorted_pair"
    assert torch.equal(want[5], got[5]), "pair_row"
    return n


def test_noalloc_permute_matches_the_workspace_version_on_two_calls():
    # a capped layer (token-order drops) and then a larger uncapped one with skew
    n1 = _compare_with_workspace_version(synth.CONFIGS["capped"])
    n2 = _compare_with_workspace_version(synth.CONFIGS["prompt"])
    assert n1 > 0 and n2 == 4096 * 8
    # the decode layer: 256 experts plus the shared expert's rows
    n3 = _compare_with_workspace_version(synth.CONFIGS["decode32"])
    assert n3 == 32 * 8 + 32
    # exactly the array's limit, 256 experts and a shared expert: the last block and the
    # widest expert stride of the fixed array are both in use
    big = synth.LayerConfig("noalloc_limit", T=b.NOALLOC_MAX_PAIRS // 8, d=64, f=64, E=256, k=8,
                            has_shared=True, f_shared=64)
    n4 = _compare_with_workspace_version(big)
    assert n4 == b.NOALLOC_MAX_PAIRS + big.T


def test_noalloc_permute_rejects_sizes_beyond_its_array():
    # 40000 tokens x top-8 = 320000 pairs, more than the fixed array holds
    p = b.params(T=40000, d_model=64, d_ff=64, E=16, k=8)
    status = b.lib().moe_permute_noalloc(ctypes.byref(p), None, None, None, None, None, None, None, None, None)
    assert status == 2  # MOE_ERR_WORKSPACE_TOO_SMALL, before any launch
    assert 40000 * 8 > b.NOALLOC_MAX_PAIRS
