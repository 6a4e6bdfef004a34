"""Backward of the expert FFN (moe_expert_ffn_backward) against the fp64 oracle.

The upstream gradient dout is seeded N(0, 1) (synth.dout); every gradient —
dx, the three expert weight gradients of every expert (zeros for experts
without rows), the routing-weight gradient d topk_w, dlogits and the shared
expert's weight gradients — is compared element by element with
oracle.backward: rel-L2 <= 1e-2, and every element within 3e-2 * rms(ref)
plus 2^-6 of its own magnitude. The second term is the 16-bit operand
rounding carried by large elements: with one token a weight gradient is an
outer product, whose largest element is ~20x its rms, so an error relative to
each element (fp16: 2^-11 per rounded operand) reaches a few percent of rms.
The GPU multiplies the bf16 gate/up weights by bf16 operands and the fp16
W_down copy and the weight gradients by fp16 operands, accumulating in fp32.
Small layers span several M-tiles per expert with ragged tails, capacity
drops, a shared expert, skew, k = E and a firing clamp; the prompt workload
runs at full size. Two calls give the same bits.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from mixture_experts_routed_04_b200 import binding as b
from synth.device import expert_f64, shared_f64, upload

pytestmark = pytest.mark.gpu

REL_L2, MAX_ABS_RMS, ELEM_REL = 1e-2, 3e-2, 2.0 ** -6

LAYERS = {
    "tiny": synth.CONFIGS["tiny"],
    "ragged": synth.LayerConfig("ragged", T=700, d=192, f=320, E=6, k=3),
    "ragged_capped": synth.LayerConfig("ragged_capped", T=700, d=192, f=320, E=6, k=3, capacity_factor=0.8),
    "e1_dense": synth.LayerConfig("e1_dense", T=37, d=64, f=64, E=1, k=1),
    "k_equals_E": synth.LayerConfig("k_equals_E", T=50, d=128, f=128, E=4, k=4),
    "single_token": synth.LayerConfig("single_token", T=1, d=128, f=256, E=8, k=2),
    "shared_small": synth.LayerConfig("shared_small", T=20, d=256, f=192, E=16, k=4, has_shared=True,
                                      f_shared=192),
    "zipf_small": synth.LayerConfig("zipf_small", T=512, d=256, f=256, E=32, k=4, bias="zipf"),
    "clamp_fires": synth.LayerConfig("clamp_fires", T=96, d=128, f=192, E=4, k=2, swiglu_limit=0.5),
}


def check_close(got, ref, what):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert np.isfinite(got).all(), f"{what}: non-finite"
    diff = got - ref
    rel = np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-300)
    rms = float(np.sqrt(np.mean(ref ** 2)))
    excess = np.abs(diff) - (MAX_ABS_RMS * rms + ELEM_REL * np.abs(ref))
    worst = float(excess.max()) if diff.size else -1.0
    assert rel <= REL_L2 and worst <= 0.0, \
        f"{what}: rel-L2 {rel:.3e} (<= {REL_L2}), worst element over its bound by {worst:.3e}"


def dout_of(cfg):
    return synth.dout(cfg)


def run_backward(cfg, d, dout):
    p = b.params_for(cfg, down_dtype=b.DOWN_F16)
    T, E, k, dm, f = cfg.T, cfg.E, cfg.k, cfg.d, cfg.f
    Et = E + int(cfg.has_shared)
    rows = b.max_rows(p)
    i32 = dict(dtype=torch.int32, device="cuda")
    f32 = dict(dtype=torch.float32, device="cuda")
    idx, w = torch.empty(T, k, **i32), torch.empty(T, k, **f32)
    counts, kept, offsets = torch.empty(Et, **i32), torch.empty(Et, **i32), torch.empty(Et + 1, **i32)
    st, sp, pr = torch.empty(rows, **i32), torch.empty(rows, **i32), torch.empty(T * k, **i32)
    b.route(p, d["logits"], idx, w, b.workspace(p, b.WS_ROUTE))
    b.permute(p, idx, counts, kept, offsets, st, sp, pr, b.workspace(p, b.WS_PERMUTE))
    # the backward multiplies the fp16 copy of W_down, prepared once as for the forward
    sh = (d["shared_gate"], d["shared_up"], b.prepare_down_f16(d["shared_down"])) if cfg.has_shared else None
    W = b.weights(d["w_gate"], d["w_up"], b.prepare_down_f16(d["w_down"]), shared=sh)
    nan = float("nan")
    outs = dict(dx=torch.full((T, dm), nan, **f32), dw_gate=torch.full((E, dm, f), nan, **f32),
                dw_up=torch.full((E, dm, f), nan, **f32), dw_down=torch.full((E, f, dm), nan, **f32),
                d_topk_w=torch.full((T, k), nan, **f32), dlogits=torch.full((T, E), nan, **f32))
    shg = None
    if cfg.has_shared:
        shg = tuple(torch.full(s, nan, **f32) for s in ((dm, f), (dm, f), (f, dm)))
    G = b.grads(outs["dx"], outs["dw_gate"], outs["dw_up"], outs["dw_down"], outs["d_topk_w"], outs["dlogits"],
                shared=shg)
    ws = b.workspace(p, b.WS_BACKWARD)
    dout_d = torch.from_numpy(dout).cuda()
    b.expert_ffn_backward(p, d["x"], idx, w, offsets, st, sp, pr, W, dout_d, G, ws)
    torch.cuda.synchronize()
    assert b.get_error(ws) == 0
    res = {key: t.cpu().numpy().astype(np.float64) for key, t in outs.items()}
    if shg is not None:
        res["dshared"] = tuple(t.cpu().numpy().astype(np.float64) for t in shg)
    return res


def reference(cfg, dout):
    x = synth.bf16_bits_to_f32(synth.x_bits(cfg)).astype(np.float64)
    sh = shared_f64(cfg) if cfg.has_shared else None
    return oracle.backward(x, synth.logits(cfg), cfg.k, lambda e: expert_f64(cfg, e), cfg.swiglu_limit, dout,
                           cfg.capacity_factor, shared=sh)


def compare(name, got, ref):
    for key in ("dx", "d_topk_w", "dlogits"):
        check_close(got[key], ref[key], f"{name} {key}")
    for key in ("dw_gate", "dw_up", "dw_down"):
        check_close(got[key], ref[key], f"{name} {key}")
        for e in range(ref[key].shape[0]):
            if np.abs(ref[key][e]).max() == 0.0:
                assert np.abs(got[key][e]).max() == 0.0, f"{name} {key}[{e}] of an expert without rows"
    if "dshared" in ref:
        for i, key in enumerate(("dshared_gate", "dshared_up", "dshared_down")):
            check_close(got["dshared"][i], ref["dshared"][i], f"{name} {key}")


@pytest.mark.parametrize("name", list(LAYERS))
def test_backward_small_layers(name):
    cfg = LAYERS[name]
    d = upload(cfg, "cuda")
    dout = dout_of(cfg)
    got = run_backward(cfg, d, dout)
    compare(name, got, reference(cfg, dout))


def test_backward_prompt_full_size_and_deterministic():
    cfg = synth.CONFIGS["prompt"]
    d = upload(cfg, "cuda")
    dout = dout_of(cfg)
    got = run_backward(cfg, d, dout)
    compare("prompt", got, reference(cfg, dout))
    again = run_backward(cfg, d, dout)
    for key in ("dx", "dw_gate", "dw_up", "dw_down", "d_topk_w", "dlogits"):
        assert np.array_equal(got[key], again[key]), f"{key} differs between two calls"
