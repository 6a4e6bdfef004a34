"""GPU path against the fp64 oracle, through the C ABI, on the seeded inputs.

Bar: routing indices, counts, offsets, sorted lists and drop decisions are
bit-exact; routing weights within 1e-6; the layer output (fp32) and the
per-row expert outputs y_rows (fp16) within rel-L2 <= 1e-2 and
max-abs <= 3e-2 * rms(reference); the bf16 output option is the fp32 output
rounded once.

Small layers (several M-tiles per expert, ragged tails, partial N-tiles) are
compared element by element on every kernel variant and both forms of W_down
(bf16 as given, fp16 prepared at load time). The stated workloads are compared
at full size in the launch configuration the benchmark times (moe_forward,
automatic variant choice, W_down prepared as fp16): routing and permutation in
full, and every output element (with sampled tokens from the per-token
definition beside it), and the bf16 output option on every workload.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
from mixture_experts_routed_04_b200 import binding as b
from synth.device import expert_f64, shared_f64, upload

pytestmark = pytest.mark.gpu

REL_L2, MAX_ABS_RMS = 1e-2, 3e-2

SMALL = {
    "tiny": synth.CONFIGS["tiny"],
    # several M-tiles per expert with a ragged tail; f=320 and d=192 leave partial N-tiles
    "ragged": synth.LayerConfig("ragged", T=700, d=192, f=320, E=6, k=3),
    "ragged_capped": synth.LayerConfig("ragged_capped", T=700, d=192, f=320, E=6, k=3, capacity_factor=0.8),
    "e1_dense": synth.LayerConfig("e1_dense", T=37, d=64, f=64, E=1, k=1),
    "k_equals_E": synth.LayerConfig("k_equals_E", T=50, d=128, f=128, E=4, k=4),
    "single_token": synth.LayerConfig("single_token", T=1, d=128, f=256, E=8, k=2),
    "shared_small": synth.LayerConfig("shared_small", T=20, d=256, f=192, E=16, k=4, has_shared=True,
                                      f_shared=192),
    "zipf_small": synth.LayerConfig("zipf_small", T=512, d=256, f=256, E=32, k=4, bias="zipf"),
    # 32 touched experts x 5 gate/up tiles >= 148 SMs: the automatic choice keeps every expert
    # on the tiles, so a forced streaming variant must still launch the streaming kernels
    "many_experts": synth.LayerConfig("many_experts", T=8, d=128, f=640, E=32, k=4),
    # d_ff too wide for the streaming down kernel's h buffer: the K-split gate/up partials go
    # through the separate reduce kernel (at d_ff <= 2136 the down kernel sums them itself)
    "wide_ff": synth.LayerConfig("wide_ff", T=3, d=256, f=2176, E=4, k=2),
    # two tokens with a shared expert: every expert streams and the streaming down kernel
    # also does the combine (a 256-column block of d=320 is partial)
    "two_tokens": synth.LayerConfig("two_tokens", T=2, d=320, f=256, E=8, k=3, has_shared=True, f_shared=256),
    # 257 experts with the shared one, above the front kernel's batch: the permutation's scan
    # runs as its own launch (one thread per expert no longer fits a scatter block), and the
    # automatic choice mixes streaming (experts of a few rows) with tiles (the shared expert)
    "scan_launch": synth.LayerConfig("scan_launch", T=96, d=128, f=128, E=256, k=2, has_shared=True,
                                     f_shared=128),
}
Q4_SMALL = {
    "q4_tiny": synth.CONFIGS["tiny"].replace(name="q4_tiny", weight_format="q4g32"),
    "q4_ragged": synth.LayerConfig("q4_ragged", T=700, d=192, f=320, E=6, k=3, weight_format="q4g32"),
    "q4_zipf": synth.LayerConfig("q4_zipf", T=512, d=256, f=256, E=32, k=4, bias="zipf", weight_format="q4g32"),
    "q4_capped": synth.LayerConfig("q4_capped", T=300, d=128, f=192, E=8, k=2, capacity_factor=0.9,
                                   weight_format="q4g32"),
}
FULL = ["prompt", "capped", "decode1", "decode8", "decode32"]
VARIANTS = {"auto": b.VARIANT_AUTO, "tensor": b.VARIANT_TENSOR, "stream": b.VARIANT_STREAM}


def check_close(got, ref, what):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    diff = got - ref
    rel = np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-300)
    rms = float(np.sqrt(np.mean(ref ** 2)))
    mx = float(np.abs(diff).max()) if diff.size else 0.0
    assert rel <= REL_L2 and mx <= MAX_ABS_RMS * rms, \
        f"{what}: rel-L2 {rel:.3e} (<= {REL_L2}), max-abs {mx:.3e} (<= {MAX_ABS_RMS * rms:.3e})"


def f64(t):
    return t.float().cpu().numpy().astype(np.float64)


# --------------------------------------------------------------------------- oracle side

def expert_ref(cfg, e, scale=1.0):
    """(W_gate, W_up, W_down) float64 of expert e, as the layer's weights define them."""
    if cfg.weight_format == "q4g32":
        W = tuple(oracle.dequant_q4g32(*synth.expert_q4_weights(cfg, e, w)) for w in ("gate", "up", "down"))
    else:
        W = expert_f64(cfg, e)
    return (W[0] * scale, W[1] * scale, W[2])


_REF = {}


def reference(cfg, scale=1.0):
    key = (cfg, scale)
    if key not in _REF:
        x = synth.bf16_bits_to_f32(synth.x_bits(cfg)).astype(np.float64)
        sh = shared_f64(cfg) if cfg.has_shared else None
        _REF[key] = oracle.forward(x, synth.logits(cfg), cfg.k, lambda e: expert_ref(cfg, e, scale),
                                   cfg.swiglu_limit, cfg.capacity_factor, shared=sh)
    return _REF[key]


def routing_reference(cfg):
    idx, w = oracle.route(synth.logits(cfg), cfg.k)
    cap = oracle.capacity(cfg.T, cfg.k, cfg.E, cfg.capacity_factor)
    perm = oracle.permute(idx, cfg.E, cap, shared_T=cfg.T if cfg.has_shared else 0)
    return idx, w, perm


# --------------------------------------------------------------------------- device side

_DEV = {}


def device_inputs(cfg, experts=None, scale=1.0):
    key = (cfg, scale)
    if key not in _DEV:
        _DEV.clear()
        torch.cuda.empty_cache()
        d = upload(cfg, "cuda", experts=experts)
        if scale != 1.0:
            d["w_gate"].mul_(scale)
            d["w_up"].mul_(scale)
        if cfg.weight_format == "bf16":  # load-time fp16 copies of W_down
            d["w_down_f16"] = b.prepare_down_f16(d["w_down"])
            if cfg.has_shared:
                d["shared_down_f16"] = b.prepare_down_f16(d["shared_down"])
        _DEV[key] = d
    return _DEV[key]


def W_of(d, down_f16):
    dn = "w_down_f16" if down_f16 else "w_down"
    sh = None
    if "shared_gate" in d:
        sh = (d["shared_gate"], d["shared_up"], d["shared_down_f16" if down_f16 else "shared_down"])
    return b.weights(d["w_gate"], d["w_up"], d[dn], d.get("s_gate"), d.get("s_up"), d.get("s_down"), shared=sh)


def P_of(cfg, variant, down_f16, **kw):
    return b.params_for(cfg, variant=variant, down_dtype=b.DOWN_F16 if down_f16 else b.DOWN_BF16, **kw)


def run_steps(cfg, d, variant, down_f16, **kw):
    p = P_of(cfg, variant, down_f16, **kw)
    T, E, k = cfg.T, cfg.E, cfg.k
    Et = E + int(cfg.has_shared)
    rows = b.max_rows(p)
    dev = "cuda"
    i32 = dict(dtype=torch.int32, device=dev)
    topk_idx, topk_w = torch.empty(T, k, **i32), torch.empty(T, k, dtype=torch.float32, device=dev)
    counts, kept, offsets = torch.empty(Et, **i32), torch.empty(Et, **i32), torch.empty(Et + 1, **i32)
    st, sp = torch.full((rows,), -7, **i32), torch.full((rows,), -7, **i32)
    pr = torch.empty(T * k, **i32)
    y = torch.zeros(rows, cfg.d, dtype=torch.float16, device=dev)
    out = torch.empty(T, cfg.d, dtype=torch.float32, device=dev)
    wss = [b.workspace(p, w) for w in (b.WS_ROUTE, b.WS_PERMUTE, b.WS_EXPERT_FFN, b.WS_COMBINE)]
    b.route(p, d["logits"], topk_idx, topk_w, wss[0])
    b.permute(p, topk_idx, counts, kept, offsets, st, sp, pr, wss[1])
    b.expert_ffn(p, d["x"], offsets, st, sp, topk_w, W_of(d, down_f16), y, wss[2])
    b.combine(p, y, pr, offsets, out, wss[3])
    torch.cuda.synchronize()
    for ws in wss:
        assert b.get_error(ws) == 0
    n = int(offsets[-1])
    return {"idx": topk_idx.cpu().numpy(), "w": topk_w.cpu().numpy(), "counts": counts.cpu().numpy(),
            "kept": kept.cpu().numpy(), "offsets": offsets.cpu().numpy(), "sorted_token": st[:n].cpu().numpy(),
            "sorted_pair": sp[:n].cpu().numpy(), "pair_row": pr.cpu().numpy(), "y": f64(y[:n]),
            "out": f64(out)}


def run_forward(cfg, d, variant=b.VARIANT_AUTO, down_f16=True, **kw):
    p = P_of(cfg, variant, down_f16 and cfg.weight_format == "bf16", **kw)
    ws = b.workspace(p, b.WS_FORWARD)
    out = torch.empty(cfg.T, cfg.d, dtype=torch.float32, device="cuda")
    counts = torch.empty(cfg.E + int(cfg.has_shared), dtype=torch.int32, device="cuda")
    b.forward(p, d["x"], d["logits"], W_of(d, down_f16 and cfg.weight_format == "bf16"), out, ws,
              counts_out=counts)
    torch.cuda.synchronize()
    assert b.get_error(ws) == 0
    return out, counts.cpu().numpy()


def check_routing(cfg, got):
    idx, w, perm = routing_reference(cfg)
    assert (got["idx"] == idx).all(), "topk_idx differs"
    np.testing.assert_allclose(got["w"], w, rtol=0, atol=1e-6)
    for key in ("counts", "kept", "offsets", "sorted_token", "sorted_pair", "pair_row"):
        assert (got[key] == perm[key]).all(), f"{key} differs"
    return idx, w, perm


def check_layer(name, cfg, got, scale=1.0):
    out, it = reference(cfg, scale)
    w_row = np.array([it["w"].reshape(-1)[p] if p >= 0 else 1.0 for p in it["sorted_pair"]])
    check_close(got["y"], it["y"] * w_row[:, None], f"{name} y_rows")
    check_close(got["out"], out, f"{name} out")
    return out, it


# --------------------------------------------------------------------------- tests

def test_library_is_in_tree():
    import os
    assert os.path.dirname(b.LIB_PATH).endswith("mixture_experts_routed_04_b200")
    b.lib()


@pytest.mark.parametrize("down", ["bf16", "f16"])
@pytest.mark.parametrize("variant", list(VARIANTS))
@pytest.mark.parametrize("name", list(SMALL))
def test_small_layers_every_variant(name, variant, down):
    cfg = SMALL[name]
    d = device_inputs(cfg)
    f16 = down == "f16"
    got = run_steps(cfg, d, VARIANTS[variant], f16)
    check_routing(cfg, got)
    out, it = check_layer(f"{name}/{variant}/{down}", cfg, got)
    # the fused entry point gives the same bits as the step-by-step calls
    fout, counts = run_forward(cfg, d, VARIANTS[variant], f16)
    assert (counts == it["counts"]).all()
    assert np.array_equal(f64(fout), got["out"])


TILES = {"one": b.TILE_ONE, "pair": b.TILE_PAIR}


@pytest.mark.parametrize("down", ["bf16", "f16"])
@pytest.mark.parametrize("tile", list(TILES))
@pytest.mark.parametrize("name", list(SMALL))
def test_small_layers_tile_shapes(name, tile, down):
    """Every expert on the tcgen05 tiles, one SM per 128-row tile or SM pairs on 256-row tiles
    (the pair kernels cover the bf16 gate/up and the fp16 down; bf16 W_down stays on one SM)."""
    cfg = SMALL[name]
    d = device_inputs(cfg)
    f16 = down == "f16"
    got = run_steps(cfg, d, b.VARIANT_TENSOR, f16, tile_ctas=TILES[tile])
    check_routing(cfg, got)
    check_layer(f"{name}/{tile}/{down}", cfg, got)
    fout, _ = run_forward(cfg, d, b.VARIANT_TENSOR, f16, tile_ctas=TILES[tile])
    assert np.array_equal(f64(fout), got["out"])


def test_prompt_both_tile_shapes():
    """The prompt workload at full size with each tile shape, against the per-token definition
    on sampled tokens, and the two shapes against each other on every element."""
    cfg = synth.CONFIGS["prompt"]
    idx, w, perm = routing_reference(cfg)
    d = device_inputs(cfg)
    x = synth.bf16_bits_to_f32(synth.x_bits(cfg)).astype(np.float64)
    rng = np.random.default_rng(11)
    toks = sorted(set([0, cfg.T - 1] + rng.choice(cfg.T, 48, replace=False).tolist()))
    ref = oracle.token_outputs(toks, x, idx, w, perm["pair_row"], lambda e: expert_ref(cfg, e), cfg.swiglu_limit)
    outs = {}
    for tile, t in TILES.items():
        out, counts = run_forward(cfg, d, tile_ctas=t)
        assert (counts == perm["counts"]).all()
        check_close(f64(out)[toks], ref, f"prompt/{tile} sampled tokens")
        outs[tile] = f64(out)
    check_close(outs["pair"], outs["one"], "prompt pair vs one SM per tile")


@pytest.mark.parametrize("variant", ["auto", "tensor"])
@pytest.mark.parametrize("name", list(Q4_SMALL))
def test_q4g32_layers(name, variant):
    cfg = Q4_SMALL[name]
    d = device_inputs(cfg)
    got = run_steps(cfg, d, VARIANTS[variant], False)
    check_routing(cfg, got)
    check_layer(f"{name}/{variant}", cfg, got)
    fout, _ = run_forward(cfg, d, VARIANTS[variant])
    assert np.array_equal(f64(fout), got["out"])


def test_q4g32_streaming_variant_is_refused():
    cfg = Q4_SMALL["q4_tiny"]
    p = b.params_for(cfg, variant=b.VARIANT_STREAM)
    with pytest.raises(b.MoeError):
        b.workspace(p, b.WS_FORWARD)


@pytest.mark.parametrize("down", ["bf16", "f16"])
def test_clamp_fires_and_matches(down):
    cfg = SMALL["tiny"]
    scale = 32.0  # exact in bf16; pre-activations reach well past the clamp at 7
    d = device_inputs(cfg, scale=scale)
    for v in ("tensor", "stream"):
        got = run_steps(cfg, d, VARIANTS[v], down == "f16")
        check_layer(f"clamp/{v}/{down}", cfg, got, scale=scale)
    _, it = reference(cfg, scale)
    x = synth.bf16_bits_to_f32(synth.x_bits(cfg)).astype(np.float64)
    g = x[:1] @ expert_ref(cfg, int(it["idx"][0, 0]), scale)[0]
    assert np.abs(g).max() > 7.0


@pytest.mark.parametrize("name", FULL)
def test_full_size_workloads(name):
    cfg = synth.CONFIGS[name]
    idx, w, perm = routing_reference(cfg)
    touched = np.unique(idx[perm["pair_row"].reshape(idx.shape) >= 0])
    d = device_inputs(cfg, experts=touched)
    got = run_steps(cfg, d, b.VARIANT_AUTO, True)
    check_routing(cfg, got)
    # every output element, the oracle drawing each touched expert's weights as it goes
    x = synth.bf16_bits_to_f32(synth.x_bits(cfg)).astype(np.float64)
    sh = shared_f64(cfg) if cfg.has_shared else None
    ref, it = oracle.forward(x, synth.logits(cfg), cfg.k, lambda e: expert_ref(cfg, e), cfg.swiglu_limit,
                             cfg.capacity_factor, shared=sh)
    check_close(got["out"], ref, f"{name} full output (step calls)")
    w_row = np.array([it["w"].reshape(-1)[p] if p >= 0 else 1.0 for p in it["sorted_pair"]])
    check_close(got["y"], it["y"] * w_row[:, None], f"{name} y_rows")
    fout, counts = run_forward(cfg, d)
    assert (counts == perm["counts"]).all()
    check_close(f64(fout), ref, f"{name} full output (moe_forward)")
    # and a few tokens from the per-token definition, which never permutes
    toks = [0, cfg.T // 2, cfg.T - 1]
    one = oracle.token_outputs(toks, x, idx, w, perm["pair_row"], lambda e: expert_ref(cfg, e), cfg.swiglu_limit,
                               shared=sh)
    check_close(f64(fout)[toks], one, f"{name} per-token definition")


def test_full_size_quantised_workload():
    """The T=32768 Q4G32 layer: every output element against the oracle's whole layer (each
    expert's weights dequantised exactly as q * s), plus sampled tokens from the per-token
    definition, which never permutes."""
    cfg = synth.CONFIGS["quant"]
    d = device_inputs(cfg)
    got = run_steps(cfg, d, b.VARIANT_AUTO, False)
    idx, w, perm = check_routing(cfg, got)
    x = synth.bf16_bits_to_f32(synth.x_bits(cfg)).astype(np.float64)
    cache = {}

    def experts(e):
        if e not in cache:
            cache[e] = expert_ref(cfg, e)
        return cache[e]

    ref, it = oracle.forward(x, synth.logits(cfg), cfg.k, experts, cfg.swiglu_limit, cfg.capacity_factor)
    check_close(got["out"], ref, "quant full output (step calls)")
    w_row = np.array([it["w"].reshape(-1)[p] for p in it["sorted_pair"]])
    check_close(got["y"], it["y"] * w_row[:, None], "quant y_rows")
    fout, _ = run_forward(cfg, d)
    check_close(f64(fout), ref, "quant full output (moe_forward)")
    rng = np.random.default_rng(7)
    toks = sorted(set([0, cfg.T - 1] + rng.choice(cfg.T, 16, replace=False).tolist()))
    one = oracle.token_outputs(toks, x, idx, w, perm["pair_row"], experts, cfg.swiglu_limit)
    check_close(f64(fout)[toks], one, "quant per-token definition")


BF16_ULP_REL = 2.0 ** -8  # one rounding to bf16 (8 significant bits) moves a value by at most this, relative


@pytest.mark.parametrize("name", ["tiny"] + FULL + ["quant"])
def test_bf16_output_every_workload(name):
    """The bf16 output option on every stated workload at full size: it equals the fp32 output
    rounded once (nearest even); against the oracle, rel-L2 <= 1e-2 and every element within
    3e-2 * rms(out) plus the one bf16 rounding (2^-8 of the element). On the capped layer most
    tokens lose every pair, rms(out) is small, and that rounding alone exceeds 3e-2 * rms on a
    few elements, hence the second term. Prints the measured max-abs / rms."""
    cfg = synth.CONFIGS[name]
    idx, w, perm = routing_reference(cfg)
    touched = np.unique(idx[perm["pair_row"].reshape(idx.shape) >= 0])
    d = device_inputs(cfg, experts=None if cfg.weight_format == "q4g32" else touched)
    f32_out, _ = run_forward(cfg, d)
    p = P_of(cfg, b.VARIANT_AUTO, cfg.weight_format == "bf16", out_dtype=b.OUT_BF16)
    ws = b.workspace(p, b.WS_FORWARD)
    out = torch.empty(cfg.T, cfg.d, dtype=torch.bfloat16, device="cuda")
    b.forward(p, d["x"], d["logits"], W_of(d, cfg.weight_format == "bf16"), out, ws)
    torch.cuda.synchronize()
    assert b.get_error(ws) == 0
    assert torch.equal(out.view(torch.int16), f32_out.to(torch.bfloat16).view(torch.int16))
    x = synth.bf16_bits_to_f32(synth.x_bits(cfg)).astype(np.float64)
    sh = shared_f64(cfg) if cfg.has_shared else None
    cache = {}

    def experts(e):
        if e not in cache:
            cache[e] = expert_ref(cfg, e)
        return cache[e]

    ref, _ = oracle.forward(x, synth.logits(cfg), cfg.k, experts, cfg.swiglu_limit, cfg.capacity_factor,
                            shared=sh)
    got = f64(out)
    diff = np.abs(got - ref)
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    rms = float(np.sqrt(np.mean(ref ** 2)))
    print(f"bf16 output {name}: rel-L2 {rel:.3e}, max-abs/rms {diff.max() / rms:.3e}")
    assert rel <= REL_L2, f"{name} bf16 output rel-L2 {rel:.3e}"
    bound = MAX_ABS_RMS * rms + BF16_ULP_REL * np.abs(ref)
    assert (diff <= bound).all(), f"{name} bf16 output: max excess {(diff - bound).max():.3e}"


@pytest.mark.parametrize("name", ["tiny", "single_token", "shared_small", "k_equals_E", "small_capped"])
def test_fused_front_matches_separate_kernels(name):
    """moe_forward with T <= 64 runs routing, permutation and schedule as one kernel; the layer
    must equal, bit for bit, the separate route / permute / expert_ffn / combine calls."""
    cfg = SMALL.get(name) or synth.LayerConfig("small_capped", T=64, d=128, f=128, E=8, k=2, capacity_factor=0.6)
    assert cfg.T <= 64
    d = device_inputs(cfg)
    steps = run_steps(cfg, d, b.VARIANT_AUTO, True)
    out, counts = run_forward(cfg, d)
    assert np.array_equal(f64(out), steps["out"])
    assert np.array_equal(counts, steps["counts"])


def test_forward_is_deterministic():
    cfg = synth.CONFIGS["prompt"].replace(T=1024)
    d = device_inputs(cfg)
    a, _ = run_forward(cfg, d)
    c, _ = run_forward(cfg, d)
    assert torch.equal(a.view(torch.int32), c.view(torch.int32))


def test_down_forms_agree():
    """W_down as bf16 (converted per tile) and prepared fp16 give the same bits."""
    cfg = SMALL["ragged"]
    d = device_inputs(cfg)
    for v in (b.VARIANT_TENSOR, b.VARIANT_STREAM):
        a, _ = run_forward(cfg, d, v, down_f16=False)
        c, _ = run_forward(cfg, d, v, down_f16=True)
        assert torch.equal(a.view(torch.int32), c.view(torch.int32))


def test_forward_host_matches_device():
    cfg = SMALL["ragged"]
    d = device_inputs(cfg)
    ref_out, _ = run_forward(cfg, d)
    p = P_of(cfg, b.VARIANT_AUTO, True)
    ws = b.workspace(p, b.WS_FORWARD_HOST)
    x_h = d["x"].cpu().pin_memory()
    l_h = d["logits"].cpu().pin_memory()
    o_h = torch.empty(cfg.T, cfg.d, dtype=torch.float32).pin_memory()
    b.forward_host(p, x_h, l_h, W_of(d, True), o_h, ws)
    assert torch.equal(o_h.view(torch.int32), ref_out.cpu().view(torch.int32))


def test_forward_host_async_pipeline_matches_device():
    """Four steps on two streams (separate workspaces and pinned buffers), copies overlapping kernels."""
    cfg = SMALL["ragged"]
    d = device_inputs(cfg)
    ref_out, _ = run_forward(cfg, d)
    p = P_of(cfg, b.VARIANT_AUTO, True)
    W = W_of(d, True)
    slots = [dict(stream=torch.cuda.Stream(), ws=b.workspace(p, b.WS_FORWARD_HOST),
                  x=d["x"].cpu().pin_memory(), l=d["logits"].cpu().pin_memory(),
                  o=torch.full((cfg.T, cfg.d), float("nan"), dtype=torch.float32).pin_memory()) for _ in range(2)]
    for i in range(4):
        sl = slots[i % 2]
        b.forward_host_async(p, sl["x"], sl["l"], W, sl["o"], sl["ws"], stream=sl["stream"])
    torch.cuda.synchronize()
    for sl in slots:
        assert b.get_error(sl["ws"]) == 0
        assert torch.equal(sl["o"].view(torch.int32), ref_out.cpu().view(torch.int32))


def test_bf16_output_option():
    cfg = SMALL["ragged"]
    d = device_inputs(cfg)
    f32_out, _ = run_forward(cfg, d)
    p = P_of(cfg, b.VARIANT_AUTO, True, out_dtype=b.OUT_BF16)
    ws = b.workspace(p, b.WS_FORWARD)
    out = torch.empty(cfg.T, cfg.d, dtype=torch.bfloat16, device="cuda")
    b.forward(p, d["x"], d["logits"], W_of(d, True), out, ws)
    torch.cuda.synchronize()
    assert b.get_error(ws) == 0
    # the bf16 output is the fp32 output rounded once (to nearest even)
    assert torch.equal(out.view(torch.int16), f32_out.to(torch.bfloat16).view(torch.int16))
    ref, _ = reference(cfg)
    assert np.linalg.norm(f64(out) - ref) / np.linalg.norm(ref) <= REL_L2


def test_weight_conversion_is_exact_rounding():
    rng = np.random.default_rng(5)
    vals = np.concatenate([rng.standard_normal(10000).astype(np.float32) * 0.02,
                           # 65280 is the largest bf16 value inside fp16's range (65504 rounds to 65536 in bf16)
                           np.array([0.0, -0.0, 1e-7, -3e-6, 6.1e-5, 65280.0, -65280.0, 1.0, 2.0 ** -17], np.float32)])
    bits = synth.f32_to_bf16_bits(vals)
    src = torch.from_numpy(bits.view(np.int16)).cuda()
    dst = torch.empty(src.numel(), dtype=torch.float16, device="cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    b.convert_bf16_to_f16(src, dst, err_ws=ws)
    want = synth.bf16_bits_to_f32(bits).astype(np.float16)  # round to nearest even
    assert np.array_equal(dst.cpu().numpy().view(np.uint16), want.view(np.uint16))
    assert b.get_error(ws) == 0
    big = torch.from_numpy(synth.f32_to_bf16_bits(np.array([1e6] * 8, np.float32)).view(np.int16)).cuda()
    b.convert_bf16_to_f16(big, torch.empty(8, dtype=torch.float16, device="cuda"), err_ws=ws)
    assert b.get_error(ws) & b.DEVERR_RANGE


def test_out_of_range_expert_ids_are_flagged():
    cfg = SMALL["tiny"]
    p = b.params_for(cfg)
    T, k, E = cfg.T, cfg.k, cfg.E
    idx = torch.randint(0, E, (T, k), dtype=torch.int32, device="cuda")
    idx[3, 1] = E  # out of range
    idx[5, 0] = -2
    i32 = dict(dtype=torch.int32, device="cuda")
    rows = b.max_rows(p)
    bufs = [torch.empty(E, **i32), torch.empty(E, **i32), torch.empty(E + 1, **i32), torch.empty(rows, **i32),
            torch.empty(rows, **i32), torch.empty(T * k, **i32)]
    ws = b.workspace(p, b.WS_PERMUTE)
    b.permute(p, idx, *bufs, ws)
    assert b.get_error(ws) & b.DEVERR_BOUNDS
    pr = bufs[5].cpu().numpy().reshape(T, k)
    assert pr[3, 1] == -1 and pr[5, 0] == -1
    assert int(bufs[0].sum()) == T * k - 2
    b.clear_error(ws)
    assert b.get_error(ws) == 0


def test_empty_batch():
    """T = 0: every call succeeds without a launch; counts and offsets come back zero."""
    cfg = synth.LayerConfig("empty", T=0, d=128, f=128, E=8, k=2, has_shared=True, f_shared=128)
    p = b.params_for(cfg)
    Et = cfg.E + 1
    i32 = dict(dtype=torch.int32, device="cuda")
    counts = torch.full((Et,), -3, **i32)
    ws = b.workspace(p, b.WS_FORWARD)
    st = b.lib().moe_forward(ctypes.byref(p), None, None, None, None, ctypes.c_void_p(counts.data_ptr()),
                             ctypes.c_void_p(ws.data_ptr()), ws.numel(), None)
    torch.cuda.synchronize()
    assert st == 0 and int(counts.abs().sum()) == 0
    bufs = [torch.full((Et,), -3, **i32), torch.full((Et,), -3, **i32), torch.full((Et + 1,), -3, **i32),
            torch.empty(1, **i32), torch.empty(1, **i32), torch.empty(1, **i32)]
    wsp = b.workspace(p, b.WS_PERMUTE)
    b.permute(p, torch.empty(1, 2, **i32), *bufs, wsp)
    torch.cuda.synchronize()
    assert all(int(t.abs().sum()) == 0 for t in bufs[:3])
    assert b.get_error(ws) == 0 and b.get_error(wsp) == 0


@pytest.mark.parametrize("name", ["tiny", "prompt", "capped", "decode1", "decode32", "quant"])
def test_route_stats_against_oracle(name):
    """moe_route_stats: the routing bit-identical to moe_route; kept, balance, z and aux against
    the oracle's router telemetry (fp64) within 1e-5 relative; each token's want exact where the
    fp64 cumulative mass is not within 1e-5 of 90% at the decision, and otherwise one of the two
    counts on either side of it; two calls bit-identical."""
    cfg = synth.CONFIGS[name]
    T, E, k = cfg.T, cfg.E, cfg.k
    p = b.params_for(cfg)
    lg_np = synth.logits(cfg)
    lg = torch.from_numpy(lg_np).cuda()
    i32 = dict(dtype=torch.int32, device="cuda")
    f32 = dict(dtype=torch.float32, device="cuda")
    ref_idx, ref_w = torch.empty(T, k, **i32), torch.empty(T, k, **f32)
    b.route(p, lg, ref_idx, ref_w, b.workspace(p, b.WS_ROUTE))
    ws = b.workspace(p, b.WS_ROUTE_STATS)
    zw = 1e-3
    runs = []
    for _ in range(2):
        idx, w = torch.full((T, k), -1, **i32), torch.full((T, k), float("nan"), **f32)
        stats, kept = torch.full((5,), float("nan"), **f32), torch.full((T,), float("nan"), **f32)
        want, est = torch.full((T,), -1, **i32), torch.full((2, E), float("nan"), **f32)
        b.route_stats(p, lg, idx, w, stats, ws, z_weight=zw, kept_tok=kept, want_tok=want, expert_stats=est)
        torch.cuda.synchronize()
        assert b.get_error(ws) == 0
        runs.append([t.cpu().numpy() for t in (idx, w, stats, kept, want, est)])
    for a, c in zip(*runs):
        assert np.array_equal(a.view(np.uint8), c.view(np.uint8)), "two calls differ"
    idx, w, stats, kept, want, est = runs[0]
    assert np.array_equal(idx, ref_idx.cpu().numpy())
    assert np.array_equal(w.view(np.int32), ref_w.cpu().numpy().view(np.int32))
    r = oracle.router_telemetry(lg_np, k, z_weight=zw)
    for i, key in enumerate(("kept", "balance", "z", "aux")):
        got = stats[[0, 2, 3, 4][i]]
        np.testing.assert_allclose(got, r[key], rtol=1e-5, err_msg=key)
    np.testing.assert_allclose(kept, r["kept_tok"], rtol=0, atol=1e-5)
    np.testing.assert_allclose(est[0], r["frac"], rtol=1e-6, atol=0)
    np.testing.assert_allclose(est[1], r["prob_mean"], rtol=1e-5, atol=1e-8)
    # want: the fp64 cumulative mass of the sorted probabilities decides it
    x = lg_np.astype(np.float64)
    pr = np.exp(x - x.max(1, keepdims=True))
    pr /= pr.sum(1, keepdims=True)
    cum = np.cumsum(-np.sort(-pr, axis=1), axis=1)
    ref_want = r["want_tok"]
    near = np.abs(cum[np.arange(T), ref_want - 1] - 0.9) < 1e-5
    near |= (ref_want > 1) & (np.abs(cum[np.arange(T), np.maximum(ref_want - 2, 0)] - 0.9) < 1e-5)
    exact = ~near
    assert np.array_equal(want[exact], ref_want[exact])
    assert (np.abs(want[near] - ref_want[near]) <= 1).all()
    np.testing.assert_allclose(stats[1], r["want_k"], rtol=0, atol=near.sum() / T + 1e-6)
