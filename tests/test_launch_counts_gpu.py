"""moe_launch_count against the launches the library itself records.

With per-kernel event timing on (moe_profile_enable), every kernel launch of the
library is counted. One call of each entry point must launch exactly the number of
kernels moe_launch_count reports for it — across the paths the fusions choose
between: the single-block front kernel (with and without the row gather), the
separate routing and permutation kernels, the tile and streaming variants, the
K-split reduce folded into the streaming down kernel or not, the combine inside
the streaming down kernel or not, the Q4G32 tiles, the backward and the telemetry.
The benchmark's gpu_launches figure is this count times the steps.
"""
import pytest
import torch

import synth
from mixture_experts_routed_04_b200 import binding as b
from synth.device import upload

pytestmark = pytest.mark.gpu

LAYERS = {
    # front kernel with the gather; every expert streams; K-split folded; combine in the down kernel
    "single_token": synth.LayerConfig("single_token", T=1, d=128, f=256, E=8, k=2),
    # two tokens with a shared expert: no K split (d_model 320), combine in the down kernel
    "two_tokens": synth.LayerConfig("two_tokens", T=2, d=320, f=256, E=8, k=3, has_shared=True, f_shared=256),
    # front kernel without the gather (64 tokens x 4 pairs of 2 KB rows: above its 96 KB)
    "front_64": synth.LayerConfig("front_64", T=64, d=1024, f=256, E=16, k=4),
    # separate routing and permutation kernels
    "ragged": synth.LayerConfig("ragged", T=700, d=192, f=320, E=6, k=3),
    # d_ff too wide for the down kernel's h buffer: the separate K-split reduce
    "wide_ff": synth.LayerConfig("wide_ff", T=3, d=256, f=2176, E=4, k=2),
    # 257 experts: the permutation's scan as its own launch
    "scan_launch": synth.LayerConfig("scan_launch", T=96, d=128, f=128, E=256, k=2, has_shared=True,
                                     f_shared=128),
    "q4_capped": synth.LayerConfig("q4_capped", T=300, d=128, f=192, E=8, k=2, capacity_factor=0.9,
                                   weight_format="q4g32"),
}
VARIANTS = {"auto": b.VARIANT_AUTO, "tensor": b.VARIANT_TENSOR, "stream": b.VARIANT_STREAM}


def launches_of(fn):
    fn()  # warm: first-call set-up (tensor map encoding, attributes) outside the count
    torch.cuda.synchronize()
    b.profile_collect()
    b.profile_enable(True)
    try:
        fn()
        torch.cuda.synchronize()
        prof = b.profile_collect()
    finally:
        b.profile_enable(False)
    return sum(cnt for _, cnt in prof.values())


def weights_of(cfg, d):
    if cfg.weight_format != "bf16":
        return b.weights(d["w_gate"], d["w_up"], d["w_down"], d.get("s_gate"), d.get("s_up"), d.get("s_down"))
    sh = None
    if cfg.has_shared:
        sh = (d["shared_gate"], d["shared_up"], b.prepare_down_f16(d["shared_down"]))
    return b.weights(d["w_gate"], d["w_up"], b.prepare_down_f16(d["w_down"]), shared=sh)


@pytest.mark.parametrize("variant", list(VARIANTS))
@pytest.mark.parametrize("name", list(LAYERS))
def test_forward_launches_match_the_count(name, variant):
    cfg = LAYERS[name]
    if cfg.weight_format != "bf16" and variant == "stream":
        pytest.skip("Q4G32 runs on the tiles only")
    d = upload(cfg, "cuda")
    down = b.DOWN_F16 if cfg.weight_format == "bf16" else b.DOWN_BF16
    p = b.params_for(cfg, variant=VARIANTS[variant], down_dtype=down)
    W = weights_of(cfg, d)
    ws = b.workspace(p, b.WS_FORWARD)
    out = torch.empty(cfg.T, cfg.d, dtype=torch.float32, device="cuda")
    n = launches_of(lambda: b.forward(p, d["x"], d["logits"], W, out, ws))
    assert b.get_error(ws) == 0
    assert n == b.launch_count(p, b.WS_FORWARD), f"{name} {variant}: {n} launches recorded"


def test_backward_and_telemetry_launches_match_the_count():
    cfg = LAYERS["ragged"]
    d = upload(cfg, "cuda")
    p = b.params_for(cfg, down_dtype=b.DOWN_F16)
    T, E, k, dm, f = cfg.T, cfg.E, cfg.k, cfg.d, cfg.f
    rows = b.max_rows(p)
    i32 = dict(dtype=torch.int32, device="cuda")
    f32 = dict(dtype=torch.float32, device="cuda")
    idx, w = torch.empty(T, k, **i32), torch.empty(T, k, **f32)
    counts, kept, offsets = torch.empty(E, **i32), torch.empty(E, **i32), torch.empty(E + 1, **i32)
    st, sp, pr = torch.empty(rows, **i32), torch.empty(rows, **i32), torch.empty(T * k, **i32)
    b.route(p, d["logits"], idx, w, b.workspace(p, b.WS_ROUTE))
    b.permute(p, idx, counts, kept, offsets, st, sp, pr, b.workspace(p, b.WS_PERMUTE))
    W = weights_of(cfg, d)
    G = b.grads(torch.empty(T, dm, **f32), torch.empty(E, dm, f, **f32), torch.empty(E, dm, f, **f32),
                torch.empty(E, f, dm, **f32), torch.empty(T, k, **f32), torch.empty(T, E, **f32))
    dout = torch.randn(T, dm, **f32)
    wsb = b.workspace(p, b.WS_BACKWARD)
    n = launches_of(lambda: b.expert_ffn_backward(p, d["x"], idx, w, offsets, st, sp, pr, W, dout, G, wsb))
    assert b.get_error(wsb) == 0
    assert n == b.launch_count(p, b.WS_BACKWARD)  # dlogits given: the routing gradient too
    stats = torch.empty(5, **f32)
    wss = b.workspace(p, b.WS_ROUTE_STATS)
    idx2, w2 = torch.empty(T, k, **i32), torch.empty(T, k, **f32)
    n = launches_of(lambda: b.route_stats(p, d["logits"], idx2, w2, stats, wss))
    assert n == b.launch_count(p, b.WS_ROUTE_STATS)
