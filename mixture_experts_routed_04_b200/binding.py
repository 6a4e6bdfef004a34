"""Thin Python binding of the C ABI in ``include/moe.h`` (ctypes).

Argument marshalling only: every step of the layer runs in the CUDA kernels of
``libmoe_b200.so``. PyTorch supplies device memory and the current stream. If
the library has not been built, loading it raises ``MoeError``; there is no
fallback of any kind.

Tensors are passed by ``data_ptr()``: x and bf16 weights as ``torch.bfloat16``
(or int16 bit patterns), y_rows as ``torch.float16``, the layer output as
``torch.float32`` (default) or ``torch.bfloat16`` (out_dtype=OUT_BF16). Calls are asynchronous on
``torch.cuda.current_stream()`` unless a stream is given.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libmoe_b200.so")

MOE_OK = 0
MOE_ERR_DEVICE = 6  # moe_get_error: the device error word is set
STATUS = {0: "ok", 1: "invalid argument", 2: "workspace too small", 3: "unsupported configuration",
          4: "CUDA error", 5: "misaligned pointer", 6: "device error word set"}
DEVERR_TIMEOUT, DEVERR_BOUNDS, DEVERR_RANGE = 0x1, 0x2, 0x4
OUT_F32, OUT_BF16 = 0, 1
DOWN_BF16, DOWN_F16 = 0, 1
WEIGHTS_BF16, WEIGHTS_Q4G32 = 0, 1
VARIANT_AUTO, VARIANT_TENSOR, VARIANT_STREAM = 0, 1, 2
TILE_AUTO, TILE_ONE, TILE_PAIR = 0, 1, 2
WS_ROUTE, WS_PERMUTE, WS_EXPERT_FFN, WS_COMBINE, WS_FORWARD, WS_FORWARD_HOST, WS_ROUTE_STATS, WS_BACKWARD = range(8)

# every entry point declared in include/moe.h
EXPORTS = ("moe_version", "moe_status_string", "moe_capacity", "moe_max_rows", "moe_workspace_size",
           "moe_route", "moe_permute", "moe_expert_ffn", "moe_combine", "moe_forward", "moe_forward_host",
           "moe_get_error", "moe_clear_error", "moe_set_wait_limit_ns", "moe_launch_count",
           "moe_profile_enable", "moe_profile_collect", "moe_convert_bf16_to_f16",
           "moe_permute_noalloc", "moe_forward_host_async", "moe_wait_selftest", "moe_tile_ctas",
           "moe_route_stats", "moe_expert_ffn_backward", "moe_variant_table")
NOALLOC_MAX_PAIRS = 262144  # MOE_NOALLOC_MAX_PAIRS

# kernel ids (MOE_K_*), in order
KERNELS = ("route", "perm_count", "perm_scan", "perm_scatter", "schedule", "gather", "tc_gateup", "tc_down",
           "stream_gateup", "stream_reduce", "stream_down", "combine", "convert", "front", "route_stats",
           "bwd_gemm", "bwd_small")


class MoeError(RuntimeError):
    pass


class Params(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("d_model", ctypes.c_int32), ("d_ff", ctypes.c_int32),
                ("E", ctypes.c_int32), ("k", ctypes.c_int32), ("capacity_factor", ctypes.c_float),
                ("swiglu_limit", ctypes.c_float), ("weight_format", ctypes.c_int32),
                ("has_shared", ctypes.c_int32), ("d_ff_shared", ctypes.c_int32),
                ("variant", ctypes.c_int32), ("stream_max_rows", ctypes.c_int32), ("out_dtype", ctypes.c_int32),
                ("down_dtype", ctypes.c_int32), ("tile_ctas", ctypes.c_int32)]


class Weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("w_gate", "w_up", "w_down", "s_gate", "s_up", "s_down",
                                               "shared_gate", "shared_up", "shared_down")]


class Grads(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("dx", "dw_gate", "dw_up", "dw_down", "d_topk_w", "dlogits",
                                               "dshared_gate", "dshared_up", "dshared_down")]


_lib = None
_P, _V, _S = ctypes.POINTER(Params), ctypes.c_void_p, ctypes.c_size_t


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise MoeError(f"{LIB_PATH} is not built; run `python -m mixture_experts_routed_04_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        sig = {
            "moe_version": ([], ctypes.c_int),
            "moe_status_string": ([ctypes.c_int], ctypes.c_char_p),
            "moe_capacity": ([_P, ctypes.POINTER(ctypes.c_int32)], ctypes.c_int),
            "moe_max_rows": ([_P, ctypes.POINTER(ctypes.c_int64)], ctypes.c_int),
            "moe_tile_ctas": ([_P, ctypes.POINTER(ctypes.c_int32)], ctypes.c_int),
            "moe_workspace_size": ([_P, ctypes.c_int], _S),
            "moe_route": ([_P, _V, _V, _V, _V, _S, _V], ctypes.c_int),
            "moe_route_stats": ([_P, _V, _V, _V, ctypes.c_float, _V, _V, _V, _V, _V, _S, _V], ctypes.c_int),
            "moe_permute": ([_P, _V, _V, _V, _V, _V, _V, _V, _V, _S, _V], ctypes.c_int),
            "moe_expert_ffn": ([_P, _V, _V, _V, _V, _V, ctypes.POINTER(Weights), _V, _V, _S, _V], ctypes.c_int),
            "moe_combine": ([_P, _V, _V, _V, _V, _V, _S, _V], ctypes.c_int),
            "moe_forward": ([_P, _V, _V, ctypes.POINTER(Weights), _V, _V, _V, _S, _V], ctypes.c_int),
            "moe_forward_host": ([_P, _V, _V, ctypes.POINTER(Weights), _V, _V, _S, _V], ctypes.c_int),
            "moe_forward_host_async": ([_P, _V, _V, ctypes.POINTER(Weights), _V, _V, _S, _V], ctypes.c_int),
            "moe_wait_selftest": ([_V, ctypes.c_uint64, _V], ctypes.c_int),
            "moe_get_error": ([_V, ctypes.POINTER(ctypes.c_uint32), _V], ctypes.c_int),
            "moe_clear_error": ([_V, _V], ctypes.c_int),
            "moe_set_wait_limit_ns": ([ctypes.c_uint64], ctypes.c_int),
            "moe_launch_count": ([_P, ctypes.c_int, ctypes.POINTER(ctypes.c_int)], ctypes.c_int),
            "moe_profile_enable": ([ctypes.c_int], ctypes.c_int),
            "moe_profile_collect": ([ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int64)], ctypes.c_int),
            "moe_convert_bf16_to_f16": ([_V, _V, ctypes.c_int64, _V, _V], ctypes.c_int),
            "moe_permute_noalloc": ([_P, _V, _V, _V, _V, _V, _V, _V, _V, _V], ctypes.c_int),
            "moe_variant_table": ([ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_int32), ctypes.c_int],
                                  ctypes.c_int),
            "moe_expert_ffn_backward": ([_P, _V, _V, _V, _V, _V, _V, _V, ctypes.POINTER(Weights), _V,
                                         ctypes.POINTER(Grads), _V, _S, _V], ctypes.c_int),
        }
        for name, (args, res) in sig.items():
            fn = getattr(L, name)
            fn.argtypes, fn.restype = args, res
        _lib = L
    return _lib


def params(T, d_model, d_ff, E, k, capacity_factor=0.0, swiglu_limit=7.0, weight_format=WEIGHTS_BF16,
           has_shared=0, d_ff_shared=0, variant=VARIANT_AUTO, stream_max_rows=-1, out_dtype=OUT_F32,
           down_dtype=DOWN_BF16, tile_ctas=TILE_AUTO) -> Params:
    return Params(T, d_model, d_ff, E, k, capacity_factor, swiglu_limit, weight_format, int(has_shared),
                  d_ff_shared if has_shared else 0, variant, stream_max_rows, out_dtype, down_dtype, tile_ctas)


def params_for(cfg, **over) -> Params:
    """Params of a ``synth.LayerConfig``-like object (fields T, d, f, E, k, ...)."""
    kw = dict(T=cfg.T, d_model=cfg.d, d_ff=cfg.f, E=cfg.E, k=cfg.k, capacity_factor=cfg.capacity_factor,
              swiglu_limit=cfg.swiglu_limit,
              weight_format=WEIGHTS_Q4G32 if cfg.weight_format == "q4g32" else WEIGHTS_BF16,
              has_shared=int(cfg.has_shared), d_ff_shared=cfg.f_shared)
    kw.update(over)
    return params(**kw)


def check(status: int, what: str = "") -> None:
    if status != MOE_OK:
        raise MoeError(f"{what}: {STATUS.get(status, status)}")


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def capacity(p: Params):
    v = ctypes.c_int32()
    check(lib().moe_capacity(ctypes.byref(p), ctypes.byref(v)), "moe_capacity")
    return None if v.value < 0 else v.value


def tile_ctas(p: Params) -> int:
    """SMs per tcgen05 tile these params use (TILE_ONE or TILE_PAIR)."""
    v = ctypes.c_int32()
    check(lib().moe_tile_ctas(ctypes.byref(p), ctypes.byref(v)), "moe_tile_ctas")
    return v.value


def max_rows(p: Params) -> int:
    v = ctypes.c_int64()
    check(lib().moe_max_rows(ctypes.byref(p), ctypes.byref(v)), "moe_max_rows")
    return v.value


def workspace_size(p: Params, which: int) -> int:
    return int(lib().moe_workspace_size(ctypes.byref(p), which))


def workspace(p: Params, which: int, device="cuda"):
    """A zeroed device workspace of the size `which` needs (256-byte aligned)."""
    import torch
    n = workspace_size(p, which)
    if n == 0:
        raise MoeError("invalid parameters")
    ws = torch.zeros(n, dtype=torch.uint8, device=device)
    assert ws.data_ptr() % 256 == 0
    return ws


def weights(w_gate, w_up, w_down, s_gate=None, s_up=None, s_down=None, shared=None) -> Weights:
    sh = shared or (None, None, None)
    W = Weights(*(None if t is None else t.data_ptr() for t in (w_gate, w_up, w_down, s_gate, s_up, s_down, *sh)))
    W._keep = (w_gate, w_up, w_down, s_gate, s_up, s_down, *sh)  # keep the tensors alive
    return W


def route(p, logits, topk_idx, topk_w, ws, stream=None):
    check(lib().moe_route(ctypes.byref(p), _p(logits), _p(topk_idx), _p(topk_w), _p(ws), ws.numel(),
                          _stream(stream)), "moe_route")


STATS = ("kept", "want_k", "balance", "z", "aux")  # moe_route_stats stats[0..4]


def route_stats(p, logits, topk_idx, topk_w, stats, ws, z_weight=1e-3, kept_tok=None, want_tok=None,
                expert_stats=None, stream=None):
    """moe_route_stats: moe_route plus the router telemetry (stats: device fp32 [5], see STATS)."""
    check(lib().moe_route_stats(ctypes.byref(p), _p(logits), _p(topk_idx), _p(topk_w), float(z_weight), _p(stats),
                                _p(kept_tok), _p(want_tok), _p(expert_stats), _p(ws), ws.numel(),
                                _stream(stream)), "moe_route_stats")


def permute(p, topk_idx, counts, kept, offsets, sorted_token, sorted_pair, pair_row, ws, stream=None):
    check(lib().moe_permute(ctypes.byref(p), _p(topk_idx), _p(counts), _p(kept), _p(offsets), _p(sorted_token),
                            _p(sorted_pair), _p(pair_row), _p(ws), ws.numel(), _stream(stream)), "moe_permute")


def permute_noalloc(p, topk_idx, counts, kept, offsets, sorted_token, sorted_pair, pair_row, err_word,
                    stream=None):
    """moe_permute with the library's fixed scratch array instead of a workspace (one stream only)."""
    check(lib().moe_permute_noalloc(ctypes.byref(p), _p(topk_idx), _p(counts), _p(kept), _p(offsets),
                                    _p(sorted_token), _p(sorted_pair), _p(pair_row), _p(err_word),
                                    _stream(stream)), "moe_permute_noalloc")


def expert_ffn(p, x, offsets, sorted_token, sorted_pair, topk_w, W: Weights, y_rows, ws, stream=None):
    check(lib().moe_expert_ffn(ctypes.byref(p), _p(x), _p(offsets), _p(sorted_token), _p(sorted_pair), _p(topk_w),
                               ctypes.byref(W), _p(y_rows), _p(ws), ws.numel(), _stream(stream)), "moe_expert_ffn")


def combine(p, y_rows, pair_row, offsets, out, ws, stream=None):
    check(lib().moe_combine(ctypes.byref(p), _p(y_rows), _p(pair_row), _p(offsets), _p(out), _p(ws), ws.numel(),
                            _stream(stream)), "moe_combine")


def grads(dx, dw_gate, dw_up, dw_down, d_topk_w, dlogits=None, shared=None) -> Grads:
    sh = shared or (None, None, None)
    ts = (dx, dw_gate, dw_up, dw_down, d_topk_w, dlogits, *sh)
    G = Grads(*(None if t is None else t.data_ptr() for t in ts))
    G._keep = ts
    return G


def expert_ffn_backward(p, x, topk_idx, topk_w, offsets, sorted_token, sorted_pair, pair_row, W: Weights, dout,
                        G: Grads, ws, stream=None):
    """moe_expert_ffn_backward: gradients of the layer for dout (fp32 [T, d]) into G (fp32)."""
    check(lib().moe_expert_ffn_backward(ctypes.byref(p), _p(x), _p(topk_idx), _p(topk_w), _p(offsets),
                                        _p(sorted_token), _p(sorted_pair), _p(pair_row), ctypes.byref(W), _p(dout),
                                        ctypes.byref(G), _p(ws), ws.numel(), _stream(stream)),
          "moe_expert_ffn_backward")


def forward(p, x, logits, W: Weights, out, ws, counts_out=None, stream=None):
    check(lib().moe_forward(ctypes.byref(p), _p(x), _p(logits), ctypes.byref(W), _p(out), _p(counts_out), _p(ws),
                            ws.numel(), _stream(stream)), "moe_forward")


def forward_host(p, x_host, logits_host, W: Weights, out_host, ws, stream=None):
    """moe_forward_host: host (CPU, ideally pinned) x/logits/out; synchronises the stream."""
    check(lib().moe_forward_host(ctypes.byref(p), _p(x_host), _p(logits_host), ctypes.byref(W), _p(out_host),
                                 _p(ws), ws.numel(), _stream(stream)), "moe_forward_host")


def forward_host_async(p, x_host, logits_host, W: Weights, out_host, ws, stream=None):
    """moe_forward_host_async: as forward_host, enqueued on the stream without synchronising."""
    check(lib().moe_forward_host_async(ctypes.byref(p), _p(x_host), _p(logits_host), ctypes.byref(W),
                                       _p(out_host), _p(ws), ws.numel(), _stream(stream)), "moe_forward_host_async")


def wait_selftest(err_ws, limit_ns, stream=None):
    """moe_wait_selftest: a bounded wait on a barrier nothing completes; sets DEVERR_TIMEOUT."""
    check(lib().moe_wait_selftest(_p(err_ws), int(limit_ns), _stream(stream)), "moe_wait_selftest")


def get_error(ws, stream=None) -> int:
    v = ctypes.c_uint32()
    st = lib().moe_get_error(_p(ws), ctypes.byref(v), _stream(stream))
    if st not in (MOE_OK, MOE_ERR_DEVICE):
        check(st, "moe_get_error")
    return v.value


def clear_error(ws, stream=None) -> None:
    check(lib().moe_clear_error(_p(ws), _stream(stream)), "moe_clear_error")


def set_wait_limit_ns(ns: int) -> None:
    check(lib().moe_set_wait_limit_ns(ns), "moe_set_wait_limit_ns")


def variant_table():
    """[(tiles_per_sm, max_rows), ...]: the measured rows of the default variant choice."""
    n = lib().moe_variant_table(None, None, 0)
    a, r = (ctypes.c_float * n)(), (ctypes.c_int32 * n)()
    lib().moe_variant_table(a, r, n)
    return [(float(a[i]), int(r[i])) for i in range(n)]


def launch_count(p: Params, which: int) -> int:
    v = ctypes.c_int()
    check(lib().moe_launch_count(ctypes.byref(p), which, ctypes.byref(v)), "moe_launch_count")
    return v.value


def profile_enable(on: bool = True) -> None:
    check(lib().moe_profile_enable(int(on)), "moe_profile_enable")


def profile_collect() -> dict:
    """{kernel name: (total ms, launches)} since the last collect (waits for the events)."""
    n = len(KERNELS)
    ms = (ctypes.c_double * n)()
    cnt = (ctypes.c_int64 * n)()
    check(lib().moe_profile_collect(ms, cnt), "moe_profile_collect")
    return {KERNELS[i]: (ms[i], cnt[i]) for i in range(n)}


def convert_bf16_to_f16(src, dst, err_ws=None, stream=None) -> None:
    """Load-time weight preparation: dst (fp16) = src (bf16), elementwise."""
    assert src.numel() == dst.numel()
    check(lib().moe_convert_bf16_to_f16(_p(src), _p(dst), src.numel(), _p(err_ws), _stream(stream)),
          "moe_convert_bf16_to_f16")


def prepare_down_f16(w_down, stream=None):
    """fp16 copy of a bf16 W_down (or shared W_down), for down_dtype=DOWN_F16."""
    import torch
    out = torch.empty(w_down.shape, dtype=torch.float16, device=w_down.device)
    convert_bf16_to_f16(w_down, out, stream=stream)
    return out
