"""Seeded synthetic inputs for the routed MoE expert FFN.

This module only draws numbers. It holds none of the method's arithmetic (no
routing, no permutation, no FFN), so both the fp64 oracle and the CUDA path can
take their inputs from it without sharing any computation.

Every tensor comes from its own stream, ``numpy.random.default_rng([seed,
stream, e])``: one stream per tensor kind and, for weights, one per expert. Any
expert's weights can therefore be regenerated on their own, which lets the
oracle pull only the experts a sampled token touches.

Value recipe (the workloads of the task's five layer configurations):

* x: N(0, 1) fp32, rounded to bf16 (round-to-nearest-even).
* upstream gradient (backward): N(0, 1) fp32.
* router logits: N(0, 1) fp32, plus a per-expert bias:
  - ``zipf``: expert e gets a rank r_e (a seeded permutation of 1..E) and
    bias 3.0 * (1 - ln r_e / ln E), i.e. the log of a Zipf law rescaled to
    [0, 3.0]; the exponent s=1.1 cancels under that rescale. The literal
    reading 3.0 * r^-1.1 is kept as ``zipf_literal``.
  - ``hot``: +4.0 on 8 seeded distinct experts.
  - ``balanced`` (timing sweeps only): +16 on experts (t*k + j) mod touched,
    j < k, so every one of ``touched`` experts gets exactly T*k/touched pairs.
* expert weights W_gate, W_up [d, f] and W_down [f, d]: N(0, 0.02) fp32 → bf16.
* Q4G32 weights (self-defined 4-bit format): the same N(0, 0.02) draws,
  quantised per group of 32 along K with one fp16 scale per group (see
  ``quantize_q4g32``). Quantising is how the *inputs* are made; the path under
  test only dequantises.

bf16 tensors are returned as ``uint16`` bit patterns so that no library
rounding mode is involved; ``bf16_bits_to_f32`` widens them exactly.
"""
from __future__ import annotations

import dataclasses
import math
from concurrent.futures import ThreadPoolExecutor

import numpy as np

# stream ids, one per tensor kind
S_LOGITS, S_X, S_ZIPF_RANK, S_HOT, S_DOUT = 1, 2, 3, 4, 5
S_WG, S_WU, S_WD = 10, 11, 12
S_SWG, S_SWU, S_SWD = 20, 21, 22

WEIGHT_STD = 0.02


@dataclasses.dataclass(frozen=True)
class LayerConfig:
    name: str
    T: int
    d: int
    f: int
    E: int
    k: int
    capacity_factor: float = 0.0
    bias: str = "none"  # none | zipf | zipf_literal | hot | balanced
    touched: int = 0  # balanced: experts 0..touched-1 share the pairs evenly
    has_shared: bool = False
    f_shared: int = 0
    weight_format: str = "bf16"  # bf16 | q4g32
    swiglu_limit: float = 7.0
    seed: int = 0

    def replace(self, **kw) -> "LayerConfig":
        return dataclasses.replace(self, **kw)


# The five layer configurations (sizes as stated for the workload), seed 0.
CONFIGS = {
    "tiny": LayerConfig("tiny", T=64, d=128, f=256, E=8, k=2),
    "prompt": LayerConfig("prompt", T=4096, d=2048, f=768, E=128, k=8, bias="zipf"),
    "capped": LayerConfig("capped", T=8192, d=1024, f=2048, E=128, k=2,
                          capacity_factor=1.5, bias="hot"),
    "decode1": LayerConfig("decode1", T=1, d=4096, f=1536, E=256, k=8,
                           has_shared=True, f_shared=1536),
    "decode8": LayerConfig("decode8", T=8, d=4096, f=1536, E=256, k=8,
                           has_shared=True, f_shared=1536),
    "decode32": LayerConfig("decode32", T=32, d=4096, f=1536, E=256, k=8,
                            has_shared=True, f_shared=1536),
    "quant": LayerConfig("quant", T=32768, d=2048, f=768, E=128, k=8, bias="zipf",
                         weight_format="q4g32"),
}


def _rng(seed: int, stream: int, e: int = 0) -> np.random.Generator:
    return np.random.default_rng([seed, stream, e])


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even); return the uint16 bits.

    Inputs are finite normals here; NaN/Inf are not produced by this module.
    """
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 exactly."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _normal_bf16(seed: int, stream: int, e: int, shape, std: float) -> np.ndarray:
    z = _rng(seed, stream, e).standard_normal(shape, dtype=np.float32)
    if std != 1.0:
        z *= np.float32(std)
    return f32_to_bf16_bits(z)


# --------------------------------------------------------------------------- router

def expert_bias(cfg: LayerConfig) -> np.ndarray:
    """Per-expert logit bias (fp32) for the configuration's bias mode."""
    E = cfg.E
    if cfg.bias == "none":
        return np.zeros(E, np.float32)
    if cfg.bias in ("zipf", "zipf_literal"):
        rank = _rng(cfg.seed, S_ZIPF_RANK).permutation(E) + 1  # rank of expert e
        if cfg.bias == "zipf":
            b = 3.0 * (1.0 - np.log(rank) / math.log(E)) if E > 1 else np.full(E, 3.0)
        else:
            b = 3.0 * rank.astype(np.float64) ** -1.1
        return b.astype(np.float32)
    if cfg.bias == "hot":
        hot = _rng(cfg.seed, S_HOT).permutation(E)[: min(8, E)]
        b = np.zeros(E, np.float32)
        b[hot] = 4.0
        return b
    raise ValueError(cfg.bias)


def logits(cfg: LayerConfig) -> np.ndarray:
    """Router logits [T, E] fp32: N(0,1) plus the per-expert bias; with ``balanced``,
    +16 on experts (t*k + j) mod touched for j < k instead, so those k experts are token t's
    choice and every touched expert receives T*k/touched pairs (timing sweeps over exact
    rows per expert)."""
    z = _rng(cfg.seed, S_LOGITS).standard_normal((cfg.T, cfg.E), dtype=np.float32)
    if cfg.bias == "balanced":
        n = cfg.touched if cfg.touched else cfg.E
        t = np.arange(cfg.T)[:, None]
        cols = (t * cfg.k + np.arange(cfg.k)[None, :]) % n
        z[np.arange(cfg.T)[:, None], cols] += np.float32(16.0)
        return z
    return z + expert_bias(cfg)[None, :]


def dout(cfg: LayerConfig) -> np.ndarray:
    """Upstream gradient dL/d out [T, d] fp32 ~ N(0, 1), for the backward."""
    return _rng(cfg.seed, S_DOUT).standard_normal((cfg.T, cfg.d), dtype=np.float32)


def x_bits(cfg: LayerConfig) -> np.ndarray:
    """Token activations [T, d] as bf16 bits."""
    return _normal_bf16(cfg.seed, S_X, 0, (cfg.T, cfg.d), 1.0)


# --------------------------------------------------------------------------- bf16 weights

def expert_weight_bits(cfg: LayerConfig, e: int, which: str) -> np.ndarray:
    """One expert's bf16 weight bits. which: 'gate'/'up' → [d, f]; 'down' → [f, d]."""
    if which == "gate":
        return _normal_bf16(cfg.seed, S_WG, e, (cfg.d, cfg.f), WEIGHT_STD)
    if which == "up":
        return _normal_bf16(cfg.seed, S_WU, e, (cfg.d, cfg.f), WEIGHT_STD)
    if which == "down":
        return _normal_bf16(cfg.seed, S_WD, e, (cfg.f, cfg.d), WEIGHT_STD)
    raise ValueError(which)


def shared_weight_bits(cfg: LayerConfig, which: str) -> np.ndarray:
    fs = cfg.f_shared
    if which == "gate":
        return _normal_bf16(cfg.seed, S_SWG, 0, (cfg.d, fs), WEIGHT_STD)
    if which == "up":
        return _normal_bf16(cfg.seed, S_SWU, 0, (cfg.d, fs), WEIGHT_STD)
    if which == "down":
        return _normal_bf16(cfg.seed, S_SWD, 0, (fs, cfg.d), WEIGHT_STD)
    raise ValueError(which)


def all_expert_weight_bits(cfg: LayerConfig, which: str, threads: int = 8) -> np.ndarray:
    """Stacked [E, ...] bf16 weight bits, experts drawn in parallel threads."""
    shape = (cfg.d, cfg.f) if which in ("gate", "up") else (cfg.f, cfg.d)
    out = np.empty((cfg.E,) + shape, np.uint16)

    def one(e):
        out[e] = expert_weight_bits(cfg, e, which)

    with ThreadPoolExecutor(max_workers=threads) as ex:
        list(ex.map(one, range(cfg.E)))
    return out


# --------------------------------------------------------------------------- Q4G32 weights
#
# Self-defined format. A matrix with reduction dim K and output dim N is stored
# K-major: packed bytes [N, K/2]. Each row is K/8 little-endian 32-bit words;
# word i holds k = 8i..8i+7, nibble position p (bits 4p..4p+3) holding
# k = 8i + (0, 2, 4, 6, 1, 3, 5, 7)[p]: the pair (k, k+1) sits 16 bits apart,
# which lets a kernel turn one masked word into two fp16 values at once. Each
# nibble u = q + 8 with q in [-7, 7]. Scales are fp16, group-major [K/32, N]:
# one per group of 32 consecutive k of each column. The weight is q * s.

Q4_GROUP = 32
Q4_NIBBLE_K = (0, 2, 4, 6, 1, 3, 5, 7)  # k offset (within a word) of nibble position p


def pack_q4_rows(u: np.ndarray) -> np.ndarray:
    """Pack nibbles u [N, K] (values 0..15) into bytes [N, K/2] in the word order above."""
    N, K = u.shape
    u = u.astype(np.uint32).reshape(N, K // 8, 8)
    words = np.zeros((N, K // 8), np.uint32)
    for p, kk in enumerate(Q4_NIBBLE_K):
        words |= u[:, :, kk] << np.uint32(4 * p)
    return words.astype("<u4").view(np.uint8).reshape(N, K // 2)


def quantize_q4g32(w_kn: np.ndarray):
    """Quantise an fp32 [K, N] matrix to (packed uint8 [N, K/2], scales fp16 [K/32, N]).

    Per group: s = fp16(max|w| / 7) (1.0 if the group is all zero);
    q = clip(rint(w / s), -7, 7) with the fp16-rounded s.
    """
    K, N = w_kn.shape
    assert K % Q4_GROUP == 0
    wt = np.ascontiguousarray(w_kn.T, dtype=np.float32)  # [N, K]
    g = wt.reshape(N, K // Q4_GROUP, Q4_GROUP)
    amax = np.abs(g).max(axis=2)
    s16 = (amax / np.float32(7.0)).astype(np.float16)
    s16[s16 == 0] = np.float16(1.0)
    q = np.rint(g / s16.astype(np.float32)[:, :, None])
    q = np.clip(q, -7, 7).astype(np.int8).reshape(N, K)
    packed = pack_q4_rows((q + 8).astype(np.uint8))
    return packed, np.ascontiguousarray(s16.T)


def expert_q4_weights(cfg: LayerConfig, e: int, which: str):
    """One expert's Q4G32 weights for 'gate'/'up' (K=d, N=f) or 'down' (K=f, N=d)."""
    stream = {"gate": S_WG, "up": S_WU, "down": S_WD}[which]
    shape = (cfg.d, cfg.f) if which in ("gate", "up") else (cfg.f, cfg.d)
    z = _rng(cfg.seed, stream, e).standard_normal(shape, dtype=np.float32) * np.float32(WEIGHT_STD)
    return quantize_q4g32(z)


def all_expert_q4_weights(cfg: LayerConfig, which: str, threads: int = 8):
    K, N = (cfg.d, cfg.f) if which in ("gate", "up") else (cfg.f, cfg.d)
    packed = np.empty((cfg.E, N, K // 2), np.uint8)
    scales = np.empty((cfg.E, K // Q4_GROUP, N), np.float16)

    def one(e):
        packed[e], scales[e] = expert_q4_weights(cfg, e, which)

    with ThreadPoolExecutor(max_workers=threads) as ex:
        list(ex.map(one, range(cfg.E)))
    return packed, scales
