"""Place the seeded synthetic inputs in device memory (PyTorch tensors).

Input logistics only: draws come from ``synth``; nothing here computes any part
of the layer. Experts that are not listed are filled with NaN bf16 so that a
kernel reading an untouched expert's weights shows up in the outputs.
"""
from __future__ import annotations

from concurrent.futures import ThreadPoolExecutor

import numpy as np

import synth


def _bf16(bits: np.ndarray, device):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(torch.bfloat16)


def upload(cfg: synth.LayerConfig, device="cuda", experts=None, threads: int = 8):
    """Return dict: x [T,d] bf16, logits [T,E] f32, w_gate/w_up [E,d,f], w_down [E,f,d] bf16
    (or Q4G32 packed/scales), shared_* when cfg.has_shared. ``experts``: iterable of
    expert ids to fill (default: all); the others hold NaN."""
    import torch
    out = {"x": _bf16(synth.x_bits(cfg), device),
           "logits": torch.from_numpy(synth.logits(cfg)).to(device)}
    E, d, f = cfg.E, cfg.d, cfg.f
    ids = list(range(E)) if experts is None else sorted(set(int(e) for e in experts))
    if cfg.weight_format == "q4g32":
        shapes = {"gate": (f, d), "up": (f, d), "down": (d, f)}  # [N, K]
        for w, (N, K) in shapes.items():
            pk = torch.zeros((E, N, K // 2), dtype=torch.uint8, device=device)
            sc = torch.full((E, K // 32, N), float("nan"), dtype=torch.float16, device=device)

            def one(e, w=w, pk=pk, sc=sc):
                p, s = synth.expert_q4_weights(cfg, e, w)
                return e, p, s

            with ThreadPoolExecutor(max_workers=threads) as ex:
                for e, p, s in ex.map(one, ids):
                    pk[e].copy_(torch.from_numpy(p))
                    sc[e].copy_(torch.from_numpy(s))
            out["w_" + w], out["s_" + w] = pk, sc
    else:
        for w in ("gate", "up", "down"):
            shape = (E, d, f) if w != "down" else (E, f, d)
            t = torch.full(shape, float("nan"), dtype=torch.bfloat16, device=device)

            def one(e, w=w):
                return e, synth.expert_weight_bits(cfg, e, w)

            with ThreadPoolExecutor(max_workers=threads) as ex:
                for e, bits in ex.map(one, ids):
                    t[e].copy_(_bf16(bits, "cpu"))
            out["w_" + w] = t
    if cfg.has_shared:
        for w in ("gate", "up", "down"):
            out["shared_" + w] = _bf16(synth.shared_weight_bits(cfg, w), device)
    return out


def expert_f64(cfg: synth.LayerConfig, e: int):
    """(W_gate [d,f], W_up [d,f], W_down [f,d]) of one expert as float64 (CPU)."""
    if cfg.weight_format == "q4g32":
        raise ValueError("use the oracle's dequantisation for Q4G32")
    return tuple(synth.bf16_bits_to_f32(synth.expert_weight_bits(cfg, e, w)).astype(np.float64)
                 for w in ("gate", "up", "down"))


def shared_f64(cfg: synth.LayerConfig):
    return tuple(synth.bf16_bits_to_f32(synth.shared_weight_bits(cfg, w)).astype(np.float64)
                 for w in ("gate", "up", "down"))
