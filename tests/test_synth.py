"""The seeded generator: bf16 rounding, determinism, per-expert streams, workload shapes."""
import numpy as np

import synth


def test_bf16_round_nearest_even():
    vals = np.array([1.0, 1.0 + 2**-8, 1.0 + 3 * 2**-8, 1.0 + 2**-8 + 2**-20, -2.5, 3.0e-39], np.float32)
    bits = synth.f32_to_bf16_bits(vals)
    # 1+2^-8 is a tie between 1.0 and 1+2^-7: to even (1.0); 1+3*2^-8 ties to 1+2^-6 (even)
    want = [0x3F80, 0x3F80, 0x3F82, 0x3F81, 0xC020, 0x0021]
    assert bits.tolist() == want
    assert (synth.bf16_bits_to_f32(bits)[:3] == np.array([1.0, 1.0, 1.0 + 2**-6], np.float32)).all()


def test_deterministic_and_per_expert_streams():
    cfg = synth.CONFIGS["tiny"]
    a = synth.expert_weight_bits(cfg, 3, "gate")
    assert (a == synth.expert_weight_bits(cfg, 3, "gate")).all()
    assert not (a == synth.expert_weight_bits(cfg, 4, "gate")).all()
    stacked = synth.all_expert_weight_bits(cfg, "gate")
    assert (stacked[3] == a).all()
    assert (synth.logits(cfg) == synth.logits(cfg)).all()


def test_workload_shapes_and_stats():
    c = synth.CONFIGS
    assert synth.logits(c["prompt"]).shape == (4096, 128)
    assert synth.x_bits(c["tiny"]).shape == (64, 128)
    w = synth.bf16_bits_to_f32(synth.expert_weight_bits(c["tiny"], 0, "down"))
    assert w.shape == (256, 128) and abs(w.std() - 0.02) < 0.002
    b = synth.expert_bias(c["prompt"])
    assert abs(b.max() - 3.0) < 1e-6 and abs(b.min()) < 1e-6
    hot = synth.expert_bias(c["capped"])
    assert (hot == 4.0).sum() == 8 and (hot == 0.0).sum() == 120
    packed, s = synth.expert_q4_weights(c["tiny"], 0, "gate")
    assert packed.shape == (256, 64) and s.shape == (4, 256) and s.dtype == np.float16
    lo, hi = packed & 15, packed >> 4
    assert lo.min() >= 1 and hi.max() <= 15  # nibbles are q+8 with q in [-7, 7]
