"""Planted mistakes in the oracle, on the CPU: every plausible slip below — a
dropped term, a wrong sign, index, operand or rounding, a misread drop rule —
must make at least one of the pins in test_oracle_pins.py fail.

Each mutant is a fresh module built from the oracle's source text with one
edit; the oracle itself is never modified. The pins are run against the mutant
by pointing test_oracle_pins' ``oracle`` at it; an assertion or an error raised
by the mistake both count as caught. A control run checks that the unedited
text passes every pin, so a catch is never the harness's own failure.
"""
import types

import numpy as np
import pytest

import oracle
import test_oracle_pins as pins

with open(oracle.__file__) as _fh:
    SRC = _fh.read()

# name -> (text in the oracle, replacement)
MUTATIONS = {
    "backward: silu derivative without its second term": (
        "dg = dh * uc * sg * (1.0 + gc * (1.0 - sg)) * pass_g",
        "dg = dh * uc * sg * pass_g"),
    "backward: clamp passes the gradient outside its range": (
        "pass_g, pass_u = np.abs(g) <= limit, np.abs(u) <= limit",
        "pass_g = pass_u = np.ones(g.shape, bool)"),
    "backward: h recomputed without the clamp": (
        "    h = swiglu_clamped(g, u, limit)\n    dh = dy @ wd.T",
        "    h = swiglu_clamped(g, u, 0.0)\n    dh = dy @ wd.T"),
    "backward: down-projection gradient transposed operands": (
        "x_rows.T @ du, h.T @ dy, h @ wd",
        "x_rows.T @ du, dy.T @ h, h @ wd"),
    "backward: input gradient without the up branch": (
        "return dg @ wg.T + du @ wu.T, x_rows.T @ dg",
        "return dg @ wg.T, x_rows.T @ dg"),
    "backward: expert sees dout without the gate weight": (
        "dy = wf[pairs][:, None] * dout[rows]",
        "dy = dout[rows]"),
    "backward: routing gradient without the weighted mean": (
        "dsel = w * (d_w - (w * d_w).sum(axis=1, keepdims=True))",
        "dsel = w * d_w"),
    "telemetry: kept measured after renormalisation": (
        "kept_tok = np.take_along_axis(probs, idx.astype(np.int64), axis=1).sum(axis=1)",
        "kept_tok = np.take_along_axis(probs, idx.astype(np.int64), axis=1).sum(axis=1)\n"
        "    kept_tok = kept_tok / kept_tok"),
    "telemetry: want off by one": (
        "want_tok = (cum < WANT_MASS).sum(axis=1) + 1",
        "want_tok = (cum < WANT_MASS).sum(axis=1)"),
    "telemetry: want at half the mass": (
        'WANT_MASS = 0.9  #',
        'WANT_MASS = 0.5  #'),
    "telemetry: balance without the factor n": (
        "balance = float((frac * prob_mean).sum() * E)",
        "balance = float((frac * prob_mean).sum())"),
    "telemetry: share of last choices instead of first": (
        "frac = np.bincount(idx[:, 0], minlength=E)",
        "frac = np.bincount(idx[:, -1], minlength=E)"),
    "telemetry: logsumexp without the max": (
        "lse = mx[:, 0] + np.log(ex.sum(axis=1))",
        "lse = np.log(ex.sum(axis=1))"),
    "route: top-k of the full softmax, not renormalised": (
        "    m = sel[:, :1]\n    ex = np.exp(sel - m)\n    w = ex / ex.sum(axis=1, keepdims=True)\n",
        "    full = np.exp(lg.astype(np.float64) - lg.max(axis=1, keepdims=True).astype(np.float64))\n"
        "    full /= full.sum(axis=1, keepdims=True)\n"
        "    w = np.take_along_axis(full, order, axis=1)\n"),
    "route: ties to the higher expert index": (
        'order = np.argsort(-lg, axis=1, kind="stable")[:, :k]',
        'order = (lg.shape[1] - 1 - np.argsort(-lg[:, ::-1], axis=1, kind="stable"))[:, :k]'),
    "route: the k smallest logits (sign)": (
        'order = np.argsort(-lg, axis=1, kind="stable")[:, :k]',
        'order = np.argsort(lg, axis=1, kind="stable")[:, :k]'),
    "capacity: rounded down": (
        "return int(math.ceil(cf * T * k / E))",
        "return int(math.floor(cf * T * k / E))"),
    "capacity: fair share without k": (
        "return int(math.ceil(cf * T * k / E))",
        "return int(math.ceil(cf * T / E))"),
    "permute: overflow dropped from the front (last tokens kept)": (
        "keep = np.ones(order.size, bool) if cap is None else rank < cap",
        "keep = np.ones(order.size, bool) if cap is None else rank >= counts[e_sorted] - cap"),
    "permute: token of a pair by the wrong division": (
        "sorted_token = sorted_pair // k",
        "sorted_token = sorted_pair % k"),
    "permute: kept counts not clamped": (
        "kept = counts if cap is None else np.minimum(counts, cap)",
        "kept = counts"),
    "silu: wrong sign in the sigmoid": (
        "return z / (1.0 + np.exp(-z))",
        "return z / (1.0 + np.exp(z))"),
    "swiglu: only the gate clamped": (
        "        u = np.clip(u, -limit, limit)\n",
        ""),
    "swiglu: gate and up swapped": (
        "return silu(g) * u",
        "return silu(u) * g"),
    "expert_ffn: W_gate used for the up projection": (
        "u = x_rows @ np.asarray(w_up, dtype=np.float64)",
        "u = x_rows @ np.asarray(w_gate, dtype=np.float64)"),
    "dequant: nibble bias 7": (
        ".astype(np.float64) - 8.0",
        ".astype(np.float64) - 7.0"),
    "dequant: nibbles in natural order": (
        "enumerate((0, 2, 4, 6, 1, 3, 5, 7))",
        "enumerate((0, 1, 2, 3, 4, 5, 6, 7))"),
    "dequant: scale groups reversed": (
        "return q.T * s",
        "return q.T * s[::-1]"),
    "combine: gate weight dropped": (
        "out[ok] += w[ok, j:j + 1] * y_rows[r[ok]]",
        "out[ok] += y_rows[r[ok]]"),
    "combine: kept weights renormalised after a drop": (
        "    for j in range(k):\n        r = pr[:, j]",
        "    kw = np.where(pr >= 0, w, 0.0).sum(axis=1, keepdims=True)\n"
        "    w = w / np.where(kw > 0, kw, 1.0)\n"
        "    for j in range(k):\n        r = pr[:, j]"),
    "combine: shared expert not added": (
        "        out += y_rows[shared_base:shared_base + T]",
        "        pass"),
    "forward: capacity ignored": (
        'perm = permute(idx, E, cap, shared_T=T if shared is not None else 0)',
        'perm = permute(idx, E, None, shared_T=T if shared is not None else 0)'),
    "token_outputs: gate weight dropped": (
        "acc += float(w[t, j]) * expert_ffn(",
        "acc += expert_ffn("),
}


def _module(src):
    mod = types.ModuleType("oracle_mutant")
    mod.__file__ = oracle.__file__
    exec(compile(src, "oracle_mutant", "exec"), mod.__dict__)
    return mod


def _pin_calls():
    """Every pin of test_oracle_pins with each of its parameter sets."""
    calls = []
    for name in sorted(dir(pins)):
        fn = getattr(pins, name)
        if not name.startswith("test_") or not callable(fn):
            continue
        marks = [m for m in getattr(fn, "pytestmark", []) if m.name == "parametrize"]
        if not marks:
            calls.append((name, fn, {}))
            continue
        assert len(marks) == 1, name
        names = [a.strip() for a in marks[0].args[0].split(",")]
        for v in marks[0].args[1]:
            vals = tuple(v) if len(names) > 1 else (v,)
            calls.append((f"{name}{vals}", fn, dict(zip(names, vals))))
    return calls


def _first_failing_pin(mod, monkeypatch):
    monkeypatch.setattr(pins, "oracle", mod)
    for label, fn, kw in _pin_calls():
        try:
            with np.errstate(all="ignore"):
                fn(**kw)
        except Exception:  # an assertion, or an error the mistake causes
            return label
    return None


def test_unedited_oracle_passes_every_pin(monkeypatch):
    assert len(_pin_calls()) >= 20
    assert _first_failing_pin(_module(SRC), monkeypatch) is None


@pytest.mark.parametrize("name", list(MUTATIONS))
def test_planted_mistake_is_caught(name, monkeypatch):
    old, new = MUTATIONS[name]
    assert SRC.count(old) == 1, f"mutation site not unique: {name}"
    caught = _first_failing_pin(_module(SRC.replace(old, new)), monkeypatch)
    assert caught is not None, f"no pin catches: {name}"
