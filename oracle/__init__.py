"""fp64 CPU oracle for the routed mixture-of-experts expert FFN.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import, call or run
this package: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` use it. It shares no code with the CUDA library; both take
their inputs from the ``synth`` generator alone.

It is the plain definition of what the path computes, in float64, with no
blocking, fusion or reordering beyond what the definition states. Sources:

* "mini-AGI PR #3" (gt50/mini-AGI, files diff), ``minagi/pool.py``, the
  ``requested(scores)`` router hunk: full softmax ``probs`` of the router
  logits, the top-k ``idx``/``w``, ``w`` renormalised after the telemetry has
  read its pre-normalisation mass; then the flatten / ``argsort`` by expert /
  ``bincount`` hunk, and the capacity-drop hunk (``keep`` mask over the sorted
  pairs, ``counts.clamp(max=limit)``).
* the same pages' ``configs/strix_halo_large.yaml`` ``capacity_factor`` comment:
  the most of a batch one expert may take, as a multiple of its fair share; the
  rest is dropped; 0 removes the cap.
* "mini-AGI PR #4" ``minagi/pool.py`` ``experts()``/``run()``: per expert,
  ``silu(x W1) * (x W3)`` then ``W2``, gathered back in pair order.
* "Strata PR #4366" (DS4_FAT_ROWS), "Approach": the SwiGLU is clamped.
* "TensorFold PR #1607", "What this changes": served plans with "256 + shared"
  experts (an always-on shared expert).

Readings taken where the pages are silent:
top-k ties go to the lower expert index; the capacity is
``ceil(cf * T * k / E)`` with cf widened from float32; overflow is dropped in
token order and the kept weights are NOT renormalised; the clamp bounds both
the gate and the up pre-activation to [-L, L]; the shared expert is un-gated
(weight 1) and holds every token.

Pins: every function here is checked in ``tests/test_oracle_pins.py`` against
closed forms, brute force on tiny inputs, invariants and special cases.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "route", "router_telemetry", "capacity", "permute", "silu", "swiglu_clamped", "expert_ffn",
    "dequant_q4g32", "combine", "forward", "token_outputs",
    "swiglu_clamped_backward", "expert_ffn_backward", "route_backward", "backward",
]


# --------------------------------------------------------------------------- route

def route(logits: np.ndarray, k: int):
    """Top-k experts per token and their weights.

    mini-AGI PR #3, ``requested()``: ``probs = softmax(logits)``, ``idx, w`` =
    top-k of ``probs``, then ``w / w.sum(-1)``. Renormalising the top-k of a
    full softmax equals a softmax over the k selected logits, which is what is
    computed here (in float64).

    The ranking compares the given float32 logits exactly; ties go to the lower
    expert index (stable sort of the negated values). NaN logits are outside
    the contract.

    Returns idx int32 [T, k] (descending logit order) and w float64 [T, k].
    """
    lg = np.asarray(logits, dtype=np.float32)
    T, E = lg.shape
    if not 1 <= k <= E:
        raise ValueError("need 1 <= k <= E")
    order = np.argsort(-lg, axis=1, kind="stable")[:, :k]
    sel = np.take_along_axis(lg, order, axis=1).astype(np.float64)
    m = sel[:, :1]
    ex = np.exp(sel - m)
    w = ex / ex.sum(axis=1, keepdims=True)
    return order.astype(np.int32), w


# --------------------------------------------------------------------------- router telemetry

WANT_MASS = 0.9  # "the smallest number of experts covering 90% of the probability mass"


def router_telemetry(logits: np.ndarray, k: int, z_weight: float = 1e-3):
    """Router telemetry and auxiliary losses of one batch, float64.

    mini-AGI PR #3, ``requested()`` telemetry hunk, on the full softmax
    ``probs`` of each token's logits and its top-k ``idx``:

    * ``kept``: the top-k probability mass measured BEFORE the top-k weights
      are renormalised (afterwards it is 1 by construction), averaged over the
      tokens: mean_t sum_j probs[t, idx[t, j]].
    * ``want_k``: per token, the smallest number of experts whose
      probabilities sum to at least 90% of the mass (the largest ones first);
      averaged over the tokens like ``kept``.
    * ``balance``: ``(frac * probs.mean(0)).sum() * n`` with ``frac[e]`` the
      share of tokens whose first choice ``idx[t, 0]`` is e and n = E.
    * ``z``: ``logsumexp(logits, -1).pow(2).mean()``.
    * ``aux`` = balance + z_weight * z (the hunk's default weight is 1e-3).

    The page keeps exponential moving averages of ``1 - kept`` ("pressure")
    and of ``want`` across calls; those running averages are the caller's
    state, so the per-batch values are what is returned.

    Returns a dict: per-token ``kept_tok`` [T], ``want_tok`` [T] (int), ``lse``
    [T]; per-expert ``frac`` [E], ``prob_mean`` [E]; scalars ``kept``,
    ``want_k``, ``balance``, ``z``, ``aux``.
    """
    lg = np.asarray(logits, dtype=np.float32)
    T, E = lg.shape
    idx, _ = route(lg, k)
    x = lg.astype(np.float64)
    mx = x.max(axis=1, keepdims=True)
    ex = np.exp(x - mx)
    lse = mx[:, 0] + np.log(ex.sum(axis=1))
    probs = ex / ex.sum(axis=1, keepdims=True)
    kept_tok = np.take_along_axis(probs, idx.astype(np.int64), axis=1).sum(axis=1)
    srt = -np.sort(-probs, axis=1)  # largest first
    cum = np.cumsum(srt, axis=1)
    want_tok = (cum < WANT_MASS).sum(axis=1) + 1  # first m with cum[m-1] >= 0.9
    want_tok = np.minimum(want_tok, E)
    frac = np.bincount(idx[:, 0], minlength=E).astype(np.float64) / T
    prob_mean = probs.mean(axis=0)
    balance = float((frac * prob_mean).sum() * E)
    z = float(np.mean(lse ** 2))
    return {"kept_tok": kept_tok, "want_tok": want_tok.astype(np.int64), "lse": lse, "frac": frac,
            "prob_mean": prob_mean, "kept": float(kept_tok.mean()), "want_k": float(want_tok.mean()),
            "balance": balance, "z": z, "aux": balance + z_weight * z}


# --------------------------------------------------------------------------- capacity

def capacity(T: int, k: int, E: int, capacity_factor: float):
    """Rows one expert may take, or None for no cap.

    mini-AGI ``capacity_factor``: a multiple of an expert's fair share T*k/E;
    0 removes the cap. The rounding up (ceil) is the stated workload's. The
    factor is read as float32 (the boundary passes it so) and widened.
    """
    cf = float(np.float32(capacity_factor))
    if cf <= 0.0:
        return None
    return int(math.ceil(cf * T * k / E))


# --------------------------------------------------------------------------- permute

def permute(idx: np.ndarray, E: int, cap=None, shared_T: int = 0):
    """Group the (token, expert) pairs by expert, in token order, and drop overflow.

    mini-AGI PR #3, ``requested()``: ``flat_e``/``tok`` flattened, ``order =
    argsort(flat_e)``, ``counts = bincount(e_sorted)``; with a capacity,
    ``keep`` = the pairs whose slot is below the limit, the rest counted as
    dropped and filtered out, ``counts.clamp(max=limit)``.

    Pair p = t*k + j. Within an expert, rows are in ascending p, which is
    ascending token (a token's k experts are distinct). A pair of rank >= cap
    in its expert is dropped: ``pair_row[p] = -1``.

    With ``shared_T > 0`` an always-on shared expert is appended as expert
    index E holding every token 0..T-1 in order (``sorted_pair = -1``).

    Returns a dict of int32/int64 arrays: counts, kept, offsets, sorted_token,
    sorted_pair, pair_row.
    """
    idx = np.asarray(idx)
    T, k = idx.shape
    flat_e = idx.reshape(-1).astype(np.int64)
    counts = np.bincount(flat_e, minlength=E).astype(np.int64)
    order = np.argsort(flat_e, kind="stable")  # pairs grouped by expert, ascending p
    e_sorted = flat_e[order]
    first = np.concatenate([[0], np.cumsum(counts)[:-1]])
    rank = np.arange(order.size) - first[e_sorted]
    keep = np.ones(order.size, bool) if cap is None else rank < cap
    kept = counts if cap is None else np.minimum(counts, cap)
    sorted_pair = order[keep]
    sorted_token = sorted_pair // k
    if shared_T:
        counts = np.concatenate([counts, [shared_T]])
        kept = np.concatenate([kept, [shared_T]])
        sorted_token = np.concatenate([sorted_token, np.arange(shared_T)])
        sorted_pair = np.concatenate([sorted_pair, np.full(shared_T, -1)])
    offsets = np.concatenate([[0], np.cumsum(kept)])
    pair_row = np.full(T * k, -1, np.int64)
    n_routed = int(keep.sum())
    pair_row[sorted_pair[:n_routed]] = np.arange(n_routed)
    return {
        "counts": counts.astype(np.int32), "kept": kept.astype(np.int32),
        "offsets": offsets.astype(np.int32), "sorted_token": sorted_token.astype(np.int32),
        "sorted_pair": sorted_pair.astype(np.int32), "pair_row": pair_row.astype(np.int32),
    }


# --------------------------------------------------------------------------- FFN

def silu(z):
    """silu(z) = z * sigmoid(z) = z / (1 + exp(-z)), float64."""
    z = np.asarray(z, dtype=np.float64)
    return z / (1.0 + np.exp(-z))


def swiglu_clamped(g, u, limit: float):
    """Clamped SwiGLU: silu(clamp(g, -L, L)) * clamp(u, -L, L).

    Strata PR #4366, "Approach": the fat-rows route applies a clamped SwiGLU.
    The bound L (7.0 for the stated workloads) applies to both the gate and
    the up pre-activation. ``limit <= 0`` means no clamp.
    """
    g = np.asarray(g, dtype=np.float64)
    u = np.asarray(u, dtype=np.float64)
    if limit > 0:
        g = np.clip(g, -limit, limit)
        u = np.clip(u, -limit, limit)
    return silu(g) * u


def expert_ffn(x_rows, w_gate, w_up, w_down, limit: float):
    """One expert on its rows: y = swiglu(x Wg, x Wu) Wd, all float64.

    mini-AGI PR #4, ``experts()``: ``h = silu(x W1) * (x W3)``, ``y = h W2``
    (W_gate, W_up are [d, f]; W_down is [f, d]). No intermediate rounding.
    """
    x_rows = np.asarray(x_rows, dtype=np.float64)
    g = x_rows @ np.asarray(w_gate, dtype=np.float64)
    u = x_rows @ np.asarray(w_up, dtype=np.float64)
    h = swiglu_clamped(g, u, limit)
    return h @ np.asarray(w_down, dtype=np.float64)


def dequant_q4g32(packed: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Q4G32 (self-defined) → float64 [K, N]: w[k, n] = q * s exactly.

    packed uint8 [N, K/2]: each row is K/8 little-endian 32-bit words; word i
    holds k = 8i..8i+7, nibble position p (bits 4p..4p+3) holding
    k = 8i + (0, 2, 4, 6, 1, 3, 5, 7)[p]; each nibble u = q + 8.
    scales fp16 [K/32, N]: one scale per group of 32 consecutive k of a column.
    """
    packed = np.asarray(packed, dtype=np.uint8)
    N, K2 = packed.shape
    K = 2 * K2
    words = packed.reshape(N, K // 8, 4).astype(np.uint32)
    words = words[:, :, 0] | (words[:, :, 1] << 8) | (words[:, :, 2] << 16) | (words[:, :, 3] << 24)
    q = np.empty((N, K // 8, 8), np.float64)
    for p, kk in enumerate((0, 2, 4, 6, 1, 3, 5, 7)):
        q[:, :, kk] = ((words >> (4 * p)) & 0xF).astype(np.float64) - 8.0
    q = q.reshape(N, K)
    s = np.repeat(np.asarray(scales, dtype=np.float16).astype(np.float64), 32, axis=0)  # [K, N]
    return q.T * s


# --------------------------------------------------------------------------- combine

def combine(y_rows, pair_row, w, T: int, k: int, shared_rows=None, shared_base: int = 0):
    """Gate-weighted sum back to token order.

    mini-AGI PR #4, ``run()``: expert outputs are read back in pair order
    (``y[e_sorted, slot]``) and each token's k outputs are weighted by ``w`` and
    summed. A dropped pair (``pair_row = -1``) adds nothing; the remaining
    weights are not renormalised. With a shared expert its row
    ``shared_base + t`` is added with weight 1.
    """
    d = y_rows.shape[1]
    out = np.zeros((T, d), np.float64)
    pr = np.asarray(pair_row).reshape(T, k)
    w = np.asarray(w, dtype=np.float64).reshape(T, k)
    for j in range(k):
        r = pr[:, j]
        ok = r >= 0
        out[ok] += w[ok, j:j + 1] * y_rows[r[ok]]
    if shared_rows:
        out += y_rows[shared_base:shared_base + T]
    return out


# --------------------------------------------------------------------------- forward

def forward(x, logits, k: int, experts, limit: float, capacity_factor: float = 0.0,
            shared=None):
    """The whole layer: route → permute → per-expert FFN → combine, float64.

    x: [T, d] (any float dtype; widened exactly). logits: [T, E] float32.
    experts: callable e -> (W_gate [d,f], W_up [d,f], W_down [f,d]).
    shared: None or (W_gate, W_up, W_down) of the always-on shared expert.
    Returns (out [T, d] float64, dict of intermediates).
    """
    x = np.asarray(x, dtype=np.float64)
    T = x.shape[0]
    E = np.asarray(logits).shape[1]
    idx, w = route(logits, k)
    cap = capacity(T, k, E, capacity_factor)
    perm = permute(idx, E, cap, shared_T=T if shared is not None else 0)
    off, tok = perm["offsets"], perm["sorted_token"]
    y = np.zeros((int(off[-1]), x.shape[1]), np.float64)
    for e in range(E):
        a, b = int(off[e]), int(off[e + 1])
        if b > a:
            y[a:b] = expert_ffn(x[tok[a:b]], *experts(e), limit)
    if shared is not None:
        a, b = int(off[E]), int(off[E + 1])
        y[a:b] = expert_ffn(x[tok[a:b]], *shared, limit)
    out = combine(y, perm["pair_row"], w, T, k,
                  shared_rows=shared is not None, shared_base=int(off[E]))
    return out, {"idx": idx, "w": w, "cap": cap, "y": y, **perm}


def token_outputs(tokens, x, idx, w, pair_row, experts, limit: float, shared=None):
    """Outputs of selected tokens, each from its own definition.

    out[t] = sum over kept j of w[t, j] * FFN_{idx[t, j]}(x[t])  (+ shared(x[t])).
    Used to check full-size runs on sampled tokens without running the layer.
    """
    x = np.asarray(x)
    T, k = idx.shape
    pr = np.asarray(pair_row).reshape(T, k)
    res = []
    for t in tokens:
        xt = np.asarray(x[t:t + 1], dtype=np.float64)
        acc = np.zeros((1, x.shape[1]), np.float64)
        for j in range(k):
            if pr[t, j] >= 0:
                acc += float(w[t, j]) * expert_ffn(xt, *experts(int(idx[t, j])), limit)
        if shared is not None:
            acc += expert_ffn(xt, *shared, limit)
        res.append(acc[0])
    return np.stack(res) if res else np.zeros((0, x.shape[1]))


# --------------------------------------------------------------------------- backward

def swiglu_clamped_backward(g, u, dh, limit: float):
    """Gradients of h = silu(clamp(g)) * clamp(u) with respect to g and u, float64.

    d silu(z)/dz = s(z) * (1 + z * (1 - s(z))), s the logistic sigmoid. The
    clamp passes the gradient where -L <= v <= L and stops it outside (its
    derivative there is 0); ``limit <= 0`` means no clamp.
    """
    g = np.asarray(g, dtype=np.float64)
    u = np.asarray(u, dtype=np.float64)
    dh = np.asarray(dh, dtype=np.float64)
    if limit > 0:
        gc, uc = np.clip(g, -limit, limit), np.clip(u, -limit, limit)
        pass_g, pass_u = np.abs(g) <= limit, np.abs(u) <= limit
    else:
        gc, uc = g, u
        pass_g = pass_u = np.ones(g.shape, bool)
    sg = 1.0 / (1.0 + np.exp(-gc))
    dg = dh * uc * sg * (1.0 + gc * (1.0 - sg)) * pass_g
    du = dh * gc * sg * pass_u
    return dg, du


def expert_ffn_backward(x_rows, w_gate, w_up, w_down, limit: float, dy):
    """Backward of ``expert_ffn`` for the rows of one expert, float64.

    Given dy = dL/dy for y = swiglu(x Wg, x Wu) Wd: dh = dy Wd^T,
    dWd = h^T dy, (dg, du) from ``swiglu_clamped_backward``, dx = dg Wg^T +
    du Wu^T, dWg = x^T dg, dWu = x^T du. mini-AGI PR #3's tests/test_dispatch.py
    checks that these expert-weight gradients are the same on every dispatch
    path; this is their definition.

    Returns (dx [n, d], dWg [d, f], dWu [d, f], dWd [f, d], y [n, d]), y being
    the forward output (the routing-weight gradient needs it).
    """
    x_rows = np.asarray(x_rows, dtype=np.float64)
    wg, wu, wd = (np.asarray(w, dtype=np.float64) for w in (w_gate, w_up, w_down))
    dy = np.asarray(dy, dtype=np.float64)
    g, u = x_rows @ wg, x_rows @ wu
    h = swiglu_clamped(g, u, limit)
    dh = dy @ wd.T
    dg, du = swiglu_clamped_backward(g, u, dh, limit)
    return dg @ wg.T + du @ wu.T, x_rows.T @ dg, x_rows.T @ du, h.T @ dy, h @ wd


def route_backward(logits, k: int, d_w):
    """Gradient of the routing weights' softmax over the k selected logits.

    w_j = exp(l_j) / sum_i exp(l_i) over the selected; dl_j = w_j (dw_j -
    sum_i w_i dw_i) for the selected experts, 0 for the others (the top-k
    choice itself is piecewise constant). Returns dlogits [T, E] float64.
    """
    lg = np.asarray(logits, dtype=np.float32)
    T, E = lg.shape
    idx, w = route(lg, k)
    d_w = np.asarray(d_w, dtype=np.float64).reshape(T, k)
    dsel = w * (d_w - (w * d_w).sum(axis=1, keepdims=True))
    out = np.zeros((T, E), np.float64)
    np.put_along_axis(out, idx.astype(np.int64), dsel, axis=1)
    return out


def backward(x, logits, k: int, experts, limit: float, dout, capacity_factor: float = 0.0, shared=None):
    """Gradients of the layer for an upstream gradient dout = dL/dout, float64.

    out[t] = sum over kept j of w[t, j] * FFN_{idx[t, j]}(x[t]) (+ shared(x[t])).
    So a kept pair's expert sees dy = w[t, j] * dout[t]; dw[t, j] =
    <dout[t], FFN_{idx[t, j]}(x[t])> (0 for a dropped pair, whose weight is
    not renormalised away); dx[t] sums its pairs' input gradients (and the
    shared expert's, with dy = dout[t]); dlogits from ``route_backward``.

    Returns a dict: dx [T, d], dw_gate/dw_up [E, d, f], dw_down [E, f, d],
    d_topk_w [T, k], dlogits [T, E], and with a shared expert
    dshared = (dWg, dWu, dWd).
    """
    x = np.asarray(x, dtype=np.float64)
    dout = np.asarray(dout, dtype=np.float64)
    T, d = x.shape
    E = np.asarray(logits).shape[1]
    idx, w = route(logits, k)
    cap = capacity(T, k, E, capacity_factor)
    perm = permute(idx, E, cap)
    off, tok, sp = perm["offsets"], perm["sorted_token"], perm["sorted_pair"]
    f = np.asarray(experts(0)[0]).shape[1] if E else 0
    dx = np.zeros((T, d), np.float64)
    dwg, dwu, dwd = np.zeros((E, d, f)), np.zeros((E, d, f)), np.zeros((E, f, d))
    d_w = np.zeros(T * k, np.float64)
    wf = w.reshape(-1)
    for e in range(E):
        a, b = int(off[e]), int(off[e + 1])
        if b == a:
            continue
        rows, pairs = tok[a:b], sp[a:b]
        dy = wf[pairs][:, None] * dout[rows]
        dxr, dwg[e], dwu[e], dwd[e], y = expert_ffn_backward(x[rows], *experts(e), limit, dy)
        np.add.at(dx, rows, dxr)
        d_w[pairs] = (dout[rows] * y).sum(axis=1)
    res = {"dx": dx, "dw_gate": dwg, "dw_up": dwu, "dw_down": dwd, "d_topk_w": d_w.reshape(T, k),
           "dlogits": route_backward(logits, k, d_w), "idx": idx, "w": w, **perm}
    if shared is not None:
        dxs, sg, su, sd, _ = expert_ffn_backward(x, *shared, limit, dout)
        res["dx"] = dx + dxs
        res["dshared"] = (sg, su, sd)
    return res
