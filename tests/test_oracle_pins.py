"""Pins for the fp64 oracle: closed forms, brute force, invariants, golden cases.

Each check ties the oracle to something other than its own code: hand-worked
golden fixtures (tests/golden/, each citing its source), brute force over all
k-subsets, pure-Python loop versions of the definitions, closed forms and
symmetry properties. A plausible mistake (dropped term, wrong sign, transposed
operand, wrong tie-break, renormalising after a drop) fails at least one.
"""
import itertools
import math
import os

import numpy as np
import pytest

import oracle
import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _lines(name):
    with open(os.path.join(GOLD, name)) as fh:
        return [ln.strip() for ln in fh if ln.strip() and not ln.startswith("#")]


# --------------------------------------------------------------------------- route

def test_route_golden_cases():
    for ln in _lines("route_cases.txt"):
        k, lg, ix, w = [p.split() for p in ln.split("|")]
        k = int(k[0])
        logits = np.array([[float(v) for v in lg]], np.float32)
        idx, ww = oracle.route(logits, k)
        assert idx[0].tolist() == [int(v) for v in ix], ln
        np.testing.assert_allclose(ww[0], [float(v) for v in w], rtol=0, atol=1e-12)


def test_route_brute_force_topk():
    """Over all k-subsets, the top-k set is the one with the largest logit sum."""
    rng = np.random.default_rng(11)
    for E in (2, 3, 5, 8):
        for k in range(1, E + 1):
            lg = rng.standard_normal((20, E)).astype(np.float32)
            idx, w = oracle.route(lg, k)
            for t in range(lg.shape[0]):
                best = max(itertools.combinations(range(E), k),
                           key=lambda s: sum(float(lg[t, e]) for e in s))
                want = sorted(best, key=lambda e: -float(lg[t, e]))
                assert idx[t].tolist() == want
                # softmax over the selected, by its definition with Python floats
                ex = [math.exp(float(lg[t, e]) - float(lg[t, want[0]])) for e in want]
                np.testing.assert_allclose(w[t], [v / sum(ex) for v in ex], rtol=1e-13)


def test_route_equals_renormalised_full_softmax():
    """The pages' procedure: full softmax, take top-k, divide by their sum."""
    from scipy.special import softmax
    lg = np.random.default_rng(5).standard_normal((50, 16)).astype(np.float32) * 3
    idx, w = oracle.route(lg, 4)
    probs = softmax(lg.astype(np.float64), axis=1)
    sel = np.take_along_axis(probs, idx.astype(np.int64), axis=1)
    np.testing.assert_allclose(w, sel / sel.sum(1, keepdims=True), rtol=1e-12)
    # shift invariance of the weights, and they sum to one
    idx2, w2 = oracle.route(lg + np.float32(0.0), 4)
    np.testing.assert_allclose(w.sum(1), 1.0, rtol=1e-14)
    assert (idx2 == idx).all()


def test_route_k1_and_k2_closed_forms():
    lg = np.random.default_rng(3).standard_normal((30, 6)).astype(np.float32)
    _, w1 = oracle.route(lg, 1)
    assert (w1 == 1.0).all()
    idx, w2 = oracle.route(lg, 2)
    a = lg[np.arange(30), idx[:, 0]].astype(np.float64)
    b = lg[np.arange(30), idx[:, 1]].astype(np.float64)
    np.testing.assert_allclose(w2[:, 0], 1.0 / (1.0 + np.exp(b - a)), rtol=1e-14)
    assert (a >= b).all()


# --------------------------------------------------------------------------- router telemetry

def test_router_telemetry_golden_cases():
    for ln in _lines("router_telemetry_cases.txt"):
        k, lg, kept, want, lse, bal = [p.split() for p in ln.split("|")]
        logits = np.array([[float(v) for v in lg]], np.float32)
        r = oracle.router_telemetry(logits, int(k[0]), z_weight=0.0)
        np.testing.assert_allclose(r["kept"], float(kept[0]), rtol=0, atol=1e-12)
        assert r["want_k"] == float(want[0]) and int(r["want_tok"][0]) == int(want[0]), ln
        np.testing.assert_allclose(r["lse"][0], float(lse[0]), rtol=1e-14)
        np.testing.assert_allclose(r["z"], float(lse[0]) ** 2, rtol=1e-13)
        np.testing.assert_allclose(r["balance"], float(bal[0]), rtol=1e-12)
        np.testing.assert_allclose(r["aux"], r["balance"], rtol=0, atol=0)


def test_router_telemetry_want_by_brute_force():
    """want = the size of the smallest set of experts of mass >= 0.9, over every subset."""
    rng = np.random.default_rng(21)
    for E in (2, 3, 5, 7):
        lg = (rng.standard_normal((25, E)) * 2.5).astype(np.float32)
        r = oracle.router_telemetry(lg, 1)
        for t in range(lg.shape[0]):
            ex = [math.exp(float(v)) for v in lg[t]]
            p = [v / sum(ex) for v in ex]
            best = min(len(s) for m in range(1, E + 1) for s in itertools.combinations(range(E), m)
                       if sum(p[e] for e in s) >= 0.9)
            assert int(r["want_tok"][t]) == best
            np.testing.assert_allclose(r["kept_tok"][t], max(p), rtol=1e-13)


def test_router_telemetry_loop_definitions():
    """Every output from Python-float loops over the definitions (first choice, mean probability,
    logsumexp), against the oracle's array code; kept == 1 when k == E."""
    rng = np.random.default_rng(8)
    T, E, k, zw = 40, 6, 2, 0.01
    lg = (rng.standard_normal((T, E)) * 2).astype(np.float32)
    r = oracle.router_telemetry(lg, k, z_weight=zw)
    probs, lses, firsts, kept = [], [], [], []
    for t in range(T):
        vals = [float(v) for v in lg[t]]
        s = sum(math.exp(v) for v in vals)
        p = [math.exp(v) / s for v in vals]
        probs.append(p)
        lses.append(math.log(s))
        top = sorted(range(E), key=lambda e: (-vals[e], e))
        firsts.append(top[0])
        kept.append(sum(p[e] for e in top[:k]))
    frac = [firsts.count(e) / T for e in range(E)]
    pm = [sum(probs[t][e] for t in range(T)) / T for e in range(E)]
    bal = E * sum(frac[e] * pm[e] for e in range(E))
    z = sum(v * v for v in lses) / T
    np.testing.assert_allclose(r["frac"], frac, rtol=0, atol=0)
    np.testing.assert_allclose(r["prob_mean"], pm, rtol=1e-12)
    np.testing.assert_allclose(r["kept"], sum(kept) / T, rtol=1e-12)
    np.testing.assert_allclose(r["balance"], bal, rtol=1e-12)
    np.testing.assert_allclose(r["z"], z, rtol=1e-12)
    np.testing.assert_allclose(r["aux"], bal + zw * z, rtol=1e-12)
    np.testing.assert_allclose(oracle.router_telemetry(lg, E)["kept"], 1.0, rtol=1e-14)


def test_router_telemetry_balance_extremes():
    """balance = E when every token sends all its mass to one expert; about 1 when each expert
    is the sole first choice of an equal share of tokens (the loss's minimum)."""
    E = 16
    lg = np.zeros((64, E), np.float32)
    lg[:, 5] = 60.0
    r = oracle.router_telemetry(lg, 2)
    np.testing.assert_allclose(r["balance"], E, rtol=1e-12)
    assert r["want_k"] == 1.0
    lg2 = np.zeros((4 * E, E), np.float32)
    lg2[np.arange(4 * E), np.arange(4 * E) % E] = 60.0
    np.testing.assert_allclose(oracle.router_telemetry(lg2, 2)["balance"], 1.0, rtol=1e-12)


# --------------------------------------------------------------------------- capacity

def test_capacity_golden():
    for ln in _lines("capacity_cases.txt"):
        T, k, E, cf, want = ln.split()
        got = oracle.capacity(int(T), int(k), int(E), float(cf))
        assert got == (None if want == "none" else int(want)), ln


# --------------------------------------------------------------------------- permute

def _permute_loop(idx, E, cap):
    """Plain per-expert loop: walk the tokens in order, each expert takes rows until full."""
    T, k = idx.shape
    rows = {e: [] for e in range(E)}
    counts = [0] * E
    for t in range(T):
        for j in range(k):
            e = int(idx[t, j])
            counts[e] += 1
            if cap is None or len(rows[e]) < cap:
                rows[e].append((t, t * k + j))
    pair_row = [-1] * (T * k)
    sorted_token, offsets = [], [0]
    for e in range(E):
        for (t, p) in rows[e]:
            pair_row[p] = len(sorted_token)
            sorted_token.append(t)
        offsets.append(len(sorted_token))
    return counts, offsets, sorted_token, pair_row


def test_permute_golden_drop_order():
    g = {}
    for ln in _lines("drop_order.txt"):
        key, *vals = ln.split()
        g[key] = [int(v) for v in vals]
    idx = np.array(g["idx"], np.int32)[:, None]
    p = oracle.permute(idx, g["E"][0], g["cap"][0])
    for key in ("counts", "kept", "offsets", "sorted_token", "pair_row"):
        assert p[key].tolist() == g[key], key


@pytest.mark.parametrize("cap", [None, 1, 3, 7])
def test_permute_matches_loop(cap):
    rng = np.random.default_rng(7)
    for E, k, T in ((4, 2, 9), (8, 3, 40), (5, 5, 12), (16, 1, 50)):
        lg = rng.standard_normal((T, E)).astype(np.float32)
        idx, _ = oracle.route(lg, k)
        p = oracle.permute(idx, E, cap)
        counts, offsets, st, pr = _permute_loop(idx, E, cap)
        assert p["counts"].tolist() == counts
        assert p["offsets"].tolist() == offsets
        assert p["sorted_token"].tolist() == st
        assert p["pair_row"].tolist() == pr


def test_permute_invariants_capped_workload():
    cfg = synth.CONFIGS["capped"]
    idx, _ = oracle.route(synth.logits(cfg), cfg.k)
    cap = oracle.capacity(cfg.T, cfg.k, cfg.E, cfg.capacity_factor)
    assert cap == 192
    p = oracle.permute(idx, cfg.E, cap)
    assert p["counts"].sum() == cfg.T * cfg.k
    assert (p["kept"] <= cap).all()
    P = int(p["offsets"][-1])
    assert p["kept"].sum() == P and (np.diff(p["offsets"]) >= 0).all()
    dropped = cfg.T * cfg.k - P
    assert dropped > 0.5 * cfg.T * cfg.k  # the +4 bias crowds 8 experts: most pairs drop
    # every kept pair once, pair_row the inverse of sorted_pair
    sp = p["sorted_pair"]
    assert len(set(sp.tolist())) == P
    assert (p["pair_row"][sp] == np.arange(P)).all()
    assert ((p["pair_row"] >= 0).sum()) == P
    # tokens ascend inside each expert
    st = p["sorted_token"]
    for e in range(cfg.E):
        seg = st[p["offsets"][e]:p["offsets"][e + 1]]
        assert (np.diff(seg) > 0).all()


def test_permute_shared_expert_rows():
    idx = np.array([[0, 1], [1, 2], [0, 2]], np.int32)
    p = oracle.permute(idx, 3, None, shared_T=3)
    assert p["offsets"].tolist() == [0, 2, 4, 6, 9]
    assert p["sorted_token"][6:].tolist() == [0, 1, 2]
    assert p["sorted_pair"][6:].tolist() == [-1, -1, -1]
    assert p["kept"].tolist() == [2, 2, 2, 3]


# --------------------------------------------------------------------------- FFN

def test_swiglu_golden_points():
    for ln in _lines("swiglu_points.txt"):
        g, u, L, want = (float(v) for v in ln.split())
        got = float(oracle.swiglu_clamped(np.array([g]), np.array([u]), L)[0])
        assert got == pytest.approx(want, rel=1e-14, abs=1e-15), ln


def _ffn_loops(x, wg, wu, wd, L):
    """SwiGLU FFN with explicit Python loops (no matrix library)."""
    d, f = len(wg), len(wg[0])
    out = []
    for row in x:
        h = []
        for n in range(f):
            g = sum(row[i] * wg[i][n] for i in range(d))
            u = sum(row[i] * wu[i][n] for i in range(d))
            if L > 0:
                g, u = min(max(g, -L), L), min(max(u, -L), L)
            h.append(g / (1.0 + math.exp(-g)) * u)
        out.append([sum(h[n] * wd[n][i] for n in range(f)) for i in range(d)])
    return np.array(out)


@pytest.mark.parametrize("scale,L,d,f", [(1.0, 7.0, 5, 7), (20.0, 7.0, 5, 7), (20.0, 0.0, 5, 7),
                                         (1.0, 7.0, 6, 6)])
def test_expert_ffn_matches_loops(scale, L, d, f):
    rng = np.random.default_rng(2)
    # non-square and square shapes: a transposed operand fails either way
    x = rng.standard_normal((4, d))
    wg, wu = rng.standard_normal((d, f)) * scale, rng.standard_normal((d, f)) * scale
    wd = rng.standard_normal((f, d))
    got = oracle.expert_ffn(x, wg, wu, wd, L)
    want = _ffn_loops(x.tolist(), wg.tolist(), wu.tolist(), wd.tolist(), L)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)
    if scale == 20.0 and L > 0:
        unclamped = _ffn_loops(x.tolist(), wg.tolist(), wu.tolist(), wd.tolist(), 0.0)
        assert np.abs(unclamped - want).max() > 1.0  # the clamp fires in this case


def test_e1_top1_is_dense_ffn():
    """E=1, k=1: routing weight 1, every token kept → the layer is one dense FFN."""
    cfg = synth.LayerConfig("e1", T=12, d=16, f=24, E=1, k=1)
    x = synth.bf16_bits_to_f32(synth.x_bits(cfg)).astype(np.float64)
    W = [synth.bf16_bits_to_f32(synth.expert_weight_bits(cfg, 0, w)) for w in ("gate", "up", "down")]
    out, inter = oracle.forward(x, synth.logits(cfg), 1, lambda e: W, 7.0)
    assert (inter["w"] == 1.0).all()
    dense = _ffn_loops(x.tolist(), *(w.astype(np.float64).tolist() for w in W), 7.0)
    np.testing.assert_allclose(out, dense, rtol=1e-12, atol=1e-14)


# --------------------------------------------------------------------------- whole layer

def _layer_loops(x, lg, k, Ws, L, cap, shared=None):
    """The layer straight from its definition: per token, sum of weighted expert
    outputs, with the capacity drop decided by a running per-expert count."""
    T, E = lg.shape
    taken = [0] * E
    out = np.zeros_like(x)
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-float(lg[t, e]), e))[:k]
        ex = [math.exp(float(lg[t, e]) - float(lg[t, order[0]])) for e in order]
        for e, v in zip(order, ex):
            taken[e] += 1
            if cap is not None and taken[e] > cap:
                continue  # dropped: contributes nothing, the others are not renormalised
            y = _ffn_loops([x[t].tolist()], *(w.tolist() for w in Ws[e]), L)[0]
            out[t] += v / sum(ex) * y
        if shared is not None:
            out[t] += _ffn_loops([x[t].tolist()], *(w.tolist() for w in shared), L)[0]
    return out


@pytest.mark.parametrize("cf,shared", [(0.0, False), (1.0, False), (0.5, True)])
def test_forward_matches_per_token_loops(cf, shared):
    rng = np.random.default_rng(9)
    T, d, f, E, k = 9, 4, 6, 3, 2
    x = rng.standard_normal((T, d))
    lg = rng.standard_normal((T, E)).astype(np.float32)
    Ws = [tuple(rng.standard_normal(s) * 0.7 for s in ((d, f), (d, f), (f, d))) for _ in range(E)]
    sh = tuple(rng.standard_normal(s) * 0.7 for s in ((d, f), (d, f), (f, d))) if shared else None
    out, inter = oracle.forward(x, lg, k, lambda e: Ws[e], 7.0, cf, shared=sh)
    cap = oracle.capacity(T, k, E, cf)
    want = _layer_loops(x, lg, k, Ws, 7.0, cap, sh)
    np.testing.assert_allclose(out, want, rtol=1e-12, atol=1e-12)
    if cf > 0:
        assert (inter["pair_row"] < 0).any()


def test_token_permutation_equivariance():
    cfg = synth.CONFIGS["tiny"]
    x = synth.bf16_bits_to_f32(synth.x_bits(cfg)).astype(np.float64)
    lg = synth.logits(cfg)
    Ws = {e: [synth.bf16_bits_to_f32(synth.expert_weight_bits(cfg, e, w)) for w in ("gate", "up", "down")]
          for e in range(cfg.E)}
    out, _ = oracle.forward(x, lg, cfg.k, Ws.__getitem__, 7.0)
    perm = np.random.default_rng(4).permutation(cfg.T)
    out_p, _ = oracle.forward(x[perm], lg[perm], cfg.k, Ws.__getitem__, 7.0)
    np.testing.assert_allclose(out_p, out[perm], rtol=1e-12, atol=1e-15)
    # linear in W_down
    Ws2 = {e: [w[0], w[1], 2 * w[2]] for e, w in Ws.items()}
    out2, _ = oracle.forward(x, lg, cfg.k, Ws2.__getitem__, 7.0)
    np.testing.assert_allclose(out2, 2 * out, rtol=1e-12, atol=1e-15)


def test_all_dropped_token_is_zero_or_shared():
    # every token picks expert 0 (bias), cap 1: only token 0 is served
    T, E, k, d, f = 4, 2, 1, 3, 5
    rng = np.random.default_rng(1)
    lg = np.array([[5.0, 0.0]] * T, np.float32)
    x = rng.standard_normal((T, d))
    W = tuple(rng.standard_normal(s) for s in ((d, f), (d, f), (f, d)))
    out, inter = oracle.forward(x, lg, k, lambda e: W, 7.0, capacity_factor=0.5)
    assert inter["cap"] == 1
    assert np.abs(out[1:]).max() == 0.0 and np.abs(out[0]).max() > 0
    out_s, _ = oracle.forward(x, lg, k, lambda e: W, 7.0, capacity_factor=0.5, shared=W)
    np.testing.assert_allclose(out_s[1:], oracle.expert_ffn(x[1:], *W, 7.0), rtol=1e-13)


def test_token_outputs_match_forward():
    cfg = synth.CONFIGS["tiny"].replace(capacity_factor=1.0)
    x = synth.bf16_bits_to_f32(synth.x_bits(cfg)).astype(np.float64)
    lg = synth.logits(cfg)
    Ws = {e: [synth.bf16_bits_to_f32(synth.expert_weight_bits(cfg, e, w)) for w in ("gate", "up", "down")]
          for e in range(cfg.E)}
    out, it = oracle.forward(x, lg, cfg.k, Ws.__getitem__, 7.0, cfg.capacity_factor)
    toks = [0, 5, 17, 63]
    got = oracle.token_outputs(toks, x, it["idx"], it["w"], it["pair_row"], Ws.__getitem__, 7.0)
    np.testing.assert_allclose(got, out[toks], rtol=1e-12, atol=1e-15)


# --------------------------------------------------------------------------- Q4G32

def test_q4g32_golden_bytes():
    packed = np.full((2, 32), 0x88, np.uint8)  # N=2 rows, K=64
    packed[0, 0], packed[0, 2], packed[0, 6], packed[0, 16], packed[1, 0] = 0x9F, 0x18, 0x8C, 0xB7, 0x2E
    scales = np.array([[0.5, 0.25], [2.0, 1.0]], np.float16)  # [K/32, N]
    w = oracle.dequant_q4g32(packed, scales)  # [K=64, N=2]
    want = np.zeros((64, 2))
    for ln in _lines("q4g32_bytes.txt"):
        n, k, v = ln.split()
        want[int(k), int(n)] = float(v)
    assert (w == want).all()


def test_q4g32_round_trip_and_error_bound():
    rng = np.random.default_rng(0)
    # exactly representable: every group holds +-7 so the scale is exactly 0.25
    q = rng.integers(-7, 8, size=(64, 6))
    q[0::32, :] = 7
    w = q * 0.25
    packed, s = synth.quantize_q4g32(w.astype(np.float32))
    assert s.shape == (2, 6) and (s == np.float16(0.25)).all()
    assert (oracle.dequant_q4g32(packed, s) == w).all()
    # general case: error at most half a step (plus the fp16 rounding of the scale)
    w = rng.standard_normal((128, 40)).astype(np.float32) * 0.02
    packed, s = synth.quantize_q4g32(w)
    err = np.abs(oracle.dequant_q4g32(packed, s) - w)
    step = np.repeat(s.astype(np.float64), 32, axis=0)
    assert (err <= step * (0.5 + 7 * 2.0 ** -10) + 1e-12).all()


# --------------------------------------------------------------------------- backward

def _tiny_layer(seed, T=7, d=8, f=6, E=4, k=2, wscale=0.5):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, d))
    lg = (rng.standard_normal((T, E)) * 2).astype(np.float32)
    Ws = [tuple(rng.standard_normal(s) * wscale for s in ((d, f), (d, f), (f, d))) for _ in range(E)]
    dout = rng.standard_normal((T, d))
    return x, lg, Ws, dout


def _loss(x, lg, Ws, dout, k, limit, cf=0.0, shared=None):
    out, _ = oracle.forward(x, lg, k, lambda e: Ws[e], limit, cf, shared=shared)
    return float((out * dout).sum())


@pytest.mark.parametrize("limit,cf,shared", [(7.0, 0.0, False), (1.5, 0.0, False), (7.0, 0.6, False),
                                             (1.5, 0.0, True)])
def test_backward_against_central_differences(limit, cf, shared):
    """Every gradient of L = <dout, out> against central differences of the forward oracle
    (fp64, step 1e-6), with the clamp firing (limit 1.5), a capacity drop and a shared expert."""
    x, lg, Ws, dout = _tiny_layer(4)
    k, E = 2, len(Ws)
    sh = tuple(np.random.default_rng(9).standard_normal(s) * 0.5 for s in ((8, 6), (8, 6), (6, 8))) \
        if shared else None
    g = oracle.backward(x, lg, k, lambda e: Ws[e], limit, dout, cf, shared=sh)
    eps = 1e-6

    def fd(mut):
        plus, minus = mut(eps), mut(-eps)
        return (plus - minus) / (2 * eps)

    for t, c in [(0, 0), (3, 5), (6, 7)]:
        def mx(h, t=t, c=c):
            xx = x.copy()
            xx[t, c] += h
            return _loss(xx, lg, Ws, dout, k, limit, cf, sh)
        np.testing.assert_allclose(g["dx"][t, c], fd(mx), rtol=1e-6, atol=1e-8)
    for e in range(E):
        for wi, key, (i, j) in ((0, "dw_gate", (1, 2)), (1, "dw_up", (7, 0)), (2, "dw_down", (5, 3))):
            def mw(h, e=e, wi=wi, i=i, j=j):
                W2 = [list(w) for w in Ws]
                W2[e][wi] = W2[e][wi].copy()
                W2[e][wi][i, j] += h
                return _loss(x, lg, [tuple(w) for w in W2], dout, k, limit, cf, sh)
            np.testing.assert_allclose(g[key][e, i, j], fd(mw), rtol=1e-6, atol=1e-8)
    for t in range(0, 7, 2):
        for ee in range(E):
            def ml(h, t=t, ee=ee):
                l2 = lg.astype(np.float64).copy()
                l2[t, ee] += h
                # the router reads float32 logits: perturb in float64 through the weights only
                return _loss_logits64(x, l2, Ws, dout, k, limit, cf, sh)
            np.testing.assert_allclose(g["dlogits"][t, ee], fd(ml), rtol=1e-5, atol=1e-7)
    if sh is not None:
        def msh(h):
            s2 = (sh[0].copy(), sh[1], sh[2])
            s2[0][2, 3] += h
            return _loss(x, lg, Ws, dout, k, limit, cf, s2)
        np.testing.assert_allclose(g["dshared"][0][2, 3], fd(msh), rtol=1e-6, atol=1e-8)


def _loss_logits64(x, lg64, Ws, dout, k, limit, cf, sh):
    """The layer with the routing weights taken from float64 logits (same top-k choice): the
    softmax over the selected, as the forward defines it, without the float32 input rounding."""
    lg32 = lg64.astype(np.float32)
    idx, _ = oracle.route(lg32, k)
    sel = np.take_along_axis(lg64, idx.astype(np.int64), axis=1)
    w = np.exp(sel - sel[:, :1])
    w /= w.sum(1, keepdims=True)
    T, E = lg64.shape
    cap = oracle.capacity(T, k, E, cf)
    perm = oracle.permute(idx, E, cap)
    y = np.zeros((int(perm["offsets"][-1]), x.shape[1]))
    for e in range(E):
        a, b = int(perm["offsets"][e]), int(perm["offsets"][e + 1])
        if b > a:
            y[a:b] = oracle.expert_ffn(x[perm["sorted_token"][a:b]], *Ws[e], limit)
    out = oracle.combine(y, perm["pair_row"], w, T, k)
    if sh is not None:
        out = out + oracle.expert_ffn(x, *sh, limit)
    return float((out * dout).sum())


def test_backward_dense_case_against_autograd():
    """E = 1, k = 1: the layer is a dense clamped-SwiGLU FFN; torch autograd (float64) of that
    FFN written out separately gives the same dx and weight gradients."""
    import torch
    rng = np.random.default_rng(2)
    T, d, f, L = 9, 12, 10, 2.0
    x = rng.standard_normal((T, d))
    W = tuple(rng.standard_normal(s) for s in ((d, f), (d, f), (f, d)))
    dout = rng.standard_normal((T, d))
    g = oracle.backward(x, np.zeros((T, 1), np.float32), 1, lambda e: W, L, dout)
    xt = torch.tensor(x, requires_grad=True)
    Wt = [torch.tensor(w, requires_grad=True) for w in W]
    gg = torch.clamp(xt @ Wt[0], -L, L)
    uu = torch.clamp(xt @ Wt[1], -L, L)
    out = (torch.nn.functional.silu(gg) * uu) @ Wt[2]
    (out * torch.tensor(dout)).sum().backward()
    np.testing.assert_allclose(g["dx"], xt.grad.numpy(), rtol=1e-12, atol=1e-12)
    for key, t in zip(("dw_gate", "dw_up", "dw_down"), Wt):
        np.testing.assert_allclose(g[key][0], t.grad.numpy(), rtol=1e-12, atol=1e-12)
    assert np.abs(g["dlogits"]).max() == 0.0  # one expert, weight 1: no routing gradient


def test_route_backward_closed_form_k2():
    """k = 2: w0 = sigmoid(l0 - l1), so dl0 = w0 w1 (dw0 - dw1) = -dl1."""
    lg = np.array([[0.3, 2.0, -1.0, 1.1]], np.float32)
    dw = np.array([[0.7, -0.4]])
    dl = oracle.route_backward(lg, 2, dw)
    a, c = 2.0, float(np.float32(1.1))
    w0 = 1.0 / (1.0 + math.exp(c - a))
    np.testing.assert_allclose(dl[0, 1], w0 * (1 - w0) * (0.7 + 0.4), rtol=1e-12)
    np.testing.assert_allclose(dl[0, 3], -dl[0, 1], rtol=1e-12)
    assert dl[0, 0] == 0.0 and dl[0, 2] == 0.0
