"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each pin takes an ``oracle.Oracle`` and raises AssertionError when the oracle
disagrees with:
  * a hand-worked closed-form example (tests/golden/handworked_micro.json),
  * library special cases (tau=0 is the unmasked dense MoE layer, computed
    here with torch fp64 softmax/topk/silu/matmul; tau=+inf leaves only the
    shared expert),
  * brute-force per-neuron enumeration on tiny inputs,
  * invariants of the definition (nested masks, exact decomposition of the
    output difference between two thresholds, the calibrated keep fraction),
  * a stable-sort ranking of the router probabilities with deliberate ties.

The same pins run against deliberately broken copies of the oracle in
test_oracle_mutants.py, which shows each plausible mistake fails one of them.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch
import torch.nn.functional as F

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _bf16(a):
    return torch.as_tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)


def _bits(t):
    return None if t is None else t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _rand_layer(seed, d, E, f, k, S, T, scale_x=1.0):
    g = torch.Generator().manual_seed(seed)

    def rn(*shape, std):
        return (torch.randn(*shape, generator=g) * std).to(torch.bfloat16)

    W = dict(w_router=rn(E, d, std=d ** -0.5), w_gate=rn(E, d, f, std=d ** -0.5),
             w_up=rn(E, d, f, std=d ** -0.5), w_down=rn(E, f, d, std=f ** -0.5))
    if S:
        W.update(ws_gate=rn(S, d, f, std=d ** -0.5), ws_up=rn(S, d, f, std=d ** -0.5),
                 ws_down=rn(S, f, d, std=f ** -0.5))
    else:
        W.update(ws_gate=None, ws_up=None, ws_down=None)
    x = rn(T, d, std=scale_x)
    return x, W


def _call(o, x, W, k, tau, active=None, tau_shared=0.0):
    args = {n: _bits(t) for n, t in W.items()}
    return o.forward(_bits(x), **args, top_k=k, tau=tau, active=active, tau_shared=tau_shared)


def _torch_dense(x, W, k, with_routed=True, with_shared=True):
    """The unmasked dense MoE layer from torch fp64 library calls."""
    xd = x.double()
    logits = xd @ W["w_router"].double().T
    p = torch.softmax(logits, dim=-1)
    # stable descending sort = top-k with ties to the lower index
    order = np.argsort(-p.numpy(), axis=1, kind="stable")[:, :k]
    idx = torch.as_tensor(order)
    y = torch.zeros_like(xd)
    if with_routed:
        for t in range(x.shape[0]):
            for r in range(k):
                e = int(idx[t, r])
                g = xd[t] @ W["w_gate"][e].double()
                u = xd[t] @ W["w_up"][e].double()
                y[t] += p[t, e] * ((F.silu(g) * u) @ W["w_down"][e].double())
    if with_shared and W["ws_gate"] is not None:
        for s in range(W["ws_gate"].shape[0]):
            g = xd @ W["ws_gate"][s].double()
            u = xd @ W["ws_up"][s].double()
            y += (F.silu(g) * u) @ W["ws_down"][s].double()
    return y.numpy(), idx.numpy(), p.numpy(), logits.numpy()


def _rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


# ---------------------------------------------------------------- pins

def pin_handworked(o):
    """Closed-form micro layer worked by hand (golden fixture)."""
    with open(os.path.join(GOLDEN, "handworked_micro.json")) as fh:
        G = json.load(fh)

    def sig(z):
        return 1.0 / (1.0 + math.exp(-z))

    def ev(s):
        return float(eval(s, {"__builtins__": {}}, {"sig": sig, "inf": math.inf}))

    x = _bf16(G["x"])
    W = {n: _bf16(G[n]) for n in ("w_router", "w_gate", "w_up", "w_down",
                                    "ws_gate", "ws_up", "ws_down")}
    for case in G["cases"]:
        tau = ev(case["tau"])
        r = _call(o, x, W, G["top_k"], tau)
        assert np.array_equal(r.topk_idx, np.array(G["topk_idx"])), ("idx", r.topk_idx)
        want_w = np.array([[ev(v) for v in row] for row in G["topk_w"]])
        assert np.allclose(r.topk_w, want_w, rtol=1e-14, atol=0), ("w", r.topk_w, want_w)
        assert np.array_equal(r.active, np.array(case["active"], dtype=np.uint8)), \
            ("active", case["tau"], r.active)
        want_y = np.array([[ev(v) for v in row] for row in case["y"]])
        assert np.allclose(r.y, want_y, rtol=1e-13, atol=1e-14), ("y", case["tau"], r.y, want_y)


def pin_tau0_is_dense(o):
    """tau = 0 keeps every neuron: the layer is the unmasked dense MoE (torch fp64)."""
    for seed, S in ((11, 1), (12, 0), (13, 2)):
        x, W = _rand_layer(seed, d=64, E=6, f=48, k=3, S=S, T=5)
        r = _call(o, x, W, 3, 0.0)
        y, idx, p, logits = _torch_dense(x, W, 3)
        assert np.array_equal(r.topk_idx, idx), ("idx", r.topk_idx, idx)
        assert _rel(r.y, y) < 1e-12, ("y", _rel(r.y, y))
        assert r.active.all()


def pin_tauinf_is_shared_only(o):
    """tau = +inf keeps no routed neuron: only the shared experts remain (0 without one)."""
    for seed, S in ((21, 1), (22, 2), (23, 0)):
        x, W = _rand_layer(seed, d=64, E=6, f=48, k=2, S=S, T=4)
        r = _call(o, x, W, 2, math.inf)
        y, *_ = _torch_dense(x, W, 2, with_routed=False)
        if S == 0:
            assert not r.y.any()
        else:
            assert _rel(r.y, y) < 1e-12, ("y", _rel(r.y, y))
        assert not r.active.any()


def pin_bruteforce(o):
    """Per-neuron enumeration with scalar Python arithmetic on a tiny layer."""
    d, E, f, k, S, T = 16, 4, 8, 2, 1, 3
    x, W = _rand_layer(31, d, E, f, k, S, T, scale_x=1.0)
    X = x.float().double().tolist()
    Wr = W["w_router"].double().tolist()
    Wg = W["w_gate"].double().tolist()
    Wu = W["w_up"].double().tolist()
    Wd = W["w_down"].double().tolist()
    Sg, Su, Sd = (W["ws_gate"].double().tolist(), W["ws_up"].double().tolist(),
                  W["ws_down"].double().tolist())

    def silu(z):
        return z / (1.0 + math.exp(-z))

    # every selected neuron's score, then a threshold that splits them
    scores, plan = [], []
    for t in range(T):
        lg = [sum(X[t][i] * Wr[e][i] for i in range(d)) for e in range(E)]
        m = max(lg)
        ex = [math.exp(v - m) for v in lg]
        p = [v / sum(ex) for v in ex]
        chosen = sorted(range(E), key=lambda e: (-p[e], e))[:k]
        for e in chosen:
            for j in range(f):
                g = sum(X[t][i] * Wg[e][i][j] for i in range(d))
                u = sum(X[t][i] * Wu[e][i][j] for i in range(d))
                scores.append(abs(silu(g)))
                plan.append((t, e, j, p[e], silu(g) * u))
    tau = float(np.float32(sorted(scores)[len(scores) // 2] * 1.0001))
    y = [[0.0] * d for _ in range(T)]
    act = {}
    for (t, e, j, pe, h), s in zip(plan, scores):
        on = np.float32(s) >= np.float32(tau)
        act[(t, e, j)] = on
        if on:
            for i in range(d):
                y[t][i] += pe * h * Wd[e][j][i]
    for t in range(T):
        for s_ in range(S):
            for j in range(f):
                g = sum(X[t][i] * Sg[s_][i][j] for i in range(d))
                u = sum(X[t][i] * Su[s_][i][j] for i in range(d))
                for i in range(d):
                    y[t][i] += silu(g) * u * Sd[s_][j][i]
    r = _call(o, x, W, k, tau)
    for t in range(T):
        for r_ in range(k):
            e = int(r.topk_idx[t, r_])
            for j in range(f):
                assert bool(r.active[t, r_, j]) == bool(act[(t, e, j)]), ("active", t, e, j)
    assert _rel(r.y, np.array(y)) < 1e-12, ("y", _rel(r.y, np.array(y)))


def pin_mask_override(o):
    """A given mask replaces the threshold: scalar-Python enumeration under an
    arbitrary seeded mask (unrelated to any threshold), on a tiny layer."""
    d, E, f, k, S, T = 16, 4, 8, 2, 1, 3
    x, W = _rand_layer(33, d, E, f, k, S, T, scale_x=1.0)
    X = x.float().double().tolist()
    Wr = W["w_router"].double().tolist()
    Wg, Wu, Wd = (W["w_gate"].double().tolist(), W["w_up"].double().tolist(),
                  W["w_down"].double().tolist())
    Sg, Su, Sd = (W["ws_gate"].double().tolist(), W["ws_up"].double().tolist(),
                  W["ws_down"].double().tolist())

    def silu(z):
        return z / (1.0 + math.exp(-z))

    mask = (np.random.default_rng(34).random((T, k, f)) < 0.5).astype(np.uint8)
    mask[0, 0, :] = 1          # one pair fully on, one fully off
    mask[1, 1, :] = 0
    y = [[0.0] * d for _ in range(T)]
    want_score = np.zeros((T, k, f))
    for t in range(T):
        lg = [sum(X[t][i] * Wr[e][i] for i in range(d)) for e in range(E)]
        m = max(lg)
        ex = [math.exp(v - m) for v in lg]
        p = [v / sum(ex) for v in ex]
        chosen = sorted(range(E), key=lambda e: (-p[e], e))[:k]
        for r_, e in enumerate(chosen):
            for j in range(f):
                g = sum(X[t][i] * Wg[e][i][j] for i in range(d))
                u = sum(X[t][i] * Wu[e][i][j] for i in range(d))
                want_score[t, r_, j] = abs(silu(g))
                if mask[t, r_, j]:
                    for i in range(d):
                        y[t][i] += p[e] * silu(g) * u * Wd[e][j][i]
        for s_ in range(S):
            for j in range(f):
                g = sum(X[t][i] * Sg[s_][i][j] for i in range(d))
                u = sum(X[t][i] * Su[s_][i][j] for i in range(d))
                for i in range(d):
                    y[t][i] += silu(g) * u * Sd[s_][j][i]
    # tau = 0 would keep every neuron and +inf none: the mask alone must decide
    for tau in (0.0, math.inf):
        r = _call(o, x, W, k, tau, active=mask)
        assert np.array_equal(r.active, mask), ("active echo", tau)
        assert np.allclose(r.score, want_score, rtol=1e-12, atol=1e-15), "scores"
        assert _rel(r.y, np.array(y)) < 1e-12, ("y", tau, _rel(r.y, np.array(y)))


def pin_shared_threshold(o):
    """The shared-expert threshold: +inf removes the shared experts (torch fp64
    routed-only layer); tau_s equal to a shared neuron's own score keeps it (>=);
    scalar-Python enumeration at that tau_s; shared scores = |silu(x Ws_g)|."""
    d, E, f, k, S, T = 16, 4, 8, 2, 2, 3
    x, W = _rand_layer(35, d, E, f, k, S, T, scale_x=1.0)
    r_inf = _call(o, x, W, k, 0.0, tau_shared=math.inf)
    y_routed, *_ = _torch_dense(x, W, k, with_shared=False)
    assert _rel(r_inf.y, y_routed) < 1e-12, ("tau_s=inf", _rel(r_inf.y, y_routed))
    X = x.float().double().tolist()
    Wr = W["w_router"].double().tolist()
    Wg, Wu, Wd = (W["w_gate"].double().tolist(), W["w_up"].double().tolist(),
                  W["w_down"].double().tolist())
    Sg, Su, Sd = (W["ws_gate"].double().tolist(), W["ws_up"].double().tolist(),
                  W["ws_down"].double().tolist())

    def silu(z):
        return z / (1.0 + math.exp(-z))

    sh = []   # (t, s, j, silu(g), u)
    for t in range(T):
        for s_ in range(S):
            for j in range(f):
                g = sum(X[t][i] * Sg[s_][i][j] for i in range(d))
                u = sum(X[t][i] * Su[s_][i][j] for i in range(d))
                sh.append((t, s_, j, silu(g), u))
    scores = sorted(abs(a) for (_, _, _, a, _) in sh)
    tau_s = float(np.float32(scores[len(scores) // 2]))   # one shared neuron sits exactly on it
    y = [[0.0] * d for _ in range(T)]
    for t in range(T):
        lg = [sum(X[t][i] * Wr[e][i] for i in range(d)) for e in range(E)]
        m = max(lg)
        ex = [math.exp(v - m) for v in lg]
        p = [v / sum(ex) for v in ex]
        for e in sorted(range(E), key=lambda e: (-p[e], e))[:k]:   # tau = 0: every routed neuron
            for j in range(f):
                g = sum(X[t][i] * Wg[e][i][j] for i in range(d))
                u = sum(X[t][i] * Wu[e][i][j] for i in range(d))
                for i in range(d):
                    y[t][i] += p[e] * silu(g) * u * Wd[e][j][i]
    kept = 0
    for (t, s_, j, a, u) in sh:
        if np.float32(abs(a)) >= np.float32(tau_s):
            kept += 1
            for i in range(d):
                y[t][i] += a * u * Sd[s_][j][i]
    assert 0 < kept < len(sh)
    r = _call(o, x, W, k, 0.0, tau_shared=tau_s)
    assert _rel(r.y, np.array(y)) < 1e-12, ("y", _rel(r.y, np.array(y)))
    want = np.array([[[abs(silu(sum(X[t][i] * Sg[s_][i][j] for i in range(d)))) for j in range(f)]
                      for s_ in range(S)] for t in range(T)])
    assert np.allclose(r.score_shared, want, rtol=1e-12, atol=1e-15), "shared scores"


def pin_nested_masks(o):
    """tau1 < tau2  =>  A(tau2) is a subset of A(tau1), for every pair."""
    x, W = _rand_layer(41, d=64, E=8, f=64, k=2, S=1, T=6)
    prev = None
    for tau in (0.0, 0.1, 0.5, 1.0, 2.0, math.inf):
        r = _call(o, x, W, 2, tau)
        if prev is not None:
            assert np.array_equal(r.topk_idx, prev.topk_idx)
            assert not np.any(r.active & ~prev.active), ("not nested at", tau)
        prev = r


def pin_threshold_decomposition(o):
    """y(t1) - y(t2) equals the sum of the contributions of neurons with t1 <= s < t2."""
    d, E, f, k, S, T = 48, 5, 40, 2, 1, 4
    x, W = _rand_layer(51, d, E, f, k, S, T)
    t1, t2 = 0.3, 0.9
    r1, r2 = _call(o, x, W, k, t1), _call(o, x, W, k, t2)
    xd = x.double()
    p = torch.softmax(xd @ W["w_router"].double().T, dim=-1).numpy()
    diff = np.zeros((T, d))
    for t in range(T):
        for r_ in range(k):
            e = int(r1.topk_idx[t, r_])
            g = (xd[t] @ W["w_gate"][e].double())
            u = (xd[t] @ W["w_up"][e].double())
            a = F.silu(g).numpy()
            s32 = np.abs(a).astype(np.float32)
            band = (s32 >= np.float32(t1)) & (s32 < np.float32(t2))
            h = a * u.numpy() * band
            diff[t] += p[t, e] * (h @ W["w_down"][e].double().numpy())
    got = r1.y - r2.y
    assert _rel(got, diff) < 1e-10, ("decomposition", _rel(got, diff))


def pin_router_ranking(o):
    """Router weights are softmax(x Wr^T)[top-k]; ties go to the lower expert index."""
    d, E, f, k, T = 32, 8, 16, 3, 6
    x, W = _rand_layer(61, d, E, f, k, 0, T)
    wr = W["w_router"].clone()
    wr[5] = wr[1]          # experts 1 and 5 always tie
    wr[6] = wr[2]          # experts 2 and 6 always tie
    W["w_router"] = wr
    r = _call(o, x, W, k, 0.5)
    logits = (x.double() @ wr.double().T).numpy()
    assert np.allclose(r.logits, logits, rtol=1e-13, atol=1e-13), "logits"
    p = torch.softmax(torch.as_tensor(logits), dim=-1).numpy()
    assert np.allclose(p.sum(1), 1.0, atol=1e-12)
    want = np.argsort(-p, axis=1, kind="stable")[:, :k]
    assert np.array_equal(r.topk_idx, want), ("idx", r.topk_idx, want)
    assert np.allclose(r.topk_w, np.take_along_axis(p, want, 1), rtol=1e-13, atol=0), "w"
    # the routing weight is softmax over all E, not renormalised over the top-k
    assert np.all(r.topk_w.sum(1) < 1.0 - 1e-6)


def pin_calibration(o):
    """tau(q) = floor(q N)-th order statistic; kept fraction within 1/N of 1 - q."""
    rng = np.random.default_rng(71)
    s = np.abs(rng.standard_normal(10007))
    for q in (0.0, 0.5, 0.8, 0.9, 0.95, 0.98):
        tau64 = o._lib.oracle_calibrate_tau(o._ptr(s), s.size, q)
        if q == 0.0:
            assert tau64 == 0.0
            continue
        assert tau64 == np.partition(s, int(math.floor(q * s.size)))[int(math.floor(q * s.size))]
        keep = float(np.mean(s >= tau64))
        assert abs(keep - (1 - q)) <= 1.0 / s.size + 1e-15, (q, keep)
    assert math.isinf(o._lib.oracle_calibrate_tau(o._ptr(s), s.size, 1.0))


def _rank_brute(row, r):
    """Scalar-Python rank rule: neuron j is kept iff fewer than r non-NaN
    scores beat it, a score beating j when it is larger in float32, or equal
    with a lower index; NaN is never kept and beats nobody."""
    v = [np.float32(z) for z in row]
    keep = []
    for j, vj in enumerate(v):
        if vj != vj:
            keep.append(0)
            continue
        above = sum(1 for i, vi in enumerate(v) if vi == vi and (vi > vj or (vi == vj and i < j)))
        keep.append(1 if above < r else 0)
    return keep


def pin_rank_bruteforce(o):
    """The per-pair rank budget against a scalar enumeration of its rule, on
    scores with exact ties, NaN, zeros, +inf and a pair that is distinct in
    double but tied in float; the kept count is min(r, non-NaN) and budgets
    nest."""
    rng = np.random.default_rng(81)
    f = 12
    rows = [np.abs(rng.standard_normal(f)),
            np.round(np.abs(rng.standard_normal(f)) * 2) / 2,     # many exact ties
            np.zeros(f),                                        # all tied: lowest indices
            np.array([1.0, math.nan, 0.5, 1.0, math.inf, 0.0, math.nan, 0.5, 2.0, 1.0, 0.25, 0.0]),
            np.array([0.5] * 10 + [1.0, 1.0 + 1e-12])]           # float tie, double order reversed
    s = np.array(rows)
    prev = None
    for r in range(0, f + 2):
        m = o.rank_mask(s, r)
        want = np.array([_rank_brute(row, r) for row in rows], np.uint8)
        assert np.array_equal(m, want), ("rank mask", r, m.tolist(), want.tolist())
        n_valid = (~np.isnan(s)).sum(axis=1)
        assert np.array_equal(m.sum(axis=1), np.minimum(r, n_valid)), ("count", r)
        if prev is not None:
            assert np.all(prev <= m), ("nesting", r)
        prev = m
    assert o.rank_mask(s[4:5], 1)[0, 10] == 1   # 1.0 and 1.0+1e-12 tie in float: index 10 wins


def pin_rank_layer(o):
    """The layer under a rank budget: budget 0 is the shared-only layer (tau =
    +inf), budget >= f the unmasked one (tau = 0); one pair with distinct
    float scores equals the threshold layer at its r-th largest score; a zero
    token keeps its r lowest neurons; a scalar-Python enumeration of the whole
    layer at r = 3."""
    d, E, f, k, S, T = 16, 4, 8, 2, 1, 3
    x, W = _rand_layer(83, d, E, f, k, S, T, scale_x=1.0)
    args = {n: _bits(t) for n, t in W.items()}
    xb = _bits(x)
    inf_ = _call(o, x, W, k, math.inf)
    zero = _call(o, x, W, k, 0.0)
    assert _rel(o.forward_budget(xb, **args, top_k=k, budget=0).y, inf_.y) < 1e-15
    assert _rel(o.forward_budget(xb, **args, top_k=k, budget=f).y, zero.y) < 1e-15
    assert _rel(o.forward_budget(xb, **args, top_k=k, budget=f + 5).y, zero.y) < 1e-15
    # one token, one expert: the budget is the threshold at the r-th largest score
    x1, W1 = _rand_layer(84, d, 4, 16, 1, 0, 1, scale_x=1.0)
    a1 = {n: _bits(t) for n, t in W1.items()}
    sc = _call(o, x1, W1, 1, 0.0).score.reshape(-1).astype(np.float32)
    assert len(set(sc.tolist())) == sc.size
    for r in (1, 5, 11):
        tau = float(np.sort(sc)[::-1][r - 1])
        rb = o.forward_budget(_bits(x1), **a1, top_k=1, budget=r)
        rt = _call(o, x1, W1, 1, tau)
        assert np.array_equal(rb.active, rt.active) and int(rb.active.sum()) == r, ("threshold", r)
        assert _rel(rb.y, rt.y) < 1e-15
    # a zero token: every score is 0, a tie broken toward the lower index
    x0 = x.clone()
    x0[1] = 0
    r0 = o.forward_budget(_bits(x0), **args, top_k=k, budget=3)
    assert np.array_equal(r0.active[1], np.array([[1, 1, 1, 0, 0, 0, 0, 0]] * k, np.uint8))
    # scalar enumeration of the layer at r = 3
    X = x.float().double().tolist()
    Wr = W["w_router"].double().tolist()
    Wg, Wu, Wd = (W["w_gate"].double().tolist(), W["w_up"].double().tolist(),
                  W["w_down"].double().tolist())
    Sg, Su, Sd = (W["ws_gate"].double().tolist(), W["ws_up"].double().tolist(),
                  W["ws_down"].double().tolist())

    def silu(z):
        return z / (1.0 + math.exp(-z))

    r = 3
    y = [[0.0] * d for _ in range(T)]
    for t in range(T):
        lg = [sum(X[t][i] * Wr[e][i] for i in range(d)) for e in range(E)]
        mx = max(lg)
        ex = [math.exp(v - mx) for v in lg]
        p = [v / sum(ex) for v in ex]
        for e in sorted(range(E), key=lambda e: (-p[e], e))[:k]:
            gs = [sum(X[t][i] * Wg[e][i][j] for i in range(d)) for j in range(f)]
            keep = _rank_brute([abs(silu(g)) for g in gs], r)
            for j in range(f):
                if keep[j]:
                    u = sum(X[t][i] * Wu[e][i][j] for i in range(d))
                    for i in range(d):
                        y[t][i] += p[e] * silu(gs[j]) * u * Wd[e][j][i]
        for s_ in range(S):
            for j in range(f):
                g = sum(X[t][i] * Sg[s_][i][j] for i in range(d))
                u = sum(X[t][i] * Su[s_][i][j] for i in range(d))
                for i in range(d):
                    y[t][i] += silu(g) * u * Sd[s_][j][i]
    rb = o.forward_budget(xb, **args, top_k=k, budget=r)
    assert _rel(rb.y, np.array(y)) < 1e-12, ("layer", _rel(rb.y, np.array(y)))
    assert np.all(rb.active.sum(axis=2) == r)


def _capacity_sorted(idx, w, E, C):
    """Each expert's pairs sorted by (float32 weight descending, token
    ascending); the first C are kept (C < 0: all)."""
    T, k = idx.shape
    keep = np.zeros((T, k), np.uint8)
    for e in range(E):
        pairs = [(t, r) for t in range(T) for r in range(k) if idx[t, r] == e]
        pairs.sort(key=lambda tr: (-float(np.float32(w[tr])), tr[0]))
        for t, r in (pairs if C < 0 else pairs[:C]):
            keep[t, r] = 1
    return keep


def pin_capacity_bruteforce(o):
    """Capacity-aware token drop against a per-expert sort: random routings
    with exact weight ties, a pair tied in float but ordered in double, every
    capacity from none to above T; kept count per expert = min(load, C);
    capacities nest."""
    rng = np.random.default_rng(91)
    T, k, E = 12, 3, 5
    idx = np.zeros((T, k), np.int32)
    for t in range(T):
        idx[t] = rng.choice(E, size=k, replace=False)
    w = np.round(rng.random((T, k)) * 4) / 8 + 0.05        # many exact ties
    w[2, 0], w[7, 0] = 0.3, 0.3 + 1e-12                    # equal in float: token 2 first
    idx[2, 0] = idx[7, 0] = 1
    prev = None
    for C in range(-1, T + 2):
        got = o.capacity_keep(idx, w, E, C)
        want = _capacity_sorted(idx, w, E, C)
        assert np.array_equal(got, want), ("capacity", C)
        for e in range(E):
            load = int((idx == e).sum())
            assert int(got[idx == e].sum()) == (load if C < 0 else min(load, C)), ("count", C, e)
        if prev is not None and C > 0:
            assert np.all(prev <= got), ("nesting", C)
        prev = got
    assert o.capacity_keep(idx, w, E, -1).all() and not o.capacity_keep(idx, w, E, 0).any()
    assert o.capacity(1.0, 16, 8, 64) == 2 and o.capacity(1.25, 16, 8, 64) == 3 and o.capacity(0.0, 16, 8, 64) == -1


def pin_capacity_layer(o):
    """The layer under capacity-aware token drop at tau = 0 against a torch
    fp64 composition of the routed SwiGLU experts over the kept pairs only
    (kept set from the per-expert sort), plus the shared expert; a capacity
    of at least T equals the layer without it."""
    d, E, f, k, S, T = 16, 4, 8, 2, 1, 7
    x, W = _rand_layer(93, d, E, f, k, S, T, scale_x=1.0)
    args = {n: _bits(t) for n, t in W.items()}
    xb = _bits(x)
    _, idx, p, _ = _torch_dense(x, W, k)
    w = np.take_along_axis(p, idx, axis=1)
    for gamma in (0.5, 0.8, 1.0):
        C = o.capacity(gamma, T, k, E)
        assert 0 < C < T
        keep = _capacity_sorted(idx, w, E, C)
        assert 0 < keep.sum() < T * k
        xd = x.double()
        y = torch.zeros_like(xd)
        for t in range(T):
            for r in range(k):
                if keep[t, r]:
                    e = int(idx[t, r])
                    g = xd[t] @ W["w_gate"][e].double()
                    u = xd[t] @ W["w_up"][e].double()
                    y[t] += p[t, e] * ((F.silu(g) * u) @ W["w_down"][e].double())
        for s_ in range(S):
            g = xd @ W["ws_gate"][s_].double()
            u = xd @ W["ws_up"][s_].double()
            y += (F.silu(g) * u) @ W["ws_down"][s_].double()
        r = o.forward_capacity(xb, **args, top_k=k, tau=0.0, gamma=gamma)
        assert _rel(r.y, y.numpy()) < 1e-12, ("layer", gamma, _rel(r.y, y.numpy()))
        assert np.array_equal(r.active.any(axis=2), keep.astype(bool))
    big = o.forward_capacity(xb, **args, top_k=k, tau=0.0, gamma=100.0)
    assert _rel(big.y, _call(o, x, W, k, 0.0).y) < 1e-15


ALL_PINS = [pin_handworked, pin_tau0_is_dense, pin_tauinf_is_shared_only, pin_bruteforce,
            pin_mask_override, pin_shared_threshold, pin_nested_masks, pin_threshold_decomposition,
            pin_router_ranking, pin_calibration, pin_rank_bruteforce, pin_rank_layer,
            pin_capacity_bruteforce, pin_capacity_layer]


def run_all(o):
    """Run every pin; return {name: None (passed) | error text}."""
    out = {}
    for pin in ALL_PINS:
        try:
            pin(o)
            out[pin.__name__] = None
        except Exception as exc:  # noqa: BLE001 - a mutant may fail in any way
            out[pin.__name__] = f"{type(exc).__name__}: {str(exc)[:200]}"
    return out
