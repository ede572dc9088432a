"""Helpers for comparing the CUDA path with the CPU oracle on the same seeded inputs.

Acceptance rules (the layer's own stated bar):
  * router top-k indices equal, except tokens whose k-th and (k+1)-th oracle
    logits are within 1e-5 * max|logit| (a near tie that fp32 may order
    either way -- 1e-5 is several hundred times the fp32 accumulation error of
    a 4096-long dot product of these magnitudes); such tokens are excluded;
  * active-neuron sets equal, except neurons whose oracle score lies within
    1e-3 * tau of tau;
  * per token, ||y_gpu - y_oracle|| / ||y_oracle|| <= 1e-2 for every token
    except near-tie router tokens; when the oracle output is exactly zero the
    GPU output must be exactly zero.
A calibrated tau is itself the score of one routed neuron, so that neuron
sits exactly on the threshold and either decision is correct.  A token with
a band neuron that the GPU decided the other way is therefore compared with
the oracle evaluated under the GPU's own mask (the oracle's `active` input),
not dropped: its expected output is the one whose active set equals the
GPU's.  Where the GPU's mask is not exported (the dense branch), every
combination of the token's threshold-band decisions is evaluated and the
GPU output must match one of them.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import moe_inputs as mi
import oracle

TIE_REL = 1e-5
BAND_REL = 1e-3
OUT_REL_L2 = 1e-2


def host_inputs(W, x):
    return oracle.layer_inputs(W, x)


def calibrate(o, inputs, top_k, sparsity, nthreads=0):
    """tau from the oracle's scores of the routed pairs (see oracle.calibrate_tau)."""
    if sparsity <= 0:
        return 0.0
    r = o.forward(**inputs, top_k=top_k, tau=math.inf, nthreads=nthreads)
    return o.calibrate_tau(r.score, sparsity)


def near_tie_tokens(logits, k):
    E = logits.shape[1]
    if k >= E:
        return np.zeros(logits.shape[0], bool)
    s = -np.sort(-logits, axis=1)
    gap = s[:, k - 1] - s[:, k]
    return gap <= TIE_REL * np.abs(logits).max(axis=1)


def check_router(ref, idx_gpu, w_gpu, k):
    tie = near_tie_tokens(ref.logits, k)
    ok = np.all(ref.topk_idx == idx_gpu, axis=1) | tie
    assert ok.all(), f"router mismatch at tokens {np.where(~ok)[0][:10]}"
    wdiff = np.abs(ref.topk_w - w_gpu)[~tie]
    assert wdiff.size == 0 or wdiff.max() <= 1e-5 + 1e-4 * np.abs(ref.topk_w[~tie]).max(), wdiff.max()
    return tie


def check_active(ref, tau, idx_lists, cnt, tie):
    """idx_lists [T][k][f] (first cnt valid), cnt [T][k].

    Returns (tokens with a band neuron decided differently, number of band
    neurons, the GPU's mask [T][k][f] bool)."""
    T, k, f = ref.active.shape
    gpu = np.zeros((T, k, f), bool)
    for t in range(T):
        for r in range(k):
            c = int(cnt[t, r])
            lst = idx_lists[t, r, :c].astype(np.int64)
            assert np.all(np.diff(lst) > 0), f"list not ascending at ({t},{r})"
            gpu[t, r, lst] = True
    band = np.abs(ref.score - tau) <= BAND_REL * abs(tau)
    ref_on = ref.active.astype(bool)
    diff = gpu != ref_on
    bad = diff & ~band
    bad[tie] = False
    assert not bad.any(), f"{int(bad.sum())} active-set mismatches outside the band, first at {np.argwhere(bad)[:5]}"
    flipped = np.any(diff & band, axis=(1, 2))
    return flipped, int(band.sum()), gpu


def gpu_mask_from_lists(idx_lists, cnt, f):
    """[T][k][f] bool from the ascending active lists (first cnt valid)."""
    T, k = cnt.shape
    gpu = np.zeros((T, k, f), bool)
    for t in range(T):
        for r in range(k):
            c = int(cnt[t, r])
            lst = idx_lists[t, r, :c].astype(np.int64)
            assert np.all(np.diff(lst) > 0), f"list not ascending at ({t},{r})"
            gpu[t, r, lst] = True
    return gpu


def check_rank_mask(o, scores, budget, gpu_mask, tie, band_rel=BAND_REL):
    """The CUDA path's per-pair rank selection against the oracle's scores.

    Exact: every pair keeps min(budget, f) neurons (the inputs hold no NaN).
    Valid: no kept neuron scores (oracle, rounded to float) below a dropped one
    by more than band_rel of the larger; the GPU's fp32 g may order two
    neurons that close the other way.  Returns (tokens whose selection differs
    from the oracle's rank mask, the oracle's rank mask)."""
    T, k, f = scores.shape
    want = o.rank_mask(scores, budget).astype(bool)
    cnt = gpu_mask.sum(axis=2)
    assert np.all(cnt[~tie] == min(budget, f)), f"kept counts {np.unique(cnt[~tie])}, want {min(budget, f)}"
    s = scores.astype(np.float32).astype(np.float64)
    for t in range(T):
        if tie[t]:
            continue
        for r in range(k):
            kept, dropped = s[t, r][gpu_mask[t, r]], s[t, r][~gpu_mask[t, r]]
            if kept.size and dropped.size:
                lo, hi = kept.min(), dropped.max()
                assert lo >= hi - band_rel * max(abs(hi), 1e-30), (t, r, lo, hi)
    differ = np.any(gpu_mask != want, axis=(1, 2)) & ~tie
    return differ, want


def expected_under_gpu_mask(o, inputs, top_k, tau, ref, gpu_mask, flipped, tie, nthreads=0, tau_shared=0.0):
    """The oracle's output per token, where a token whose band neuron the GPU
    decided the other way is evaluated under the GPU's mask instead."""
    y = ref.y.copy()
    rows = np.where(flipped & ~tie)[0]
    if rows.size:
        sub = dict(inputs)
        sub["x"] = inputs["x"][rows]
        r2 = o.forward(**sub, top_k=top_k, tau=tau, active=gpu_mask[rows], want_scores=True,
                       nthreads=nthreads, tau_shared=tau_shared)
        assert np.array_equal(r2.topk_idx, ref.topk_idx[rows])
        y[rows] = r2.y
    return y


def check_output_any_band_decision(o, inputs, top_k, tau, ref, out_gpu, tie, band_rel, max_band=8,
                                   nthreads=0, tau_shared=0.0):
    """Output check for a path whose mask is not exported: a token with n
    neurons within band_rel*tau of tau must match the oracle under one of the
    2**n decisions of those neurons (all other neurons as the oracle decides).
    Returns (worst rel L2, number of tokens that needed the enumeration)."""
    y = out_gpu.float().cpu().double().numpy() if torch.is_tensor(out_gpu) else out_gpu
    amb = np.abs(ref.score - tau) <= band_rel * abs(tau)
    worst, n_amb = 0.0, 0
    for t in range(y.shape[0]):
        if tie[t]:
            continue
        pos = np.argwhere(amb[t])
        if pos.shape[0] == 0:
            worst = max(worst, check_output(ref.y[t:t + 1], y[t:t + 1]))
            continue
        n_amb += 1
        assert pos.shape[0] <= max_band, f"token {t}: {pos.shape[0]} band neurons"
        sub = dict(inputs)
        sub["x"] = inputs["x"][t:t + 1]
        best = math.inf
        for combo in range(1 << pos.shape[0]):
            mask = ref.active[t:t + 1].astype(bool).copy()
            for b, (r, j) in enumerate(pos):
                mask[0, r, j] = bool((combo >> b) & 1)
            yc = o.forward(**sub, top_k=top_k, tau=tau, active=mask, want_scores=False,
                           nthreads=nthreads, tau_shared=tau_shared).y[0]
            nr = np.linalg.norm(yc)
            rel = np.linalg.norm(y[t] - yc) / nr if nr > 0 else (0.0 if not np.any(y[t]) else math.inf)
            best = min(best, rel)
        assert best <= OUT_REL_L2, f"token {t}: rel L2 {best:.3e} under every band decision"
        worst = max(worst, best)
    return worst, n_amb


def check_output(ref_y, out_gpu, exclude=None):
    y = out_gpu.float().cpu().double().numpy() if torch.is_tensor(out_gpu) else out_gpu
    T = ref_y.shape[0]
    exclude = np.zeros(T, bool) if exclude is None else exclude
    worst = 0.0
    for t in range(T):
        if exclude[t]:
            continue
        nr = np.linalg.norm(ref_y[t])
        if nr == 0.0:
            assert not np.any(y[t]), f"token {t}: expected exact zeros"
            continue
        rel = np.linalg.norm(y[t] - ref_y[t]) / nr
        worst = max(worst, rel)
        assert rel <= OUT_REL_L2, f"token {t}: rel L2 {rel:.3e} > {OUT_REL_L2}"
    return worst


def gpu_layer(shape, device="cuda", max_tokens=4096, weights=None):
    from intra_expert_activation_router_b200 import MoESparseLayer
    W = weights if weights is not None else mi.make_weights(shape, device=device)
    layer = MoESparseLayer.from_weights(W, shape.top_k, max_tokens=max_tokens)
    return layer, W


def threshold_off_scores(scores, q, eps=1e-4):
    """A threshold near the q-quantile of `scores` that no score lies within
    eps (relative) of: halfway between two neighbouring scores, so that fp32
    and fp64 scores decide every neuron alike."""
    s = np.sort(np.asarray(scores, dtype=np.float64).reshape(-1))
    m = int(math.floor(q * s.size))
    for delta in range(s.size):
        for mm in (m + delta, m - delta):
            if 1 <= mm < s.size:
                tau = float(np.float32(0.5 * (s[mm - 1] + s[mm])))
                if tau > 0 and not np.any(np.abs(s - tau) <= eps * tau):
                    return tau
    raise AssertionError("no threshold clear of the scores")
