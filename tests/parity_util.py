"""Helpers for comparing the CUDA path with the CPU oracle on the same seeded inputs.

Acceptance rules (the layer's own stated bar):
  * router top-k indices equal, except tokens whose k-th and (k+1)-th oracle
    logits are within 1e-5 * max|logit| (a near tie that fp32 may order
    either way -- 1e-5 is several hundred times the fp32 accumulation error of
    a 4096-long dot product of these magnitudes); such tokens are excluded;
  * active-neuron sets equal, except neurons whose oracle score lies within
    1e-3 * tau of tau;
  * per token, ||y_gpu - y_oracle|| / ||y_oracle|| <= 1e-2, excluding tokens
    with a near-tie router or a band neuron decided differently; when the
    oracle output is exactly zero the GPU output must be exactly zero.
A calibrated tau is itself the score of one routed neuron, so that neuron
sits exactly on the threshold and either decision is correct; flips inside
the band are therefore allowed (and their tokens excluded from the output
comparison), while near ties must stay rare.
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
    """idx_lists [T][k][f] (first cnt valid), cnt [T][k]; returns tokens with a flipped band neuron."""
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
    return flipped, int(band.sum())


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
