"""The dense tensor-core branch (tcgen05 grouped GEMMs) against the CPU oracle
and against the sparse branch, through the C ABI.

The dense branch rounds h to bf16 before the down projection, so outputs are
compared at the layer's 1e-2 relative-L2 bar.  Its mask is decided on
tensor-core fp32 gate values, where a neuron scoring within 1e-5*tau of tau
may go either way; such a token must match the oracle under one of the
decisions of its band neurons (every combination is evaluated).  Only
near-tie router tokens are left out of the output check.
"""

import numpy as np
import pytest
import torch

import moe_inputs as mi
import oracle
from tests import parity_util as pu

pytestmark = pytest.mark.gpu

# the dense branch's mask is decided on tensor-core fp32 gate values (sums of
# 2048 to 4096 products in a different order from the oracle's fp64 sums):
# neurons this close to tau may go either way
DENSE_BAND_REL = 1e-5


@pytest.fixture(scope="module")
def o():
    return oracle.load()


_cache = {}


def layer_for(name):
    if name not in _cache:
        for k in list(_cache):
            _cache.pop(k)[0].close()
        torch.cuda.empty_cache()
        sh = mi.SHAPES[name]
        layer, W = pu.gpu_layer(sh, max_tokens=4096)
        _cache[name] = (layer, W, oracle.layer_inputs(W, torch.zeros(1, sh.d_model, dtype=torch.bfloat16)))
    return _cache[name]


def run_dense(o, name, T, q, sample=None, masked=True):
    import intra_expert_activation_router_b200 as m
    sh = mi.SHAPES[name]
    layer, W, host = layer_for(name)
    x = mi.make_x(sh, T, device="cuda")
    inputs = dict(host)
    inputs["x"] = mi.bf16_bits(x)
    cal = dict(inputs)
    cal["x"] = inputs["x"][:64]
    tau = pu.calibrate(o, cal, sh.top_k, q) if masked else 0.0
    if masked:
        layer.set_path(m.MOE_PATH_DENSE)
        out = layer.forward(x, tau)
        layer.set_path(m.MOE_PATH_AUTO)
    else:
        out = layer.dense_forward(x)
    torch.cuda.synchronize()
    st = layer.stats()
    assert st["path"] == m.MOE_PATH_DENSE and st["device_error"] == 0
    rows = np.arange(T) if sample is None else np.sort(
        np.random.default_rng(7 * T + 1).choice(T, size=min(sample, T), replace=False))
    sub = dict(inputs)
    sub["x"] = inputs["x"][rows]
    ref = o.forward(**sub, top_k=sh.top_k, tau=tau)
    tie = pu.near_tie_tokens(ref.logits, sh.top_k)
    assert tie.sum() <= max(1, len(rows) // 50)
    band = DENSE_BAND_REL if masked and 0 < tau < np.inf else 0.0
    pu.check_output_any_band_decision(o, sub, sh.top_k, tau, ref, out[torch.as_tensor(rows, device="cuda")],
                                      tie, band)
    return layer, x, tau, out


def test_tiny_dense_masked(o):
    run_dense(o, "tiny", 16, 0.9)


def test_tiny_dense_unmasked(o):
    run_dense(o, "tiny", 16, 0.0, masked=False)


@pytest.mark.parametrize("T", [1, 64, 257, 1000, 4096])
def test_olmoe_dense(o, T):
    run_dense(o, "olmoe", T, 0.9, sample=None if T <= 64 else 12)


def test_olmoe_dense_unmasked_baseline(o):
    run_dense(o, "olmoe", 300, 0.0, sample=12, masked=False)


@pytest.mark.parametrize("T", [8, 128])
def test_dsv2lite_dense_shared(o, T):
    run_dense(o, "dsv2lite", T, 0.8, sample=None if T <= 8 else 12)


def test_large_dense(o):
    run_dense(o, "large", 64, 0.98, sample=8)


@pytest.mark.parametrize("name,T", [("olmoe", 64), ("olmoe", 1000), ("dsv2lite", 8), ("dsv2lite", 128)])
def test_dense_deterministic_combine(o, name, T):
    """moe_set_deterministic on the dense branch: each (token, slot) row of
    the down GEMM's epilogue written once, the k + S rows of a token summed in
    order: oracle parity as for the atomic combine, and repeats bit-identical."""
    import intra_expert_activation_router_b200 as m
    layer, W, host = layer_for(name)
    layer.set_deterministic(True)
    try:
        layer, x, tau, out = run_dense(o, name, T, 0.9, sample=None if T <= 64 else 12)
        assert layer.stats()["deterministic"] == 1
        layer.set_path(m.MOE_PATH_DENSE)
        reps = [layer.forward(x, tau).clone() for _ in range(3)]
        torch.cuda.synchronize()
        for u in reps:
            assert torch.equal(u, out)
    finally:
        layer.set_deterministic(False)
        layer.set_path(m.MOE_PATH_AUTO)


def test_dense_matches_sparse(o):
    """Both branches of the same layer at the same tau agree (up to h's bf16 rounding)."""
    import intra_expert_activation_router_b200 as m
    sh = mi.SHAPES["olmoe"]
    layer, W, host = layer_for("olmoe")
    x = mi.make_x(sh, 48, device="cuda")
    tau = layer.calibrate_tau(x, 0.9)
    layer.set_path(m.MOE_PATH_SPARSE)
    ys = layer.forward(x, tau).float()
    layer.set_path(m.MOE_PATH_DENSE)
    yd = layer.forward(x, tau).float()
    layer.set_path(m.MOE_PATH_AUTO)
    torch.cuda.synchronize()
    rel = ((yd - ys).norm(dim=1) / ys.norm(dim=1)).cpu().numpy()
    # a rare band neuron decided differently moves one token by a few percent
    assert np.sum(rel > 1e-2) <= 2 and np.median(rel) < 5e-3


def test_auto_switch_picks_by_batch(o):
    import intra_expert_activation_router_b200 as m
    sh = mi.SHAPES["olmoe"]
    layer, W, host = layer_for("olmoe")
    layer.set_t_star(32)
    for T, want in ((32, m.MOE_PATH_SPARSE), (33, m.MOE_PATH_DENSE)):
        x = mi.make_x(sh, T, device="cuda")
        layer.forward(x, 1.0)
        assert layer.stats()["path"] == want
    layer.set_t_star(16)


@pytest.mark.parametrize("name,q", [("olmoe", 0.9), ("dsv2lite", 0.9), ("large", 0.98)])
def test_tuned_switch_point_selects_by_batch(o, name, q):
    """moe_tune_t_star measures both branches on the device; AUTO then takes the
    sparse branch up to the measured T* and the dense branch above it."""
    import intra_expert_activation_router_b200 as m
    sh = mi.SHAPES[name]
    layer, W, host = layer_for(name)
    x = mi.make_x(sh, 64, device="cuda")
    tau = layer.calibrate_tau(x, q)
    t_star = layer.tune_t_star(x, tau)
    try:
        assert 1 <= t_star <= 64, t_star
        assert layer.stats()["t_star"] == t_star
        for T in sorted({1, t_star, min(t_star + 1, 64), 64}):
            layer.forward(x[:T].contiguous(), tau)
            want = m.MOE_PATH_SPARSE if T <= t_star else m.MOE_PATH_DENSE
            assert layer.stats()["path"] == want, (T, t_star)
    finally:
        layer.set_t_star(16)


def test_dense_unsupported_shape_rejected():
    import intra_expert_activation_router_b200 as m
    sh = mi.custom_shape(264, 4, 32, 4, 0)   # d not a multiple of 256: no dense branch
    W = mi.make_weights(sh, device="cuda")
    layer = m.MoESparseLayer.from_weights(W, 4, max_tokens=16)
    x = mi.make_x(sh, 4, device="cuda")
    with pytest.raises(m.MoeError) as ei:
        layer.dense_forward(x)
    assert ei.value.code == m.MOE_ENOTSUP
    layer.set_t_star(0)          # AUTO above T* falls back to the sparse branch on such shapes
    layer.forward(x, 0.5)
    torch.cuda.synchronize()
    assert layer.stats()["path"] == m.MOE_PATH_SPARSE
    layer.close()
