"""CUDA path vs the CPU oracle, through the C ABI, on the five workloads' shapes.

Every comparison uses the same seeded bf16 inputs on both sides.  Small
batches are compared token by token in full; the big batches (and the
6.44 GB layer) on a seeded sample of tokens, which the oracle computes one
by one -- tokens are independent, so a sampled token's expected output is
exact.
"""
import math

import numpy as np
import pytest
import torch

import moe_inputs as mi
import oracle
from tests import parity_util as pu

pytestmark = pytest.mark.gpu

NTHREADS = 0   # oracle: all host cores


@pytest.fixture(scope="module")
def o():
    return oracle.load()


_layers = {}


def layer_for(name, max_tokens=4096):
    key = (name, max_tokens)
    if key not in _layers:
        for k_ in list(_layers):
            if k_[0] != name:
                _layers.pop(k_)[0].close()
        torch.cuda.empty_cache()
        sh = mi.SHAPES[name]
        layer, W = pu.gpu_layer(sh, max_tokens=max_tokens)
        _layers[key] = (layer, W, oracle.layer_inputs(W, torch.zeros(1, sh.d_model, dtype=torch.bfloat16)))
    return _layers[key]


def run_case(o, name, T, q, sample=None, check_lists=True):
    sh = mi.SHAPES[name]
    layer, W, host = layer_for(name)
    x = mi.make_x(sh, T, device="cuda")
    inputs = dict(host)
    inputs["x"] = mi.bf16_bits(x)
    # tau: the oracle's calibration on (at most) the first 64 tokens of the batch
    cal = dict(inputs)
    cal["x"] = inputs["x"][:64]
    tau = pu.calibrate(o, cal, sh.top_k, q, NTHREADS)
    # the sparse GPU path on the whole batch (large batches would otherwise switch to dense)
    import intra_expert_activation_router_b200 as m
    layer.set_path(m.MOE_PATH_SPARSE)
    out = layer.forward(x, tau)
    layer.set_path(m.MOE_PATH_AUTO)
    idx, w = layer.router(x)
    out_dbg = torch.empty_like(x)
    lists, cnt = layer.active_lists(x, tau, out=out_dbg) if check_lists else (None, None)
    torch.cuda.synchronize()
    rows = np.arange(T) if sample is None else np.sort(
        np.random.default_rng(1000 * T + int(q * 100)).choice(T, size=min(sample, T), replace=False))
    sub = dict(inputs)
    sub["x"] = inputs["x"][rows]
    ref = o.forward(**sub, top_k=sh.top_k, tau=tau, nthreads=NTHREADS, want_scores=check_lists)
    tie = pu.check_router(ref, idx.cpu().numpy()[rows], w.cpu().numpy()[rows], sh.top_k)
    y_expect = ref.y
    flipped = np.zeros(len(rows), bool)
    trows = torch.as_tensor(rows, device="cuda")
    if check_lists:
        flipped, _, gmask = pu.check_active(ref, tau, lists.cpu().numpy().view(np.uint16)[rows],
                                            cnt.cpu().numpy()[rows], tie)
        # a token whose threshold-band neuron the GPU decided the other way is
        # checked against the oracle under the GPU's mask, not dropped
        y_expect = pu.expected_under_gpu_mask(o, sub, sh.top_k, tau, ref, gmask, flipped, tie, NTHREADS)
        pu.check_output(y_expect, out_dbg[trows], tie)
    worst = pu.check_output(y_expect, out[trows], tie)
    assert tie.sum() <= max(1, len(rows) // 50), "too many near-tie tokens"
    assert flipped.sum() <= max(2, len(rows) // 20), "too many band flips"
    return tau, worst, layer


def test_tiny(o):
    tau, worst, _ = run_case(o, "tiny", 16, 0.9)
    assert 0.5 < tau < 2.0


@pytest.mark.parametrize("T", [1, 4, 16, 64])
def test_olmoe(o, T):
    run_case(o, "olmoe", T, 0.9)


@pytest.mark.parametrize("name,T", [("tiny", 1), ("tiny", 2), ("tiny", 9), ("olmoe", 2), ("olmoe", 9),
                                    ("olmoe", 17), ("olmoe", 33)])
def test_tiling_boundaries(o, name, T):
    """The kernel's (tokens per pass, 16-byte slices per thread) instantiations
    not reached above, and the batch sizes where the token tiling changes:
    one token tile up to 16 tokens, 8-token tiles from 17, 16-token tiles
    again from 33."""
    run_case(o, name, T, 0.9)


@pytest.mark.parametrize("name,T,q", [("olmoe", 1, 0.9), ("olmoe", 4, 0.9), ("olmoe", 16, 0.9), ("tiny", 16, 0.9),
                                      ("dsv2lite", 8, 0.9), ("large", 1, 0.98), ("large", 8, 0.98)])
def test_router_kernel_path(o, name, T, q):
    """Decode batches route inside the expert kernel by default; the same
    batches through the separate router kernel must match the oracle too."""
    layer, W, host = layer_for(name)
    layer.set_fused_router(False)
    try:
        run_case(o, name, T, q)
        assert layer.stats()["fused_router"] == 0
    finally:
        layer.set_fused_router(True)


@pytest.mark.parametrize("name,T,q", [("olmoe", 1, 0.9), ("olmoe", 2, 0.9), ("olmoe", 16, 0.9), ("tiny", 16, 0.9),
                                      ("dsv2lite", 8, 0.9), ("large", 1, 0.98), ("olmoe", 40, 0.9)])
def test_one_launch_forward(o, name, T, q):
    """Routing and the combine inside the expert kernel (one launch per
    forward) against the oracle; 40 tokens exceed one token tile, so that
    forward falls back to the router kernel and the conversion kernel."""
    layer, W, host = layer_for(name)
    layer.set_fused_router(True, one_launch=True)
    try:
        for _ in range(2):   # counters left for the next forward must be reset by the kernel itself
            run_case(o, name, T, q)
        assert layer.stats()["fused_router"] == (2 if T <= 16 else 0)
    finally:
        layer.set_fused_router(True)


def test_in_kernel_routing_is_used_for_decode_batches(o):
    sh = mi.SHAPES["olmoe"]
    layer, W, host = layer_for("olmoe")
    for T, want in ((1, 1), (16, 1), (17, 0)):
        x = mi.make_x(sh, T, device="cuda")
        layer.forward(x, 1.0)
        st = layer.stats()
        assert st["fused_router"] == want and st["rc"] == 0, (T, st)
    # the workspace copy of the plan that the statistics use is the kernel's own
    x = mi.make_x(sh, 16, device="cuda")
    idx, _ = layer.router(x)
    layer.forward(x, 1.0)
    st = layer.stats()
    assert st["n_touched"] == len(np.unique(idx.cpu().numpy()))


@pytest.mark.parametrize("T", [1, 8, 32, 128])
@pytest.mark.parametrize("q", [0.0, 0.5, 0.8, 0.9, 0.95])
def test_dsv2lite(o, T, q):
    run_case(o, "dsv2lite", T, q, sample=None if T <= 32 else 24)


@pytest.mark.parametrize("T", [1, 16, 64])
def test_large(o, T):
    run_case(o, "large", T, 0.98, sample=None if T <= 16 else 12)


@pytest.mark.parametrize("T", [3, 13, 100, 257, 1000, 4096])
def test_crossover_sparse_sampled(o, T):
    run_case(o, "crossover", T, 0.9, sample=None if T <= 13 else 12, check_lists=T <= 1000)


@pytest.mark.parametrize("name,T,qs", [
    ("tiny", 16, (0.5, 0.9, 0.98)),
    ("olmoe", 16, (0.5, 0.9, 0.98)),
    ("dsv2lite", 8, (0.5, 0.8, 0.9, 0.95)),
    ("large", 1, (0.98,)),
])
def test_calibrate_tau_matches_oracle(o, name, T, qs):
    """The library's on-GPU threshold (an exact radix select over its fp32
    scores) against the oracle's order statistic of its fp64 scores."""
    sh = mi.SHAPES[name]
    layer, W, host = layer_for(name)
    x = mi.make_x(sh, T, device="cuda")
    inputs = dict(host)
    inputs["x"] = mi.bf16_bits(x)
    ref = o.forward(**inputs, top_k=sh.top_k, tau=math.inf, nthreads=NTHREADS)
    idx, w = layer.router(x)
    torch.cuda.synchronize()
    tie = pu.check_router(ref, idx.cpu().numpy(), w.cpu().numpy(), sh.top_k)
    assert not tie.any(), "a near-tie token would make the two populations differ"
    s = np.sort(ref.score.reshape(-1))
    N = s.size
    eps = 1e-4   # fp32 gate sums of up to 4096 products against fp64 ones
    for q in qs:
        tau_g = layer.calibrate_tau(x, q)
        m = int(math.floor(q * N))
        # the GPU's tau is the m-th smallest score, up to the fp32 noise of the scores
        lo, hi = tau_g * (1 - eps), tau_g * (1 + eps)
        assert np.sum(s < lo) <= m < np.sum(s <= hi), (q, tau_g, s[m])
        assert abs(tau_g - o.calibrate_tau(ref.score, q)) <= 2 * eps * tau_g + (s[min(m + 1, N - 1)] - s[m])
        # about 1 - q of the routed neurons are kept
        band = int(np.sum((s >= lo) & (s <= hi)))
        assert abs(int(np.sum(s >= tau_g)) - (N - m)) <= 1 + band
    assert layer.calibrate_tau(x, 0.0) == 0.0
    assert layer.calibrate_tau(x, -0.5) == 0.0
    assert math.isinf(layer.calibrate_tau(x, 1.0))


@pytest.mark.parametrize("name,T,q,q_s", [("dsv2lite", 8, 0.9, 0.5), ("dsv2lite", 32, 0.9, 0.8),
                                          ("tiny", 16, 0.9, 0.5), ("large", 1, 0.98, 0.9)])
def test_shared_threshold(o, name, T, q, q_s):
    """The shared experts' own threshold (looser than the routed one): the
    sparse branch (in-kernel routing at 8 and 16 tokens, token tiles at 32)
    and the dense branch against the oracle with the same two thresholds."""
    import intra_expert_activation_router_b200 as m
    sh = mi.SHAPES[name]
    layer, W, host = layer_for(name)
    x = mi.make_x(sh, T, device="cuda")
    inputs = dict(host)
    inputs["x"] = mi.bf16_bits(x)
    tau = pu.calibrate(o, inputs, sh.top_k, q, NTHREADS)
    r0 = o.forward(**inputs, top_k=sh.top_k, tau=math.inf, nthreads=NTHREADS)
    tau_s = pu.threshold_off_scores(r0.score_shared, q_s)
    ref = o.forward(**inputs, top_k=sh.top_k, tau=tau, tau_shared=tau_s, nthreads=NTHREADS)
    kept = float(np.mean(r0.score_shared >= tau_s))
    assert 0.0 < kept < 1.0
    layer.set_shared_tau(tau_s)
    try:
        layer.set_path(m.MOE_PATH_SPARSE)
        out = layer.forward(x, tau)
        out_dbg = torch.empty_like(x)
        lists, cnt = layer.active_lists(x, tau, out=out_dbg)
        idx, w = layer.router(x)
        torch.cuda.synchronize()
        tie = pu.check_router(ref, idx.cpu().numpy(), w.cpu().numpy(), sh.top_k)
        flipped, _, gmask = pu.check_active(ref, tau, lists.cpu().numpy().view(np.uint16), cnt.cpu().numpy(), tie)
        y_expect = pu.expected_under_gpu_mask(o, inputs, sh.top_k, tau, ref, gmask, flipped, tie, NTHREADS, tau_s)
        pu.check_output(y_expect, out, tie)
        pu.check_output(y_expect, out_dbg, tie)
        # the unmasked shared experts would give another layer: the threshold is applied
        ref_dense_shared = o.forward(**inputs, top_k=sh.top_k, tau=tau, nthreads=NTHREADS, want_scores=False)
        assert np.linalg.norm(ref_dense_shared.y - ref.y) > 0.05 * np.linalg.norm(ref.y)
        layer.set_path(m.MOE_PATH_DENSE)
        out_d = layer.forward(x, tau)
        torch.cuda.synchronize()
        pu.check_output_any_band_decision(o, inputs, sh.top_k, tau, ref, out_d, tie, 1e-5, nthreads=NTHREADS,
                                          tau_shared=tau_s)
    finally:
        layer.set_shared_tau(0.0)
        layer.set_path(m.MOE_PATH_AUTO)


@pytest.mark.parametrize("name,T,qs", [("tiny", 16, (0.5, 0.9)), ("dsv2lite", 8, (0.5, 0.8, 0.95)),
                                       ("large", 1, (0.5, 0.9))])
def test_calibrate_tau_shared_matches_oracle(o, name, T, qs):
    sh = mi.SHAPES[name]
    layer, W, host = layer_for(name)
    x = mi.make_x(sh, T, device="cuda")
    inputs = dict(host)
    inputs["x"] = mi.bf16_bits(x)
    ref = o.forward(**inputs, top_k=sh.top_k, tau=math.inf, nthreads=NTHREADS)
    s = np.sort(ref.score_shared.reshape(-1))
    N = s.size
    eps = 1e-4
    for q in qs:
        tau_g = layer.calibrate_tau_shared(x, q)
        mq = int(math.floor(q * N))
        lo, hi = tau_g * (1 - eps), tau_g * (1 + eps)
        assert np.sum(s < lo) <= mq < np.sum(s <= hi), (q, tau_g, s[mq])
        band = int(np.sum((s >= lo) & (s <= hi)))
        assert abs(int(np.sum(s >= tau_g)) - (N - mq)) <= 1 + band
    assert layer.calibrate_tau_shared(x, 0.0) == 0.0
    assert math.isinf(layer.calibrate_tau_shared(x, 1.0))


def test_gate_values_beyond_fp16_range(o):
    """|g| up to ~1e6, far above the fp16 range: the sparse path keeps silu(g)
    finite and matches the oracle (routed and shared experts)."""
    from intra_expert_activation_router_b200 import MoESparseLayer
    sh = mi.custom_shape(256, 8, 64, 2, 1, seed_base=7300)
    W = mi.make_weights(sh, device="cuda")
    W.w_gate = (W.w_gate.float() * 2e5).to(torch.bfloat16)
    W.ws_gate = (W.ws_gate.float() * 2e5).to(torch.bfloat16)
    layer = MoESparseLayer.from_weights(W, sh.top_k, max_tokens=16)
    x = mi.make_x(sh, 16, device="cuda")
    inputs = oracle.layer_inputs(W, x)
    tau = pu.calibrate(o, inputs, sh.top_k, 0.7)
    assert tau > 65504.0
    out = layer.forward(x, tau)
    idx, w = layer.router(x)
    lists, cnt = layer.active_lists(x, tau)
    torch.cuda.synchronize()
    assert bool(torch.isfinite(out.float()).all())
    ref = o.forward(**inputs, top_k=sh.top_k, tau=tau)
    tie = pu.check_router(ref, idx.cpu().numpy(), w.cpu().numpy(), sh.top_k)
    flipped, _, gmask = pu.check_active(ref, tau, lists.cpu().numpy().view(np.uint16), cnt.cpu().numpy(), tie)
    pu.check_output(pu.expected_under_gpu_mask(o, inputs, sh.top_k, tau, ref, gmask, flipped, tie), out, tie)
    layer.close()


def test_tau_extremes(o):
    sh = mi.SHAPES["dsv2lite"]
    layer, W, host = layer_for("dsv2lite")
    x = mi.make_x(sh, 5, device="cuda")
    inputs = dict(host)
    inputs["x"] = mi.bf16_bits(x)
    for tau in (0.0, -1.0, math.inf):
        out = layer.forward(x, tau)
        ref = o.forward(**inputs, top_k=sh.top_k, tau=tau, want_scores=False)
        pu.check_output(ref.y, out)
    # no shared expert and tau = +inf: exactly zero
    layer2, W2, host2 = layer_for("olmoe")
    x2 = mi.make_x(mi.SHAPES["olmoe"], 3, device="cuda")
    out2 = layer2.forward(x2, math.inf)
    assert not out2.float().abs().sum().item()


def test_repeat_and_interleave(o):
    """Workspace state (accumulators, tickets) resets itself between calls."""
    sh = mi.SHAPES["olmoe"]
    layer, W, host = layer_for("olmoe")
    xa, xb = mi.make_x(sh, 16, device="cuda"), mi.make_x(sh, 5, device="cuda", seed=99)
    a1 = layer.forward(xa, 1.0).clone()
    b1 = layer.forward(xb, 1.0).clone()
    a2 = layer.forward(xa, 1.0).clone()
    b2 = layer.forward(xb, 1.0).clone()
    torch.cuda.synchronize()
    for u, v in ((a1, a2), (b1, b2)):
        d = (u.float() - v.float()).abs()
        tol = u.float().abs() * 2.0 ** -7 + 1e-6     # fp32 atomics may reorder: <= 1 bf16 ulp
        assert bool((d <= tol).all())


@pytest.mark.parametrize("name,T,mode", [("olmoe", 1, "fused"), ("olmoe", 16, "fused"), ("olmoe", 16, "one_launch"),
                                         ("olmoe", 16, "kernel"), ("olmoe", 40, "kernel"), ("dsv2lite", 8, "fused"),
                                         ("dsv2lite", 8, "one_launch"), ("tiny", 16, "kernel"), ("large", 1, "fused")])
def test_deterministic_combine(o, name, T, mode):
    """moe_set_deterministic: every (token, slot, neuron block) contribution in
    a row of its own, a token's rows summed in one fixed order.  The output
    against the oracle as everywhere else; repeated forwards, interleaved with
    another batch, bit-identical; with the capacity drop on, dropped pairs'
    rows (never written) read as zero, and the next forward without the drop
    is the plain deterministic one again."""
    import intra_expert_activation_router_b200 as m
    sh = mi.SHAPES[name]
    q = 0.98 if name == "large" else 0.9
    layer, W, host = layer_for(name)
    layer.set_fused_router(mode != "kernel", one_launch=(mode == "one_launch"))
    layer.set_deterministic(True)
    try:
        tau, worst, _ = run_case(o, name, T, q)
        st = layer.stats()
        assert st["deterministic"] == 1 and st["device_error"] == 0
        assert st["fused_router"] == ({"kernel": 0, "fused": 1, "one_launch": 2}[mode] if T <= 16 else 0)
        layer.set_path(m.MOE_PATH_SPARSE)
        x = mi.make_x(sh, T, device="cuda")
        xo = mi.make_x(sh, 7, device="cuda", seed=5)
        outs = []
        for _ in range(4):
            outs.append(layer.forward(x, tau).clone())
            layer.forward(xo, tau)
        torch.cuda.synchronize()
        for u in outs[1:]:
            assert torch.equal(u, outs[0])
        if name != "large":   # capacity drop: only where gamma = 1 drops pairs at this T
            layer.set_capacity(1.0)
            try:
                layer.set_deterministic(False)
                plain = layer.forward(x, tau).clone()
                layer.set_deterministic(True)
                c1 = layer.forward(x, tau).clone()
                c2 = layer.forward(x, tau).clone()
                torch.cuda.synchronize()
                C = -(-T * sh.top_k // sh.n_experts)
                assert layer.stats()["capacity"] == (C if C < T else -1)
                assert torch.equal(c1, c2)
                dd = (c1.float() - plain.float()).abs()
                assert bool((dd <= plain.float().abs() * 2.0 ** -7 + 1e-6).all())
            finally:
                layer.set_capacity(0.0)
            again = layer.forward(x, tau)
            torch.cuda.synchronize()
            assert torch.equal(again, outs[0])
    finally:
        layer.set_deterministic(False)
        layer.set_fused_router(True)
        layer.set_path(m.MOE_PATH_AUTO)


@pytest.mark.parametrize("T,fused", [(1, True), (16, True), (16, False)])
def test_traced_kernel(o, T, fused):
    """moe_set_trace switches the sparse path to the traced instantiation of
    the expert kernel: with the deterministic combine its output is bit-equal
    to the untraced kernel's, every CTA that ran stamps a start and an end
    (end >= start), the item counts add up to the forward's work items, and
    turning tracing off goes back to the untraced kernel."""
    import intra_expert_activation_router_b200 as m
    sh = mi.SHAPES["olmoe"]
    layer, W, host = layer_for("olmoe")
    x = mi.make_x(sh, T, device="cuda")
    layer.set_path(m.MOE_PATH_SPARSE)
    layer.set_fused_router(fused)
    layer.set_deterministic(True)
    words = 2 * 148 * 64 + 1024
    buf = torch.zeros(words, dtype=torch.int64, device="cuda")
    try:
        plain = layer.forward(x, 1.0).clone()
        m.moe_set_trace(layer.h, buf, words * 8)
        traced = layer.forward(x, 1.0).clone()
        m.moe_set_trace(layer.h, None)
        again = layer.forward(x, 1.0).clone()
        torch.cuda.synchronize()
        assert layer.stats()["device_error"] == 0
        assert torch.equal(traced, plain) and torch.equal(again, plain)
        b = buf.cpu().numpy()
        router = words // 2
        et = b[router:router + (words - router) // 64 * 64].reshape(-1, 64)
        ran = et[:, 0] > 0
        assert ran.sum() >= 8
        assert (et[ran, 62] >= et[ran, 0]).all()
        st = layer.stats()
        assert int(et[ran, 63].sum()) >= st["n_touched"] * (sh.d_ff // 128)
    finally:
        m.moe_set_trace(layer.h, None)
        layer.set_deterministic(False)
        layer.set_fused_router(True)
        layer.set_path(m.MOE_PATH_AUTO)


@pytest.mark.parametrize("name,T,mode", [("dsv2lite", 2, "fused"), ("dsv2lite", 4, "fused"), ("dsv2lite", 4, "kernel"),
                                         ("tiny", 4, "fused"), ("tiny", 4, "one_launch"), ("large", 2, "fused"),
                                         ("large", 4, "fused")])
def test_dense_shared_items_split(o, name, T, mode):
    """Layers whose shared experts run without a threshold split those heavy
    items: by the gate's K stages with the records shared (one and two
    tokens, where the grid allows) or by records, each part streaming the
    whole gate (more tokens).  Both part counts (2, and 4 where every claim
    has an SM) and both routing modes, against the oracle."""
    layer, W, host = layer_for(name)
    layer.set_fused_router(mode != "kernel", one_launch=(mode == "one_launch"))
    try:
        for _ in range(2):   # counters the split uses must be reset by the forward itself
            run_case(o, name, T, 0.98 if name == "large" else 0.9)
        assert layer.stats()["device_error"] == 0
    finally:
        layer.set_fused_router(True)


def test_host_pointer_entry(o):
    from intra_expert_activation_router_b200 import moe_sparse_forward_host
    sh = mi.SHAPES["olmoe"]
    layer, W, host = layer_for("olmoe")
    x = mi.make_x(sh, 7, device="cuda")
    dev = layer.forward(x, 1.0)
    xh = x.cpu().pin_memory()
    oh = torch.empty_like(xh).pin_memory()
    moe_sparse_forward_host(layer.h, xh, 7, 1.0, oh)
    d = (oh.float() - dev.cpu().float()).abs()
    assert bool((d <= dev.cpu().float().abs() * 2.0 ** -7 + 1e-6).all())


def test_stats_match_oracle(o):
    sh = mi.SHAPES["olmoe"]
    layer, W, host = layer_for("olmoe")
    T = 16
    x = mi.make_x(sh, T, device="cuda")
    inputs = dict(host)
    inputs["x"] = mi.bf16_bits(x)
    tau = pu.calibrate(o, inputs, sh.top_k, 0.9)
    layer.forward(x, tau)
    st = layer.stats()
    ref = o.forward(**inputs, top_k=sh.top_k, tau=tau)
    assert st["n_touched"] == len(np.unique(ref.topk_idx))
    band = int((np.abs(ref.score - tau) <= pu.BAND_REL * tau).sum())
    assert abs(st["n_active"] - int(ref.active.sum())) <= band
    uni = 0
    for e in np.unique(ref.topk_idx):
        rows = np.argwhere(ref.topk_idx == e)
        uni += int(np.any(ref.active[rows[:, 0], rows[:, 1]], axis=0).sum())
    assert abs(st["n_union"] - uni) <= band
    d, f = sh.d_model, sh.d_ff
    want = st["n_touched"] * d * f * 2 + 4 * d * st["n_union"] + sh.n_experts * d * 2 + 4 * T * d
    assert st["alg_bytes"] == pytest.approx(want)


@pytest.mark.parametrize("dims", [
    dict(d=264, E=4, f=32, k=4, S=0, T=9),     # E == k, one chunk, d not a multiple of 256
    dict(d=64, E=16, f=96, k=1, S=1, T=37),    # top-1, ragged token count
    dict(d=128, E=1024, f=64, k=2, S=0, T=5),  # the largest expert count
    dict(d=2048, E=8, f=64, k=2, S=3, T=40),   # many shared experts, T == max_tokens
])
def test_edge_shapes(o, dims):
    sh = mi.custom_shape(dims["d"], dims["E"], dims["f"], dims["k"], dims["S"])
    W = mi.make_weights(sh, device="cuda")
    from intra_expert_activation_router_b200 import MoESparseLayer
    layer = MoESparseLayer.from_weights(W, sh.top_k, max_tokens=dims["T"])
    x = mi.make_x(sh, dims["T"], device="cuda")
    inputs = oracle.layer_inputs(W, x)
    tau = pu.calibrate(o, inputs, sh.top_k, 0.7)
    out = layer.forward(x, tau)
    idx, w = layer.router(x)
    lists, cnt = layer.active_lists(x, tau)
    torch.cuda.synchronize()
    ref = o.forward(**inputs, top_k=sh.top_k, tau=tau)
    tie = pu.check_router(ref, idx.cpu().numpy(), w.cpu().numpy(), sh.top_k)
    flipped, _, gmask = pu.check_active(ref, tau, lists.cpu().numpy().view(np.uint16), cnt.cpu().numpy(), tie)
    pu.check_output(pu.expected_under_gpu_mask(o, inputs, sh.top_k, tau, ref, gmask, flipped, tie), out, tie)
    layer.close()


def test_argument_errors_live_handle():
    import intra_expert_activation_router_b200 as m
    sh = mi.SHAPES["tiny"]
    layer, W, host = layer_for("tiny", max_tokens=32)
    x = mi.make_x(sh, 4, device="cuda")
    out = torch.empty_like(x)
    for T in (0, -1, 33):
        with pytest.raises(m.MoeError) as ei:
            m.moe_sparse_forward(layer.h, x, T, 1.0, out)
        assert ei.value.code == m.MOE_EINVAL
    with pytest.raises(m.MoeError) as ei:
        m.moe_sparse_forward(layer.h, x, 4, float("nan"), out)
    assert ei.value.code == m.MOE_EINVAL
    with pytest.raises(m.MoeError) as ei:
        m.moe_sparse_forward(layer.h, x.data_ptr() + 2, 4, 1.0, out)
    assert ei.value.code == m.MOE_EALIGN
    with pytest.raises(m.MoeError) as ei:
        m.moe_sparse_forward(layer.h, x, 4, 1.0, x)
    assert ei.value.code == m.MOE_EINVAL
    with pytest.raises(m.MoeError) as ei:
        m.moe_set_path(layer.h, 7)
    assert ei.value.code == m.MOE_EINVAL
    # the layer class rejects an output it cannot fill, before any launch
    for bad in (torch.empty(3, sh.d_model, dtype=torch.bfloat16, device="cuda"),
                torch.empty(4, sh.d_model, dtype=torch.float32, device="cuda"),
                torch.empty(4, sh.d_model, dtype=torch.bfloat16),
                torch.empty(sh.d_model, 4, dtype=torch.bfloat16, device="cuda").t()):
        with pytest.raises(ValueError):
            layer.forward(x, 1.0, out=bad)
    # the handle still works after the rejected calls
    layer.forward(x, 1.0)
    torch.cuda.synchronize()
    # destroyed handles are rejected, not dereferenced
    h = m.moe_sparse_create(dict(w_router=W.w_router, w_gate=W.w_gate, w_up=W.w_up, w_down=W.w_down,
                                 ws_gate=W.ws_gate, ws_up=W.ws_up, ws_down=W.ws_down),
                            sh.n_experts, sh.top_k, sh.d_model, sh.d_ff, sh.n_shared, 8)
    m.moe_sparse_destroy(h)
    with pytest.raises(m.MoeError) as ei:
        m.moe_sparse_forward(h, x, 4, 1.0, out)
    assert ei.value.code == m.MOE_EHANDLE


def _rank_case(o, layer, inputs, x, top_k, budget, tau_s=0.0):
    """One rank-budget forward (and its debug lists) against the oracle."""
    out = layer.forward(x, 0.5)   # tau is unused for the routed experts under a budget
    out_dbg = torch.empty_like(x)
    lists, cnt = layer.active_lists(x, 0.5, out=out_dbg)
    idx, w = layer.router(x)
    torch.cuda.synchronize()
    ref = o.forward_budget(**inputs, top_k=top_k, budget=budget, nthreads=NTHREADS, tau_shared=tau_s)
    tie = pu.check_router(ref, idx.cpu().numpy(), w.cpu().numpy(), top_k)
    f = ref.score.shape[2]
    gmask = pu.gpu_mask_from_lists(lists.cpu().numpy().view(np.uint16), cnt.cpu().numpy(), f)
    differ, want = pu.check_rank_mask(o, ref.score, budget, gmask, tie)
    assert np.array_equal(ref.active.astype(bool)[~tie], want[~tie])
    y = ref.y.copy()
    rows = np.where(differ)[0]
    if rows.size:   # a near-equal pair of scores ordered the other way: the layer under the GPU's choice
        sub = dict(inputs)
        sub["x"] = inputs["x"][rows]
        y[rows] = o.forward(**sub, top_k=top_k, tau=0.0, active=gmask[rows], nthreads=NTHREADS,
                            tau_shared=tau_s).y
    pu.check_output(y, out, tie)
    pu.check_output(y, out_dbg, tie)
    return gmask, ref


@pytest.mark.parametrize("name,T,frac", [("tiny", 16, 0.1), ("olmoe", 1, 0.1), ("olmoe", 4, 0.1),
                                         ("olmoe", 16, 0.1), ("olmoe", 40, 0.05), ("dsv2lite", 8, 0.1),
                                         ("large", 1, 0.02)])
def test_rank_budget(o, name, T, frac):
    """Per-pair rank budget (each routed pair keeps its r highest scores):
    exact counts, a valid selection under the oracle's scores, and the layer
    output against the oracle under that selection; in-kernel-routing sizes,
    a token-tile size (40) and shapes with shared experts."""
    import intra_expert_activation_router_b200 as m
    sh = mi.SHAPES[name]
    layer, W, host = layer_for(name)
    x = mi.make_x(sh, T, device="cuda")
    inputs = dict(host)
    inputs["x"] = mi.bf16_bits(x)
    budget = max(1, int(round(frac * sh.d_ff)))
    layer.set_rank_budget(budget)
    try:
        _rank_case(o, layer, inputs, x, sh.top_k, budget)
        st = layer.stats()
        assert st["path"] == m.MOE_PATH_SPARSE and st["device_error"] == 0
    finally:
        layer.set_rank_budget(-1)


@pytest.mark.parametrize("name,T", [("olmoe", 16), ("dsv2lite", 8)])
def test_rank_budget_deterministic(o, name, T):
    """The rank budget's two passes (general kernel instantiation) with the
    deterministic combine: oracle parity under the GPU's selection, and
    repeats bit-identical."""
    sh = mi.SHAPES[name]
    layer, W, host = layer_for(name)
    x = mi.make_x(sh, T, device="cuda")
    inputs = dict(host)
    inputs["x"] = mi.bf16_bits(x)
    budget = max(1, int(round(0.1 * sh.d_ff)))
    layer.set_rank_budget(budget)
    layer.set_deterministic(True)
    try:
        _rank_case(o, layer, inputs, x, sh.top_k, budget)
        reps = [layer.forward(x, 0.5).clone() for _ in range(3)]
        torch.cuda.synchronize()
        assert layer.stats()["deterministic"] == 1 and layer.stats()["device_error"] == 0
        for u in reps[1:]:
            assert torch.equal(u, reps[0])
    finally:
        layer.set_deterministic(False)
        layer.set_rank_budget(-1)


def test_rank_budget_edges_and_shared_threshold(o):
    """Budget 0 (the shared experts alone), budget = d_ff and above (the
    unmasked layer), a looser shared threshold beside the budget, the dense
    path refused, and the threshold restored afterwards."""
    import intra_expert_activation_router_b200 as m
    sh = mi.SHAPES["dsv2lite"]
    layer, W, host = layer_for("dsv2lite")
    T = 8
    x = mi.make_x(sh, T, device="cuda")
    inputs = dict(host)
    inputs["x"] = mi.bf16_bits(x)
    try:
        for budget in (0, sh.d_ff, sh.d_ff + 100):
            layer.set_rank_budget(budget)
            gmask, ref = _rank_case(o, layer, inputs, x, sh.top_k, budget)
            assert int(gmask.sum()) == T * sh.top_k * min(budget, sh.d_ff)
        r_inf = o.forward(**inputs, top_k=sh.top_k, tau=math.inf, nthreads=NTHREADS, want_scores=False)
        layer.set_rank_budget(0)
        pu.check_output(r_inf.y, layer.forward(x, 0.5))
        r0 = o.forward(**inputs, top_k=sh.top_k, tau=math.inf, nthreads=NTHREADS)
        tau_s = pu.threshold_off_scores(r0.score_shared, 0.5)
        layer.set_shared_tau(tau_s)
        layer.set_rank_budget(141)
        _rank_case(o, layer, inputs, x, sh.top_k, 141, tau_s)
        layer.set_path(m.MOE_PATH_DENSE)
        with pytest.raises(m.MoeError):
            layer.forward(x, 0.5)
        layer.set_path(m.MOE_PATH_AUTO)
        layer.set_rank_budget(-1)
        layer.set_shared_tau(0.0)
        tau = pu.calibrate(o, inputs, sh.top_k, 0.9, NTHREADS)
        ref = o.forward(**inputs, top_k=sh.top_k, tau=tau, nthreads=NTHREADS)
        out = layer.forward(x, tau)
        lists, cnt = layer.active_lists(x, tau)
        torch.cuda.synchronize()
        tie = np.zeros(T, bool)
        flipped, _, gm = pu.check_active(ref, tau, lists.cpu().numpy().view(np.uint16), cnt.cpu().numpy(), tie)
        pu.check_output(pu.expected_under_gpu_mask(o, inputs, sh.top_k, tau, ref, gm, flipped, tie, NTHREADS), out)
    finally:
        layer.set_rank_budget(-1)
        layer.set_shared_tau(0.0)
        layer.set_path(m.MOE_PATH_AUTO)


def test_rank_budget_exact_ties():
    """Exact ties: gate columns repeated four times give four identical scores
    per neuron group, and a zero token scores 0 everywhere; the selection must
    keep the lower indices of a tied group first (checked on the GPU's own
    mask, no tolerance), and the zero token keeps neurons 0..r-1."""
    import intra_expert_activation_router_b200 as m
    sh = mi.SHAPES["tiny"]
    W = mi.make_weights(sh, device="cuda")
    q = sh.d_ff // 4
    W.w_gate.copy_(W.w_gate[:, :, :q].repeat(1, 1, 4))
    layer = m.MoESparseLayer.from_weights(W, sh.top_k, max_tokens=64)
    try:
        for T in (16, 40):
            x = mi.make_x(sh, T, device="cuda")
            x[1] = 0
            for budget in (1, 6, 50, 130):   # 6, 50, 130 cut inside a group of four
                layer.set_rank_budget(budget)
                layer.forward(x, 0.5)
                lists, cnt = layer.active_lists(x, 0.5)
                torch.cuda.synchronize()
                g = pu.gpu_mask_from_lists(lists.cpu().numpy().view(np.uint16), cnt.cpu().numpy(), sh.d_ff)
                assert np.all(g.sum(axis=2) == budget)
                grp = g.reshape(T, sh.top_k, 4, q)   # [.., member, j]: member m is neuron m*q + j
                assert np.all(grp[:, :, 1:, :] <= grp[:, :, :-1, :]), "a tied group kept a higher index first"
                assert np.all(g[1, :, :budget]) and not np.any(g[1, :, budget:])
                assert layer.stats()["device_error"] == 0
    finally:
        layer.close()


@pytest.mark.parametrize("name,T,gamma,path", [("tiny", 16, 1.0, "sparse"), ("olmoe", 16, 1.0, "sparse"),
                                               ("olmoe", 16, 1.5, "sparse"), ("olmoe", 40, 1.0, "sparse"),
                                               ("olmoe", 256, 1.25, "dense"), ("dsv2lite", 32, 1.0, "sparse"),
                                               ("dsv2lite", 32, 1.0, "dense")])
def test_capacity_drop(o, name, T, gamma, path):
    """Capacity-aware token drop: each expert keeps at most ceil(gamma T k / E)
    pairs, the ones with the largest routing weight.  The kept pairs are
    compared with the oracle's exactly, except experts whose cut falls between
    weights within 1e-6 of each other (fp32 softmax against the oracle's
    rounding); the output against the oracle under the GPU's kept set and mask."""
    import intra_expert_activation_router_b200 as m
    sh = mi.SHAPES[name]
    layer, W, host = layer_for(name)
    x = mi.make_x(sh, T, device="cuda")
    inputs = dict(host)
    inputs["x"] = mi.bf16_bits(x)
    g32 = float(np.float32(gamma))
    C = oracle.Oracle.capacity(g32, T, sh.top_k, sh.n_experts)
    assert 0 < C < T
    tau = pu.calibrate(o, inputs, sh.top_k, 0.9, NTHREADS)
    ref = o.forward_capacity(**inputs, top_k=sh.top_k, tau=tau, gamma=g32, nthreads=NTHREADS)
    layer.set_capacity(gamma)
    try:
        layer.set_path(m.MOE_PATH_SPARSE if path == "sparse" else m.MOE_PATH_DENSE)
        out = layer.forward(x, tau)
        st = layer.stats()
        assert st["capacity"] == C and st["device_error"] == 0
        idx, w = layer.router(x)
        torch.cuda.synchronize()
        tie = pu.check_router(ref, idx.cpu().numpy(), w.cpu().numpy(), sh.top_k)
        keep_ref = ref.active.any(axis=2)
        # experts whose C-th and (C+1)-th weights are within 1e-6: either order is right
        wr = ref.topk_w.astype(np.float32)
        amb_e = set()
        for e in np.unique(ref.topk_idx):
            ws_ = np.sort(wr[ref.topk_idx == e])[::-1]
            if ws_.size > C and ws_[C - 1] - ws_[C] <= 1e-6 * ws_[C - 1]:
                amb_e.add(int(e))
        assert len(amb_e) <= 2, amb_e
        amb = np.isin(ref.topk_idx, list(amb_e))
        if path == "sparse":
            lists, cnt = layer.active_lists(x, tau)
            torch.cuda.synchronize()
            cnt = cnt.cpu().numpy()
            keep_gpu = cnt > 0
            ok = ~amb & ~tie[:, None]
            assert np.array_equal(keep_gpu[ok], keep_ref[ok]), "kept pairs differ"
            flipped, _, gm = pu.check_active(ref, tau, lists.cpu().numpy().view(np.uint16), cnt, tie | amb.any(axis=1))
            y = pu.expected_under_gpu_mask(o, inputs, sh.top_k, tau, ref, gm, flipped, tie, NTHREADS)
            pu.check_output(y, out, tie | amb.any(axis=1))
        else:
            import dataclasses
            sc = ref.score.copy()
            sc[~keep_ref] = -1.0   # a dropped pair's neurons are never near the threshold
            pu.check_output_any_band_decision(o, inputs, sh.top_k, tau, dataclasses.replace(ref, score=sc), out,
                                              tie | amb.any(axis=1), 1e-5, nthreads=NTHREADS)
        # a large factor drops nothing: the plain layer
        layer.set_capacity(1000.0)
        out2 = layer.forward(x, tau)
        assert layer.stats()["capacity"] == -1
        ref2 = o.forward(**inputs, top_k=sh.top_k, tau=tau, nthreads=NTHREADS)
        if path == "dense":
            pu.check_output_any_band_decision(o, inputs, sh.top_k, tau, ref2, out2, tie, 1e-5, nthreads=NTHREADS)
    finally:
        layer.set_capacity(0.0)
        layer.set_path(m.MOE_PATH_AUTO)


def test_capacity_limits(o):
    """A capacity below T on more than 4096 pairs is refused; gamma <= 0 turns
    the drop off; NaN is rejected."""
    import intra_expert_activation_router_b200 as m
    sh = mi.SHAPES["olmoe"]
    layer, W, host = layer_for("olmoe")
    x = mi.make_x(sh, 1024, device="cuda")
    layer.set_capacity(1.0)
    try:
        with pytest.raises(m.MoeError) as ei:
            layer.forward(x, 1.0)
        assert ei.value.code == m.MOE_ENOTSUP
        layer.set_capacity(-1.0)
        layer.forward(x[:8], 1.0)
        assert layer.stats()["capacity"] == -1
        with pytest.raises(m.MoeError):
            layer.set_capacity(float("nan"))
    finally:
        layer.set_capacity(0.0)
