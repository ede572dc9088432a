"""Failure detection without a GPU fault, trap or hang.

* A bounded device wait is made to run out: a test-only hook makes the expert
  kernel's gate lane publish no work item (and issue no copy), so the other
  agents' bounded polls for work expire.  The kernel must record its error
  code and return; moe_query_stats must report MOE_EDEVICE; the next forward
  on the same handle must match the oracle again.
* Host-side allocation failure: MOE_INJECT_ALLOC_FAIL makes a named device
  allocation report failure; the call returns MOE_ENOMEM and leaks nothing.
"""
import numpy as np
import pytest
import torch

import moe_inputs as mi
import oracle
from tests import parity_util as pu

pytestmark = pytest.mark.gpu

GET_ITEM_TIMEOUT = 50   # the code a consumer records when no work item is published in time


@pytest.fixture(scope="module")
def o():
    return oracle.load()


def _check_against_oracle(o, W, sh, x, tau, out):
    inputs = oracle.layer_inputs(W, x)
    ref = o.forward(**inputs, top_k=sh.top_k, tau=tau)
    # band tokens may legitimately differ: compare the rest (the full band
    # treatment is in the parity tests; here the point is recovery)
    band = np.any(np.abs(ref.score - tau) <= pu.BAND_REL * tau, axis=(1, 2))
    tie = pu.near_tie_tokens(ref.logits, sh.top_k)
    pu.check_output(ref.y, out, band | tie)


@pytest.mark.parametrize("name,T", [("tiny", 16), ("olmoe", 40)])
def test_bounded_wait_runs_out_and_handle_recovers(o, name, T):
    import intra_expert_activation_router_b200 as m
    sh = mi.SHAPES[name]
    W = mi.make_weights(sh, device="cuda")
    layer = m.MoESparseLayer.from_weights(W, sh.top_k, max_tokens=64)
    layer.set_path(m.MOE_PATH_SPARSE)   # T = 40 would otherwise take the dense branch
    try:
        x = mi.make_x(sh, T, device="cuda")
        tau = layer.calibrate_tau(x, 0.9)
        good = layer.forward(x, tau).clone()
        assert layer.stats()["rc"] == m.MOE_OK
        # 1. the injected forward: its waits run out, it reports, its output is zero
        m.moe_debug_inject(layer.h, m.MOE_INJECT_WITHHOLD_ITEMS)
        bad = layer.forward(x, tau)
        torch.cuda.synchronize()
        st = layer.stats()
        assert st["rc"] == m.MOE_EDEVICE and st["device_error"] == GET_ITEM_TIMEOUT
        assert not bad.float().abs().sum().item()
        # 2. the error was read and cleared; the next forward is correct
        again = layer.forward(x, tau)
        torch.cuda.synchronize()
        assert layer.stats()["rc"] == m.MOE_OK
        _check_against_oracle(o, W, sh, x, tau, again)
        d = (again.float() - good.float()).abs()
        assert bool((d <= good.float().abs() * 2.0 ** -7 + 1e-6).all())
        # 3. an error is kept across later forwards until it is read
        m.moe_debug_inject(layer.h, m.MOE_INJECT_WITHHOLD_ITEMS)
        layer.forward(x, tau)
        later = layer.forward(x, tau)
        torch.cuda.synchronize()
        st = layer.stats()
        assert st["rc"] == m.MOE_EDEVICE and st["device_error"] == GET_ITEM_TIMEOUT
        _check_against_oracle(o, W, sh, x, tau, later)
        assert layer.stats()["rc"] == m.MOE_OK
        # 4. an injection can be cancelled
        m.moe_debug_inject(layer.h, m.MOE_INJECT_WITHHOLD_ITEMS)
        m.moe_debug_inject(layer.h, m.MOE_INJECT_NONE)
        layer.forward(x, tau)
        assert layer.stats()["rc"] == m.MOE_OK
        with pytest.raises(m.MoeError):
            m.moe_debug_inject(layer.h, 7)
    finally:
        layer.close()


def test_allocation_failure_injection(o, monkeypatch):
    import intra_expert_activation_router_b200 as m
    sh = mi.SHAPES["olmoe"]   # 1 GB of repacked weights: a leak would show
    W = mi.make_weights(sh, device="cuda")
    warm = m.MoESparseLayer.from_weights(W, sh.top_k, max_tokens=16)   # loads the module
    warm.close()
    torch.cuda.synchronize()
    for what in ("weights", "workspace"):
        monkeypatch.setenv("MOE_INJECT_ALLOC_FAIL", what)
        free0 = torch.cuda.mem_get_info()[0]
        with pytest.raises(m.MoeError) as ei:
            m.MoESparseLayer.from_weights(W, sh.top_k, max_tokens=16)
        assert ei.value.code == m.MOE_ENOMEM
        torch.cuda.synchronize()
        assert abs(torch.cuda.mem_get_info()[0] - free0) <= (64 << 20), what
    monkeypatch.setenv("MOE_INJECT_ALLOC_FAIL", "scores")
    layer = m.MoESparseLayer.from_weights(W, sh.top_k, max_tokens=16)
    try:
        x = mi.make_x(sh, 16, device="cuda")
        with pytest.raises(m.MoeError) as ei:
            layer.calibrate_tau(x, 0.9)
        assert ei.value.code == m.MOE_ENOMEM
        monkeypatch.setenv("MOE_INJECT_ALLOC_FAIL", "rank")
        with pytest.raises(m.MoeError) as ei:   # the rank budget's buffers: the threshold stays in force
            layer.set_rank_budget(50)
        assert ei.value.code == m.MOE_ENOMEM
        monkeypatch.setenv("MOE_INJECT_ALLOC_FAIL", "deterministic")
        with pytest.raises(m.MoeError) as ei:   # the deterministic combine's rows: atomics stay in force
            layer.set_deterministic(True)
        assert ei.value.code == m.MOE_ENOMEM
        monkeypatch.delenv("MOE_INJECT_ALLOC_FAIL")
        tau = layer.calibrate_tau(x, 0.9)   # the handle is still usable
        out = layer.forward(x, tau)
        torch.cuda.synchronize()
        assert layer.stats()["rc"] == m.MOE_OK and layer.stats()["deterministic"] == 0
        _check_against_oracle(o, W, sh, x, tau, out)
    finally:
        layer.close()
