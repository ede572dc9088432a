"""The allocation-free router entry point, for callers that cannot call
cudaMalloc (servers that reserve all device memory up front in their own
arena, custom operators inside a framework that owns the allocator, paths
that cannot afford an allocation's implicit synchronisation), against the
handle-based router of the same library and against the CPU oracle.

Kept in its own file, collected last, so a failure here comes after every
other test has run.  It creates its own inputs and passes when run alone.
"""
import numpy as np
import pytest
import torch

import moe_inputs as mi
import oracle
from tests import parity_util as pu

pytestmark = pytest.mark.gpu

SHAPES = {
    "tiny": mi.SHAPES["tiny"],
    "olmoe": mi.SHAPES["olmoe"],
    "large": mi.SHAPES["large"],
    # the largest expert count: the selection's 32-bit "taken" mask is full
    "e1024": mi.custom_shape(128, 1024, 32, 8, 0, name="e1024"),
}


@pytest.mark.parametrize("name,T", [("tiny", 16), ("olmoe", 37), ("large", 5), ("e1024", 9)])
def test_noalloc_router_matches_handle_router_and_oracle(name, T):
    import intra_expert_activation_router_b200 as m
    sh = SHAPES[name]
    g = torch.Generator(device="cuda").manual_seed(11 + T)
    w_router = (torch.randn(sh.n_experts, sh.d_model, generator=g, device="cuda") * sh.d_model ** -0.5).to(torch.bfloat16)
    # a handle with the same router (the expert weights do not affect routing)
    f = 32
    zeros = torch.zeros(sh.n_experts, sh.d_model, f, dtype=torch.bfloat16, device="cuda")
    down = torch.zeros(sh.n_experts, f, sh.d_model, dtype=torch.bfloat16, device="cuda")
    h = m.moe_sparse_create(dict(w_router=w_router, w_gate=zeros, w_up=zeros, w_down=down),
                            sh.n_experts, sh.top_k, sh.d_model, f, 0, T)
    try:
        x = mi.make_x(sh, T, device="cuda")
        idx_ref = torch.empty(T, sh.top_k, dtype=torch.int32, device="cuda")
        w_ref = torch.empty(T, sh.top_k, dtype=torch.float32, device="cuda")
        m.moe_debug_router(h, x, T, idx_ref, w_ref)
        torch.cuda.synchronize()
        # the oracle's routing of the same bf16 inputs (near-tie tokens excluded)
        zh = np.zeros((sh.n_experts, sh.d_model, f), np.uint16)
        ref = oracle.load().forward(mi.bf16_bits(x), mi.bf16_bits(w_router), zh, zh,
                                    np.zeros((sh.n_experts, f, sh.d_model), np.uint16),
                                    top_k=sh.top_k, tau=float("inf"), want_scores=False)
        for _call in range(2):   # two calls in a row share the fixed scratch
            idx = torch.full((T, sh.top_k), -1, dtype=torch.int32, device="cuda")
            w = torch.full((T, sh.top_k), -1.0, dtype=torch.float32, device="cuda")
            m.moe_router_topk_noalloc(x, T, w_router, sh.n_experts, sh.d_model, sh.top_k, idx, w)
            torch.cuda.synchronize()
            assert torch.equal(idx.cpu(), idx_ref.cpu())
            wr, wn = w_ref.cpu().numpy(), w.cpu().numpy()
            assert np.abs(wr - wn).max() <= 1e-5 + 1e-4 * np.abs(wr).max()
            tie = pu.check_router(ref, idx.cpu().numpy(), wn, sh.top_k)
            assert tie.sum() <= 1
    finally:
        m.moe_sparse_destroy(h)


def test_noalloc_router_rejects_oversized():
    import intra_expert_activation_router_b200 as m
    x = torch.zeros(8, 16, dtype=torch.bfloat16, device="cuda")
    wr = torch.zeros(1024, 16, dtype=torch.bfloat16, device="cuda")
    idx = torch.zeros(8, 1, dtype=torch.int32, device="cuda")
    w = torch.zeros(8, 1, dtype=torch.float32, device="cuda")
    # 4096 tokens x 1024 experts of fp32 logits exceed the fixed scratch: rejected before launch
    rc = m.raw_call("moe_router_topk_noalloc", x.data_ptr(), 4096, wr.data_ptr(), 1024, 16, 1,
                    idx.data_ptr(), w.data_ptr(), None)
    assert rc == m.MOE_ENOTSUP
