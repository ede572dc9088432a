"""The allocation-free router entry point (for callers that cannot call
cudaMalloc: servers with a pre-reserved memory arena, custom operators inside a
framework that owns the allocator, latency-critical paths) against the
handle-based router of the same library.

Kept in its own file, collected last, so a failure here comes after every
other test has run.  It creates its own inputs and passes when run alone.
"""
import numpy as np
import pytest
import torch

import moe_inputs as mi

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,T", [("tiny", 16), ("olmoe", 37), ("large", 5)])
def test_noalloc_router_matches_handle_router(name, T):
    import intra_expert_activation_router_b200 as m
    sh = mi.SHAPES[name]
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
        for _call in range(2):   # two calls in a row share the fixed scratch
            idx = torch.full((T, sh.top_k), -1, dtype=torch.int32, device="cuda")
            w = torch.full((T, sh.top_k), -1.0, dtype=torch.float32, device="cuda")
            m.moe_router_topk_noalloc(x, T, w_router, sh.n_experts, sh.d_model, sh.top_k, idx, w)
            torch.cuda.synchronize()
            assert torch.equal(idx.cpu(), idx_ref.cpu())
            wr, wn = w_ref.cpu().numpy(), w.cpu().numpy()
            assert np.abs(wr - wn).max() <= 1e-5 + 1e-4 * np.abs(wr).max()
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
