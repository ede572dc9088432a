"""Routed-expert MoE layer with intra-expert activation sparsity, for B200 (sm_100a).

The computation runs in libmoe_sparse.so (hand-written CUDA behind the C ABI
in include/moe_sparse.h); this package is its ctypes binding plus a small
convenience class.  The library is loaded on first use of any binding name;
if it is missing that access raises ImportError -- there is no fallback.
The build module (``python -m intra_expert_activation_router_b200.build``)
does not need the library.
"""
_BINDING_NAMES = {
    "EXPORTED", "LIB_PATH", "MOE_EALIGN", "MOE_ECUDA", "MOE_EDEVICE", "MOE_EHANDLE", "MOE_EINVAL",
    "MOE_ENOMEM", "MOE_ENOTSUP", "MOE_OK", "MOE_PATH_AUTO", "MOE_PATH_DENSE", "MOE_PATH_SPARSE",
    "MoeError", "moe_debug_active", "moe_debug_router", "moe_dense_forward", "moe_query_stats",
    "moe_set_path", "moe_set_t_star", "moe_sparse_create", "moe_sparse_destroy",
    "moe_sparse_forward", "moe_sparse_forward_host", "moe_strerror", "raw_call",
    "moe_calibrate_tau", "moe_set_launch_events", "moe_set_trace", "moe_router_topk_noalloc",
    "moe_debug_inject", "MOE_INJECT_NONE", "MOE_INJECT_WITHHOLD_ITEMS", "moe_set_fused_router",
    "moe_set_shared_tau", "moe_calibrate_tau_shared", "moe_tune_t_star", "moe_set_rank_budget", "moe_set_capacity",
    "moe_set_deterministic",
}


def __getattr__(name):
    if name in _BINDING_NAMES:
        from . import _binding
        return getattr(_binding, name)
    if name == "MoESparseLayer":
        from .layer import MoESparseLayer
        return MoESparseLayer
    raise AttributeError(name)


__all__ = sorted(_BINDING_NAMES | {"MoESparseLayer"})
