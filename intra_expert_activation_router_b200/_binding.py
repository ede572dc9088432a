"""ctypes binding of libmoe_sparse.so -- argument marshalling only.

Every function here has the name and argument order of the C entry point in
include/moe_sparse.h.  Tensor arguments may be torch tensors (their
data_ptr() is passed) or plain integer addresses; a stream may be a
torch.cuda.Stream, an integer cudaStream_t or None (the current torch
stream when torch has CUDA, else the legacy default stream).  A nonzero
return code raises MoeError.  All arithmetic runs in the CUDA library; if
the library is missing this module raises at import, there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_sparse.so")

MOE_OK = 0
MOE_EINVAL = -1
MOE_ENOMEM = -2
MOE_ECUDA = -3
MOE_EALIGN = -4
MOE_EHANDLE = -5
MOE_EDEVICE = -6
MOE_ENOTSUP = -7

MOE_INJECT_NONE = 0
MOE_INJECT_WITHHOLD_ITEMS = 1

MOE_PATH_AUTO = 0
MOE_PATH_SPARSE = 1
MOE_PATH_DENSE = 2


class MoeError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {moe_strerror(code)} ({code})")


class moe_weights(ctypes.Structure):
    _fields_ = [("w_router", ctypes.c_void_p), ("w_gate", ctypes.c_void_p),
                ("w_up", ctypes.c_void_p), ("w_down", ctypes.c_void_p),
                ("ws_gate", ctypes.c_void_p), ("ws_up", ctypes.c_void_p),
                ("ws_down", ctypes.c_void_p)]


class moe_stats(ctypes.Structure):
    _fields_ = [("path", ctypes.c_int), ("n_tokens", ctypes.c_int), ("n_touched", ctypes.c_int),
                ("t_star", ctypes.c_int), ("n_active", ctypes.c_longlong),
                ("n_union", ctypes.c_longlong), ("alg_bytes", ctypes.c_double),
                ("dense_bytes", ctypes.c_double), ("device_error", ctypes.c_int),
                ("fused_router", ctypes.c_int),
                ("capacity", ctypes.c_int), ("deterministic", ctypes.c_int)]

    def as_dict(self):
        return {n: getattr(self, n) for n, _ in self._fields_}


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing; build it with "
                          "`python -m intra_expert_activation_router_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    sig = {
        "moe_sparse_create": (I, [ctypes.POINTER(moe_weights), I, I, I, I, I, I, ctypes.POINTER(P)]),
        "moe_sparse_forward": (I, [P, P, I, F, P, P]),
        "moe_dense_forward": (I, [P, P, I, P, P]),
        "moe_sparse_forward_host": (I, [P, P, I, F, P, P]),
        "moe_sparse_destroy": (None, [P]),
        "moe_set_path": (I, [P, I]),
        "moe_set_t_star": (I, [P, I]),
        "moe_debug_router": (I, [P, P, I, P, P, P]),
        "moe_debug_active": (I, [P, P, I, F, P, P, P, P]),
        "moe_query_stats": (I, [P, ctypes.POINTER(moe_stats)]),
        "moe_calibrate_tau": (I, [P, P, I, ctypes.c_double, ctypes.POINTER(F), P]),
        "moe_set_launch_events": (I, [P, ctypes.POINTER(P), I]),
        "moe_set_trace": (I, [P, P, ctypes.c_longlong]),
        "moe_router_topk_noalloc": (I, [P, I, P, I, I, I, P, P, P]),
        "moe_debug_inject": (I, [P, I]),
        "moe_set_fused_router": (I, [P, I]),
        "moe_set_shared_tau": (I, [P, F]),
        "moe_set_rank_budget": (I, [P, I]),
        "moe_set_capacity": (I, [P, F]),
        "moe_set_deterministic": (I, [P, I]),
        "moe_calibrate_tau_shared": (I, [P, P, I, ctypes.c_double, ctypes.POINTER(F), P]),
        "moe_tune_t_star": (I, [P, P, I, F, ctypes.POINTER(I), P]),
        "moe_strerror": (ctypes.c_char_p, [I]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()
EXPORTED = ("moe_sparse_create", "moe_sparse_forward", "moe_dense_forward",
            "moe_sparse_forward_host", "moe_sparse_destroy", "moe_set_path", "moe_set_t_star",
            "moe_debug_router", "moe_debug_active", "moe_query_stats", "moe_strerror",
            "moe_calibrate_tau", "moe_set_launch_events", "moe_set_trace", "moe_router_topk_noalloc",
            "moe_debug_inject", "moe_set_fused_router", "moe_set_shared_tau", "moe_calibrate_tau_shared",
            "moe_tune_t_star", "moe_set_rank_budget", "moe_set_capacity", "moe_set_deterministic")


def _addr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if hasattr(t, "data_ptr"):
        return t.data_ptr()
    raise TypeError(f"expected a tensor or an address, got {type(t).__name__}")


def _stream(s):
    if s is None:
        try:
            import torch
            if torch.cuda.is_available():
                return torch.cuda.current_stream().cuda_stream
        except ImportError:
            pass
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(rc, where):
    if rc != MOE_OK:
        raise MoeError(rc, where)


def moe_strerror(code: int) -> str:
    return _lib.moe_strerror(int(code)).decode()


def moe_sparse_create(weights: dict, E: int, top_k: int, d_model: int, d_ff: int,
                      n_shared: int, max_tokens: int = 0) -> int:
    """weights: dict with w_router, w_gate, w_up, w_down[, ws_gate, ws_up, ws_down]."""
    w = moe_weights(*[_addr(weights.get(n)) for n, _ in moe_weights._fields_])
    h = ctypes.c_void_p()
    _check(_lib.moe_sparse_create(ctypes.byref(w), E, top_k, d_model, d_ff, n_shared,
                                  max_tokens, ctypes.byref(h)), "moe_sparse_create")
    return h.value


def moe_sparse_forward(h, x, T: int, tau: float, out, stream=None):
    _check(_lib.moe_sparse_forward(h, _addr(x), T, tau, _addr(out), _stream(stream)),
           "moe_sparse_forward")


def moe_dense_forward(h, x, T: int, out, stream=None):
    _check(_lib.moe_dense_forward(h, _addr(x), T, _addr(out), _stream(stream)), "moe_dense_forward")


def moe_sparse_forward_host(h, x_host, T: int, tau: float, out_host, stream=None):
    _check(_lib.moe_sparse_forward_host(h, _addr(x_host), T, tau, _addr(out_host),
                                        _stream(stream)), "moe_sparse_forward_host")


def moe_sparse_destroy(h):
    _lib.moe_sparse_destroy(h)


def moe_set_path(h, path: int):
    _check(_lib.moe_set_path(h, path), "moe_set_path")


def moe_set_t_star(h, t_star: int):
    _check(_lib.moe_set_t_star(h, t_star), "moe_set_t_star")


def moe_debug_router(h, x, T: int, idx_out, w_out, stream=None):
    _check(_lib.moe_debug_router(h, _addr(x), T, _addr(idx_out), _addr(w_out), _stream(stream)),
           "moe_debug_router")


def moe_debug_active(h, x, T: int, tau: float, idx_out, cnt_out, out=None, stream=None):
    _check(_lib.moe_debug_active(h, _addr(x), T, tau, _addr(idx_out), _addr(cnt_out), _addr(out),
                                 _stream(stream)), "moe_debug_active")


def moe_query_stats(h) -> dict:
    st = moe_stats()
    rc = _lib.moe_query_stats(h, ctypes.byref(st))
    d = st.as_dict()
    if rc not in (MOE_OK, MOE_EDEVICE):
        raise MoeError(rc, "moe_query_stats")
    d["rc"] = rc
    return d


def moe_calibrate_tau(h, x, T: int, sparsity: float, stream=None) -> float:
    tau = ctypes.c_float()
    _check(_lib.moe_calibrate_tau(h, _addr(x), T, float(sparsity), ctypes.byref(tau), _stream(stream)),
           "moe_calibrate_tau")
    return tau.value


def moe_set_launch_events(h, events):
    """events: three cudaEvent_t handles (ints or torch.cuda.Event), or None to stop."""
    if not events:
        _check(_lib.moe_set_launch_events(h, None, 0), "moe_set_launch_events")
        return
    hs = [e if isinstance(e, int) else e.cuda_event for e in events]
    arr = (ctypes.c_void_p * len(hs))(*hs)
    _check(_lib.moe_set_launch_events(h, arr, len(hs)), "moe_set_launch_events")


def moe_set_trace(h, buf, nbytes: int = 0):
    """buf: an int64 CUDA tensor (or address) receiving phase timestamps; None turns tracing off."""
    if buf is None:
        _check(_lib.moe_set_trace(h, None, 0), "moe_set_trace")
        return
    n = nbytes or (buf.numel() * buf.element_size())
    _check(_lib.moe_set_trace(h, _addr(buf), n), "moe_set_trace")


def moe_router_topk_noalloc(x, T: int, w_router, E: int, d_model: int, top_k: int, idx_out, w_out,
                            stream=None):
    """Router softmax top-k without a handle or any allocation (fixed device scratch)."""
    _check(_lib.moe_router_topk_noalloc(_addr(x), T, _addr(w_router), E, d_model, top_k, _addr(idx_out),
                                        _addr(w_out), _stream(stream)), "moe_router_topk_noalloc")


def moe_set_shared_tau(h, tau_shared: float):
    _check(_lib.moe_set_shared_tau(h, float(tau_shared)), "moe_set_shared_tau")


def moe_set_capacity(h, gamma: float):
    _check(_lib.moe_set_capacity(h, float(gamma)), "moe_set_capacity")


def moe_set_deterministic(h, enable: bool):
    _check(_lib.moe_set_deterministic(h, 1 if enable else 0), "moe_set_deterministic")


def moe_set_rank_budget(h, r: int):
    _check(_lib.moe_set_rank_budget(h, int(r)), "moe_set_rank_budget")


def moe_calibrate_tau_shared(h, x, T: int, sparsity: float, stream=None) -> float:
    tau = ctypes.c_float()
    _check(_lib.moe_calibrate_tau_shared(h, _addr(x), T, float(sparsity), ctypes.byref(tau), _stream(stream)),
           "moe_calibrate_tau_shared")
    return tau.value


def moe_tune_t_star(h, x, T_max: int, tau: float, stream=None) -> int:
    """Measure both branches at batch sizes up to T_max and set the AUTO switch point; returns it."""
    t = ctypes.c_int()
    _check(_lib.moe_tune_t_star(h, _addr(x), T_max, float(tau), ctypes.byref(t), _stream(stream)),
           "moe_tune_t_star")
    return t.value


def moe_set_fused_router(h, mode: int):
    _check(_lib.moe_set_fused_router(h, int(mode)), "moe_set_fused_router")


def moe_debug_inject(h, kind: int):
    """Test-only fault for the next sparse forward (MOE_INJECT_*)."""
    _check(_lib.moe_debug_inject(h, kind), "moe_debug_inject")


def raw_call(name: str, *args) -> int:
    """Call an entry point with raw ctypes arguments and return its code (for argument tests)."""
    return getattr(_lib, name)(*args)
