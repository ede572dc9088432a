"""CPU oracle of the masked routed-expert MoE layer -- TEST INFRASTRUCTURE.

Only the tests, the smoke check and the benchmark's CPU-baseline leg may use
this package.  The product path (the CUDA library and its Python binding)
never imports it.

The arithmetic lives in ``moe_oracle.c`` (plain fp64 C, see its header for
the definition and the passages it follows).  This module compiles it with
gcc and marshals numpy arrays through ctypes; it adds no arithmetic of its
own except the threshold calibration's choice of population (the scores of
the pairs the router selected), which is stated in ``calibrate_tau``.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
import tempfile
from dataclasses import dataclass

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "moe_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")


def build(src: str = SRC, out: str = LIB, openmp: bool = True) -> str:
    """Compile the oracle C source into a shared library (gcc -O2, OpenMP)."""
    cmd = ["gcc", "-O2", "-std=c11", "-shared", "-fPIC", "-o", out, src, "-lm"]
    if openmp:
        cmd.insert(1, "-fopenmp")
    subprocess.run(cmd, check=True)
    return out


def _needs_build(src, out):
    return not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src)


_P = ctypes.c_void_p


@dataclass
class OracleResult:
    y: np.ndarray            # [T][d] float64
    topk_idx: np.ndarray     # [T][k] int32
    topk_w: np.ndarray       # [T][k] float64
    logits: np.ndarray       # [T][E] float64
    score: np.ndarray | None   # [T][k][f] float64
    active: np.ndarray | None  # [T][k][f] uint8
    score_shared: np.ndarray | None = None   # [T][S][f] float64


class Oracle:
    """ctypes wrapper around one compiled oracle library."""

    def __init__(self, path: str | None = None):
        if path is None:
            path = LIB
            if _needs_build(SRC, LIB):
                build()
        self.path = path
        self._lib = ctypes.CDLL(path)
        f = self._lib.oracle_moe_forward
        f.restype = ctypes.c_int
        f.argtypes = [_P, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                      ctypes.c_int, _P, _P, _P, _P, _P, _P, _P, ctypes.c_float, ctypes.c_float,
                      ctypes.c_int, _P, _P, _P, _P, _P, _P, _P, _P]
        c = self._lib.oracle_calibrate_tau
        c.restype = ctypes.c_double
        c.argtypes = [_P, ctypes.c_long, ctypes.c_double]
        rm = self._lib.oracle_rank_mask
        rm.restype = ctypes.c_int
        rm.argtypes = [_P, ctypes.c_long, ctypes.c_int, ctypes.c_int, _P]
        ck = self._lib.oracle_capacity_keep
        ck.restype = ctypes.c_int
        ck.argtypes = [_P, _P, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, _P]

    @staticmethod
    def _ptr(a):
        return None if a is None else a.ctypes.data_as(ctypes.c_void_p)

    def forward(self, x, w_router, w_gate, w_up, w_down, ws_gate=None, ws_up=None,
                ws_down=None, *, top_k: int, tau: float, want_scores: bool = True,
                nthreads: int = 0, active=None, tau_shared: float = 0.0) -> OracleResult:
        """All weight/x arguments are uint16 numpy arrays of bf16 bits (x @ W layout).

        ``active``: optional [T][top_k][d_ff] mask (nonzero = active) that
        replaces the threshold decision for each (token, rank) pair; ``tau``
        is then unused.  It evaluates the layer under a given decision, e.g.
        the CUDA path's for neurons whose score sits on the threshold.

        ``tau_shared``: shared-expert neurons count iff |silu(g)| >= tau_shared
        (<= 0, the default: every shared neuron)."""
        arrs = [np.ascontiguousarray(a, dtype=np.uint16) if a is not None else None
                for a in (x, w_router, w_gate, w_up, w_down, ws_gate, ws_up, ws_down)]
        x, wr, wg, wu, wd, wsg, wsu, wsd = arrs
        T, d = x.shape
        E = wr.shape[0]
        f = wg.shape[2]
        S = 0 if wsg is None else wsg.shape[0]
        k = int(top_k)
        y = np.zeros((T, d), np.float64)
        idx = np.zeros((T, k), np.int32)
        w = np.zeros((T, k), np.float64)
        lg = np.zeros((T, E), np.float64)
        sc = np.zeros((T, k, f), np.float64) if want_scores else None
        ac = np.zeros((T, k, f), np.uint8) if want_scores else None
        ssh = np.zeros((T, S, f), np.float64) if (want_scores and S > 0) else None
        ain = None
        if active is not None:
            ain = np.ascontiguousarray(np.asarray(active) != 0, dtype=np.uint8)
            if ain.shape != (T, k, f):
                raise ValueError(f"active must be [{T}][{k}][{f}], got {ain.shape}")
        rc = self._lib.oracle_moe_forward(
            self._ptr(x), T, d, f, E, k, S, self._ptr(wr), self._ptr(wg), self._ptr(wu),
            self._ptr(wd), self._ptr(wsg), self._ptr(wsu), self._ptr(wsd),
            ctypes.c_float(tau), ctypes.c_float(tau_shared), int(nthreads), self._ptr(y), self._ptr(idx),
            self._ptr(w), self._ptr(lg), self._ptr(sc), self._ptr(ac), self._ptr(ain), self._ptr(ssh))
        if rc != 0:
            raise RuntimeError(f"oracle_moe_forward failed ({rc})")
        return OracleResult(y, idx, w, lg, sc, ac, ssh)

    def rank_mask(self, scores: np.ndarray, budget: int) -> np.ndarray:
        """Per pair (the last axis holds one pair's f scores), 1 for the
        ``budget`` largest scores compared in float, ties to the lower index,
        NaN never kept; see ``oracle_rank_mask``."""
        s = np.ascontiguousarray(scores, dtype=np.float64)
        f = s.shape[-1]
        out = np.zeros(s.shape, np.uint8)
        rc = self._lib.oracle_rank_mask(self._ptr(s), s.size // f, f, int(budget), self._ptr(out))
        if rc != 0:
            raise RuntimeError(f"oracle_rank_mask failed ({rc})")
        return out

    def forward_budget(self, x, w_router, w_gate, w_up, w_down, ws_gate=None, ws_up=None,
                       ws_down=None, *, top_k: int, budget: int, nthreads: int = 0,
                       tau_shared: float = 0.0) -> OracleResult:
        """The layer with a rank budget in place of the routed threshold: each
        selected pair keeps its ``budget`` highest-scoring neurons
        (``rank_mask`` of its scores); the shared experts keep their
        ``tau_shared`` rule.  Composition of three oracle calls: the scores
        (forward at tau = 0), the rank mask, the layer under that mask."""
        args = (x, w_router, w_gate, w_up, w_down, ws_gate, ws_up, ws_down)
        first = self.forward(*args, top_k=top_k, tau=0.0, nthreads=nthreads, tau_shared=tau_shared)
        mask = self.rank_mask(first.score, budget)
        res = self.forward(*args, top_k=top_k, tau=0.0, nthreads=nthreads, active=mask,
                           tau_shared=tau_shared)
        res.score = first.score
        return res

    @staticmethod
    def capacity(gamma: float, T: int, top_k: int, E: int) -> int:
        """The per-expert capacity C = ceil(gamma * N), N = T * top_k / E the
        mean number of pairs per expert; gamma <= 0: no capacity (-1)."""
        if not gamma > 0:
            return -1
        return int(math.ceil(gamma * (T * top_k) / E))

    def capacity_keep(self, topk_idx: np.ndarray, topk_w: np.ndarray, E: int, C: int) -> np.ndarray:
        """[T][k] 1 for the pairs each expert keeps under capacity C (see
        ``oracle_capacity_keep``)."""
        idx = np.ascontiguousarray(topk_idx, dtype=np.int32)
        w = np.ascontiguousarray(topk_w, dtype=np.float64)
        T, k = idx.shape
        keep = np.zeros((T, k), np.uint8)
        rc = self._lib.oracle_capacity_keep(self._ptr(idx), self._ptr(w), T, k, int(E), int(C), self._ptr(keep))
        if rc != 0:
            raise RuntimeError(f"oracle_capacity_keep failed ({rc})")
        return keep

    def forward_capacity(self, x, w_router, w_gate, w_up, w_down, ws_gate=None, ws_up=None,
                         ws_down=None, *, top_k: int, tau: float, gamma: float, nthreads: int = 0,
                         tau_shared: float = 0.0) -> OracleResult:
        """The layer with capacity-aware token drop at capacity factor gamma:
        the routing, then each expert's kept pairs (``capacity_keep``), then
        the layer with the dropped pairs' neurons all inactive (a dropped pair
        contributes nothing).  ``active`` of the result is the threshold mask
        with the dropped pairs cleared."""
        args = (x, w_router, w_gate, w_up, w_down, ws_gate, ws_up, ws_down)
        first = self.forward(*args, top_k=top_k, tau=tau, nthreads=nthreads, tau_shared=tau_shared)
        T = first.topk_idx.shape[0]
        E = first.logits.shape[1]
        C = self.capacity(gamma, T, top_k, E)
        keep = self.capacity_keep(first.topk_idx, first.topk_w, E, C)
        active = first.active * keep[:, :, None]
        res = self.forward(*args, top_k=top_k, tau=tau, nthreads=nthreads, active=active, tau_shared=tau_shared)
        res.score = first.score
        return res

    def calibrate_tau(self, scores: np.ndarray, sparsity: float) -> float:
        """tau = the floor(q*N)-th smallest of the routed pairs' scores s = |silu(g)|.

        The population is the T*k*f scores of the (token, expert) pairs the
        router selected; shared-expert scores are excluded (they are never
        masked).  The result is returned as a float32-representable value,
        which is how the layer receives it."""
        s = np.ascontiguousarray(scores, dtype=np.float64).reshape(-1)
        t = self._lib.oracle_calibrate_tau(self._ptr(s), s.size, float(sparsity))
        return float(np.float32(t))


_default = None


def load() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle()
    return _default


def build_variant(src_text: str, workdir: str | None = None) -> Oracle:
    """Compile a modified copy of the oracle source (used to plant mistakes in tests)."""
    workdir = workdir or tempfile.mkdtemp(prefix="oracle_variant_")
    src = os.path.join(workdir, "variant.c")
    with open(src, "w") as fh:
        fh.write(src_text)
    out = os.path.join(workdir, "libvariant.so")
    build(src, out, openmp=False)
    return Oracle(out)


def layer_inputs(weights, x):
    """Convert moe_inputs tensors to the bf16-bit numpy arrays the oracle takes."""
    import torch  # local: only used to view bf16 tensors as raw bits

    def bits(t):
        if t is None:
            return None
        return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)

    return dict(x=bits(x), w_router=bits(weights.w_router), w_gate=bits(weights.w_gate),
                w_up=bits(weights.w_up), w_down=bits(weights.w_down),
                ws_gate=bits(weights.ws_gate), ws_up=bits(weights.ws_up),
                ws_down=bits(weights.ws_down))
