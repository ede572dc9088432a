"""MoESparseLayer: owns one library handle; torch supplies device memory and streams."""
from __future__ import annotations

import torch

from . import _binding as B


class MoESparseLayer:
    """Routed-expert MoE layer with intra-expert activation sparsity.

    Weights are bf16 CUDA tensors in the x @ W layout (w_router [E][d],
    w_gate/w_up [E][d][f], w_down [E][f][d], optional shared ws_* with a
    leading n_shared dimension).  The library copies and repacks them, so the
    caller's tensors may be freed after construction.
    """

    def __init__(self, w_router, w_gate, w_up, w_down, ws_gate=None, ws_up=None, ws_down=None,
                 top_k: int = 8, max_tokens: int = 4096):
        for t in (w_router, w_gate, w_up, w_down, ws_gate, ws_up, ws_down):
            if t is not None and (t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous()):
                raise ValueError("weights must be contiguous bf16 CUDA tensors")
        self.E, self.d_model = w_router.shape
        self.d_ff = w_gate.shape[2]
        self.n_shared = 0 if ws_gate is None else ws_gate.shape[0]
        self.top_k = top_k
        self.max_tokens = max_tokens
        self.h = B.moe_sparse_create(
            dict(w_router=w_router, w_gate=w_gate, w_up=w_up, w_down=w_down, ws_gate=ws_gate,
                 ws_up=ws_up, ws_down=ws_down),
            self.E, top_k, self.d_model, self.d_ff, self.n_shared, max_tokens)

    @classmethod
    def from_weights(cls, W, top_k, max_tokens=4096):
        return cls(W.w_router, W.w_gate, W.w_up, W.w_down, W.ws_gate, W.ws_up, W.ws_down,
                   top_k=top_k, max_tokens=max_tokens)

    def _check_x(self, x):
        if x.dtype != torch.bfloat16 or not x.is_cuda or not x.is_contiguous():
            raise ValueError("x must be a contiguous bf16 CUDA tensor")
        if x.dim() != 2 or x.shape[1] != self.d_model:
            raise ValueError(f"x must be [T][{self.d_model}]")

    @staticmethod
    def _out_like(x, out):
        """`out`, or a new tensor like x; the library writes T x d_model bf16 values there."""
        if out is None:
            return torch.empty_like(x)
        if (out.dtype != torch.bfloat16 or out.device != x.device or not out.is_contiguous()
                or out.shape != x.shape):
            raise ValueError(f"out must be a contiguous bf16 tensor of shape {tuple(x.shape)} on {x.device}")
        return out

    def forward(self, x, tau: float, out=None, stream=None):
        self._check_x(x)
        out = self._out_like(x, out)
        B.moe_sparse_forward(self.h, x, x.shape[0], float(tau), out, stream)
        return out

    def dense_forward(self, x, out=None, stream=None):
        self._check_x(x)
        out = self._out_like(x, out)
        B.moe_dense_forward(self.h, x, x.shape[0], out, stream)
        return out

    def set_path(self, path: int):
        B.moe_set_path(self.h, path)

    def set_t_star(self, t_star: int):
        B.moe_set_t_star(self.h, t_star)

    def tune_t_star(self, x, tau: float, stream=None) -> int:
        """Measure both branches on batches of x's first rows (up to all of x) and set T*."""
        self._check_x(x)
        return B.moe_tune_t_star(self.h, x, x.shape[0], float(tau), stream)

    def set_shared_tau(self, tau_shared: float):
        """The shared experts' own threshold on later masked forwards (<= 0: dense)."""
        B.moe_set_shared_tau(self.h, float(tau_shared))

    def set_rank_budget(self, r: int):
        """Keep each routed pair's r highest-scoring neurons on later masked
        forwards instead of thresholding at tau (r < 0: back to the threshold)."""
        B.moe_set_rank_budget(self.h, int(r))

    def set_capacity(self, gamma: float):
        """Capacity-aware token drop on later forwards: each expert keeps at most
        ceil(gamma * T * top_k / E) pairs, the ones with the largest routing
        weight (gamma <= 0: off)."""
        B.moe_set_capacity(self.h, float(gamma))

    def set_deterministic(self, enable: bool = True):
        """Combine each token's contributions in one fixed order on later
        forwards (bit-identical repeats), instead of fp32 atomics."""
        B.moe_set_deterministic(self.h, bool(enable))

    def calibrate_tau_shared(self, x, sparsity: float, stream=None) -> float:
        """tau_shared keeping about 1 - sparsity of the shared experts' neurons of this batch."""
        self._check_x(x)
        return B.moe_calibrate_tau_shared(self.h, x, x.shape[0], sparsity, stream)

    def set_fused_router(self, enable, one_launch: bool = False):
        """Route decode batches inside the expert kernel (the default); with
        one_launch also combine there, so a forward is a single launch."""
        B.moe_set_fused_router(self.h, (2 if one_launch else 1) if enable else 0)

    def router(self, x, stream=None):
        self._check_x(x)
        T = x.shape[0]
        idx = torch.empty((T, self.top_k), dtype=torch.int32, device=x.device)
        w = torch.empty((T, self.top_k), dtype=torch.float32, device=x.device)
        B.moe_debug_router(self.h, x, T, idx, w, stream)
        return idx, w

    def active_lists(self, x, tau: float, out=None, stream=None):
        self._check_x(x)
        T = x.shape[0]
        idx = torch.empty((T, self.top_k, self.d_ff), dtype=torch.int16, device=x.device)
        cnt = torch.empty((T, self.top_k), dtype=torch.int32, device=x.device)
        out = None if out is None else self._out_like(x, out)
        B.moe_debug_active(self.h, x, T, float(tau), idx, cnt, out, stream)
        return idx, cnt

    def calibrate_tau(self, x, sparsity: float, stream=None) -> float:
        """tau keeping about 1 - sparsity of the routed neurons of this batch (on the GPU)."""
        self._check_x(x)
        return B.moe_calibrate_tau(self.h, x, x.shape[0], sparsity, stream)

    def stats(self):
        return B.moe_query_stats(self.h)

    def close(self):
        if getattr(self, "h", None):
            B.moe_sparse_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:  # noqa: BLE001 - interpreter shutdown
            pass
