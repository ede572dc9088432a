"""Seeded synthetic workloads for the routed-expert MoE layer.

This module holds shapes and random draws only.  It contains none of the
layer's arithmetic (no projection, activation, threshold or routing), so both
the CPU oracle and the CUDA path can take their inputs from here without
sharing any of the method's code.

Workloads (the five shapes the intra-expert sparsity pages evaluate on, see
"Uncovering Intra-expert Activation Sparsity for Efficient MoE Model
Execution", Methodology / Results):

  tiny      d=256,  E=8,   f=512,  k=2, 1 shared expert  (correctness size)
  olmoe     d=2048, E=64,  f=1024, k=8, no shared expert  (decode layer)
  dsv2lite  d=2048, E=64,  f=1408, k=6, 2 shared experts
  large     d=4096, E=256, f=1024, k=8, 1 shared expert   (6.44 GB of experts)
  crossover olmoe shapes, T swept 1..4096

Weight convention is ``x @ W``:
  w_router [E][d], w_gate/w_up [E][d][f], w_down [E][f][d]
  ws_gate/ws_up [S][d][f], ws_down [S][f][d]
Every weight is N(0, 1/fan_in) rounded to bf16 (fan_in = d for router, gate
and up; f for down).  x is N(0, 1); the tiny workload draws it in fp32 and
rounds to bf16 with round-to-nearest-even, the others draw bf16 directly
(same thing: torch rounds fp32 draws to bf16 with RNE).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Shape:
    name: str
    d_model: int
    n_experts: int
    d_ff: int
    top_k: int
    n_shared: int
    t_values: tuple
    sparsity: tuple = (0.9,)
    seed_base: int = 0

    @property
    def expert_params(self) -> int:
        return 3 * self.n_experts * self.d_model * self.d_ff


SHAPES = {
    "tiny": Shape("tiny", 256, 8, 512, 2, 1, (16,), (0.9,), 1000),
    "olmoe": Shape("olmoe", 2048, 64, 1024, 8, 0, (1, 4, 16, 64), (0.9,), 2000),
    "dsv2lite": Shape("dsv2lite", 2048, 64, 1408, 6, 2, (1, 8, 32, 128),
                      (0.0, 0.5, 0.8, 0.9, 0.95), 3000),
    "large": Shape("large", 4096, 256, 1024, 8, 1, (1, 16, 64), (0.98,), 4000),
    "crossover": Shape("crossover", 2048, 64, 1024, 8, 0,
                       tuple(2 ** i for i in range(13)), (0.9,), 5000),
}


def custom_shape(d_model, n_experts, d_ff, top_k, n_shared, name="custom", seed_base=7000):
    return Shape(name, d_model, n_experts, d_ff, top_k, n_shared, (1,), (0.9,), seed_base)


@dataclass
class Weights:
    """bf16 tensors in the x @ W convention (see module docstring)."""
    w_router: torch.Tensor
    w_gate: torch.Tensor
    w_up: torch.Tensor
    w_down: torch.Tensor
    ws_gate: torch.Tensor | None = None
    ws_up: torch.Tensor | None = None
    ws_down: torch.Tensor | None = None
    extra: dict = field(default_factory=dict)

    def to(self, device) -> "Weights":
        def mv(t):
            return None if t is None else t.to(device)
        return Weights(mv(self.w_router), mv(self.w_gate), mv(self.w_up), mv(self.w_down),
                       mv(self.ws_gate), mv(self.ws_up), mv(self.ws_down), dict(self.extra))


def _randn_bf16(gen, shape, std, device):
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    # draw in fp32 slabs to bound peak memory, round to bf16 (RNE)
    flat = out.view(-1)
    step = 1 << 26
    for s in range(0, flat.numel(), step):
        n = min(step, flat.numel() - s)
        flat[s:s + n] = (torch.randn(n, generator=gen, device=device, dtype=torch.float32)
                         * std).to(torch.bfloat16)
    return out


def make_weights(shape: Shape, device="cpu", seed: int | None = None) -> Weights:
    """Draw every weight of the layer from one seeded generator (seed = 1000*config)."""
    seed = shape.seed_base if seed is None else seed
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    d, E, f, S = shape.d_model, shape.n_experts, shape.d_ff, shape.n_shared
    w_router = _randn_bf16(gen, (E, d), d ** -0.5, device)
    w_gate = _randn_bf16(gen, (E, d, f), d ** -0.5, device)
    w_up = _randn_bf16(gen, (E, d, f), d ** -0.5, device)
    w_down = _randn_bf16(gen, (E, f, d), f ** -0.5, device)
    ws = (None, None, None)
    if S > 0:
        ws = (_randn_bf16(gen, (S, d, f), d ** -0.5, device),
              _randn_bf16(gen, (S, d, f), d ** -0.5, device),
              _randn_bf16(gen, (S, f, d), f ** -0.5, device))
    return Weights(w_router, w_gate, w_up, w_down, *ws)


def make_x(shape: Shape, T: int, device="cpu", seed: int | None = None) -> torch.Tensor:
    """x ~ N(0,1) drawn in fp32 and rounded to bf16 (RNE); seed = 1000*config + T."""
    seed = shape.seed_base + T if seed is None else seed
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    return torch.randn((T, shape.d_model), generator=gen, device=device,
                       dtype=torch.float32).to(torch.bfloat16)


def bf16_bits(t: torch.Tensor):
    """Raw uint16 view of a bf16 tensor as a contiguous CPU numpy array."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view("uint16")
