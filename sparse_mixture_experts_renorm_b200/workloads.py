"""Seeded synthetic workloads for the MoE forward pass.

This module only draws inputs: shapes, value distributions and the seed. It
holds none of the layer's arithmetic, and it is the one module that both the
CUDA path's harnesses and the oracle's tests use, so that both sides see the
same stored tensors.

The shapes follow the pages' Mixtral-style workloads: the Mixtral MoE Block
page ("Structure" table and exported PyTorch: d=4096, 8 experts, top-2,
I=14336, input 1 x 4096 x 4096), and KempnerForge's ModelConfig FFN sizing
(computed_ffn_hidden_dim / computed_expert_ffn_hidden_dim), which gives
I=2816 at d=1024 and I=1408 at d=2048 with an expert multiplier of 0.25.
The pages use no public dataset; these synthetic draws stand in for one.

Draw recipe: one ``torch.Generator`` seeded with ``seed`` on the target
device, draws in the order x, W_router, W_gate, W_up, W_down, each
``torch.randn`` in fp32 scaled by its std and then cast to the workload
dtype. The skewed workload's router bias is the deterministic
``b_e = 0.5 * ln(1 / (e + 1))``.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    d: int
    E: int
    k: int
    I: int
    renorm: bool
    dtype: str  # "f32" or "bf16"
    x_std: float = 1.0
    w_std: float = 0.02
    router_std: float = 0.02
    zipf_bias: bool = False
    note: str = ""

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def active_flops(self) -> float:
        """Active-expert FLOPs of one forward: 6*d*I*k*T + 2*d*E*T."""
        return 6.0 * self.d * self.I * self.k * self.T + 2.0 * self.d * self.E * self.T

    def replace(self, **kw) -> "Workload":
        d = dict(self.__dict__)
        d.update(kw)
        return Workload(**d)


WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", T=64, d=128, E=4, k=2, I=256, renorm=True, dtype="f32",
                         router_std=0.5, note="tiny fp32, router std 0.5 to avoid near ties"),
    "small_bf16": Workload("small_bf16", T=4096, d=1024, E=8, k=2, I=2816, renorm=True, dtype="bf16"),
    "mixtral_prefill": Workload("mixtral_prefill", T=4096, d=4096, E=8, k=2, I=14336, renorm=True,
                                dtype="bf16", note="Mixtral-shape prefill, batch 1 x seq 4096"),
    "fine_grained": Workload("fine_grained", T=16384, d=2048, E=64, k=6, I=1408, renorm=False,
                             dtype="bf16", zipf_bias=True,
                             note="64 fine-grained experts, top-6, no renorm, Zipf-like router bias"),
    "mixtral_decode": Workload("mixtral_decode", T=32, d=4096, E=8, k=2, I=14336, renorm=True,
                               dtype="bf16", note="Mixtral-shape decode, weight streaming"),
}


@dataclass
class Inputs:
    wl: Workload
    x: torch.Tensor  # [T, d]
    w_router: torch.Tensor  # [E, d]
    b_router: torch.Tensor | None  # [E] fp32
    w_gate: torch.Tensor  # [E, I, d]
    w_up: torch.Tensor  # [E, I, d]
    w_down: torch.Tensor  # [E, d, I]
    extra: dict = field(default_factory=dict)


def zipf_bias(E: int) -> torch.Tensor:
    return torch.tensor([0.5 * math.log(1.0 / (e + 1)) for e in range(E)], dtype=torch.float32)


def _randn(shape, std, gen, device, dtype):
    t = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def make_inputs(wl: Workload, device="cpu", seed: int = 0) -> Inputs:
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    dt = wl.torch_dtype
    x = _randn((wl.T, wl.d), wl.x_std, gen, device, dt)
    w_router = _randn((wl.E, wl.d), wl.router_std, gen, device, dt)
    w_gate = _randn((wl.E, wl.I, wl.d), wl.w_std, gen, device, dt)
    w_up = _randn((wl.E, wl.I, wl.d), wl.w_std, gen, device, dt)
    w_down = _randn((wl.E, wl.d, wl.I), wl.w_std, gen, device, dt)
    b = zipf_bias(wl.E).to(device) if wl.zipf_bias else None
    return Inputs(wl, x, w_router, b, w_gate, w_up, w_down)


@dataclass
class OptionInputs:
    """Tensors of the layer's options: the RMSNorm weight and the shared
    experts' weights (None where unused)."""
    norm_weight: torch.Tensor | None  # [d]
    shared_gate: torch.Tensor | None  # [S, I, d]
    shared_up: torch.Tensor | None  # [S, I, d]
    shared_down: torch.Tensor | None  # [S, d, I]


def make_option_inputs(wl: Workload, device="cpu", seed: int = 0, n_shared: int = 0,
                       norm_weight: bool = False) -> OptionInputs:
    """Draws, from a generator seeded with ``seed + 7919``, in this order: the
    RMSNorm weight ``1 + 0.1 * N(0, 1)`` (when asked for), then the shared
    experts' gate, up and down weights with the workload's weight std."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed + 7919)
    dt = wl.torch_dtype
    nw = None
    if norm_weight:
        nw = (1.0 + _randn((wl.d,), 0.1, gen, device, torch.float32)).to(dt)
    sg = su = sd = None
    if n_shared:
        sg = _randn((n_shared, wl.I, wl.d), wl.w_std, gen, device, dt)
        su = _randn((n_shared, wl.I, wl.d), wl.w_std, gen, device, dt)
        sd = _randn((n_shared, wl.d, wl.I), wl.w_std, gen, device, dt)
    return OptionInputs(nw, sg, su, sd)


def make_tokens(wl: Workload, T: int, device="cpu", seed: int = 1) -> torch.Tensor:
    """A fresh batch of activations with the workload's distribution."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    return _randn((T, wl.d), wl.x_std, gen, device, wl.torch_dtype)
