"""B200-native (sm_100a) forward pass of the sparse top-k Mixture-of-Experts
layer: router -> softmax -> top-k (ties to the lower index) with optional
renormalisation -> dispatch -> per-expert SwiGLU MLP -> gate-weighted combine,
plus the expert counts and the load-balancing statistic.

The Python layer only allocates device memory and marshals arguments to the
C ABI of ``libmoe_b200.so`` (``include/moe.h``); every step runs in its CUDA
kernels.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch

from . import _binding as B
from ._binding import MoEError, load_library

__all__ = ["MoEError", "MoEOutputs", "MoELayer", "HostPipeline", "moe_forward", "workspace_size", "get_permutation",
           "load_library"]


def _dtype_code(t: torch.dtype) -> int:
    if t == torch.bfloat16:
        return B.MOE_BF16
    if t == torch.float32:
        return B.MOE_F32
    raise TypeError(f"unsupported dtype {t}: the layer takes bfloat16 or float32")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def workspace_size(T: int, d: int, E: int, k: int, I: int, dtype: torch.dtype) -> int:
    lib = load_library()
    n = lib.moe_workspace_size(T, d, E, k, I, _dtype_code(dtype))
    if n == 0:
        raise MoEError(B.MOE_ERR_INVALID_ARG, B.last_error_detail(lib))
    return int(n)


@dataclass
class MoEOutputs:
    out: torch.Tensor  # [T, d] fp32
    topk_idx: torch.Tensor  # [T, k] int32
    topk_gate: torch.Tensor  # [T, k] fp32
    counts: torch.Tensor  # [E] int32
    aux: torch.Tensor  # [1] fp32
    status: torch.Tensor  # [1] int32, MOE_DEV_* bits
    workspace: torch.Tensor  # uint8, holds the dispatch order of this call


def moe_forward(x, w_router, b_router, w_gate, w_up, w_down, k: int, renorm: bool, *, out=None, topk_idx=None,
                topk_gate=None, counts=None, aux=None, workspace=None, status=None, stream=None,
                events=None) -> MoEOutputs:
    """Run the layer on ``x`` ([T, d], CUDA) with stacked expert weights
    ``w_gate``/``w_up`` [E, I, d] and ``w_down`` [E, d, I]. Buffers that are
    not given are allocated with torch; the call is asynchronous on
    ``stream`` (default: torch's current stream). ``events``: optional list
    of MOE_NUM_KERNELS + 1 timing-enabled ``torch.cuda.Event`` recorded
    around each kernel (see ``moe_forward_events`` in include/moe.h)."""
    lib = load_library()
    T, d = x.shape
    E = w_router.shape[0]
    I = w_gate.shape[1]
    dt = _dtype_code(x.dtype)
    dev = x.device
    if dev.type != "cuda":
        raise ValueError("x must be a CUDA tensor (the layer runs only on the GPU)")
    for name, t, shape in (("w_router", w_router, (E, d)), ("w_gate", w_gate, (E, I, d)), ("w_up", w_up, (E, I, d)),
                           ("w_down", w_down, (E, d, I))):
        if tuple(t.shape) != shape or t.dtype != x.dtype or t.device != dev or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous {x.dtype} CUDA tensor of shape {shape}")
    if not x.is_contiguous():
        raise ValueError("x must be contiguous")
    if b_router is not None and (b_router.dtype != torch.float32 or b_router.numel() != E or b_router.device != dev):
        raise ValueError("b_router must be a float32 CUDA tensor of E elements")
    if out is None:
        out = torch.empty((T, d), dtype=torch.float32, device=dev)
    if topk_idx is None:
        topk_idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    if topk_gate is None:
        topk_gate = torch.empty((T, k), dtype=torch.float32, device=dev)
    if counts is None:
        counts = torch.empty((E,), dtype=torch.int32, device=dev)
    if aux is None:
        aux = torch.empty((1,), dtype=torch.float32, device=dev)
    if status is None:
        status = torch.zeros((1,), dtype=torch.int32, device=dev)
    if workspace is None:
        n = lib.moe_workspace_size(T, d, E, k, I, dt)
        if n == 0:
            raise MoEError(B.MOE_ERR_INVALID_ARG, B.last_error_detail(lib))
        workspace = torch.empty((n,), dtype=torch.uint8, device=dev)
    if stream is None:
        stream = torch.cuda.current_stream(dev).cuda_stream
    args = (_ptr(x), _ptr(w_router), _ptr(b_router), _ptr(w_gate), _ptr(w_up), _ptr(w_down), T, d, E, k, I,
            int(bool(renorm)), dt, _ptr(out), _ptr(topk_idx), _ptr(topk_gate), _ptr(counts), _ptr(aux),
            _ptr(workspace), workspace.numel(), _ptr(status), ctypes.c_void_p(stream))
    if events is None:
        st = lib.moe_forward(*args)
    else:
        for ev in events:
            if not ev.cuda_event:  # torch creates the event on its first record
                ev.record(torch.cuda.current_stream(dev))
        arr = (ctypes.c_void_p * len(events))(*[ev.cuda_event for ev in events])
        st = lib.moe_forward_events(*args, arr, len(events))
    B.check(st, lib)
    return MoEOutputs(out, topk_idx, topk_gate, counts, aux, status, workspace)


def get_permutation(res: MoEOutputs, T: int, d: int, E: int, k: int, I: int, dtype: torch.dtype, stream=None):
    """(offsets [E+1], perm_tok [T*k], inv [T, k]) of the call that produced ``res``."""
    lib = load_library()
    dev = res.workspace.device
    offsets = torch.empty((E + 1,), dtype=torch.int32, device=dev)
    perm = torch.empty((T * k,), dtype=torch.int32, device=dev)
    inv = torch.empty((T, k), dtype=torch.int32, device=dev)
    if stream is None:
        stream = torch.cuda.current_stream(dev).cuda_stream
    st = lib.moe_get_permutation(_ptr(res.workspace), res.workspace.numel(), T, d, E, k, I, _dtype_code(dtype),
                                 _ptr(offsets), _ptr(perm), _ptr(inv), ctypes.c_void_p(stream))
    B.check(st, lib)
    return offsets, perm, inv


class MoELayer:
    """The layer with resident weights and preallocated outputs/workspace for a
    fixed number of tokens, for repeated calls (serving, benchmarking)."""

    def __init__(self, w_router, b_router, w_gate, w_up, w_down, k: int, renorm: bool, max_tokens: int):
        self.w_router, self.b_router = w_router, b_router
        self.w_gate, self.w_up, self.w_down = w_gate, w_up, w_down
        self.k, self.renorm = k, renorm
        self.E, self.I, self.d = w_gate.shape[0], w_gate.shape[1], w_gate.shape[2]
        self.dtype = w_gate.dtype
        dev = w_gate.device
        self.T = max_tokens
        self.out = torch.empty((max_tokens, self.d), dtype=torch.float32, device=dev)
        self.topk_idx = torch.empty((max_tokens, k), dtype=torch.int32, device=dev)
        self.topk_gate = torch.empty((max_tokens, k), dtype=torch.float32, device=dev)
        self.counts = torch.empty((self.E,), dtype=torch.int32, device=dev)
        self.aux = torch.empty((1,), dtype=torch.float32, device=dev)
        self.status = torch.zeros((1,), dtype=torch.int32, device=dev)
        self.workspace = torch.empty((workspace_size(max_tokens, self.d, self.E, k, self.I, self.dtype),),
                                     dtype=torch.uint8, device=dev)

    def __call__(self, x, stream=None, events=None) -> MoEOutputs:
        T = x.shape[0]
        if T != self.T:
            raise ValueError(f"this layer was sized for {self.T} tokens")
        return moe_forward(x, self.w_router, self.b_router, self.w_gate, self.w_up, self.w_down, self.k, self.renorm,
                           out=self.out, topk_idx=self.topk_idx, topk_gate=self.topk_gate, counts=self.counts,
                           aux=self.aux, workspace=self.workspace, status=self.status, stream=stream, events=events)

    def forward_host(self, x_host, out_host, aux_host, x_dev):
        """End-to-end call from host memory: copy ``x_host`` (pinned, [T, d])
        to the device buffer ``x_dev``, run the layer, and copy the output and
        the statistic back into the pinned ``out_host`` / ``aux_host``. All on
        torch's current stream; returns without synchronising."""
        x_dev.copy_(x_host, non_blocking=True)
        self(x_dev)
        out_host.copy_(self.out, non_blocking=True)
        aux_host.copy_(self.aux, non_blocking=True)


class HostPipeline:
    """Runs batches that live in pinned host memory through a ``MoELayer``
    with the copies overlapped: batch i+1 is copied in and batch i-1 copied
    out while batch i computes (two device buffers each for x and out, one
    stream per direction). ``submit`` returns without synchronising; the
    host output buffer may be read after ``synchronize``."""

    def __init__(self, layer: "MoELayer"):
        self.layer = layer
        dev = layer.w_gate.device
        T, d = layer.T, layer.d
        self.x_dev = [torch.empty((T, d), dtype=layer.dtype, device=dev) for _ in range(2)]
        self.out_dev = [torch.empty((T, d), dtype=torch.float32, device=dev) for _ in range(2)]
        self.aux_dev = [torch.empty((1,), dtype=torch.float32, device=dev) for _ in range(2)]
        self.compute = torch.cuda.current_stream(dev)
        self.h2d = torch.cuda.Stream(dev)
        self.d2h = torch.cuda.Stream(dev)
        self.in_ready = [torch.cuda.Event() for _ in range(2)]
        self.computed = [torch.cuda.Event() for _ in range(2)]
        self.out_free = [torch.cuda.Event() for _ in range(2)]
        self.i = 0

    def submit(self, x_host, out_host, aux_host) -> None:
        b = self.i & 1
        L = self.layer
        if self.i >= 2:
            self.h2d.wait_event(self.computed[b])  # x buffer b no longer read
        with torch.cuda.stream(self.h2d):
            self.x_dev[b].copy_(x_host, non_blocking=True)
            self.in_ready[b].record(self.h2d)
        self.compute.wait_event(self.in_ready[b])
        if self.i >= 2:
            self.compute.wait_event(self.out_free[b])  # out buffer b copied out
        moe_forward(self.x_dev[b], L.w_router, L.b_router, L.w_gate, L.w_up, L.w_down, L.k, L.renorm,
                    out=self.out_dev[b], topk_idx=L.topk_idx, topk_gate=L.topk_gate, counts=L.counts,
                    aux=self.aux_dev[b], workspace=L.workspace, status=L.status,
                    stream=self.compute.cuda_stream)
        self.computed[b].record(self.compute)
        self.d2h.wait_event(self.computed[b])
        with torch.cuda.stream(self.d2h):
            out_host.copy_(self.out_dev[b], non_blocking=True)
            aux_host.copy_(self.aux_dev[b], non_blocking=True)
            self.out_free[b].record(self.d2h)
        self.i += 1

    def synchronize(self) -> None:
        self.d2h.synchronize()
        self.compute.synchronize()
