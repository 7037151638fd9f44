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

__all__ = ["MoEError", "MoEOptions", "MoEOutputs", "MoELayer", "HostPipeline", "moe_forward", "workspace_size",
           "get_permutation", "launch_plan", "load_library"]


def _dtype_code(t: torch.dtype) -> int:
    if t == torch.bfloat16:
        return B.MOE_BF16
    if t == torch.float32:
        return B.MOE_F32
    raise TypeError(f"unsupported dtype {t}: the layer takes bfloat16 or float32")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


@dataclass
class MoEOptions:
    """Options of the layer (``moe_options`` in include/moe.h).

    norm_form: 0 none, 1 torch's nn.RMSNorm x/sqrt(mean x^2 + eps)*w, 2 the
    form w*x/(sqrt(mean x^2) + eps); norm_weight: [d] in the layer dtype or
    None for ones. shared_*: weights of the shared experts ([S, I, d],
    [S, I, d], [S, d, I]) or None. capacity_factor: 0 = no dropping.
    z_loss: also compute the router z-loss statistic. fold_combine: fold the
    combine into the down GEMM for every top-k (atomic fp32 adds: with k > 2
    the result is not bit-reproducible between runs; k = 2 always folds)."""
    norm_form: int = 0
    norm_eps: float = 1e-5
    norm_weight: torch.Tensor | None = None
    shared_gate: torch.Tensor | None = None
    shared_up: torch.Tensor | None = None
    shared_down: torch.Tensor | None = None
    capacity_factor: float = 0.0
    z_loss: bool = False
    fold_combine: bool = False

    @property
    def n_shared(self) -> int:
        return 0 if self.shared_gate is None else int(self.shared_gate.shape[0])

    def to_c(self, dropped=None, z_loss=None) -> B.moe_options:
        o = B.moe_options()
        o.struct_bytes = ctypes.sizeof(B.moe_options)
        o.norm_form = int(self.norm_form)
        o.norm_eps = float(self.norm_eps)
        o.norm_weight = None if self.norm_weight is None else self.norm_weight.data_ptr()
        o.n_shared = self.n_shared
        if self.n_shared:
            o.shared_gate = self.shared_gate.data_ptr()
            o.shared_up = self.shared_up.data_ptr()
            o.shared_down = self.shared_down.data_ptr()
        o.capacity_factor = float(self.capacity_factor)
        o.dropped = None if dropped is None else dropped.data_ptr()
        o.z_loss = None if z_loss is None else z_loss.data_ptr()
        o.fold_combine = 1 if self.fold_combine else 0
        return o


def workspace_size(T: int, d: int, E: int, k: int, I: int, dtype: torch.dtype,
                   options: MoEOptions | None = None) -> int:
    lib = load_library()
    if options is None:
        n = lib.moe_workspace_size(T, d, E, k, I, _dtype_code(dtype))
    else:
        opt = options.to_c()
        n = lib.moe_workspace_size_ex(T, d, E, k, I, _dtype_code(dtype), ctypes.byref(opt))
    if n == 0:
        raise MoEError(B.MOE_ERR_INVALID_ARG, B.last_error_detail(lib))
    return int(n)


def launch_plan(T: int, d: int, E: int, k: int, I: int, dtype: torch.dtype, n_shared: int = 0,
                norm_form: int = 0, norm_weight: bool = False, fold_combine: bool = False) -> int:
    """The library's launch plan for a call of this shape (``moe_launch_plan``:
    MOE_PLAN_* bits saying which kernels are merged). A host-side query: the
    weight pointers it passes are placeholders that nothing dereferences."""
    lib = load_library()
    o = B.moe_options()
    o.struct_bytes = ctypes.sizeof(B.moe_options)
    o.norm_form = int(norm_form)
    o.norm_eps = 1e-5
    o.norm_weight = 256 if norm_weight else None
    o.n_shared = int(n_shared)
    if n_shared:
        o.shared_gate = o.shared_up = o.shared_down = 256
    o.fold_combine = 1 if fold_combine else 0
    plan = lib.moe_launch_plan(T, d, E, k, I, _dtype_code(dtype), ctypes.byref(o))
    if plan < 0:
        raise MoEError(B.MOE_ERR_INVALID_ARG, B.last_error_detail(lib))
    return int(plan)


def _check_options(options: MoEOptions, x, E: int, I: int):
    d = x.shape[1]
    if options.norm_weight is not None:
        w = options.norm_weight
        if w.dtype != x.dtype or w.numel() != d or w.device != x.device or not w.is_contiguous():
            raise ValueError(f"norm_weight must be a contiguous {x.dtype} CUDA tensor of {d} elements")
    if options.n_shared:
        S = options.n_shared
        for name, t, shape in (("shared_gate", options.shared_gate, (S, I, d)),
                               ("shared_up", options.shared_up, (S, I, d)),
                               ("shared_down", options.shared_down, (S, d, I))):
            if t is None or tuple(t.shape) != shape or t.dtype != x.dtype or t.device != x.device \
                    or not t.is_contiguous():
                raise ValueError(f"{name} must be a contiguous {x.dtype} CUDA tensor of shape {shape}")


@dataclass
class MoEOutputs:
    out: torch.Tensor  # [T, d] fp32
    topk_idx: torch.Tensor  # [T, k] int32
    topk_gate: torch.Tensor  # [T, k] fp32
    counts: torch.Tensor  # [E] int32
    aux: torch.Tensor  # [1] fp32
    status: torch.Tensor  # [1] int32, MOE_DEV_* bits
    workspace: torch.Tensor  # uint8, holds the dispatch order of this call
    z_loss: torch.Tensor | None = None  # [1] fp32 when options.z_loss
    dropped: torch.Tensor | None = None  # [1] int32 when options.capacity_factor > 0


def moe_forward(x, w_router, b_router, w_gate, w_up, w_down, k: int, renorm: bool, *, out=None, topk_idx=None,
                topk_gate=None, counts=None, aux=None, workspace=None, status=None, stream=None,
                events=None, options: MoEOptions | None = None, z_loss=None, dropped=None) -> MoEOutputs:
    """Run the layer on ``x`` ([T, d], CUDA) with stacked expert weights
    ``w_gate``/``w_up`` [E, I, d] and ``w_down`` [E, d, I]. Buffers that are
    not given are allocated with torch; the call is asynchronous on
    ``stream`` (default: torch's current stream). ``events``: optional list
    of MOE_NUM_KERNELS + 1 timing-enabled ``torch.cuda.Event`` recorded
    around each kernel (see ``moe_forward_events`` in include/moe.h).
    ``options``: RMSNorm, shared experts, capacity, z-loss (``MoEOptions``)."""
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
    if options is not None:
        _check_options(options, x, E, I)
        if options.z_loss and z_loss is None:
            z_loss = torch.empty((1,), dtype=torch.float32, device=dev)
        if options.capacity_factor > 0 and dropped is None:
            dropped = torch.empty((1,), dtype=torch.int32, device=dev)
    if workspace is None:
        workspace = torch.empty((workspace_size(T, d, E, k, I, x.dtype, options),), dtype=torch.uint8, device=dev)
    if stream is None:
        stream = torch.cuda.current_stream(dev).cuda_stream
    head = (_ptr(x), _ptr(w_router), _ptr(b_router), _ptr(w_gate), _ptr(w_up), _ptr(w_down), T, d, E, k, I,
            int(bool(renorm)), dt)
    tail = (_ptr(out), _ptr(topk_idx), _ptr(topk_gate), _ptr(counts), _ptr(aux), _ptr(workspace), workspace.numel(),
            _ptr(status), ctypes.c_void_p(stream))
    arr, n_ev = None, 0
    if events is not None:
        for ev in events:
            if not ev.cuda_event:  # torch creates the event on its first record
                ev.record(torch.cuda.current_stream(dev))
        arr = (ctypes.c_void_p * len(events))(*[ev.cuda_event for ev in events])
        n_ev = len(events)
    if options is not None:
        opt = options.to_c(dropped=dropped, z_loss=z_loss if options.z_loss else None)
        st = lib.moe_forward_ex(*head, ctypes.byref(opt), *tail, arr, n_ev)
    elif events is None:
        st = lib.moe_forward(*head, *tail)
    else:
        st = lib.moe_forward_events(*head, *tail, arr, n_ev)
    B.check(st, lib)
    return MoEOutputs(out, topk_idx, topk_gate, counts, aux, status, workspace,
                      z_loss if options is not None and options.z_loss else None, dropped)


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

    def __init__(self, w_router, b_router, w_gate, w_up, w_down, k: int, renorm: bool, max_tokens: int,
                 options: MoEOptions | None = None):
        self.options = options
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
        self.z_loss = torch.empty((1,), dtype=torch.float32, device=dev)
        self.dropped = torch.empty((1,), dtype=torch.int32, device=dev)
        self.workspace = torch.empty((workspace_size(max_tokens, self.d, self.E, k, self.I, self.dtype, options),),
                                     dtype=torch.uint8, device=dev)

    def __call__(self, x, stream=None, events=None) -> MoEOutputs:
        T = x.shape[0]
        if T != self.T:
            raise ValueError(f"this layer was sized for {self.T} tokens")
        return moe_forward(x, self.w_router, self.b_router, self.w_gate, self.w_up, self.w_down, self.k, self.renorm,
                           out=self.out, topk_idx=self.topk_idx, topk_gate=self.topk_gate, counts=self.counts,
                           aux=self.aux, workspace=self.workspace, status=self.status, stream=stream, events=events,
                           options=self.options, z_loss=self.z_loss, dropped=self.dropped)

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
    """Runs batches that live in host memory through a ``MoELayer`` with the
    library's native pipeline (``moe_pipeline_*`` in include/moe.h): batch
    i+1 is copied in and batch i-1 copied out while batch i computes (two
    device slots each for x, out and aux, allocated here with torch; one
    stream per copy direction inside the library; compute on torch's
    current stream). ``submit`` returns without synchronising; the host
    output buffers may be read after ``synchronize``. Pinned host buffers
    let the copies overlap."""

    def __init__(self, layer: "MoELayer"):
        self.layer = layer
        lib = load_library()
        dev = layer.w_gate.device
        T, d = layer.T, layer.d
        self.x_dev = [torch.empty((T, d), dtype=layer.dtype, device=dev) for _ in range(2)]
        self.out_dev = [torch.empty((T, d), dtype=torch.float32, device=dev) for _ in range(2)]
        self.aux_dev = [torch.empty((1,), dtype=torch.float32, device=dev) for _ in range(2)]
        self.compute = torch.cuda.current_stream(dev)
        desc = B.moe_layer_desc()
        desc.struct_bytes = ctypes.sizeof(B.moe_layer_desc)
        desc.w_router = layer.w_router.data_ptr()
        desc.b_router = None if layer.b_router is None else layer.b_router.data_ptr()
        desc.w_gate, desc.w_up, desc.w_down = layer.w_gate.data_ptr(), layer.w_up.data_ptr(), layer.w_down.data_ptr()
        desc.T, desc.d, desc.E, desc.k, desc.I = T, d, layer.E, layer.k, layer.I
        desc.renorm = int(bool(layer.renorm))
        desc.dtype = _dtype_code(layer.dtype)
        self._opt = None
        if layer.options is not None:
            o = layer.options
            self._opt = o.to_c(dropped=layer.dropped if o.capacity_factor > 0 else None,
                               z_loss=layer.z_loss if o.z_loss else None)
            desc.opt = ctypes.pointer(self._opt)
        desc.workspace = layer.workspace.data_ptr()
        desc.workspace_bytes = layer.workspace.numel()
        desc.topk_idx, desc.topk_gate = layer.topk_idx.data_ptr(), layer.topk_gate.data_ptr()
        desc.counts, desc.status_dev = layer.counts.data_ptr(), layer.status.data_ptr()
        for b in range(2):
            desc.x_dev[b] = self.x_dev[b].data_ptr()
            desc.out_dev[b] = self.out_dev[b].data_ptr()
            desc.aux_dev[b] = self.aux_dev[b].data_ptr()
        handle = ctypes.c_void_p()
        B.check(lib.moe_pipeline_create(ctypes.byref(desc), ctypes.c_void_p(self.compute.cuda_stream),
                                        ctypes.byref(handle)), lib)
        self._lib = lib
        self._p = handle

    def stream(self, which: int) -> torch.cuda.ExternalStream:
        """One of the pipeline's streams (B.MOE_PIPELINE_COPY_IN / _COMPUTE /
        _COPY_OUT), e.g. to record timing events on it."""
        ptr = self._lib.moe_pipeline_stream(self._p, which)
        return torch.cuda.ExternalStream(ptr, device=self.layer.w_gate.device)

    def submit(self, x_host, out_host, aux_host=None) -> None:
        L = self.layer
        if tuple(x_host.shape) != (L.T, L.d) or x_host.dtype != L.dtype or x_host.device.type != "cpu" \
                or not x_host.is_contiguous():
            raise ValueError(f"x_host must be a contiguous host tensor [{L.T}, {L.d}] of {L.dtype}")
        if tuple(out_host.shape) != (L.T, L.d) or out_host.dtype != torch.float32 \
                or out_host.device.type != "cpu" or not out_host.is_contiguous():
            raise ValueError(f"out_host must be a contiguous host float32 tensor [{L.T}, {L.d}]")
        if aux_host is not None and (aux_host.numel() != 1 or aux_host.dtype != torch.float32
                                     or aux_host.device.type != "cpu"):
            raise ValueError("aux_host must be a host float32 tensor of one element")
        B.check(self._lib.moe_pipeline_submit(self._p, _ptr(x_host), _ptr(out_host), _ptr(aux_host)), self._lib)

    def synchronize(self) -> None:
        B.check(self._lib.moe_pipeline_synchronize(self._p), self._lib)

    def close(self) -> None:
        if self._p is not None and self._p.value:
            B.check(self._lib.moe_pipeline_destroy(self._p), self._lib)
        self._p = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
