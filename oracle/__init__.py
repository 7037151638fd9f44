"""fp64 CPU oracle for the sparse top-k MoE forward pass (ctypes wrapper).

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s ``cpu_baseline`` leg (and its ``--impl reference`` arm) may
import this package. It shares no code with the CUDA path; the arithmetic
lives in ``moe_oracle.c`` and this module only marshals arguments.

Parity status: every function here is pinned by ``tests/test_oracle.py``
(brute force on tiny inputs, a dense library SwiGLU for E=1/k=1 and k=E,
zero-router ties, uniform-routing aux values, the stable-sort dispatch order,
the Mixtral parameter count; for the options: torch's rms_norm and worked
values of the other RMSNorm form, scipy's logsumexp and closed forms of the
z-loss, hand-worked capacity cases, and shared experts against a dense torch
SwiGLU).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

F32, BF16, F64 = 0, 1, 2

_lib = None


def build(force: bool = False) -> str:
    """Compile ``moe_oracle.c`` into ``liboracle.so`` with gcc + OpenMP."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.run(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"],
            check=True,
        )
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _bind(lib):
    P, I64, I32, D = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_double
    lib.oracle_num_threads.restype = I32
    lib.oracle_set_num_threads.argtypes = [I32]
    lib.oracle_round_bf16.argtypes = [P, I64, P]
    lib.oracle_rmsnorm.argtypes = [P, I32, P, I32, I64, I64, D, I32, P]
    lib.oracle_router_logits.argtypes = [P, I32, P, I32, P, I64, I64, I32, P]
    lib.oracle_softmax.argtypes = [P, I64, I32, P]
    lib.oracle_z_loss.argtypes = [P, I64, I32]
    lib.oracle_z_loss.restype = D
    lib.oracle_gates.argtypes = [P, I64, I32, I32, P, I32, P]
    lib.oracle_topk.argtypes = [P, I64, I32, I32, I32, P, P, P]
    lib.oracle_stats.argtypes = [P, P, I64, I32, I32, P, P, P]
    lib.oracle_capacity.argtypes = [D, I64, I32, I32]
    lib.oracle_capacity.restype = I64
    lib.oracle_dispatch.argtypes = [P, I64, I32, I32, I64, P, P, P]
    lib.oracle_dispatch.restype = I64
    lib.oracle_expert_rows.argtypes = [P, I32, P, P, P, I32, I64, I64, I64, P, P, P]
    lib.oracle_moe_tokens.argtypes = [P, I32, P, P, P, I32, I64, I64, I32, I64, P, P, P, P, I32, P, P, P, P]
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = _bind(ctypes.CDLL(build()))
    return _lib


class use_library:
    """Context manager that routes this module's calls to another build of
    the oracle source (used by the tests that plant mistakes in a copy)."""

    def __init__(self, path: str):
        self.path = path

    def __enter__(self):
        global _lib
        self._saved = _lib
        _lib = _bind(ctypes.CDLL(self.path))
        return self

    def __exit__(self, *exc):
        global _lib
        _lib = self._saved
        return False


def _as_stored(a):
    """Return (contiguous numpy array of the stored bits, dtype flag)."""
    try:
        import torch

        if isinstance(a, torch.Tensor):
            a = a.detach().to("cpu").contiguous()
            if a.dtype == torch.bfloat16:
                return a.view(torch.int16).numpy().view(np.uint16), BF16
            if a.dtype == torch.float32:
                return a.numpy(), F32
            if a.dtype == torch.float64:
                return a.numpy(), F64
            raise TypeError(f"oracle takes fp32, bf16 or fp64 tensors, got {a.dtype}")
    except ImportError:  # pragma: no cover - torch is always present here
        pass
    a = np.ascontiguousarray(a)
    if a.dtype == np.float32:
        return a, F32
    if a.dtype == np.float64:
        return a, F64
    if a.dtype == np.uint16:
        return a, BF16
    raise TypeError(f"oracle takes float32, float64 or bf16-bit (uint16) arrays, got {a.dtype}")


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return _load().oracle_num_threads()


def set_num_threads(n: int) -> None:
    _load().oracle_set_num_threads(int(n))


def round_bf16(a) -> np.ndarray:
    """fp64 values rounded (via fp32) to the nearest bf16, ties to even."""
    lib = _load()
    a = np.ascontiguousarray(a, dtype=np.float64)
    out = np.empty_like(a)
    lib.oracle_round_bf16(_ptr(a), a.size, _ptr(out))
    return out


def rmsnorm(x, weight=None, eps: float = 1e-5, form: int = 1) -> np.ndarray:
    """The pre-MoE RMSNorm of every token in fp64: form 1 is torch's
    nn.RMSNorm (eps under the root), form 2 the page's w*x/(rms+eps)."""
    lib = _load()
    xs, dt = _as_stored(x)
    T, d = xs.shape
    ws, wdt = (None, 0) if weight is None else _as_stored(weight)
    out = np.empty((T, d), dtype=np.float64)
    lib.oracle_rmsnorm(_ptr(xs), dt, _ptr(ws), wdt, T, d, float(eps), int(form), _ptr(out))
    return out


def router_logits(x, w_router, b_router=None) -> np.ndarray:
    """Router logits ``[T, E]`` in fp64 (bias included)."""
    lib = _load()
    xs, dt = _as_stored(x)
    ws, wdt = _as_stored(w_router)
    T, d = xs.shape
    E = ws.shape[0]
    b = None if b_router is None else np.ascontiguousarray(np.asarray(b_router, dtype=np.float32))
    logits = np.empty((T, E), dtype=np.float64)
    lib.oracle_router_logits(_ptr(xs), dt, _ptr(ws), wdt, _ptr(b), T, d, E, _ptr(logits))
    return logits


def softmax(logits: np.ndarray) -> np.ndarray:
    lib = _load()
    logits = np.ascontiguousarray(logits, dtype=np.float64)
    T, E = logits.shape
    probs = np.empty((T, E), dtype=np.float64)
    lib.oracle_softmax(_ptr(logits), T, E, _ptr(probs))
    return probs


def router_probs(x, w_router, b_router=None) -> np.ndarray:
    """Softmax router probabilities ``[T, E]`` in fp64."""
    return softmax(router_logits(x, w_router, b_router))


def z_loss(logits: np.ndarray) -> float:
    """Router z-loss statistic: mean over tokens of logsumexp(logits)^2."""
    lib = _load()
    logits = np.ascontiguousarray(logits, dtype=np.float64)
    T, E = logits.shape
    return float(lib.oracle_z_loss(_ptr(logits), T, E))


def capacity(capacity_factor: float, T: int, k: int, E: int) -> int:
    """Assignments an expert may keep, or -1 (no limit) when the factor is <= 0."""
    return int(_load().oracle_capacity(float(capacity_factor), T, k, E))


def topk(probs: np.ndarray, k: int, renorm: bool):
    """(topk_idx int32 [T,k], gates fp64 [T,k], gap fp64 [T])."""
    lib = _load()
    probs = np.ascontiguousarray(probs, dtype=np.float64)
    T, E = probs.shape
    idx = np.empty((T, k), dtype=np.int32)
    gate = np.empty((T, k), dtype=np.float64)
    gap = np.empty((T,), dtype=np.float64)
    lib.oracle_topk(_ptr(probs), T, E, k, int(renorm), _ptr(idx), _ptr(gate), _ptr(gap))
    return idx, gate, gap


def gates_for(probs: np.ndarray, idx: np.ndarray, renorm: bool) -> np.ndarray:
    """Gates of an arbitrary choice of experts per token."""
    lib = _load()
    probs = np.ascontiguousarray(probs, dtype=np.float64)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T, E = probs.shape
    k = idx.shape[1]
    gate = np.empty((T, k), dtype=np.float64)
    lib.oracle_gates(_ptr(probs), T, E, k, _ptr(idx), int(renorm), _ptr(gate))
    return gate


def stats(probs: np.ndarray, idx: np.ndarray):
    """(counts int64 [E], mean_prob fp64 [E], aux float)."""
    lib = _load()
    probs = np.ascontiguousarray(probs, dtype=np.float64)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T, E = probs.shape
    k = idx.shape[1] if idx.ndim == 2 else 1
    counts = np.zeros((E,), dtype=np.int64)
    mean_prob = np.zeros((E,), dtype=np.float64)
    aux = np.zeros((1,), dtype=np.float64)
    lib.oracle_stats(_ptr(probs), _ptr(idx), T, E, k, _ptr(counts), _ptr(mean_prob), _ptr(aux))
    return counts, mean_prob, float(aux[0])


def dispatch(idx: np.ndarray, E: int, cap: int = -1):
    """(offsets int64 [E+1], perm_tok int32 [R], inv int32 [T,k], dropped):
    R kept rows; inv is -1 for a dropped slot; cap < 0 keeps everything."""
    lib = _load()
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T, k = idx.shape
    offsets = np.zeros((E + 1,), dtype=np.int64)
    perm = np.zeros((T * k,), dtype=np.int32)
    inv = np.zeros((T, k), dtype=np.int32)
    dropped = lib.oracle_dispatch(_ptr(idx), T, k, E, int(cap), _ptr(offsets), _ptr(perm), _ptr(inv))
    return offsets, perm[:int(offsets[E])].copy(), inv, int(dropped)


def expert_rows(x, w_gate, w_up, w_down, tok, expert) -> np.ndarray:
    """``SwiGLU_e(x[t])`` in fp64 for each requested (token, expert) row."""
    lib = _load()
    xs, xdt = _as_stored(x)
    g, dt = _as_stored(w_gate)
    u, _ = _as_stored(w_up)
    dn, _ = _as_stored(w_down)
    d = xs.shape[1]
    I = g.shape[1]
    tok = np.ascontiguousarray(tok, dtype=np.int32)
    expert = np.ascontiguousarray(expert, dtype=np.int32)
    n = tok.shape[0]
    y = np.empty((n, d), dtype=np.float64)
    lib.oracle_expert_rows(_ptr(xs), xdt, _ptr(g), _ptr(u), _ptr(dn), dt, d, I, n, _ptr(tok), _ptr(expert), _ptr(y))
    return y


def moe_tokens(x, w_gate, w_up, w_down, tok, idx, gate, keep=None, shared=None) -> np.ndarray:
    """``out[i] = sum_j keep[i,j] gate[i,j] SwiGLU_{idx[i,j]}(x[tok[i]])
    + sum_s SharedSwiGLU_s(x[tok[i]])`` in fp64. ``shared`` is None or the
    (gate [S,I,d], up [S,I,d], down [S,d,I]) weights of the shared experts;
    ``idx``/``gate`` may have zero columns (shared experts alone)."""
    lib = _load()
    xs, xdt = _as_stored(x)
    g, dt = _as_stored(w_gate)
    u, _ = _as_stored(w_up)
    dn, _ = _as_stored(w_down)
    d = xs.shape[1]
    I = g.shape[1]
    tok = np.ascontiguousarray(tok, dtype=np.int32)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    gate = np.ascontiguousarray(gate, dtype=np.float64)
    ntok, k = idx.shape
    kp = None if keep is None else np.ascontiguousarray(keep, dtype=np.int8)
    if shared is not None:
        sg, sgdt = _as_stored(shared[0])
        su, _ = _as_stored(shared[1])
        sd, _ = _as_stored(shared[2])
        assert sgdt == dt, "shared and routed experts must share a dtype"
        ns = sg.shape[0]
    else:
        sg = su = sd = None
        ns = 0
    out = np.empty((ntok, d), dtype=np.float64)
    lib.oracle_moe_tokens(_ptr(xs), xdt, _ptr(g), _ptr(u), _ptr(dn), dt, d, I, k, ntok, _ptr(tok), _ptr(idx),
                          _ptr(gate), _ptr(kp), ns, _ptr(sg), _ptr(su), _ptr(sd), _ptr(out))
    return out


@dataclass
class OracleResult:
    probs: np.ndarray  # [T, E] fp64
    topk_idx: np.ndarray  # [T, k] int32
    topk_gate: np.ndarray  # [T, k] fp64
    gap: np.ndarray  # [T] fp64, p_(k) - p_(k+1)
    counts: np.ndarray  # [E] int64, assignments before any capacity drop
    mean_prob: np.ndarray  # [E] fp64
    aux: float
    offsets: np.ndarray  # [E+1] int64, of the kept rows
    perm_tok: np.ndarray  # [R] int32, R kept rows
    inv: np.ndarray  # [T, k] int32, -1 for a dropped slot
    tokens: np.ndarray  # [n] int32, the tokens whose output rows were evaluated
    out: np.ndarray  # [n, d] fp64
    logits: np.ndarray = None  # [T, E] fp64
    z_loss: float = 0.0
    capacity: int = -1  # assignments an expert may keep, -1 = no limit
    dropped: int = 0  # assignments dropped by the capacity
    xhat: np.ndarray = None  # [T, d] fp64 normalised input, when a norm was applied


def forward(x, w_router, b_router, w_gate, w_up, w_down, k: int, renorm: bool, tokens=None, *, norm_form: int = 0, norm_weight=None, norm_eps: float = 1e-5,
            capacity_factor: float = 0.0, shared=None) -> OracleResult:
    """The whole layer. Routing, statistics and dispatch cover every token;
    the expert output is evaluated for ``tokens`` (all tokens if None).

    Options: ``norm_form`` 1 or 2 applies the pre-MoE RMSNorm (weight
    ``norm_weight`` or ones, ``norm_eps``) before the router and the experts;
    ``capacity_factor`` > 0 caps every expert at ceil(cf*T*k/E) assignments;
    ``shared`` = (gate, up, down) adds shared experts with weight 1."""
    xin = x
    xhat = None
    if norm_form:
        xhat = rmsnorm(x, norm_weight, norm_eps, norm_form)
        xin = xhat
    logits = router_logits(xin, w_router, b_router)
    probs = softmax(logits)
    T, E = probs.shape
    idx, gate, gap = topk(probs, k, renorm)
    counts, mean_prob, aux = stats(probs, idx)
    cap = capacity(capacity_factor, T, k, E)
    offsets, perm, inv, dropped = dispatch(idx, E, cap)
    if tokens is None:
        tokens = np.arange(T, dtype=np.int32)
    tokens = np.asarray(tokens, dtype=np.int32)
    keep = (inv[tokens] >= 0) if cap >= 0 else None
    out = moe_tokens(xin, w_gate, w_up, w_down, tokens, idx[tokens], gate[tokens], keep=keep, shared=shared)
    return OracleResult(probs, idx, gate, gap, counts, mean_prob, aux, offsets, perm, inv, tokens, out,
                        logits=logits, z_loss=z_loss(logits), capacity=cap, dropped=dropped, xhat=xhat)
