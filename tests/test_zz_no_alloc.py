"""moe_forward_noalloc, the entry point that allocates nothing, against
moe_forward, the entry point that takes a caller workspace.

Some callers of this library can't call cudaMalloc while they run the layer:
code inside an engine or plugin whose framework owns every device
allocation, or a serving loop that forbids allocation after warm-up so that
its memory use stays fixed. For them the library keeps its scratch in a fixed
16 MiB array of its own. Both entry points run the same kernels on the same
inputs, so the results must be bit-identical. The test calls the no-alloc
entry point through the C ABI twice in a row, on two different batches (so
the second call cannot pass by reading what the first one left in the shared
array), then without a status word of the caller (the library then keeps
and clears its own status word inside the shared array) once on a batch
with a non-finite value, which sets that word, and once on a clean batch;
every output is compared with the ordinary entry point bit for bit. This file is collected last so that a run stopping at the first
failure has already run every other test.
"""
import ctypes

import pytest
import torch

from sparse_mixture_experts_renorm_b200 import _binding as B
from sparse_mixture_experts_renorm_b200 import moe_forward
from sparse_mixture_experts_renorm_b200.workloads import WORKLOADS, make_inputs, make_tokens

pytestmark = pytest.mark.gpu


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _forward_noalloc(lib, inp, x, wl, with_status=True):
    dev = x.device
    out = torch.empty((wl.T, wl.d), dtype=torch.float32, device=dev)
    idx = torch.empty((wl.T, wl.k), dtype=torch.int32, device=dev)
    gate = torch.empty((wl.T, wl.k), dtype=torch.float32, device=dev)
    counts = torch.empty((wl.E,), dtype=torch.int32, device=dev)
    aux = torch.empty((1,), dtype=torch.float32, device=dev)
    status = torch.zeros((1,), dtype=torch.int32, device=dev) if with_status else None
    st = lib.moe_forward_noalloc(_p(x), _p(inp.w_router), _p(inp.b_router), _p(inp.w_gate), _p(inp.w_up),
                                 _p(inp.w_down), wl.T, wl.d, wl.E, wl.k, wl.I, int(wl.renorm), B.MOE_BF16, _p(out),
                                 _p(idx), _p(gate), _p(counts), _p(aux), _p(status),
                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == B.MOE_OK, B.last_error_detail(lib)
    return out, idx, gate, counts, aux, status


def test_noalloc_matches_the_workspace_entry_point_on_two_calls_in_a_row():
    lib = B.load_library()
    wl = WORKLOADS["mixtral_decode"]  # a 32-token decode batch: about 3.3 MB of scratch
    need = lib.moe_workspace_size(wl.T, wl.d, wl.E, wl.k, wl.I, B.MOE_BF16)
    assert 0 < need <= B.MOE_NOALLOC_SCRATCH_BYTES
    inp = make_inputs(wl, "cuda", 0)
    batches = [inp.x, make_tokens(wl, wl.T, "cuda", seed=7)]
    for x in batches:
        ref = moe_forward(x, inp.w_router, inp.b_router, inp.w_gate, inp.w_up, inp.w_down, wl.k, wl.renorm)
        out, idx, gate, counts, aux, status = _forward_noalloc(lib, inp, x, wl)
        torch.cuda.synchronize()
        assert int(status.item()) == 0 and int(ref.status.item()) == 0
        _assert_identical(ref, out, idx, gate, counts, aux)


def test_noalloc_without_a_status_word():
    """With status_dev NULL the entry point keeps its status word in the
    shared array and clears it itself. A first such call on a batch with a
    non-finite value sets that word (MOE_DEV_NONFINITE); the next call on a
    clean batch must still succeed and match the workspace entry point."""
    lib = B.load_library()
    wl = WORKLOADS["mixtral_decode"]
    inp = make_inputs(wl, "cuda", 0)
    bad = make_tokens(wl, wl.T, "cuda", seed=11)
    bad[3, 5] = float("inf")
    _forward_noalloc(lib, inp, bad, wl, with_status=False)
    torch.cuda.synchronize()
    x = make_tokens(wl, wl.T, "cuda", seed=12)
    ref = moe_forward(x, inp.w_router, inp.b_router, inp.w_gate, inp.w_up, inp.w_down, wl.k, wl.renorm)
    out, idx, gate, counts, aux, _ = _forward_noalloc(lib, inp, x, wl, with_status=False)
    torch.cuda.synchronize()
    assert int(ref.status.item()) == 0
    _assert_identical(ref, out, idx, gate, counts, aux)


def _assert_identical(ref, out, idx, gate, counts, aux):
    assert torch.equal(idx, ref.topk_idx)
    assert torch.equal(counts, ref.counts)
    assert torch.equal(gate, ref.topk_gate)
    assert torch.equal(aux, ref.aux)
    assert torch.isfinite(out).all()
    assert torch.equal(out, ref.out)


def test_noalloc_rejects_a_shape_beyond_its_scratch():
    lib = B.load_library()
    wl = WORKLOADS["mixtral_prefill"]  # needs ~430 MB of scratch
    assert lib.moe_workspace_size(wl.T, wl.d, wl.E, wl.k, wl.I, B.MOE_BF16) > B.MOE_NOALLOC_SCRATCH_BYTES
    fake = ctypes.c_void_p(4096)  # never dereferenced: the size check comes first
    st = lib.moe_forward_noalloc(fake, fake, None, fake, fake, fake, wl.T, wl.d, wl.E, wl.k, wl.I, 1, B.MOE_BF16,
                                 fake, fake, fake, None, None, None, None)
    assert st == B.MOE_ERR_WORKSPACE
    assert "static scratch" in B.last_error_detail(lib)
