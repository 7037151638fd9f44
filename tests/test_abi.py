"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every entry point declared in include/moe.h, sizes its workspace, and
rejects bad arguments with the documented status before launching anything
(the validation rules of KempnerForge's ModelConfig.__post_init__ and of
axonml-nn's MoERouter::new: top_k > 0, top_k <= num_experts, positive dims)."""
import ctypes
import os
import re

import pytest

from sparse_mixture_experts_renorm_b200 import _binding as B
from sparse_mixture_experts_renorm_b200 import build as build_mod

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return B.load_library()


def header_functions():
    text = open(os.path.join(ROOT, "include", "moe.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:size_t|moe_status|int|void\s*\*|const char\s*\*)\s*(moe_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_entry_points():
    assert set(B.EXPORTED) <= set(header_functions())


def test_library_exports_every_declared_symbol(lib):
    for name in header_functions():
        assert hasattr(lib, name), name


def test_kernel_names(lib):
    names = B.kernel_names(lib)
    assert names[0] == "router_topk" and names[-1] == "combine" and len(names) == B.MOE_NUM_KERNELS
    assert lib.moe_kernel_name(B.MOE_NUM_KERNELS) is None


def test_forward_events_needs_events(lib):
    fake = ctypes.c_void_p(4096)
    arr = (ctypes.c_void_p * 3)()
    st = lib.moe_forward_events(fake, fake, None, fake, fake, fake, 8, 128, 4, 2, 256, 1, B.MOE_F32, fake, fake, fake,
                                None, None, fake, 1 << 40, None, None, arr, 3)
    assert st == B.MOE_ERR_INVALID_ARG


def test_workspace_size(lib):
    n = lib.moe_workspace_size(4096, 4096, 8, 2, 14336, B.MOE_BF16)
    R = 4096 * 2
    # at least the expert-contiguous x, the hidden activations and the fp32 expert outputs
    assert n >= R * 4096 * 2 + R * 14336 * 2 + R * 4096 * 4
    assert n < R * 4096 * 2 + R * 14336 * 2 + R * 4096 * 4 + 64 * 1024 * 1024
    assert lib.moe_workspace_size(0, 128, 4, 2, 256, B.MOE_F32) > 0


@pytest.mark.parametrize("T,d,E,k,I,dt,expect", [
    (-1, 128, 4, 2, 256, B.MOE_F32, B.MOE_ERR_INVALID_ARG),
    (8, 0, 4, 2, 256, B.MOE_F32, B.MOE_ERR_INVALID_ARG),
    (8, 128, 0, 1, 256, B.MOE_F32, B.MOE_ERR_INVALID_ARG),
    (8, 128, 4, 0, 256, B.MOE_F32, B.MOE_ERR_INVALID_ARG),
    (8, 128, 4, 5, 256, B.MOE_F32, B.MOE_ERR_INVALID_ARG),
    (8, 128, 4, 2, 0, B.MOE_F32, B.MOE_ERR_INVALID_ARG),
    (8, 128, 4, 2, 256, 7, B.MOE_ERR_INVALID_ARG),
    (8, 128, 300, 2, 256, B.MOE_F32, B.MOE_ERR_UNSUPPORTED),
    (8, 128, 16, 9, 256, B.MOE_F32, B.MOE_ERR_UNSUPPORTED),
    (8, 96, 4, 2, 256, B.MOE_BF16, B.MOE_ERR_UNSUPPORTED),
    (8, 128, 4, 2, 200, B.MOE_BF16, B.MOE_ERR_UNSUPPORTED),
    (8, 130, 4, 2, 256, B.MOE_F32, B.MOE_ERR_UNSUPPORTED),
])
def test_shape_validation(lib, T, d, E, k, I, dt, expect):
    assert lib.moe_workspace_size(T, d, E, k, I, dt) == 0
    fake = ctypes.c_void_p(4096)  # never dereferenced: validation fails first
    st = lib.moe_forward(fake, fake, None, fake, fake, fake, T, d, E, k, I, 1, dt, fake, fake, fake, None, None,
                         fake, 1 << 40, None, None)
    assert st == expect
    assert len(B.last_error_detail(lib)) > 0


def test_null_pointers_and_workspace(lib):
    fake = ctypes.c_void_p(4096)
    args = dict(T=8, d=128, E=4, k=2, I=256)
    st = lib.moe_forward(None, fake, None, fake, fake, fake, 8, 128, 4, 2, 256, 1, B.MOE_F32, fake, fake, fake, None,
                         None, fake, 1 << 40, None, None)
    assert st == B.MOE_ERR_INVALID_ARG
    assert "NULL" in B.last_error_detail(lib)
    need = lib.moe_workspace_size(*args.values(), B.MOE_F32)
    st = lib.moe_forward(fake, fake, None, fake, fake, fake, 8, 128, 4, 2, 256, 1, B.MOE_F32, fake, fake, fake, None,
                         None, fake, need - 1, None, None)
    assert st == B.MOE_ERR_WORKSPACE
    st = lib.moe_forward(fake, fake, None, fake, fake, fake, 8, 128, 4, 2, 256, 1, B.MOE_F32, fake, fake, fake, None,
                         None, None, need, None, None)
    assert st == B.MOE_ERR_WORKSPACE
    st = lib.moe_forward(fake, fake, None, fake, fake, fake, 8, 128, 4, 2, 256, 2, B.MOE_F32, fake, fake, fake, None,
                         None, fake, need, None, None)
    assert st == B.MOE_ERR_INVALID_ARG
    misaligned = ctypes.c_void_p(4096 + 8)
    st = lib.moe_forward(misaligned, fake, None, fake, fake, fake, 8, 128, 4, 2, 256, 1, B.MOE_F32, fake, fake, fake,
                         None, None, fake, need, None, None)
    assert st == B.MOE_ERR_INVALID_ARG
    st = lib.moe_forward(fake, fake, None, fake, fake, fake, 8, 128, 4, 2, 256, 1, B.MOE_F32, fake, fake, fake, None,
                         None, ctypes.c_void_p(4096 + 16), need, None, None)
    assert st == B.MOE_ERR_INVALID_ARG
    assert "256-byte" in B.last_error_detail(lib)


def test_get_permutation_validation(lib):
    fake = ctypes.c_void_p(4096)
    st = lib.moe_get_permutation(fake, 16, 8, 128, 4, 2, 256, B.MOE_F32, None, None, None, None)
    assert st == B.MOE_ERR_WORKSPACE
    st = lib.moe_get_permutation(fake, 1 << 30, 8, 128, 4, 5, 256, B.MOE_F32, None, None, None, None)
    assert st == B.MOE_ERR_INVALID_ARG


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(RuntimeError, match="missing"):
        B.load_library(str(tmp_path / "nope.so"))


def test_selftest_argument_checks(lib):
    assert lib.moe_selftest_wait_timeout(None, 50_000_000, None) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_selftest_wait_timeout(ctypes.c_void_p(4096), 10, None) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_selftest_wait_timeout(ctypes.c_void_p(4096), 10**10, None) == B.MOE_ERR_INVALID_ARG


def _opts(**kw):
    o = B.moe_options()
    o.struct_bytes = ctypes.sizeof(B.moe_options)
    for k, v in kw.items():
        setattr(o, k, v)
    return o


def test_options_struct_size_matches_the_library(lib):
    o = _opts()
    assert lib.moe_workspace_size_ex(64, 128, 4, 2, 128, B.MOE_BF16, ctypes.byref(o)) == \
        lib.moe_workspace_size(64, 128, 4, 2, 128, B.MOE_BF16)
    assert lib.moe_workspace_size_ex(64, 128, 4, 2, 128, B.MOE_BF16, None) == \
        lib.moe_workspace_size(64, 128, 4, 2, 128, B.MOE_BF16)


def test_options_grow_the_workspace(lib):
    base = lib.moe_workspace_size(4096, 4096, 8, 2, 14336, B.MOE_BF16)
    sh = _opts(n_shared=1, shared_gate=4096, shared_up=4096, shared_down=4096)
    # one more copy of x (T*d bf16), T more hidden rows (bf16) and T more fp32 output rows
    grow = lib.moe_workspace_size_ex(4096, 4096, 8, 2, 14336, B.MOE_BF16, ctypes.byref(sh)) - base
    assert 4096 * (4096 * 2 + 14336 * 2 + 4096 * 4) <= grow < 4096 * (4096 * 2 + 14336 * 2 + 4096 * 4) + 4096
    nm = _opts(norm_form=B.MOE_NORM_RMS, norm_eps=1e-5)
    assert lib.moe_workspace_size_ex(4096, 4096, 8, 2, 14336, B.MOE_BF16, ctypes.byref(nm)) > base


@pytest.mark.parametrize("field,value,msg", [
    ("struct_bytes", 8, "struct_bytes"),
    ("norm_form", 3, "norm_form"),
    ("n_shared", 9, "n_shared"),
    ("n_shared", -1, "n_shared"),
    ("capacity_factor", -0.5, "capacity_factor"),
    ("capacity_factor", float("nan"), "capacity_factor"),
    ("capacity_factor", float("inf"), "capacity_factor"),
])
def test_invalid_options_are_rejected(lib, field, value, msg):
    o = _opts(**{field: value})
    assert lib.moe_workspace_size_ex(64, 128, 4, 2, 128, B.MOE_BF16, ctypes.byref(o)) == 0
    assert msg in B.last_error_detail(lib)
    fake = ctypes.c_void_p(4096)
    st = lib.moe_forward_ex(fake, fake, None, fake, fake, fake, 64, 128, 4, 2, 128, 1, B.MOE_BF16, ctypes.byref(o),
                            fake, fake, fake, None, None, fake, 1 << 30, None, None, None, 0)
    assert st == B.MOE_ERR_INVALID_ARG


def test_invalid_norm_eps_and_missing_shared_weights(lib):
    fake = ctypes.c_void_p(4096)
    for o in (_opts(norm_form=1, norm_eps=-1.0), _opts(norm_form=1, norm_eps=float("nan")),
              _opts(n_shared=1), _opts(n_shared=1, shared_gate=4096, shared_up=4104, shared_down=4096),
              _opts(norm_form=1, norm_weight=4100)):
        st = lib.moe_forward_ex(fake, fake, None, fake, fake, fake, 64, 128, 4, 2, 128, 1, B.MOE_BF16,
                                ctypes.byref(o), fake, fake, fake, None, None, fake, 1 << 30, None, None, None, 0)
        assert st == B.MOE_ERR_INVALID_ARG, B.last_error_detail(lib)


def test_forward_ex_event_count_is_checked(lib):
    fake = ctypes.c_void_p(4096)
    evs = (ctypes.c_void_p * 3)(4096, 4096, 4096)
    st = lib.moe_forward_ex(fake, fake, None, fake, fake, fake, 64, 128, 4, 2, 128, 1, B.MOE_BF16, None,
                            fake, fake, fake, None, None, fake, 1 << 30, None, None, evs, 3)
    assert st == B.MOE_ERR_INVALID_ARG


def test_launch_plan(lib):
    """Which kernels a call merges: the combine into the down GEMM for bf16
    k = 2 without shared experts; both projections into one kernel for bf16
    batches of 1..32 tokens; the routing scan into the router for bf16
    batches of one router block (1..128 tokens) with at most 16 experts, else
    into the permute while router blocks x E <= 4096; an extra split of
    w * W_r for the bf16 norm with a weight; -1 for invalid arguments."""
    bf, f32 = B.MOE_BF16, B.MOE_F32
    assert lib.moe_launch_plan(32, 4096, 8, 2, 14336, bf, None) == (B.MOE_PLAN_FUSED_COMBINE | B.MOE_PLAN_FUSED_GEMMS
                                                                     | B.MOE_PLAN_FUSED_SCAN)
    assert lib.moe_launch_plan(33, 4096, 8, 2, 14336, bf, None) == B.MOE_PLAN_FUSED_COMBINE | B.MOE_PLAN_FUSED_SCAN
    assert lib.moe_launch_plan(129, 4096, 8, 2, 14336, bf, None) == (B.MOE_PLAN_FUSED_COMBINE
                                                                      | B.MOE_PLAN_PERMUTE_SCAN)
    assert lib.moe_launch_plan(100, 256, 17, 2, 256, bf, None) == (B.MOE_PLAN_FUSED_COMBINE  # E > 16
                                                                   | B.MOE_PLAN_PERMUTE_SCAN)
    assert lib.moe_launch_plan(4096, 4096, 8, 2, 14336, bf, None) == (B.MOE_PLAN_FUSED_COMBINE
                                                                       | B.MOE_PLAN_PERMUTE_SCAN)
    assert lib.moe_launch_plan(16384, 2048, 64, 6, 1408, bf, None) == 0  # 128 blocks x 64 experts
    assert lib.moe_launch_plan(65664, 4096, 8, 2, 14336, bf, None) == B.MOE_PLAN_FUSED_COMBINE  # 513 x 8
    assert lib.moe_launch_plan(64, 128, 4, 2, 256, f32, None) == B.MOE_PLAN_PERMUTE_SCAN
    assert lib.moe_launch_plan(0, 4096, 8, 2, 14336, bf, None) == B.MOE_PLAN_FUSED_COMBINE
    o = B.moe_options()
    o.struct_bytes = ctypes.sizeof(B.moe_options)
    o.norm_form, o.norm_eps, o.norm_weight = B.MOE_NORM_RMS, 1e-5, 256
    o.n_shared = 1
    o.shared_gate = o.shared_up = o.shared_down = 256
    assert lib.moe_launch_plan(32, 4096, 8, 2, 14336, bf, ctypes.byref(o)) == (B.MOE_PLAN_FUSED_GEMMS
                                                                           | B.MOE_PLAN_ROUTER_WEIGHT_SPLIT
                                                                           | B.MOE_PLAN_FUSED_SCAN)
    assert lib.moe_launch_plan(32, 4096, 8, 9, 14336, bf, None) == -1  # k > E
    # fold_combine: the combine in the down GEMM for every k (bf16, no shared experts)
    f = B.moe_options()
    f.struct_bytes = ctypes.sizeof(B.moe_options)
    f.fold_combine = 1
    assert lib.moe_launch_plan(16384, 2048, 64, 6, 1408, bf, ctypes.byref(f)) == B.MOE_PLAN_FUSED_COMBINE
    assert lib.moe_launch_plan(32, 4096, 8, 1, 14336, bf, ctypes.byref(f)) == (B.MOE_PLAN_FUSED_COMBINE
                                                                           | B.MOE_PLAN_FUSED_GEMMS
                                                                           | B.MOE_PLAN_FUSED_SCAN)
    assert lib.moe_launch_plan(64, 128, 4, 3, 256, f32, ctypes.byref(f)) == B.MOE_PLAN_PERMUTE_SCAN
    f.n_shared = 1
    f.shared_gate = f.shared_up = f.shared_down = 256
    assert lib.moe_launch_plan(16384, 2048, 64, 6, 1408, bf, ctypes.byref(f)) == 0


def test_pipeline_rejects_bad_arguments_before_any_cuda_call(lib):
    """moe_pipeline_create validates its description on the host: a NULL
    handle pointer or description, a short struct, an invalid shape and
    missing device slots are refused before a stream or event is made."""
    h = ctypes.c_void_p()
    assert lib.moe_pipeline_create(None, None, ctypes.byref(h)) == B.MOE_ERR_INVALID_ARG
    desc = B.moe_layer_desc()
    desc.struct_bytes = ctypes.sizeof(B.moe_layer_desc)
    assert lib.moe_pipeline_create(ctypes.byref(desc), None, None) == B.MOE_ERR_INVALID_ARG
    desc.struct_bytes = 8
    assert lib.moe_pipeline_create(ctypes.byref(desc), None, ctypes.byref(h)) == B.MOE_ERR_INVALID_ARG
    desc.struct_bytes = ctypes.sizeof(B.moe_layer_desc)
    desc.T, desc.d, desc.E, desc.k, desc.I, desc.renorm, desc.dtype = 32, 4096, 8, 9, 14336, 1, B.MOE_BF16
    assert lib.moe_pipeline_create(ctypes.byref(desc), None, ctypes.byref(h)) == B.MOE_ERR_INVALID_ARG  # k > E
    desc.k = 2
    assert lib.moe_pipeline_create(ctypes.byref(desc), None, ctypes.byref(h)) == B.MOE_ERR_INVALID_ARG  # no slots
    assert "x_dev" in B.last_error_detail(lib)
    assert h.value is None
    assert lib.moe_pipeline_destroy(None) == B.MOE_OK
    assert lib.moe_pipeline_stream(None, 0) is None


def _c_layout(struct, fields, tmp_path):
    """sizeof and offsetof of `fields` of `struct` as gcc lays out the
    declarations of include/moe.h (a host program compiled for this test)."""
    import subprocess

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    lines = [f'printf("%zu\\n", sizeof({struct}));'] + [f'printf("%zu\\n", offsetof({struct}, {f}));' for f in fields]
    src = tmp_path / "layout.c"
    src.write_text("#include <stdio.h>\n#include <stddef.h>\n#include \"moe.h\"\nint main(void) {\n"
                   + "\n".join(lines) + "\nreturn 0;\n}\n")
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c99", "-I", os.path.join(root, "include"), str(src), "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()
    return int(out[0]), [int(v) for v in out[1:]]


@pytest.mark.parametrize("cls,struct", [(B.moe_options, "moe_options"), (B.moe_layer_desc, "moe_layer_desc")])
def test_ctypes_structs_match_the_header(cls, struct, tmp_path):
    """The binding's ctypes mirrors of the option and pipeline structs have
    the header's size and field offsets (a field added on one side only
    would shift every later field)."""
    names = [f[0] for f in cls._fields_]
    size, offsets = _c_layout(struct, names, tmp_path)
    assert ctypes.sizeof(cls) == size
    assert [getattr(cls, n).offset for n in names] == offsets
