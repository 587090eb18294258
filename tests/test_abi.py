"""The C-ABI library: it builds, loads, exports every symbol include/nabla.h
declares, and rejects bad arguments before touching the GPU."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    text = open(os.path.join(ROOT, "include", "nabla.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^NABLA_API [\w\s\*]*?\b((?:nabla|bsa)_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def nl():
    import block_sparse_attention_23_b200 as nl
    nl.build()
    return nl


def test_header_declares_the_boundary():
    names = _declared_functions()
    for required in ("nabla_build_mask", "bsa_fwd", "bsa_fwd_with_mask", "nabla_workspace_size",
                     "nabla_last_error", "nabla_query_status"):
        assert required in names


def test_library_exports_every_declared_symbol(nl):
    lib = nl.lib()
    for name in _declared_functions():
        assert hasattr(lib, name), name
    assert set(_declared_functions()) <= set(nl.EXPORTED)


def test_no_torch_types_in_signatures():
    text = open(os.path.join(ROOT, "include", "nabla.h")).read()
    assert "torch" not in text.lower().replace("pytorch", "")
    assert "extern \"C\"" in text


def test_version_and_workspace_sizes(nl):
    lib = nl.lib()
    assert lib.nabla_version() >= 100
    s = nl.make_shape(1, 40, 76800, 128, (5, 12, 20))
    n_fwd = nl.workspace_size(s, nl.OP_FWD)
    n_build = nl.workspace_size(s, nl.OP_BUILD_MASK)
    n_mask = nl.workspace_size(s, nl.OP_FWD_WITH_MASK)
    assert n_fwd == 256
    # raster token order: the header plus tile-major copies of K and V
    r = nl.make_shape(1, 40, 76800, 128, (5, 12, 20), nl.LAYOUT_RASTER)
    assert nl.workspace_size(r, nl.OP_FWD) == 256 + 2 * 40 * 76800 * 128 * 2
    assert nl.workspace_size(r, nl.OP_FWD_WITH_MASK) == n_mask + 2 * 40 * 76800 * 128 * 2
    nb = 1200
    # pooled Q and K + reduced map + bitmap + counts
    assert n_build >= 2 * 40 * nb * 128 * 4 + 40 * nb * nb * 4
    assert n_mask >= 40 * nb * nb * 4


@pytest.mark.parametrize("shape,status", [
    ((1, 1, 100, 64), 2),          # S % 64 != 0
    ((1, 1, 128, 96), 2),          # d unsupported
    ((0, 1, 128, 64), 1),          # bad size
    ((1, 1, 64 * 4097, 64), 2),    # nb > 4096
])
def test_bad_shapes_rejected(nl, shape, status):
    s = nl.make_shape(*shape)
    assert nl.lib().nabla_workspace_size(ctypes.byref(s), 0) == 0
    prm = nl._MaskParams(0.2, 0, 0, 0, 0)
    null = ctypes.c_void_p(0)
    dummy = ctypes.c_void_p(1 << 20)
    rc = nl.lib().nabla_build_mask(ctypes.byref(s), ctypes.byref(prm), dummy, dummy, null, dummy,
                                   dummy, 10, null, dummy, null)
    assert rc == status


def test_argument_errors_before_any_cuda_call(nl):
    lib = nl.lib()
    null = ctypes.c_void_p(0)
    a = ctypes.c_void_p(1 << 20)
    s = nl.make_shape(1, 1, 128, 64, (1, 1, 2))
    prm = nl._MaskParams(0.2, 0, 0, 0, 0)
    assert lib.nabla_build_mask(None, ctypes.byref(prm), a, a, null, a, a, 4, null, a, null) == 1
    assert lib.nabla_build_mask(ctypes.byref(s), None, a, a, null, a, a, 4, null, a, null) == 1
    bad = nl._MaskParams(1.5, 0, 0, 0, 0)
    assert lib.nabla_build_mask(ctypes.byref(s), ctypes.byref(bad), a, a, null, a, a, 4, null, a,
                                null) == 2
    wrong_grid = nl.make_shape(1, 1, 128, 64, (1, 1, 3))
    assert lib.nabla_build_mask(ctypes.byref(wrong_grid), ctypes.byref(prm), a, a, null, a, a, 4,
                                null, a, null) == 1
    neg = nl._MaskParams(0.2, 1, -1, 0, 0)
    assert lib.nabla_build_mask(ctypes.byref(s), ctypes.byref(neg), a, a, null, a, a, 4, null, a,
                                null) == 1
    # null q / misaligned pointers
    assert lib.bsa_fwd(ctypes.byref(s), null, a, a, a, a, 0.0, a, null, a, null) == 1
    odd = ctypes.c_void_p((1 << 20) + 2)
    assert lib.bsa_fwd(ctypes.byref(s), odd, a, a, a, a, 0.0, a, null, a, null) == 1
    assert lib.bsa_fwd_with_mask(ctypes.byref(s), a, a, a, null, 0.0, a, null, a, null) == 1
    assert lib.bsa_fwd(ctypes.byref(s), a, a, a, a, a, float("nan"), a, null, a, null) == 1
    assert "scale" in lib.nabla_last_error().decode()
    assert lib.nabla_selftest_mma(7, a, a, a, a, null) == 1


def test_product_path_has_no_cpu_fallback(nl):
    import torch
    if torch.cuda.is_available():
        pytest.skip("CUDA present")
    q = torch.zeros((1, 1, 64, 64), dtype=torch.bfloat16)
    with pytest.raises(RuntimeError):
        nl.bsa_fwd_with_mask(q, q, q, torch.ones((1, 1, 1, 1), dtype=torch.uint8))


def test_package_does_not_import_oracle():
    pkg = os.path.join(ROOT, "block_sparse_attention_23_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".c")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f
                assert "nabla_oracle" not in text, f


def test_topk_argument_checked(nl):
    lib = nl.lib()
    null = ctypes.c_void_p(0)
    a = ctypes.c_void_p(1 << 20)
    s = nl.make_shape(1, 1, 128, 64, (1, 1, 2))
    prm = nl._MaskParams(0.2, 0, 0, 0, 0, -3)
    assert lib.nabla_build_mask(ctypes.byref(s), ctypes.byref(prm), a, a, null, a, a, 4, null, a,
                                null) == 1
    assert lib.nabla_version() >= 200


def test_reorder_arguments_checked(nl):
    lib = nl.lib()
    null = ctypes.c_void_p(0)
    a, b = ctypes.c_void_p(1 << 20), ctypes.c_void_p(1 << 21)
    good = nl.make_shape(1, 2, 128, 64, (1, 1, 2))
    bad_s = nl.make_shape(1, 2, 192, 64, (1, 1, 2))
    bad_d = nl.make_shape(1, 2, 128, 60, (1, 1, 2))
    f = lib.nabla_reorder_tokens
    assert f(None, 0, a, b, null) == 1
    assert f(ctypes.byref(bad_s), 0, a, b, null) == 1
    assert f(ctypes.byref(bad_d), 0, a, b, null) == 2
    assert f(ctypes.byref(good), 7, a, b, null) == 1
    assert f(ctypes.byref(good), 0, null, b, null) == 1
    assert f(ctypes.byref(good), 0, a, a, null) == 1
    assert f(ctypes.byref(good), 1, ctypes.c_void_p((1 << 20) + 8), b, null) == 1


def test_layout_arguments_checked(nl):
    lib = nl.lib()
    null = ctypes.c_void_p(0)
    a = ctypes.c_void_p(1 << 20)
    no_grid = nl.make_shape(1, 1, 128, 64, (0, 0, 0), nl.LAYOUT_RASTER)
    bad = nl.make_shape(1, 1, 128, 64, (1, 1, 2), 7)
    raster = nl.make_shape(1, 1, 128, 64, (1, 1, 2), nl.LAYOUT_RASTER)
    f = lib.bsa_fwd
    assert f(ctypes.byref(no_grid), a, a, a, a, a, ctypes.c_float(0), a, a, a, null) == 1
    assert f(ctypes.byref(bad), a, a, a, a, a, ctypes.c_float(0), a, a, a, null) == 1
    # the backward and the energy kernel take tile-major tokens only
    assert lib.bsa_bwd(ctypes.byref(raster), a, a, a, a, a, a, a, a, ctypes.c_float(0), a, a, a,
                       a, null) == 2
    assert lib.nabla_block_energy(ctypes.byref(raster), a, a, a, a, a, ctypes.c_float(0), a,
                                  null, a, null) == 2
    assert lib.nabla_version() >= 210


def test_layer_host_arguments_checked(nl):
    lib = nl.lib()
    null = ctypes.c_void_p(0)
    a = ctypes.c_void_p(1 << 20)
    s = nl.make_shape(1, 40, 76800, 128, (5, 12, 20))
    prm = nl._MaskParams(0.2, 1, 1, 2, 2, 0)
    one = lib.nabla_layer_host_workspace_size(ctypes.byref(s), 4)
    # two slots of 4 heads (Q, K, V, O and LSE) beyond one chunk's mask workspace
    assert one >= 2 * (4 * 4 * 76800 * 128 * 2 + 4 * 76800 * 4)
    assert one > lib.nabla_layer_host_workspace_size(ctypes.byref(s), 2)
    assert lib.nabla_layer_host_workspace_size(ctypes.byref(s), 0) == 0
    bad = nl.make_shape(1, 40, 76800, 96, (5, 12, 20))
    assert lib.nabla_layer_host_workspace_size(ctypes.byref(bad), 4) == 0
    f = lib.nabla_layer_host
    assert f(ctypes.byref(s), ctypes.byref(prm), a, a, a, a, a, 0, a, null) == 1
    assert f(ctypes.byref(s), ctypes.byref(prm), a, null, a, a, a, 4, a, null) == 1
    assert f(ctypes.byref(bad), ctypes.byref(prm), a, a, a, a, a, 4, a, null) == 1
    raster = nl.make_shape(1, 40, 76800, 128, (5, 12, 20), nl.LAYOUT_RASTER)
    assert f(ctypes.byref(raster), ctypes.byref(prm), a, a, a, a, a, 4, a, null) == 2
    # the workspace must be 256-byte aligned
    assert f(ctypes.byref(s), ctypes.byref(prm), a, a, a, a, a, 4,
             ctypes.c_void_p((1 << 20) + 16), null) == 1
    assert lib.nabla_version() >= 220


@pytest.mark.parametrize("heads,hpc", [(40, 8), (40, 4), (40, 1), (40, 64), (1, 4), (2, 8),
                                       (3, 2), (24, 6), (96, 16), (7, 7)])
def test_layer_host_chunk_schedule(nl, heads, hpc):
    sizes = nl.layer_host_chunks(heads, hpc)
    assert sum(sizes) == heads
    assert all(1 <= s <= hpc for s in sizes)
    assert sizes[0] == 1
    # ramp: each chunk at most twice the one before it until the full size
    for a, b in zip(sizes, sizes[1:]):
        if a < hpc // 2:
            assert b <= 2 * a
    assert nl.layer_host_chunks(0, hpc) == [] and nl.layer_host_chunks(heads, 0) == []


def test_layer_host_schedule_wan(nl):
    assert nl.layer_host_chunks(40, 8) == [1, 2, 4, 8, 8, 8, 7, 2]


def test_layer_host_rejects_bad_mask_params_before_queuing(nl):
    # the mask parameters are checked before any copy or CUDA call
    lib = nl.lib()
    null = ctypes.c_void_p(0)
    a = ctypes.c_void_p(1 << 20)
    s = nl.make_shape(1, 4, 1024, 64, (4, 2, 2))
    f = lib.nabla_layer_host
    bad_thr = nl._MaskParams(1.5, 0, 0, 0, 0, 0)
    assert f(ctypes.byref(s), ctypes.byref(bad_thr), a, a, a, a, a, 2, a, null) == 2
    bad_topk = nl._MaskParams(0.2, 0, 0, 0, 0, -1)
    assert f(ctypes.byref(s), ctypes.byref(bad_topk), a, a, a, a, a, 2, a, null) == 1
    bad_sta = nl._MaskParams(0.2, 1, -1, 0, 0, 0)
    assert f(ctypes.byref(s), ctypes.byref(bad_sta), a, a, a, a, a, 2, a, null) == 1
    no_grid = nl.make_shape(1, 4, 1024, 64, (4, 2, 3))
    ok = nl._MaskParams(0.2, 0, 0, 0, 0, 0)
    assert f(ctypes.byref(no_grid), ctypes.byref(ok), a, a, a, a, a, 2, a, null) == 1


def test_forward_refuses_a_workspace_too_small_for_raster_order(nl):
    """A raster-order forward writes tile-major K/V copies into its workspace:
    the binding refuses a buffer sized for tile-major tokens before any device
    call (the check bsa_fwd and bsa_fwd_with_mask run first)."""
    import torch
    shape = nl.make_shape(1, 2, 64 * 6, 64, (1, 2, 3), nl.LAYOUT_RASTER)
    small = nl.Workspace(torch.empty(256, dtype=torch.uint8), nl.OP_FWD)
    with pytest.raises(ValueError, match="workspace holds 256 bytes"):
        nl._check_workspace(small, shape, nl.OP_FWD)
    big = nl.Workspace(torch.empty(nl.workspace_size(shape, nl.OP_FWD), dtype=torch.uint8), nl.OP_FWD)
    nl._check_workspace(big, shape, nl.OP_FWD)


def test_exact_pass_counter_query_rejects_null(nl):
    lib = nl.lib()
    assert lib.nabla_query_exact_passes(None, None) == -1
    assert "NULL" in lib.nabla_last_error().decode()
    lib.nabla_set_exact_reference(0)          # the default; a no-op without a GPU


def test_diagnostics_reject_bad_arguments_before_any_cuda_call(nl):
    """The stage-timing and self-test calls check their arguments on the host
    (no GPU needed to see the rejections)."""
    lib = nl.lib()
    s = nl.make_shape(1, 2, 64 * 12, 128, (1, 3, 4))
    prm = nl._MaskParams(0.2, 0, 0, 0, 0, 0)
    a = ctypes.c_void_p(1 << 20)
    # a null ms_out is refused before the build runs
    rc = lib.nabla_build_mask_stage_ms(ctypes.byref(s), ctypes.byref(prm), a, a, a, a, 10, a, a,
                                       None, None)
    assert rc == 1 and "ms_out" in lib.nabla_last_error().decode()
    assert lib.nabla_selftest_fp64_tflops(None, None) == 1
    assert lib.nabla_selftest_fp64_exp_rate(None, None) == 1
    assert lib.nabla_selftest_ex2_rate(None, None) == 1
    assert lib.nabla_selftest_mma_pair(2, a, a, a, a, None) == 1
    assert "variant" in lib.nabla_last_error().decode()
    assert lib.nabla_selftest_mma_pair(0, None, a, a, a, None) == 1



def test_calibration_xattn_and_init_arguments_checked(nl):
    """The calibration calls, the XAttention builder and the workspace initialiser
    reject bad arguments on the host, before any CUDA call (no GPU needed)."""
    lib = nl.lib()
    null = ctypes.c_void_p(0)
    a = ctypes.c_void_p(1 << 20)
    s = nl.make_shape(1, 2, 64 * 12, 128, (1, 3, 4))
    assert lib.nabla_workspace_init(None, None) == 1
    # nabla_calib_accumulate: eps outside [0, 1] (or NaN) is unsupported, null buffers invalid
    assert lib.nabla_calib_accumulate(None, a, 0.1, a, None) == 1
    assert lib.nabla_calib_accumulate(ctypes.byref(s), a, 1.5, a, None) == 2
    assert lib.nabla_calib_accumulate(ctypes.byref(s), a, float("nan"), a, None) == 2
    assert lib.nabla_calib_accumulate(ctypes.byref(s), null, 0.1, a, None) == 1
    assert lib.nabla_calib_accumulate(ctypes.byref(s), a, 0.1, null, None) == 1
    # nabla_calib_finalize: at least one vote, both buffers given
    assert lib.nabla_calib_finalize(ctypes.byref(s), a, 0, a, None) == 1
    assert "min_votes" in lib.nabla_last_error().decode()
    assert lib.nabla_calib_finalize(ctypes.byref(s), null, 1, a, None) == 1
    assert lib.nabla_calib_finalize(ctypes.byref(s), a, 1, null, None) == 1
    # nabla_build_mask_xattn
    prm = nl._MaskParams(0.2, 0, 0, 0, 0, 0)

    def xattn(shape, params, stride, q=a, row_ptr=a, cap=10, col=a, ws=a):
        return lib.nabla_build_mask_xattn(shape, params, stride, q, a, null, null, row_ptr, col,
                                          cap, null, ws, None)

    assert xattn(ctypes.byref(s), None, 8) == 1
    assert xattn(ctypes.byref(s), ctypes.byref(prm), 5) == 2
    assert "stride" in lib.nabla_last_error().decode()
    assert xattn(ctypes.byref(s), ctypes.byref(nl._MaskParams(1.5, 0, 0, 0, 0, 0)), 8) == 2
    assert xattn(ctypes.byref(s), ctypes.byref(nl._MaskParams(0.2, 0, 0, 0, 0, -1)), 8) == 1
    assert xattn(ctypes.byref(s), ctypes.byref(nl._MaskParams(0.2, 1, -1, 0, 0, 0)), 8) == 1
    bad_grid = nl.make_shape(1, 2, 64 * 12, 128, (1, 3, 5))
    assert xattn(ctypes.byref(bad_grid), ctypes.byref(nl._MaskParams(0.2, 1, 1, 1, 1, 0)), 8) == 1
    assert xattn(ctypes.byref(s), ctypes.byref(prm), 8, q=null) == 1
    assert xattn(ctypes.byref(s), ctypes.byref(prm), 8, cap=-1) == 1
    assert xattn(ctypes.byref(s), ctypes.byref(prm), 8, col=null) == 1
    assert xattn(ctypes.byref(s), ctypes.byref(prm), 8, q=ctypes.c_void_p((1 << 20) + 8)) == 1
    assert xattn(ctypes.byref(s), ctypes.byref(prm), 8, ws=ctypes.c_void_p((1 << 20) + 16)) == 1
    raster = nl.make_shape(1, 2, 64 * 12, 128, (1, 3, 4), nl.LAYOUT_RASTER)
    assert xattn(ctypes.byref(raster), ctypes.byref(prm), 8) == 2
