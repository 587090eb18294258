"""bsa_fwd_with_mask_static: the attention entry point for callers that cannot
allocate device memory (memory-pool runtimes, code running inside another
framework's graph capture, fixed-budget hosts).  It keeps its block CSR in a
fixed library-owned device array instead of a caller workspace.

The GPU test calls it through the C ABI twice in a row, with different masks
and inputs, and checks each result against bsa_fwd_with_mask (the entry point
with a caller workspace) within the attention tolerance used throughout the
tests, and against the fp64 oracle.  This file is named to be collected last."""
import ctypes

import numpy as np
import pytest

from _parity import compare_attention, to_device_bf16


@pytest.fixture(scope="module")
def nl():
    import block_sparse_attention_23_b200 as nl
    nl.build()
    nl.lib()
    return nl


def test_oversized_shape_rejected_before_any_cuda_call(nl):
    lib = nl.lib()
    s = nl.make_shape(1, 40, 76800, 128)        # 57.6 M blocks: far beyond 32 MiB
    a = ctypes.c_void_p(1 << 20)
    rc = lib.bsa_fwd_with_mask_static(ctypes.byref(s), a, a, a, a, 0.0, a, a, None, None)
    assert rc == 2                              # NABLA_ERR_UNSUPPORTED
    msg = lib.nabla_last_error().decode()
    assert "scratch" in msg and str(32 * 1024 * 1024) in msg
    assert rc == 2 and lib.bsa_fwd_with_mask_static(None, a, a, a, a, 0.0, a, a, None, None) == 1


def test_invalid_arguments_rejected_before_any_work(nl):
    """Every argument check runs before the entry point touches the shared
    scratch or the GPU: a raster tile grid that does not cover S/64, a
    misaligned pointer, a non-finite scale."""
    lib = nl.lib()
    a = ctypes.c_void_p(1 << 20)
    bad_grid = nl.make_shape(1, 2, 64 * 30, 128, (3, 2, 4), nl.LAYOUT_RASTER)   # 24 != 30
    rc = lib.bsa_fwd_with_mask_static(ctypes.byref(bad_grid), a, a, a, a, 0.0, a, a, None, None)
    assert rc == 1 and "tile grid" in lib.nabla_last_error().decode()
    s = nl.make_shape(1, 2, 64 * 30, 128)
    odd = ctypes.c_void_p((1 << 20) + 8)
    rc = lib.bsa_fwd_with_mask_static(ctypes.byref(s), odd, a, a, a, 0.0, a, a, None, None)
    assert rc == 1 and "alignment" in lib.nabla_last_error().decode()
    rc = lib.bsa_fwd_with_mask_static(ctypes.byref(s), a, a, a, a, float("inf"), a, a, None, None)
    assert rc == 1 and "finite" in lib.nabla_last_error().decode()
    rc = lib.bsa_fwd_with_mask_static(ctypes.byref(s), a, a, a, None, 0.0, a, a, None, None)
    assert rc == 1


def _call_static(nl, shape, q, k, v, mask, o, lse, status):
    import torch
    rc = nl.lib().bsa_fwd_with_mask_static(
        ctypes.byref(shape), ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
        ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(mask.data_ptr()), ctypes.c_float(0.0),
        ctypes.c_void_p(o.data_ptr()), ctypes.c_void_p(lse.data_ptr()),
        ctypes.c_void_p(status.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, nl.lib().nabla_last_error().decode()


@pytest.mark.gpu
def test_static_scratch_matches_workspace_entry_point_twice(nl, synth_mod, oracle_mod):
    """Two calls in a row with different masks and inputs: each result against
    bsa_fwd_with_mask (same tolerance as every attention test) and, as an
    independent check, against the fp64 oracle on every row."""
    import torch
    B, H, nb, d = 1, 6, 96, 128
    S = 64 * nb
    shape = nl.make_shape(B, H, S, d)
    for call, (p, seed) in enumerate([(0.4, 21), (0.1, 22)]):
        q16 = synth_mod.make_tensor(0, seed, B, H, S, d, pos_weight=0.0, noise_weight=1.0)
        k16 = synth_mod.make_tensor(1, seed, B, H, S, d, pos_weight=0.0, noise_weight=1.0)
        v16 = synth_mod.make_tensor(2, seed, B, H, S, d, pos_weight=0.0, noise_weight=1.0)
        q, k, v = to_device_bf16(q16), to_device_bf16(k16), to_device_bf16(v16)
        mask_np = synth_mod.make_bernoulli_mask(seed, B * H, nb, p).reshape(B, H, nb, nb)
        mask_np[0, 0, 3, :] = 0                  # one empty row
        mask = torch.from_numpy(mask_np).cuda()
        o_s = torch.full_like(q, float("nan"))
        lse_s = torch.full((B, H, S), float("nan"), dtype=torch.float32, device=q.device)
        status = torch.full((1,), -1, dtype=torch.int32, device=q.device)
        _call_static(nl, shape, q, k, v, mask, o_s, lse_s, status)
        o_w, lse_w = nl.bsa_fwd_with_mask(q, k, v, mask)
        torch.cuda.synchronize()
        assert int(status.item()) == 0, f"call {call}: device status {int(status.item())}"
        go = o_s.float().cpu().numpy().reshape(-1, d)
        gl = lse_s.cpu().numpy().reshape(-1)
        ref_o = o_w.double().cpu().numpy().reshape(-1, d)
        ref_l = lse_w.double().cpu().numpy().reshape(-1)
        compare_attention(go, gl, ref_o, ref_l)
        ro, rl = oracle_mod.masked_attention(q16, k16, v16, mask_np)
        compare_attention(go, gl, ro, rl)


@pytest.mark.gpu
def test_static_entry_raster_reads_kv_in_place(nl, synth_mod):
    """Raster token order on the allocation-free entry point: with no room for
    tile-major K/V copies, the kernel reads K and V through 5D boxes; the
    result is bitwise the tile-major one, reordered."""
    import torch
    from test_gpu_raster import to_raster, to_tile_major
    grid, B, H, d = (3, 2, 5), 1, 2, 128
    S = 64 * 30
    q16, k16, v16 = (synth_mod.make_tensor(i, 31, B, H, S, d, grid=grid) for i in range(3))
    mask_np = synth_mod.make_bernoulli_mask(31, B * H, S // 64, 0.4).reshape(B, H, S // 64, S // 64)
    mask = torch.from_numpy(mask_np).cuda()
    q, k, v = (to_device_bf16(a) for a in (q16, k16, v16))
    o_t, lse_t = nl.bsa_fwd_with_mask(q, k, v, mask, tile_grid=grid)
    qr, kr, vr = (to_device_bf16(to_raster(a, grid)) for a in (q16, k16, v16))
    shape = nl.make_shape(B, H, S, d, grid, nl.LAYOUT_RASTER)
    o_r = torch.empty_like(qr)
    lse_r = torch.empty((B, H, S), dtype=torch.float32, device=qr.device)
    status = torch.full((1,), -1, dtype=torch.int32, device=qr.device)
    _call_static(nl, shape, qr, kr, vr, mask, o_r, lse_r, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    o_back = to_tile_major(o_r.view(torch.int16).cpu().numpy(), grid)
    assert np.array_equal(o_back, o_t.view(torch.int16).cpu().numpy())
    l_back = to_tile_major(lse_r.cpu().numpy()[..., None], grid)[..., 0]
    assert np.array_equal(l_back, lse_t.cpu().numpy())
