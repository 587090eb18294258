"""Raster token order read in place (the token reorder fused into the mask
builder's pooling loads and the attention's TMA boxes and O / LSE stores).

The raster tensors are made on the host from the seeded tile-major ones by a
numpy axis permutation.  The raster path must give bit for bit the tile-major
path's mask and, moved back to tile-major order, its O and LSE (the same
values reach the same shared-memory rows), and the oracle agrees with it."""
import numpy as np
import pytest

from _parity import compare_attention, rows_with_same_mask, to_device_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nl():
    import block_sparse_attention_23_b200 as nl
    nl.lib()
    return nl


def to_raster(x, grid):
    """[..., S, d] tile-major -> raster (t, h, w) order."""
    Tt, Th, Tw = grid
    lead = x.shape[:-2]
    d = x.shape[-1]
    y = x.reshape(lead + (Tt, Th, Tw, 4, 4, 4, d))
    n = len(lead)
    perm = tuple(range(n)) + (n, n + 3, n + 1, n + 4, n + 2, n + 5, n + 6)
    return np.ascontiguousarray(y.transpose(perm)).reshape(x.shape)


def to_tile_major(x, grid):
    Tt, Th, Tw = grid
    lead = x.shape[:-2]
    d = x.shape[-1]
    y = x.reshape(lead + (Tt, 4, Th, 4, Tw, 4, d))
    n = len(lead)
    perm = tuple(range(n)) + (n, n + 2, n + 4, n + 1, n + 3, n + 5, n + 6)
    return np.ascontiguousarray(y.transpose(perm)).reshape(x.shape)


def _layer(nl, q, k, v, grid, thr, sta, layout):
    B, H, S, d = q.shape
    qd, kd, vd = to_device_bf16(q), to_device_bf16(k), to_device_bf16(v)
    rp, ci, nnz, mask = nl.nabla_build_mask(qd, kd, grid, thr, sta, want_mask=True, layout=layout)
    ws = nl.Workspace.create(nl.make_shape(B, H, S, d, grid, layout), nl.OP_FWD)
    o, lse = nl.bsa_fwd(qd, kd, vd, rp, ci, workspace=ws, tile_grid=grid, layout=layout)
    assert ws.query_status() == 0
    return (mask.cpu().numpy(), o.view(__import__("torch").int16).cpu().numpy(),
            lse.cpu().numpy())


@pytest.mark.parametrize("case", ["tiny", "small", "ragged"])
def test_raster_layer_equals_tile_major_layer(nl, oracle_mod, synth_mod, case):
    if case == "ragged":
        grid, B, H, d, thr, sta = (3, 2, 5), 2, 2, 128, 0.3, (1, 1, 1)
        S = 64 * 30
        q, k, v = (synth_mod.make_tensor(i, 4, B, H, S, d, grid=grid) for i in range(3))
    else:
        w = synth_mod.WORKLOADS[case]
        q, k, v = synth_mod.make_qkv(w)
        grid, thr, sta = w.tile_grid, w.thr, w.sta
    B, H, S, d = q.shape
    m_tm, o_tm, l_tm = _layer(nl, q, k, v, grid, thr, sta, nl.LAYOUT_TILE_MAJOR)
    qr, kr, vr = (to_raster(a, grid) for a in (q, k, v))
    m_r, o_r, l_r = _layer(nl, qr, kr, vr, grid, thr, sta, nl.LAYOUT_RASTER)
    assert np.array_equal(m_r, m_tm)                                  # same mask bits
    assert np.array_equal(to_tile_major(o_r, grid), o_tm)            # same O bits
    assert np.array_equal(to_tile_major(l_r[..., None], grid)[..., 0], l_tm)
    # and against the oracle, in tile-major order, on rows whose mask row agrees
    ora_mask = oracle_mod.build_mask(q, k, grid, thr, sta)
    rows = rows_with_same_mask(np.arange(B * H * S, dtype=np.int64), m_tm, ora_mask, S)
    ro, rl = oracle_mod.masked_attention(q, k, v, ora_mask, rows)
    go = to_tile_major(o_r, grid).view(np.uint16).astype(np.uint32) << 16
    go = go.view(np.float32).reshape(-1, d)[rows]
    gl = to_tile_major(l_r[..., None], grid)[..., 0].reshape(-1)[rows]
    compare_attention(go, gl, ro, rl)


def test_raster_static_mask_and_full_size(nl, synth_mod):
    """Wan 720p layer in raster order with a host Bernoulli mask: bitwise the
    tile-major result (all 40 heads)."""
    import torch
    w = synth_mod.WORKLOADS["wan720p"]
    q, k, v = synth_mod.make_qkv(w)
    grid = w.tile_grid
    mask = synth_mod.make_bernoulli_mask(3, w.B * w.H, w.nb, 0.3).reshape(w.B, w.H, w.nb, w.nb)
    mt = torch.from_numpy(mask).cuda()
    outs = []
    for layout, arrs in ((nl.LAYOUT_TILE_MAJOR, (q, k, v)),
                         (nl.LAYOUT_RASTER, tuple(to_raster(a, grid) for a in (q, k, v)))):
        qd, kd, vd = (to_device_bf16(a) for a in arrs)
        ws = nl.Workspace.create(nl.make_shape(w.B, w.H, w.S, w.d, grid, layout), nl.OP_FWD_WITH_MASK)
        o, lse = nl.bsa_fwd_with_mask(qd, kd, vd, mt, workspace=ws, tile_grid=grid, layout=layout)
        assert ws.query_status() == 0
        outs.append((o.view(torch.int16).cpu().numpy(), lse.cpu().numpy()))
        del qd, kd, vd, o, lse
    (o_tm, l_tm), (o_r, l_r) = outs
    assert np.array_equal(to_tile_major(o_r, grid), o_tm)
    assert np.array_equal(to_tile_major(l_r[..., None], grid)[..., 0], l_tm)
