"""XAttention antidiagonal scores and the mask selected from them, GPU vs the
fp64 oracle.  Scores: relative 2e-4 per block (the strided dot products are
fp32-accumulated bf16 MMAs, exp2 is approximate, sums are fp32; every term is
positive).  Masks: the oracle's selection on the oracle's scores, bit-exact
except rows within 1e-4 of the cut or tied to 1e-6."""
import numpy as np
import pytest

from _parity import CUT_BAND, check_csr, to_device_bf16

pytestmark = pytest.mark.gpu

S_RTOL = 2e-4


@pytest.fixture(scope="module")
def nl():
    import block_sparse_attention_23_b200 as nl
    nl.lib()
    return nl


def _gpu(nl, q, k, thr, stride, grid=None, sta=None, topk=0):
    qd, kd = to_device_bf16(q), to_device_bf16(k)
    B, H, S, d = q.shape
    ws = nl.Workspace.create(nl.make_shape(B, H, S, d, grid), nl.OP_BUILD_XATTN)
    rp, ci, nnz, mask, scores = nl.nabla_build_mask_xattn(
        qd, kd, thr, stride, tile_grid=grid, sta=sta, topk=topk, want_mask=True,
        want_scores=True, workspace=ws)
    assert ws.query_status() == 0
    return (rp.cpu().numpy(), ci.cpu().numpy(), int(nnz.item()), mask.cpu().numpy(),
            scores.cpu().numpy())


def _compare_mask(oracle_mod, gmask, omask, diag, thr):
    g = gmask.reshape(-1, gmask.shape[-1])
    o = omask.reshape(-1, omask.shape[-1])
    dg = diag.reshape(-1, 4)
    diff = (g != o).sum(axis=1)
    exempt = oracle_mod.near_cut_rows(dg, thr, CUT_BAND) | oracle_mod.near_tie_rows(dg)
    assert not ((diff > 0) & ~exempt).any(), np.nonzero((diff > 0) & ~exempt)[0][:5]
    assert diff[exempt].max(initial=0) <= 2


@pytest.mark.parametrize("name,stride", [("tiny", 8), ("tiny", 4), ("tiny", 16), ("small", 8)])
def test_xattn_scores_and_mask_parity(nl, oracle_mod, synth_mod, name, stride):
    w = synth_mod.WORKLOADS[name]
    q, k, _ = synth_mod.make_qkv(w)
    if name == "small":
        q, k = q[:, :3].copy(), k[:, :3].copy()
    B, H, S, d = q.shape
    rp, ci, nnz, gmask, gs = _gpu(nl, q, k, 0.3, stride, w.tile_grid, w.sta)
    ref = oracle_mod.xattn_scores(q, k, stride)
    np.testing.assert_allclose(gs, ref, rtol=S_RTOL, atol=0)
    np.testing.assert_allclose(gs.sum(axis=-1), 1.0, atol=1e-3)
    omask, diag = oracle_mod.select_rows(ref, w.tile_grid, 0.3, w.sta, with_diag=True)
    _compare_mask(oracle_mod, gmask, omask, diag, 0.3)
    check_csr(rp, ci, B * H * (S // 64), S // 64)
    assert nnz == int(gmask.sum())


@pytest.mark.parametrize("stride,nblocks,d", [(8, 30, 128), (4, 7, 64), (16, 5, 128)])
def test_xattn_ragged_tiles(nl, oracle_mod, synth_mod, stride, nblocks, d):
    """Strided row counts that are not multiples of the 128-row tile."""
    B, H, S = 2, 2, 64 * nblocks
    q = synth_mod.make_tensor(0, 70 + nblocks, B, H, S, d, pos_weight=0.0, noise_weight=1.0)
    k = synth_mod.make_tensor(1, 70 + nblocks, B, H, S, d, pos_weight=0.0, noise_weight=1.0)
    rp, ci, nnz, gmask, gs = _gpu(nl, q, k, 0.2, stride)
    ref = oracle_mod.xattn_scores(q, k, stride)
    np.testing.assert_allclose(gs, ref, rtol=S_RTOL, atol=0)
    omask, diag = oracle_mod.select_rows(ref, (nblocks, 1, 1), 0.2, None, with_diag=True)
    _compare_mask(oracle_mod, gmask, omask, diag, 0.2)


def test_xattn_full_size_wan_sampled_rows(nl, oracle_mod, synth_mod):
    import torch
    w = synth_mod.WORKLOADS["wan720p"]
    q, k, _ = synth_mod.make_qkv(w)
    rp, ci, nnz, gmask, gs = _gpu(nl, q, k, w.thr, 8, w.tile_grid, w.sta)
    flat = gs.reshape(-1, w.nb)
    assert np.abs(flat.sum(axis=1) - 1.0).max() < 2e-3
    rng = np.random.default_rng(3)
    rows = np.sort(rng.choice(flat.shape[0], 6, replace=False)).astype(np.int64)
    ref = oracle_mod.xattn_scores(q, k, 8, rows=rows)
    np.testing.assert_allclose(flat[rows], ref, rtol=S_RTOL, atol=0)
    check_csr(rp, ci, flat.shape[0], w.nb)
