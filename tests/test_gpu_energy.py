"""Block energy and calibrated static masks on the GPU vs the fp64 oracle.

Energy: both sides get the same fp32 LSE, computed by the oracle (its fp64
attention LSE rounded to fp32); the GPU's S = QK^T is a bf16 MMA with fp32 accumulation, exp2 is approximate and
the sums are fp32, so E agrees to a relative 2e-4 (every term is positive, so
the relative error of a block sum is at most the largest relative error of its
terms).  Calibration votes are integers: bit-exact except rows whose cut sits
within 1e-4 of 1 - eps or whose cut energies tie to 1e-6 (the GPU normalises
in fp32)."""
import math

import numpy as np
import pytest

from _parity import CUT_BAND, to_device_bf16

pytestmark = pytest.mark.gpu

E_RTOL = 2e-4


@pytest.fixture(scope="module")
def nl():
    import block_sparse_attention_23_b200 as nl
    nl.lib()
    return nl


def _csr(mask):
    import torch
    B, H, nb, _ = mask.shape
    flat = mask.reshape(-1, nb)
    counts = flat.sum(axis=1).astype(np.int64)
    row_ptr = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    col_idx = np.nonzero(flat)[1].astype(np.int32)
    if col_idx.size == 0:
        col_idx = np.zeros(1, dtype=np.int32)
    return torch.from_numpy(row_ptr).cuda(), torch.from_numpy(col_idx).cuda()


def _dense_lse(nl, qd, kd, vd):
    import torch
    B, H, S, d = qd.shape
    nb = S // 64
    full = torch.ones((B, H, nb, nb), dtype=torch.uint8, device="cuda")
    ws = nl.Workspace.create(nl.make_shape(B, H, S, d), nl.OP_FWD_WITH_MASK)
    _, lse = nl.bsa_fwd_with_mask(qd, kd, vd, full, workspace=ws)
    assert ws.query_status() == 0
    return lse


def _oracle_lse(oracle_mod, q, k, v, mask=None):
    """fp64 oracle LSE [B,H,S] rounded to fp32 (dense when mask is None)."""
    B, H, S, _ = q.shape
    if mask is None:
        _, lse = oracle_mod.dense_attention(q, k, v)
    else:
        _, lse = oracle_mod.masked_attention(q, k, v, mask)
    return lse.astype(np.float32).reshape(B, H, S)


def _gpu_energy(nl, qd, kd, lse, mask):
    B, H, S, d = qd.shape
    rp, ci = _csr(mask)
    ws = nl.Workspace.create(nl.make_shape(B, H, S, d), nl.OP_FWD)
    E, mass = nl.nabla_block_energy(qd, kd, lse, rp, ci, workspace=ws)
    assert ws.query_status() == 0
    return E.cpu().numpy(), mass.cpu().numpy()


def _random_qkv(synth_mod, B, H, S, d, seed):
    return tuple(synth_mod.make_tensor(i, seed, B, H, S, d, pos_weight=0.0, noise_weight=1.0)
                 for i in range(3))


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_energy_parity_dense_and_nabla_lists(nl, oracle_mod, synth_mod, name):
    w = synth_mod.WORKLOADS[name]
    q, k, v = synth_mod.make_qkv(w)
    if name == "small":            # keep the oracle to a few seconds: 2 heads
        q, k, v = q[:, :2].copy(), k[:, :2].copy(), v[:, :2].copy()
    B, H, S, d = q.shape
    nb = S // 64
    import torch
    qd, kd = to_device_bf16(q), to_device_bf16(k)
    lse_h = _oracle_lse(oracle_mod, q, k, v)
    lse = torch.from_numpy(lse_h).cuda()
    full = np.ones((B, H, nb, nb), dtype=np.uint8)
    E, mass = _gpu_energy(nl, qd, kd, lse, full)
    ref, ref_mass = oracle_mod.block_energy(q, k, lse_h, full)
    np.testing.assert_allclose(E, ref, rtol=E_RTOL, atol=0)
    np.testing.assert_allclose(mass, ref_mass, rtol=E_RTOL, atol=0)
    np.testing.assert_allclose(mass, 1.0, atol=2e-3)     # dense LSE: rows sum to 1
    # the NABLA mask's own block list: energy on kept blocks only, retained mass
    nm = oracle_mod.build_mask(q, k, w.tile_grid, w.thr, w.sta)
    E2, mass2 = _gpu_energy(nl, qd, kd, lse, nm)
    ref2, ref_mass2 = oracle_mod.block_energy(q, k, lse_h, nm)
    np.testing.assert_allclose(E2, ref2, rtol=E_RTOL, atol=0)
    np.testing.assert_allclose(mass2, ref_mass2, rtol=E_RTOL, atol=0)
    assert (E2[nm == 0] == 0).all()
    assert (mass2 <= mass * (1 + 1e-5)).all()


@pytest.mark.parametrize("B,H,nb,d", [(1, 1, 1, 64), (1, 2, 3, 128), (2, 3, 5, 64),
                                      (1, 1, 7, 128), (2, 1, 33, 64)])
def test_energy_edge_cases(nl, oracle_mod, synth_mod, B, H, nb, d):
    """Odd block counts (a pair with one block), empty rows and rows whose
    LSE is -inf, single-block and dense rows, both head dims."""
    import torch
    S = 64 * nb
    q, k, v = _random_qkv(synth_mod, B, H, S, d, seed=40 + nb)
    qd, kd = to_device_bf16(q), to_device_bf16(k)
    rng = np.random.default_rng(nb)
    mask = (rng.random((B, H, nb, nb)) < 0.4).astype(np.uint8)
    mask[..., 0, :] = 0
    if nb > 1:
        mask[..., 1, :] = 0
        mask[..., 1, nb - 1] = 1
    if nb > 2:
        mask[..., 2, :] = 1
    # the mask's own LSE: row block 0 is empty (LSE = -inf)
    lse_h = _oracle_lse(oracle_mod, q, k, v, mask)
    lse = torch.from_numpy(lse_h).cuda()
    E, mass = _gpu_energy(nl, qd, kd, lse, mask)
    ref, ref_mass = oracle_mod.block_energy(q, k, lse_h, mask)
    np.testing.assert_allclose(E, ref, rtol=E_RTOL, atol=0)
    np.testing.assert_allclose(mass, ref_mass, rtol=E_RTOL, atol=0)
    live = mask.sum(-1) > 0
    np.testing.assert_allclose(mass[live], 1.0, atol=2e-3)   # the mask's own LSE
    assert (mass[~live] == 0).all()


def test_energy_full_size_wan_sampled_rows(nl, oracle_mod, synth_mod):
    """Wan 720p layer, dense block list: with the GPU's own dense LSE every row
    of E sums to 1 (a property at any size); sampled block rows, whose LSE
    entries are replaced by the oracle's, agree with the oracle."""
    import torch
    w = synth_mod.WORKLOADS["wan720p"]
    q, k, v = synth_mod.make_qkv(w)
    qd, kd, vd = to_device_bf16(q), to_device_bf16(k), to_device_bf16(v)
    lse = _dense_lse(nl, qd, kd, vd)
    nb = w.nb
    BH = w.B * w.H
    rng = np.random.default_rng(7)
    rows = np.sort(rng.choice(BH * nb, 6, replace=False)).astype(np.int64)
    tok = ((rows // nb) * w.S + (rows % nb) * 64)[:, None] + np.arange(64)[None, :]
    _, ora_lse = oracle_mod.dense_attention(q, k, v, tok.reshape(-1))
    lse_flat = lse.reshape(-1)
    lse_flat[torch.from_numpy(tok.reshape(-1)).cuda()] = torch.from_numpy(
        ora_lse.astype(np.float32)).cuda()
    lse_sampled = np.full(BH * w.S, np.nan)          # the oracle reads only the sampled rows
    lse_sampled[tok.reshape(-1)] = ora_lse.astype(np.float32)
    row_ptr = torch.arange(0, BH * nb + 1, dtype=torch.int64, device="cuda").mul_(nb).to(torch.int32)
    col_idx = torch.arange(nb, dtype=torch.int32, device="cuda").repeat(BH * nb)
    ws = nl.Workspace.create(nl.make_shape(w.B, w.H, w.S, w.d), nl.OP_FWD)
    E, mass = nl.nabla_block_energy(qd, kd, lse, row_ptr, col_idx, workspace=ws)
    assert ws.query_status() == 0
    m = mass.cpu().numpy()
    assert np.abs(m - 1.0).max() < 2e-3
    full = np.ones((w.B, w.H, nb, nb), dtype=np.uint8)
    ref, _ = oracle_mod.block_energy(q, k, lse_sampled.reshape(w.B, w.H, w.S), full, rows=rows)
    got = E.reshape(-1, nb)[torch.from_numpy(rows).cuda()].cpu().numpy()
    np.testing.assert_allclose(got, ref, rtol=E_RTOL, atol=0)


def _exempt_rows(oracle_mod, energy, eps):
    """Rows whose cut lies within CUT_BAND of 1 - eps or whose cut energies tie."""
    nb = energy.shape[-1]
    flat = energy.reshape(-1, nb).astype(np.float64)
    ex = np.zeros(flat.shape[0], dtype=bool)
    for g in range(flat.shape[0]):
        z = np.clip(flat[g], 0, None).sum()
        if z <= 0:
            continue
        _, _, diag = oracle_mod.row_select(np.clip(flat[g], 0, None) / z, eps)
        ex[g] = (oracle_mod.near_cut_rows(diag[None], eps, CUT_BAND)[0] or
                 oracle_mod.near_tie_rows(diag[None])[0])
    return ex


def test_calibration_votes_and_mask_parity(nl, oracle_mod):
    import torch
    rng = np.random.default_rng(17)
    B, H, nb = 1, 3, 77
    runs = [rng.gamma(0.4, size=(B, H, nb, nb)).astype(np.float32) for _ in range(3)]
    runs[0][0, 1, 4] = 0.0                       # an all-zero row
    runs[1][0, 2, 9, :5] = -1.0                  # negative energies count as zero
    eps = 0.3
    votes_g = torch.zeros((B, H, nb, nb), dtype=torch.int32, device="cuda")
    votes_o = np.zeros((B, H, nb, nb), dtype=np.int32)
    exempt = np.zeros(B * H * nb, dtype=bool)
    for e in runs:
        nl.nabla_calib_accumulate(torch.from_numpy(e).cuda(), eps, votes_g)
        oracle_mod.calib_accumulate(e.astype(np.float64), eps, votes_o)
        exempt |= _exempt_rows(oracle_mod, e, eps)
    vg = votes_g.cpu().numpy().reshape(-1, nb)
    vo = votes_o.reshape(-1, nb)
    diff = (vg != vo).any(axis=1)
    assert not (diff & ~exempt).any(), np.nonzero(diff & ~exempt)[0][:5]
    assert exempt.sum() <= 3
    for mv in (1, 2, 3):
        mg = nl.nabla_calib_finalize(votes_g, mv).cpu().numpy()
        np.testing.assert_array_equal(mg, oracle_mod.calib_finalize(vg.reshape(votes_o.shape), mv))


def test_calibration_pipeline_to_static_mask_attention(nl, oracle_mod, synth_mod):
    """Two calibration runs (different seeds) of the tiny layer: dense LSE ->
    block energy -> votes -> static mask -> masked attention.  Each GPU stage
    runs on the oracle's result of the stage before (the oracle never reads a
    GPU result), and is compared with the oracle's result of that stage."""
    import torch
    from _parity import compare_attention
    w = synth_mod.WORKLOADS["tiny"]
    nb = w.nb
    eps = 0.15
    votes = torch.zeros((w.B, w.H, nb, nb), dtype=torch.int32, device="cuda")
    votes_o = np.zeros((w.B, w.H, nb, nb), dtype=np.int32)
    full = np.ones((w.B, w.H, nb, nb), dtype=np.uint8)
    for seed in (0, 1):
        q, k, v = synth_mod.make_qkv(w, seed=seed)
        qd, kd = to_device_bf16(q), to_device_bf16(k)
        lse_h = _oracle_lse(oracle_mod, q, k, v)
        E, _ = _gpu_energy(nl, qd, kd, torch.from_numpy(lse_h).cuda(), full)
        E_o, _ = oracle_mod.block_energy(q, k, lse_h, full)
        np.testing.assert_allclose(E, E_o, rtol=E_RTOL, atol=0)
        E_o32 = E_o.astype(np.float32)
        assert not _exempt_rows(oracle_mod, E_o32, eps).any()
        nl.nabla_calib_accumulate(torch.from_numpy(E_o32).cuda(), eps, votes)
        oracle_mod.calib_accumulate(E_o32.astype(np.float64), eps, votes_o)
    np.testing.assert_array_equal(votes.cpu().numpy(), votes_o)
    mask = nl.nabla_calib_finalize(votes, 1)
    mask_h = oracle_mod.calib_finalize(votes_o, 1)
    np.testing.assert_array_equal(mask.cpu().numpy(), mask_h)
    assert 0 < mask_h.sum() < mask_h.size
    q, k, v = synth_mod.make_qkv(w, seed=2)         # inference on a new input
    qd, kd, vd = to_device_bf16(q), to_device_bf16(k), to_device_bf16(v)
    ws = nl.Workspace.create(nl.make_shape(w.B, w.H, w.S, w.d), nl.OP_FWD_WITH_MASK)
    o, lse = nl.bsa_fwd_with_mask(qd, kd, vd, mask, workspace=ws)
    assert ws.query_status() == 0
    rows = np.arange(w.B * w.H * w.S, dtype=np.int64)
    ro, rl = oracle_mod.masked_attention(q, k, v, mask_h, rows)
    compare_attention(o.float().cpu().numpy().reshape(-1, w.d), lse.cpu().numpy().reshape(-1),
                      ro, rl)
