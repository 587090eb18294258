"""The largest supported block count (S/64 = 4096 blocks = 262,144 tokens per
head): the selection's shared-memory rows, the attention's per-CTA bitmaps and
union lists at their capacity, against the oracle on sampled rows."""
import numpy as np
import pytest

from _parity import compare_attention, compare_masks, rows_with_same_mask, to_device_bf16

pytestmark = pytest.mark.gpu


def test_max_blocks_mask_and_attention(oracle_mod, synth_mod):
    import block_sparse_attention_23_b200 as nl
    B, H, d = 1, 1, 64
    grid = (16, 16, 16)                       # 4096 tiles
    nb = 16 * 16 * 16
    S = 64 * nb
    q = synth_mod.make_tensor(0, 21, B, H, S, d, grid=grid, pos_weight=1.0, noise_weight=1.0)
    k = synth_mod.make_tensor(1, 21, B, H, S, d, grid=grid, pos_weight=1.0, noise_weight=1.0)
    v = synth_mod.make_tensor(2, 21, B, H, S, d, pos_weight=0.0, noise_weight=1.0)
    qd, kd, vd = to_device_bf16(q), to_device_bf16(k), to_device_bf16(v)
    thr, sta = 0.3, (1, 1, 1)
    rp, ci, nnz, gmask = nl.nabla_build_mask(qd, kd, grid, thr, sta, want_mask=True)
    gm = gmask.cpu().numpy()
    omask, diag, _ = oracle_mod.build_mask(q, k, grid, thr, sta, with_diag=True)
    compare_masks(gm, omask, diag, thr)
    o, lse = nl.bsa_fwd(qd, kd, vd, rp, ci)
    rng = np.random.default_rng(9)
    blocks = np.concatenate([[0, nb - 1], rng.choice(nb, 6, replace=False)])
    rows = np.sort((blocks[:, None] * 64 + rng.choice(64, 4, replace=False)[None, :]).ravel())
    rows = rows_with_same_mask(rows.astype(np.int64), gm, omask, S, min_frac=0.5)
    ro, rl = oracle_mod.masked_attention(q, k, v, omask, rows)
    go = o.float().cpu().numpy().reshape(-1, d)[rows]
    gl = lse.cpu().numpy().reshape(-1)[rows]
    compare_attention(go, gl, ro, rl)
    # a dense row reaches the list capacity of its CTA
    dense = np.zeros((B, H, nb, nb), dtype=np.uint8)
    dense[0, 0, 5, :] = 1
    dense[0, 0, np.arange(nb), np.arange(nb)] = 1
    import torch
    o2, lse2 = nl.bsa_fwd_with_mask(qd, kd, vd, torch.from_numpy(dense).cuda())
    r2 = np.array([5 * 64, 5 * 64 + 63, 7 * 64], dtype=np.int64)
    ro2, rl2 = oracle_mod.masked_attention(q, k, v, dense, r2)
    compare_attention(o2.float().cpu().numpy().reshape(-1, d)[r2], lse2.cpu().numpy().reshape(-1)[r2],
                      ro2, rl2)
