"""Host-side work counters of bench.py (CPU): the executed tile products of the
forward and the backward, counted from a block CSR, against a brute-force
restatement of each kernel's work decomposition on small random masks, plus
closed forms (dense and diagonal masks)."""
import os
import sys

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402

TILE = 2.0 * 128 * 128   # FLOPs of one 128 x 128 x d product, per unit of d


def _csr(mask):
    BH, nb, _ = mask.shape
    m = mask.reshape(BH * nb, nb)
    rp = np.concatenate([[0], np.cumsum(m.sum(1))]).astype(np.int32)
    ci = np.nonzero(m)[1].astype(np.int32)
    return torch.from_numpy(rp), torch.from_numpy(ci)


def _brute_fwd_products(mask):
    """Forward: query blocks in pairs (2g, 2g+1), the union of their lists taken
    four blocks per 256-key tile; a tile counts two units, a unit being the S
    and PV products of the 128 queries against 128 of the tile's keys."""
    BH, nb, _ = mask.shape
    total = 0
    for b in range(BH):
        for g in range(0, nb, 2):
            union = set()
            for r in range(g, min(g + 2, nb)):
                union |= set(np.nonzero(mask[b, r])[0].tolist())
            tiles = -(-len(union) // 4)
            total += 2 * tiles
    return total


def _brute_bwd_flops(mask, d):
    """Backward: the dQ kernel pairs query blocks and takes the union of their key
    blocks two per 128-key tile, three products per tile; the dK/dV kernel pairs
    key blocks and takes the union of the query blocks listing either, two per
    128-query tile, four products per tile."""
    BH, nb, _ = mask.shape
    tq = tk = 0
    for b in range(BH):
        for g in range(0, nb, 2):
            uq = set()
            uk = set()
            for r in range(g, min(g + 2, nb)):
                uq |= set(np.nonzero(mask[b, r])[0].tolist())
                uk |= set(np.nonzero(mask[b, :, r])[0].tolist())
            tq += -(-len(uq) // 2)
            tk += -(-len(uk) // 2)
    return (3 * tq + 4 * tk) * TILE * d


@pytest.mark.parametrize("seed,nb,p", [(0, 7, 0.3), (1, 8, 0.1), (2, 12, 0.6), (3, 5, 1.0)])
def test_executed_counts_match_brute_force(seed, nb, p):
    rng = np.random.default_rng(seed)
    BH = 3
    mask = rng.random((BH, nb, nb)) < p
    mask[:, np.arange(nb), np.arange(nb)] = True
    rp, ci = _csr(mask)
    d = 128
    assert bench.executed_tile_products(rp, ci, BH, nb) == _brute_fwd_products(mask)
    assert bench.bwd_executed_flops(rp, ci, BH, nb, d) == _brute_bwd_flops(mask, d)
    # the sweep's shortcut on the dense uint8 mask gives the same forward count
    kept = int(mask.sum())
    want = 8.0 * (_brute_fwd_products(mask) / 2) / kept
    assert bench.sweep_executed_over_kept(mask.reshape(1, BH, nb, nb).astype(np.uint8)) == \
        pytest.approx(want, rel=1e-12)


def test_executed_counts_closed_forms():
    d = 64
    # dense, nb = 8: every pair's union is all 8 blocks
    nb = 8
    dense = np.ones((1, nb, nb), dtype=bool)
    rp, ci = _csr(dense)
    assert bench.executed_tile_products(rp, ci, 1, nb) == (nb // 2) * 2 * (nb // 4)
    assert bench.bwd_executed_flops(rp, ci, 1, nb, d) == \
        (3 + 4) * (nb // 2) * (nb // 2) * TILE * d
    # on a dense mask the forward executes exactly the kept work
    assert bench.sweep_executed_over_kept(dense.reshape(1, 1, nb, nb)) == pytest.approx(1.0)
    # diagonal, odd nb = 5: pairs (0,1), (2,3) have unions of 2, block 4 alone has 1
    nb = 5
    diag = np.eye(nb, dtype=bool)[None]
    rp, ci = _csr(diag)
    assert bench.executed_tile_products(rp, ci, 1, nb) == 3 * 2
    assert bench.bwd_executed_flops(rp, ci, 1, nb, d) == (3 * 3 + 4 * 3) * TILE * d


def test_mask_kernel_rooflines_units():
    """Per-kernel mask rooflines from stage times: pooling and compaction against
    HBM bytes, the reduced map against the fp64 FMA rate, the selection against
    the fp64 exp rate (one exponential per map entry) with its HBM fraction."""
    BH, nb, d, S, kept = 2, 8, 128, 512, 40
    peaks = {"hbm_gbs": 1000.0}
    out = bench._mask_kernel_rooflines([1.0, 2.0, 4.0, 0.5], BH, nb, d, S, kept, peaks,
                                       fp64_peak=10.0, exp_peak=50.0)
    pool, rmap, sel, comp = out["pool"], out["reduced_map"], out["select"], out["compact"]
    nw = (nb + 31) // 32
    assert pool["bound"] == "hbm" and comp["bound"] == "hbm"
    assert pool["bytes"] == 2.0 * BH * S * d * 2 + 2.0 * BH * nb * d * 8
    assert pool["frac"] == pytest.approx(pool["bytes"] / 1e-3 / 1e9 / 1000.0)
    assert rmap["bound"] == "fp64" and rmap["flops"] == 2.0 * BH * nb * nb * d
    assert rmap["frac"] == pytest.approx(rmap["flops"] / 2e-3 / 1e12 / 10.0)
    assert sel["bound"] == "alu" and sel["entries"] == BH * nb * nb
    assert sel["achieved"] == pytest.approx(BH * nb * nb / 4e-3 / 1e9)
    assert sel["frac"] == pytest.approx(sel["achieved"] / 50.0)
    hbm_bytes = 8.0 * BH * nb * nb + 4.0 * BH * nb * nw + 4.0 * BH * nb
    assert sel["hbm_frac"] == pytest.approx(hbm_bytes / 4e-3 / 1e9 / 1000.0)
    assert comp["bytes"] == 4.0 * BH * nb * nw + 8.0 * BH * nb + 4.0 * kept
