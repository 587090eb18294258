"""NABLA mask builder on the GPU vs the fp64 oracle (bit-exact masks except
rows whose cut lies within 1e-4 of 1 - thr; those are counted)."""
import math

import numpy as np
import pytest

from _parity import check_csr, compare_masks, csr_to_mask, to_device_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nl():
    import block_sparse_attention_23_b200 as nl
    nl.lib()
    return nl


def _gpu_mask(nl, q, k, grid, thr, sta, cap=None):
    qd, kd = to_device_bf16(q), to_device_bf16(k)
    B, H, S, d = q.shape
    ws = nl.Workspace.create(nl.make_shape(B, H, S, d, grid), nl.OP_BUILD_MASK)
    row_ptr, col_idx, nnz, mask = nl.nabla_build_mask(qd, kd, grid, thr, sta, want_mask=True,
                                                      col_capacity=cap, workspace=ws)
    status = ws.query_status()
    return (row_ptr.cpu().numpy(), col_idx.cpu().numpy(), int(nnz.item()),
            mask.cpu().numpy(), status)


def _run_config(nl, oracle_mod, synth_mod, name, thr=None, sta="cfg", record=None):
    w = synth_mod.WORKLOADS[name]
    q, k, _ = synth_mod.make_qkv(w)
    thr = w.thr if thr is None else thr
    sta = w.sta if sta == "cfg" else sta
    row_ptr, col_idx, nnz, gmask, status = _gpu_mask(nl, q, k, w.tile_grid, thr, sta)
    assert status == 0
    nrows = w.B * w.H * w.nb
    check_csr(row_ptr, col_idx, nrows, w.nb)
    assert nnz == row_ptr[-1] == int(gmask.sum())
    assert np.array_equal(csr_to_mask(row_ptr, col_idx, nrows, w.nb), gmask.reshape(nrows, w.nb))
    omask, diag, _ = oracle_mod.build_mask(q, k, w.tile_grid, thr, sta, with_diag=True)
    counts = compare_masks(gmask, omask, diag, thr)
    if record is not None:
        record(f"mask {name} thr={thr}", density=float(gmask.mean()), **counts)
    return gmask


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_mask_parity_small_configs(nl, oracle_mod, synth_mod, parity_record, name):
    _run_config(nl, oracle_mod, synth_mod, name, record=parity_record)


@pytest.mark.parametrize("thr", [0.0, 0.05, 0.7, 1.0])
def test_mask_parity_thresholds(nl, oracle_mod, synth_mod, parity_record, thr):
    m = _run_config(nl, oracle_mod, synth_mod, "small", thr=thr, sta=None, record=parity_record)
    if thr == 0.0:
        assert m.min() == 1
    if thr == 1.0:
        assert (m.sum(-1) == 1).all()


@pytest.mark.parametrize("name", ["hunyuan720p", "wan720p"])
def test_mask_parity_full_size(nl, oracle_mod, synth_mod, parity_record, name):
    _run_config(nl, oracle_mod, synth_mod, name, record=parity_record)


def test_mask_geometric_rows_closed_form(nl):
    """Pooled logits L[r][c] = -c * delta for every row: each row is the
    geometric-decay model, whose kept count has a closed form."""
    nb, d, delta = 48, 64, 0.125
    x = np.zeros((nb * 64, d), dtype=np.float32)
    x[:, 0] = 8.0
    y = np.zeros((nb * 64, d), dtype=np.float32)
    y[:, 0] = np.repeat(-delta * np.arange(nb), 64)
    q = (x.view(np.uint32) >> 16).astype(np.uint16)[None, None]
    k = (y.view(np.uint32) >> 16).astype(np.uint16)[None, None]
    rho = math.exp(-delta)
    for thr in (0.2, 0.4, 0.7):
        xx = math.log(1.0 - (1.0 - thr) * (1.0 - rho ** nb)) / math.log(rho)
        want = math.ceil(xx)
        _, _, _, m, st = _gpu_mask(nl, q, k, (3, 4, 4), thr, None)
        assert st == 0
        assert (m[0, 0].sum(axis=1) == want).all()
        assert (m[0, 0][:, :want] == 1).all()


@pytest.mark.parametrize("grid,d,sta", [((1, 3, 3), 64, (1, 1, 1)), ((3, 1, 5), 128, (0, 0, 2)),
                                        ((1, 1, 1), 64, None), ((2, 5, 7), 128, (1, 2, 2))])
def test_mask_ragged_grids(nl, oracle_mod, synth_mod, grid, d, sta):
    S = 64 * grid[0] * grid[1] * grid[2]
    q = synth_mod.make_tensor(0, 3, 2, 3, S, d, grid=grid, pos_weight=1.0, noise_weight=0.7)
    k = synth_mod.make_tensor(1, 3, 2, 3, S, d, grid=grid, pos_weight=1.0, noise_weight=0.7)
    row_ptr, col_idx, nnz, gmask, st = _gpu_mask(nl, q, k, grid, 0.3, sta)
    assert st == 0
    omask, diag, _ = oracle_mod.build_mask(q, k, grid, 0.3, sta, with_diag=True)
    compare_masks(gmask, omask, diag, 0.3)


def test_mask_capacity_overflow_reported(nl, synth_mod):
    w = synth_mod.WORKLOADS["tiny"]
    q, k, _ = synth_mod.make_qkv(w)
    row_ptr, col_idx, nnz, gmask, st = _gpu_mask(nl, q, k, w.tile_grid, 0.2, None, cap=5)
    assert st == 3   # NABLA_ERR_CAPACITY; row_ptr stays exact
    assert nnz == int(gmask.sum()) == row_ptr[-1]


@pytest.mark.parametrize("name,topk", [("tiny", 3), ("small", 1), ("small", 17), ("small", 200),
                                       ("hunyuan720p", 300)])
def test_topk_mask_parity(nl, oracle_mod, synth_mod, name, topk):
    """Fixed top-k rule: the same kept sets as the oracle's (rows whose k-th and
    (k+1)-th probabilities tie to 1e-6 may swap one block)."""
    w = synth_mod.WORKLOADS[name]
    q, k, _ = synth_mod.make_qkv(w)
    qd, kd = to_device_bf16(q), to_device_bf16(k)
    row_ptr, col_idx, nnz, mask = nl.nabla_build_mask(qd, kd, w.tile_grid, w.thr, w.sta,
                                                      want_mask=True, topk=topk)
    gmask = mask.cpu().numpy()
    omask, diag, _ = oracle_mod.build_mask(q, k, w.tile_grid, w.thr, w.sta, with_diag=True,
                                           topk=topk)
    compare_masks(gmask, omask, diag, w.thr)
    if w.sta is None:
        assert (gmask.sum(-1) == min(topk, w.nb)).all()
