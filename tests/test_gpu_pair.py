"""The forward's CTA-pair kernel (opt-in: nabla_set_pair_mode) against the fp64
oracle: two CTAs walk the union of four query blocks' lists with M = 256
products, each loading half of every K and V tile.  Same bars as every
attention test (bf16 O within max-abs 2e-2 / mean-abs 2e-3, LSE within 1e-3)."""
import numpy as np
import pytest

from _parity import compare_attention, sample_rows, to_device_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture
def nl():
    import block_sparse_attention_23_b200 as nl
    nl.lib()
    nl.set_pair_mode(nl.PAIR_ALWAYS)
    yield nl
    nl.set_pair_mode(nl.PAIR_NEVER)


def _qkv(synth_mod, B, H, S, d, seed):
    return tuple(synth_mod.make_tensor(i, seed, B, H, S, d, pos_weight=0.0, noise_weight=1.0)
                 for i in range(3))


def _run(nl, q, k, v, mask, passes=None):
    import torch
    B, H, S, d = q.shape
    qd, kd, vd = to_device_bf16(q), to_device_bf16(k), to_device_bf16(v)
    ws = nl.Workspace.create(nl.make_shape(B, H, S, d), nl.OP_FWD_WITH_MASK)
    o, lse = nl.bsa_fwd_with_mask(qd, kd, vd, torch.from_numpy(mask).cuda(), workspace=ws)
    assert ws.query_status() == 0
    if passes is not None:
        assert ws.exact_passes() == passes
    return (o.float().cpu().numpy().reshape(-1, d), lse.cpu().numpy().reshape(-1))


@pytest.mark.parametrize("B,H,nb", [(1, 1, 1), (1, 2, 3), (2, 1, 5), (1, 1, 6), (1, 2, 7),
                                    (2, 1, 33)])
def test_pair_edge_cases(nl, oracle_mod, synth_mod, B, H, nb):
    """Quadruples with one to four query blocks present, empty rows, a single
    far block, a dense row, a key block no query lists."""
    d, S = 128, 64 * nb
    q, k, v = _qkv(synth_mod, B, H, S, d, seed=200 + nb)
    rng = np.random.default_rng(nb)
    mask = (rng.random((B, H, nb, nb)) < 0.4).astype(np.uint8)
    mask[..., 0, :] = 0
    if nb > 1:
        mask[..., 1, :] = 0
        mask[..., 1, nb - 1] = 1
    if nb > 2:
        mask[..., 2, :] = 1
    if nb > 3:
        mask[..., :, 3] = 0
    go, gl = _run(nl, q, k, v, mask, passes=0)
    ro, rl = oracle_mod.masked_attention(q, k, v, mask)
    compare_attention(go, gl, ro, rl)
    assert np.all(go.reshape(B * H, nb, 64, d)[:, 0] == 0.0)
    assert np.all(np.isneginf(gl.reshape(B * H, nb, 64)[:, 0]))


def test_pair_union_shapes(nl, oracle_mod, synth_mod):
    """Unions of four lists of every size modulo four, lists disjoint between
    the two CTAs of a pair, and an empty quadruple."""
    B, H, nb, d = 1, 2, 16, 128
    S = 64 * nb
    q, k, v = _qkv(synth_mod, B, H, S, d, seed=301)
    mask = np.zeros((B, H, nb, nb), dtype=np.uint8)
    for h in range(H):
        m = mask[0, h]
        # quadruple 0 (rows 0-3): empty
        m[4, (h + 3) % nb] = 1                      # quadruple 1: union of 1, in the even CTA
        m[6, [1, 2]] = 1
        m[7, [9 + h]] = 1                           # rows 6,7 (odd CTA): union of 3
        m[8, 0:5] = 1
        m[11, 5:10] = 1                             # quadruple 2: disjoint lists, union of 10
        m[12, :] = 1
        m[13, ::2] = 1
        m[14, 1::4] = 1
        m[15, [h, nb - 1 - h]] = 1                  # quadruple 3: dense union
    go, gl = _run(nl, q, k, v, mask, passes=0)
    ro, rl = oracle_mod.masked_attention(q, k, v, mask)
    compare_attention(go, gl, ro, rl)


def test_pair_rising_logits_hand_over_to_exact_pass(nl, oracle_mod):
    """Scores rising ~10 log2 units per key block outgrow the fixed reference:
    the pair pass must ask for the exact-reference recomputation, whose
    result meets the bars."""
    from test_gpu_numerics import _rising
    B, H, nb, d = 1, 2, 12, 128
    step = np.sqrt(d) * 10.0 / 1.4427
    q, k, v = _rising(B, H, nb, d, step, seed=nb)
    mask = np.ones((B, H, nb, nb), dtype=np.uint8)
    mask[:, :, 1, ::2] = 0
    go, gl = _run(nl, q, k, v, mask, passes=1)
    ro, rl = oracle_mod.masked_attention(q, k, v, mask)
    compare_attention(go, gl, ro, rl)


def test_pair_wan_layer_sampled_rows(nl, oracle_mod, synth_mod):
    """The Wan 720p-shaped layer (first 4 heads, full length) with its NABLA
    mask through bsa_fwd: every head x 16 query blocks x 64 rows."""
    w = synth_mod.WORKLOADS["wan720p"]
    q, k, v = (np.ascontiguousarray(a[:, :4]) for a in synth_mod.make_qkv(w))
    B, H, S, d = q.shape
    mask = oracle_mod.build_mask(q, k, w.tile_grid, w.thr, w.sta)
    import torch
    nb = S // 64
    flat = mask.reshape(-1, nb)
    rp = torch.from_numpy(np.concatenate([[0], np.cumsum(flat.sum(1))]).astype(np.int32)).cuda()
    ci = torch.from_numpy(np.nonzero(flat)[1].astype(np.int32)).cuda()
    qd, kd, vd = to_device_bf16(q), to_device_bf16(k), to_device_bf16(v)
    ws = nl.Workspace.create(nl.make_shape(B, H, S, d), nl.OP_FWD)
    o, lse = nl.bsa_fwd(qd, kd, vd, rp, ci, workspace=ws)
    assert ws.query_status() == 0 and ws.exact_passes() == 0
    rows = sample_rows(B, H, S, 16, 64, seed=9)
    ro, rl = oracle_mod.masked_attention(q, k, v, mask, rows)
    go = o.float().cpu().numpy().reshape(-1, d)[rows]
    gl = lse.cpu().numpy().reshape(-1)[rows]
    compare_attention(go, gl, ro, rl)
