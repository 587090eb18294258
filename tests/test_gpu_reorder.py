"""Token reordering on the GPU vs the oracle (bit-exact: it moves bytes)."""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nl():
    import block_sparse_attention_23_b200 as nl
    nl.lib()
    return nl


def _dev(a):
    import torch
    return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)


def _host(t):
    import torch
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("grid,B,H,d", [((1, 1, 1), 1, 1, 64), ((3, 2, 5), 2, 3, 64),
                                        ((2, 3, 1), 1, 2, 128), ((5, 1, 3), 1, 1, 8),
                                        ((2, 2, 2), 1, 2, 200)])
def test_reorder_parity_ragged_grids(nl, oracle_mod, grid, B, H, d):
    Tt, Th, Tw = grid
    S = 64 * Tt * Th * Tw
    rng = np.random.default_rng(sum(grid) * 7 + d)
    x = rng.integers(0, 1 << 16, size=(B, H, S, d), dtype=np.uint16)
    xd = _dev(x)
    y = nl.nabla_reorder_tokens(xd, grid, nl.TO_TILE_MAJOR)
    assert np.array_equal(_host(y), oracle_mod.reorder(x, grid, to_tile_major=True))
    z = nl.nabla_reorder_tokens(xd, grid, nl.TO_RASTER)
    assert np.array_equal(_host(z), oracle_mod.reorder(x, grid, to_tile_major=False))
    back = nl.nabla_reorder_tokens(y, grid, nl.TO_RASTER)
    assert np.array_equal(_host(back), x)


def test_reorder_full_size_wan_roundtrip_and_sampled_rows(nl, synth_mod):
    import torch
    w = synth_mod.WORKLOADS["wan720p"]
    Tt, Th, Tw = w.tile_grid
    g = torch.Generator(device="cuda").manual_seed(11)
    x = torch.randint(-32768, 32767, (w.B, w.H, w.S, w.d), dtype=torch.int16, device="cuda",
                      generator=g).view(torch.bfloat16)
    y = nl.nabla_reorder_tokens(x, w.tile_grid, nl.TO_TILE_MAJOR)
    back = nl.nabla_reorder_tokens(y, w.tile_grid, nl.TO_RASTER)
    torch.cuda.synchronize()
    assert torch.equal(back.view(torch.int16), x.view(torch.int16))
    # sampled rows against the index definition
    rng = np.random.default_rng(2)
    T, H, W = w.grid
    n = 4096
    bh = rng.integers(0, w.B * w.H, n)
    t, h, ww = rng.integers(0, T, n), rng.integers(0, H, n), rng.integers(0, W, n)
    raster = (t * H + h) * W + ww
    major = (((t // 4) * Th + h // 4) * Tw + ww // 4) * 64 + ((t % 4) * 4 + h % 4) * 4 + ww % 4
    xf = x.view(torch.int16).reshape(-1, w.d)
    yf = y.view(torch.int16).reshape(-1, w.d)
    src = torch.from_numpy(bh * w.S + raster).cuda()
    dst = torch.from_numpy(bh * w.S + major).cuda()
    assert torch.equal(xf[src], yf[dst])
