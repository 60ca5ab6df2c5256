"""Index build on the GPU against the oracle's direct loops, bit for bit."""
import math

import numpy as np
import pytest
import torch

import oracle
from local_global_attention_b200 import configs as C
from local_global_attention_b200 import inputs as I
from local_global_attention_b200 import pack3d as P

pytestmark = pytest.mark.gpu

RAGGED = I.Workload(name="ragged_6x10x20", B=2, H=2, d=96, Z=6, Y=10, X=20, window=(5, 3, 7),
                    block=(3, 5, 4), packings=I.PACKINGS, seed=21)


def coords_of(wl, packing):
    orders = np.stack([I.packing_order(packing, wl.Z, wl.Y, wl.X, wl.block, wl.seed, b)
                       for b in range(wl.B)])
    return np.stack([I.coords_of_order(orders[b], wl.Z, wl.Y, wl.X) for b in range(wl.B)])


@pytest.mark.parametrize("wl,packing", [(C.TINY, "raster"), (C.VOL16K, "morton"),
                                        (RAGGED, "random"), (RAGGED, "block"),
                                        (C.VOL65K, "raster"), (C.VOL65K, "morton"),
                                        (C.VOL65K, "block"), (C.VOL65K, "random"),
                                        (C.MICRO1M, "block")])
def test_index_bit_exact(oracle_lib, wl, packing):
    coords = coords_of(wl, packing)
    params = P.make_params(wl)
    idx = P.pack3d_build_index(params, torch.from_numpy(coords).cuda())
    assert P.pack3d_index_check(idx) == P.OK
    got = {k: v.cpu().numpy() for k, v in idx.arrays().items()}
    want = oracle.build_index(wl, coords, tile=tuple(idx.struct.tile))
    np.testing.assert_array_equal(got["vol"], want["vol"])
    np.testing.assert_array_equal(got["perm"], want["perm"])
    np.testing.assert_array_equal(got["tile_off"], want["tile_off"])
    for b in range(wl.B):
        np.testing.assert_array_equal(got["nbr_off"], want["nbr_off"][b])
    np.testing.assert_array_equal(got["nbr"], want["nbr"])
    # rotation table: cos and sin of c * base^(-2j/da), fp64 values rounded to fp32
    da, half = wl.d // 3, wl.d // 6
    rows = [c for e in (wl.Z, wl.Y, wl.X) for c in range(e)]
    tab = got["rope"].reshape(len(rows), half, 2)
    theta = wl.rope_base ** (-2.0 * np.arange(half) / da)
    ang = np.asarray(rows, np.float64)[:, None] * theta[None, :]
    np.testing.assert_allclose(tab[..., 0], np.cos(ang), rtol=0, atol=1e-7)
    np.testing.assert_allclose(tab[..., 1], np.sin(ang), rtol=0, atol=1e-7)


@pytest.mark.parametrize("fault", ["duplicate", "out_of_range", "negative"])
def test_bad_coordinates_reported_and_nothing_written(fault):
    wl = RAGGED
    coords = coords_of(wl, "random")
    if fault == "duplicate":
        coords[1, 5] = coords[1, 9]
    elif fault == "out_of_range":
        coords[0, 3, 2] = wl.X
    else:
        coords[0, 7, 0] = -1
    params = P.make_params(wl)
    idx = P.pack3d_build_index(params, torch.from_numpy(coords).cuda())
    assert P.pack3d_index_check(idx) == P.ERR_COORDS
    err = idx.arrays()["err"].cpu().numpy()
    assert err[0] & (2 if fault == "duplicate" else 1)
    g = torch.Generator().manual_seed(0)
    shp = (wl.B, wl.N, wl.H, wl.d)
    q, k, v = (torch.randn(*shp, generator=g).to(torch.bfloat16).cuda() for _ in range(3))
    out = torch.full(shp, 7.0, dtype=torch.bfloat16, device="cuda")
    lse = torch.full((wl.B, wl.H, wl.N), 7.0, device="cuda")
    ksum = torch.full((wl.B, wl.H, wl.n_blocks, wl.d), 7.0, device="cuda")
    vsum = ksum.clone()
    P.pack3d_block_summaries(params, idx, k, v, ksum, vsum)
    P.pack3d_forward(params, idx, q, k, v, ksum, vsum, out, lse)
    P.pack3d_window_forward(params, idx, q, k, v, out, lse)
    torch.cuda.synchronize()
    assert bool((out == 7.0).all()) and bool((lse == 7.0).all()) and bool((ksum == 7.0).all())
