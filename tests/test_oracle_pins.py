"""Pins of the CPU oracle against facts fixed outside the oracle itself.

Each test checks the oracle against a closed form, a textbook routine
(torch's dense scaled-dot-product attention), an invariant the paper states
("Geometry Matters in Packed 3D Attention", abstract: logits depend on
query-relative 3D displacement, summaries are means of rotated keys, results do
not depend on the memory order), a brute-force construction on tiny inputs, or
central finite differences.  They run on the CPU.
"""
import glob
import json
import math
import os
from types import SimpleNamespace

import numpy as np
import pytest
import torch
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import oracle
from local_global_attention_b200 import inputs as I

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def shape(B=1, H=1, d=12, Z=4, Y=5, X=6, window=(3, 3, 3), block=(2, 5, 3), base=100.0,
          n_tokens=0):
    return SimpleNamespace(B=B, H=H, d=d, Z=Z, Y=Y, X=X, window=window, block=block,
                           rope_base=base, scale=0.0, n_tokens=n_tokens)


def rand_inputs(s, seed=0, packing="random"):
    g = torch.Generator().manual_seed(seed)
    N = s.Z * s.Y * s.X
    grid = {n: torch.randn(s.B, N, s.H, s.d, generator=g, dtype=torch.float64) for n in "qkv"}
    grid["dout"] = torch.randn(s.B, N, s.H, s.d, generator=g, dtype=torch.float64)
    orders = np.stack([I.packing_order(packing, s.Z, s.Y, s.X, s.block, seed, b)
                       for b in range(s.B)])
    coords = np.stack([I.coords_of_order(orders[b], s.Z, s.Y, s.X) for b in range(s.B)])
    packed = {n: torch.stack([t[b][torch.from_numpy(orders[b])] for b in range(s.B)])
              for n, t in grid.items()}
    return packed, coords, orders


def rotate_complex(x, coords, base):
    """Axial rotation written as complex multiplication: pair (j, j + da/2) of
    axis segment a is the complex number x_j + i x_{j+da/2}, multiplied by
    exp(i c_a base^(-2j/da))."""
    x = np.asarray(x, np.float64)
    d = x.shape[-1]
    da, h = d // 3, d // 6
    theta = base ** (-2.0 * np.arange(h) / da)
    out = np.empty_like(x)
    for a in range(3):
        seg = x[..., a * da:(a + 1) * da]
        z = (seg[..., :h] + 1j * seg[..., h:]) * np.exp(1j * coords[..., a, None] * theta)
        out[..., a * da:a * da + h] = z.real
        out[..., a * da + h:(a + 1) * da] = z.imag
    return out


def dense_reference(s, packed, coords, b):
    """Dense softmax attention with axial RoPE for batch item b, via torch SDPA."""
    c = coords[b].astype(np.float64)[:, None, :]  # [N, 1, 3]
    qr = torch.from_numpy(rotate_complex(packed["q"][b].numpy(), c, s.rope_base))
    kr = torch.from_numpy(rotate_complex(packed["k"][b].numpy(), c, s.rope_base))
    tau = 1.0 / math.sqrt(s.d)
    q, k, v = (t.permute(1, 0, 2) for t in (qr, kr, packed["v"][b]))  # [H, N, d]
    out = torch.nn.functional.scaled_dot_product_attention(q, k, v, scale=tau)
    lse = torch.logsumexp(tau * q @ k.transpose(1, 2), dim=-1)
    return out.permute(1, 0, 2).numpy(), lse.numpy()


# ---- rotation -------------------------------------------------------------

def test_rope_matches_complex_rotation(oracle_lib):
    s = shape(B=2, H=3, d=18, Z=5, Y=3, X=7, block=(1, 1, 1))
    packed, coords, _ = rand_inputs(s, seed=1)
    got = oracle.rope(s, coords, packed["q"])
    want = rotate_complex(packed["q"].numpy(), coords.astype(np.float64)[:, :, None, :], s.rope_base)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-13)
    back = oracle.rope(s, coords, torch.from_numpy(got), transpose=True)
    np.testing.assert_allclose(back, packed["q"].numpy(), rtol=0, atol=1e-13)


def test_rope_logit_depends_only_on_displacement(oracle_lib):
    """Translating both coordinates by the same vector leaves q~.k~ unchanged."""
    s = shape(B=1, H=1, d=24, Z=40, Y=40, X=40, block=(1, 1, 1))
    rng = np.random.default_rng(3)
    N = s.Z * s.Y * s.X
    for _ in range(20):
        cq, ck = rng.integers(0, 20, 3), rng.integers(0, 20, 3)
        t = rng.integers(0, 20, 3)
        q, k = rng.standard_normal(s.d), rng.standard_normal(s.d)

        def logit(a, b):
            # rotate single rows by building a 1-token-per-coordinate input
            x = np.zeros((1, N, 1, s.d))
            coords = I.coords_of_order(np.arange(N), s.Z, s.Y, s.X)[None]
            ia = (a[0] * s.Y + a[1]) * s.X + a[2]
            ib = (b[0] * s.Y + b[1]) * s.X + b[2]
            x[0, ia, 0] = q
            rq = oracle.rope(s, coords, x)[0, ia, 0]
            x[0, ia, 0] = 0
            x[0, ib, 0] = k
            rk = oracle.rope(s, coords, x)[0, ib, 0]
            return rq @ rk

        assert abs(logit(cq, ck) - logit(cq + t, ck + t)) < 1e-12


def test_rope_same_position_cancels(oracle_lib):
    """R(c)^T R(c) = I, so q~_i . k~_i = q_i . k_i at any coordinate."""
    s = shape(B=1, H=2, d=30, Z=9, Y=4, X=11, block=(1, 1, 1))
    packed, coords, _ = rand_inputs(s, seed=4)
    qr = oracle.rope(s, coords, packed["q"])
    kr = oracle.rope(s, coords, packed["k"])
    np.testing.assert_allclose((qr * kr).sum(-1), (packed["q"] * packed["k"]).sum(-1).numpy(),
                               rtol=0, atol=1e-12)


# ---- worked examples ------------------------------------------------------

@pytest.mark.parametrize("path", sorted(glob.glob(os.path.join(GOLDEN, "closed_form_*.json"))))
def test_closed_form_worked_example(oracle_lib, path):
    fx = json.load(open(path))
    sh = fx["shape"]
    s = shape(B=1, H=1, d=sh["d"], Z=sh["Z"], Y=sh["Y"], X=sh["X"], window=tuple(sh["window"]),
              block=tuple(sh["block"]), base=sh["rope_base"])
    coords = np.asarray(fx["coords"], np.int16)[None]
    q, k, v = (np.asarray(fx[n], np.float64)[None, :, None, :] for n in "qkv")
    out, lse = oracle.forward(s, coords, q, k, v)
    np.testing.assert_allclose(out[0, :, 0], np.asarray(fx["out"]), rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse[0, 0], np.asarray(fx["lse"]), rtol=0, atol=1e-13)


def test_self_only_window_without_summaries(oracle_lib):
    """Window 1x1x1 and one block covering the volume: out_i = v_i and
    lse_i = tau q_i . k_i (the rotation cancels at equal positions)."""
    s = shape(B=2, H=2, d=12, Z=3, Y=4, X=5, window=(1, 1, 1), block=(3, 4, 5))
    packed, coords, _ = rand_inputs(s, seed=5)
    out, lse = oracle.forward(s, coords, packed["q"], packed["k"], packed["v"])
    np.testing.assert_allclose(out, packed["v"].numpy(), rtol=0, atol=1e-13)
    want = (packed["q"] * packed["k"]).sum(-1).permute(0, 2, 1).numpy() / math.sqrt(s.d)
    np.testing.assert_allclose(lse, want, rtol=0, atol=1e-13)


# ---- reductions to dense attention ----------------------------------------

@pytest.mark.parametrize("packing", ["raster", "random"])
def test_full_window_is_dense_attention(oracle_lib, packing):
    """Property (i): a window of at least 2*extent-1 per axis covers the volume,
    every block meets it, no summary is used: dense attention with axial RoPE."""
    s = shape(B=2, H=2, d=12, Z=3, Y=4, X=5, window=(5, 7, 9), block=(1, 2, 5))
    packed, coords, _ = rand_inputs(s, seed=6, packing=packing)
    out, lse = oracle.forward(s, coords, packed["q"], packed["k"], packed["v"])
    for b in range(s.B):
        ro, rl = dense_reference(s, packed, coords, b)
        np.testing.assert_allclose(out[b], ro, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[b], rl, rtol=0, atol=1e-12)


@pytest.mark.parametrize("window", [(1, 1, 1), (3, 3, 3), (3, 1, 5), (1, 5, 1)])
def test_one_token_blocks_are_dense_attention(oracle_lib, window):
    """Property (iii), special case: with 1x1x1 blocks every token is either in
    the window (exact) or its own summary (kbar = k~, vbar = v), so any window
    gives dense attention."""
    s = shape(B=1, H=2, d=18, Z=4, Y=3, X=5, window=window, block=(1, 1, 1))
    packed, coords, _ = rand_inputs(s, seed=7)
    out, lse = oracle.forward(s, coords, packed["q"], packed["k"], packed["v"])
    ro, rl = dense_reference(s, packed, coords, 0)
    np.testing.assert_allclose(out[0], ro, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse[0], rl, rtol=0, atol=1e-12)


# ---- summaries --------------------------------------------------------------

@pytest.mark.parametrize("dims,block", [((4, 6, 6), (2, 3, 2)), ((5, 6, 7), (2, 4, 3))],
                         ids=["dividing", "cut_at_edge"])
def test_summary_logit_is_mean_of_member_logits(oracle_lib, dims, block):
    """Property (iii): tau q~ . kbar_B = mean over j in B of tau q~ . k~_j, and
    vbar is the mean of the members' values; blocks found from the coordinates.
    Where an extent does not divide the volume, the last blocks hold fewer
    tokens and the means run over those."""
    Z, Y, X = dims
    s = shape(B=2, H=2, d=12, Z=Z, Y=Y, X=X, block=block)
    packed, coords, _ = rand_inputs(s, seed=8)
    ks, vs = oracle.block_summaries(s, coords, packed["k"], packed["v"])
    kr = oracle.rope(s, coords, packed["k"])
    qr = oracle.rope(s, coords, packed["q"])
    nby, nbx = -(-s.Y // s.block[1]), -(-s.X // s.block[2])
    for b in range(s.B):
        c = coords[b].astype(np.int64)
        bid = ((c[:, 0] // s.block[0]) * nby + c[:, 1] // s.block[1]) * nbx + c[:, 2] // s.block[2]
        for B in range(ks.shape[2]):
            members = np.nonzero(bid == B)[0]
            Bc = (B // (nby * nbx), (B // nbx) % nby, B % nbx)
            held = np.prod([min(e, n - i * e) for i, e, n in zip(Bc, s.block, (Z, Y, X))])
            assert members.size == held
            for h in range(s.H):
                ql = qr[b, :, h] @ ks[b, h, B]
                want = (qr[b, :, h] @ kr[b, members, h].T).mean(axis=1)
                np.testing.assert_allclose(ql, want, rtol=0, atol=1e-12)
                np.testing.assert_allclose(vs[b, h, B], packed["v"][b, members, h].mean(0).numpy(),
                                           rtol=0, atol=1e-13)


# ---- brute force on tiny volumes -------------------------------------------

def brute_force(s, packed, coords, b, window_only=False):
    """Masked dense softmax over [keys | block summaries] with the geometry
    decided by enumeration: a key is local when every axis offset is within the
    radius; a block is excluded when any voxel of its box (cut at the volume's
    edge) is local to the query; a block holding no token has no summary."""
    c = coords[b].astype(np.int64)
    N = c.shape[0]
    r = (np.asarray(s.window) - 1) // 2
    cf = c.astype(np.float64)[:, None, :]
    qr = rotate_complex(packed["q"][b].numpy(), cf, s.rope_base)
    kr = rotate_complex(packed["k"][b].numpy(), cf, s.rope_base)
    v = packed["v"][b].numpy()
    local = np.all(np.abs(c[:, None, :] - c[None, :, :]) <= r, axis=-1)  # [Nq, Nk]
    # block membership by enumeration of voxels
    blk = np.asarray(s.block)
    cells = c // blk
    keys = sorted({tuple(x) for x in cells})
    members = [np.nonzero(np.all(cells == np.asarray(kk), axis=1))[0] for kk in keys]
    boxes = [np.stack(np.meshgrid(*[np.arange(kk[a] * blk[a], min((kk[a] + 1) * blk[a], n))
                                    for a, n in enumerate((s.Z, s.Y, s.X))], indexing="ij"),
                      -1).reshape(-1, 3) for kk in keys]
    seen = np.stack([np.all(np.abs(c[:, None, :] - bx[None]) <= r, axis=-1).any(axis=1)
                     for bx in boxes], axis=1)  # [Nq, nb]
    tau = 1.0 / math.sqrt(s.d)
    outs, lses = np.zeros((N, s.H, s.d)), np.zeros((s.H, N))
    for h in range(s.H):
        logits = tau * qr[:, h] @ kr[:, h].T
        logits = np.where(local, logits, -np.inf)
        cols, vals = [logits], [v[:, h]]
        if not window_only:
            kbar = np.stack([kr[m, h].mean(0) for m in members])
            vbar = np.stack([v[m, h].mean(0) for m in members])
            cols.append(np.where(seen, -np.inf, tau * qr[:, h] @ kbar.T))
            vals.append(vbar)
        L = np.concatenate(cols, axis=1)
        V = np.concatenate(vals, axis=0)
        m = L.max(axis=1, keepdims=True)
        e = np.exp(L - m)
        outs[:, h] = (e @ V) / e.sum(1, keepdims=True)
        lses[h] = (m[:, 0] + np.log(e.sum(1)))
    return outs, lses


@pytest.mark.parametrize("cfg", [
    dict(Z=4, Y=5, X=6, window=(3, 3, 3), block=(2, 5, 3)),
    dict(Z=6, Y=4, X=4, window=(3, 1, 5), block=(3, 2, 2)),
    dict(Z=4, Y=4, X=8, window=(1, 3, 3), block=(4, 2, 4)),
    dict(Z=5, Y=5, X=5, window=(5, 5, 3), block=(5, 1, 1)),
    # extents that do not divide the volume: the last blocks are cut at its edge
    dict(Z=5, Y=5, X=7, window=(3, 3, 3), block=(2, 3, 4)),
    dict(Z=4, Y=6, X=5, window=(1, 3, 5), block=(3, 4, 2)),
])
@pytest.mark.parametrize("window_only", [False, True])
def test_brute_force_masked_softmax(oracle_lib, cfg, window_only):
    s = shape(B=2, H=2, d=12, **cfg)
    packed, coords, _ = rand_inputs(s, seed=9)
    out, lse = oracle.forward(s, coords, packed["q"], packed["k"], packed["v"],
                              window_only=window_only)
    for b in range(s.B):
        ro, rl = brute_force(s, packed, coords, b, window_only)
        np.testing.assert_allclose(out[b], ro, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[b], rl, rtol=0, atol=1e-12)


def test_sampled_forward_matches_full(oracle_lib):
    s = shape(B=2, H=3, d=12, Z=4, Y=5, X=6)
    packed, coords, _ = rand_inputs(s, seed=10)
    out, lse = oracle.forward(s, coords, packed["q"], packed["k"], packed["v"])
    rng = np.random.default_rng(0)
    N = s.Z * s.Y * s.X
    b, h, i = rng.integers(0, s.B, 50), rng.integers(0, s.H, 50), rng.integers(0, N, 50)
    so, sl = oracle.forward(s, coords, packed["q"], packed["k"], packed["v"],
                            sel=oracle.flat_index(s, b, h, i))
    np.testing.assert_array_equal(so, out[b, i, h])
    np.testing.assert_array_equal(sl, lse[b, h, i])


# ---- memory-order independence -------------------------------------------

@pytest.mark.parametrize("dims,block", [((4, 8, 8), (2, 4, 4)), ((5, 7, 8), (2, 3, 3))],
                         ids=["dividing", "cut_at_edge"])
def test_packing_equivariance_bit_exact(oracle_lib, dims, block):
    """Property (iv): raster, Morton, block-contiguous and random packings of
    the same field give the same per-voxel outputs, bit for bit."""
    Z, Y, X = dims
    s = shape(B=2, H=2, d=12, Z=Z, Y=Y, X=X, window=(3, 3, 3), block=block)
    g = torch.Generator().manual_seed(11)
    N = s.Z * s.Y * s.X
    grid = {n: torch.randn(s.B, N, s.H, s.d, generator=g, dtype=torch.float64) for n in "qkv"}
    ref = None
    for packing in I.PACKINGS:
        orders = np.stack([I.packing_order(packing, s.Z, s.Y, s.X, s.block, 3, b)
                           for b in range(s.B)])
        coords = np.stack([I.coords_of_order(orders[b], s.Z, s.Y, s.X) for b in range(s.B)])
        pk = {n: torch.stack([t[b][torch.from_numpy(orders[b])] for b in range(s.B)])
              for n, t in grid.items()}
        out, lse = oracle.forward(s, coords, pk["q"], pk["k"], pk["v"])
        raster_out = np.empty_like(out)
        raster_lse = np.empty_like(lse)
        for b in range(s.B):
            raster_out[b, orders[b]] = out[b]
            raster_lse[b][:, orders[b]] = lse[b]
        if ref is None:
            ref = (raster_out, raster_lse)
        else:
            np.testing.assert_array_equal(raster_out, ref[0])
            np.testing.assert_array_equal(raster_lse, ref[1])


def test_block_larger_than_volume_equals_the_volume_wide_block(oracle_lib):
    """A block extent beyond the volume holds the same tokens as the extent of
    the volume itself, so summaries, outputs and gradients agree bit for bit."""
    base = dict(B=2, H=2, d=12, Z=4, Y=6, X=5, window=(3, 3, 3))
    s_cut, s_fit = shape(block=(2, 3, 8), **base), shape(block=(2, 3, 5), **base)
    packed, coords, _ = rand_inputs(s_fit, seed=21)
    args = (coords, packed["q"], packed["k"], packed["v"])
    for got, want in zip(oracle.block_summaries(s_cut, coords, packed["k"], packed["v"]),
                         oracle.block_summaries(s_fit, coords, packed["k"], packed["v"])):
        np.testing.assert_array_equal(got, want)
    for got, want in zip(oracle.forward(s_cut, *args), oracle.forward(s_fit, *args)):
        np.testing.assert_array_equal(got, want)
    for got, want in zip(oracle.backward(s_cut, *args, packed["dout"]),
                         oracle.backward(s_fit, *args, packed["dout"])):
        np.testing.assert_array_equal(got, want)


# ---- backward -------------------------------------------------------------

@pytest.mark.parametrize("window_only", [False, True])
@pytest.mark.parametrize("block", [(2, 2, 3), (3, 3, 4)], ids=["dividing", "cut_at_edge"])
def test_backward_finite_differences(oracle_lib, window_only, block):
    """Central differences of sum(dout * out) against the analytic gradients,
    including the paths through the rotation and through the block means (with
    blocks cut at the volume's edge in the second case)."""
    s = shape(B=1, H=2, d=12, Z=4, Y=4, X=6, window=(3, 3, 3), block=block)
    packed, coords, _ = rand_inputs(s, seed=12)
    dq, dk, dv = oracle.backward(s, coords, packed["q"], packed["k"], packed["v"],
                                 packed["dout"], window_only=window_only)
    grads = {"q": dq, "k": dk, "v": dv}
    rng = np.random.default_rng(1)
    eps = 1e-6
    dout = packed["dout"].numpy()
    for name in "qkv":
        for _ in range(12):
            idx = tuple(int(rng.integers(0, n)) for n in packed[name].shape)
            vals = {}
            for sign in (+1, -1):
                pk = {n: packed[n].clone() for n in "qkv"}
                pk[name][idx] += sign * eps
                out, _ = oracle.forward(s, coords, pk["q"], pk["k"], pk["v"],
                                        window_only=window_only)
                vals[sign] = (out * dout).sum()
            fd = (vals[1] - vals[-1]) / (2 * eps)
            assert abs(fd - grads[name][idx]) <= 1e-6 * max(1.0, abs(fd)), (name, idx)


@pytest.mark.slow
def test_backward_finite_differences_tiny_workload(oracle_lib):
    """Same check on the 8x8x8, d = 48 tiny workload shape (fp64 inputs)."""
    from local_global_attention_b200.configs import TINY
    s = shape(B=1, H=1, d=TINY.d, Z=8, Y=8, X=8, window=TINY.window, block=TINY.block)
    packed, coords, _ = rand_inputs(s, seed=13, packing="raster")
    dq, dk, dv = oracle.backward(s, coords, packed["q"], packed["k"], packed["v"], packed["dout"])
    grads = {"q": dq, "k": dk, "v": dv}
    rng = np.random.default_rng(2)
    eps = 1e-6
    dout = packed["dout"].numpy()
    for name in "qkv":
        for _ in range(4):
            idx = tuple(int(rng.integers(0, n)) for n in packed[name].shape)
            vals = {}
            for sign in (+1, -1):
                pk = {n: packed[n].clone() for n in "qkv"}
                pk[name][idx] += sign * eps
                out, _ = oracle.forward(s, coords, pk["q"], pk["k"], pk["v"])
                vals[sign] = (out * dout).sum()
            fd = (vals[1] - vals[-1]) / (2 * eps)
            assert abs(fd - grads[name][idx]) <= 1e-6 * max(1.0, abs(fd)), (name, idx)


# ---- index ----------------------------------------------------------------

@pytest.mark.parametrize("dims,window,tile", [((8, 8, 8), (3, 3, 3), (4, 4, 8)),
                                               ((6, 10, 12), (5, 3, 7), (4, 4, 8)),
                                               ((5, 7, 9), (1, 1, 1), (2, 3, 4))])
def test_index_against_sorting(oracle_lib, dims, window, tile):
    """perm = tokens sorted by (tile, raster inside the tile) with numpy's
    lexsort; halo lists = tokens whose voxel is within r of the tile box."""
    Z, Y, X = dims
    s = shape(B=2, H=1, d=12, Z=Z, Y=Y, X=X, window=window, block=(1, 1, 1))
    _, coords, _ = rand_inputs(s, seed=14)
    ix = oracle.build_index(s, coords, tile)
    nTy, nTx = -(-Y // tile[1]), -(-X // tile[2])
    r = (np.asarray(window) - 1) // 2
    for b in range(s.B):
        c = coords[b].astype(np.int64)
        assert np.array_equal(ix["vol"][b][(c[:, 0] * Y + c[:, 1]) * X + c[:, 2]], np.arange(Z * Y * X))
        tid = ((c[:, 0] // tile[0]) * nTy + c[:, 1] // tile[1]) * nTx + c[:, 2] // tile[2]
        raster = (c[:, 0] * Y + c[:, 1]) * X + c[:, 2]
        want = np.lexsort((raster, tid))
        assert np.array_equal(ix["perm"][b], want)
        counts = np.bincount(tid, minlength=ix["tile_off"].shape[1] - 1)
        assert np.array_equal(ix["tile_off"][b], np.concatenate([[0], np.cumsum(counts)]))
        for t in range(ix["tile_off"].shape[1] - 1):
            box_lo = c[want[ix["tile_off"][b, t]]]  # first voxel of the tile = its low corner
            members = c[want[ix["tile_off"][b, t]:ix["tile_off"][b, t + 1]]]
            lo, hi = members.min(0), members.max(0)
            assert np.array_equal(lo, box_lo)
            near = np.all((c >= lo - r) & (c <= hi + r), axis=1)
            halo = np.nonzero(near)[0]
            halo = halo[np.argsort(raster[halo])]
            got = ix["nbr"][b, ix["nbr_off"][b, t]:ix["nbr_off"][b, t + 1]]
            assert np.array_equal(got, halo)


def test_index_partly_occupied_against_sorting(oracle_lib):
    """A partly occupied volume: vol holds the token at each occupied voxel and
    -1 elsewhere; perm = the tokens present sorted by (tile, raster inside the
    tile) with numpy's lexsort, tile_off their counts per tile; the halo lists
    hold, for every voxel of the widened tile box in raster order, its token
    or -1 (the box is geometry, not occupancy)."""
    tile = (2, 3, 4)
    s = shape(B=2, H=1, d=12, Z=5, Y=6, X=7, window=(3, 3, 5), block=(1, 1, 1), n_tokens=97)
    _, coords = partial_inputs(s, seed=16)
    ix = oracle.build_index(s, coords, tile)
    Z, Y, X = s.Z, s.Y, s.X
    nTz, nTy, nTx = -(-Z // tile[0]), -(-Y // tile[1]), -(-X // tile[2])
    r = (np.asarray(s.window) - 1) // 2
    for b in range(s.B):
        c = coords[b].astype(np.int64)
        raster = (c[:, 0] * Y + c[:, 1]) * X + c[:, 2]
        vol = np.full(Z * Y * X, -1)
        vol[raster] = np.arange(s.n_tokens)
        assert np.array_equal(ix["vol"][b], vol)
        tid = ((c[:, 0] // tile[0]) * nTy + c[:, 1] // tile[1]) * nTx + c[:, 2] // tile[2]
        want = np.lexsort((raster, tid))
        assert np.array_equal(ix["perm"][b], want)
        counts = np.bincount(tid, minlength=nTz * nTy * nTx)
        assert np.array_equal(ix["tile_off"][b], np.concatenate([[0], np.cumsum(counts)]))
        grid = np.stack(np.meshgrid(np.arange(Z), np.arange(Y), np.arange(X), indexing="ij"),
                        -1).reshape(-1, 3)
        for t in range(nTz * nTy * nTx):
            Tz, Ty, Tx = t // (nTy * nTx), (t // nTx) % nTy, t % nTx
            lo = np.array([Tz * tile[0], Ty * tile[1], Tx * tile[2]])
            hi = np.minimum(lo + tile, (Z, Y, X)) - 1
            near = np.all((grid >= lo - r) & (grid <= hi + r), axis=1)
            got = ix["nbr"][b, ix["nbr_off"][b, t]:ix["nbr_off"][b, t + 1]]
            assert np.array_equal(got, vol[np.nonzero(near)[0]])


def test_bad_coordinates_rejected(oracle_lib):
    s = shape(B=1, H=1, d=12, Z=2, Y=2, X=2, block=(1, 1, 1))
    _, coords, _ = rand_inputs(s, seed=15)
    dup = coords.copy()
    dup[0, 1] = dup[0, 0]
    with pytest.raises(ValueError):
        oracle.volume(s, dup)
    out = coords.copy()
    out[0, 3, 2] = 2
    with pytest.raises(ValueError):
        oracle.volume(s, out)


# ---- packed-sequence comparison mode (1-D RoPE on the packed position) -------

def packed_shape(**kw):
    s = shape(**kw)
    s.rope_mode = oracle.ROPE_PACKED
    return s


def rotate_complex_1d(x, base):
    """One-dimensional RoPE as complex multiplication: pair (j, j + d/2) is the
    complex number x_j + i x_{j+d/2}, multiplied by exp(i p base^(-2j/d)) with p
    the row's position along axis -3 (the packed index)."""
    x = np.asarray(x, np.float64)
    d = x.shape[-1]
    h = d // 2
    theta = base ** (-2.0 * np.arange(h) / d)
    pos = np.arange(x.shape[-3], dtype=np.float64)[:, None, None]
    z = (x[..., :h] + 1j * x[..., h:]) * np.exp(1j * pos * theta)
    return np.concatenate([z.real, z.imag], axis=-1)


def test_packed_rope_matches_complex_rotation(oracle_lib):
    s = packed_shape(B=2, H=3, d=18, Z=5, Y=3, X=7, block=(1, 1, 1))
    packed, coords, _ = rand_inputs(s, seed=21)
    got = oracle.rope(s, coords, packed["q"])
    want = rotate_complex_1d(packed["q"].numpy(), s.rope_base)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)
    back = oracle.rope(s, coords, torch.from_numpy(got), transpose=True)
    np.testing.assert_allclose(back, packed["q"].numpy(), rtol=0, atol=1e-12)


def test_packed_rope_logit_depends_only_on_packed_displacement(oracle_lib):
    """With the same q and k in every row, q~_i . k~_j is a function of j - i."""
    s = packed_shape(B=1, H=1, d=24, Z=4, Y=4, X=4, block=(1, 1, 1))
    rng = np.random.default_rng(4)
    N = s.Z * s.Y * s.X
    q, k = rng.standard_normal(s.d), rng.standard_normal(s.d)
    coords = I.coords_of_order(rng.permutation(N), s.Z, s.Y, s.X)[None]
    rq = oracle.rope(s, coords, np.broadcast_to(q, (1, N, 1, s.d)).copy())[0, :, 0]
    rk = oracle.rope(s, coords, np.broadcast_to(k, (1, N, 1, s.d)).copy())[0, :, 0]
    L = rq @ rk.T
    for dlt in (-7, -1, 0, 3, 11):
        diag = np.array([L[i, i + dlt] for i in range(max(0, -dlt), min(N, N - dlt))])
        np.testing.assert_allclose(diag, diag[0], rtol=0, atol=1e-11)


def test_packed_mode_full_window_is_dense_1d_rope_attention(oracle_lib):
    """Full windows and 1x1x1 blocks: dense softmax attention over the packed
    sequence with one-dimensional RoPE (torch SDPA on independently rotated
    rows)."""
    s = packed_shape(B=2, H=2, d=12, Z=3, Y=4, X=5, window=(5, 7, 9), block=(1, 1, 1))
    packed, coords, _ = rand_inputs(s, seed=22)
    out, lse = oracle.forward(s, coords, packed["q"], packed["k"], packed["v"])
    tau = 1.0 / math.sqrt(s.d)
    for b in range(s.B):
        qr = torch.from_numpy(rotate_complex_1d(packed["q"][b].numpy(), s.rope_base))
        kr = torch.from_numpy(rotate_complex_1d(packed["k"][b].numpy(), s.rope_base))
        q, k, v = (t.permute(1, 0, 2) for t in (qr, kr, packed["v"][b]))
        ro = torch.nn.functional.scaled_dot_product_attention(q, k, v, scale=tau)
        rl = torch.logsumexp(tau * q @ k.transpose(1, 2), dim=-1)
        np.testing.assert_allclose(out[b], ro.permute(1, 0, 2).numpy(), rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[b], rl.numpy(), rtol=0, atol=1e-12)


def test_packed_mode_depends_on_the_packing(oracle_lib):
    """The failure mode the pages contrast axial RoPE with: the same field under
    two packings gives the same per-voxel output with axial RoPE and different
    outputs with RoPE on the packed position."""
    res = {}
    for mode in (oracle.ROPE_AXIAL, oracle.ROPE_PACKED):
        s = shape(B=1, H=2, d=12, Z=4, Y=4, X=8, window=(3, 3, 3), block=(2, 2, 4))
        s.rope_mode = mode
        g = torch.Generator().manual_seed(23)
        N = s.Z * s.Y * s.X
        grid = {n: torch.randn(1, N, s.H, s.d, generator=g, dtype=torch.float64) for n in "qkv"}
        outs = []
        for packing in ("raster", "random"):
            order = I.packing_order(packing, s.Z, s.Y, s.X, s.block, 5, 0)
            coords = I.coords_of_order(order, s.Z, s.Y, s.X)[None]
            pk = {n: t[:, torch.from_numpy(order)] for n, t in grid.items()}
            out, _ = oracle.forward(s, coords, pk["q"], pk["k"], pk["v"])
            o = np.empty_like(out)
            o[0, order] = out[0]
            outs.append(o)
        res[mode] = np.abs(outs[0] - outs[1]).max()
    assert res[oracle.ROPE_AXIAL] == 0.0
    assert res[oracle.ROPE_PACKED] > 1e-3


# ---- partly occupied volumes ----------------------------------------------

def partial_inputs(s, seed):
    """s.n_tokens distinct voxels per batch item (seeded), in a random packed
    order, with N(0, 1) q, k, v and dout per token."""
    g = torch.Generator().manual_seed(seed)
    V = s.Z * s.Y * s.X
    coords = np.stack([I.coords_of_order(torch.randperm(V, generator=g)[:s.n_tokens].numpy(),
                                         s.Z, s.Y, s.X) for _ in range(s.B)])
    packed = {n: torch.randn(s.B, s.n_tokens, s.H, s.d, generator=g, dtype=torch.float64)
              for n in ("q", "k", "v", "dout")}
    return packed, coords


PARTIAL = [
    dict(Z=4, Y=5, X=6, window=(3, 3, 3), block=(2, 3, 4), n_tokens=70),
    dict(Z=5, Y=4, X=6, window=(3, 1, 5), block=(2, 2, 3), n_tokens=24),
]


@pytest.mark.parametrize("cfg", PARTIAL, ids=["70_of_120", "24_of_120"])
@pytest.mark.parametrize("window_only", [False, True])
def test_partly_occupied_brute_force(oracle_lib, cfg, window_only):
    """Windows and blocks hold only the tokens present; a block's summary
    averages over them, a block holding none has no summary, exclusion follows
    the block's box; checked against the enumeration of brute_force."""
    s = shape(B=2, H=2, d=12, **cfg)
    packed, coords = partial_inputs(s, seed=31)
    out, lse = oracle.forward(s, coords, packed["q"], packed["k"], packed["v"],
                              window_only=window_only)
    assert out.shape == (s.B, s.n_tokens, s.H, s.d)
    for b in range(s.B):
        ro, rl = brute_force(s, packed, coords, b, window_only)
        np.testing.assert_allclose(out[b], ro, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[b], rl, rtol=0, atol=1e-12)


def test_sparse_case_has_empty_blocks(oracle_lib):
    """The sparse case above really leaves blocks without tokens (so the
    no-summary rule is exercised)."""
    s = shape(B=2, H=2, d=12, **PARTIAL[1])
    _, coords = partial_inputs(s, seed=31)
    nblk = np.prod([-(-n // e) for n, e in zip((s.Z, s.Y, s.X), s.block)])
    for b in range(s.B):
        held = {tuple(x) for x in coords[b].astype(np.int64) // np.asarray(s.block)}
        assert len(held) < nblk


def test_partly_occupied_packing_equivariance(oracle_lib):
    """Reordering the tokens of a partly occupied volume permutes the outputs
    and changes nothing else, bit for bit."""
    s = shape(B=2, H=2, d=12, **PARTIAL[0])
    packed, coords = partial_inputs(s, seed=32)
    out, lse = oracle.forward(s, coords, packed["q"], packed["k"], packed["v"])
    g = torch.Generator().manual_seed(5)
    perm = [torch.randperm(s.n_tokens, generator=g).numpy() for _ in range(s.B)]
    c2 = np.stack([coords[b][perm[b]] for b in range(s.B)])
    pk2 = {n: torch.stack([packed[n][b][torch.from_numpy(perm[b])] for b in range(s.B)])
           for n in "qkv"}
    out2, lse2 = oracle.forward(s, c2, pk2["q"], pk2["k"], pk2["v"])
    for b in range(s.B):
        np.testing.assert_array_equal(out2[b], out[b][perm[b]])
        np.testing.assert_array_equal(lse2[b], lse[b][:, perm[b]])


def test_full_occupancy_equals_dense(oracle_lib):
    """n_tokens = Z*Y*X describes the dense volume: same results, bit for bit."""
    s0 = shape(B=2, H=2, d=12, Z=4, Y=5, X=6, block=(2, 5, 3))
    s1 = shape(B=2, H=2, d=12, Z=4, Y=5, X=6, block=(2, 5, 3), n_tokens=120)
    packed, coords, _ = rand_inputs(s0, seed=33)
    args = (coords, packed["q"], packed["k"], packed["v"])
    for got, want in zip(oracle.forward(s1, *args), oracle.forward(s0, *args)):
        np.testing.assert_array_equal(got, want)
    for got, want in zip(oracle.backward(s1, *args, packed["dout"]),
                         oracle.backward(s0, *args, packed["dout"])):
        np.testing.assert_array_equal(got, want)


def test_partly_occupied_backward_finite_differences(oracle_lib):
    """Central differences of sum(dout * out) against the analytic gradients on
    a partly occupied volume with cut and empty blocks."""
    s = shape(B=1, H=2, d=12, Z=4, Y=4, X=5, window=(3, 3, 3), block=(3, 2, 2), n_tokens=30)
    packed, coords = partial_inputs(s, seed=34)
    dq, dk, dv = oracle.backward(s, coords, packed["q"], packed["k"], packed["v"],
                                 packed["dout"])
    grads = {"q": dq, "k": dk, "v": dv}
    rng = np.random.default_rng(2)
    eps = 1e-6
    dout = packed["dout"].numpy()
    for name in "qkv":
        for _ in range(12):
            idx = tuple(int(rng.integers(0, n)) for n in packed[name].shape)
            vals = {}
            for sign in (+1, -1):
                pk = {n: packed[n].clone() for n in "qkv"}
                pk[name][idx] += sign * eps
                out, _ = oracle.forward(s, coords, pk["q"], pk["k"], pk["v"])
                vals[sign] = (out * dout).sum()
            fd = (vals[1] - vals[-1]) / (2 * eps)
            assert abs(fd - grads[name][idx]) <= 1e-6 * max(1.0, abs(fd)), (name, idx)


def test_batch_items_are_independent(oracle_lib):
    """Batch items never interact: a two-item call equals two one-item calls,
    bit for bit (so ragged batches are item-by-item calls)."""
    s2 = shape(B=2, H=2, d=12, **PARTIAL[0])
    packed, coords = partial_inputs(s2, seed=35)
    out, lse = oracle.forward(s2, coords, packed["q"], packed["k"], packed["v"])
    s1 = shape(B=1, H=2, d=12, **PARTIAL[0])
    for b in range(2):
        o1, l1 = oracle.forward(s1, coords[b:b + 1], packed["q"][b:b + 1], packed["k"][b:b + 1],
                                packed["v"][b:b + 1])
        np.testing.assert_array_equal(o1[0], out[b])
        np.testing.assert_array_equal(l1[0], lse[b])


# ---- random geometries -------------------------------------------------------

@st.composite
def geometries(draw):
    Z, Y, X = (draw(st.integers(1, 5)) for _ in range(3))
    window = tuple(draw(st.sampled_from((1, 3, 5))) for _ in range(3))
    block = tuple(draw(st.integers(1, 4)) for _ in range(3))
    V = Z * Y * X
    n = draw(st.integers(1, V))
    return dict(B=draw(st.integers(1, 2)), H=draw(st.integers(1, 2)),
                d=draw(st.sampled_from((6, 12))), Z=Z, Y=Y, X=X, window=window, block=block,
                n_tokens=0 if n == V else n), draw(st.integers(0, 2**16)), draw(st.booleans())


@settings(max_examples=40, deadline=None, derandomize=True,
          suppress_health_check=[HealthCheck.too_slow, HealthCheck.function_scoped_fixture])
@given(geometries())
def test_random_geometries_against_brute_force(oracle_lib, case):
    """Random small volumes, windows, block extents (dividing or not) and
    occupancies, with and without summaries, against brute_force."""
    cfg, seed, window_only = case
    s = shape(**cfg)
    if s.n_tokens:
        packed, coords = partial_inputs(s, seed)
    else:
        packed, coords, _ = rand_inputs(s, seed=seed)
    out, lse = oracle.forward(s, coords, packed["q"], packed["k"], packed["v"],
                              window_only=window_only)
    for b in range(s.B):
        ro, rl = brute_force(s, packed, coords, b, window_only)
        np.testing.assert_allclose(out[b], ro, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[b], rl, rtol=0, atol=1e-12)
