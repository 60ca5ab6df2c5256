"""Forward parity of the CUDA path against the CPU oracle on seeded inputs.

Small volumes (several query tiles and ragged tails) are compared element by
element over every output; the full-size workloads in the launch
configuration the benchmark times are compared on sampled queries the oracle
computes one by one (corners, faces, edges and random voxels)."""
import numpy as np
import pytest
import torch

import oracle
from local_global_attention_b200 import configs as C
from local_global_attention_b200 import inputs as I
from local_global_attention_b200 import pack3d as P

from gpu_common import assert_close, gpu_run, oracle_sample

pytestmark = pytest.mark.gpu

RAGGED96 = I.Workload(name="ragged_6x10x20_d96", B=2, H=2, d=96, Z=6, Y=10, X=20,
                      window=(5, 3, 7), block=(3, 5, 4), dtype="bf16", value_scale=1.0,
                      seed=31)
# more heads than the bulk gather of the staging pass takes (its fallback path)
HEADS10 = I.Workload(name="heads10_4x8x16_d96", B=1, H=10, d=96, Z=4, Y=8, X=16,
                     window=(3, 3, 5), block=(2, 4, 4), dtype="bf16", seed=38)
SMALL = [
    C.TINY,
    RAGGED96,
    RAGGED96.replace(name="ragged_fp32_d96", dtype="fp32", seed=32),
    I.Workload(name="odd_5x9x17_d48", B=1, H=3, d=48, Z=5, Y=9, X=17, window=(3, 5, 3),
               block=(5, 3, 17), dtype="bf16", seed=33),
    I.Workload(name="big_window_8x8x16_d96", B=1, H=2, d=96, Z=8, Y=8, X=16, window=(15, 15, 31),
               block=(2, 4, 4), dtype="bf16", seed=34),
    I.Workload(name="self_window_4x4x8_d96", B=1, H=2, d=96, Z=4, Y=8, X=8, window=(1, 1, 1),
               block=(2, 2, 2), dtype="bf16", seed=35),
    I.Workload(name="d12_fp32_6x6x6", B=2, H=2, d=12, Z=6, Y=6, X=6, window=(3, 3, 3),
               block=(2, 3, 6), dtype="fp32", seed=36),
    I.Workload(name="d24_bf16_4x12x9", B=1, H=2, d=24, Z=4, Y=12, X=9, window=(3, 5, 5),
               block=(2, 6, 3), dtype="bf16", seed=37),
    HEADS10,
]


def full_oracle(wl, inp, window_only):
    return oracle.forward(wl, inp["coords"], inp["q"], inp["k"], inp["v"], window_only=window_only)


@pytest.mark.parametrize("wl", SMALL, ids=lambda w: w.name)
@pytest.mark.parametrize("window_only", [False, True], ids=["pack3d", "window"])
def test_forward_small_full(oracle_lib, wl, window_only):
    inp = I.make_inputs(wl, "random")
    res = gpu_run(wl, inp, window_only=window_only)
    out, lse = full_oracle(wl, inp, window_only)
    assert_close(res["out"], out, wl.dtype, "out")
    assert_close(res["lse"], lse, wl.dtype, "lse")


@pytest.mark.parametrize("wl", [C.TINY, RAGGED96, C.VOL16K], ids=lambda w: w.name)
def test_block_summaries(oracle_lib, wl):
    inp = I.make_inputs(wl, wl.packings[0])
    res = gpu_run(wl, inp)
    ks, vs = oracle.block_summaries(wl, inp["coords"], inp["k"], inp["v"])
    # fp32 accumulation of exactly represented inputs: relative error ~1e-6
    np.testing.assert_allclose(res["ksum"].double().numpy(), ks, rtol=0, atol=2e-5)
    np.testing.assert_allclose(res["vsum"].double().numpy(), vs, rtol=0, atol=2e-5)


@pytest.mark.slow
def test_forward_vol16k_full(oracle_lib):
    wl = C.VOL16K
    inp = I.make_inputs(wl, "morton")
    res = gpu_run(wl, inp)
    out, lse = full_oracle(wl, inp, False)
    assert_close(res["out"], out, wl.dtype, "out")
    assert_close(res["lse"], lse, wl.dtype, "lse")


@pytest.fixture(scope="module")
def grid65k():
    return I.grid_tensors(C.VOL65K)


@pytest.mark.parametrize("packing", I.PACKINGS)
def test_forward_65k_sampled(oracle_lib, grid65k, packing):
    wl = C.VOL65K
    inp = I.make_inputs(wl, packing, grid=grid65k)
    res = gpu_run(wl, inp)
    (b, h, i), out, lse = oracle_sample(wl, inp, 48, seed=5)
    assert_close(res["out"][b, i, h], out, wl.dtype, "out")
    assert_close(res["lse"][b, h, i], lse, wl.dtype, "lse")
    wres = gpu_run(wl, inp, window_only=True)
    (b, h, i), wout, wlse = oracle_sample(wl, inp, 24, window_only=True, seed=6)
    assert_close(wres["out"][b, i, h], wout, wl.dtype, "window out")
    assert_close(wres["lse"][b, h, i], wlse, wl.dtype, "window lse")


def test_forward_65k_packing_equivariance_bit_exact(grid65k):
    """Every packing of the same field gives the same per-voxel output, bit for
    bit: all accumulation orders follow the grid, never the memory order."""
    wl = C.VOL65K
    ref = None
    for packing in I.PACKINGS:
        inp = I.make_inputs(wl, packing, grid=grid65k)
        res = gpu_run(wl, inp)
        out = I.unpack_rows(res["out"], inp["order"])
        lse = I.unpack_rows(res["lse"].permute(0, 2, 1), inp["order"])
        if ref is None:
            ref = (out, lse)
        else:
            assert torch.equal(out, ref[0]), packing
            assert torch.equal(lse, ref[1]), packing


@pytest.mark.parametrize("wl", [RAGGED96, SMALL[3]], ids=lambda w: w.name)
def test_forward_fp32_output(oracle_lib, wl):
    """bf16 inputs, fp32 output: the same kernels without the output rounding."""
    inp = I.make_inputs(wl, "random")
    res = gpu_run(wl, inp, out_fp32=True)
    assert res["out"].dtype == torch.float32
    out, lse = full_oracle(wl, inp, False)
    mx, _ = assert_close(res["out"], out, wl.dtype, "out")
    assert_close(res["lse"], lse, wl.dtype, "lse")


@pytest.mark.slow
def test_forward_micro1m_sampled(oracle_lib):
    """1M-token smooth field.  |out| reaches 4-5 here, where bf16 output
    rounding alone is up to 0.016, so the output is kept in fp32 (the inputs and
    the tensor-core arithmetic are the bf16 path's)."""
    wl = C.MICRO1M
    dev = "cuda"
    inp = I.make_inputs(wl, "block", grid=I.grid_tensors(wl, device=dev))
    res = gpu_run(wl, inp, out_fp32=True)
    (b, h, i), out, lse = oracle_sample(wl, inp, 64, seed=7)
    assert_close(res["out"][b, i, h], out, wl.dtype, "out")
    assert_close(res["lse"][b, h, i], lse, wl.dtype, "lse")


@pytest.mark.parametrize("wl", [RAGGED96, HEADS10, C.VOL16K], ids=lambda w: w.name)
def test_staged_halves(oracle_lib, wl):
    """pack3d_stage_kv with summaries computes the same summaries as
    pack3d_block_summaries (bit for bit) and stages the same grid-order keys
    and values as pack3d_forward does; pack3d_forward_staged then gives
    pack3d_forward's result, and the window-only halves pack3d_window_forward's."""
    inp = I.make_inputs(wl, "random")
    d = {k: v.cuda() for k, v in inp.items() if k != "order"}
    params = P.make_params(wl)
    idx = P.pack3d_build_index(params, d["coords"])
    ks_ref, vs_ref = P.pack3d_block_summaries(params, idx, d["k"], d["v"])
    out_ref, lse_ref = P.pack3d_forward(params, idx, d["q"], d["k"], d["v"], ks_ref, vs_ref)
    wout_ref, wlse_ref = P.pack3d_window_forward(params, idx, d["q"], d["k"], d["v"])
    # staging alone (what pack3d_forward stages) vs staging fused with the summaries
    ws_plain = P.pack3d_stage_kv(params, idx, d["k"], d["v"])
    ks = torch.full_like(ks_ref, float("nan"))
    vs = torch.full_like(vs_ref, float("nan"))
    ws = P.pack3d_stage_kv(params, idx, d["k"], d["v"], ks, vs)
    torch.cuda.synchronize()
    assert torch.equal(ks, ks_ref) and torch.equal(vs, vs_ref)
    kv_bytes = 2 * wl.B * wl.H * wl.N * wl.d * 2  # grid-order k and v (256-aligned here)
    assert torch.equal(ws[:kv_bytes], ws_plain[:kv_bytes])
    out, lse = P.pack3d_forward_staged(params, idx, d["q"], ws, with_summaries=True)
    assert torch.equal(out, out_ref) and torch.equal(lse, lse_ref)
    wout, wlse = P.pack3d_forward_staged(params, idx, d["q"], ws_plain, with_summaries=False)
    assert torch.equal(wout, wout_ref) and torch.equal(wlse, wlse_ref)
    assert P.pack3d_index_check(idx) == P.OK
    ref = oracle.forward(wl, inp["coords"], inp["q"], inp["k"], inp["v"])
    assert_close(out.cpu(), ref[0], wl.dtype, "out")


# ---- packed-sequence comparison mode (1-D RoPE on the packed index) --------

PACKED_SMALL = [
    RAGGED96.replace(name="packed_rope_ragged_d96", rope_mode=1, seed=51),
    RAGGED96.replace(name="packed_rope_ragged_fp32", dtype="fp32", rope_mode=1, seed=52),
    SMALL[3].replace(name="packed_rope_odd_d48", rope_mode=1, seed=53),
    HEADS10.replace(name="packed_rope_heads10", rope_mode=1, seed=54),
]


@pytest.mark.parametrize("wl", PACKED_SMALL, ids=lambda w: w.name)
@pytest.mark.parametrize("window_only", [False, True], ids=["pack3d", "window"])
def test_packed_rope_mode_small_full(oracle_lib, wl, window_only):
    inp = I.make_inputs(wl, "random")
    res = gpu_run(wl, inp, window_only=window_only)
    out, lse = full_oracle(wl, inp, window_only)
    assert_close(res["out"], out, wl.dtype, "out")
    assert_close(res["lse"], lse, wl.dtype, "lse")
    if not window_only:
        ks, vs = oracle.block_summaries(wl, inp["coords"], inp["k"], inp["v"])
        np.testing.assert_allclose(res["ksum"].double().numpy(), ks, rtol=0, atol=2e-5)


def test_packed_rope_mode_staged_halves(oracle_lib):
    test_staged_halves(oracle_lib, PACKED_SMALL[0])


def test_packed_rope_mode_65k(oracle_lib, grid65k):
    """The comparison mode at the benchmark shape: parity on sampled queries
    under random packing, and the failure mode the pages contrast axial RoPE
    with - the per-voxel result changes with the packing."""
    wl = C.VOL65K.replace(rope_mode=1)
    outs = []
    for packing in ("raster", "random"):
        inp = I.make_inputs(wl, packing, grid=grid65k)
        res = gpu_run(wl, inp)
        if packing == "random":
            (b, h, i), out, lse = oracle_sample(wl, inp, 32, seed=8)
            assert_close(res["out"][b, i, h], out, wl.dtype, "out")
            assert_close(res["lse"][b, h, i], lse, wl.dtype, "lse")
        outs.append(I.unpack_rows(res["out"], inp["order"]).float())
    # (axial RoPE gives bit-identical outputs here, see the equivariance test)
    assert (outs[0] - outs[1]).abs().max().item() > 1e-4


# ---- blocks cut at the volume's edge -----------------------------------------
# Where a block extent does not divide the volume, the last block along that
# axis holds only the voxels inside the volume; its summary averages over them.

CUT_SMALL = [
    I.Workload(name="cut_bf16_d96_6x10x20", B=2, H=2, d=96, Z=6, Y=10, X=20, window=(3, 5, 7),
               block=(4, 3, 8), dtype="bf16", value_scale=1.0, seed=61),
    I.Workload(name="cut_fp32_d96_5x7x19", B=1, H=2, d=96, Z=5, Y=7, X=19, window=(3, 3, 5),
               block=(2, 4, 6), dtype="fp32", seed=62),
    I.Workload(name="cut_bf16_d48_7x5x9", B=1, H=3, d=48, Z=7, Y=5, X=9, window=(3, 3, 3),
               block=(3, 2, 4), dtype="bf16", seed=63),
    # a block wider than the volume along x and z (one cut block per axis)
    I.Workload(name="cut_wide_bf16_d96_3x8x12", B=1, H=2, d=96, Z=3, Y=8, X=12,
               window=(1, 3, 3), block=(4, 3, 16), dtype="bf16", seed=64),
    # more heads than the bulk gather takes (the per-thread gather kernel)
    I.Workload(name="cut_heads10_bf16_d96_5x6x10", B=1, H=10, d=96, Z=5, Y=6, X=10,
               window=(3, 3, 5), block=(2, 4, 4), dtype="bf16", seed=65),
]


@pytest.mark.parametrize("wl", CUT_SMALL, ids=lambda w: w.name)
def test_cut_blocks_forward_and_summaries(oracle_lib, wl):
    inp = I.make_inputs(wl, "random")
    res = gpu_run(wl, inp)
    out, lse = full_oracle(wl, inp, False)
    assert_close(res["out"], out, wl.dtype, "out")
    assert_close(res["lse"], lse, wl.dtype, "lse")
    ks, vs = oracle.block_summaries(wl, inp["coords"], inp["k"], inp["v"])
    assert res["ksum"].shape[2] == wl.n_blocks
    np.testing.assert_allclose(res["ksum"].double().numpy(), ks, rtol=0, atol=2e-5)
    np.testing.assert_allclose(res["vsum"].double().numpy(), vs, rtol=0, atol=2e-5)


@pytest.mark.parametrize("wl", [CUT_SMALL[0], CUT_SMALL[3], CUT_SMALL[4]], ids=lambda w: w.name)
def test_cut_blocks_staged_halves(oracle_lib, wl):
    """The fused staging pass computes the cut blocks' summaries bit for bit as
    pack3d_block_summaries does."""
    test_staged_halves(oracle_lib, wl)
