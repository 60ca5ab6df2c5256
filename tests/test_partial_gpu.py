"""Partly occupied volumes on the GPU against the oracle.

Every batch item holds n_tokens tokens at distinct voxels; windows and blocks
hold only the tokens present, a block's summary averages over them, and a
block holding none has no summary (the oracle's reading, pinned on the CPU).
The forward and backward run on the tensor-core path (bf16, head_dim 96);
the CUDA-core paths report ERR_UNSUPPORTED for such volumes, while the block
summaries are computed for every dtype."""
import numpy as np
import pytest
import torch

import oracle
from local_global_attention_b200 import inputs as I
from local_global_attention_b200 import pack3d as P

from gpu_common import assert_close, assert_grad_close, gpu_run

pytestmark = pytest.mark.gpu

PARTIAL = [
    # 700 of 1200 voxels, blocks cut at the volume's edge
    I.Workload(name="partial_700_of_6x10x20", B=2, H=2, d=96, Z=6, Y=10, X=20, window=(3, 5, 7),
               block=(4, 3, 8), dtype="bf16", value_scale=1.0, n_tokens=700, seed=71),
    # sparse: 90 of 640 voxels in 1 x 2 x 2 blocks, most of which are empty
    I.Workload(name="sparse_90_of_5x8x16", B=2, H=2, d=96, Z=5, Y=8, X=16, window=(3, 3, 5),
               block=(1, 2, 2), dtype="bf16", value_scale=1.0, n_tokens=90, seed=72),
    # more heads than the bulk staging gather takes
    I.Workload(name="partial_heads10_4x8x16", B=1, H=10, d=96, Z=4, Y=8, X=16, window=(3, 3, 5),
               block=(2, 4, 4), dtype="bf16", n_tokens=300, seed=73),
    # the packed-sequence comparison mode (RoPE on the packed index)
    I.Workload(name="partial_packed_rope_6x10x20", B=2, H=2, d=96, Z=6, Y=10, X=20,
               window=(3, 5, 7), block=(3, 5, 4), dtype="bf16", n_tokens=500, rope_mode=1,
               seed=74),
]


@pytest.mark.parametrize("wl", PARTIAL[:3], ids=lambda w: w.name)
def test_partial_index_bit_exact(oracle_lib, wl):
    inp = I.make_inputs(wl, "random")
    params = P.make_params(wl)
    idx = P.pack3d_build_index(params, inp["coords"].cuda())
    assert P.pack3d_index_check(idx) == P.OK
    got = {k: v.cpu().numpy() for k, v in idx.arrays().items()}
    want = oracle.build_index(wl, inp["coords"], tile=tuple(idx.struct.tile))
    for name in ("vol", "perm", "tile_off", "nbr"):
        np.testing.assert_array_equal(got[name], want[name], err_msg=name)
    for b in range(wl.B):
        np.testing.assert_array_equal(got["nbr_off"], want["nbr_off"][b])
    # tokens per block, from the coordinates
    c = inp["coords"].numpy().astype(np.int64)
    nby, nbx = -(-wl.Y // wl.block[1]), -(-wl.X // wl.block[2])
    for b in range(wl.B):
        bid = ((c[b, :, 0] // wl.block[0]) * nby + c[b, :, 1] // wl.block[1]) * nbx + \
            c[b, :, 2] // wl.block[2]
        np.testing.assert_array_equal(got["bcount"][b], np.bincount(bid, minlength=wl.n_blocks))


def test_sparse_case_has_empty_blocks():
    wl = PARTIAL[1]
    inp = I.make_inputs(wl, "random")
    params = P.make_params(wl)
    idx = P.pack3d_build_index(params, inp["coords"].cuda())
    assert P.pack3d_index_check(idx) == P.OK
    counts = idx.arrays()["bcount"].cpu().numpy()
    assert (counts == 0).sum() > wl.n_blocks // 4


@pytest.mark.parametrize("wl", PARTIAL, ids=lambda w: w.name)
@pytest.mark.parametrize("window_only", [False, True], ids=["pack3d", "window"])
def test_partial_forward(oracle_lib, wl, window_only):
    inp = I.make_inputs(wl, "random")
    res = gpu_run(wl, inp, window_only=window_only)
    out, lse = oracle.forward(wl, inp["coords"], inp["q"], inp["k"], inp["v"],
                              window_only=window_only)
    assert res["out"].shape == (wl.B, wl.n_tokens, wl.H, wl.d)
    assert_close(res["out"], out, wl.dtype, "out")
    assert_close(res["lse"], lse, wl.dtype, "lse")
    if not window_only:
        ks, vs = oracle.block_summaries(wl, inp["coords"], inp["k"], inp["v"])
        np.testing.assert_allclose(res["ksum"].double().numpy(), ks, rtol=0, atol=2e-5)
        np.testing.assert_allclose(res["vsum"].double().numpy(), vs, rtol=0, atol=2e-5)


@pytest.mark.parametrize("wl", PARTIAL, ids=lambda w: w.name)
def test_partial_backward(oracle_lib, wl):
    wl = wl.replace(value_scale=1.0 / np.sqrt(96))
    inp = I.make_inputs(wl, "random", with_dout=True)
    res = gpu_run(wl, inp, with_backward=True)
    want = oracle.backward(wl, inp["coords"], inp["q"], inp["k"], inp["v"], inp["dout"])
    for name, w in zip(("dq", "dk", "dv"), want):
        assert_grad_close(res[name], w, wl.dtype, name)


def test_partial_packing_equivariance_bit_exact():
    """The same occupied voxels and values under the four packings give the
    same per-voxel outputs and gradients, bit for bit."""
    wl = PARTIAL[0].replace(value_scale=1.0 / np.sqrt(96))
    grid = I.grid_tensors(wl, with_dout=True)
    ref = None
    for packing in I.PACKINGS:
        inp = I.make_inputs(wl, packing, grid=grid)
        res = gpu_run(wl, inp, with_backward=True)
        per_voxel = {}
        for name in ("out", "dq", "dk", "dv"):
            t = torch.zeros(wl.B, wl.V, wl.H, wl.d, dtype=res[name].dtype)
            for b in range(wl.B):
                t[b].index_copy_(0, inp["order"][b], res[name][b])
            per_voxel[name] = t
        if ref is None:
            ref = per_voxel
        else:
            for name in per_voxel:
                assert torch.equal(per_voxel[name], ref[name]), (packing, name)


def test_partial_cuda_core_paths(oracle_lib):
    """fp32: the block summaries are computed (any dtype); the forward and the
    backward, which run on the CUDA cores for fp32, report ERR_UNSUPPORTED."""
    wl = PARTIAL[0].replace(dtype="fp32", name="partial_fp32")
    inp = I.make_inputs(wl, "random", with_dout=True)
    d = {k: v.cuda() for k, v in inp.items() if k != "order"}
    params = P.make_params(wl)
    idx = P.pack3d_build_index(params, d["coords"])
    assert P.pack3d_index_check(idx) == P.OK
    ks, vs = P.pack3d_block_summaries(params, idx, d["k"], d["v"])
    torch.cuda.synchronize()
    wks, wvs = oracle.block_summaries(wl, inp["coords"], inp["k"], inp["v"])
    np.testing.assert_allclose(ks.double().cpu().numpy(), wks, rtol=0, atol=2e-5)
    np.testing.assert_allclose(vs.double().cpu().numpy(), wvs, rtol=0, atol=2e-5)
    with pytest.raises(P.Pack3dError) as e:
        P.pack3d_forward(params, idx, d["q"], d["k"], d["v"], ks, vs)
    assert e.value.status == P.ERR_UNSUPPORTED
    out = torch.zeros_like(d["q"])
    lse = torch.zeros(wl.B, wl.H, wl.N, device="cuda")
    with pytest.raises(P.Pack3dError) as e:
        P.pack3d_backward(params, idx, d["q"], d["k"], d["v"], out, lse, d["dout"])
    assert e.value.status == P.ERR_UNSUPPORTED
