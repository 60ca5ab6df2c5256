"""Degenerate shapes on the GPU against the oracle, forward and backward:
a one-voxel volume (its block always meets the window: no summary term, the
output is v), one-voxel-thick planes and lines (a 1 x 1 x X line, a Z x 1 x 1
column), a block as large as the whole volume (one summary, never seen), and a
partly occupied volume holding a single token or one token per block; and a
bounded device wait that runs out (ERR_TIMEOUT, the context stays usable)."""
import numpy as np
import pytest

import oracle
from local_global_attention_b200 import inputs as I

from gpu_common import assert_close, assert_grad_close, gpu_run

pytestmark = pytest.mark.gpu

SCALE = 1.0 / np.sqrt(96)

EDGE = [
    # tensor-core path (bf16, head_dim 96) and CUDA-core path (fp32)
    I.Workload(name="one_voxel_bf16", B=1, H=2, d=96, Z=1, Y=1, X=1, window=(1, 1, 1),
               block=(1, 1, 1), dtype="bf16", value_scale=SCALE, seed=91),
    I.Workload(name="one_voxel_fp32_d12", B=2, H=1, d=12, Z=1, Y=1, X=1, window=(3, 3, 3),
               block=(1, 1, 1), dtype="fp32", seed=92),
    I.Workload(name="line_1x1x40_bf16", B=1, H=2, d=96, Z=1, Y=1, X=40, window=(1, 1, 5),
               block=(1, 1, 4), dtype="bf16", value_scale=SCALE, seed=93),
    I.Workload(name="column_12x1x1_bf16", B=2, H=1, d=96, Z=12, Y=1, X=1, window=(3, 1, 1),
               block=(3, 1, 1), dtype="bf16", value_scale=SCALE, seed=94),
    I.Workload(name="plane_1x9x20_fp32", B=1, H=2, d=96, Z=1, Y=9, X=20, window=(1, 3, 5),
               block=(1, 3, 5), dtype="fp32", seed=95),
    I.Workload(name="one_block_4x8x16_bf16", B=1, H=2, d=96, Z=4, Y=8, X=16, window=(3, 3, 3),
               block=(4, 8, 16), dtype="bf16", value_scale=SCALE, seed=96),
    I.Workload(name="single_token_of_5x8x16_bf16", B=2, H=2, d=96, Z=5, Y=8, X=16,
               window=(3, 3, 5), block=(1, 2, 2), dtype="bf16", value_scale=SCALE, n_tokens=1,
               seed=97),
    I.Workload(name="sparse_8_of_4x8x16_bf16", B=1, H=2, d=96, Z=4, Y=8, X=16, window=(1, 1, 1),
               block=(2, 4, 8), dtype="bf16", value_scale=SCALE, n_tokens=8, seed=98),
]


@pytest.mark.parametrize("wl", EDGE, ids=lambda w: w.name)
def test_edge_forward_and_backward(oracle_lib, wl):
    inp = I.make_inputs(wl, "random", with_dout=True)
    # the CUDA-core paths run dense volumes only
    backward = wl.dtype == "bf16" or not wl.n_tokens
    res = gpu_run(wl, inp, with_backward=backward)
    out, lse = oracle.forward(wl, inp["coords"], inp["q"], inp["k"], inp["v"])
    assert_close(res["out"], out, wl.dtype, "out")
    assert_close(res["lse"], lse, wl.dtype, "lse")
    if backward:
        want = oracle.backward(wl, inp["coords"], inp["q"], inp["k"], inp["v"], inp["dout"])
        for name, w in zip(("dq", "dk", "dv"), want):
            assert_grad_close(res[name], w, wl.dtype, name)


def test_one_voxel_output_is_v():
    """A single token sees only itself: out = v and lse = its own logit."""
    wl = EDGE[0]
    inp = I.make_inputs(wl, "random")
    res = gpu_run(wl, inp)
    np.testing.assert_array_equal(res["out"].float().numpy(), inp["v"].float().numpy())


def test_bounded_wait_times_out_and_the_context_stays_usable(oracle_lib):
    """A device wait on a barrier phase that nothing completes gives up after
    its poll limit and reports ERR_TIMEOUT; the next calls run normally."""
    from local_global_attention_b200 import pack3d as P
    assert P.pack3d_wait_selftest(1000) == P.ERR_TIMEOUT
    wl = EDGE[2]
    inp = I.make_inputs(wl, "random")
    res = gpu_run(wl, inp)
    out, lse = oracle.forward(wl, inp["coords"], inp["q"], inp["k"], inp["v"])
    assert_close(res["out"], out, wl.dtype, "out after the timed-out wait")
