"""The allocation-free backward (pack3d_backward_noalloc) against the backward
that takes a caller-allocated workspace.

Some callers hold no device allocator of their own (a plugin whose host
framework owns all device memory, or code that must not allocate while
running), so the library also offers the backward with its workspace in a
static device array.  This file is collected last so that a run stopping at
the first failure has already run every other test; it also passes on its
own in a fresh process."""
import numpy as np
import pytest
import torch

from local_global_attention_b200 import configs as C
from local_global_attention_b200 import inputs as I
from local_global_attention_b200 import pack3d as P

from gpu_common import assert_grad_close

pytestmark = pytest.mark.gpu

CASES = [
    I.Workload(name="ragged_bf16_6x10x20", B=2, H=2, d=96, Z=6, Y=10, X=20, window=(5, 3, 7),
               block=(3, 5, 4), dtype="bf16", value_scale=1.0 / np.sqrt(96), seed=51),
    I.Workload(name="train_shape_16x16x32_fp32", B=1, H=4, d=96, Z=16, Y=16, X=32,
               window=(7, 7, 7), block=(8, 8, 8), dtype="fp32", seed=52),
]


def prepare(wl):
    """Inputs, index, forward and the workspace backward of one case."""
    inp = I.make_inputs(wl, "random", with_dout=True)
    d = {k: v.cuda() for k, v in inp.items() if k != "order"}
    params = P.make_params(wl)
    assert P.pack3d_backward_workspace_bytes(params) <= P.NOALLOC_SCRATCH_BYTES
    idx = P.pack3d_build_index(params, d["coords"])
    assert P.pack3d_index_check(idx) == P.OK
    ksum, vsum = P.pack3d_block_summaries(params, idx, d["k"], d["v"])
    out, lse = P.pack3d_forward(params, idx, d["q"], d["k"], d["v"], ksum, vsum)
    ref = P.pack3d_backward(params, idx, d["q"], d["k"], d["v"], out, lse, d["dout"])
    return params, idx, (d["q"], d["k"], d["v"], out, lse, d["dout"]), ref


def test_noalloc_backward_matches_workspace_backward():
    """The two cases alternate (A, B, A, B), so every call but the first finds
    the scratch array filled by a call of another shape and dtype.  Each call
    must agree with the workspace backward within the stated tolerance (for
    bf16 at head_dim 96 that one runs on the tensor cores, this one on the CUDA
    cores), and the two calls of a case must agree bit for bit: the reductions
    run in a fixed order, and no call reads scratch it has not written."""
    prepared = [prepare(wl) for wl in CASES]
    first = {}
    for call in range(2):
        for wl, (params, idx, args, ref) in zip(CASES, prepared):
            got = P.pack3d_backward_noalloc(params, idx, *args)
            torch.cuda.synchronize()
            for name, g_, r_ in zip(("dq", "dk", "dv"), got, ref):
                assert_grad_close(g_.cpu(), r_.double().cpu().numpy(), wl.dtype,
                                  f"{wl.name} call {call} {name}")
            if call == 0:
                first[wl.name] = [t.clone() for t in got]
            else:
                for name, g_, f_ in zip(("dq", "dk", "dv"), got, first[wl.name]):
                    assert torch.equal(g_, f_), (wl.name, name)
    for _, idx, _, _ in prepared:
        assert P.pack3d_index_check(idx) == P.OK


def test_noalloc_rejects_shapes_beyond_the_scratch():
    wl = C.MICRO1M  # workspace 34 MiB, above the 32 MiB array
    params = P.make_params(wl)
    assert P.pack3d_backward_workspace_bytes(params) > P.NOALLOC_SCRATCH_BYTES
    x = torch.zeros(1, device="cuda")
    idx = P.Index()
    st = P.load().pack3d_backward_noalloc(
        P.ctypes.byref(params), P.ctypes.byref(idx), *([P.ctypes.c_void_p(x.data_ptr())] * 3),
        P.ctypes.c_void_p(x.data_ptr()), P.ctypes.c_void_p(x.data_ptr()),
        P.ctypes.c_void_p(x.data_ptr()), *([P.ctypes.c_void_p(x.data_ptr())] * 3), None)
    assert st == P.ERR_UNSUPPORTED
