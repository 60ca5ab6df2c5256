"""The z-slab sharded forward on one GPU: the ranks' library calls run one after
another on the same device (each on its slab with its halo planes, summaries of
its own blocks summed over the ranks), and the owned outputs, put together,
match the unsharded forward and the oracle."""
import numpy as np
import pytest
import torch

import oracle
from local_global_attention_b200 import configs as C
from local_global_attention_b200 import inputs as I
from local_global_attention_b200 import pack3d as P
from local_global_attention_b200 import sharding as S

from gpu_common import assert_close, gpu_run, oracle_sample

pytestmark = pytest.mark.gpu


def emulated_sharded_forward(wl, inp, world):
    """Every rank's calls in turn; the all-reduce of the summaries is their sum."""
    rz = (wl.window[0] - 1) // 2
    slabs = [s for s in S.plan_slabs(wl.Z, wl.block[0], rz, world) if s.owned]
    dev = {k: v.cuda() for k, v in inp.items() if k != "order"}
    calls = []
    ksum = vsum = None
    for slab in slabs:
        held_c, held = [], {"q": [], "k": [], "v": []}
        for b in range(wl.B):
            c, t = S.held_from_global(slab, dev["coords"][b],
                                      {n: dev[n][b] for n in ("q", "k", "v")})
            held_c.append(c)
            for n in held:
                held[n].append(t[n])
        hc = torch.stack(held_c).contiguous()
        hq, hk, hv = (torch.stack(held[n]).contiguous() for n in ("q", "k", "v"))
        params = P.make_params(S.slab_shape(wl, slab))
        idx = P.pack3d_build_index(params, hc)
        assert P.pack3d_index_check(idx) == P.OK
        ks, vs = P.pack3d_block_summaries(params, idx, hk, hv)
        ksum = ks if ksum is None else ksum + ks
        vsum = vs if vsum is None else vsum + vs
        calls.append((slab, params, idx, hc, hq, hk, hv))
    out = torch.zeros_like(dev["q"])
    lse = torch.zeros(wl.B, wl.H, wl.N, device="cuda")
    for slab, params, idx, hc, hq, hk, hv in calls:
        o, l = P.pack3d_forward(params, idx, hq, hk, hv, ksum, vsum)
        for b in range(wl.B):
            own = ((dev["coords"][b, :, 0] >= slab.z_lo) & (dev["coords"][b, :, 0] < slab.z_hi))
            pos = own.nonzero().squeeze(1)
            out[b].index_copy_(0, pos, o[b, :pos.numel()])
            lse[b].index_copy_(1, pos, l[b, :, :pos.numel()])
        assert P.pack3d_index_check(idx) == P.OK
    torch.cuda.synchronize()
    return out.cpu(), lse.cpu(), ksum.cpu(), vsum.cpu()


SHARD_CASES = [
    (I.Workload(name="shard_16x8x16", B=2, H=2, d=96, Z=16, Y=8, X=16, window=(5, 3, 7),
                block=(4, 4, 4), dtype="bf16", value_scale=1.0, seed=81), 2),
    (I.Workload(name="shard_cut_14x6x10", B=1, H=3, d=96, Z=14, Y=6, X=10, window=(3, 5, 3),
                block=(4, 3, 4), dtype="bf16", value_scale=1.0, seed=82), 3),
]


@pytest.mark.parametrize("wl,world", SHARD_CASES, ids=lambda x: getattr(x, "name", str(x)))
def test_sharded_forward_matches(oracle_lib, wl, world):
    inp = I.make_inputs(wl, "random")
    out, lse, ks, vs = emulated_sharded_forward(wl, inp, world)
    ref = gpu_run(wl, inp)
    # the summed summaries are the unsharded ones, bit for bit (one rank adds
    # each block, the others zeros)
    assert torch.equal(ks, ref["ksum"]) and torch.equal(vs, ref["vsum"])
    assert_close(out, ref["out"].double().numpy(), wl.dtype, "out vs unsharded")
    want_out, want_lse = oracle.forward(wl, inp["coords"], inp["q"], inp["k"], inp["v"])
    assert_close(out, want_out, wl.dtype, "out")
    assert_close(lse, want_lse, wl.dtype, "lse")


def test_sharded_forward_65k_two_slabs(oracle_lib):
    """The 65k benchmark volume cut into two z-slabs of 16 planes (+3 halo
    planes each): sampled queries against the oracle, and every output against
    the unsharded forward."""
    wl = C.VOL65K
    inp = I.make_inputs(wl, "random")
    out, lse, _, _ = emulated_sharded_forward(wl, inp, 2)
    ref = gpu_run(wl, inp)
    assert_close(out, ref["out"].double().numpy(), wl.dtype, "out vs unsharded")
    (b, h, i), o, l = oracle_sample(wl, inp, 24, seed=9)
    assert_close(out[b, i, h], o, wl.dtype, "out")
    assert_close(lse[b, h, i], l, wl.dtype, "lse")


def test_slab_calls_reject_other_paths():
    """z-slabs run the tensor-core forward of dense volumes with axial RoPE:
    the backward, fp32, the packed-RoPE mode and partly occupied volumes report
    ERR_UNSUPPORTED."""
    wl = SHARD_CASES[0][0]
    slab = S.plan_slabs(wl.Z, wl.block[0], 2, 2)[0]
    for variant in (dict(dtype="fp32"), dict(rope_mode=1)):
        shp = S.slab_shape(wl.replace(**variant), slab)
        params = P.make_params(shp)
        N = shp.Z * shp.Y * shp.X
        x = torch.zeros(wl.B, N, wl.H, wl.d, device="cuda",
                        dtype=torch.float32 if variant.get("dtype") == "fp32" else torch.bfloat16)
        idx = P.IndexBuffers(params)
        ks = torch.zeros(wl.B, wl.H, wl.n_blocks, wl.d, device="cuda")
        with pytest.raises(P.Pack3dError) as e:
            P.pack3d_forward(params, idx, x, x, x, ks, ks)
        assert e.value.status == P.ERR_UNSUPPORTED
    params = P.make_params(S.slab_shape(wl, slab))
    shp = S.slab_shape(wl, slab)
    N = shp.Z * shp.Y * shp.X
    x = torch.zeros(wl.B, N, wl.H, wl.d, device="cuda", dtype=torch.bfloat16)
    idx = P.IndexBuffers(params)
    lse = torch.zeros(wl.B, wl.H, N, device="cuda")
    with pytest.raises(P.Pack3dError) as e:
        P.pack3d_backward(params, idx, x, x, x, x, lse, x)
    assert e.value.status == P.ERR_UNSUPPORTED
