"""The z-slab sharded forward and backward on one GPU: the ranks' library calls
run one after another on the same device (each on its slab with its halo
planes; the all-reduces of the summaries and of the summary gradients are sums
over the ranks), and the owned outputs and gradients, put together, match the
unsharded calls and the oracle."""
import numpy as np
import pytest
import torch

import oracle
from local_global_attention_b200 import configs as C
from local_global_attention_b200 import inputs as I
from local_global_attention_b200 import pack3d as P
from local_global_attention_b200 import sharding as S

from gpu_common import assert_close, assert_grad_close, gpu_run, oracle_sample

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


def test_sharded_window_only_forward(oracle_lib):
    """The window-only forward on slabs needs no exchange but the halo: every
    rank's owned outputs against the unsharded window-only forward and the
    oracle."""
    wl, world = SHARD_CASES[1]
    inp = I.make_inputs(wl, "random")
    rz = (wl.window[0] - 1) // 2
    dev = {k: v.cuda() for k, v in inp.items() if k != "order"}
    out = torch.zeros_like(dev["q"])
    lse = torch.zeros(wl.B, wl.H, wl.N, device="cuda")
    for slab in (s for s in S.plan_slabs(wl.Z, wl.block[0], rz, world) if s.owned):
        held_c, held = [], {"q": [], "k": [], "v": []}
        for b in range(wl.B):
            c, t = S.held_from_global(slab, dev["coords"][b],
                                      {n: dev[n][b] for n in ("q", "k", "v")})
            held_c.append(c)
            for n in held:
                held[n].append(t[n])
        params = P.make_params(S.slab_shape(wl, slab))
        idx = P.pack3d_build_index(params, torch.stack(held_c).contiguous())
        assert P.pack3d_index_check(idx) == P.OK
        o, l = P.pack3d_window_forward(params, idx, *(torch.stack(held[n]).contiguous()
                                                      for n in ("q", "k", "v")))
        for b in range(wl.B):
            own = (dev["coords"][b, :, 0] >= slab.z_lo) & (dev["coords"][b, :, 0] < slab.z_hi)
            pos = own.nonzero().squeeze(1)
            out[b].index_copy_(0, pos, o[b, :pos.numel()])
            lse[b].index_copy_(1, pos, l[b, :, :pos.numel()])
    torch.cuda.synchronize()
    ref = gpu_run(wl, inp, window_only=True)
    assert_close(out.cpu(), ref["out"].double().numpy(), wl.dtype, "out vs unsharded")
    want_out, want_lse = oracle.forward(wl, inp["coords"], inp["q"], inp["k"], inp["v"],
                                        window_only=True)
    assert_close(out.cpu(), want_out, wl.dtype, "out")
    assert_close(lse.cpu(), want_lse, wl.dtype, "lse")


def emulated_sharded_backward(wl, inp, world, out, lse):
    """The backward of every rank in turn: held tensors (halo planes included)
    cut from the global ones, summary gradients over each rank's owned queries
    summed over the ranks, then each rank's owned dq, dk, dv.  out, lse: the
    global forward results the backward differentiates."""
    rz = (wl.window[0] - 1) // 2
    slabs = [s for s in S.plan_slabs(wl.Z, wl.block[0], rz, world) if s.owned]
    dev = {k: v.cuda() for k, v in inp.items() if k != "order"}
    dev["out"] = out.cuda()
    dev["lse_t"] = lse.cuda().transpose(1, 2)
    names = ("q", "k", "v", "out", "dout", "lse_t")
    calls = []
    ksum = vsum = None
    for slab in slabs:
        held_c, held = [], {n: [] for n in names}
        for b in range(wl.B):
            c, t = S.held_from_global(slab, dev["coords"][b], {n: dev[n][b] for n in names})
            held_c.append(c)
            for n in names:
                held[n].append(t[n])
        hc = torch.stack(held_c).contiguous()
        h = {n: torch.stack(held[n]).contiguous() for n in names}
        h["lse"] = h.pop("lse_t").transpose(1, 2).contiguous()
        params = P.make_params(S.slab_shape(wl, slab))
        idx = P.pack3d_build_index(params, hc)
        assert P.pack3d_index_check(idx) == P.OK
        ks, vs = P.pack3d_block_summaries(params, idx, h["k"], h["v"])
        ksum = ks if ksum is None else ksum + ks
        vsum = vs if vsum is None else vsum + vs
        calls.append((slab, params, idx, h))
    dks = dvs = None
    staged = []
    for slab, params, idx, h in calls:
        a, c, ws = P.pack3d_backward_summary_grads(params, idx, h["q"], h["k"], h["v"], h["out"],
                                                   h["lse"], h["dout"], ksum, vsum)
        dks = a if dks is None else dks + a
        dvs = c if dvs is None else dvs + c
        staged.append(ws)
    grads = {n: torch.zeros_like(dev[n]) for n in ("q", "k", "v")}
    for (slab, params, idx, h), ws in zip(calls, staged):
        g = [torch.zeros_like(h[n]) for n in ("q", "k", "v")]
        P.pack3d_backward_from_summary_grads(params, idx, dks, dvs, ws, *g)
        for b in range(wl.B):
            own = ((dev["coords"][b, :, 0] >= slab.z_lo) & (dev["coords"][b, :, 0] < slab.z_hi))
            pos = own.nonzero().squeeze(1)
            for n, t in zip(("q", "k", "v"), g):
                grads[n][b].index_copy_(0, pos, t[b, :pos.numel()])
        assert P.pack3d_index_check(idx) == P.OK
    torch.cuda.synchronize()
    return grads["q"].cpu(), grads["k"].cpu(), grads["v"].cpu()


@pytest.mark.parametrize("wl,world", SHARD_CASES, ids=lambda x: getattr(x, "name", str(x)))
def test_sharded_backward_matches(oracle_lib, wl, world):
    wl = wl.replace(value_scale=1.0 / np.sqrt(96))
    inp = I.make_inputs(wl, "random", with_dout=True)
    ref = gpu_run(wl, inp, with_backward=True)
    got = emulated_sharded_backward(wl, inp, world, ref["out"], ref["lse"])
    want = oracle.backward(wl, inp["coords"], inp["q"], inp["k"], inp["v"], inp["dout"])
    for name, g, w in zip(("dq", "dk", "dv"), got, want):
        assert_grad_close(g, ref[name].double().numpy(), wl.dtype, f"{name} vs unsharded")
        assert_grad_close(g, w, wl.dtype, name)


def test_two_call_backward_is_the_backward():
    """Without a slab, the two calls with nothing between them are
    pack3d_backward, bit for bit (given summaries or computed ones)."""
    wl = SHARD_CASES[0][0].replace(value_scale=1.0 / np.sqrt(96), name="two_call")
    inp = I.make_inputs(wl, "random", with_dout=True)
    ref = gpu_run(wl, inp, with_backward=True)
    d = {k: v.cuda() for k, v in inp.items() if k != "order"}
    params, idx = ref["params"], ref["index"]
    out, lse = ref["out"].cuda(), ref["lse"].cuda()
    ksum, vsum = ref["ksum"].cuda(), ref["vsum"].cuda()
    for given in (False, True):
        dks, dvs, ws = P.pack3d_backward_summary_grads(
            params, idx, d["q"], d["k"], d["v"], out, lse, d["dout"],
            ksum if given else None, vsum if given else None)
        g = [torch.empty_like(d[n]) for n in ("q", "k", "v")]
        P.pack3d_backward_from_summary_grads(params, idx, dks, dvs, ws, *g)
        torch.cuda.synchronize()
        for name, t in zip(("dq", "dk", "dv"), g):
            assert torch.equal(t.cpu(), ref[name]), (given, name)


@pytest.mark.parametrize("variant", ["partial", "packed_rope"])
def test_two_call_backward_other_modes(variant):
    """The two calls equal pack3d_backward bit for bit for a partly occupied
    volume and in the packed-sequence RoPE mode (both unsharded)."""
    base = SHARD_CASES[0][0].replace(value_scale=1.0 / np.sqrt(96), name="two_call_" + variant)
    wl = base.replace(n_tokens=1500) if variant == "partial" else base.replace(rope_mode=1)
    inp = I.make_inputs(wl, "random", with_dout=True)
    ref = gpu_run(wl, inp, with_backward=True)
    d = {k: v.cuda() for k, v in inp.items() if k != "order"}
    dks, dvs, ws = P.pack3d_backward_summary_grads(
        ref["params"], ref["index"], d["q"], d["k"], d["v"], ref["out"].cuda(),
        ref["lse"].cuda(), d["dout"])
    g = [torch.empty_like(d[n]) for n in ("q", "k", "v")]
    P.pack3d_backward_from_summary_grads(ref["params"], ref["index"], dks, dvs, ws, *g)
    torch.cuda.synchronize()
    for name, t in zip(("dq", "dk", "dv"), g):
        assert torch.equal(t.cpu(), ref[name]), name


def test_sharded_backward_65k_two_slabs(oracle_lib):
    """The 65k training shape cut into two z-slabs: every gradient against the
    unsharded backward, and one (batch item, head) slice against the oracle."""
    wl = C.TRAIN65K
    inp = I.make_inputs(wl, "random", with_dout=True)
    ref = gpu_run(wl, inp, with_backward=True)
    got = emulated_sharded_backward(wl, inp, 2, ref["out"], ref["lse"])
    for name, g in zip(("dq", "dk", "dv"), got):
        assert_grad_close(g, ref[name].double().numpy(), wl.dtype, f"{name} vs unsharded")
    one = wl.replace(B=1, H=1)
    b, h = 1, 3
    sl = {n: inp[n][b:b + 1, :, h:h + 1].contiguous() for n in ("q", "k", "v", "dout")}
    want = oracle.backward(one, inp["coords"][b:b + 1], sl["q"], sl["k"], sl["v"], sl["dout"])
    for name, g, w in zip(("dq", "dk", "dv"), got, want):
        assert_grad_close(g[b:b + 1, :, h:h + 1], w, wl.dtype, f"{name}[b={b}, h={h}]")


def test_slab_calls_reject_other_paths():
    """z-slabs run the tensor-core path of dense volumes with axial RoPE:
    fp32 and the packed-RoPE mode report ERR_UNSUPPORTED, and so does the
    one-call backward (a slab's summary gradients need the exchange between the
    two calls)."""
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


def test_sharded_entry_points_single_rank():
    """sharding.sharded_forward and sharded_backward end to end in a one-rank
    process group (gloo): the slab is the whole volume, so out, lse and the
    gradients equal the unsharded calls bit for bit."""
    import socket

    import torch.distributed as dist
    wl = SHARD_CASES[0][0].replace(value_scale=1.0 / np.sqrt(96), name="single_rank")
    inp = I.make_inputs(wl, "random", with_dout=True)
    ref = gpu_run(wl, inp, with_backward=True)
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1)
    try:
        slab = S.plan_slabs(wl.Z, wl.block[0], (wl.window[0] - 1) // 2, 1)[0]
        d = {k: v.cuda() for k, v in inp.items() if k != "order"}
        coords = d["coords"].to(torch.int16)
        out, lse = S.sharded_forward(wl, slab, coords, d["q"], d["k"], d["v"])
        dq, dk, dv = S.sharded_backward(wl, slab, coords, d["q"], d["k"], d["v"], out, lse,
                                        d["dout"])
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    assert torch.equal(out.cpu(), ref["out"]) and torch.equal(lse.cpu(), ref["lse"])
    for name, g in zip(("dq", "dk", "dv"), (dq, dk, dv)):
        assert torch.equal(g.cpu(), ref[name]), name
