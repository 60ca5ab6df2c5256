"""Shared helpers of the GPU tests: run the CUDA path through the C ABI and
compare it with the CPU oracle on the same seeded inputs."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from local_global_attention_b200 import inputs as I
from local_global_attention_b200 import pack3d as P

# Tolerances stated for the operator: bf16 inputs with fp32 accumulation
# (max-abs 2e-2, mean-abs 2e-3) and the fp32 mode (max-abs 1e-4).
TOL = {"bf16": (2e-2, 2e-3), "fp32": (1e-4, 1e-5)}


def to_cuda(inp):
    return {k: (v.cuda() if isinstance(v, torch.Tensor) and k != "order" else v)
            for k, v in inp.items()}


def gpu_run(wl, inp, window_only=False, with_backward=False, out_fp32=False):
    """Index, summaries, forward (and backward) on the GPU; CPU tensors back."""
    d = to_cuda(inp)
    params = P.make_params(wl, out_fp32=out_fp32)
    idx = P.pack3d_build_index(params, d["coords"])
    st = P.pack3d_index_check(idx)
    assert st == P.OK, P.strerror(st)
    res = {"index": idx, "params": params}
    if window_only:
        out, lse = P.pack3d_window_forward(params, idx, d["q"], d["k"], d["v"])
    else:
        ksum, vsum = P.pack3d_block_summaries(params, idx, d["k"], d["v"])
        out, lse = P.pack3d_forward(params, idx, d["q"], d["k"], d["v"], ksum, vsum)
        res["ksum"], res["vsum"] = ksum.cpu(), vsum.cpu()
    res["out"], res["lse"] = out, lse
    if with_backward:
        dq, dk, dv = P.pack3d_backward(params, idx, d["q"], d["k"], d["v"], out, lse, d["dout"])
        res["dq"], res["dk"], res["dv"] = dq.cpu(), dk.cpu(), dv.cpu()
    torch.cuda.synchronize()
    assert P.pack3d_index_check(idx) == P.OK
    res["out"], res["lse"] = out.cpu(), lse.cpu()
    return res


def errors(got, want):
    g = got.double().numpy() if isinstance(got, torch.Tensor) else np.asarray(got, np.float64)
    w = np.asarray(want, np.float64)
    assert g.shape == w.shape, (g.shape, w.shape)
    assert np.all(np.isfinite(g)), "non-finite GPU output"
    e = np.abs(g - w)
    return float(e.max()), float(e.mean())


def assert_close(got, want, dtype, what=""):
    mx, mean = errors(got, want)
    tmax, tmean = TOL[dtype]
    assert mx <= tmax and mean <= tmean, f"{what}: max-abs {mx:.3g} (<= {tmax}), mean-abs {mean:.3g} (<= {tmean})"
    return mx, mean


def assert_grad_close(got, want, dtype, what=""):
    """Gradient parity: the stated absolute bound (max-abs, mean-abs), and the
    same bound relative to the gradient's own largest magnitude when that is
    below 1, so that small gradients (bf16 dq and dk are O(1e-3) on the
    1/sqrt(96)-scaled workloads) are checked as tightly as O(1) outputs are."""
    mx, mean = assert_close(got, want, dtype, what)
    ref = float(np.abs(np.asarray(want, np.float64)).max())
    if 0.0 < ref < 1.0:
        tmax, tmean = TOL[dtype]
        assert mx <= tmax * ref and mean <= tmean * ref, (
            f"{what}: max-abs {mx:.3g} (<= {tmax * ref:.3g}), mean-abs {mean:.3g} "
            f"(<= {tmean * ref:.3g}) relative to max |{what}| = {ref:.3g}")
    return mx, mean


def sample_queries(wl, order, n, seed=0):
    """Packed indices of a query sample for one batch item: the 8 corners,
    points on faces and edges (one or two coordinates at the volume edge), and
    uniform random voxels."""
    rng = np.random.default_rng(seed)
    ext = (wl.Z, wl.Y, wl.X)
    pts = [(z, y, x) for z in (0, ext[0] - 1) for y in (0, ext[1] - 1) for x in (0, ext[2] - 1)]
    for m in range(max(0, n // 3)):
        c = [int(rng.integers(0, e)) for e in ext]
        for ax in rng.choice(3, size=1 + m % 2, replace=False):
            c[ax] = 0 if rng.integers(0, 2) == 0 else ext[ax] - 1
        pts.append(tuple(c))
    while len(pts) < n:
        pts.append(tuple(int(rng.integers(0, e)) for e in ext))
    vox = np.array([(z * ext[1] + y) * ext[2] + x for z, y, x in pts[:max(n, 8)]], np.int64)
    inv = np.empty_like(order)
    inv[order] = np.arange(order.size)
    return inv[vox]


def oracle_sample(wl, inp, n_per_bh, window_only=False, seed=0):
    """(b, h, i) sample and the oracle's out [n, d], lse [n] for it."""
    N = wl.N
    bs, hs, iis = [], [], []
    for b in range(wl.B):
        order = inp["order"][b].numpy()
        for h in range(wl.H):
            q = sample_queries(wl, order, n_per_bh, seed=seed + 97 * b + h)
            bs.append(np.full(q.size, b))
            hs.append(np.full(q.size, h))
            iis.append(q)
    b, h, i = (np.concatenate(a).astype(np.int64) for a in (bs, hs, iis))
    sel = oracle.flat_index(wl, b, h, i)
    out, lse = oracle.forward(wl, inp["coords"], inp["q"], inp["k"], inp["v"], sel=sel,
                              window_only=window_only)
    return (b, h, i), out, lse
