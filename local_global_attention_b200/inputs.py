"""Seeded synthetic workloads for the PACK3D operator.

This module only draws numbers and orders tokens; it holds none of the
operator's arithmetic (no rotation, no window, no block or softmax logic), so
both the CUDA path and the CPU oracle can be fed from it.

Memory orders ("packings") follow the four repackings the paper names in its
abstract ("Geometry Matters in Packed 3D Attention": Morton, block-contiguous
and random repacking, plus the plain raster order):

* ``raster``  - z-major, then y, then x.
* ``morton``  - ascending Morton code; bit k of x, y, z goes to bit 3k, 3k+1,
  3k+2 of the code (interleaving up to the largest extent), so the order is
  defined for non-cubic volumes too.
* ``block``   - block-contiguous: the summary blocks in raster order, raster
  order inside each block.
* ``random``  - a seeded uniform permutation (one per batch item).

A workload's tensors are drawn in fp32 in grid raster order from one
``torch.Generator`` seeded with the workload seed, in the order q, k, v, dO;
they are rounded to the working dtype and then permuted into the packing.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

PACKINGS = ("raster", "morton", "block", "random")


def raster_coords(Z: int, Y: int, X: int) -> np.ndarray:
    """(z, y, x) of every voxel in raster order, shape [Z*Y*X, 3], int64."""
    z, y, x = np.meshgrid(np.arange(Z), np.arange(Y), np.arange(X), indexing="ij")
    return np.stack([z.ravel(), y.ravel(), x.ravel()], axis=1).astype(np.int64)


def _morton_codes(c: np.ndarray, nbits: int) -> np.ndarray:
    code = np.zeros(c.shape[0], dtype=np.int64)
    for k in range(nbits):
        code |= ((c[:, 2] >> k) & 1) << (3 * k)
        code |= ((c[:, 1] >> k) & 1) << (3 * k + 1)
        code |= ((c[:, 0] >> k) & 1) << (3 * k + 2)
    return code


def packing_order(name: str, Z: int, Y: int, X: int, block=(1, 1, 1), seed: int = 0,
                  item: int = 0) -> np.ndarray:
    """Voxel raster index held by each packed slot: ``order[p]`` (int64, length N)."""
    N = Z * Y * X
    if name == "raster":
        return np.arange(N, dtype=np.int64)
    c = raster_coords(Z, Y, X)
    if name == "morton":
        nbits = max(1, int(math.ceil(math.log2(max(Z, Y, X)))))
        return np.argsort(_morton_codes(c, nbits), kind="stable").astype(np.int64)
    if name == "block":
        bz, by, bx = block
        nby, nbx = -(-Y // by), -(-X // bx)
        bid = ((c[:, 0] // bz) * nby + (c[:, 1] // by)) * nbx + (c[:, 2] // bx)
        inner = ((c[:, 0] % bz) * by + (c[:, 1] % by)) * bx + (c[:, 2] % bx)
        return np.lexsort((inner, bid)).astype(np.int64)
    if name == "random":
        g = torch.Generator().manual_seed(1_000_003 * (seed + 1) + item)
        return torch.randperm(N, generator=g).numpy().astype(np.int64)
    raise ValueError(f"unknown packing {name!r}")


def coords_of_order(order: np.ndarray, Z: int, Y: int, X: int) -> np.ndarray:
    """int16 (z, y, x) of the token in each packed slot, shape [N, 3]."""
    o = np.asarray(order, dtype=np.int64)
    x = o % X
    y = (o // X) % Y
    z = o // (X * Y)
    return np.stack([z, y, x], axis=1).astype(np.int16)


def _gauss_kernel(sigma: float, radius: int) -> torch.Tensor:
    t = torch.arange(-radius, radius + 1, dtype=torch.float64)
    w = torch.exp(-0.5 * (t / sigma) ** 2)
    return (w / w.sum()).to(torch.float32)


def _blur_axis(f: torch.Tensor, axis: int, w: torch.Tensor) -> torch.Tensor:
    """Convolve the [Z, Y, X, C] field along one spatial axis, reflect boundary."""
    r = (w.numel() - 1) // 2
    moved = f.movedim(axis, -1)
    shp = moved.shape
    flat = moved.reshape(-1, 1, shp[-1])
    out = torch.nn.functional.conv1d(
        torch.nn.functional.pad(flat, (r, r), mode="reflect"), w.view(1, 1, -1).to(f.device))
    return out.reshape(shp).movedim(-1, axis)


def smooth_field(gen: torch.Generator, Z, Y, X, C, sigma=2.0, radius=8, noise=0.1,
                 device="cpu") -> torch.Tensor:
    """Gaussian-blurred N(0,1) noise, each channel rescaled to unit std, plus
    N(0, noise^2) noise. Shape [Z*Y*X, C], fp32, raster order."""
    f = torch.randn(Z, Y, X, C, generator=gen, dtype=torch.float32)
    n = torch.randn(Z, Y, X, C, generator=gen, dtype=torch.float32)
    f = f.to(device)
    w = _gauss_kernel(sigma, radius)
    for ax in range(3):
        f = _blur_axis(f, ax, w)
    f = f / f.reshape(-1, C).std(dim=0).clamp_min(1e-12)
    f = f + noise * n.to(device)
    return f.reshape(Z * Y * X, C).cpu()


@dataclass
class Workload:
    """Shapes, sizes and value recipe of one synthetic PACK3D workload."""
    name: str
    B: int
    H: int
    d: int
    Z: int
    Y: int
    X: int
    window: tuple
    block: tuple
    dtype: str = "bf16"          # "bf16" or "fp32"
    values: str = "normal"       # "normal" or "smooth"
    value_scale: float = 1.0     # multiplies the N(0,1) draws ("normal" only)
    rope_base: float = 100.0
    rope_mode: int = 0           # 0: axial RoPE on grid coordinates; 1: 1-D RoPE on the packed position
    n_tokens: int = 0            # 0: dense; > 0: that many tokens per item at distinct voxels
    packings: tuple = ("raster",)
    seed: int = 0
    backward: bool = False
    note: str = ""
    extra: dict = field(default_factory=dict)

    @property
    def V(self) -> int:
        return self.Z * self.Y * self.X

    @property
    def N(self) -> int:
        """Tokens per batch item."""
        return self.n_tokens or self.V

    @property
    def n_blocks(self) -> int:
        # the last block along an axis is cut at the volume's edge when the
        # extent does not divide the volume
        return (-(-self.Z // self.block[0])) * (-(-self.Y // self.block[1])) * (-(-self.X // self.block[2]))

    def replace(self, **kw) -> "Workload":
        d = dict(self.__dict__)
        d.update(kw)
        return Workload(**d)


def grid_tensors(wl: Workload, with_dout: bool = False, device="cpu"):
    """q, k, v (and dO) in grid raster order, fp32, shape [B, V, H, d] (one
    row per voxel; a partly occupied workload takes the rows of its tokens).

    Drawn from one generator seeded with ``wl.seed``, in the order q, k, v, dO."""
    g = torch.Generator().manual_seed(wl.seed)
    names = ["q", "k", "v"] + (["dout"] if with_dout else [])
    out = {}
    for nm in names:
        if wl.values == "normal" or nm == "dout":
            t = torch.randn(wl.B, wl.V, wl.H, wl.d, generator=g, dtype=torch.float32)
            if nm != "dout":
                t = t * wl.value_scale
        elif wl.values == "smooth":
            t = torch.empty(wl.B, wl.V, wl.H, wl.d, dtype=torch.float32)
            for b in range(wl.B):
                t[b] = smooth_field(g, wl.Z, wl.Y, wl.X, wl.H * wl.d, device=device).view(
                    wl.V, wl.H, wl.d)
        else:
            raise ValueError(wl.values)
        out[nm] = t
    return out


def torch_dtype(name: str) -> torch.dtype:
    return {"bf16": torch.bfloat16, "fp32": torch.float32}[name]


def make_inputs(wl: Workload, packing: str, with_dout: bool = False, grid=None, device="cpu"):
    """Packed inputs of a workload under one packing.

    Returns a dict with ``q, k, v`` (and ``dout``) as ``[B, N, H, d]`` tensors in
    packed order and the working dtype, ``coords`` as int16 ``[B, N, 3]`` and
    ``order`` as int64 ``[B, N]`` (voxel raster index of each packed slot).
    ``grid`` may pass tensors already drawn by :func:`grid_tensors`, so several
    packings share one field."""
    if grid is None:
        grid = grid_tensors(wl, with_dout=with_dout, device=device)
    dt = torch_dtype(wl.dtype)
    orders = np.stack([packing_order(packing, wl.Z, wl.Y, wl.X, wl.block, wl.seed, b)
                       for b in range(wl.B)])
    if wl.n_tokens:
        # a partly occupied volume: a seeded set of n_tokens voxels per item,
        # packed in the packing's order restricted to the set
        kept = []
        for b in range(wl.B):
            gen = torch.Generator().manual_seed(7_000_003 * (wl.seed + 1) + b)
            held = np.zeros(wl.V, bool)
            held[torch.randperm(wl.V, generator=gen)[:wl.n_tokens].numpy()] = True
            kept.append(orders[b][held[orders[b]]])
        orders = np.stack(kept)
    coords = np.stack([coords_of_order(orders[b], wl.Z, wl.Y, wl.X) for b in range(wl.B)])
    res = {"coords": torch.from_numpy(coords), "order": torch.from_numpy(orders)}
    idx = torch.from_numpy(orders)
    for nm, t in grid.items():
        r = t.to(dt)
        res[nm] = torch.stack([r[b].index_select(0, idx[b]) for b in range(wl.B)]).contiguous()
    return res


def unpack_rows(t: torch.Tensor, order: torch.Tensor) -> torch.Tensor:
    """Inverse of the packing along dim 1: packed [B, N, ...] -> raster [B, N, ...]
    (dense volumes)."""
    out = torch.empty_like(t)
    for b in range(t.shape[0]):
        out[b].index_copy_(0, order[b].to(t.device), t[b])
    return out
