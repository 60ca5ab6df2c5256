"""Spatial sharding of the PACK3D forward along z, one process per GPU.

A volume too large for one GPU is cut into z-slabs.  Rank r owns a contiguous
run of block rows (planes [z_lo, z_hi), aligned to the block extent bz) and the
tokens in it.  The operator's two branches need different exchanges:

* the local window of a query in the slab reaches rz planes into each
  neighbour: the ranks swap their boundary planes (a halo exchange, the only
  token data that crosses the interconnect), so every rank holds planes
  [h_lo, h_hi) = its slab widened by rz and clipped to the volume;
* the block summaries are needed by every query: each rank computes the
  summaries of the blocks it owns (zeros for the others) and one all-reduce
  (sum) gives every rank all of them, exactly (each block's term comes from
  one rank, the others add zeros).

Each rank then calls the library on its slab with its halo planes, as a volume
of Z_total planes starting at plane z_origin = h_lo, owning the local planes
[z_lo - h_lo, z_hi - h_lo): RoPE angles and the block grid follow the global
planes, and outputs are written for the owned tokens only.  The window of an
owned query lies inside the held planes, and the axial RoPE logits depend only
on coordinate differences, so the owned outputs equal the unsharded ones.

The backward (sharded_backward) needs one more exchange.  The gradient of a
block summary sums over every query of the volume, so each rank computes the
partial sum over its owned queries (pack3d_backward_summary_grads) and an
all-reduce adds them; the rank then finishes dq, dk, dv of its owned tokens
(pack3d_backward_from_summary_grads).  The keys of a slab also receive
gradient from the queries in its halo planes, so the halo exchange carries q,
k, v, out, lse and dout.

Host-side orchestration only: the arithmetic runs in the library's kernels; this
module selects, exchanges and reduces tensors with torch.distributed (NCCL on
GPUs, gloo for the CPU tests).  Each slab must be at least rz planes thick, so
that a rank's halo comes from its two neighbours only.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Slab:
    rank: int
    world: int
    z_lo: int  # owned global planes [z_lo, z_hi)
    z_hi: int
    h_lo: int  # held global planes [h_lo, h_hi): owned + halo
    h_hi: int

    @property
    def owned(self) -> bool:
        return self.z_hi > self.z_lo


def plan_slabs(Z: int, bz: int, rz: int, world: int) -> list[Slab]:
    """Block rows split as evenly as possible over the ranks (rank r: rows
    [r nbz / world, (r + 1) nbz / world)), each slab widened by rz halo planes
    and clipped to the volume."""
    nbz = -(-Z // bz)
    slabs = []
    for r in range(world):
        b0, b1 = r * nbz // world, (r + 1) * nbz // world
        z_lo, z_hi = min(b0 * bz, Z), min(b1 * bz, Z)
        if z_hi > z_lo and z_hi - z_lo < rz and world > 1:
            raise ValueError(f"slab of rank {r} ({z_hi - z_lo} planes) thinner than the "
                             f"window radius {rz}: use fewer ranks")
        slabs.append(Slab(r, world, z_lo, z_hi, max(z_lo - rz, 0) if z_hi > z_lo else z_lo,
                          min(z_hi + rz, Z) if z_hi > z_lo else z_hi))
    return slabs


def slab_shape(shape, slab: Slab):
    """The shape of one rank's library call: its held planes as the volume,
    Z_total / z_origin / own_lo / own_hi describing where they sit."""
    fields = dict(Z=slab.h_hi - slab.h_lo, Z_total=shape.Z, z_origin=slab.h_lo,
                  own_lo=slab.z_lo - slab.h_lo, own_hi=slab.z_hi - slab.h_lo)
    if dataclasses.is_dataclass(shape):
        extra = {k: v for k, v in fields.items() if k in {f.name for f in dataclasses.fields(shape)}}
        out = dataclasses.replace(shape, **extra)
        for k, v in fields.items():
            if k not in extra:
                object.__setattr__(out, k, v)
        return out
    out = type("SlabShape", (), {})()
    out.__dict__.update(shape.__dict__)
    out.__dict__.update(fields)
    return out


def select_planes(coords: torch.Tensor, tensors: dict, z_lo: int, z_hi: int):
    """Rows (tokens) of one batch item whose z lies in [z_lo, z_hi), in their
    packed order: (coords [n, 3], {name: [n, ...]})."""
    keep = (coords[:, 0] >= z_lo) & (coords[:, 0] < z_hi)
    idx = keep.nonzero().squeeze(1)
    return coords.index_select(0, idx), {k: t.index_select(0, idx) for k, t in tensors.items()}


def held_from_global(slab: Slab, coords: torch.Tensor, tensors: dict):
    """The tokens a rank holds after the halo exchange, taken directly from one
    batch item's global packed arrays (for running the ranks one after another
    on one device): owned tokens first, then the planes below, then above, with
    coordinates made local (z - h_lo)."""
    parts = [select_planes(coords, tensors, lo, hi)
             for lo, hi in ((slab.z_lo, slab.z_hi), (slab.h_lo, slab.z_lo),
                            (slab.z_hi, slab.h_hi))]
    c = torch.cat([p[0] for p in parts])
    c = c - torch.tensor([slab.h_lo, 0, 0], dtype=c.dtype, device=c.device)
    return c, {k: torch.cat([p[1][k] for p in parts]) for k in tensors}


def _swap(send: torch.Tensor, peer: int, recv_like_rows: int, group):
    import torch.distributed as dist
    recv = torch.empty((recv_like_rows,) + tuple(send.shape[1:]), dtype=send.dtype,
                       device=send.device)
    ops = [dist.P2POp(dist.isend, send.contiguous(), peer, group),
           dist.P2POp(dist.irecv, recv, peer, group)]
    for req in dist.batch_isend_irecv(ops):
        req.wait()
    return recv


def exchange_halo(slab: Slab, coords: torch.Tensor, tensors: dict, rz: int, group=None):
    """Halo exchange for one batch item.  `coords` [n_own, 3] (global z) and
    `tensors` {name: [n_own, ...]} hold the rank's owned tokens in its packed
    order.  Returns the held tokens - the owned ones first, then those received
    from the rank below, then from the rank above - with coordinates made local
    (z - h_lo)."""
    import torch.distributed as dist
    names = sorted(tensors)
    parts_c, parts_t = [coords], {k: [tensors[k]] for k in names}
    for peer, lo, hi in ((slab.rank - 1, slab.z_lo, slab.z_lo + rz),
                         (slab.rank + 1, slab.z_hi - rz, slab.z_hi)):
        if peer < 0 or peer >= slab.world or not slab.owned:
            continue
        c_out, t_out = select_planes(coords, tensors, lo, hi)
        n_out = torch.tensor([c_out.shape[0]], dtype=torch.int64, device=coords.device)
        n_in = _swap(n_out, peer, 1, group)
        n = int(n_in.item())
        parts_c.append(_swap(c_out, peer, n, group))
        for k in names:
            parts_t[k].append(_swap(t_out[k], peer, n, group))
    held_c = torch.cat(parts_c)
    held_c = held_c - torch.tensor([slab.h_lo, 0, 0], dtype=held_c.dtype, device=held_c.device)
    return held_c, {k: torch.cat(parts_t[k]) for k in names}


def allreduce_summaries(ksum: torch.Tensor, vsum: torch.Tensor, group=None):
    """Every rank computed the summaries of its own blocks and zeros for the
    others; the sum over ranks is every block's summary."""
    import torch.distributed as dist
    dist.all_reduce(ksum, op=dist.ReduceOp.SUM, group=group)
    dist.all_reduce(vsum, op=dist.ReduceOp.SUM, group=group)
    return ksum, vsum


def sharded_forward(shape, slab: Slab, coords: torch.Tensor, q, k, v, group=None):
    """The PACK3D forward of this rank's owned tokens.  coords [B, n_own, 3]
    (global z), q, k, v [B, n_own, H, d] on this rank's GPU.  Returns out
    [B, n_own, H, d] and lse [B, H, n_own] for the owned tokens, in their
    packed order."""
    from . import pack3d as P
    rz = (shape.window[0] - 1) // 2
    hc, held = _held_batch(slab, coords, {"q": q, "k": k, "v": v}, rz, group)
    hq, hk, hv = held["q"], held["k"], held["v"]
    params = P.make_params(slab_shape(shape, slab))
    idx = P.pack3d_build_index(params, hc)
    ksum, vsum = P.pack3d_block_summaries(params, idx, hk, hv)
    allreduce_summaries(ksum, vsum, group)
    out, lse = P.pack3d_forward(params, idx, hq, hk, hv, ksum, vsum)
    n_own = coords.shape[1]
    return out[:, :n_own], lse[:, :, :n_own]


def _held_batch(slab: Slab, coords: torch.Tensor, tensors: dict, rz: int, group):
    """Halo exchange of every batch item; the held coordinates [B, n_held, 3]
    and tensors {name: [B, n_held, ...]}."""
    held_c, held = [], {n: [] for n in tensors}
    for b in range(coords.shape[0]):
        c, t = exchange_halo(slab, coords[b], {n: x[b] for n, x in tensors.items()}, rz, group)
        held_c.append(c)
        for n in held:
            held[n].append(t[n])
    return (torch.stack(held_c).contiguous(),
            {n: torch.stack(x).contiguous() for n, x in held.items()})


def sharded_backward(shape, slab: Slab, coords: torch.Tensor, q, k, v, out, lse, dout,
                     group=None):
    """Gradients of sum(dout * out) with respect to this rank's owned q, k, v.
    coords [B, n_own, 3] (global z); q, k, v, out, dout [B, n_own, H, d] and lse
    [B, H, n_own] as sharded_forward returned them.  Returns dq, dk, dv
    [B, n_own, H, d].  The summaries of the whole volume are computed again
    (one pass over the held keys and values and an all-reduce)."""
    from . import pack3d as P
    rz = (shape.window[0] - 1) // 2
    hc, held = _held_batch(slab, coords, {"q": q, "k": k, "v": v, "out": out, "dout": dout,
                                          "lse": lse.transpose(1, 2)}, rz, group)
    params = P.make_params(slab_shape(shape, slab))
    idx = P.pack3d_build_index(params, hc)
    ksum, vsum = P.pack3d_block_summaries(params, idx, held["k"], held["v"])
    allreduce_summaries(ksum, vsum, group)
    hlse = held["lse"].transpose(1, 2).contiguous()
    dks, dvs, ws = P.pack3d_backward_summary_grads(params, idx, held["q"], held["k"], held["v"],
                                                   held["out"], hlse, held["dout"], ksum, vsum)
    # the gradient of a summary sums over the queries of every rank
    allreduce_summaries(dks, dvs, group)
    dq, dk, dv = (torch.zeros_like(held[n]) for n in ("q", "k", "v"))
    P.pack3d_backward_from_summary_grads(params, idx, dks, dvs, ws, dq, dk, dv)
    n_own = coords.shape[1]
    return dq[:, :n_own], dk[:, :n_own], dv[:, :n_own]
