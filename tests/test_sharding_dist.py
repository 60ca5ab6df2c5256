"""Host logic of the z-slab sharding on CPU: the slab plan, the halo exchange
(single and batched, as the forward and the backward run it) and the summary
all-reduce as two gloo ranks (torch.distributed, the same calls
NCCL runs on GPUs)."""
import json
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from local_global_attention_b200 import sharding as S  # noqa: E402


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("Z,bz,rz,world", [(32, 8, 3, 2), (32, 8, 3, 4), (30, 4, 2, 3), (9, 4, 1, 2)])
def test_plan_covers_the_volume(Z, bz, rz, world):
    slabs = S.plan_slabs(Z, bz, rz, world)
    owned = sorted((s.z_lo, s.z_hi) for s in slabs if s.owned)
    assert owned[0][0] == 0 and owned[-1][1] == Z
    for (a0, a1), (b0, b1) in zip(owned, owned[1:]):
        assert a1 == b0  # contiguous, disjoint
    for s in slabs:
        if s.owned:
            assert s.z_lo % bz == 0  # whole block rows
            assert s.h_lo == max(s.z_lo - rz, 0) and s.h_hi == min(s.z_hi + rz, Z)


def test_plan_rejects_slabs_thinner_than_the_halo():
    with pytest.raises(ValueError):
        S.plan_slabs(8, 1, 3, 4)


def voxel_value(c, ch):
    """A distinct value per (voxel, channel) of the synthetic field."""
    return (c[:, 0] * 1000 + c[:, 1] * 100 + c[:, 2]).double()[:, None] + ch[None, :] / 10.0


def worker(rank, world, port, out_dir, Z, Y, X, bz, rz):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import torch.distributed as dist
    dist.init_process_group("gloo")
    slab = S.plan_slabs(Z, bz, rz, world)[rank]
    # the rank's owned tokens, in a seeded random packing
    zz, yy, xx = torch.meshgrid(torch.arange(slab.z_lo, slab.z_hi), torch.arange(Y),
                                torch.arange(X), indexing="ij")
    coords = torch.stack([zz.flatten(), yy.flatten(), xx.flatten()], 1).to(torch.int16)
    coords = coords[torch.randperm(coords.shape[0], generator=torch.Generator().manual_seed(rank))]
    ch = torch.arange(3)
    vals = voxel_value(coords.long(), ch)
    held_c, held = S.exchange_halo(slab, coords, {"val": vals}, rz)
    gc = held_c.long() + torch.tensor([slab.h_lo, 0, 0])
    # summaries: this rank fills the blocks it owns, zeros elsewhere
    nb = -(-Z // bz)
    ks = torch.zeros(nb, 2)
    for B in range(slab.z_lo // bz, -(-slab.z_hi // bz)):
        ks[B] = torch.tensor([B + 1.0, -(B + 1.0)])
    vs = ks.clone() * 2
    S.allreduce_summaries(ks, vs)
    # batched exchange as the backward runs it: two items, and a per-head
    # row tensor laid out [B, H, n] (as lse is) exchanged through its transpose
    cb = torch.stack([coords, coords.flip(0)])
    lse = torch.stack([voxel_value(c.long(), ch).T for c in cb])  # [2, 3, n]
    hb_c, hb = S._held_batch(slab, cb, {"lse_t": lse.transpose(1, 2)}, rz, None)
    batch_ok = all(
        torch.equal(hb["lse_t"][b].T,
                    voxel_value(hb_c[b].long() + torch.tensor([slab.h_lo, 0, 0]), ch).T)
        for b in range(2))
    res = {
        "batch_ok": bool(batch_ok),
        "held": sorted(map(tuple, gc.tolist())),
        "values_ok": bool(torch.equal(held["val"], voxel_value(gc, ch))),
        "own_first": bool(torch.equal(held_c[:coords.shape[0]].long() + torch.tensor([slab.h_lo, 0, 0]),
                                      coords.long())),
        "ks": ks.tolist(), "vs": vs.tolist(), "slab": [slab.h_lo, slab.h_hi],
    }
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump(res, f)
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_halo_exchange_and_summary_allreduce(tmp_path, world):
    Z, Y, X, bz, rz = 12, 3, 4, 4, 2
    mp.spawn(worker, args=(world, free_port(), str(tmp_path), Z, Y, X, bz, rz), nprocs=world,
             join=True)
    nb = -(-Z // bz)
    for r in range(world):
        res = json.load(open(tmp_path / f"rank{r}.json"))
        h_lo, h_hi = res["slab"]
        want = sorted([z, y, x] for z in range(h_lo, h_hi) for y in range(Y) for x in range(X))
        assert res["held"] == want  # every voxel of the held planes, once
        assert res["values_ok"] and res["own_first"] and res["batch_ok"]
        assert res["ks"] == [[B + 1.0, -(B + 1.0)] for B in range(nb)]
        assert res["vs"] == [[2 * (B + 1.0), -2 * (B + 1.0)] for B in range(nb)]
