"""PACK3D forward throughput on B200.

One step is the whole forward hot path over one batch of synthetic input at
the 65,536-token shape (volume 32 x 32 x 64, batch 2, 8 heads, head_dim 96,
window 7^3, blocks 8^3, bf16, random packing): index build from the batch's
coordinates, block summaries, and the PACK3D forward with LSE.  ``value`` is
tokens/s (B * N per step) with inputs resident in HBM; ``e2e`` measures the
same through the C ABI from pinned host buffers, copies included.  The
window-only mode is timed alongside.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

With N > 1 (one process per GPU under torchrun) every rank runs its own batch
(weak scaling; the operator has no cross-rank data path) and the time is the
maximum over ranks.  ``--impl reference`` times the CPU oracle on the host
cores on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "PACK3D fwd tokens/s at 65k tokens bf16; % of BF16 tensor peak and HBM roofline"
UNIT = "tokens/s"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
PROFILE_SUMMARY = os.path.join(ROOT, "profiles", "forward_tc_vol_32x32x64.md")
# the attention kernel's source and the headers it includes
TC_SOURCES = [os.path.join(ROOT, "local_global_attention_b200", "csrc", f)
              for f in ("attn_tc.cu", "tc_attn_common.cuh", "tc_primitives.cuh",
                        "pack3d_internal.cuh")]


def peaks():
    try:
        with open(PEAKS_FILE) as f:
            return json.load(f), "measured"
    except (OSError, ValueError):
        return FALLBACK_PEAKS, "fallback"


def workload(name):
    from local_global_attention_b200 import configs as C
    return C.BY_NAME[name]


def algorithmic_work(wl):
    """Useful FLOPs of one forward (local and summary terms, 4 d per term) and
    the minimum HBM bytes (q, k, v read, out written, lse written, plus the
    summary builder's read of k and v)."""
    def axis_hist(ext, r):
        # number of window positions per coordinate along one axis
        c = np.arange(ext)
        return np.minimum(c + r, ext - 1) - np.maximum(c - r, 0) + 1
    rz, ry, rx = ((w - 1) // 2 for w in wl.window)
    wz, wy, wx = axis_hist(wl.Z, rz), axis_hist(wl.Y, ry), axis_hist(wl.X, rx)
    local_terms = wz.sum() * wy.sum() * wx.sum()  # sum over queries of |W(i)|

    def blocks_met(ext, r, bsz):
        c = np.arange(ext)
        lo = np.maximum(c - r, 0) // bsz
        hi = np.minimum(c + r, ext - 1) // bsz
        return hi - lo + 1
    nb = wl.n_blocks
    met = (blocks_met(wl.Z, rz, wl.block[0])[:, None, None] *
           blocks_met(wl.Y, ry, wl.block[1])[None, :, None] *
           blocks_met(wl.X, rx, wl.block[2])[None, None, :])
    sum_terms = (nb - met).sum()
    per_bh_local = 4.0 * wl.d * local_terms
    per_bh_sum = 4.0 * wl.d * sum_terms
    BH = wl.B * wl.H
    esz = 2
    rows = wl.B * wl.N * wl.H * wl.d
    hbm = rows * esz * 4 + wl.B * wl.H * wl.N * 4 + rows * esz * 2
    # backward: S recomputed (2d), dP = dO.v (2d), dq, dk and dv updates (2d
    # each): 10 d FLOPs per local and per summary term
    per_bh_bwd = 10.0 * wl.d * (local_terms + sum_terms)
    return {"local_flop": BH * per_bh_local, "summary_flop": BH * per_bh_sum,
            "bwd_flop": BH * per_bh_bwd,
            "flop": BH * (per_bh_local + per_bh_sum), "hbm_bytes": hbm,
            "fwd_bytes": rows * esz * 4 + wl.B * wl.H * wl.N * 4}


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        # wait (up to 3 s) for the first sample, so that sampling already runs
        # when the timed region starts
        self.first = None
        if self.proc is not None:
            import select
            r, _, _ = select.select([self.proc.stdout], [], [], 3.0)
            if r:
                self.first = self.proc.stdout.readline()
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            # the sample taken before the timed region is left out
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup(n_gpus):
    """One process per GPU (torchrun env).  NCCL on GPUs; gloo where there is
    none (the CPU tests of this host logic)."""
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        timeout = datetime.timedelta(seconds=120)
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=timeout,
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group("gloo", timeout=timeout)
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    """Maximum of a per-rank time over all ranks (every rank gets it)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_workload(wl, rank):
    """Weak scaling: every rank runs its own batch of the same shape (seed
    offset by the rank), so there is no data-path collective."""
    return wl.replace(seed=wl.seed + 1000 * rank)


def whole_job_rate(tokens_per_rank, world, ms):
    """Tokens/s of the whole job: all ranks' tokens over the slowest rank's time."""
    return tokens_per_rank * world / (ms * 1e-3)


def run_config(wl, packing, world):
    """The workload a line is quoted on; both arms print the same one."""
    B, N, H, d = wl.B, wl.N, wl.H, wl.d
    return {
        "workload": f"{wl.name}: {N} tokens x batch {B}, {H} heads, head_dim {d}, "
                    f"window {'x'.join(map(str, wl.window))}, blocks "
                    f"{'x'.join(map(str, wl.block))} ({wl.n_blocks} summaries), {packing} packing",
        "step": "index build + block summaries fused with key/value staging + attention (out, lse)",
        "global_batch": B * world,
        "seq_len": N,
        "parallelism": f"replicas x{world} (independent batches, no collective)",
        "l2": "inputs larger than L2: q, k, v = "
              f"{3 * B * N * H * d * 2 / 1e6:.0f} MB per step, no flush",
    }


class Runner:
    """One workload on this GPU: its inputs in HBM, index, workspace and the
    calls of one step, made through the C ABI (ctypes) on one stream."""

    def __init__(self, wl, inp, packed_rope=False):
        import ctypes

        import torch

        from local_global_attention_b200 import pack3d as P
        self.torch, self.ctypes, self.P = torch, ctypes, P
        self.wl = wl
        self.dev = {k: v.cuda() for k, v in inp.items() if k != "order"}
        self.params = P.make_params(wl)
        if packed_rope:
            self.params.rope_mode = P.ROPE_PACKED
        self.idx = P.IndexBuffers(self.params)
        B, N, H, d = wl.B, wl.N, wl.H, wl.d
        self.ksum = torch.empty(B, H, wl.n_blocks, d, dtype=torch.float32, device="cuda")
        self.vsum = torch.empty_like(self.ksum)
        self.out = torch.empty_like(self.dev["q"])
        self.lse = torch.empty(B, H, N, dtype=torch.float32, device="cuda")
        self.ws_bytes = P.pack3d_forward_workspace_bytes(self.params)
        self.ws = torch.empty(max(self.ws_bytes, 1), dtype=torch.uint8, device="cuda")
        self.stream = torch.cuda.current_stream()
        self.lib = P.load()
        self.sp = ctypes.c_void_p(self.stream.cuda_stream)
        self.pp, self.ip = ctypes.byref(self.params), ctypes.byref(self.idx.struct)
        self.phase_events = []

    def ptr(self, t):
        return self.ctypes.c_void_p(t.data_ptr())

    def event(self):
        e = self.torch.cuda.Event(enable_timing=True)
        e.record(self.stream)
        return e

    def step(self, window=False, record=False, bufs=None, res=None):
        """Index build; block summaries computed in the pass that stages the
        rotated keys and the values in grid order (pack3d_stage_kv); the
        attention (pack3d_forward_staged).  With record, CUDA events between
        the three phases."""
        c_size = self.ctypes.c_size_t
        d_ = self.dev if bufs is None else bufs
        o_, l_ = (self.out, self.lse) if res is None else res
        ev = [self.event()] if record else None
        rc = self.lib.pack3d_build_index(self.pp, self.ptr(d_["coords"]), self.ip, self.sp)
        if record:
            ev.append(self.event())
        rc |= self.lib.pack3d_stage_kv(self.pp, self.ip, self.ptr(d_["k"]), self.ptr(d_["v"]),
                                       None if window else self.ptr(self.ksum),
                                       None if window else self.ptr(self.vsum),
                                       self.ptr(self.ws), c_size(self.ws_bytes), self.sp)
        if record:
            ev.append(self.event())
        rc |= self.lib.pack3d_forward_staged(self.pp, self.ip, self.ptr(d_["q"]),
                                             self.ptr(self.ws), c_size(self.ws_bytes),
                                             0 if window else 1, self.ptr(o_), self.ptr(l_),
                                             self.sp)
        if record:
            ev.append(self.event())
            self.phase_events.append(ev)
        if rc:
            raise RuntimeError(f"pack3d call failed: {rc}")

    def phase_ms(self):
        """Mean ms of (index build, staging + summaries, attention) over the
        recorded steps."""
        ev = self.phase_events
        return [statistics.mean(e[i].elapsed_time(e[i + 1]) for e in ev) for i in range(3)]

    def timed(self, steps, warmup, world, window=False, record=False):
        """ms per step over `steps` timed steps (barrier + synchronize on both
        sides, CUDA events on the launching stream, max over ranks) and the
        number of library kernels launched in the timed region."""
        torch = self.torch
        self.phase_events = []
        for _ in range(warmup):
            self.step(window=window)
        torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        n0 = self.P.pack3d_kernel_launches()
        t0 = self.event()
        for _ in range(steps):
            self.step(window=window, record=record)
        t1 = self.event()
        n1 = self.P.pack3d_kernel_launches()
        torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        st = self.P.pack3d_index_check(self.idx)
        if st != self.P.OK:
            raise RuntimeError(f"index status {self.P.strerror(st)}")
        return max_over_ranks(t0.elapsed_time(t1) / steps, world), n1 - n0

    def time_calls(self, fn, calls, warmup=3):
        """Mean ms of fn() over `calls` back-to-back calls (CUDA events)."""
        for _ in range(warmup):
            fn()
        self.torch.cuda.synchronize()
        t0 = self.event()
        for _ in range(calls):
            fn()
        t1 = self.event()
        self.torch.cuda.synchronize()
        return t0.elapsed_time(t1) / calls

    def block_summaries(self):
        rc = self.lib.pack3d_block_summaries(self.pp, self.ip, self.ptr(self.dev["k"]),
                                             self.ptr(self.dev["v"]), self.ptr(self.ksum),
                                             self.ptr(self.vsum), self.sp)
        if rc:
            raise RuntimeError(f"pack3d_block_summaries failed: {rc}")


def kernel_sources_sha256():
    """sha256 over the attention kernel's source files, in order, with line
    comments and blank lines dropped (a comment edit leaves the kernel as it
    was profiled)."""
    h = hashlib.sha256()
    for f in TC_SOURCES:
        for line in open(f, encoding="utf-8"):
            code = line.split("//", 1)[0].rstrip()
            if code:
                h.update(code.encode() + b"\n")
    return h.hexdigest()


def profile_value(key):
    """A figure from the committed ncu summary of the attention kernel, if it
    was taken on the current kernel source; else None."""
    try:
        text = open(PROFILE_SUMMARY).read()
    except OSError:
        return None
    m_sha = re.search(r"source_sha256:\s*([0-9a-f]{64})", text)
    m = re.search(key + r":\s*([0-9.eE+]+)", text)
    if not (m_sha and m):
        return None
    sha = kernel_sources_sha256()
    return float(m.group(1)) if sha == m_sha.group(1) else None


def backward_runner(r, wl):
    """A closure that runs pack3d_backward once through the C ABI on the
    runner's inputs and the forward's out and lse (computed here), with
    dO ~ N(0, 1)."""
    import ctypes

    import torch

    from local_global_attention_b200 import pack3d as P
    B, N, H, d = wl.B, wl.N, wl.H, wl.d
    g_do = torch.Generator().manual_seed(wl.seed + 7)
    dout = torch.randn(B, N, H, d, generator=g_do).to(r.dev["q"].dtype).cuda()
    dq, dk, dv = (torch.empty_like(r.dev["q"]) for _ in range(3))
    nbytes = P.pack3d_backward_workspace_bytes(r.params)
    ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device="cuda")
    r.step()  # the forward the backward reads
    ptr = r.ptr
    keep = (dout, dq, dk, dv, ws)

    def backward():
        _ = keep
        rc = r.lib.pack3d_backward(r.pp, r.ip, ptr(r.dev["q"]), ptr(r.dev["k"]), ptr(r.dev["v"]),
                                   ptr(r.out), ptr(r.lse), ptr(dout), ptr(dq), ptr(dk), ptr(dv),
                                   ptr(ws), ctypes.c_size_t(nbytes), r.sp)
        if rc:
            raise RuntimeError(f"pack3d_backward failed: {rc}")
    return backward


def micro1m_line(args, pk):
    """The 1,048,576-token microscopy-shaped workload (smooth field, block
    packing): PACK3D step and window-only step, with the attention kernel's
    useful FLOP rate.  Its summary term (1,024 blocks) dwarfs the local one."""
    import torch

    from local_global_attention_b200 import configs as C
    from local_global_attention_b200 import inputs as I
    wl = C.MICRO1M
    t_gen = time.perf_counter()
    inp = I.make_inputs(wl, "block", grid=I.grid_tensors(wl, device="cuda"))
    t_gen = time.perf_counter() - t_gen
    r = Runner(wl, inp)
    steps = max(3, min(args.steps, 20))
    ms, launches = r.timed(steps, args.warmup, 1, record=True)
    idx_ms, stage_ms, attn_ms = r.phase_ms()
    wms, _ = r.timed(steps, args.warmup, 1, window=True, record=True)
    w_attn = r.phase_ms()[2]
    work = algorithmic_work(wl)
    tf = work["flop"] / (attn_ms * 1e-3) / 1e12
    res = {
        "workload": f"{wl.name}: {wl.N} tokens x batch {wl.B}, {wl.H} heads, head_dim {wl.d}, "
                    f"window {'x'.join(map(str, wl.window))}, blocks "
                    f"{'x'.join(map(str, wl.block))} ({wl.n_blocks} summaries), block packing, "
                    "smooth random field",
        "ms_per_step": ms, "value": wl.B * wl.N / (ms * 1e-3), "unit": UNIT, "steps": steps,
        "phases_ms": {"index": idx_ms, "stage_and_summaries": stage_ms, "attention": attn_ms},
        "attention_tflops_useful": tf, "attention_frac_of_burst_peak": tf / pk["bf16_tflops"],
        "local_flop": work["local_flop"], "summary_flop": work["summary_flop"],
        "window_only": {"ms_per_step": wms, "attention_ms": w_attn,
                        "pack3d_over_window": ms / wms},
        "gpu_launches_per_step": launches / steps,
        "input_generation_s": t_gen,
    }
    del r, inp
    torch.cuda.empty_cache()
    return res


def cuda_core_line(args, dtype="fp32", d=96):
    """A configuration the CUDA-core kernels run, at the 65k shape: the fp32
    mode (1e-4 bound), or bf16 at a head dim other than 96.  Index build,
    block summaries and forward through the C ABI, a few timed steps, with the
    useful FLOP rate against the fp32 FMA peak (148 SMs x 128 lanes x 2 FLOP
    at the clock sampled here)."""
    import torch

    from local_global_attention_b200 import configs as C
    from local_global_attention_b200 import inputs as I
    from local_global_attention_b200 import pack3d as P
    name = f"vol_32x32x64_{dtype}" + ("" if d == 96 else f"_d{d}")
    wl = C.VOL65K.replace(dtype=dtype, d=d, value_scale=1.0 / math.sqrt(d), name=name)
    inp = I.make_inputs(wl, "random")
    dev = {k: v.cuda() for k, v in inp.items() if k != "order"}
    params = P.make_params(wl)
    idx = P.IndexBuffers(params)
    ksum = torch.empty(wl.B, wl.H, wl.n_blocks, wl.d, device="cuda")
    vsum = torch.empty_like(ksum)
    out = torch.empty_like(dev["q"])
    lse = torch.empty(wl.B, wl.H, wl.N, device="cuda")

    def step():
        P.pack3d_build_index(params, dev["coords"], idx)
        P.pack3d_block_summaries(params, idx, dev["k"], dev["v"], ksum, vsum)
        P.pack3d_forward(params, idx, dev["q"], dev["k"], dev["v"], ksum, vsum, out=out, lse=lse)

    steps = 3
    for _ in range(3):
        step()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    assert P.pack3d_index_check(idx) == P.OK
    ms = e0.elapsed_time(e1) / steps
    work = algorithmic_work(wl)
    tf = work["flop"] / (ms * 1e-3) / 1e12
    res = {"workload": f"vol_32x32x64 in {dtype}, head_dim {d} (same shape and seed layout, "
                       "CUDA-core kernels)",
           "ms_per_step": ms, "value": wl.B * wl.N / (ms * 1e-3), "unit": UNIT, "steps": steps,
           "tflops_useful_whole_step": tf}
    del dev, inp, out, lse, ksum, vsum, idx
    torch.cuda.empty_cache()
    return res


def run_ours(args):
    import ctypes

    import torch

    from local_global_attention_b200 import inputs as I
    from local_global_attention_b200 import pack3d as P

    world, rank, local = dist_setup(args.gpus)
    wl = workload(args.workload)
    wl_r = rank_workload(wl, rank)
    inp = I.make_inputs(wl_r, args.packing)
    r = Runner(wl_r, inp)
    B, N, H, d = wl.B, wl.N, wl.H, wl.d

    with ClockSampler(local) as clk:
        ms, launches = r.timed(args.steps, args.warmup, world, record=True)
    idx_ms, stage_ms, fwd_ms = r.phase_ms()
    pk, pk_src = peaks()
    work = algorithmic_work(wl)
    tokens = B * N * world
    if args.only == "forward":
        # the forward step alone, then three pack3d_block_summaries calls (a
        # short run for profilers); one line, no extras
        for _ in range(3):
            r.block_summaries()
        torch.cuda.synchronize()
        if rank == 0:
            print(json.dumps({"metric": METRIC, "value": whole_job_rate(B * N, world, ms),
                              "unit": UNIT, "n_gpus": world, "steps": args.steps,
                              "ms_per_step": ms, "only": "forward"}), flush=True)
        return

    if args.only == "backward":
        # the forward once, then the backward calls alone (a short run for
        # profilers); one line, no extras
        bwd = backward_runner(r, wl_r)
        bwd_ms = r.time_calls(bwd, max(1, args.steps), warmup=args.warmup)
        if rank == 0:
            print(json.dumps({"metric": "backward ms per call", "value": bwd_ms, "unit": "ms",
                              "only": "backward", "steps": args.steps}), flush=True)
        return

    window_ms, _ = r.timed(args.steps, args.warmup, world, window=True)
    # the packed-sequence comparison mode (1-D RoPE on the packed index): its own
    # params and index (the rotation table differs), the same step
    r_pk = Runner(wl_r, inp, packed_rope=True)
    packed_ms, _ = r_pk.timed(args.steps, args.warmup, world)
    del r_pk
    # pack3d_block_summaries alone (HBM-bound: k and v read once)
    sum_ms = r.time_calls(r.block_summaries, 20)

    # the backward (dq, dk, dv from the forward's out and lse) at the same shape,
    # with dO ~ N(0, 1)
    backward = backward_runner(r, wl_r)
    bw_steps = max(3, min(args.steps, 20))
    bwd_ms = max_over_ranks(r.time_calls(backward, bw_steps), world)
    if P.pack3d_index_check(r.idx) != P.OK:
        raise RuntimeError("index status after the backward")

    # End to end through the C ABI: every step copies its inputs from pinned
    # host memory and reads its outputs back.  Two device buffer sets and two
    # copy streams let step i's upload, step i-1's compute and step i-2's
    # download overlap (PCIe is full duplex); every byte of every step is still
    # copied inside the timed region.
    stream = r.stream
    names = ("coords", "q", "k", "v")
    host = {k: inp[k].pin_memory() for k in names}
    sets = [r.dev, {k: torch.empty_like(r.dev[k]) for k in names}]
    results = [(r.out, r.lse), (torch.empty_like(r.out), torch.empty_like(r.lse))]
    host_res = [(torch.empty(r.out.shape, dtype=r.out.dtype).pin_memory(),
                 torch.empty(r.lse.shape, dtype=r.lse.dtype).pin_memory()) for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    computed = [None, None]  # compute of the last step on buffer set b done
    drained = [None, None]   # download of the last step on buffer set b done

    def e2e_step(i):
        b = i % 2
        with torch.cuda.stream(s_in):
            if computed[b] is not None:
                s_in.wait_event(computed[b])
            for k_ in names:
                sets[b][k_].copy_(host[k_], non_blocking=True)
            ready = torch.cuda.Event()
            ready.record(s_in)
        stream.wait_event(ready)
        if drained[b] is not None:
            stream.wait_event(drained[b])
        r.step(bufs=sets[b], res=results[b])
        ev = torch.cuda.Event()
        ev.record(stream)
        computed[b] = ev
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev)
            host_res[b][0].copy_(results[b][0], non_blocking=True)
            host_res[b][1].copy_(results[b][1], non_blocking=True)
            dr = torch.cuda.Event()
            dr.record(s_out)
            drained[b] = dr

    for i in range(args.warmup):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_in.wait_event(e0)
    for i in range(args.steps):
        e2e_step(i)
    for ev in drained:
        stream.wait_event(ev)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world)
    h2d = sum(host[k_].numel() * host[k_].element_size() for k_ in host)
    d2h = sum(t.numel() * t.element_size() for t in host_res[0])
    del sets, results, host_res, host

    micro = None
    if args.micro1m and world == 1:
        micro = micro1m_line(args, pk)
    fp32 = cuda_core_line(args) if args.micro1m and world == 1 else None
    d48 = cuda_core_line(args, "bf16", 48) if args.micro1m and world == 1 else None

    if rank != 0:
        barrier(world)
        return
    achieved = work["flop"] / (fwd_ms * 1e-3) / 1e12
    local_achieved = work["local_flop"] / (fwd_ms * 1e-3) / 1e12
    peak_tf = pk["bf16_tflops"]
    stage_bytes = work["fwd_bytes"] - wl.B * wl.H * wl.N * 4  # k, v read + grid copies written
    line = {
        "metric": METRIC,
        "value": whole_job_rate(B * N, world, ms),
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1)/sqrt(96) q, k, v; random packing)",
        "config": run_config(wl, args.packing, world),
        "gpu_launches": launches,
        "gpu_launches_note": "library kernel launches issued inside the timed region "
                             "(pack3d_kernel_launches before and after)",
        "roofline": {
            "bound": "tensor",
            "kernel": "k_forward_tc (local window + summaries, tcgen05)",
            "achieved": achieved,
            "peak": peak_tf,
            "unit": "TFLOP/s",
            "frac": achieved / peak_tf,
            "peak_source": f"{pk_src} bf16_tflops (burst: a ~1 ms kernel timed alone)",
            "local_frac": local_achieved / peak_tf,
            "local_note": "local-window FLOPs only (the summary terms left out)",
            "tensor_pipe_active_pct_ncu": profile_value("tensor_pipe_active_pct"),
            "traffic": profile_value("dram_bytes_per_launch"),
            "algorithmic_flop_per_launch": work["flop"],
            "forward_ms": fwd_ms,
            "forward_hbm_frac": (work["fwd_bytes"] / (fwd_ms * 1e-3) / 1e9) / pk["hbm_gbs"],
        },
        "memory_bound": {
            "unit": "GB/s", "peak": pk["hbm_gbs"], "peak_source": f"{pk_src} hbm_gbs (copy)",
            "stage_and_summaries": {
                "kernel": "k_summaries_bulk<1>", "ms": stage_ms,
                "algorithmic_bytes": stage_bytes,
                "achieved": stage_bytes / (stage_ms * 1e-3) / 1e9,
                "frac": stage_bytes / (stage_ms * 1e-3) / 1e9 / pk["hbm_gbs"]},
            "block_summaries": {
                "kernel": "k_summaries_bulk<0> (pack3d_block_summaries)", "ms": sum_ms,
                "algorithmic_bytes": stage_bytes / 2,
                "achieved": stage_bytes / 2 / (sum_ms * 1e-3) / 1e9,
                "frac": stage_bytes / 2 / (sum_ms * 1e-3) / 1e9 / pk["hbm_gbs"]},
            "index_build_ms": idx_ms,
        },
        "backward": {
            "ms_per_call": bwd_ms,
            "calls": bw_steps,
            "kernels": "attn_bwd_tc.cu (tcgen05: staging, summary gradients, dq, dk/dv)",
            "roofline": {"bound": "tensor", "unit": "TFLOP/s",
                         "achieved": work["bwd_flop"] / (bwd_ms * 1e-3) / 1e12,
                         "peak": peak_tf,
                         "frac": work["bwd_flop"] / (bwd_ms * 1e-3) / 1e12 / peak_tf,
                         "peak_source": f"{pk_src} bf16_tflops (burst)",
                         "algorithmic_flop_per_call": work["bwd_flop"],
                         "note": "whole call (staging included) against the useful FLOPs: "
                                 "10 d per window key and per unmasked summary of each query"},
        },
        "window_only": {"ms_per_step": window_ms, "value": tokens / (window_ms * 1e-3),
                        "pack3d_over_window": ms / window_ms},
        "packed_rope_mode": {"ms_per_step": packed_ms, "value": tokens / (packed_ms * 1e-3),
                             "note": "comparison mode: 1-D RoPE on the packed index, same step"},
        "e2e": {"value": tokens / (e2e_ms * 1e-3), "unit": UNIT, "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "clocks": clk.summary(),
    }
    if micro is not None:
        line["micro1m"] = micro
    if fp32 is not None:
        clock_mhz = (line.get("clocks") or {}).get("sm_mhz") or 1965.0
        fma_peak = 148 * 128 * 2 * clock_mhz / 1e6  # TFLOP/s
        fp32["fp32_fma_peak_tflops"] = fma_peak
        fp32["frac_of_fma_peak"] = fp32["tflops_useful_whole_step"] / fma_peak
        line["fp32_mode"] = fp32
        d48["fp32_fma_peak_tflops"] = fma_peak
        d48["frac_of_fma_peak"] = d48["tflops_useful_whole_step"] / fma_peak
        line["bf16_head_dim_48"] = d48
    if not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_baseline(wl, inp, args.cpu_sample)
    barrier(world)
    print(json.dumps(line), flush=True)


def cpu_baseline(wl, inp, n_tokens, seed=0):
    """The CPU oracle on a bounded sample: n_tokens query positions (all heads
    of each), timed on the host cores; tokens/s of the same workload."""
    import oracle
    oracle.build()
    rng = np.random.default_rng(seed)
    N = wl.N
    bs = rng.integers(0, wl.B, n_tokens)
    iis = rng.integers(0, N, n_tokens)
    b = np.repeat(bs, wl.H)
    i = np.repeat(iis, wl.H)
    h = np.tile(np.arange(wl.H), n_tokens)
    sel = oracle.flat_index(wl, b, h, i)
    t0 = time.perf_counter()
    ks, vs = oracle.block_summaries(wl, inp["coords"], inp["k"], inp["v"])
    oracle.forward(wl, inp["coords"], inp["q"], inp["k"], inp["v"], sel=sel, summaries=(ks, vs))
    dt = time.perf_counter() - t0
    return {"value": n_tokens / dt, "unit": UNIT, "cores": oracle.max_threads(), "kind": "oracle",
            "sample": f"{n_tokens} random query tokens x {wl.H} heads of {wl.name} "
                      f"(block summaries of the whole batch included), {dt:.1f} s"}


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    from local_global_attention_b200 import inputs as I
    wl = workload(args.workload)
    inp = I.make_inputs(wl, args.packing)
    oracle.build()
    ks, vs = oracle.block_summaries(wl, inp["coords"], inp["k"], inp["v"])
    rng = np.random.default_rng(1)
    # sample per step sized so that the whole run takes about a minute of CPU
    n = 256

    def one():
        b = rng.integers(0, wl.B, n)
        i = rng.integers(0, wl.N, n)
        sel = oracle.flat_index(wl, np.repeat(b, wl.H), np.tile(np.arange(wl.H), n),
                                np.repeat(i, wl.H))
        t0 = time.perf_counter()
        oracle.forward(wl, inp["coords"], inp["q"], inp["k"], inp["v"], sel=sel,
                       summaries=(ks, vs))
        return time.perf_counter() - t0

    per_tok = one() / n  # calibration
    n = int(max(16, min(args.cpu_sample // 4, 60.0 / max(per_tok, 1e-9) /
                        (args.steps + args.warmup))))
    for _ in range(args.warmup):
        one()
    times = [one() for _ in range(args.steps)]
    per_token = sum(times) / (n * args.steps)
    value = 1.0 / per_token
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * sum(times) / len(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (same workload and seed as the CUDA arm)",
        "config": run_config(wl, args.packing, world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.max_threads(),
                         "kind": "oracle",
                         "sample": f"each step {n} random query tokens x {wl.H} heads of "
                                   f"{wl.name} (block summaries precomputed)"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="vol_32x32x64")
    ap.add_argument("--packing", default="random")
    ap.add_argument("--cpu-sample", type=int, default=32768,
                    help="query tokens the CPU oracle computes for the baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", default="all", choices=["all", "forward", "backward"],
                    help="forward / backward: time that alone and print a short line "
                         "(for profiler runs)")
    ap.add_argument("--no-micro1m", dest="micro1m", action="store_false",
                    help="skip the 1M-token workload and the CUDA-core sections (fp32 mode, "
                         "bf16 at head dim 48)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)
    if int(os.environ.get("WORLD_SIZE", "1")) > 1 and args.impl == "ours":
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
