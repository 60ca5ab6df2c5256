"""The five synthetic PACK3D workloads, by shape.

Sizes follow the operator's stated evaluation settings: a tiny fp32 volume the
CPU oracle finishes in seconds, a 16k-token Morton-packed volume, the
65k-token operator under all four packings (the shape the paper's abstract
quotes its latency claim at), a 1M-token anisotropic microscopy-shaped smooth
field (a synthetic stand-in for the WTC-11 hiPSC volumes the paper evaluates on,
which are not available here), and a training step at the 65k shape.
"""
import math

from .inputs import Workload

TINY = Workload(
    name="tiny_8x8x8", B=1, H=1, d=48, Z=8, Y=8, X=8, window=(3, 3, 3), block=(4, 4, 4),
    dtype="fp32", values="normal", value_scale=1.0, packings=("raster",), seed=0,
    note="512 tokens, 16 channels per axis, RoPE base 100, 8 summaries, fp32")

VOL16K = Workload(
    name="vol_16x32x32", B=1, H=8, d=96, Z=16, Y=32, X=32, window=(7, 7, 7), block=(8, 8, 8),
    dtype="bf16", values="normal", value_scale=1.0 / math.sqrt(96), packings=("morton",), seed=1,
    note="16,384 tokens, 32 summaries, Morton packing, forward only")

VOL65K = Workload(
    name="vol_32x32x64", B=2, H=8, d=96, Z=32, Y=32, X=64, window=(7, 7, 7), block=(8, 8, 8),
    dtype="bf16", values="normal", value_scale=1.0 / math.sqrt(96),
    packings=("raster", "morton", "block", "random"), seed=2,
    note="65,536 tokens x batch 2, 128 summaries, four packings")

MICRO1M = Workload(
    name="micro_64x128x128", B=1, H=4, d=96, Z=64, Y=128, X=128, window=(5, 7, 7),
    block=(4, 16, 16), dtype="bf16", values="smooth", packings=("block",), seed=3,
    note="1,048,576 tokens, 1,024 summaries, smooth random field, block-contiguous")

TRAIN65K = Workload(
    name="train_32x32x64", B=2, H=8, d=96, Z=32, Y=32, X=64, window=(7, 7, 7), block=(8, 8, 8),
    dtype="bf16", values="normal", value_scale=1.0 / math.sqrt(96), packings=("random",),
    seed=4, backward=True,
    note="65k-token training step: forward + backward, dO ~ N(0,1), random packing")

ALL = (TINY, VOL16K, VOL65K, MICRO1M, TRAIN65K)
BY_NAME = {w.name: w for w in ALL}
