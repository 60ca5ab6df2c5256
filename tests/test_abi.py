"""The C-ABI library builds, loads and exports every entry point the header
declares; host-side argument checks work without a GPU (no CUDA call is made)."""
import ctypes
import os
import re
from types import SimpleNamespace

import pytest

from local_global_attention_b200 import build as B
from local_global_attention_b200 import pack3d as P

HEADER = os.path.join(B.ROOT, "include", "pack3d.h")


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"PACK3D_API\s+[\w\s\*]+?\b(pack3d_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    B.build()
    return P.load()


def test_header_declares_the_operator_calls():
    names = declared_symbols()
    for n in ("pack3d_build_index", "pack3d_block_summaries", "pack3d_forward",
              "pack3d_window_forward", "pack3d_backward"):
        assert n in names
    assert set(names) == set(P.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def shape(**kw):
    base = dict(B=2, H=8, d=96, Z=32, Y=32, X=64, window=(7, 7, 7), block=(8, 8, 8),
                rope_base=100.0, dtype="bf16")
    base.update(kw)
    return SimpleNamespace(**base)


def test_index_bytes_and_argument_checks(lib):
    p = P.make_params(shape())
    n = lib.pack3d_index_bytes(ctypes.byref(p))
    N = 32 * 32 * 64
    assert n >= 4 * (2 * 2 * N)  # vol + perm at least
    for bad in (dict(window=(6, 7, 7)), dict(block=(0, 8, 8)),
                dict(d=90), dict(d=0), dict(rope_base=0.0), dict(Z=0)):
        assert lib.pack3d_index_bytes(ctypes.byref(P.make_params(shape(**bad)))) == 0, bad
    # shapes the library is not built for report ERR_UNSUPPORTED, not ERR_ARG:
    # head dims outside 12/24/48/96
    idx = P.Index()
    st = lib.pack3d_index_init(ctypes.byref(P.make_params(shape(d=36))), ctypes.c_void_p(256),
                               ctypes.c_size_t(1 << 30), ctypes.byref(idx))
    assert st == P.ERR_UNSUPPORTED
    # block extents that do not divide the volume are the operator with the
    # last blocks cut at the edge: accepted
    assert lib.pack3d_index_bytes(ctypes.byref(P.make_params(shape(block=(5, 8, 8))))) > 0
    assert lib.pack3d_index_init(ctypes.byref(P.make_params(shape(block=(0, 8, 8)))),
                                 ctypes.c_void_p(256), ctypes.c_size_t(1 << 30),
                                 ctypes.byref(idx)) == P.ERR_ARG
    # misaligned or short buffers are rejected before any device access
    assert lib.pack3d_index_init(ctypes.byref(p), ctypes.c_void_p(257), ctypes.c_size_t(n),
                                 ctypes.byref(idx)) == P.ERR_ARG
    assert lib.pack3d_index_init(ctypes.byref(p), ctypes.c_void_p(256), ctypes.c_size_t(n - 1),
                                 ctypes.byref(idx)) == P.ERR_ARG
    assert lib.pack3d_index_init(ctypes.byref(p), ctypes.c_void_p(1 << 20), ctypes.c_size_t(n),
                                 ctypes.byref(idx)) == P.OK
    assert tuple(idx.tile) == (4, 4, 8)
    assert idx.n_tiles == 8 * 8 * 8
    # halo list length: product over axes of the clipped tile extents
    assert idx.n_halo == (7 + 7 + 6 * 10) ** 2 * (11 + 11 + 6 * 14)


def test_null_pointers_rejected_without_cuda(lib):
    p = P.make_params(shape())
    idx = P.Index()
    assert lib.pack3d_build_index(ctypes.byref(p), None, ctypes.byref(idx), None) == P.ERR_ARG
    assert lib.pack3d_forward(ctypes.byref(p), ctypes.byref(idx), None, None, None, None, None,
                              None, ctypes.c_size_t(0), None, None, None) == P.ERR_ARG
    assert lib.pack3d_backward(ctypes.byref(p), None, *([None] * 10), ctypes.c_size_t(0),
                               None) == P.ERR_ARG


def test_strerror(lib):
    for st in (P.OK, P.ERR_ARG, P.ERR_COORDS, P.ERR_CUDA, P.ERR_TIMEOUT, P.ERR_UNSUPPORTED):
        assert P.strerror(st)
    assert P.strerror(12345) == "unknown status"


def test_forward_workspace_size_and_checks(lib):
    """The tensor-core forward's workspace: grid-order copies of the rotated
    keys and of the values plus bf16 summary copies (256-byte aligned
    sections); none for the CUDA-core paths.  A missing, short or misaligned
    workspace is rejected before anything is launched."""
    al = lambda x: (x + 255) // 256 * 256
    p = P.make_params(shape())
    vol = 2 * 8 * 32 * 32 * 64 * 96 * 2
    summ = 2 * 8 * (4 * 4 * 8) * 96 * 2
    need = lib.pack3d_forward_workspace_bytes(ctypes.byref(p))
    assert need == 2 * al(vol) + 2 * al(summ)
    assert lib.pack3d_forward_workspace_bytes(ctypes.byref(P.make_params(shape(dtype="fp32")))) == 0
    assert lib.pack3d_forward_workspace_bytes(ctypes.byref(P.make_params(shape(d=48)))) == 0
    idx = P.Index()
    assert lib.pack3d_index_init(ctypes.byref(p), ctypes.c_void_p(1 << 20), ctypes.c_size_t(1 << 40),
                                 ctypes.byref(idx)) == P.OK
    fake = ctypes.c_void_p(1 << 30)
    for ws, nbytes in ((None, need), (ctypes.c_void_p((1 << 32) + 16), need),
                       (ctypes.c_void_p(1 << 32), need - 1)):
        assert lib.pack3d_forward(ctypes.byref(p), ctypes.byref(idx), fake, fake, fake, fake, fake,
                                  ws, ctypes.c_size_t(nbytes), fake, fake, None) == P.ERR_ARG
        assert lib.pack3d_window_forward(ctypes.byref(p), ctypes.byref(idx), fake, fake, fake, ws,
                                         ctypes.c_size_t(nbytes), fake, fake, None) == P.ERR_ARG


def simt_backward_bytes(wl):
    """Workspace of the CUDA-core backward: delta [B][H][N] + k/v summaries and
    their gradients (4 x [B][H][nb][d] fp32, each 256-byte aligned) + the
    d = 96 summary kernel's per-split partial sums (2 x splits x
    [B][H][nb][d]); the splits fill one wave of two CTAs per SM (148 SMs) over
    B*H*ceil(nb/64) groups, at most one per query tile and at most 32."""
    def a256(x):
        return (x + 255) // 256 * 256
    nb, nT = wl.n_blocks, -(-wl.Z // 4) * -(-wl.Y // 4) * -(-wl.X // 8)
    ns = 4 * wl.B * wl.H * nb * wl.d
    splits = 0
    if wl.d == 96:
        splits = max(1, min(296 // (wl.B * wl.H * -(-nb // 64)), nT, 32))
    return a256(4 * wl.B * wl.H * wl.N) + 4 * a256(ns) + 2 * splits * ns


def test_noalloc_scratch_holds_the_training_shape(lib):
    """The allocation-free backward runs the CUDA-core kernels; the static
    array (its size stated in the header) holds their workspace at the
    65k-token training shape."""
    from local_global_attention_b200 import configs as C
    hdr = open(HEADER).read()
    m = re.search(r"#define PACK3D_NOALLOC_SCRATCH_BYTES \(\(size_t\)(\d+) << 20\)", hdr)
    assert m and (int(m.group(1)) << 20) == P.NOALLOC_SCRATCH_BYTES
    assert 0 < simt_backward_bytes(C.TRAIN65K) <= P.NOALLOC_SCRATCH_BYTES


def test_backward_workspace_layout(lib):
    """bf16 at head_dim 96 runs the tensor-core backward, whose workspace holds
    grid-order copies of rotated k, v, rotated q and dO (4 x [B][H][N][96]
    bf16), per-voxel (lse, delta) pairs padded to 16 bytes, the same as 16 bf16
    contraction channels per voxel (32 bytes), the fp32 summaries,
    their bf16 copies, the summary gradients, and the summary role's per-split
    partial sums (2 x splits x [B][H][nb][96] fp32; the splits fill one wave of
    148 CTAs over B*H*ceil(nb/128) row tiles, at most 64); every section
    256-byte aligned.  Other dtypes and head dims run the CUDA-core backward."""
    from local_global_attention_b200 import configs as C

    def a256(x):
        return (x + 255) // 256 * 256

    for wl in (C.TRAIN65K, C.VOL16K):
        nb = wl.n_blocks
        vox = wl.B * wl.H * wl.N
        s32 = 4 * wl.B * wl.H * nb * wl.d
        chunks = -(-wl.Z // 2) * -(-wl.Y // 2) * -(-wl.X // 16)
        groups = wl.B * wl.H * -(-nb // 128)
        splits = max(1, min(-(-148 // groups), chunks, 64))
        want = (4 * a256(vox * 96 * 2) + a256(vox * 16) + a256(vox * 32) + 2 * a256(s32) +
                2 * a256(s32 // 2) +
                2 * a256(s32) + a256(splits * 2 * s32))
        assert lib.pack3d_backward_workspace_bytes(ctypes.byref(P.make_params(wl))) == want
    for wl in (C.TINY, C.TRAIN65K.replace(dtype="fp32")):
        assert lib.pack3d_backward_workspace_bytes(ctypes.byref(P.make_params(wl))) == \
            simt_backward_bytes(wl)


def test_size_limits(lib):
    """The header's limits: extents up to 32767 per axis and
    B * N * H * head_dim below 2^31 (32-bit element offsets); beyond them the
    shape is rejected before anything is sized or launched."""
    ok = shape(B=1, H=1, d=96, Z=1, Y=1, X=32767, window=(1, 1, 1), block=(1, 1, 1))
    assert lib.pack3d_index_bytes(ctypes.byref(P.make_params(ok))) > 0
    for bad in (dict(X=32768), dict(Z=-1)):
        s = shape(B=1, H=1, d=96, Z=1, Y=1, X=32767, window=(1, 1, 1), block=(1, 1, 1))
        s.__dict__.update(bad)
        assert lib.pack3d_index_bytes(ctypes.byref(P.make_params(s))) == 0, bad
    # 3 x 8 heads x 2^20 tokens x 96 = 1.125 * 2^31 elements: too many
    big = shape(B=3, H=8, d=96, Z=64, Y=128, X=128, window=(5, 7, 7), block=(4, 16, 16))
    assert lib.pack3d_index_bytes(ctypes.byref(P.make_params(big))) == 0
    # two items fit (0.75 * 2^31)
    fits = shape(B=2, H=8, d=96, Z=64, Y=128, X=128, window=(5, 7, 7), block=(4, 16, 16))
    assert lib.pack3d_index_bytes(ctypes.byref(P.make_params(fits))) > 0


def test_backward_rejects_unbuilt_halo_before_any_launch(lib):
    """The CUDA-core backward stages one halo row (the tile's 8 columns widened
    by the window radius on both sides and clipped to the volume) at a time, so
    rows longer than its staging buffer report ERR_UNSUPPORTED.  The check runs on
    the host before anything is launched: here, on a machine without a GPU, a
    launch would have returned ERR_CUDA instead.  The allocation-free variant
    rejects the same shape the same way."""
    wide = shape(B=1, H=1, d=96, Z=4, Y=4, X=200, window=(1, 1, 161), block=(4, 4, 8),
                 dtype="fp32")
    p = P.make_params(wide)
    idx = P.Index()
    assert lib.pack3d_index_init(ctypes.byref(p), ctypes.c_void_p(1 << 20),
                                 ctypes.c_size_t(1 << 40), ctypes.byref(idx)) == P.OK
    need = lib.pack3d_backward_workspace_bytes(ctypes.byref(p))
    fake = ctypes.c_void_p(1 << 30)
    assert lib.pack3d_backward(ctypes.byref(p), ctypes.byref(idx), *([fake] * 9),
                               ctypes.c_void_p(1 << 32), ctypes.c_size_t(need),
                               None) == P.ERR_UNSUPPORTED
    assert lib.pack3d_backward_noalloc(ctypes.byref(p), ctypes.byref(idx), *([fake] * 9),
                                       None) == P.ERR_UNSUPPORTED
    # bf16 at head_dim 96: pack3d_backward runs the tensor-core kernels, which
    # stream halo chunks and have no such limit; the allocation-free backward
    # runs the CUDA-core kernels and rejects the shape as well
    pb = P.make_params(shape(B=1, H=1, d=96, Z=4, Y=4, X=200, window=(1, 1, 161),
                             block=(4, 4, 8)))
    assert lib.pack3d_backward_noalloc(ctypes.byref(pb), ctypes.byref(idx), *([fake] * 9),
                                       None) == P.ERR_UNSUPPORTED


def test_kernel_launch_counter_without_cuda(lib):
    """The launch counter is host-side: readable without a GPU, and calls that
    are rejected before launching leave it unchanged."""
    n0 = P.pack3d_kernel_launches()
    p = P.make_params(shape())
    idx = P.Index()
    assert lib.pack3d_forward(ctypes.byref(p), ctypes.byref(idx), None, None, None, None, None,
                              None, ctypes.c_size_t(0), None, None, None) == P.ERR_ARG
    assert P.pack3d_kernel_launches() == n0


def test_partly_occupied_params(lib):
    """n_tokens: 0 is a dense volume; 1 .. Z*Y*X tokens at distinct voxels is a
    partly occupied one (the index holds the same arrays, the coordinate volume
    sized by voxels, the permutation by tokens); outside that range the params
    are rejected."""
    dense = P.make_params(shape(B=1, H=2, d=96, Z=4, Y=8, X=16, block=(2, 4, 4)))
    part = P.make_params(shape(B=1, H=2, d=96, Z=4, Y=8, X=16, block=(2, 4, 4), n_tokens=100))
    assert lib.pack3d_index_bytes(ctypes.byref(part)) > 0
    # the permutation shrinks with the token count
    assert lib.pack3d_index_bytes(ctypes.byref(part)) <= lib.pack3d_index_bytes(ctypes.byref(dense))
    for bad in (-1, 4 * 8 * 16 + 1):
        p = P.make_params(shape(B=1, H=2, d=96, Z=4, Y=8, X=16, block=(2, 4, 4), n_tokens=bad))
        assert lib.pack3d_index_bytes(ctypes.byref(p)) == 0, bad
    idx = P.Index()
    assert lib.pack3d_index_init(ctypes.byref(part), ctypes.c_void_p(1 << 20),
                                 ctypes.c_size_t(1 << 30), ctypes.byref(idx)) == P.OK
    assert idx.bcount and idx.bocc and idx.bocc > idx.bcount


def test_two_call_backward_checks_without_cuda(lib):
    """The two-call backward: missing pointers, a short workspace and a slab
    call without the whole volume's summaries are ERR_ARG; the CUDA-core shapes
    and slabs of the packed-RoPE mode are ERR_UNSUPPORTED; all of it before any
    launch (the counter does not move)."""
    n0 = P.pack3d_kernel_launches()
    fake = ctypes.c_void_p(1 << 30)
    ws = ctypes.c_void_p(1 << 32)

    def index_for(p):
        idx = P.Index()
        assert lib.pack3d_index_init(ctypes.byref(p), ctypes.c_void_p(1 << 20),
                                     ctypes.c_size_t(1 << 40), ctypes.byref(idx)) == P.OK
        return idx

    def first(p, idx, ksum, nbytes):
        return lib.pack3d_backward_summary_grads(ctypes.byref(p), ctypes.byref(idx),
                                                 *([fake] * 6), ksum, ksum, fake, fake, ws,
                                                 ctypes.c_size_t(nbytes), None)

    def second(p, idx, nbytes, dq=fake):
        return lib.pack3d_backward_from_summary_grads(ctypes.byref(p), ctypes.byref(idx), fake,
                                                      fake, ws, ctypes.c_size_t(nbytes), dq,
                                                      fake, fake, None)

    dense = shape(B=1, H=2, d=96, Z=16, Y=8, X=16, block=(4, 4, 4), window=(5, 3, 7))
    p = P.make_params(dense)
    idx = index_for(p)
    need = lib.pack3d_backward_workspace_bytes(ctypes.byref(p))
    assert need > 0
    assert first(p, idx, None, need - 1) == P.ERR_ARG
    assert second(p, idx, need - 1) == P.ERR_ARG
    assert second(p, idx, need, dq=None) == P.ERR_ARG
    assert lib.pack3d_backward_summary_grads(ctypes.byref(p), ctypes.byref(idx), None,
                                             *([fake] * 5), None, None, fake, fake, ws,
                                             ctypes.c_size_t(need), None) == P.ERR_ARG
    # given summaries: both or neither
    assert lib.pack3d_backward_summary_grads(ctypes.byref(p), ctypes.byref(idx), *([fake] * 6),
                                             fake, None, fake, fake, ws, ctypes.c_size_t(need),
                                             None) == P.ERR_ARG
    # CUDA-core shapes
    p32 = P.make_params(SimpleNamespace(**{**dense.__dict__, "dtype": "fp32"}))
    idx32 = index_for(p32)
    assert first(p32, idx32, None, 1 << 40) == P.ERR_UNSUPPORTED
    assert second(p32, idx32, 1 << 40) == P.ERR_UNSUPPORTED
    # a z-slab (planes 0 .. 11 of 16, owning 0 .. 8) needs the given summaries
    slab = SimpleNamespace(**{**dense.__dict__, "Z": 11, "Z_total": 16, "z_origin": 0,
                              "own_lo": 0, "own_hi": 8})
    ps = P.make_params(slab)
    idxs = index_for(ps)
    need_s = lib.pack3d_backward_workspace_bytes(ctypes.byref(ps))
    assert first(ps, idxs, None, need_s) == P.ERR_ARG
    assert lib.pack3d_backward(ctypes.byref(ps), ctypes.byref(idxs), *([fake] * 9), ws,
                               ctypes.c_size_t(need_s), None) == P.ERR_UNSUPPORTED
    psr = P.make_params(SimpleNamespace(**{**slab.__dict__, "rope_mode": 1}))
    idxr = index_for(psr)
    assert first(psr, idxr, fake, 1 << 40) == P.ERR_UNSUPPORTED
    assert P.pack3d_kernel_launches() == n0


def test_wait_selftest_argument_checks_without_cuda(lib):
    """A poll count of 0 or above 2^24 is rejected before anything is launched."""
    n0 = P.pack3d_kernel_launches()
    assert lib.pack3d_wait_selftest(ctypes.c_uint32(0), None) == P.ERR_ARG
    assert lib.pack3d_wait_selftest(ctypes.c_uint32((1 << 24) + 1), None) == P.ERR_ARG
    assert P.pack3d_kernel_launches() == n0
