"""Python binding of the PACK3D C ABI (include/pack3d.h) over ctypes.

Argument marshalling only: every step of the operator runs in the CUDA
library ``_build/libpack3d.so``.  Tensors are torch CUDA tensors; the functions
keep the C names and pass ``data_ptr()`` and the current (or given) stream.
If the library is missing or no CUDA device is present, the calls raise; there
is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

from . import build as _build

BF16, FP32 = 0, 1
ROPE_AXIAL, ROPE_PACKED = 0, 1  # axial RoPE on grid coordinates / 1-D RoPE on the packed index
OK, ERR_ARG, ERR_COORDS, ERR_CUDA, ERR_TIMEOUT, ERR_UNSUPPORTED = 0, -1, -2, -3, -4, -5

EXPORTS = ("pack3d_index_bytes", "pack3d_index_init", "pack3d_build_index", "pack3d_index_check",
           "pack3d_block_summaries", "pack3d_forward_workspace_bytes", "pack3d_forward",
           "pack3d_window_forward", "pack3d_stage_kv", "pack3d_forward_staged",
           "pack3d_backward_workspace_bytes", "pack3d_backward", "pack3d_backward_summary_grads",
           "pack3d_backward_from_summary_grads", "pack3d_backward_noalloc",
           "pack3d_kernel_launches", "pack3d_wait_selftest", "pack3d_strerror")


class Params(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("B", "H", "head_dim", "Z", "Y", "X", "wz", "wy", "wx", "bz", "by", "bx")] + [
        ("rope_base", ctypes.c_float), ("scale", ctypes.c_float), ("dtype", ctypes.c_int32),
        ("out_fp32", ctypes.c_int32), ("rope_mode", ctypes.c_int32), ("n_tokens", ctypes.c_int32),
        ("Z_total", ctypes.c_int32), ("z_origin", ctypes.c_int32), ("own_lo", ctypes.c_int32),
        ("own_hi", ctypes.c_int32)]


class Index(ctypes.Structure):
    _fields_ = [("vol", ctypes.c_void_p), ("perm", ctypes.c_void_p),
                ("tile_off", ctypes.c_void_p), ("nbr_off", ctypes.c_void_p),
                ("nbr", ctypes.c_void_p), ("rope", ctypes.c_void_p), ("err", ctypes.c_void_p),
                ("bcount", ctypes.c_void_p), ("bocc", ctypes.c_void_p),
                ("tile", ctypes.c_int32 * 3), ("n_tiles", ctypes.c_int32),
                ("n_halo", ctypes.c_int64)]


class Pack3dError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {strerror(status)} ({status})")
        self.status = status


_lib = None


def library_path() -> str:
    return _build.LIB


def load(build_if_missing: bool = True):
    """Load libpack3d.so (building it in-tree first if it is missing)."""
    global _lib
    if _lib is None:
        path = _build.LIB
        if not os.path.exists(path):
            if not build_if_missing:
                raise OSError(f"PACK3D CUDA library not built: {path}")
            _build.build()
        lib = ctypes.CDLL(path)
        P = ctypes.POINTER
        vp = ctypes.c_void_p
        lib.pack3d_index_bytes.argtypes = [P(Params)]
        lib.pack3d_index_bytes.restype = ctypes.c_size_t
        lib.pack3d_index_init.argtypes = [P(Params), vp, ctypes.c_size_t, P(Index)]
        lib.pack3d_build_index.argtypes = [P(Params), vp, P(Index), vp]
        lib.pack3d_index_check.argtypes = [P(Index), vp]
        lib.pack3d_block_summaries.argtypes = [P(Params), P(Index), vp, vp, vp, vp, vp]
        lib.pack3d_forward_workspace_bytes.argtypes = [P(Params)]
        lib.pack3d_forward_workspace_bytes.restype = ctypes.c_size_t
        lib.pack3d_forward.argtypes = [P(Params), P(Index), vp, vp, vp, vp, vp, vp,
                                       ctypes.c_size_t, vp, vp, vp]
        lib.pack3d_window_forward.argtypes = [P(Params), P(Index), vp, vp, vp, vp,
                                              ctypes.c_size_t, vp, vp, vp]
        lib.pack3d_stage_kv.argtypes = [P(Params), P(Index), vp, vp, vp, vp, vp, ctypes.c_size_t,
                                        vp]
        lib.pack3d_forward_staged.argtypes = [P(Params), P(Index), vp, vp, ctypes.c_size_t,
                                              ctypes.c_int, vp, vp, vp]
        lib.pack3d_backward_workspace_bytes.argtypes = [P(Params)]
        lib.pack3d_backward_workspace_bytes.restype = ctypes.c_size_t
        lib.pack3d_backward.argtypes = [P(Params), P(Index), vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                        vp, ctypes.c_size_t, vp]
        lib.pack3d_backward_summary_grads.argtypes = [P(Params), P(Index), vp, vp, vp, vp, vp,
                                                      vp, vp, vp, vp, vp, vp, ctypes.c_size_t,
                                                      vp]
        lib.pack3d_backward_from_summary_grads.argtypes = [P(Params), P(Index), vp, vp, vp,
                                                           ctypes.c_size_t, vp, vp, vp, vp]
        lib.pack3d_backward_noalloc.argtypes = [P(Params), P(Index), vp, vp, vp, vp, vp, vp, vp,
                                                vp, vp, vp]
        lib.pack3d_wait_selftest.argtypes = [ctypes.c_uint32, vp]
        lib.pack3d_kernel_launches.argtypes = []
        lib.pack3d_kernel_launches.restype = ctypes.c_uint64
        lib.pack3d_strerror.argtypes = [ctypes.c_int]
        lib.pack3d_strerror.restype = ctypes.c_char_p
        for name in EXPORTS:
            getattr(lib, name).restype = getattr(lib, name).restype or ctypes.c_int
        _lib = lib
    return _lib


def pack3d_kernel_launches() -> int:
    """Kernels the library has launched in this process so far."""
    return int(load().pack3d_kernel_launches())


def pack3d_wait_selftest(polls: int = 1000, stream=None) -> int:
    """Status of a bounded device wait that runs out (ERR_TIMEOUT expected)."""
    return int(load().pack3d_wait_selftest(ctypes.c_uint32(polls), _stream(stream)))


def strerror(status: int) -> str:
    return load().pack3d_strerror(int(status)).decode()


def _check(status: int, what: str):
    if status != OK:
        raise Pack3dError(status, what)


def make_params(shape, dtype=None, scale: float = 0.0, out_fp32: bool = False) -> Params:
    """Params from any object with ``B, H, d, Z, Y, X, window, block, rope_base``
    (and ``dtype`` "bf16"/"fp32" unless given, ``rope_mode`` 0, ``n_tokens`` 0
    (a dense volume) and no z-slab (``Z_total``, ``z_origin``, ``own_lo``,
    ``own_hi``) unless set).  ``out_fp32`` makes the forward output fp32 for
    bf16 inputs."""
    dt = dtype if dtype is not None else getattr(shape, "dtype", "bf16")
    code = {"bf16": BF16, "fp32": FP32, torch.bfloat16: BF16, torch.float32: FP32}[dt]
    w, b = tuple(shape.window), tuple(shape.block)
    return Params(shape.B, shape.H, shape.d, shape.Z, shape.Y, shape.X, w[0], w[1], w[2],
                  b[0], b[1], b[2], float(shape.rope_base), float(scale), code, int(bool(out_fp32)),
                  int(getattr(shape, "rope_mode", 0) or 0), int(getattr(shape, "n_tokens", 0) or 0),
                  *(int(getattr(shape, f, 0) or 0) for f in ("Z_total", "z_origin", "own_lo",
                                                             "own_hi")))


def out_dtype(params: Params, like: torch.Tensor) -> torch.dtype:
    return torch.float32 if params.out_fp32 else like.dtype


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("PACK3D tensors must be CUDA tensors")
        if t is not None and not t.is_contiguous():
            raise ValueError("PACK3D tensors must be contiguous")


class IndexBuffers:
    """A built index: the caller-owned device buffer and the C struct over it."""

    def __init__(self, params: Params, device=None):
        lib = load()
        self.params = params
        nbytes = lib.pack3d_index_bytes(ctypes.byref(params))
        if nbytes == 0:
            raise Pack3dError(ERR_ARG, "pack3d_index_bytes")
        self.buffer = torch.empty(nbytes + 256, dtype=torch.uint8, device=device or "cuda")
        base = self.buffer.data_ptr()
        off = (-base) % 256
        self.struct = Index()
        _check(lib.pack3d_index_init(ctypes.byref(params), ctypes.c_void_p(base + off),
                                     ctypes.c_size_t(nbytes), ctypes.byref(self.struct)),
               "pack3d_index_init")
        self.nbytes = nbytes

    # Views of the index arrays (for tests and inspection).
    def _view(self, field, count, dtype):
        ptr = getattr(self.struct, field)
        off = ptr - self.buffer.data_ptr()
        esz = torch.tensor([], dtype=dtype).element_size()
        return self.buffer[off:off + count * esz].view(dtype)

    def arrays(self):
        p, s = self.params, self.struct
        V = p.Z * p.Y * p.X
        N = p.n_tokens or V
        T = s.n_tiles
        nb = (-(-(p.Z_total or p.Z) // p.bz)) * (-(-p.Y // p.by)) * (-(-p.X // p.bx))
        return {
            "vol": self._view("vol", p.B * V, torch.int32).view(p.B, V),
            "bcount": self._view("bcount", p.B * nb, torch.int32).view(p.B, nb),
            "perm": self._view("perm", p.B * N, torch.int32).view(p.B, N),
            "tile_off": self._view("tile_off", p.B * (T + 1), torch.int32).view(p.B, T + 1),
            "nbr_off": self._view("nbr_off", T + 1, torch.int32),
            "nbr": self._view("nbr", p.B * s.n_halo, torch.int32).view(p.B, s.n_halo),
            "rope": self._view("rope", 2 * (p.Z + p.Y + p.X) * (p.head_dim // 6), torch.float32),
            "err": self._view("err", 2, torch.int32),
        }


def pack3d_build_index(params: Params, coords: torch.Tensor, index: IndexBuffers = None,
                       stream=None) -> IndexBuffers:
    _need_cuda(coords)
    if coords.dtype != torch.int16:
        raise ValueError("coords must be int16 [B, N, 3]")
    if index is None:
        index = IndexBuffers(params, device=coords.device)
    _check(load().pack3d_build_index(ctypes.byref(params), _ptr(coords),
                                     ctypes.byref(index.struct), _stream(stream)),
           "pack3d_build_index")
    return index


def pack3d_index_check(index: IndexBuffers, stream=None) -> int:
    """Synchronise and return the index status code (0, ERR_COORDS, ERR_TIMEOUT)."""
    return int(load().pack3d_index_check(ctypes.byref(index.struct), _stream(stream)))


def _dims(params):
    return params.B, params.n_tokens or params.Z * params.Y * params.X, params.H, params.head_dim


def n_blocks(params: Params) -> int:
    """Blocks of the volume (a z-slab: of the whole volume); blocks that do not
    divide the volume are cut at its edge, so the counts round up."""
    Zg = params.Z_total or params.Z
    return (-(-Zg // params.bz)) * (-(-params.Y // params.by)) * (-(-params.X // params.bx))


def pack3d_block_summaries(params: Params, index: IndexBuffers, k, v, ksum=None, vsum=None,
                           stream=None):
    _need_cuda(k, v)
    B, N, H, d = _dims(params)
    nb = n_blocks(params)
    if ksum is None:
        ksum = torch.empty(B, H, nb, d, dtype=torch.float32, device=k.device)
    if vsum is None:
        vsum = torch.empty(B, H, nb, d, dtype=torch.float32, device=k.device)
    _need_cuda(ksum, vsum)
    _check(load().pack3d_block_summaries(ctypes.byref(params), ctypes.byref(index.struct),
                                         _ptr(k), _ptr(v), _ptr(ksum), _ptr(vsum),
                                         _stream(stream)), "pack3d_block_summaries")
    return ksum, vsum


def pack3d_forward_workspace_bytes(params: Params) -> int:
    return int(load().pack3d_forward_workspace_bytes(ctypes.byref(params)))


def _forward_workspace(params, workspace, device):
    nbytes = pack3d_forward_workspace_bytes(params)
    if workspace is None and nbytes:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)
    if workspace is None:
        return None, 0
    _need_cuda(workspace)
    return workspace, workspace.numel() * workspace.element_size()


def pack3d_forward(params: Params, index: IndexBuffers, q, k, v, ksum, vsum, out=None, lse=None,
                   workspace=None, stream=None):
    _need_cuda(q, k, v, ksum, vsum)
    B, N, H, d = _dims(params)
    out = torch.empty_like(q, dtype=out_dtype(params, q)) if out is None else out
    lse = torch.empty(B, H, N, dtype=torch.float32, device=q.device) if lse is None else lse
    _need_cuda(out, lse)
    ws, nbytes = _forward_workspace(params, workspace, q.device)
    _check(load().pack3d_forward(ctypes.byref(params), ctypes.byref(index.struct), _ptr(q),
                                 _ptr(k), _ptr(v), _ptr(ksum), _ptr(vsum),
                                 None if ws is None else _ptr(ws), ctypes.c_size_t(nbytes),
                                 _ptr(out), _ptr(lse), _stream(stream)), "pack3d_forward")
    return out, lse


def pack3d_window_forward(params: Params, index: IndexBuffers, q, k, v, out=None, lse=None,
                          workspace=None, stream=None):
    _need_cuda(q, k, v)
    B, N, H, d = _dims(params)
    out = torch.empty_like(q, dtype=out_dtype(params, q)) if out is None else out
    lse = torch.empty(B, H, N, dtype=torch.float32, device=q.device) if lse is None else lse
    _need_cuda(out, lse)
    ws, nbytes = _forward_workspace(params, workspace, q.device)
    _check(load().pack3d_window_forward(ctypes.byref(params), ctypes.byref(index.struct),
                                        _ptr(q), _ptr(k), _ptr(v),
                                        None if ws is None else _ptr(ws),
                                        ctypes.c_size_t(nbytes), _ptr(out), _ptr(lse),
                                        _stream(stream)), "pack3d_window_forward")
    return out, lse


def pack3d_stage_kv(params: Params, index: IndexBuffers, k, v, ksum=None, vsum=None,
                    workspace=None, stream=None):
    """Stage rotated keys and values in grid order (and bf16 summaries) for
    pack3d_forward_staged; returns the workspace."""
    _need_cuda(k, v)
    ws, nbytes = _forward_workspace(params, workspace, k.device)
    _check(load().pack3d_stage_kv(ctypes.byref(params), ctypes.byref(index.struct), _ptr(k),
                                  _ptr(v), None if ksum is None else _ptr(ksum),
                                  None if vsum is None else _ptr(vsum),
                                  None if ws is None else _ptr(ws), ctypes.c_size_t(nbytes),
                                  _stream(stream)), "pack3d_stage_kv")
    return ws


def pack3d_forward_staged(params: Params, index: IndexBuffers, q, workspace, with_summaries=True,
                          out=None, lse=None, stream=None):
    _need_cuda(q, workspace)
    B, N, H, d = _dims(params)
    out = torch.empty_like(q, dtype=out_dtype(params, q)) if out is None else out
    lse = torch.empty(B, H, N, dtype=torch.float32, device=q.device) if lse is None else lse
    _need_cuda(out, lse)
    _check(load().pack3d_forward_staged(ctypes.byref(params), ctypes.byref(index.struct), _ptr(q),
                                        _ptr(workspace),
                                        ctypes.c_size_t(workspace.numel() *
                                                        workspace.element_size()),
                                        int(bool(with_summaries)), _ptr(out), _ptr(lse),
                                        _stream(stream)), "pack3d_forward_staged")
    return out, lse


def pack3d_backward_workspace_bytes(params: Params) -> int:
    return int(load().pack3d_backward_workspace_bytes(ctypes.byref(params)))


def pack3d_backward(params: Params, index: IndexBuffers, q, k, v, out, lse, dout, dq=None,
                    dk=None, dv=None, workspace=None, stream=None):
    _need_cuda(q, k, v, out, lse, dout)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    nbytes = pack3d_backward_workspace_bytes(params)
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    _need_cuda(dq, dk, dv, workspace)
    _check(load().pack3d_backward(ctypes.byref(params), ctypes.byref(index.struct), _ptr(q),
                                  _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(dout), _ptr(dq),
                                  _ptr(dk), _ptr(dv), _ptr(workspace),
                                  ctypes.c_size_t(workspace.numel() * workspace.element_size()),
                                  _stream(stream)), "pack3d_backward")
    return dq, dk, dv


def pack3d_backward_summary_grads(params: Params, index: IndexBuffers, q, k, v, out, lse, dout,
                                  ksum=None, vsum=None, dks=None, dvs=None, workspace=None,
                                  stream=None):
    """First half of the two-call backward: stages the inputs into `workspace`
    (allocated when None) and returns (dks, dvs, workspace), the summary
    gradients [B, H, nb, d] fp32 over the call's owned queries."""
    _need_cuda(q, k, v, out, lse, dout)
    B, N, H, d = _dims(params)
    nb = n_blocks(params)
    dks = torch.empty(B, H, nb, d, dtype=torch.float32, device=q.device) if dks is None else dks
    dvs = torch.empty(B, H, nb, d, dtype=torch.float32, device=q.device) if dvs is None else dvs
    if workspace is None:
        workspace = torch.empty(pack3d_backward_workspace_bytes(params), dtype=torch.uint8,
                                device=q.device)
    _need_cuda(dks, dvs, workspace)
    if ksum is not None:
        _need_cuda(ksum, vsum)
    _check(load().pack3d_backward_summary_grads(
        ctypes.byref(params), ctypes.byref(index.struct), _ptr(q), _ptr(k), _ptr(v), _ptr(out),
        _ptr(lse), _ptr(dout), _ptr(ksum), _ptr(vsum), _ptr(dks), _ptr(dvs), _ptr(workspace),
        ctypes.c_size_t(workspace.numel() * workspace.element_size()), _stream(stream)),
        "pack3d_backward_summary_grads")
    return dks, dvs, workspace


def pack3d_backward_from_summary_grads(params: Params, index: IndexBuffers, dks, dvs, workspace,
                                       dq, dk, dv, stream=None):
    """Second half: dq, dk, dv of the owned tokens from the staged workspace and
    the summary gradients of the whole volume."""
    _need_cuda(dks, dvs, workspace, dq, dk, dv)
    _check(load().pack3d_backward_from_summary_grads(
        ctypes.byref(params), ctypes.byref(index.struct), _ptr(dks), _ptr(dvs), _ptr(workspace),
        ctypes.c_size_t(workspace.numel() * workspace.element_size()), _ptr(dq), _ptr(dk),
        _ptr(dv), _stream(stream)), "pack3d_backward_from_summary_grads")
    return dq, dk, dv


NOALLOC_SCRATCH_BYTES = 32 << 20


def pack3d_backward_noalloc(params: Params, index: IndexBuffers, q, k, v, out, lse, dout,
                            dq=None, dk=None, dv=None, stream=None):
    """pack3d_backward without a workspace argument: the library's static
    device scratch array (NOALLOC_SCRATCH_BYTES) stands in for it.  Calls that
    overlap on the GPU share that array and race; the first call on a device
    looks the array up and should precede any stream capture."""
    _need_cuda(q, k, v, out, lse, dout)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _need_cuda(dq, dk, dv)
    _check(load().pack3d_backward_noalloc(ctypes.byref(params), ctypes.byref(index.struct),
                                          _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
                                          _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv),
                                          _stream(stream)), "pack3d_backward_noalloc")
    return dq, dk, dv


class Pack3D:
    """Convenience wrapper: one operator shape, its index, and the calls."""

    def __init__(self, shape, dtype=None, scale: float = 0.0, out_fp32: bool = False):
        self.params = make_params(shape, dtype, scale, out_fp32)
        self.index = None

    def build_index(self, coords, stream=None, check=True):
        self.index = pack3d_build_index(self.params, coords, self.index, stream)
        if check:
            st = pack3d_index_check(self.index, stream)
            _check(st, "pack3d_index_check")
        return self.index

    def forward(self, q, k, v, stream=None):
        ksum, vsum = pack3d_block_summaries(self.params, self.index, k, v, stream=stream)
        return pack3d_forward(self.params, self.index, q, k, v, ksum, vsum, stream=stream)

    def window_forward(self, q, k, v, stream=None):
        return pack3d_window_forward(self.params, self.index, q, k, v, stream=stream)

    def backward(self, q, k, v, out, lse, dout, stream=None):
        return pack3d_backward(self.params, self.index, q, k, v, out, lse, dout, stream=stream)
