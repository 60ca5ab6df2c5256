"""CPU fp64 oracle of the PACK3D operator (test infrastructure).

Thin ctypes wrapper around ``pack3d_oracle.c``.  Only the tests, the smoke
check and the benchmark's CPU-baseline leg use this package; the CUDA library
never does, and this package never touches the CUDA library.  Every numeric
step lives in the C file, which states the definition it follows.

Functions take a *shape* object with attributes ``B, H, d, Z, Y, X, window,
block, rope_base`` (and optionally ``scale``, ``rope_mode`` and ``n_tokens``)
and torch tensors or numpy arrays in packed order; bf16 inputs are passed as
their exact bit patterns, fp32 and fp64 as is.  Outputs are fp64 numpy arrays.
``n_tokens`` > 0 describes a partly occupied volume: every batch item holds
that many tokens at distinct voxels (coords [B, n_tokens, 3]); 0 or absent
means one token per voxel.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pack3d_oracle.c")
_LIB_DIR = os.path.join(_HERE, "_build")
_LIB = os.path.join(_LIB_DIR, "liboracle.so")

F32, BF16, F64 = 0, 1, 2
ERR = {0: "ok", -1: "bad argument", -2: "bad coordinates", -3: "out of memory"}


class Params(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("B", "H", "d", "Z", "Y", "X", "wz", "wy", "wx", "bz", "by", "bx")] + [
        ("base", ctypes.c_double), ("scale", ctypes.c_double), ("rope_mode", ctypes.c_int32),
        ("n_tokens", ctypes.c_int32)]

# rope_mode: 0 = axial RoPE on grid coordinates (PACK3D); 1 = one-dimensional
# RoPE on the packed position (the packed-sequence comparison mode)
ROPE_AXIAL, ROPE_PACKED = 0, 1


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain -O2, no fast-math) if needed."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        os.makedirs(_LIB_DIR, exist_ok=True)
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-std=c11", "-Wall", "-shared",
                               "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P = ctypes.POINTER
        vp, i64p = ctypes.c_void_p, P(ctypes.c_int64)
        _lib.oracle_volume.argtypes = [P(Params), vp, vp]
        _lib.oracle_build_index.argtypes = [P(Params), vp, ctypes.c_int, ctypes.c_int,
                                            ctypes.c_int, vp, vp, vp, vp, vp]
        _lib.oracle_rope.argtypes = [P(Params), vp, vp, ctypes.c_int, ctypes.c_int, vp]
        _lib.oracle_block_summaries.argtypes = [P(Params), vp, vp, vp, ctypes.c_int, vp, vp]
        _lib.oracle_forward.argtypes = [P(Params), vp, vp, vp, vp, ctypes.c_int, vp, vp,
                                        ctypes.c_int, vp, ctypes.c_int64, vp, vp]
        _lib.oracle_backward.argtypes = [P(Params), vp, vp, vp, vp, vp, ctypes.c_int,
                                         ctypes.c_int, vp, vp, vp]
        _lib.oracle_max_threads.restype = ctypes.c_int
    return _lib


def max_threads() -> int:
    return int(lib().oracle_max_threads())


def params(shape) -> Params:
    w, b = tuple(shape.window), tuple(shape.block)
    return Params(shape.B, shape.H, shape.d, shape.Z, shape.Y, shape.X, w[0], w[1], w[2],
                  b[0], b[1], b[2], float(shape.rope_base), float(getattr(shape, "scale", 0.0) or 0.0),
                  int(getattr(shape, "rope_mode", 0) or 0), int(getattr(shape, "n_tokens", 0) or 0))


def n_tokens(shape) -> int:
    """Tokens per batch item: n_tokens when the volume is partly occupied, else Z*Y*X."""
    return int(getattr(shape, "n_tokens", 0) or 0) or shape.Z * shape.Y * shape.X


def _as_input(x):
    """(numpy array kept alive, dtype code) for a tensor or array."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous()
            if x.dtype == torch.bfloat16:
                return x.view(torch.int16).numpy().view(np.uint16), BF16
            if x.dtype == torch.float32:
                return x.numpy(), F32
            if x.dtype == torch.float64:
                return x.numpy(), F64
            raise TypeError(x.dtype)
    except ImportError:  # pragma: no cover
        pass
    x = np.ascontiguousarray(x)
    if x.dtype == np.float32:
        return x, F32
    if x.dtype == np.float64:
        return x, F64
    if x.dtype == np.uint16:
        return x, BF16
    raise TypeError(x.dtype)


def _coords(c):
    try:
        import torch
        if isinstance(c, torch.Tensor):
            c = c.cpu().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(c, dtype=np.int16)


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(rc):
    if rc != 0:
        raise ValueError(f"oracle: {ERR.get(rc, rc)}")


def volume(shape, coords):
    c = _coords(coords)
    vol = np.empty((shape.B, shape.Z * shape.Y * shape.X), dtype=np.int32)
    _check(lib().oracle_volume(ctypes.byref(params(shape)), _ptr(c), _ptr(vol)))
    return vol


def build_index(shape, coords, tile=(4, 4, 8)):
    """vol, perm, tile_off, nbr_off, nbr (halo lists) for query tiles ``tile``
    (vol and nbr hold -1 at the empty voxels of a partly occupied volume, perm
    only the tokens present)."""
    c = _coords(coords)
    p = params(shape)
    V = shape.Z * shape.Y * shape.X
    nT = -(-shape.Z // tile[0]) * -(-shape.Y // tile[1]) * -(-shape.X // tile[2])
    vol = np.empty((shape.B, V), np.int32)
    perm = np.empty((shape.B, n_tokens(shape)), np.int32)
    toff = np.empty((shape.B, nT + 1), np.int32)
    noff = np.empty((shape.B, nT + 1), np.int64)
    _check(lib().oracle_build_index(ctypes.byref(p), _ptr(c), tile[0], tile[1], tile[2],
                                    _ptr(vol), _ptr(perm), _ptr(toff), _ptr(noff), None))
    nbr = np.empty((shape.B, int(noff[0, -1])), np.int32)
    _check(lib().oracle_build_index(ctypes.byref(p), _ptr(c), tile[0], tile[1], tile[2],
                                    _ptr(vol), _ptr(perm), _ptr(toff), _ptr(noff), _ptr(nbr)))
    return {"vol": vol, "perm": perm, "tile_off": toff, "nbr_off": noff, "nbr": nbr}


def rope(shape, coords, x, transpose=False):
    """R(c_i) x_i (or R(c_i)^T x_i) for every row, fp64 [B, N, H, d]."""
    c = _coords(coords)
    a, dt = _as_input(x)
    out = np.empty((shape.B, n_tokens(shape), shape.H, shape.d), np.float64)
    _check(lib().oracle_rope(ctypes.byref(params(shape)), _ptr(c), _ptr(a), dt,
                             int(bool(transpose)), _ptr(out)))
    return out


def block_summaries(shape, coords, k, v):
    """(kbar, vbar), fp64 [B, H, nb, d]: block means of rotated k and of v."""
    c = _coords(coords)
    ka, dt = _as_input(k)
    va, dt2 = _as_input(v)
    assert dt == dt2
    nb = (-(-shape.Z // shape.block[0])) * (-(-shape.Y // shape.block[1])) * (-(-shape.X // shape.block[2]))
    ks = np.empty((shape.B, shape.H, nb, shape.d), np.float64)
    vs = np.empty_like(ks)
    _check(lib().oracle_block_summaries(ctypes.byref(params(shape)), _ptr(c), _ptr(ka),
                                        _ptr(va), dt, _ptr(ks), _ptr(vs)))
    return ks, vs


def forward(shape, coords, q, k, v, sel=None, window_only=False, summaries=None):
    """Operator output.

    ``sel`` (int64 flat indices ``(b*H + h)*N + i``) picks queries; the result
    is then ``out [len(sel), d]`` and ``lse [len(sel)]``.  Without ``sel`` all
    queries are computed and returned as ``out [B, N, H, d]`` and ``lse [B, H, N]``.
    """
    c = _coords(coords)
    qa, dt = _as_input(q)
    ka, _ = _as_input(k)
    va, _ = _as_input(v)
    N = n_tokens(shape)
    full = sel is None
    if full:
        sel = np.arange(shape.B * shape.H * N, dtype=np.int64)
    sel = np.ascontiguousarray(sel, dtype=np.int64)
    if window_only:
        ks = vs = np.zeros(1, np.float64)
    else:
        ks, vs = summaries if summaries is not None else block_summaries(shape, coords, k, v)
        ks, vs = np.ascontiguousarray(ks, np.float64), np.ascontiguousarray(vs, np.float64)
    out = np.empty((sel.size, shape.d), np.float64)
    lse = np.empty(sel.size, np.float64)
    _check(lib().oracle_forward(ctypes.byref(params(shape)), _ptr(c), _ptr(qa), _ptr(ka),
                                _ptr(va), dt, _ptr(ks), _ptr(vs), int(bool(window_only)),
                                _ptr(sel), sel.size, _ptr(out), _ptr(lse)))
    if full:
        out = out.reshape(shape.B, shape.H, N, shape.d).transpose(0, 2, 1, 3).copy()
        lse = lse.reshape(shape.B, shape.H, N)
    return out, lse


def backward(shape, coords, q, k, v, dout, window_only=False):
    """(dq, dk, dv) of sum(dout * out), fp64 [B, N, H, d], packed order."""
    c = _coords(coords)
    qa, dt = _as_input(q)
    ka, _ = _as_input(k)
    va, _ = _as_input(v)
    da, _ = _as_input(dout)
    shp = (shape.B, n_tokens(shape), shape.H, shape.d)
    dq, dk, dv = (np.zeros(shp, np.float64) for _ in range(3))
    _check(lib().oracle_backward(ctypes.byref(params(shape)), _ptr(c), _ptr(qa), _ptr(ka),
                                 _ptr(va), _ptr(da), dt, int(bool(window_only)), _ptr(dq),
                                 _ptr(dk), _ptr(dv)))
    return dq, dk, dv


def flat_index(shape, b, h, i):
    """Flat query selector ``(b*H + h)*N + i`` used by :func:`forward`."""
    N = n_tokens(shape)
    return (np.asarray(b, np.int64) * shape.H + np.asarray(h, np.int64)) * N + np.asarray(i, np.int64)
