"""Float64 CPU oracle for block-causal ReLU linear attention with 3D RoPE.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may use this package; the product path
(``block_causal_linear_rope_b200``) never imports it, and this package never
imports the product.  The arithmetic lives in ``blin_oracle.c`` (plain C,
double precision, OpenMP over rows); this file only marshals numpy arrays.

Functions and the passages they follow (SANA-Video pages):
  grid            token -> (t, y, x) and block id (talk transcript, block-causal
                  walk-through; blocks of F latent frames)
  rope            3D RoPE rotation (talk transcript, 3D RoPE for linear attention)
  attention_rows  explicit O(N^2) masked double sum, RoPE in the numerator only
                  (talk transcript block cache; news article, positional
                  encoding paragraph)
  recurrence      state form S_i = S_{i-1} + block contribution, all rows
                  (talk transcript, state review)
  tconv           causal block temporal convolution with its one-frame cache
                  (talk transcript, causal-FFN passage)
  nvfp4_decode    NVFP4 block-scaled 4-bit values (news article, NVFP4 /
                  SVDQuant paragraph): E2M1 codes x E4M3 block scale x global

The RoPE pairing/frequency schedule is a reading of silent pages; it is pinned
to a library RoPE in the tests, not to the pages.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "blin_oracle.c")
_LIB = os.path.join(_HERE, "_blin_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle into a shared library next to its source."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        L = ctypes.c_long
        lib.blin_oracle_grid.argtypes = [L, L, L, L, L, P, P]
        lib.blin_oracle_grid.restype = None
        lib.blin_oracle_rope.argtypes = [P, P, ctypes.c_int, P, ctypes.c_double, P]
        lib.blin_oracle_rope.restype = None
        lib.blin_oracle_pairsum.argtypes = [P, P, P, L, P, P, P, P, L, L, ctypes.c_int, P,
                                            ctypes.c_double, P, P, ctypes.c_int]
        lib.blin_oracle_pairsum.restype = ctypes.c_int
        lib.blin_oracle_finish.argtypes = [P, P, L, ctypes.c_int, ctypes.c_double, P]
        lib.blin_oracle_finish.restype = None
        lib.blin_oracle_recurrence.argtypes = [P, P, P, P, P, L, L, ctypes.c_int, P,
                                               ctypes.c_double, ctypes.c_double, P, P, P, P, P,
                                               ctypes.c_int]
        lib.blin_oracle_recurrence.restype = ctypes.c_int
        lib.blin_oracle_tconv.argtypes = [P, P, P, P, L, L, L, L, L, L, P]
        lib.blin_oracle_tconv.restype = None
        lib.blin_oracle_e2m1.argtypes = [ctypes.c_int]
        lib.blin_oracle_e2m1.restype = ctypes.c_double
        lib.blin_oracle_e4m3.argtypes = [ctypes.c_int]
        lib.blin_oracle_e4m3.restype = ctypes.c_double
        lib.blin_oracle_nvfp4_decode.argtypes = [P, P, L, ctypes.c_int, ctypes.c_double, P]
        lib.blin_oracle_nvfp4_decode.restype = None
        _lib = lib
    return _lib


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _f32(x) -> np.ndarray:
    return np.ascontiguousarray(x, dtype=np.float32)


def _i64(x) -> np.ndarray:
    return np.ascontiguousarray(x, dtype=np.int64)


def _split(split: Sequence[int]) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(split, dtype=np.int32))


def grid(T: int, Hg: int, Wg: int, F: int, t0: int = 0):
    """Positions [N,3] (absolute t, y, x) and absolute block ids [N]."""
    N = T * Hg * Wg
    pos = np.zeros((N, 3), np.int64)
    blk = np.zeros((N,), np.int64)
    _load().blin_oracle_grid(T, Hg, Wg, F, t0, _p(pos), _p(blk))
    return pos, blk


def rope(u, pos, split: Sequence[int], theta: float) -> np.ndarray:
    """R_p u for one position p=(t,y,x); u is a float64 d-vector."""
    u = np.ascontiguousarray(u, dtype=np.float64)
    out = np.empty_like(u)
    _load().blin_oracle_rope(_p(u), _p(out), u.shape[-1], _p(_split(split)), float(theta),
                             _p(_i64(pos)))
    return out


class PairSum:
    """Running explicit double sum for a fixed set of query rows.

    Keys may be fed in several calls, in ascending token order, so long
    sequences never need to be held whole.
    """

    def __init__(self, q, qpos, qblk, split, theta: float, nthreads: int = 0):
        self.q = _f32(q)
        self.BH, self.nq, self.d = self.q.shape
        self.qpos, self.qblk = _i64(qpos), _i64(qblk)
        self.split, self.theta, self.nthreads = _split(split), float(theta), nthreads
        self.num = np.zeros((self.BH, self.nq, self.d), np.float64)
        self.den = np.zeros((self.BH, self.nq), np.float64)

    def add_keys(self, k, v, kpos, kblk) -> None:
        k, v = _f32(k), _f32(v)
        assert k.shape == v.shape and k.shape[0] == self.BH and k.shape[2] == self.d
        rc = _load().blin_oracle_pairsum(
            _p(self.q), _p(self.qpos), _p(self.qblk), self.nq, _p(k), _p(v), _p(_i64(kpos)),
            _p(_i64(kblk)), k.shape[1], self.BH, self.d, _p(self.split), self.theta,
            _p(self.num), _p(self.den), self.nthreads)
        if rc != 0:
            raise MemoryError("oracle pair sum: allocation failed")

    def result(self, eps: float) -> np.ndarray:
        out = np.empty_like(self.num)
        _load().blin_oracle_finish(_p(self.num), _p(self.den), self.BH * self.nq, self.d,
                                   float(eps), _p(out))
        return out


def attention_rows(q, k, v, pos, blk, rows, split, theta: float, eps: float,
                   nthreads: int = 0) -> np.ndarray:
    """Explicit O(N^2) block-causal sum for the query rows ``rows`` of one call.

    q, k, v: [BH, N, d] (or [B, H, N, d]) float32 values.  Returns [BH, len(rows), d].
    """
    q, k, v = (np.asarray(a) for a in (q, k, v))
    d = q.shape[-1]
    q = q.reshape(-1, q.shape[-2], d)
    k = k.reshape(-1, k.shape[-2], d)
    v = v.reshape(-1, v.shape[-2], d)
    rows = _i64(rows)
    ps = PairSum(q[:, rows, :], pos[rows], blk[rows], split, theta, nthreads)
    ps.add_keys(k, v, pos, blk)
    return ps.result(eps)


def recurrence(q, k, v, pos, blk, split, theta: float, eps: float, S_in=None, z_in=None,
               nthreads: int = 0):
    """State-form oracle over all rows.  Returns (out [BH,N,d], S [BH,d,d], z [BH,d])."""
    q, k, v = (np.asarray(a) for a in (q, k, v))
    d = q.shape[-1]
    N = q.shape[-2]
    q = _f32(q.reshape(-1, N, d))
    k = _f32(k.reshape(-1, N, d))
    v = _f32(v.reshape(-1, N, d))
    BH = q.shape[0]
    out = np.zeros((BH, N, d), np.float64)
    S_out = np.zeros((BH, d, d), np.float64)
    z_out = np.zeros((BH, d), np.float64)
    S_in = None if S_in is None else np.ascontiguousarray(S_in, dtype=np.float64).reshape(BH, d, d)
    z_in = None if z_in is None else np.ascontiguousarray(z_in, dtype=np.float64).reshape(BH, d)
    rc = _load().blin_oracle_recurrence(_p(q), _p(k), _p(v), _p(_i64(pos)), _p(_i64(blk)), BH, N,
                                        d, _p(_split(split)), float(theta), float(eps), _p(S_in),
                                        _p(z_in), _p(out), _p(S_out), _p(z_out), nthreads)
    if rc != 0:
        raise MemoryError("oracle recurrence: allocation failed")
    return out, S_out, z_out


def tconv(x, w, bias, F: int, t0: int = 0, prev=None):
    """Causal block temporal convolution over frames t0 .. t0+T-1.

    x: [B, T, HW, C] values (float32); w: [C, 3] taps (previous, current, next);
    bias: [C] or None; prev: [B, HW, C] previous frame (the cache) or None.
    Returns (y [B, T, HW, C] float64, the call's last frame [B, HW, C] float64)."""
    x = _f32(x)
    B, T, HW, C = x.shape
    w = np.ascontiguousarray(w, dtype=np.float64).reshape(C, 3)
    bias = None if bias is None else np.ascontiguousarray(bias, dtype=np.float64).reshape(C)
    prev = None if prev is None else np.ascontiguousarray(prev, dtype=np.float64).reshape(B, HW, C)
    y = np.zeros((B, T, HW, C), np.float64)
    _load().blin_oracle_tconv(_p(x), _p(prev), _p(w), _p(bias), B, T, HW, C, int(t0), int(F), _p(y))
    last = x[:, -1].astype(np.float64) if T > 0 else prev
    return y, last


def e2m1(code: int) -> float:
    return float(_load().blin_oracle_e2m1(int(code)))


def e4m3(code: int) -> float:
    return float(_load().blin_oracle_e4m3(int(code)))


def nvfp4_decode(data, scale, d: int, global_scale: float) -> np.ndarray:
    """data [..., d/2] uint8, scale [..., d/16] uint8 -> float64 values [..., d]."""
    data = np.ascontiguousarray(data, dtype=np.uint8)
    scale = np.ascontiguousarray(scale, dtype=np.uint8)
    lead = data.shape[:-1]
    rows = int(np.prod(lead)) if lead else 1
    out = np.empty(lead + (d,), np.float64)
    _load().blin_oracle_nvfp4_decode(_p(data), _p(scale), rows, int(d), float(global_scale), _p(out))
    return out


def exact_f32(x64: np.ndarray) -> np.ndarray:
    """float32 copy of float64 values that float32 holds exactly (raises otherwise), for the
    float32-input oracle routines."""
    x32 = np.ascontiguousarray(x64, dtype=np.float32)
    if not np.array_equal(x32.astype(np.float64), x64):
        raise ValueError("values are not exact in float32")
    return x32
