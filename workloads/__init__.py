"""Seeded synthetic workloads for block-causal linear attention with 3D RoPE.

This module only draws random numbers and changes number formats (float32 ->
bfloat16 with round-to-nearest-even).  It holds none of the attention
arithmetic, so both the CUDA path and the float64 oracle can take their inputs
from it without sharing any of the method.

Generator: ``numpy.random.default_rng([seed, tensor_id, block_id])`` with
tensor ids Q=0, K=1, V=2, Q-scale=3, K-scale=4.  Each latent block of ``F``
frames is drawn from its own stream, so a long autoregressive run can be
regenerated one block at a time and a one-shot prefill is the concatenation of
the same per-block draws.

Shapes follow the SANA-Video pages: latent grids of 21 frames at 30x52 (480p)
and 45x80 (720p), blocks of 3 latent frames, 70 heads of width 32; a
minute-long run streams 80 such blocks.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Optional, Tuple

import numpy as np

TENSOR_Q, TENSOR_K, TENSOR_V, TENSOR_QSCALE, TENSOR_KSCALE = 0, 1, 2, 3, 4
TENSOR_CONV_X, TENSOR_CONV_W, TENSOR_CONV_BIAS = 5, 6, 7
# The 4-bit E2M1 magnitudes, by code (bit 3 is the sign): a format definition.
E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], np.float32)


@dataclass(frozen=True)
class Workload:
    """One problem shape.  ``dtype`` is the storage type handed to the kernels."""

    name: str
    B: int
    H: int
    d: int
    dtype: str  # "f32" or "bf16"
    T: int
    Hg: int
    Wg: int
    F: int
    split: Tuple[int, int, int]
    theta: float = 10000.0
    eps: float = 1e-6
    dist: str = "normal"  # "normal" or "lognormal_qk"
    seed: int = 0
    t0: int = 0  # first absolute latent frame of this call
    steps: int = 1  # >1: streamed through block_step, one block per call

    @property
    def HW(self) -> int:
        return self.Hg * self.Wg

    @property
    def N(self) -> int:
        return self.T * self.HW

    def block_frame_ranges(self):
        """Absolute frame ranges [f0, f1) of the blocks this call touches."""
        out = []
        f = self.t0
        end = self.t0 + self.T
        while f < end:
            f1 = min((f // self.F + 1) * self.F, end)
            out.append((f, f1))
            f = f1
        return out

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


CONFIGS = {
    # Tiny case the O(N^2) oracle finishes instantly; also streamed 4x.
    "tiny": Workload("tiny", B=1, H=2, d=32, dtype="f32", T=12, Hg=4, Wg=4, F=3,
                     split=(8, 12, 12)),
    # 480p-like prefill: 21 x 30 x 52 latent, 7 blocks of 3 frames.
    "480p": Workload("480p", B=1, H=70, d=32, dtype="bf16", T=21, Hg=30, Wg=52, F=3,
                     split=(8, 12, 12)),
    # 720p-like prefill with per-channel lognormal Q/K scales.
    "720p": Workload("720p", B=1, H=70, d=32, dtype="bf16", T=21, Hg=45, Wg=80, F=3,
                     split=(8, 12, 12), dist="lognormal_qk"),
    # Minute-long decode: 80 calls of one 3-frame block (T=240 in total).
    "decode": Workload("decode", B=1, H=70, d=32, dtype="bf16", T=240, Hg=30, Wg=52, F=3,
                       split=(8, 12, 12), steps=80),
    # Wider heads, batched, one-frame blocks.
    "wide": Workload("wide", B=4, H=32, d=64, dtype="bf16", T=21, Hg=30, Wg=52, F=1,
                     split=(16, 24, 24)),
}


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (round to nearest, ties to even); returns uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = ((u >> 16) & 1) + 0x7FFF
    return ((u + r) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to float32."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _normal(seed: int, tensor_id: int, block_id: int, shape) -> np.ndarray:
    rng = np.random.default_rng([seed, tensor_id, block_id])
    return rng.standard_normal(size=shape, dtype=np.float32)


def channel_scales(w: Workload, tensor_id: int) -> Optional[np.ndarray]:
    """Per-(batch, head, channel) lognormal(0,1) factors, fixed over tokens."""
    if w.dist != "lognormal_qk" or tensor_id not in (TENSOR_Q, TENSOR_K):
        return None
    sid = TENSOR_QSCALE if tensor_id == TENSOR_Q else TENSOR_KSCALE
    rng = np.random.default_rng([w.seed, sid, 0])
    return rng.lognormal(0.0, 1.0, size=(w.B, w.H, 1, w.d)).astype(np.float32)


def block_tensor(w: Workload, tensor_id: int, block_id: int, frames: int) -> np.ndarray:
    """Draw one block's tensor [B, H, frames*Hg*Wg, d] in float32 storage values.

    For bf16 workloads the returned float32 values are exactly the bfloat16
    values handed to the GPU.
    """
    shape = (w.B, w.H, frames * w.HW, w.d)
    x = _normal(w.seed, tensor_id, block_id, shape)
    sc = channel_scales(w, tensor_id)
    if sc is not None:
        x = x * sc
    if w.dtype == "bf16":
        x = bf16_bits_to_f32(f32_to_bf16_bits(x))
    return x


def call_tensors(w: Workload):
    """Q, K, V for one call covering frames [t0, t0+T): [B,H,N,d] float32 values.

    Blocks are keyed by their absolute block index t // F, so a prefill and a
    block-by-block stream of the same frames see identical values.
    """
    out = []
    for tid in (TENSOR_Q, TENSOR_K, TENSOR_V):
        parts = [block_tensor(w, tid, f0 // w.F, f1 - f0) for (f0, f1) in w.block_frame_ranges()]
        out.append(np.ascontiguousarray(np.concatenate(parts, axis=2)) if parts else
                   np.zeros((w.B, w.H, 0, w.d), np.float32))
    return tuple(out)


def as_storage(x: np.ndarray, dtype: str) -> np.ndarray:
    """Storage array for the kernels: float32 as is, bf16 as uint16 bit patterns."""
    if dtype == "f32":
        return np.ascontiguousarray(x, dtype=np.float32)
    return f32_to_bf16_bits(x)


# ----------------------------------------------------------------------------- temporal convolution
@dataclass(frozen=True)
class ConvWorkload:
    """Causal block temporal convolution of the Mix-FFN: tokens [B, T*Hg*Wg, C] of
    C channels (channels innermost), blocks of F frames.  C defaults to the
    attention's width (70 heads x 32); the pages do not state the FFN's own."""

    name: str
    B: int
    C: int
    T: int
    Hg: int
    Wg: int
    F: int
    dtype: str = "bf16"
    seed: int = 0
    t0: int = 0

    @property
    def HW(self) -> int:
        return self.Hg * self.Wg

    @property
    def N(self) -> int:
        return self.T * self.HW

    def with_(self, **kw) -> "ConvWorkload":
        return replace(self, **kw)


CONV_CONFIGS = {
    "conv-tiny": ConvWorkload("conv-tiny", B=2, C=16, T=7, Hg=3, Wg=5, F=3, dtype="f32"),
    "conv-480p": ConvWorkload("conv-480p", B=1, C=2240, T=21, Hg=30, Wg=52, F=3),
}


def conv_tensors(w: ConvWorkload):
    """x [B, T, HW, C] (one stream per frame, keyed by the absolute frame), taps [C, 3]
    and bias [C] (float32 values; x bf16-representable for bf16 workloads)."""
    frames = []
    for t in range(w.t0, w.t0 + w.T):
        x = _normal(w.seed, TENSOR_CONV_X, t, (w.B, 1, w.HW, w.C))
        if w.dtype == "bf16":
            x = bf16_bits_to_f32(f32_to_bf16_bits(x))
        frames.append(x)
    x = np.ascontiguousarray(np.concatenate(frames, axis=1)) if frames else np.zeros((w.B, 0, w.HW, w.C), np.float32)
    taps = 0.5 * _normal(w.seed, TENSOR_CONV_W, 0, (w.C, 3))
    bias = 0.1 * _normal(w.seed, TENSOR_CONV_BIAS, 0, (w.C,))
    return x, taps, bias


# ----------------------------------------------------------------------------- NVFP4 inputs
def nvfp4_encode(x: np.ndarray, global_scale: float):
    """Quantise float32 [..., d] to NVFP4: per 16 consecutive elements an E4M3 scale
    (the block's max |x| / (6 * global), rounded to E4M3 by torch), then each element
    x / (scale * global) rounded to the nearest E2M1 value (ties to the even code).
    Returns (data [..., d/2] uint8, even elements in the low nibble;
    scale [..., d/16] uint8).  A number-format conversion of the inputs only."""
    import torch
    x = np.ascontiguousarray(x, dtype=np.float32)
    d = x.shape[-1]
    blocks = x.reshape(x.shape[:-1] + (d // 16, 16))
    amax = np.abs(blocks).max(axis=-1)
    s_f = (amax / (6.0 * global_scale)).astype(np.float32)
    s_t = torch.from_numpy(s_f).to(torch.float8_e4m3fn)
    scale = s_t.view(torch.uint8).numpy().copy()
    s_val = s_t.float().numpy().astype(np.float64)
    denom = s_val[..., None] * float(global_scale)
    v = np.divide(blocks, denom, out=np.zeros(blocks.shape, np.float64), where=denom > 0)
    mag = np.minimum(np.abs(v), 6.0)
    grid = E2M1_GRID.astype(np.float64)
    dist = np.abs(mag[..., None] - grid)
    idx = np.argmin(dist, axis=-1)  # the lower code on a tie between neighbours
    nxt = np.minimum(idx + 1, 7)
    tie_up = (idx % 2 == 1) & (np.take_along_axis(dist, nxt[..., None], -1)[..., 0] == np.take_along_axis(dist, idx[..., None], -1)[..., 0])
    idx = np.where(tie_up, nxt, idx)  # ties go to the even code
    code = (idx | np.where((v < 0) & (idx > 0), 8, 0)).astype(np.uint8).reshape(x.shape)
    data = (code[..., 0::2] | (code[..., 1::2] << 4)).astype(np.uint8)
    return data, scale


def nvfp4_global_scale(x: np.ndarray) -> float:
    """A power-of-two global scale putting the largest block scale near E4M3's top (448):
    powers of two keep every dequantised value exact in float32 and bfloat16."""
    amax = float(np.abs(x).max())
    if amax == 0.0:
        return 1.0
    return float(2.0 ** np.ceil(np.log2(amax / (6.0 * 448.0))))


def nvfp4_call_tensors(w: Workload):
    """Q, K, V of a call as NVFP4: ((data, scale, global) x 3), drawn like call_tensors in float32
    and then quantised; one global scale per tensor."""
    out = []
    w32 = w.with_(dtype="f32")
    for x in call_tensors(w32):
        g = nvfp4_global_scale(x)
        data, scale = nvfp4_encode(x, g)
        out.append((data, scale, g))
    return tuple(out)
