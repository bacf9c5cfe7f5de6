"""Shared helpers for the GPU parity tests: run the CUDA path, run the oracle, compare."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import workloads

TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16}
# max|o - o_ref| / max|o_ref| bounds: fp32 storage on CUDA cores, bf16 storage
# with fp32 accumulation on tensor cores.
TOL = {"f32": 1e-4, "bf16": 2e-2}


def dev(x: np.ndarray, dtype: str) -> torch.Tensor:
    """Exact device copy (bf16 workloads already hold bf16-representable values)."""
    return torch.from_numpy(np.ascontiguousarray(x)).to(device="cuda", dtype=TORCH_DT[dtype])


def host(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy()


def rel_err(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.abs(got - ref).max() / max(np.abs(ref).max(), 1e-300))


def run_prefill(blin, w: workloads.Workload, q, k, v, state=None) -> np.ndarray:
    o = blin.prefill(dev(q, w.dtype), dev(k, w.dtype), dev(v, w.dtype), grid=(w.T, w.Hg, w.Wg),
                     block_frames=w.F, rope_split=w.split, theta=w.theta, eps=w.eps, state=state)
    torch.cuda.synchronize()
    return host(o)


def oracle_all_rows(w: workloads.Workload, q, k, v, S=None, z=None):
    """State-form oracle over every row of a call (positions from the grid)."""
    pos, blk = oracle.grid(w.T, w.Hg, w.Wg, w.F, w.t0)
    return oracle.recurrence(q, k, v, pos, blk, w.split, w.theta, w.eps, S, z)


def sample_rows(w: workloads.Workload, per_block: int = 8, seed: int = 0) -> np.ndarray:
    """First and last token of every block plus `per_block` seeded rows per block."""
    rng = np.random.default_rng([seed, 99])
    rows = []
    tok = 0
    for (f0, f1) in w.block_frame_ranges():
        n = (f1 - f0) * w.HW
        rows += [tok, tok + n - 1]
        rows += list(tok + rng.integers(0, n, size=min(per_block, n)))
        tok += n
    return np.unique(np.array(rows, dtype=np.int64))
