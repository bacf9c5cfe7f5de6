"""NVFP4 Q/K/V through the tensor-core kernels (news article, NVFP4 / SVDQuant paragraph).

The kernels decode the 4-bit values in shared memory and apply the global
scales in fp32.  With power-of-two global scales every step scales exactly,
so the outputs must equal, bit for bit, those of the bf16 path on the decoded
values; and they must match the float64 oracle run on the decoded values.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from _support import TOL, dev, host, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def blin():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import block_causal_linear_rope_b200 as m
    yield m
    assert m.device_status() == 0, "a kernel wait ran out"


def _inputs(blin, w):
    """Device NVFP4 operands and the decoded float64 values of q, k, v."""
    ops, dec = [], []
    for data, scale, g in workloads.nvfp4_call_tensors(w):
        ops.append(blin.Nvfp4Tensor(torch.from_numpy(data), torch.from_numpy(scale), g))
        dec.append(oracle.nvfp4_decode(data, scale, w.d, g))
    return ops, dec


@pytest.mark.parametrize("d", [32, 64])
def test_nvfp4_prefill_matches_bf16_path_and_oracle(blin, d):
    split = (8, 12, 12) if d == 32 else (16, 24, 24)
    w = workloads.Workload("nvfp4", B=2, H=3, d=d, dtype="bf16", T=7, Hg=9, Wg=23, F=3, split=split, seed=29)
    (q4, k4, v4), dec = _inputs(blin, w)
    got = blin.prefill_nvfp4(q4, k4, v4, (w.T, w.Hg, w.Wg), w.F, w.split, w.theta, w.eps)
    q, k, v = (oracle.exact_f32(x) for x in dec)
    want = blin.prefill(dev(q, "bf16"), dev(k, "bf16"), dev(v, "bf16"), (w.T, w.Hg, w.Wg), w.F, w.split,
                        w.theta, w.eps)
    torch.cuda.synchronize()
    assert torch.equal(got, want), "NVFP4 path differs from the bf16 path on the decoded values"
    pos, blk = oracle.grid(w.T, w.Hg, w.Wg, w.F)
    ref, _, _ = oracle.recurrence(q, k, v, pos, blk, w.split, w.theta, w.eps)
    assert rel_err(host(got).reshape(ref.shape), ref) <= TOL["bf16"]


def test_nvfp4_480p_bitwise_bf16_path(blin):
    w = workloads.CONFIGS["480p"].with_(seed=31)
    (q4, k4, v4), dec = _inputs(blin, w)
    st_a, st_b = blin.BlockState(w.B, w.H, w.d), blin.BlockState(w.B, w.H, w.d)
    got = blin.prefill_nvfp4(q4, k4, v4, (w.T, w.Hg, w.Wg), w.F, w.split, w.theta, w.eps, state=st_a)
    q, k, v = (dev(oracle.exact_f32(x), "bf16") for x in dec)
    want = blin.prefill(q, k, v, (w.T, w.Hg, w.Wg), w.F, w.split, w.theta, w.eps, state=st_b)
    torch.cuda.synchronize()
    assert torch.equal(got, want)
    Sa, za = st_a.to_host()
    Sb, zb = st_b.to_host()
    assert torch.equal(Sa, Sb) and torch.equal(za, zb)


def test_nvfp4_block_steps_equal_prefill(blin):
    w = workloads.Workload("nvfp4-steps", B=1, H=5, d=32, dtype="bf16", T=9, Hg=30, Wg=52, F=3, split=(8, 12, 12),
                           seed=37)
    (q4, k4, v4), _ = _inputs(blin, w)
    st_a = blin.BlockState(w.B, w.H, w.d)
    full = blin.prefill_nvfp4(q4, k4, v4, (w.T, w.Hg, w.Wg), w.F, w.split, w.theta, w.eps, state=st_a)
    st_b = blin.BlockState(w.B, w.H, w.d)
    outs = []
    for f0 in range(0, w.T, w.F):
        n0, n1 = f0 * w.HW, (f0 + w.F) * w.HW
        part = [blin.Nvfp4Tensor(x.data[:, :, n0:n1], x.scale[:, :, n0:n1], x.global_scale) for x in (q4, k4, v4)]
        outs.append(blin.block_step_nvfp4(*part, w.Hg, w.Wg, w.F, w.split, st_b, theta=w.theta, eps=w.eps,
                                          block_frames=w.F))
    torch.cuda.synchronize()
    assert torch.equal(torch.cat(outs, dim=2), full)
    Sa, za = st_a.to_host()
    Sb, zb = st_b.to_host()
    assert torch.equal(Sa, Sb) and torch.equal(za, zb)


def test_nvfp4_needs_the_tensor_core_path(blin):
    w = workloads.Workload("nvfp4-split", B=1, H=2, d=32, dtype="bf16", T=3, Hg=4, Wg=8, F=3, split=(16, 8, 8))
    (q4, k4, v4), _ = _inputs(blin, w)
    with pytest.raises(blin.BlinError, match="BLIN_ERR_SHAPE"):
        blin.prefill_nvfp4(q4, k4, v4, (w.T, w.Hg, w.Wg), w.F, w.split)
