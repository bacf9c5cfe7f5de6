"""Strided Q/K/V/O (the QKV projection's own layout) against contiguous calls.

News article, SVDQuant paragraph: the QKV projections feed this attention.
A fused projection writes [B, N, 3, H, d]; reading Q, K and V in place (no
transpose into [B, H, N, d]) must give exactly the contiguous results.
"""
import numpy as np
import pytest
import torch

import workloads
from _support import TOL, dev, host, oracle_all_rows, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def blin():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import block_causal_linear_rope_b200 as m
    yield m
    assert m.device_status() == 0, "a kernel wait ran out"


def _fused_views(q, k, v):
    """Pack contiguous [B, H, N, d] q, k, v into one [B, N, 3, H, d] buffer; return it and
    its three [B, H, N, d] views."""
    B, H, N, d = q.shape
    buf = torch.stack([q, k, v], dim=0).permute(1, 3, 0, 2, 4).contiguous()  # [B, N, 3, H, d]
    views = [buf[:, :, i].permute(0, 2, 1, 3) for i in range(3)]
    return buf, views


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("d", [32, 64])
def test_fused_qkv_layout_prefill_is_bitwise_contiguous(blin, dtype, d):
    split = (8, 12, 12) if d == 32 else (16, 24, 24)
    w = workloads.Workload("strided", B=2, H=5, d=d, dtype=dtype, T=7, Hg=9, Wg=23, F=3, split=split, seed=17)
    q, k, v = (dev(x, dtype) for x in workloads.call_tensors(w))
    want = blin.prefill(q, k, v, (w.T, w.Hg, w.Wg), w.F, w.split, w.theta, w.eps)
    path = blin.last_path()
    buf, (qv, kv, vv) = _fused_views(q, k, v)
    assert not qv.is_contiguous()
    # output straight into a [B, N, H, d] buffer (the out projection's input layout)
    obuf = torch.full((w.B, w.N, w.H, w.d), float("nan"), device="cuda", dtype=q.dtype)
    got = blin.prefill(qv, kv, vv, (w.T, w.Hg, w.Wg), w.F, w.split, w.theta, w.eps, out=obuf.permute(0, 2, 1, 3))
    assert blin.last_path() == path
    torch.cuda.synchronize()
    assert torch.equal(got, want)
    assert torch.equal(obuf.permute(0, 2, 1, 3), want)
    ref, _, _ = oracle_all_rows(w, *workloads.call_tensors(w))
    assert rel_err(host(want).reshape(-1, w.N, w.d), ref) <= TOL[dtype]


def test_fused_qkv_layout_block_steps(blin):
    w = workloads.Workload("strided-steps", B=1, H=6, d=32, dtype="bf16", T=6, Hg=30, Wg=52, F=3, split=(8, 12, 12),
                           seed=19)
    q, k, v = (dev(x, "bf16") for x in workloads.call_tensors(w))
    st_a = blin.BlockState(w.B, w.H, w.d)
    want = blin.prefill(q, k, v, (w.T, w.Hg, w.Wg), w.F, w.split, w.theta, w.eps, state=st_a)
    st_b = blin.BlockState(w.B, w.H, w.d)
    outs = []
    for f0 in (0, 3):
        n0, n1 = f0 * w.HW, (f0 + 3) * w.HW
        _, (qv, kv, vv) = _fused_views(q[:, :, n0:n1], k[:, :, n0:n1], v[:, :, n0:n1])
        outs.append(blin.block_step(qv, kv, vv, w.Hg, w.Wg, 3, w.split, st_b, theta=w.theta, eps=w.eps,
                                    block_frames=w.F))
    torch.cuda.synchronize()
    assert torch.equal(torch.cat(outs, dim=2), want)
    Sa, za = st_a.to_host()
    Sb, zb = st_b.to_host()
    assert torch.equal(Sa, Sb) and torch.equal(za, zb)
