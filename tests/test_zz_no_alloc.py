"""blin_prefill_static: prefill for callers that cannot allocate device memory.

Some callers have no device allocator of their own (for example a plugin in a
host framework that owns all device memory), so they cannot hand blin_prefill
a workspace.  blin_prefill_static runs the same computation with a fixed
scratch area inside the library.  This file is named to be collected last.
The test calls the new entry point through the C ABI twice in a row, first on
the 480p workload and then on a smaller shape (so the second call runs over
the first call's leftovers in the shared scratch), and checks each result
against blin_prefill with a caller-provided workspace: the same kernels on the
same inputs, so the outputs must agree bit for bit.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads
from _support import TOL, dev, host, rel_err

pytestmark = pytest.mark.gpu


def _call_static(blin, w, q, k, v, out):
    g = blin._geom(w.T, w.Hg, w.Wg, w.F, w.split, w.theta, w.eps)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return blin.lib.blin_prefill_static(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                                        ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(out.data_ptr()),
                                        blin.BF16 if w.dtype == "bf16" else blin.F32, w.B, w.H, w.d,
                                        ctypes.byref(g), None, stream)


def test_static_scratch_prefill_matches_workspace_prefill_twice():
    assert torch.cuda.is_available()
    import block_causal_linear_rope_b200 as blin

    assert blin.lib.blin_prefill_static_capacity() == 32 << 20
    big = workloads.CONFIGS["480p"].with_(seed=3)
    small = workloads.Workload("small", B=1, H=5, d=32, dtype="bf16", T=7, Hg=9, Wg=21, F=3, split=(8, 12, 12), seed=4)
    for w in (big, small):  # two calls in a row: the second reuses the first one's scratch contents
        assert blin.workspace_size(w.B, w.H, w.d, (w.T, w.Hg, w.Wg), w.F, w.split) <= 32 << 20
        q, k, v = workloads.call_tensors(w)
        qd, kd, vd = dev(q, w.dtype), dev(k, w.dtype), dev(v, w.dtype)
        out = torch.full_like(qd, float("nan"))
        rc = _call_static(blin, w, qd, kd, vd, out)
        assert rc == 0, blin.lib.blin_last_error().decode()
        want = blin.prefill(qd, kd, vd, (w.T, w.Hg, w.Wg), w.F, w.split, w.theta, w.eps)
        torch.cuda.synchronize()
        assert torch.equal(out, want), f"{w.name}: static-scratch prefill differs from blin_prefill"
        # and both are the method's result
        assert rel_err(host(out).reshape(-1, w.N, w.d)[:2], _oracle_two_heads(w, q, k, v)) <= TOL[w.dtype]


def _oracle_two_heads(w, q, k, v):
    import oracle
    pos, blk = oracle.grid(w.T, w.Hg, w.Wg, w.F)
    two = lambda x: np.ascontiguousarray(x.reshape(-1, w.N, w.d)[:2])
    ref, _, _ = oracle.recurrence(two(q), two(k), two(v), pos, blk, w.split, w.theta, w.eps)
    return ref


def test_static_scratch_rejects_shapes_beyond_capacity():
    import block_causal_linear_rope_b200 as blin

    w = workloads.CONFIGS["wide"]  # needs more scratch than the fixed area holds
    assert blin.workspace_size(w.B, w.H, w.d, (w.T, w.Hg, w.Wg), w.F, w.split) > 32 << 20
    x = torch.zeros(16, device="cuda", dtype=torch.bfloat16)
    rc = _call_static(blin, w, x, x, x, x)
    assert rc == -5  # BLIN_ERR_WORKSPACE, before any launch
    assert "static area holds" in blin.lib.blin_last_error().decode()
