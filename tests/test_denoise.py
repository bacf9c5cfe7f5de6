"""Denoising loop on one block: K read-only block steps, then one commit.

Talk transcript, hybrid autoregressive + diffusion passage: video is generated
block by block, and each block is denoised over several steps; block-cache
walk-through: the cache takes a block's contribution once that block's
computation is finished.  So every denoising step reads the cache of the
earlier blocks plus the step's own (noisy) block, and only the finished block
is added to the cache.  Each step's K and V are new, so each step recomputes
its block's contribution.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from _support import TOL, dev, host, rel_err

pytestmark = pytest.mark.gpu

K_STEPS = 4


@pytest.fixture(scope="module")
def blin():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import block_causal_linear_rope_b200 as m
    yield m
    assert m.device_status() == 0, "a kernel wait ran out"


def _block(w, t0, seed):
    return workloads.call_tensors(w.with_(T=w.F, t0=t0, seed=seed))


def _oracle_step(w, q, k, v, t0, S, z):
    pos, blk = oracle.grid(w.F, w.Hg, w.Wg, w.F, t0)
    return oracle.recurrence(q, k, v, pos, blk, w.split, w.theta, w.eps, S, z)


@pytest.mark.parametrize("d", [32, 64])
def test_denoise_steps_then_commit(blin, d):
    split = (8, 12, 12) if d == 32 else (16, 24, 24)
    w = workloads.Workload("denoise", B=1, H=6, d=d, dtype="bf16", T=9, Hg=30, Wg=52, F=3, split=split, seed=21)
    st = blin.BlockState(w.B, w.H, w.d)
    S_o = z_o = None
    # two finished blocks in the cache (oracle cache built by the oracle alone)
    for b in range(2):
        q, k, v = _block(w, 3 * b, w.seed)
        blin.block_step(dev(q, "bf16"), dev(k, "bf16"), dev(v, "bf16"), w.Hg, w.Wg, 3, w.split, st,
                        theta=w.theta, eps=w.eps, block_frames=w.F)
        _, S_o, z_o = _oracle_step(w, q, k, v, 3 * b, S_o, z_o)
    S_prev, z_prev = st.to_host()
    # K denoising steps of block 2: fresh Q, K, V each step, cache read only
    for s in range(K_STEPS):
        q, k, v = _block(w, 6, 1000 + s)
        o = blin.block_step(dev(q, "bf16"), dev(k, "bf16"), dev(v, "bf16"), w.Hg, w.Wg, 3, w.split, st,
                            theta=w.theta, eps=w.eps, commit=False, block_frames=w.F)
        ref, _, _ = _oracle_step(w, q, k, v, 6, S_o, z_o)
        assert rel_err(host(o).reshape(ref.shape), ref) <= TOL["bf16"], f"denoise step {s}"
        S_s, z_s = st.to_host()
        assert torch.equal(S_s, S_prev) and torch.equal(z_s, z_prev) and st.t_next == 6
    # the finished block is committed once
    q, k, v = _block(w, 6, w.seed)
    o_c = blin.block_step(dev(q, "bf16"), dev(k, "bf16"), dev(v, "bf16"), w.Hg, w.Wg, 3, w.split, st,
                          theta=w.theta, eps=w.eps, block_frames=w.F)
    S_c, z_c = st.to_host()
    assert st.t_next == 9
    # same cache, one committed step and no denoising steps: identical bits
    st2 = blin.BlockState(w.B, w.H, w.d)
    st2.from_host(S_prev, z_prev, 6)
    o_2 = blin.block_step(dev(q, "bf16"), dev(k, "bf16"), dev(v, "bf16"), w.Hg, w.Wg, 3, w.split, st2,
                          theta=w.theta, eps=w.eps, block_frames=w.F)
    S_2, z_2 = st2.to_host()
    assert torch.equal(o_c, o_2)
    assert torch.equal(S_c, S_2) and torch.equal(z_c, z_2)
    ref, S_ref, z_ref = _oracle_step(w, q, k, v, 6, S_o, z_o)
    assert rel_err(host(o_c).reshape(ref.shape), ref) <= TOL["bf16"]
    assert rel_err(S_c.numpy().reshape(S_ref.shape), S_ref) <= 5e-3
    assert rel_err(z_c.numpy().reshape(z_ref.shape), z_ref) <= 1e-5


def test_denoise_loop_replays_as_a_cuda_graph(blin):
    """K read-only steps plus the commit, captured once and replayed: same bits as eager calls."""
    w = workloads.Workload("denoise-graph", B=1, H=4, d=32, dtype="bf16", T=3, Hg=30, Wg=52, F=3,
                           split=(8, 12, 12), seed=5)
    steps = [tuple(dev(x, "bf16") for x in _block(w, 0, 50 + s)) for s in range(K_STEPS + 1)]
    outs = [torch.empty_like(steps[0][0]) for _ in steps]

    def loop(st):
        for s, (q, k, v) in enumerate(steps):
            blin.block_step(q, k, v, w.Hg, w.Wg, 3, w.split, st, theta=w.theta, eps=w.eps,
                            commit=s == K_STEPS, out=outs[s], block_frames=w.F)

    st_e = blin.BlockState(w.B, w.H, w.d)
    loop(st_e)
    torch.cuda.synchronize()
    eager = [o.clone() for o in outs]
    S_e, z_e = st_e.to_host()
    st_g = blin.BlockState(w.B, w.H, w.d)
    st_g.reserve(3 * w.HW)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        loop(st_g)
    # capture recorded the commit's t_next advance on the host; start the replay from frame 0
    st_g.reset()
    torch.cuda.synchronize()
    g.replay()
    torch.cuda.synchronize()
    for a, b in zip(outs, eager):
        assert torch.equal(a, b)
    S_g, z_g = st_g.to_host()
    assert torch.equal(S_g, S_e) and torch.equal(z_g, z_e)
    del g
