"""CUDA path vs the float64 oracle, element by element, on seeded inputs.

Small grids run the whole O(N^2) pair sum; full-size workloads (480p, 720p,
wide, minute-long decode) are checked on every row against the oracle's state
form and on sampled rows against the explicit pair sum.  Bound:
max|o - o_ref| / max|o_ref| <= 1e-4 (fp32 storage) / 2e-2 (bf16 storage).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from _support import TOL, dev, host, oracle_all_rows, rel_err, run_prefill, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def blin():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import block_causal_linear_rope_b200 as m
    yield m
    assert m.device_status() == 0, "a kernel wait ran out"


def _pairsum_all(w, q, k, v):
    pos, blk = oracle.grid(w.T, w.Hg, w.Wg, w.F, w.t0)
    return oracle.attention_rows(q, k, v, pos, blk, np.arange(w.N), w.split, w.theta, w.eps)


# --------------------------------------------------------------------------- tiny
def test_tiny_fp32_prefill_matches_pair_sum(blin):
    w = workloads.CONFIGS["tiny"]
    q, k, v = workloads.call_tensors(w)
    got = run_prefill(blin, w, q, k, v).reshape(-1, w.N, w.d)
    ref = _pairsum_all(w, q, k, v)
    assert rel_err(got, ref) <= TOL["f32"]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_tiny_streamed_equals_prefill_bitwise(blin, dtype):
    w = workloads.CONFIGS["tiny"].with_(dtype=dtype)
    q, k, v = workloads.call_tensors(w)
    st_a = blin.BlockState(w.B, w.H, w.d)
    full = run_prefill(blin, w, q, k, v, state=st_a)
    st_b = blin.BlockState(w.B, w.H, w.d)
    outs = []
    for (f0, f1) in w.block_frame_ranges():
        qb, kb, vb = workloads.call_tensors(w.with_(t0=f0, T=f1 - f0))
        ob = blin.block_step(dev(qb, dtype), dev(kb, dtype), dev(vb, dtype), w.Hg, w.Wg, f1 - f0, w.split,
                             st_b, theta=w.theta, eps=w.eps, block_frames=w.F)
        outs.append(host(ob))
    streamed = np.concatenate(outs, axis=2)
    np.testing.assert_array_equal(streamed, full)
    Sa, za = st_a.to_host()
    Sb, zb = st_b.to_host()
    assert torch.equal(Sa, Sb) and torch.equal(za, zb)
    assert st_a.t_next == st_b.t_next == w.T
    ref, S_ref, z_ref = oracle_all_rows(w, q, k, v)
    assert rel_err(full.reshape(-1, w.N, w.d), ref) <= TOL[dtype]
    assert rel_err(Sa.numpy().reshape(S_ref.shape), S_ref) <= TOL[dtype] / 4
    assert rel_err(za.numpy().reshape(z_ref.shape), z_ref) <= 1e-6


# --------------------------------------------------------------------------- edge shapes
EDGE = [
    # (T, Hg, Wg, F): ragged 128-row tiles, tiny frames, single block, one token per block
    (7, 5, 37, 2), (5, 3, 3, 2), (4, 1, 1, 1), (3, 9, 14, 8), (9, 11, 13, 3), (2, 40, 40, 1),
]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("shape", EDGE)
@pytest.mark.parametrize("d", [32, 64])
def test_edge_shapes_match_oracle(blin, dtype, shape, d):
    T, Hg, Wg, F = shape
    split = (8, 12, 12) if d == 32 else (16, 24, 24)
    w = workloads.Workload("edge", B=2, H=3, d=d, dtype=dtype, T=T, Hg=Hg, Wg=Wg, F=F, split=split, seed=7)
    q, k, v = workloads.call_tensors(w)
    qd, kd, vd = dev(q, dtype), dev(k, dtype), dev(v, dtype)
    # canary rows after the output must survive
    pad = 300
    buf = torch.full((w.B * w.H * w.N + pad, d), 7.0, device="cuda", dtype=qd.dtype)
    out = buf[: w.B * w.H * w.N].view(w.B, w.H, w.N, d)
    blin.prefill(qd, kd, vd, grid=(T, Hg, Wg), block_frames=F, rope_split=split, theta=w.theta, eps=w.eps, out=out)
    torch.cuda.synchronize()
    assert bool((buf[w.B * w.H * w.N:] == 7.0).all()), "wrote past the output"
    got = host(out).reshape(-1, w.N, d)
    ref, _, _ = oracle_all_rows(w, q, k, v)
    assert rel_err(got, ref) <= TOL[dtype]


def test_unsupported_split_runs_on_cuda_cores(blin):
    """A RoPE split without a tensor-core variant still matches the oracle."""
    w = workloads.Workload("split", B=1, H=2, d=32, dtype="bf16", T=6, Hg=4, Wg=9, F=2, split=(16, 8, 8), seed=3)
    q, k, v = workloads.call_tensors(w)
    got = run_prefill(blin, w, q, k, v).reshape(-1, w.N, w.d)
    assert blin.last_path() == "cuda_core"
    ref, _, _ = oracle_all_rows(w, q, k, v)
    assert rel_err(got, ref) <= TOL["bf16"]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_zero_query_rows_give_exact_zero(blin, dtype):
    w = workloads.Workload("zq", B=1, H=2, d=32, dtype=dtype, T=4, Hg=6, Wg=10, F=2, split=(8, 12, 12))
    q, k, v = workloads.call_tensors(w)
    q[:, :, ::5, :] = -np.abs(q[:, :, ::5, :])
    got = run_prefill(blin, w, q, k, v)
    assert (got[:, :, ::5, :] == 0.0).all()


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_block_mask_is_exact(blin, dtype):
    """v_m = one-hot of its block: outputs of block b are exactly 0 in columns > b."""
    w = workloads.Workload("mask", B=1, H=2, d=32, dtype=dtype, T=11, Hg=7, Wg=9, F=2, split=(8, 12, 12))
    q, k, _ = workloads.call_tensors(w)
    pos, blk = oracle.grid(w.T, w.Hg, w.Wg, w.F)
    v = np.zeros_like(q)
    v[:, :, np.arange(w.N), blk] = 1.0
    st = blin.BlockState(w.B, w.H, w.d)
    got = run_prefill(blin, w, q, k, v, state=st)
    for n in range(0, w.N, 17):
        assert (got[:, :, n, blk[n] + 1:] == 0.0).all()
    # z after the call counts phi(k) exactly for 0/1 keys
    kk = np.zeros_like(k)
    kk[..., 0] = 1.0
    st2 = blin.BlockState(w.B, w.H, w.d)
    run_prefill(blin, w, q, kk, v, state=st2)
    _, z = st2.to_host()
    assert (z[..., 0] == w.N).all() and (z[..., 1:] == 0).all()


# --------------------------------------------------------------------------- cache semantics
def test_prefill_continuation_from_state(blin):
    """Two prefill calls through a cache, the second starting mid-block.

    Rows of the second call see the whole block (cache + own frames), so they
    equal the one-shot result; rows of the first call's unfinished block can
    only see the frames that exist so far, i.e. the one-shot result of the
    first call's frames alone.  The final cache equals the one-shot cache.
    """
    w = workloads.Workload("cont", B=1, H=4, d=32, dtype="bf16", T=10, Hg=6, Wg=11, F=3, split=(8, 12, 12), seed=5)
    q, k, v = workloads.call_tensors(w)
    ref, S_ref, z_ref = oracle_all_rows(w, q, k, v)
    st = blin.BlockState(w.B, w.H, w.d)
    T1 = 4
    n1 = T1 * w.HW
    w1, w2 = w.with_(T=T1), w.with_(T=w.T - T1, t0=T1)
    sl1, sl2 = (slice(None), slice(None), slice(0, n1)), (slice(None), slice(None), slice(n1, None))
    o1 = run_prefill(blin, w1, q[sl1], k[sl1], v[sl1], state=st)
    assert st.t_next == T1
    o2 = run_prefill(blin, w2, q[sl2], k[sl2], v[sl2], state=st)
    ref1, _, _ = oracle_all_rows(w1, q[sl1], k[sl1], v[sl1])
    assert rel_err(o1.reshape(-1, n1, w.d), ref1) <= TOL["bf16"]
    assert rel_err(o2.reshape(-1, w.N - n1, w.d), ref[:, n1:]) <= TOL["bf16"]
    assert st.t_next == w.T
    S, z = st.to_host()
    assert rel_err(S.numpy().reshape(S_ref.shape), S_ref) <= 5e-3
    assert rel_err(z.numpy().reshape(z_ref.shape), z_ref) <= 1e-5


def test_commit_zero_is_read_only(blin):
    w = workloads.Workload("c0", B=1, H=3, d=32, dtype="bf16", T=6, Hg=8, Wg=8, F=3, split=(8, 12, 12), seed=9)
    st = blin.BlockState(w.B, w.H, w.d)
    q0, k0, v0 = (dev(x, "bf16") for x in workloads.call_tensors(w.with_(T=3)))
    blin.block_step(q0, k0, v0, w.Hg, w.Wg, 3, w.split, st)
    S0, z0 = st.to_host()
    q1, k1, v1 = (dev(x, "bf16") for x in workloads.call_tensors(w.with_(T=3, t0=3)))
    a = host(blin.block_step(q1, k1, v1, w.Hg, w.Wg, 3, w.split, st, commit=False))
    S1, z1 = st.to_host()
    assert torch.equal(S0, S1) and torch.equal(z0, z1) and st.t_next == 3
    b = host(blin.block_step(q1, k1, v1, w.Hg, w.Wg, 3, w.split, st, commit=True))
    np.testing.assert_array_equal(a, b)
    assert st.t_next == 6


def test_checkpoint_resume_is_bitwise(blin):
    w = workloads.Workload("ck", B=1, H=5, d=32, dtype="bf16", T=12, Hg=10, Wg=13, F=3, split=(8, 12, 12), seed=11)
    blocks = [tuple(dev(x, "bf16") for x in workloads.call_tensors(w.with_(T=3, t0=3 * i))) for i in range(4)]
    st = blin.BlockState(w.B, w.H, w.d)
    ref = [host(blin.block_step(*b, w.Hg, w.Wg, 3, w.split, st)) for b in blocks]
    S_ref, z_ref = st.to_host()
    st1 = blin.BlockState(w.B, w.H, w.d)
    got = [host(blin.block_step(*b, w.Hg, w.Wg, 3, w.split, st1)) for b in blocks[:2]]
    S, z = st1.to_host()
    t = st1.t_next
    st1.free()
    st2 = blin.BlockState(w.B, w.H, w.d)
    st2.from_host(S, z, t)
    got += [host(blin.block_step(*b, w.Hg, w.Wg, 3, w.split, st2)) for b in blocks[2:]]
    for a, b in zip(got, ref):
        np.testing.assert_array_equal(a, b)
    S2, z2 = st2.to_host()
    assert torch.equal(S2, S_ref) and torch.equal(z2, z_ref)


# --------------------------------------------------------------------------- full-size workloads
def _full_size(blin, name, heads=None, per_block=4):
    w = workloads.CONFIGS[name]
    q, k, v = workloads.call_tensors(w)
    got = run_prefill(blin, w, q, k, v)
    hsel = slice(None) if heads is None else heads
    qs, ks, vs = (x.reshape(-1, w.N, w.d)[hsel] for x in (q, k, v))
    got = got.reshape(-1, w.N, w.d)[hsel]
    ref, _, _ = oracle.recurrence(qs, ks, vs, *oracle.grid(w.T, w.Hg, w.Wg, w.F), w.split, w.theta, w.eps)
    err = rel_err(got, ref)
    per_block = []
    tok = 0
    for (f0, f1) in w.block_frame_ranges():
        sl = slice(tok, tok + (f1 - f0) * w.HW)
        per_block.append(rel_err(got[:, sl], ref[:, sl]))
        tok = sl.stop
    print(f"{name}: max rel err {err:.3e}; per block {['%.1e' % e for e in per_block]}")
    assert err <= TOL[w.dtype]
    # explicit pair sum on sampled rows of the first two heads of the selection
    rows = sample_rows(w, per_block=2)
    pos, blk = oracle.grid(w.T, w.Hg, w.Wg, w.F)
    two = slice(0, 2)
    pr = oracle.attention_rows(qs[two], ks[two], vs[two], pos, blk, rows, w.split, w.theta, w.eps)
    assert rel_err(got[two][:, rows], pr) <= TOL[w.dtype]
    np.testing.assert_allclose(ref[two][:, rows], pr, rtol=1e-9, atol=1e-12 * np.abs(pr).max())


def test_480p_prefill(blin):
    _full_size(blin, "480p")


def test_720p_lognormal_prefill(blin):
    _full_size(blin, "720p")


def test_wide_d64_prefill(blin):
    _full_size(blin, "wide", heads=slice(0, 128, 8))


def test_minute_long_decode(blin):
    """80 blocks through block_step: constant memory, outputs vs the oracle on blocks 0, 1, 39, 79."""
    w = workloads.CONFIGS["decode"]
    heads = np.arange(0, w.H, 10)  # oracle on 7 of the 70 heads
    check = {0, 1, 39, 79}
    st = blin.BlockState(w.B, w.H, w.d)
    assert st.nbytes == 70 * (32 * 32 + 32) * 4 == 295680
    st.reserve(3 * w.HW)
    torch.cuda.synchronize()
    mem0 = None
    S_o = z_o = None
    worst = 0.0
    for blk_i in range(w.steps):
        wb = w.with_(T=3, t0=3 * blk_i)
        q, k, v = workloads.call_tensors(wb)
        o = blin.block_step(dev(q, "bf16"), dev(k, "bf16"), dev(v, "bf16"), w.Hg, w.Wg, 3, w.split, st,
                            theta=w.theta, eps=w.eps, block_frames=w.F)
        got = host(o)[0, heads]
        del o
        torch.cuda.synchronize()
        # free device memory as the driver sees it: counts the library's own
        # allocations (state, scratch), which PyTorch's allocator statistics do not
        mem = torch.cuda.mem_get_info()[0]
        mem0 = mem if mem0 is None else mem0
        assert mem == mem0, "device memory changed during decode"
        sub = lambda x: np.ascontiguousarray(x[0, heads])
        ref, S_o, z_o = oracle.recurrence(sub(q), sub(k), sub(v), *oracle.grid(3, w.Hg, w.Wg, w.F, 3 * blk_i),
                                          w.split, w.theta, w.eps, S_o, z_o)
        if blk_i in check:
            e = rel_err(got, ref)
            worst = max(worst, e)
            print(f"decode block {blk_i}: rel err {e:.3e}")
            assert e <= TOL["bf16"]
    assert st.t_next == 240
    S, z = st.to_host()
    assert rel_err(S.numpy()[0, heads], S_o) <= 5e-3
    assert rel_err(z.numpy()[0, heads], z_o) <= 1e-5


# --------------------------------------------------------------------------- bitwise streaming, multi-chunk blocks
def _stream_blocks(blin, w, qd, kd, vd, st):
    """Feed a prefill-shaped call block by block through block_step; returns the concatenated output."""
    outs = []
    for (f0, f1) in w.block_frame_ranges():
        n0, n1 = (f0 - w.t0) * w.HW, (f1 - w.t0) * w.HW
        outs.append(blin.block_step(qd[:, :, n0:n1].contiguous(), kd[:, :, n0:n1].contiguous(),
                                    vd[:, :, n0:n1].contiguous(), w.Hg, w.Wg, f1 - f0, w.split, st,
                                    theta=w.theta, eps=w.eps, block_frames=w.F))
    return torch.cat(outs, dim=2)


@pytest.mark.parametrize("name", ["480p", "wide"])
def test_full_size_streamed_equals_prefill_bitwise(blin, name):
    """Every block of the workload through block_step == one prefill, bit for bit (O, S, z).

    480p blocks are 4,680 tokens (several state chunks per block, reduced in a
    fixed order); the block steps also use smaller output groups than the
    prefill, which must not change any output bit.
    """
    w = workloads.CONFIGS[name]
    q, k, v = workloads.call_tensors(w)
    qd, kd, vd = dev(q, w.dtype), dev(k, w.dtype), dev(v, w.dtype)
    st_a = blin.BlockState(w.B, w.H, w.d)
    full = blin.prefill(qd, kd, vd, (w.T, w.Hg, w.Wg), w.F, w.split, w.theta, w.eps, state=st_a)
    assert blin.last_path() == "tensor_core"
    st_b = blin.BlockState(w.B, w.H, w.d)
    streamed = _stream_blocks(blin, w, qd, kd, vd, st_b)
    assert blin.last_path() == "tensor_core"
    torch.cuda.synchronize()
    assert torch.equal(streamed, full), "streamed block outputs differ from the prefill"
    Sa, za = st_a.to_host()
    Sb, zb = st_b.to_host()
    assert torch.equal(Sa, Sb) and torch.equal(za, zb), "streamed cache differs from the prefill's"
    assert st_a.t_next == st_b.t_next == w.T


def test_decode_block_through_prefill_state_bitwise(blin):
    """Prefill 3 decode-sized blocks into a cache, then block_step the 4th: the 4th block's rows
    and the final cache equal a one-shot prefill of all 4 blocks, bit for bit."""
    w = workloads.CONFIGS["decode"].with_(T=12, steps=1)
    q, k, v = workloads.call_tensors(w)
    qd, kd, vd = dev(q, "bf16"), dev(k, "bf16"), dev(v, "bf16")
    st_full = blin.BlockState(w.B, w.H, w.d)
    full = blin.prefill(qd, kd, vd, (w.T, w.Hg, w.Wg), w.F, w.split, w.theta, w.eps, state=st_full)
    n3 = 9 * w.HW
    st = blin.BlockState(w.B, w.H, w.d)
    head = blin.prefill(qd[:, :, :n3].contiguous(), kd[:, :, :n3].contiguous(), vd[:, :, :n3].contiguous(),
                        (9, w.Hg, w.Wg), w.F, w.split, w.theta, w.eps, state=st)
    last = blin.block_step(qd[:, :, n3:].contiguous(), kd[:, :, n3:].contiguous(), vd[:, :, n3:].contiguous(),
                           w.Hg, w.Wg, 3, w.split, st, theta=w.theta, eps=w.eps, block_frames=w.F)
    torch.cuda.synchronize()
    assert torch.equal(head, full[:, :, :n3])
    assert torch.equal(last, full[:, :, n3:])
    S1, z1 = st.to_host()
    S2, z2 = st_full.to_host()
    assert torch.equal(S1, S2) and torch.equal(z1, z2)
    # and the rows agree with the oracle
    ref, _, _ = oracle_all_rows(w, q, k, v)
    assert rel_err(host(full).reshape(-1, w.N, w.d), ref) <= TOL["bf16"]


def test_block_step_after_prefill_ending_mid_block(blin):
    """A prefill that stops inside a block, then block steps that finish it and go on.

    The block length is part of the call: a step whose frames would cross a
    block boundary is rejected (BLIN_ERR_SHAPE), the state untouched.  Steps
    that finish the open block see the whole block (cache + own frames), so
    their rows equal the one-shot rows; the final cache equals the one-shot one.
    """
    w = workloads.Workload("mid", B=1, H=4, d=32, dtype="bf16", T=9, Hg=12, Wg=20, F=3, split=(8, 12, 12), seed=13)
    q, k, v = workloads.call_tensors(w)
    ref, S_ref, z_ref = oracle_all_rows(w, q, k, v)
    qd, kd, vd = dev(q, "bf16"), dev(k, "bf16"), dev(v, "bf16")
    HW = w.HW
    st = blin.BlockState(w.B, w.H, w.d)
    sl = lambda a, f0, f1: a[:, :, f0 * HW:f1 * HW].contiguous()
    blin.prefill(sl(qd, 0, 4), sl(kd, 0, 4), sl(vd, 0, 4), (4, w.Hg, w.Wg), w.F, w.split, w.theta, w.eps, state=st)
    assert st.t_next == 4
    S0, z0 = st.to_host()
    # frames 4, 5, 6 would cross from block 1 into block 2
    with pytest.raises(blin.BlinError, match="BLIN_ERR_SHAPE"):
        blin.block_step(sl(qd, 4, 7), sl(kd, 4, 7), sl(vd, 4, 7), w.Hg, w.Wg, 3, w.split, st,
                        theta=w.theta, eps=w.eps, block_frames=w.F)
    S1, z1 = st.to_host()
    assert st.t_next == 4 and torch.equal(S0, S1) and torch.equal(z0, z1)
    o45 = blin.block_step(sl(qd, 4, 6), sl(kd, 4, 6), sl(vd, 4, 6), w.Hg, w.Wg, 2, w.split, st,
                          theta=w.theta, eps=w.eps, block_frames=w.F)
    o68 = blin.block_step(sl(qd, 6, 9), sl(kd, 6, 9), sl(vd, 6, 9), w.Hg, w.Wg, 3, w.split, st,
                          theta=w.theta, eps=w.eps, block_frames=w.F)
    torch.cuda.synchronize()
    assert rel_err(host(o45).reshape(-1, 2 * HW, w.d), ref[:, 4 * HW:6 * HW]) <= TOL["bf16"]
    assert rel_err(host(o68).reshape(-1, 3 * HW, w.d), ref[:, 6 * HW:]) <= TOL["bf16"]
    assert st.t_next == 9
    S, z = st.to_host()
    assert rel_err(S.numpy().reshape(S_ref.shape), S_ref) <= 5e-3
    assert rel_err(z.numpy().reshape(z_ref.shape), z_ref) <= 1e-5


def test_head_subsets_give_the_same_bits(blin):
    """Heads are independent: a call over all heads equals calls over head subsets, bit for bit
    (the state chunks of a block depend on the block alone, not on how many heads share a call)."""
    w = workloads.CONFIGS["480p"].with_(H=24, seed=23)
    q, k, v = (dev(x, "bf16") for x in workloads.call_tensors(w))
    want = blin.prefill(q, k, v, (w.T, w.Hg, w.Wg), w.F, w.split, w.theta, w.eps)
    parts = [blin.prefill(q[:, a:b].contiguous(), k[:, a:b].contiguous(), v[:, a:b].contiguous(),
                          (w.T, w.Hg, w.Wg), w.F, w.split, w.theta, w.eps) for a, b in ((0, 1), (1, 9), (9, 24))]
    torch.cuda.synchronize()
    assert torch.equal(torch.cat(parts, dim=1), want)
