"""Pins for the float64 oracle, against things other than the oracle itself.

Each test ties one part of the oracle to brute force, a closed form, a
textbook/library routine or an invariant, so that a dropped term, a wrong sign,
index or transposed operand in it fails here.  CPU only.
"""
import itertools

import numpy as np
import pytest
import torch

import oracle
import workloads


def _rand(shape, seed, scale=1.0):
    return (np.random.default_rng(seed).standard_normal(shape) * scale).astype(np.float32)


# --------------------------------------------------------------------------- a0: grid + blocks
@pytest.mark.parametrize("T,Hg,Wg,F,t0", [(12, 4, 4, 3, 0), (7, 3, 5, 3, 0), (5, 1, 1, 1, 4),
                                           (4, 2, 3, 3, 5), (9, 2, 2, 4, 6)])
def test_grid_matches_enumeration(T, Hg, Wg, F, t0):
    pos, blk = oracle.grid(T, Hg, Wg, F, t0)
    # brute force: walk the video from frame 0, counting a new block every F frames
    block_of_frame, b, run = {}, 0, 0
    for f in range(t0 + T):
        if run == F:
            b, run = b + 1, 0
        block_of_frame[f] = b
        run += 1
    want_pos = [(t0 + t, y, x) for t in range(T) for y in range(Hg) for x in range(Wg)]
    assert [tuple(p) for p in pos.tolist()] == want_pos
    assert blk.tolist() == [block_of_frame[p[0]] for p in want_pos]


# --------------------------------------------------------------------------- RoPE
def _library_rope_section(u_sec, p, theta):
    """Rotate one axis section with the transformers (Llama) RoPE.

    The library pairs feature j with j + d_a/2; the oracle pairs (2j, 2j+1).
    The permutation between the two layouts is applied around the call.
    """
    from transformers import LlamaConfig
    from transformers.models.llama.modeling_llama import LlamaRotaryEmbedding, apply_rotary_pos_emb

    da = len(u_sec)
    cfg = LlamaConfig(hidden_size=64, num_attention_heads=1, head_dim=da, rope_theta=theta)
    rot = LlamaRotaryEmbedding(cfg)
    half = np.concatenate([u_sec[0::2], u_sec[1::2]])
    x = torch.tensor(half, dtype=torch.float64).view(1, 1, 1, da)
    cos, sin = rot(x, torch.tensor([[p]]))
    y, _ = apply_rotary_pos_emb(x, x, cos, sin)
    y = y.view(-1).numpy()
    out = np.empty(da)
    out[0::2], out[1::2] = y[: da // 2], y[da // 2:]
    return out


@pytest.mark.parametrize("split", [(8, 12, 12), (16, 24, 24)])
def test_rope_matches_library_per_axis(split):
    d = sum(split)
    u = np.random.default_rng(3).standard_normal(d)
    for p in [(0, 0, 0), (1, 2, 3), (17, 29, 51), (239, 44, 79)]:
        got = oracle.rope(u, p, split, 10000.0)
        off = 0
        for a in range(3):
            sec = slice(off, off + split[a])
            want = _library_rope_section(u[sec], p[a], 10000.0)
            np.testing.assert_allclose(got[sec], want, rtol=0, atol=2e-5 * max(1, p[a]) ** 0.5)
            off += split[a]


def test_rope_is_rotation_with_relative_property():
    split = (8, 12, 12)
    rng = np.random.default_rng(4)
    u, w = rng.standard_normal(32), rng.standard_normal(32)
    for p, q in [((3, 1, 2), (7, 5, 0)), ((0, 9, 9), (4, 0, 1)), ((200, 40, 70), (1, 2, 3))]:
        Ru = oracle.rope(u, p, split, 1e4)
        assert np.linalg.norm(Ru) == pytest.approx(np.linalg.norm(u), rel=1e-14)
        assert Ru @ oracle.rope(w, p, split, 1e4) == pytest.approx(u @ w, rel=1e-12)
        # <R_p u, R_q w> = <u, R_{q-p} w>: depends on the offset only
        lhs = Ru @ oracle.rope(w, q, split, 1e4)
        diff = tuple(b - a for a, b in zip(p, q))
        rhs = u @ oracle.rope(w, diff, split, 1e4)
        assert lhs == pytest.approx(rhs, rel=1e-10, abs=1e-12)
    # position 0 is the identity
    np.testing.assert_array_equal(oracle.rope(u, (0, 0, 0), split, 1e4), u)


# --------------------------------------------------------------------------- sums
def _small_case(seed=0, T=7, Hg=3, Wg=5, F=3, H=2, d=32, t0=0):
    N = T * Hg * Wg
    q, k, v = (_rand((H, N, d), seed + i) for i in range(3))
    pos, blk = oracle.grid(T, Hg, Wg, F, t0)
    return q, k, v, pos, blk


@pytest.mark.parametrize("shape", [dict(), dict(T=12, Hg=4, Wg=4, F=3), dict(T=5, Hg=2, Wg=3, F=2, t0=3),
                                   dict(T=4, Hg=2, Wg=2, F=1, d=64)])
def test_pair_sum_equals_state_recurrence(shape):
    d = shape.get("d", 32)
    split = (8, 12, 12) if d == 32 else (16, 24, 24)
    q, k, v, pos, blk = _small_case(**shape)
    rows = np.arange(q.shape[1])
    a = oracle.attention_rows(q, k, v, pos, blk, rows, split, 1e4, 1e-6)
    b, _, _ = oracle.recurrence(q, k, v, pos, blk, split, 1e4, 1e-6)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-12 * np.abs(b).max())


def test_single_block_is_noncausal_linear_attention():
    """F >= T: every token sees every token; textbook matrix form."""
    split = (8, 12, 12)
    q, k, v, pos, blk = _small_case(T=4, Hg=3, Wg=2, F=8)
    assert (blk == 0).all()
    eps = 1e-3
    rows = np.arange(q.shape[1])
    got = oracle.attention_rows(q, k, v, pos, blk, rows, split, 1e4, eps)
    for h in range(q.shape[0]):
        fq, fk = np.maximum(q[h], 0).astype(np.float64), np.maximum(k[h], 0).astype(np.float64)
        rq = np.stack([oracle.rope(fq[n], pos[n], split, 1e4) for n in range(len(fq))])
        rk = np.stack([oracle.rope(fk[n], pos[n], split, 1e4) for n in range(len(fk))])
        num = (rq @ rk.T) @ v[h].astype(np.float64)
        den = (fq @ fk.T) @ np.ones(len(fk)) + eps
        np.testing.assert_allclose(got[h], num / den[:, None], rtol=1e-11, atol=1e-13)


def test_identity_rope_constant_value_closed_form():
    """All angles zero and v_m = c: o_n = c * s_n / (s_n + eps), s_n = phi(q_n).sum_{m<=b(n)} phi(k_m)."""
    H, T, Hg, Wg, F, d = 2, 6, 2, 3, 2, 32
    N = T * Hg * Wg
    q, k = _rand((H, N, d), 11), _rand((H, N, d), 12)
    c = _rand((d,), 13)
    v = np.broadcast_to(c, (H, N, d)).copy()
    _, blk = oracle.grid(T, Hg, Wg, F)
    pos = np.zeros((N, 3), np.int64)
    eps = 0.5  # large, so a misplaced eps is visible
    got = oracle.attention_rows(q, k, v, pos, blk, np.arange(N), (8, 12, 12), 1e4, eps)
    rec, _, _ = oracle.recurrence(q, k, v, pos, blk, (8, 12, 12), 1e4, eps)
    for h in range(H):
        fk = np.maximum(k[h], 0).astype(np.float64)
        block_sum = {b: fk[blk == b].sum(0) for b in np.unique(blk)}
        z = np.stack([sum(block_sum[c_] for c_ in block_sum if c_ <= b) for b in blk])
        s = (np.maximum(q[h], 0).astype(np.float64) * z).sum(1)
        want = c[None, :].astype(np.float64) * (s / (s + eps))[:, None]
        np.testing.assert_allclose(got[h], want, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(rec[h], want, rtol=1e-12, atol=1e-14)


def test_integer_bookkeeping_probe():
    """k = e_0, v_m = e_{b(m)}, no rotation: the state holds exact block counts."""
    H, T, Hg, Wg, F, d = 1, 10, 2, 3, 3, 32
    N = T * Hg * Wg
    _, blk = oracle.grid(T, Hg, Wg, F)
    pos = np.zeros((N, 3), np.int64)
    k = np.zeros((H, N, d), np.float32)
    k[..., 0] = 1.0
    v = np.zeros((H, N, d), np.float32)
    v[0, np.arange(N), blk] = 1.0
    q = np.zeros((H, N, d), np.float32)
    q[..., 0] = 2.0
    eps = 0.25
    out, S, z = oracle.recurrence(q, k, v, pos, blk, (8, 12, 12), 1e4, eps)
    L = np.bincount(blk)
    assert S[0, 0, : len(L)].tolist() == L.tolist()
    assert z[0, 0] == N and not S[0, 1:].any() and not z[0, 1:].any()
    cnt = np.cumsum(L)
    for n in range(N):
        b = blk[n]
        want = np.zeros(d)
        want[: b + 1] = 2.0 * L[: b + 1] / (2.0 * cnt[b] + eps)
        np.testing.assert_allclose(out[0, n], want, rtol=1e-15)
    rows = oracle.attention_rows(q, k, v, pos, blk, np.arange(N), (8, 12, 12), 1e4, eps)
    np.testing.assert_allclose(rows, out, rtol=1e-15)


def test_single_token_blocks_closed_form():
    """One token per block at a non-zero position: first output is (s v)/(s + eps)."""
    H, d, eps = 2, 32, 1e-2
    q, k, v = (_rand((H, 5, d), 20 + i) for i in range(3))
    pos, blk = oracle.grid(5, 1, 1, 1, t0=7)
    got = oracle.attention_rows(q, k, v, pos, blk, np.arange(5), (8, 12, 12), 1e4, eps)
    s = (np.maximum(q[:, 0], 0).astype(np.float64) * np.maximum(k[:, 0], 0)).sum(-1)
    want = s[:, None] * v[:, 0] / (s[:, None] + eps)
    np.testing.assert_allclose(got[:, 0], want, rtol=1e-12)


def test_two_token_worked_example():
    """Hand-derived: d=6 split (2,2,2), token 1 at t=1 rotates its t-pair by 1 rad.

    q_1 = (1,0,0,0,0,0), k_0 = (0,1,0,0,0,0), k_1 = (0,0,1,0,0,0):
      num_1 = (R_1 q_1 . k_0) v_0 + (R_1 q_1 . R_1 k_1) v_1 = sin(1) v_0 + 0 * v_1
      den_1 = q_1.k_0 + q_1.k_1 + eps = eps
    """
    q = np.zeros((1, 2, 6), np.float32)
    k = np.zeros((1, 2, 6), np.float32)
    q[0, 1, 0] = 1.0
    k[0, 0, 1] = 1.0
    k[0, 1, 2] = 1.0
    v = np.array([[[1, 2, 3, 4, 5, 6], [-1, -1, -1, -1, -1, -1]]], np.float32)
    pos, blk = oracle.grid(2, 1, 1, 1)
    eps = 0.125
    got = oracle.attention_rows(q, k, v, pos, blk, [1], (2, 2, 2), 1e4, eps)
    np.testing.assert_allclose(got[0, 0], np.sin(1.0) * np.arange(1, 7) / eps, rtol=1e-14)


def test_zero_query_gives_exact_zero():
    q, k, v, pos, blk = _small_case(seed=30)
    q[:, ::3, :] = -np.abs(q[:, ::3, :])
    out, _, _ = oracle.recurrence(q, k, v, pos, blk, (8, 12, 12), 1e4, 1e-6)
    assert (out[:, ::3, :] == 0.0).all()
    rows = oracle.attention_rows(q, k, v, pos, blk, np.arange(0, q.shape[1], 3), (8, 12, 12), 1e4, 1e-6)
    assert (rows == 0.0).all()


def test_shift_invariance_of_positions():
    """Shifting every t, y or x by a constant (blocks unchanged) leaves o unchanged."""
    q, k, v, pos, blk = _small_case(seed=40)
    rows = np.arange(q.shape[1])
    base = oracle.attention_rows(q, k, v, pos, blk, rows, (8, 12, 12), 1e4, 1e-6)
    for shift in [(5, 0, 0), (0, 11, 0), (0, 0, 23), (100, 3, 7)]:
        got = oracle.attention_rows(q, k, v, pos + np.array(shift), blk, rows, (8, 12, 12), 1e4, 1e-6)
        np.testing.assert_allclose(got, base, rtol=1e-9, atol=1e-12)
    # whole-block shift of the grid origin keeps the block structure
    pos2, blk2 = oracle.grid(7, 3, 5, 3, t0=9)
    got = oracle.attention_rows(q, k, v, pos2, blk2 - blk2[0], rows, (8, 12, 12), 1e4, 1e-6)
    np.testing.assert_allclose(got, base, rtol=1e-9, atol=1e-12)


def test_streamed_blocks_equal_one_shot():
    """Carrying (S, z) block by block equals the one-shot prefill (both oracle forms)."""
    w = workloads.CONFIGS["tiny"]
    q, k, v = workloads.call_tensors(w)
    pos, blk = oracle.grid(w.T, w.Hg, w.Wg, w.F)
    full, S_full, z_full = oracle.recurrence(q, k, v, pos, blk, w.split, w.theta, w.eps)
    S = z = None
    outs = []
    for (f0, f1) in w.block_frame_ranges():
        wb = w.with_(t0=f0, T=f1 - f0)
        qb, kb, vb = workloads.call_tensors(wb)
        pb, bb = oracle.grid(wb.T, w.Hg, w.Wg, w.F, f0)
        o, S, z = oracle.recurrence(qb, kb, vb, pb, bb, w.split, w.theta, w.eps, S, z)
        outs.append(o)
    np.testing.assert_array_equal(np.concatenate(outs, 1), full)
    np.testing.assert_array_equal(S, S_full)
    np.testing.assert_array_equal(z, z_full)
    # explicit sum with keys streamed block by block gives the same bits
    rows = np.arange(0, w.N, 7)
    ps = oracle.PairSum(q.reshape(-1, w.N, w.d)[:, rows], pos[rows], blk[rows], w.split, w.theta)
    for (f0, f1) in w.block_frame_ranges():
        sl = slice(f0 * w.HW, f1 * w.HW)
        ps.add_keys(k.reshape(-1, w.N, w.d)[:, sl], v.reshape(-1, w.N, w.d)[:, sl], pos[sl], blk[sl])
    one = oracle.attention_rows(q, k, v, pos, blk, rows, w.split, w.theta, w.eps)
    np.testing.assert_array_equal(ps.result(w.eps), one)


def test_scale_of_value_is_linear_and_eps_small_limit():
    """o is linear in V; with eps -> 0 and all-positive features, o is a convex mix of v rows."""
    q, k, v, pos, blk = _small_case(seed=50)
    rows = np.arange(q.shape[1])
    zero = np.zeros((q.shape[1], 3), np.int64)
    a = oracle.attention_rows(q, k, v, zero, blk, rows, (8, 12, 12), 1e4, 0.0)
    b = oracle.attention_rows(q, k, 4 * v, zero, blk, rows, (8, 12, 12), 1e4, 0.0)  # exact in fp32
    np.testing.assert_allclose(b, 4 * a, rtol=1e-12)
    # without rotation and eps the weights are non-negative and sum to one
    ones = oracle.attention_rows(q, k, np.ones_like(v), zero, blk, rows, (8, 12, 12), 1e4, 0.0)
    live = np.maximum(q, 0).sum(-1) > 0
    np.testing.assert_allclose(ones[live], 1.0, rtol=1e-12)


def test_positive_scaling_of_q_and_k_cancels_without_eps():
    """phi is positively homogeneous and o = num / den: with eps = 0, doubling q or k (exact in
    binary floating point) leaves every output bit unchanged.  A missing normalisation, phi
    applied after RoPE, or eps inside the dot product would break it."""
    q, k, v, pos, blk = _small_case(seed=60)
    rows = np.arange(q.shape[1])
    base = oracle.attention_rows(q, k, v, pos, blk, rows, (8, 12, 12), 1e4, 0.0)
    live = np.maximum(q, 0).sum(-1) > 0  # rows whose phi(q) is zero are 0 / 0 without eps
    for q2, k2 in ((2 * q, k), (q, 2 * k), (0.5 * q, 4 * k)):
        out = oracle.attention_rows(q2, k2, v, pos, blk, rows, (8, 12, 12), 1e4, 0.0)
        np.testing.assert_array_equal(out[live], base[live])


def test_keys_without_a_positive_feature_contribute_nothing():
    """A key whose features are all negative has phi(k) = 0, so it adds nothing to S or z: its
    value rows may be anything.  Using k instead of phi(k) in the numerator or the denominator
    would make them matter."""
    q, k, v, pos, blk = _small_case(seed=70)
    rng = np.random.default_rng(71)
    dead = rng.random(k.shape[1]) < 0.3
    k = k.copy()
    k[:, dead] = -np.abs(k[:, dead])
    v2 = v.copy()
    v2[:, dead] = _rand(v2[:, dead].shape, 72, scale=100.0)
    rows = np.arange(q.shape[1])
    a = oracle.attention_rows(q, k, v, pos, blk, rows, (8, 12, 12), 1e4, 1e-6)
    b = oracle.attention_rows(q, k, v2, pos, blk, rows, (8, 12, 12), 1e4, 1e-6)
    np.testing.assert_array_equal(a, b)
    s1, _, _ = oracle.recurrence(q, k, v, pos, blk, (8, 12, 12), 1e4, 1e-6)
    s2, _, _ = oracle.recurrence(q, k, v2, pos, blk, (8, 12, 12), 1e4, 1e-6)
    np.testing.assert_array_equal(s1, s2)


def test_golden_fixture_unchanged():
    """The oracle still produces the recorded tiny-workload rows bit for bit."""
    import json
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "tiny_oracle_rows.json")
    doc = json.load(open(path))
    w = workloads.CONFIGS["tiny"]
    q, k, v = workloads.call_tensors(w)
    pos, blk = oracle.grid(w.T, w.Hg, w.Wg, w.F)
    out = oracle.attention_rows(q, k, v, pos, blk, doc["rows"], w.split, w.theta, w.eps)
    want = np.array([[[float.fromhex(x) for x in r] for r in h] for h in doc["out"]])
    np.testing.assert_array_equal(out, want)
