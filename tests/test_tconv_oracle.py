"""Pins of the float64 temporal-convolution oracle (causal FFN with a one-frame cache).

Talk transcript, causal-FFN passage: a zero token sits between two blocks in
causal training (a block never sees the next block); the next block sees the
previous block's last token, which is cached and put in front of it.
"""
import numpy as np

import oracle


def same_conv(a, taps):
    """Zero-padded convolution along t, as long as `a`, with taps (previous, current, next):
    numpy's full convolution (which flips its kernel) centred on `a`."""
    return np.convolve(a, taps[::-1])[1:1 + len(a)]


def test_hand_worked_example():
    # T = 4 frames of one pixel and one channel, blocks of F = 2, taps (10, 100, 1000), bias 0.5:
    #   t0: 0*10 + 1*100 + 2*1000          + .5 = 2100.5   (nothing before the video)
    #   t1: 1*10 + 2*100 + 0 (next block)  + .5 =  210.5   (zero pad after the block)
    #   t2: 2*10 + 3*100 + 4*1000          + .5 = 4320.5   (previous block's last frame)
    #   t3: 3*10 + 4*100 + 0 (video ends)  + .5 =  430.5
    x = np.array([1, 2, 3, 4], np.float32).reshape(1, 4, 1, 1)
    y, last = oracle.tconv(x, [[10, 100, 1000]], [0.5], F=2)
    assert y.ravel().tolist() == [2100.5, 210.5, 4320.5, 430.5]
    assert last.ravel().tolist() == [4.0]


def test_identity_tap_returns_the_input():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((2, 7, 5, 6)).astype(np.float32)
    w = np.zeros((6, 3))
    w[:, 1] = 1.0
    y, _ = oracle.tconv(x, w, None, F=3)
    np.testing.assert_array_equal(y, x.astype(np.float64))


def test_single_block_is_numpy_same_convolution():
    """One block covering the call: a zero-padded 'same' convolution along t (numpy's)."""
    rng = np.random.default_rng(2)
    B, T, HW, C = 1, 9, 4, 3
    x = rng.standard_normal((B, T, HW, C)).astype(np.float32)
    w = rng.standard_normal((C, 3))
    bias = rng.standard_normal(C)
    y, _ = oracle.tconv(x, w, bias, F=T)
    for s in range(HW):
        for c in range(C):
            want = same_conv(x[0, :, s, c].astype(np.float64), w[c]) + bias[c]
            np.testing.assert_allclose(y[0, :, s, c], want, rtol=1e-14, atol=1e-14)


def test_blocks_are_same_convolutions_plus_the_carried_frame():
    """Several blocks: each block is a zero-padded 'same' convolution of its own frames, and a
    block's first frame also gets the previous tap times the previous block's last frame."""
    rng = np.random.default_rng(3)
    B, T, HW, C, F = 2, 10, 3, 2, 3
    x = rng.standard_normal((B, T, HW, C)).astype(np.float32)
    w = rng.standard_normal((C, 3))
    y, _ = oracle.tconv(x, w, None, F=F)
    xd = x.astype(np.float64)
    for b in range(B):
        for s in range(HW):
            for c in range(C):
                for f0 in range(0, T, F):
                    f1 = min(f0 + F, T)
                    want = same_conv(xd[b, f0:f1, s, c], w[c])
                    if f0 > 0:
                        want[0] += w[c, 0] * xd[b, f0 - 1, s, c]
                    np.testing.assert_allclose(y[b, f0:f1, s, c], want, rtol=1e-13, atol=1e-13)


def test_streamed_calls_carry_the_cache():
    """Calls split at block boundaries, each handed the previous call's last frame, give the
    one-shot result; a call that ends inside a block leaves that block's last given frame
    without its next neighbour (it is not given yet)."""
    rng = np.random.default_rng(4)
    B, T, HW, C, F = 1, 12, 5, 4, 3
    x = rng.standard_normal((B, T, HW, C)).astype(np.float32)
    w = rng.standard_normal((C, 3))
    bias = rng.standard_normal(C)
    full, _ = oracle.tconv(x, w, bias, F=F)
    parts, prev = [], None
    for f0 in range(0, T, F):
        y, prev = oracle.tconv(x[:, f0:f0 + F], w, bias, F=F, t0=f0, prev=prev)
        parts.append(y)
    np.testing.assert_array_equal(np.concatenate(parts, axis=1), full)
    # mid-block split: frames 0..4 then 5..11 (block 1 = frames 3, 4, 5)
    y1, prev = oracle.tconv(x[:, :5], w, bias, F=F)
    y2, _ = oracle.tconv(x[:, 5:], w, bias, F=F, t0=5, prev=prev)
    np.testing.assert_array_equal(y1[:, :4], full[:, :4])
    assert not np.allclose(y1[:, 4], full[:, 4])  # frame 5 was not given yet
    np.testing.assert_allclose(y1[:, 4], full[:, 4] - w[:, 2] * x[:, 5].astype(np.float64), rtol=1e-13, atol=1e-13)
    np.testing.assert_array_equal(y2, full[:, 5:])


def test_linear_in_x_and_zero_before_the_video():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((1, 6, 2, 3)).astype(np.float32)
    w = rng.standard_normal((3, 3))
    y1, _ = oracle.tconv(x, w, None, F=2)
    y2, _ = oracle.tconv(2 * x, w, None, F=2)
    np.testing.assert_allclose(y2, 2 * y1, rtol=1e-14)
    # at t0 = 0 a `prev` frame is ignored: nothing comes before the video
    y3, _ = oracle.tconv(x, w, None, F=2, t0=0, prev=np.full((1, 2, 3), 7.0))
    np.testing.assert_array_equal(y3, y1)
