"""Causal block temporal convolution (CUDA) against the float64 oracle.

Talk transcript, causal-FFN passage: a zero token separates blocks in causal
training; a block's first frame sees the previous block's last frame, cached.
Bound: |y - y_ref| <= 2^-8 |y_ref| + 1e-5 * max|y_ref| for bf16 storage (one
bf16 rounding of an fp32 sum of three products), 1e-6 relative for fp32.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from _support import TORCH_DT

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def blin():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import block_causal_linear_rope_b200 as m
    yield m


def _dev(w, x):
    return torch.from_numpy(np.ascontiguousarray(x.reshape(w.B, -1, w.C))).to("cuda", TORCH_DT[w.dtype])


def _check(w, got, ref):
    got = got.float().cpu().numpy().reshape(ref.shape).astype(np.float64)
    if w.dtype == "f32":
        assert np.abs(got - ref).max() <= 1e-6 * max(np.abs(ref).max(), 1e-30)
    else:
        assert (np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-5 * np.abs(ref).max()).all()


CASES = [("conv-tiny", {}), ("conv-tiny", {"dtype": "bf16"}), ("conv-tiny", {"F": 1}), ("conv-tiny", {"F": 10}),
         ("conv-tiny", {"T": 1}), ("conv-tiny", {"Hg": 1, "Wg": 1, "C": 8}), ("conv-tiny", {"B": 3, "C": 24, "T": 11})]


@pytest.mark.parametrize("name,kw", CASES)
def test_one_call_matches_oracle(blin, name, kw):
    w = workloads.CONV_CONFIGS[name].with_(**kw)
    x, taps, bias = workloads.conv_tensors(w)
    y = blin.tconv(_dev(w, x), torch.from_numpy(taps), torch.from_numpy(bias), (w.T, w.Hg, w.Wg), w.F)
    torch.cuda.synchronize()
    ref, _ = oracle.tconv(x, taps, bias, F=w.F)
    _check(w, y, ref)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_streamed_blocks_equal_one_call_bitwise(blin, dtype):
    w = workloads.CONV_CONFIGS["conv-tiny"].with_(dtype=dtype, T=12, C=32)
    x, taps, bias = workloads.conv_tensors(w)
    xd = _dev(w, x)
    tt, bt = torch.from_numpy(taps), torch.from_numpy(bias)
    full = blin.tconv(xd, tt, bt, (w.T, w.Hg, w.Wg), w.F)
    st = blin.TConvState(w.B, w.C, w.Hg, w.Wg, dtype=TORCH_DT[dtype])
    assert st.nbytes == w.B * w.HW * w.C * (2 if dtype == "bf16" else 4)
    parts = []
    for f0 in range(0, w.T, w.F):
        xb = xd[:, f0 * w.HW:(f0 + w.F) * w.HW].contiguous()
        # a denoising pass first: reads the cache, leaves it alone
        blin.tconv(xb, tt, bt, (w.F, w.Hg, w.Wg), w.F, state=st, commit=False)
        assert st.t_next == f0
        parts.append(blin.tconv(xb, tt, bt, (w.F, w.Hg, w.Wg), w.F, state=st))
    torch.cuda.synchronize()
    assert st.t_next == w.T
    assert torch.equal(torch.cat(parts, dim=1), full)
    ref, _ = oracle.tconv(x, taps, bias, F=w.F)
    _check(w, full, ref)


def test_call_ending_inside_a_block(blin):
    """Frames 0..4 then 5..11 with blocks of 3: the first call's last frame has no next
    neighbour yet; the second call's first frame sees frame 4 through the cache."""
    w = workloads.CONV_CONFIGS["conv-tiny"].with_(T=12)
    x, taps, bias = workloads.conv_tensors(w)
    xd = _dev(w, x)
    tt, bt = torch.from_numpy(taps), torch.from_numpy(bias)
    st = blin.TConvState(w.B, w.C, w.Hg, w.Wg, dtype=torch.float32)
    y1 = blin.tconv(xd[:, :5 * w.HW].contiguous(), tt, bt, (5, w.Hg, w.Wg), w.F, state=st)
    y2 = blin.tconv(xd[:, 5 * w.HW:].contiguous(), tt, bt, (7, w.Hg, w.Wg), w.F, state=st)
    torch.cuda.synchronize()
    r1, last = oracle.tconv(x[:, :5], taps, bias, F=w.F)
    r2, _ = oracle.tconv(x[:, 5:], taps, bias, F=w.F, t0=5, prev=last)
    _check(w, y1, r1)
    _check(w, y2, r2)


def test_full_size_480p_channels(blin):
    w = workloads.CONV_CONFIGS["conv-480p"]
    x, taps, bias = workloads.conv_tensors(w)
    y = blin.tconv(_dev(w, x), torch.from_numpy(taps), torch.from_numpy(bias), (w.T, w.Hg, w.Wg), w.F)
    torch.cuda.synchronize()
    ref, _ = oracle.tconv(x, taps, bias, F=w.F)
    _check(w, y, ref)


def test_rejects_bad_arguments(blin):
    x = torch.zeros(1, 12, 12, device="cuda", dtype=torch.bfloat16)  # C = 12: not a multiple of 8
    with pytest.raises(blin.BlinError, match="BLIN_ERR_SHAPE"):
        blin.tconv(x, torch.zeros(12, 3), None, (3, 2, 2), 3)
    x = torch.zeros(1, 12, 16, device="cuda", dtype=torch.bfloat16)
    with pytest.raises(blin.BlinError, match="BLIN_ERR_INVALID_ARG"):
        blin.tconv(x, torch.zeros(16, 3), None, (3, 2, 2), 0)
