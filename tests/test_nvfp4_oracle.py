"""Pins of the oracle's NVFP4 decoding (news article, NVFP4 / SVDQuant paragraph).

E4M3 against torch's float8_e4m3fn for all 256 codes; E2M1 against the
format's table; the block layout against hand-built bytes; and the encoder's
round trip (inputs are drawn in float32, then quantised) within half a step.
"""
import numpy as np
import torch

import oracle
import workloads


def test_e4m3_matches_torch_for_every_code():
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    got = np.array([oracle.e4m3(c) for c in range(256)])
    nan = np.isnan(ref)
    assert (np.isnan(got) == nan).all()
    np.testing.assert_array_equal(got[~nan], ref[~nan].astype(np.float64))


def test_e2m1_table():
    want = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert [oracle.e2m1(c) for c in range(8)] == want
    assert [oracle.e2m1(8 + c) for c in range(8)] == [-v for v in want]


def test_encoder_rounds_to_nearest_with_ties_to_even():
    # scale 1 (E4M3 0x38), global 1: values straight onto the E2M1 grid
    x = np.array([[0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.3, 6.0, 0.1, 2.6, -5.1, 6.0, 0.0, 1.0, 4.4]], np.float32)
    x = np.concatenate([x, x], axis=1) * np.float32(1.0)
    x[0, 31] = 6.0  # both blocks reach 6: scale exactly 1
    x[0, 15] = 6.0
    data, scale = workloads.nvfp4_encode(x, 1.0)
    assert scale.tolist() == [[0x38, 0x38]]
    y = oracle.nvfp4_decode(data, scale, 32, 1.0)[0, :16]
    assert y.tolist() == [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0, -0.5, 6.0, 0.0, 3.0, -6.0, 6.0, 0.0, 1.0, 6.0]


def test_block_layout_by_hand():
    # one row of d = 32: element 2i in the low nibble of byte i; scale byte j for elements 16j..16j+15
    d = 32
    codes = np.array([i % 16 for i in range(d)], np.uint8)
    data = (codes[0::2] | (codes[1::2] << 4)).reshape(1, 16)
    scale = np.array([[0x38, 0x40]], np.uint8)  # E4M3 1.0 and 2.0
    got = oracle.nvfp4_decode(data, scale, d, 0.25)
    want = [oracle.e2m1(c) * (1.0 if i < 16 else 2.0) * 0.25 for i, c in enumerate(codes)]
    assert got.ravel().tolist() == want
    assert oracle.e4m3(0x38) == 1.0 and oracle.e4m3(0x40) == 2.0


def test_encode_round_trip_within_half_a_step():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((64, 32)).astype(np.float32) * rng.lognormal(0, 1, (64, 1)).astype(np.float32)
    g = workloads.nvfp4_global_scale(x)
    data, scale = workloads.nvfp4_encode(x, g)
    y = oracle.nvfp4_decode(data, scale, 32, g)
    blocks_x = x.reshape(64, 2, 16).astype(np.float64)
    blocks_y = y.reshape(64, 2, 16)
    s = np.array([[oracle.e4m3(c) for c in row] for row in scale]) * g
    # E2M1 steps are at most 2 units of scale (between 4 and 6): rounding moves a value by at most 1
    assert (np.abs(blocks_x - blocks_y) <= s[..., None] * 1.0 + 1e-12).all()
    # values on the grid come back exactly
    exact = blocks_y / np.where(s[..., None] > 0, s[..., None], 1)
    assert np.isin(np.abs(exact), [0, 0.5, 1, 1.5, 2, 3, 4, 6]).all()
