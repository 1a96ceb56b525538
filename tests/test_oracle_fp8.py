"""Pins of the oracle's e4m3 quantisation (the fp8 variant's Q/K/V copies).

The encoder and decoder are written from the OCP 8-bit floating point format definition
(E4M3: bias 7, 3 mantissa bits, no infinities, NaN = S.1111.111, max finite 448).  They
are pinned against PyTorch's independent float8_e4m3fn conversion, against closed forms
(saturation, midpoints, power-of-two scaling) and against the format's error bound.
"""
import numpy as np
import pytest
import torch

import oracle as O



def _torch_codes(y: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(y, dtype=np.float32)).to(torch.float8_e4m3fn) \
        .view(torch.uint8).numpy()


def test_decode_table_matches_library():
    codes = np.arange(256, dtype=np.uint8)
    mine = O.e4m3_decode(codes)
    lib = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(lib)
    assert nan.sum() == 2 and set(codes[nan].tolist()) == {0x7F, 0xFF}
    assert np.isnan(mine[nan]).all()
    np.testing.assert_array_equal(mine[~nan], lib[~nan])
    assert mine[0x7E] == 448.0 and mine[0x01] == 2.0 ** -9 and mine[0x08] == 2.0 ** -6


def test_encode_matches_library_inside_range():
    rng = np.random.default_rng(3)
    mag = np.exp2(rng.uniform(-12, np.log2(448.0), 200_000))
    y = (mag * rng.choice([-1.0, 1.0], mag.size)).astype(np.float32)
    y = np.concatenate([y, np.float32([0.0, -0.0, 448.0, -448.0, 2.0 ** -9, 2.0 ** -10, 2.0 ** -11])])
    np.testing.assert_array_equal(O.e4m3_encode(y), _torch_codes(y))


def test_midpoints_round_to_even_mantissa():
    vals = O.e4m3_decode(np.arange(0x7F, dtype=np.uint8))          # 0 .. 448, increasing
    assert np.all(np.diff(vals) > 0)
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)          # exact in fp32
    assert np.all(mids.astype(np.float64) == (vals[:-1] + vals[1:]) / 2)
    got = O.e4m3_encode(mids)
    lo = np.arange(0x7E, dtype=np.uint8)
    want = np.where(lo % 2 == 0, lo, lo + 1).astype(np.uint8)      # the even code of the two
    np.testing.assert_array_equal(got, want)
    np.testing.assert_array_equal(got, _torch_codes(mids))


def test_saturates_above_max_finite():
    y = np.float32([448.0001, 460.0, 464.0, 500.0, 1e30, -449.0, -1e30])
    np.testing.assert_array_equal(O.e4m3_encode(y), np.uint8([0x7E] * 5 + [0xFE] * 2))


def test_relative_error_bound_in_normal_range():
    rng = np.random.default_rng(4)
    y = np.exp2(rng.uniform(-6, np.log2(448.0), 100_000)).astype(np.float32)
    back = O.e4m3_decode(O.e4m3_encode(y))
    assert np.max(np.abs(back - y) / y) <= 2.0 ** -4


def _shape(B, H, N, d):
    return O.make_shape(B, H, N, d, 16, 0.5)


def test_quantize_blocks_closed_forms():
    rng = np.random.default_rng(5)
    B, H, N, d = 2, 3, 150, 64                      # blocks of 64, 64, 22 tokens
    x = rng.standard_normal((B, N, H, d)).astype(np.float32)
    x[1, 64:128, 2] = 0.0                            # an all-zero block
    s = _shape(B, H, N, d)
    codes, scales = O.quantize_blocks(s, x)
    assert scales.shape == (B, H, 3)
    assert scales[1, 2, 1] == 1.0 and not codes[1, 64:128, 2].any()
    for b in range(B):
        for h in range(H):
            for i in range(3):
                blk = x[b, 64 * i:min(N, 64 * i + 64), h]
                amax = np.abs(blk).max()
                if amax == 0:
                    continue
                assert scales[b, h, i] == np.float32(amax) / np.float32(448.0)
                # the element of largest magnitude lands on +-448 (code 0x7E / 0xFE)
                at = np.unravel_index(np.argmax(np.abs(blk)), blk.shape)
                assert codes[b, 64 * i + at[0], h, at[1]] & 0x7F == 0x7E
    deq = O.dequantize_blocks(s, codes, scales)
    rep = np.repeat(scales.astype(np.float64), 64, axis=2)[:, :, :N].transpose(0, 2, 1)[..., None]
    # error of each element: at most half the e4m3 spacing at its magnitude
    # (2^-4 relative in the normal range, 2^-10 * scale below it)
    bound = np.maximum(np.abs(x) * 2.0 ** -4, 2.0 ** -10 * rep)
    assert np.all(np.abs(deq - x) <= bound)


def test_quantize_blocks_power_of_two_scaling_and_head_independence():
    rng = np.random.default_rng(6)
    B, H, N, d = 1, 2, 200, 128
    x = rng.standard_normal((B, N, H, d)).astype(np.float32)
    s = _shape(B, H, N, d)
    c0, s0 = O.quantize_blocks(s, x)
    x2 = x.copy()
    x2[:, :, 1] *= 4.0                              # exact in fp32
    c1, s1 = O.quantize_blocks(s, x2)
    np.testing.assert_array_equal(c0, c1)
    np.testing.assert_array_equal(s1[:, 0], s0[:, 0])
    np.testing.assert_array_equal(s1[:, 1], 4.0 * s0[:, 1])


def test_quantize_ragged_block_ignores_nothing_past_n():
    # the 8-token tail block has its own scale from its own 8 tokens
    rng = np.random.default_rng(7)
    x = rng.standard_normal((1, 72, 1, 64)).astype(np.float32)
    x[0, 64:] *= 1e-3
    codes, scales = O.quantize_blocks(_shape(1, 1, 72, 64), x)
    assert scales[0, 0, 1] == np.float32(np.abs(x[0, 64:]).max()) / np.float32(448.0)
