"""Pins of the oracle's other 4-bit codebooks (FP4 E2M1 and absmax INT4), used to test the
pages' format claim that NF4 suits normally distributed weights better ("QLoRA in LLMs" §5;
"Idea one: NF4", goodomens.studio)."""

from fractions import Fraction

import numpy as np
import pytest

from oracle import nf4_oracle as O


def test_fp4_levels_are_the_e2m1_values_over_six():
    mags = [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2), Fraction(3),
            Fraction(4), Fraction(6)]
    want = [-m / 6 for m in reversed(mags)] + [m / 6 for m in mags]
    got = O.fp4_codebook()
    assert got.dtype == np.float32 and got.size == 16
    assert np.array_equal(got, np.array([float(v) for v in want], np.float32))
    assert np.signbit(got[7]) and not np.signbit(got[8]) and got[7] == got[8] == 0.0
    assert got[0] == -1.0 and got[15] == 1.0 and np.all(np.diff(got) >= 0)


def test_int4_levels_are_k_over_seven():
    got = O.int4_codebook()
    assert np.array_equal(got, np.array([float(Fraction(k, 7)) for k in range(-8, 8)], np.float32))
    assert got[8] == 0.0 and got[1] == -1.0 and got[15] == 1.0


@pytest.mark.parametrize("cb", [0, 1, 2])
def test_codes_are_the_nearest_level(cb):
    """Brute force: each code's level is a nearest level of x = w / c1 (fp64 distance), and
    every block holds its absmax at a +-1 level."""
    levels = O.codebook_levels(cb)
    rng = np.random.default_rng(cb)
    W = (rng.standard_normal((6, 256)) * 0.02).astype(np.float32)
    p = O.quantize_with(W, cb)
    codes = O.unpack_nibbles(p.codes).reshape(-1, 64)
    blocks = W.reshape(-1, 64).astype(np.float64)
    c1 = np.abs(blocks).max(1)
    x = blocks / c1[:, None]
    d_code = np.abs(levels[codes].astype(np.float64) - x)
    d_best = np.min(np.abs(levels.astype(np.float64)[None, None, :] - x[..., None]), axis=-1)
    assert np.all(d_code <= d_best + 1e-7)


@pytest.mark.parametrize("cb", [0, 1, 2])
def test_all_zero_block_takes_the_zero_level(cb):
    W = np.zeros((2, 128), np.float32)
    p = O.quantize_with(W, cb)
    codes = O.unpack_nibbles(p.codes)
    assert np.all(codes == O.CODEBOOK_ZERO_CODE[cb])
    assert O.codebook_levels(cb)[O.CODEBOOK_ZERO_CODE[cb]] == 0.0


def test_nf4_codebook_id_is_nf4():
    W = (np.random.default_rng(3).standard_normal((4, 192)) * 0.02).astype(np.float32)
    a, b = O.quantize_with(W, 0), O.nf4_quantize(W)
    assert np.array_equal(a.codes, b.codes) and np.array_equal(a.absmax_q8, b.absmax_q8)


def test_nf4_has_the_lowest_error_on_normal_weights():
    """The pages' claim, on synthetic N(0, 0.02) weights in 64-blocks with double-quantized
    scales: NF4's mean squared reconstruction error is below FP4's and INT4's."""
    W = (np.random.default_rng(0).standard_normal((256, 4096)) * 0.02).astype(np.float32)
    mse = {}
    for cb in (0, 1, 2):
        p = O.quantize_with(W, cb)
        deq = O.nf4_dequantize_f32(p, O.codebook_levels(cb)).astype(np.float64)
        mse[cb] = float(np.mean((deq - W) ** 2))
    assert mse[0] < mse[1] and mse[0] < mse[2], mse


@pytest.mark.parametrize("cb", [1, 2])
def test_representable_blocks_reproduce_themselves(cb):
    """A block made of the codebook's own levels times k = q8 * s2 (exact in fp32) keeps its
    codes and 8-bit scales, and dequantizes to the bf16 rounding of itself, bit for bit. The
    codes avoid the levels the encoder never chooses: FP4's +0 (a zero weight takes the -0
    code, the lower of two equal levels) and INT4's -8/7 (below -1)."""
    q = O.codebook_levels(cb)
    rng = np.random.default_rng(20 + cb)
    s2 = np.float32(2.0 ** -8)
    q8 = np.array([255] + list(rng.integers(1, 256, 255)), np.uint8)
    k = (q8.astype(np.float32) * s2).astype(np.float32)
    codes = rng.integers(1, 16, (256, 64)).astype(np.uint8)
    if cb == 1:
        codes[codes == 8] = 7
    codes[:, 0] = 15                      # level +1: every block reaches its absmax exactly
    W = (q[codes] * k[:, None]).astype(np.float32).reshape(4, 4096)
    p = O.quantize_with(W, cb)
    assert np.array_equal(O.unpack_nibbles(p.codes).reshape(256, 64), codes)
    assert np.array_equal(p.absmax_q8, q8)
    assert p.absmax_s2[0] == s2
    assert np.array_equal(O.dequantize_bits_with(p, cb), O.bf16_bits_rne(W))
