"""Pins of the oracle's blockwise NF4 quantizer, double quantization and dequantization.

Each test checks the oracle against something other than itself:
* brute force: an fp64 nearest-level search over all 16 levels;
* hand-built blocks whose codes, packed bytes and scales are known in advance;
* the round-trip error bound implied by nearest-level coding, the 8-bit scale step and the
  bf16 rounding;
* the pages' statements: blocks of 64 with an absmax scale ("QLoRA in LLMs" sections 2-3),
  outliers inflate the step of their group ("What determines the rounding error?"), double
  quantization changes the scales but not the 4-bit codes (section 6), the textbook INT8
  example (section 2, "Choose a scale, then round").
"""

import json
import os

import numpy as np
import pytest

from oracle import nf4_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_w(o, h, seed, sigma=0.02):
    return (np.random.default_rng(seed).standard_normal((o, h)) * sigma).astype(np.float32)


def test_codes_agree_with_fp64_nearest_level_search():
    W = _rand_w(8, 192, 3)
    codes = O.nf4_codes(W).reshape(-1, 64)
    q64 = O.nf4_codebook().astype(np.float64)
    w64 = W.reshape(-1, 64).astype(np.float64)
    c1 = np.max(np.abs(w64), axis=1, keepdims=True)
    xhat64 = w64 / c1
    brute = np.argmin(np.abs(xhat64[..., None] - q64), axis=-1)
    differ = codes != brute
    # any disagreement may only sit within fp32 rounding of a decision threshold
    mids = O.nf4_midpoints().astype(np.float64)
    for b, k in zip(*np.nonzero(differ)):
        assert np.min(np.abs(mids - xhat64[b, k])) < 1e-6
    assert differ.mean() < 1e-3


def test_known_block_codes_and_nibble_order():
    q = O.nf4_codebook()
    pattern = np.tile(np.arange(16, dtype=np.uint8), 4)         # codes 0..15, four times
    W = q[pattern].reshape(1, 64).astype(np.float32)             # absmax is exactly 1
    packed = O.nf4_quantize(W)
    assert np.array_equal(O.unpack_nibbles(packed.codes), pattern)
    expected = np.tile(np.array([0x01, 0x23, 0x45, 0x67, 0x89, 0xAB, 0xCD, 0xEF], np.uint8), 4)
    assert np.array_equal(packed.codes, expected)                # element 2j in the high nibble
    assert packed.absmax_q8.tolist() == [255]
    assert packed.absmax_s2.dtype == np.float32 and packed.absmax_s2[0] == np.float32(1.0) / np.float32(255.0)


def test_negative_extreme_and_scale_invariance():
    q = O.nf4_codebook()
    pattern = np.random.default_rng(5).integers(0, 16, 64).astype(np.uint8)
    pattern[10] = 0                                              # -1 * c: the extreme is negative
    pattern[20] = 7
    for c in [np.float32(0.37), np.float32(3.0e-5), np.float32(12.5)]:
        W = (q[pattern] * c).astype(np.float32).reshape(1, 64)
        assert np.array_equal(O.nf4_codes(W), pattern)


def test_zero_block_and_all_zero_group():
    W = np.zeros((2, 128), np.float32)
    W[1, 64:] = _rand_w(1, 64, 9)
    p = O.nf4_quantize(W)
    codes = O.unpack_nibbles(p.codes).reshape(-1, 64)
    assert np.all(codes[:3] == O.ZERO_CODE)
    assert p.absmax_q8[:3].tolist() == [0, 0, 0] and p.absmax_q8[3] == 255
    deq = O.nf4_dequantize(p)
    assert np.all(deq[0] == 0) and np.all(deq[1, :64] == 0)
    Z = O.nf4_quantize(np.zeros((1, 64), np.float32))
    assert Z.absmax_s2[0] == 0.0 and Z.absmax_q8[0] == 0
    assert np.all(O.nf4_dequantize(Z) == 0)


def test_partial_last_group_uses_its_own_max():
    W = _rand_w(3, 64 * 100, 11)          # 300 blocks: one full group, one of 44
    W[2, -1] = 5.0                        # the last block of the partial group is huge
    p = O.nf4_quantize(W)
    c1 = O.block_absmax(W)
    assert p.absmax_s2.size == 2
    assert p.absmax_s2[0] == np.float32(np.max(c1[:256])) / np.float32(255)
    assert p.absmax_s2[1] == np.float32(5.0) / np.float32(255)
    assert p.absmax_q8[299] == 255


def test_idempotent_on_representable_blocks():
    """A block equal to q[code] * k, with k = q8 * s2 exactly, reproduces itself (up to the
    final bf16 rounding) and keeps its codes and 8-bit scale."""
    q = O.nf4_codebook()
    rng = np.random.default_rng(7)
    s2 = np.float32(2.0 ** -8)
    q8 = np.array([255] + list(rng.integers(1, 256, 255)), np.uint8)
    k = (q8.astype(np.float32) * s2).astype(np.float32)
    codes = rng.integers(0, 16, (256, 64)).astype(np.uint8)
    codes[:, 0] = 15                      # every block reaches its absmax exactly
    W = (q[codes] * k[:, None]).astype(np.float32).reshape(4, 4096)
    p = O.nf4_quantize(W)
    assert np.array_equal(O.unpack_nibbles(p.codes).reshape(256, 64), codes)
    assert np.array_equal(p.absmax_q8, q8)
    assert p.absmax_s2[0] == s2
    assert np.array_equal(O.nf4_dequantize(p), O.bf16_round(W))


def test_round_trip_error_bound():
    W = _rand_w(16, 1024, 13)
    p = O.nf4_quantize(W)
    deq = O.nf4_dequantize(p).astype(np.float64)
    q = O.nf4_codebook().astype(np.float64)
    mids = O.nf4_midpoints().astype(np.float64)
    lo = np.concatenate([[-1.0], mids])
    hi = np.concatenate([mids, [1.0]])
    g = np.maximum(q - lo, hi - q)                       # half-width of each code's cell
    codes = O.unpack_nibbles(p.codes).reshape(-1, 64)
    c1 = O.block_absmax(W).astype(np.float64)[:, None]
    s2 = p.absmax_s2.astype(np.float64)[np.arange(codes.shape[0]) // 256][:, None]
    # bf16 rounding moves a value by at most half an ulp: 2^-8 of it at the bottom of a binade
    bound = c1 * g[codes] + np.abs(q[codes]) * s2 / 2 + 2.0 ** -8 * np.abs(deq.reshape(-1, 64)) \
        + 1e-6 * c1
    err = np.abs(W.astype(np.float64).reshape(-1, 64) - deq.reshape(-1, 64))
    assert np.all(err <= bound)


def test_double_quant_changes_scales_not_codes():
    W = _rand_w(8, 2048, 17)
    codes_plain = O.nf4_codes(W)
    p = O.nf4_quantize(W)
    assert np.array_equal(O.unpack_nibbles(p.codes), codes_plain)
    c1 = O.block_absmax(W)
    k = O.block_scales(p.absmax_q8, p.absmax_s2)
    s2 = p.absmax_s2[np.arange(c1.size) // 256]
    assert np.all(np.abs(k.astype(np.float64) - c1) <= s2.astype(np.float64) * 0.5 * (1 + 1e-6))
    no_dq = O.dequantize_without_double_quant(codes_plain, c1, 8, 2048)
    with_dq = O.nf4_dequantize(p)
    q = O.nf4_codebook()
    bound = np.abs(q[codes_plain].reshape(8, 2048)) * s2.repeat(64).reshape(8, 2048) \
        + 2.0 ** -8 * np.maximum(np.abs(no_dq), np.abs(with_dq)) + 1e-12
    assert np.all(np.abs(no_dq - with_dq) <= bound)


def test_outliers_inflate_their_blocks():
    W = _rand_w(64, 4096, 19)
    clean = W.copy()
    rng = np.random.default_rng(23)
    pos = rng.permutation(W.size)[: W.size // 100]
    W.reshape(-1)[pos] = np.where(rng.integers(0, 2, pos.size) == 1, 0.16, -0.16).astype(np.float32)
    has = np.zeros(W.size, bool)
    has[pos] = True
    blk_has = has.reshape(-1, 64).any(axis=1)
    c1 = O.block_absmax(W)
    assert np.all(np.isclose(c1[blk_has], 0.16))
    err = np.abs(O.nf4_dequantize(O.nf4_quantize(W)) - W).reshape(-1, 64)
    normal = ~has.reshape(-1, 64)
    e_out = err[blk_has][normal[blk_has]].mean()
    e_clean = err[~blk_has].mean()
    assert e_out > 1.5 * e_clean
    # the clean matrix has no such blocks
    assert np.max(O.block_absmax(clean)) < 0.16


def test_nonfinite_input_is_rejected():
    W = _rand_w(1, 64, 29)
    W[0, 5] = np.nan
    with pytest.raises(ValueError):
        O.nf4_quantize(W)


def test_textbook_int8_example():
    g = json.load(open(os.path.join(GOLDEN, "int8_textbook.json")))
    group = np.array([-g["group_absmax"], g["weight"], 0.5, g["group_absmax"]], np.float32)
    codes, scale = O.absmax_int_quantize(group, g["qmax"], signed=True)
    assert abs(float(scale) - g["step"]) < 1e-7
    assert codes[1] == g["code"] and codes[0] == -127 and codes[3] == 127
    back = O.absmax_int_dequantize(codes, scale)
    assert abs(float(back[1]) - g["dequantized"]) < 1e-6
    assert abs(abs(float(back[1]) - g["weight"]) - g["error"]) < 1e-6
    vals = O.absmax_int_dequantize(np.array(g["step_examples"]["codes"]), np.float32(0.01))
    assert np.allclose(vals, g["step_examples"]["values"], atol=1e-7)
    _, big = O.absmax_int_quantize(np.array([g["outlier_example"]["absmax"], 0.3], np.float32),
                                   g["qmax"], signed=True)
    assert abs(float(big) - g["outlier_example"]["step"]) < 1e-7


def test_unsigned_second_level_matches_textbook_scheme():
    """The 8-bit scale codes are the textbook absmax scheme with qmax = 255 on non-negative
    values (UINT8: "QLoRA in LLMs" section 1)."""
    c1 = np.abs(_rand_w(1, 700, 31)).reshape(-1)
    q8, s2 = O.double_quantize(c1)
    for g in range(s2.size):
        seg = c1[g * 256:(g + 1) * 256]
        codes, scale = O.absmax_int_quantize(seg, 255, signed=False)
        assert scale == s2[g]
        assert np.array_equal(codes, q8[g * 256:(g + 1) * 256].astype(np.int64))


def test_second_level_ties_round_half_to_even():
    """c1 / s2 exactly halfway between two integers rounds to the even one, as Python's
    built-in round does: one group whose largest scale is 255 * 2^-8 (so s2 = 2^-8 exactly)
    and whose other scales are (k + 1/2) * 2^-8, k = 0 .. 254."""
    c1 = [255.0 * 2.0 ** -8] + [(k + 0.5) * 2.0 ** -8 for k in range(255)]
    W = np.zeros((256, 64), np.float32)
    W[:, 0] = np.array(c1, np.float32)
    W[:, 1] = -0.5 * W[:, 0]              # a second, smaller weight in every block
    p = O.nf4_quantize(W.reshape(4, 4096))
    assert p.absmax_s2[0] == np.float32(2.0 ** -8)
    want = [255] + [round(k + 0.5) for k in range(255)]
    assert [int(v) for v in p.absmax_q8] == want
    assert any(w % 2 == 0 and w < k + 0.5 for k, w in enumerate(want[1:]))  # ties went down too


def test_dequantize_multiplies_level_by_the_block_scale():
    """w' = bf16(level * k) with k = fp32(q8 * s2): each product formed exactly in double and
    rounded once to fp32, then to bf16 by torch's cast. The (level, q8, s2) triples are chosen
    where the other order, (level * q8) * s2, gives a different bf16 weight, so a swapped order
    fails; the fp32 values before the bf16 rounding are compared on a random block set too."""
    import torch

    def bf16_bits(x):
        return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16) \
            .view(torch.int16).numpy().view(np.uint16)

    q = O.nf4_codebook()
    found = []                                   # (s2, q8, code) where the orders differ
    for seed in range(40):
        r = np.random.default_rng(seed)
        s2 = r.uniform(1e-5, 1e-3, 64).astype(np.float32)
        q8 = r.integers(1, 256, (64, 256)).astype(np.float32)
        k = (q8.astype(np.float64) * s2[:, None]).astype(np.float32)
        exact = (q.astype(np.float64)[None, None, :] * k[..., None]).astype(np.float32)
        other = ((q[None, None, :] * q8[..., None]).astype(np.float32) * s2[:, None, None])
        i, j, c = np.nonzero(bf16_bits(exact) != bf16_bits(other.astype(np.float32)))
        found += [(s2[a], int(q8[a, b]), int(cc)) for a, b, cc in zip(i, j, c)]
        if len(found) >= 8:
            break
    assert len(found) >= 8
    # one group per triple: its first block holds the triple's scale code and only its code
    ng = len(found)
    rng = np.random.default_rng(1)
    codes = rng.integers(0, 16, (ng * 256, 64)).astype(np.uint8)
    q8 = rng.integers(1, 256, ng * 256).astype(np.uint8)
    s2 = np.array([f[0] for f in found], np.float32)
    for g, (_, qq, cc) in enumerate(found):
        q8[g * 256], codes[g * 256] = qq, cc
    p = O.NF4Packed(O.pack_nibbles(codes.reshape(-1)), q8, s2, ng * 256, 64, None)
    k = (q8.astype(np.float64) * s2[np.arange(ng * 256) // 256].astype(np.float64)).astype(np.float32)
    exact = (q[codes].astype(np.float64) * k[:, None].astype(np.float64)).astype(np.float32)
    assert np.array_equal(O.nf4_dequantize_f32(p), exact)
    assert np.array_equal(O.nf4_dequantize_bits(p), bf16_bits(exact))


def test_weight_on_a_threshold_takes_the_lower_code():
    """x = w / c1 equal to a threshold m[i] (the tie of two nearest levels) gives code i, the
    lower level, and a weight one fp32 step above it gives code i + 1. Blocks have c1 = 1 so
    that x equals the weight exactly."""
    mids = O.nf4_midpoints()
    W = np.zeros((15, 2, 64), np.float32)
    W[:, :, 0] = 1.0
    W[:, 0, 1] = mids
    W[:, 1, 1] = np.nextafter(mids, np.float32(2.0))
    codes = O.unpack_nibbles(O.nf4_quantize(W.reshape(15, 128)).codes).reshape(15, 2, 64)
    assert np.array_equal(codes[:, 0, 1], np.arange(15))
    assert np.array_equal(codes[:, 1, 1], np.arange(1, 16))
