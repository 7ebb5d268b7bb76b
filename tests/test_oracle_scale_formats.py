"""Pins of the oracle's other 8-bit formats for the block scales ("QLoRA in LLMs" §1: FP8 E4M3
has 4 exponent and 3 fraction bits; §2 "Choose a scale, then round": symmetric absmax to
-127 .. 127).

E4M3 decoding and round-to-nearest-even encoding are checked against torch's float8_e4m3fn
(an independent implementation) on every code, on random values, on every midpoint (the ties)
and in the subnormal range; the signed scheme against the textbook worked example; every format
against its rounding bound; and the codes are the same whatever the scale format."""

import json
import os

import numpy as np
import torch

from oracle import nf4_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_e4m3_decoding_matches_torch_on_every_code():
    codes = np.arange(256)
    mine = O.e4m3_value(codes)
    ref = torch.tensor(codes, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    assert np.array_equal(np.isnan(mine), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(mine[ok], ref[ok])
    # the format's landmarks
    assert O.e4m3_value(0x7E) == 448.0 and O.e4m3_value(0x01) == 2.0 ** -9
    assert O.e4m3_value(0x08) == 2.0 ** -6 and np.isnan(O.e4m3_value(0x7F))
    assert O.e4m3_value(0x38) == 1.0


def test_e4m3_encoding_matches_torch():
    rng = np.random.default_rng(0)
    vals = O.e4m3_value(np.arange(0x7F)).astype(np.float64)
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)          # exact ties
    x = np.concatenate([rng.uniform(0, 448, 200_000), rng.uniform(0, 2.0 ** -5, 20_000),
                        vals, mids]).astype(np.float32)
    mine = O.e4m3_encode(x)
    ref = torch.tensor(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(mine, ref)
    # ties go to the even code
    assert np.all(O.e4m3_encode(mids) % 2 == 0)
    # saturation above the largest finite value
    assert list(O.e4m3_encode(np.array([448.0, 455.0, 470.0, 1e6], np.float32))) == [0x7E] * 4


def test_signed_scales_reproduce_the_textbook_example():
    g = json.load(open(os.path.join(GOLDEN, "int8_textbook.json")))
    # a group of block scales whose largest is the example's 1.27: the step is 0.01 and the
    # example weight's magnitude 0.826 becomes 83
    c1 = np.array([g["group_absmax"], abs(g["weight"]), 0.0], dtype=np.float32)
    q8, s2 = O.double_quantize_with(c1, O.SCALES_S8)
    assert np.isclose(s2[0], g["step"], rtol=1e-6)
    assert list(q8.view(np.int8)) == [g["qmax"], abs(g["code"]), 0]
    k = O.scale_code_values(q8, O.SCALES_S8) * s2[0]
    assert np.isclose(k[1], abs(g["dequantized"]), rtol=1e-6)


def _c1(n=5000, seed=1):
    rng = np.random.default_rng(seed)
    c1 = np.abs(rng.standard_normal(n)).astype(np.float32) * np.float32(0.05)
    c1[::97] *= np.float32(8.0)           # outlier blocks
    c1[5] = 0.0
    return c1


def test_each_format_within_its_rounding_bound():
    c1 = _c1()
    g = np.arange(c1.size) // O.GROUP
    for fmt in (O.SCALES_U8, O.SCALES_S8, O.SCALES_E4M3):
        q8, s2 = O.double_quantize_with(c1, fmt)
        k = (O.scale_code_values(q8, fmt) * s2[g]).astype(np.float64)
        err = np.abs(k - c1.astype(np.float64))
        if fmt == O.SCALES_E4M3:
            # half a unit in the last place: 2^-4 relative for normals, 2^-10 s2 below 2^-6
            bound = np.maximum(2.0 ** -4 * c1, 2.0 ** -10 * s2[g]) * (1 + 1e-6) + 1e-12
        else:
            bound = 0.5 * s2[g].astype(np.float64) * (1 + 1e-5) + 1e-12
        assert np.all(err <= bound), fmt
        vals = O.scale_code_values(q8, fmt)
        assert np.all(vals >= 0)                       # absmax scales are never negative
        top = O.E4M3_MAX if fmt == O.SCALES_E4M3 else (127 if fmt == O.SCALES_S8 else 255)
        assert vals.max() == top                       # each group's largest maps to the top code


def test_codes_do_not_depend_on_the_scale_format():
    rng = np.random.default_rng(2)
    W = (rng.standard_normal((24, 640)) * 0.02).astype(np.float32)
    ps = [O.quantize_format(W, 0, f) for f in (O.SCALES_U8, O.SCALES_S8, O.SCALES_E4M3)]
    for p in ps[1:]:
        assert np.array_equal(p.codes, ps[0].codes)
    # the default format is the plain quantizer, bit for bit
    ref = O.nf4_quantize(W)
    assert np.array_equal(ps[0].absmax_q8, ref.absmax_q8)
    assert np.array_equal(O.dequantize_bits_format(ps[0], 0, O.SCALES_U8), O.nf4_dequantize_bits(ref))


def test_error_ordering_on_normal_weights():
    # half the codes (signed) or 3 fraction bits (E4M3) cost reconstruction accuracy
    rng = np.random.default_rng(3)
    W = (rng.standard_normal((256, 4096)) * 0.02).astype(np.float32)
    err = []
    for f in (O.SCALES_U8, O.SCALES_S8, O.SCALES_E4M3):
        d = O.bf16_bits_to_f32(O.dequantize_bits_format(O.quantize_format(W, 0, f), 0, f))
        err.append(float(((d - W) ** 2).mean()))
    assert err[0] < err[1] < err[2]


def _bf16_bits(x):
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16) \
        .view(torch.int16).numpy().view(np.uint16)


def test_format_dequantize_multiplies_level_by_the_block_scale():
    """In every scale format w' = bf16(level * k), k = fp32(value(q8) * s2): the products are
    formed exactly in double and rounded once (value(q8) has at most 8 significant bits),
    then cast to bf16 by torch. The (value, s2) pairs are picked where the other order,
    (level * value) * s2, gives another bf16 weight for some level, so a swapped order fails."""
    q = O.nf4_codebook()
    codes_of = {O.SCALES_U8: np.arange(1, 256), O.SCALES_S8: np.arange(1, 128),
                O.SCALES_E4M3: np.arange(0x08, 0x7F)}
    for fmt, cand in codes_of.items():
        vals = O.scale_code_values(cand.astype(np.uint8), fmt).astype(np.float64)
        found = []                                      # (s2, code byte, level index)
        for seed in range(5000):
            s2 = np.float32(np.random.default_rng(seed).uniform(1e-5, 1e-3))
            k = (vals * np.float64(s2)).astype(np.float32)
            exact = (q.astype(np.float64)[None, :] * k[:, None]).astype(np.float32)
            other = ((q[None, :] * vals.astype(np.float32)[:, None]).astype(np.float32) * s2)
            i, c = np.nonzero(_bf16_bits(exact) != _bf16_bits(other.astype(np.float32)))
            found += [(s2, int(cand[a]), int(b)) for a, b in zip(i, c)]
            if len(found) >= 2:
                break
        assert len(found) >= 2, fmt
        ng = len(found)
        rng = np.random.default_rng(2)
        codes = rng.integers(0, 16, (ng * 256, 64)).astype(np.uint8)
        q8 = rng.choice(cand, ng * 256).astype(np.uint8)
        s2 = np.array([f[0] for f in found], np.float32)
        for g, (_, qq, cc) in enumerate(found):
            q8[g * 256], codes[g * 256] = qq, cc
        p = O.NF4Packed(O.pack_nibbles(codes.reshape(-1)), q8, s2, ng * 256, 64, None)
        v = O.scale_code_values(q8, fmt).astype(np.float64)
        k = (v * s2[np.arange(ng * 256) // 256].astype(np.float64)).astype(np.float32)
        exact = (q[codes].astype(np.float64) * k[:, None].astype(np.float64)).astype(np.float32)
        got = O.dequantize_bits_format(p, 0, fmt)
        assert np.array_equal(got, _bf16_bits(exact)), fmt
