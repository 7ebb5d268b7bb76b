"""Pins of the oracle's NF4 codebook and bf16 rounding against facts outside the oracle.

* Standard-normal quantiles: an independent implementation (Python's statistics.NormalDist,
  Wichura's AS241 rational approximation) rebuilds the codebook to within 1 fp32 ulp.
* The pages' properties ("QLoRA in LLMs" section 5; "Idea one: NF4"; "Key Components"):
  16 levels, exact zero, ends normalised to -1 and +1, levels sit at normal quantiles, and
  for normal data every level is used about equally often.
* bf16 rounding ("QLoRA in LLMs" section 1): agrees with torch's fp32 -> bf16 cast.
"""

import os
import statistics

import numpy as np
import pytest
import torch

from oracle import nf4_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "nf4_codebook.txt")


def _ulp_diff_f32(a, b):
    ia = np.asarray(a, np.float32).view(np.int32).astype(np.int64)
    ib = np.asarray(b, np.float32).view(np.int32).astype(np.int64)
    return np.abs(ia - ib)


def test_codebook_shape_and_exact_points():
    q = O.nf4_codebook()
    assert q.dtype == np.float32 and q.shape == (16,)
    assert np.all(np.diff(q) > 0), "levels must be distinct and ascending"
    assert q[O.ZERO_CODE] == 0.0 and q[0] == -1.0 and q[15] == 1.0
    assert (q > 0).sum() == 8 and (q < 0).sum() == 7


def test_quantile_function_against_stdlib():
    nd = statistics.NormalDist()
    for p in [1e-6, 0.01, 0.2, 0.5, 0.61, 0.9, 0.96770833, 0.999999]:
        a, b = O.normal_quantile(p), nd.inv_cdf(p)
        # the quantile is only as well defined as p itself: one ulp of p over the density
        cond = 4 * np.spacing(p) / nd.pdf(b)
        assert abs(a - b) <= cond + 1e-13 * max(1.0, abs(b)), (p, a, b)


def test_codebook_rebuilt_with_stdlib_quantiles():
    nd = statistics.NormalDist()
    pos_p, neg_p = O.nf4_construction_probabilities()
    top = nd.inv_cdf(O.nf4_tail_probability())
    ref = sorted([nd.inv_cdf(p) / top for p in pos_p]
                 + [-nd.inv_cdf(p) / top for p in neg_p] + [0.0])
    assert np.max(_ulp_diff_f32(O.nf4_codebook(), np.array(ref, np.float32))) <= 1


def test_midpoints():
    q = O.nf4_codebook().astype(np.float64)
    m = O.nf4_midpoints()
    assert m.shape == (15,)
    assert np.all(m.astype(np.float64) > q[:-1]) and np.all(m.astype(np.float64) < q[1:])
    assert np.max(np.abs(m.astype(np.float64) - (q[:-1] + q[1:]) / 2)) <= 6e-8


def test_golden_table_matches_oracle():
    levels, mids = {}, {}
    with open(GOLDEN) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            kind, idx, hexv, _ = line.split()
            val = np.array([int(hexv, 16)], np.uint32).view(np.float32)[0]
            (levels if kind == "level" else mids)[int(idx)] = val
    assert np.array_equal(np.array([levels[i] for i in range(16)], np.float32), O.nf4_codebook())
    assert np.array_equal(np.array([mids[i] for i in range(15)], np.float32), O.nf4_midpoints())


@pytest.fixture(scope="module")
def normal_draws():
    n = 10_000_000
    z = np.random.default_rng(0).standard_normal(n)
    return z / O.normal_quantile(O.nf4_tail_probability())


def test_levels_sit_at_normal_quantiles(normal_draws):
    """Empirical CDF of scaled N(0,1) draws at each level equals its construction
    probability (within 5/sqrt(N)): the levels are normal quantiles, correctly scaled."""
    x = np.sort(normal_draws)
    n = x.size
    q = O.nf4_codebook_f64()
    pos_p, neg_p = O.nf4_construction_probabilities()
    pos_levels = sorted(q[q > 0], reverse=True)        # descending: p = delta, ...
    neg_levels = sorted(q[q < 0])                      # ascending: -1 first
    for lvl, p in zip(pos_levels, pos_p):
        cdf = np.searchsorted(x, lvl, side="right") / n
        assert abs(cdf - p) <= 5 / np.sqrt(n), (lvl, cdf, p)
    for lvl, p in zip(neg_levels, neg_p):
        cdf = np.searchsorted(x, lvl, side="right") / n
        assert abs(cdf - (1 - p)) <= 5 / np.sqrt(n), (lvl, cdf, 1 - p)


def test_equal_occupancy_for_normal_data(normal_draws):
    """Nearest-level occupancy of normal data is close to 1/16 for every code."""
    q = O.nf4_codebook_f64()
    mids = (q[:-1] + q[1:]) / 2
    codes = np.searchsorted(mids, normal_draws, side="left")
    occ = np.bincount(codes, minlength=16) / normal_draws.size
    assert np.all(occ >= 0.85 / 16) and np.all(occ <= 1.20 / 16), occ * 16


def test_bf16_rounding_matches_torch_cast():
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.standard_normal(100_000).astype(np.float32),
        (rng.standard_normal(10_000) * 1e-30).astype(np.float32),
        (rng.standard_normal(10_000) * 1e30).astype(np.float32),
        # exact ties between two bf16 values, both parities of the kept bit
        (np.arange(0, 4096, dtype=np.uint32) << 16 | 0x8000).view(np.float32),
        np.array([0.0, -0.0, np.inf, -np.inf, 3.3895314e38, 1e-45], np.float32),
    ])
    ours = O.bf16_bits_rne(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    nan_bits = O.bf16_bits_rne(np.array([np.nan], np.float32))
    assert np.isnan(O.bf16_bits_to_f32(nan_bits))[0]
    # NaNs whose payload lies only in the 16 bits the rounding drops stay NaN (not infinity),
    # as torch's cast keeps them NaN
    odd = np.array([0x7F800001, 0xFF800001, 0x7F80FFFF, 0x7FFFFFFF], np.uint32).view(np.float32)
    assert np.all(np.isnan(O.bf16_bits_to_f32(O.bf16_bits_rne(odd))))
    assert torch.isnan(torch.from_numpy(odd).to(torch.bfloat16)).all()
