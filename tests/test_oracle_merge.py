"""Pins of the oracle's adapter merge ("QLoRA in LLMs" §11): against explicit loops, the
special cases that reduce it to a known matrix, its linearity, and the defining identity
that the merged weight gives the unmerged layer's output."""

import numpy as np

from oracle import nf4_oracle as O


def _case(o=12, h=128, r=16, seed=0):
    rng = np.random.default_rng(seed)
    Wt = (rng.standard_normal((o, h)) * 0.02).astype(np.float32)
    Wdq = O.nf4_dequantize(O.nf4_quantize(Wt))
    L1 = O.bf16_round(rng.standard_normal((h, r)).astype(np.float32) * 0.01)
    L2 = O.bf16_round(rng.standard_normal((r, o)).astype(np.float32) * 0.01)
    return Wdq, L1, L2


def test_merge_against_explicit_loops():
    Wdq, L1, L2 = _case(o=5, h=64, r=16, seed=1)
    s = 0.75
    got = O.merge_adapters(Wdq, L1, L2, s)
    for j in range(5):
        for k in range(0, 64, 7):
            ref = float(Wdq[j, k]) + s * sum(float(L2[c, j]) * float(L1[k, c]) for c in range(16))
            assert abs(got[j, k] - ref) <= 1e-15 * max(1.0, abs(ref))


def test_merge_special_cases():
    Wdq, L1, L2 = _case(seed=2)
    assert np.array_equal(O.merge_adapters(Wdq, np.zeros_like(L1), L2, 3.0), Wdq.astype(np.float64))
    assert np.array_equal(O.merge_adapters(Wdq, L1, L2, 0.0), Wdq.astype(np.float64))
    got = O.merge_adapters(np.zeros_like(Wdq), L1, L2, 2.0)
    np.testing.assert_allclose(got, 2.0 * (L1.astype(np.float64) @ L2.astype(np.float64)).T, rtol=1e-14)


def test_merge_is_linear_in_s():
    Wdq, L1, L2 = _case(seed=3)
    a = O.merge_adapters(Wdq, L1, L2, 0.5) - Wdq
    b = O.merge_adapters(Wdq, L1, L2, 1.5) - Wdq
    np.testing.assert_allclose(b, 3.0 * a, rtol=1e-13, atol=1e-18)


def test_merged_weight_reproduces_the_unmerged_layer():
    Wdq, L1, L2 = _case(o=24, h=192, r=32, seed=4)
    X = O.bf16_round(np.random.default_rng(5).standard_normal((7, 192)).astype(np.float32))
    s = 0.25
    Y_unmerged, _ = O.qlora_linear_fwd(X, Wdq, L1, L2, s)
    Y_merged = X.astype(np.float64) @ O.merge_adapters(Wdq, L1, L2, s).T
    np.testing.assert_allclose(Y_merged, Y_unmerged, rtol=1e-12, atol=1e-15)


def test_merge_bound_covers_fp32_evaluation():
    """An fp32 evaluation (products summed in fp32, scaled, added to W') stays inside the
    stated bound; the bound is not vacuous (below 1e-4 of the largest merged weight)."""
    Wdq, L1, L2 = _case(o=16, h=256, r=64, seed=6)
    s = np.float32(0.25)
    acc = np.zeros((16, 256), np.float32)
    for c in range(64):
        acc = (acc + np.outer(L2[c].astype(np.float32), L1[:, c].astype(np.float32))).astype(np.float32)
    got = (Wdq.astype(np.float32) + (s * acc).astype(np.float32)).astype(np.float64)
    ref = O.merge_adapters(Wdq, L1, L2, float(s))
    bound = O.merge_error_bound(Wdq, L1, L2, float(s))
    assert np.all(np.abs(got - ref) <= bound)
    assert np.max(bound) < 1e-4 * np.max(np.abs(ref))
