"""Pins of the oracle's LoRA dropout ("QLoRA in LLMs" §12: a LoRA dropout of 0.05 in the
example configuration; the reading puts it on the adapter branch's input, scaled by 1/(1-p)).

The generator is pinned by its published known-answer vectors, the mask by its statistics and
its element-to-word layout, the products by what must hold whatever the mask: no dropout
reduces them to the plain layer, their average over masks is the plain layer, and the
adjoint, bilinearity and finite-difference identities for one fixed mask."""

import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import nf4_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_philox_known_answers():
    kat = json.load(open(os.path.join(GOLDEN, "philox4x32_10_kat.json")))
    assert kat["rounds"] == 10
    for v in kat["vectors"]:
        ctr = np.array([[int(x, 16) for x in v["counter"]]], dtype=np.uint64)
        key = np.array([int(x, 16) for x in v["key"]], dtype=np.uint64)
        got = O.philox4x32_10(ctr, key)[0]
        assert [int(x) for x in got] == [int(x, 16) for x in v["output"]]


def test_philox_is_a_function_of_counter_and_key_only():
    ctr = np.array([[i, 0, 0, 0] for i in range(64)], dtype=np.uint64)
    a = O.philox4x32_10(ctr, (7, 9))
    b = O.philox4x32_10(ctr[::-1], (7, 9))[::-1]
    assert np.array_equal(a, b)
    assert not np.array_equal(a, O.philox4x32_10(ctr, (7, 10)))


def test_threshold():
    assert O.dropout_threshold(0.0) == 0
    assert O.dropout_threshold(0.5) == 2 ** 31
    assert O.dropout_threshold(0.25) == 2 ** 30
    p32 = float(np.float32(0.05))
    assert O.dropout_threshold(0.05) == math.floor(Fraction(p32) * 2 ** 32)
    for bad in (-0.1, 1.0, 1.5, float("nan")):
        with pytest.raises(ValueError):
            O.dropout_threshold(bad)


def test_mask_layout_against_known_answer():
    # seed 0 is key (0, 0); elements 0..3 take the four words of counter 0 in order
    kat = json.load(open(os.path.join(GOLDEN, "philox4x32_10_kat.json")))["vectors"][0]
    words = [int(x, 16) for x in kat["output"]]
    for p in (0.3, 0.5, 0.7, 0.9):
        thr = O.dropout_threshold(p)
        keep = O.dropout_keep_mask(1, 64, p, 0)
        assert list(keep[0, :4]) == [w >= thr for w in words]


def test_mask_depends_on_the_element_index_only():
    big = O.dropout_keep_mask(24, 128, 0.5, 1234)
    assert np.array_equal(O.dropout_keep_mask(5, 128, 0.5, 1234), big[:5])
    # the same flat index in another shape takes the same draw
    assert np.array_equal(O.dropout_keep_mask(12, 256, 0.5, 1234).reshape(-1), big.reshape(-1))
    # the high half of the seed is part of the key
    assert not np.array_equal(O.dropout_keep_mask(24, 128, 0.5, 1234 + (1 << 32)), big)


def test_mask_statistics():
    t, h, p = 512, 1024, 0.05
    keep = O.dropout_keep_mask(t, h, p, 2024)
    drop = ~keep
    n = t * h
    sigma = math.sqrt(p * (1 - p) / n)
    assert abs(drop.mean() - p) < 5 * sigma
    # per-column and per-row counts: chi-square against the binomial, within 6 standard
    # deviations of its mean (dof = number of cells)
    for counts, m in ((drop.sum(axis=0), t), (drop.sum(axis=1), h)):
        e = m * p
        chi2 = float(((counts - e) ** 2 / (e * (1 - p))).sum())
        dof = counts.size
        assert abs(chi2 - dof) < 6 * math.sqrt(2 * dof)
    # neighbouring elements (same counter and across counters) are independent
    f = drop.reshape(-1)
    for lag in (1, 3, 4, 5, h):
        both = (f[:-lag] & f[lag:]).mean()
        assert abs(both - p * p) < 5 * math.sqrt(p * p * (1 - p * p) / (n - lag))
    # another seed gives an independent mask
    other = ~O.dropout_keep_mask(t, h, p, 2025)
    assert abs((drop & other).mean() - p * p) < 5 * math.sqrt(p * p / n)
    # p = 0 keeps everything
    assert O.dropout_keep_mask(8, 64, 0.0, 99).all()


def _case(t=6, h=64, o=48, r=16, seed=0):
    rng = np.random.default_rng(seed)
    Wt = (rng.standard_normal((o, h)) * 0.02).astype(np.float32)
    Wdq = O.nf4_dequantize(O.nf4_quantize(Wt))
    X = O.bf16_round(rng.standard_normal((t, h)).astype(np.float32))
    L1 = O.bf16_round(rng.standard_normal((h, r)).astype(np.float32) * 0.05)
    L2 = O.bf16_round(rng.standard_normal((r, o)).astype(np.float32) * 0.05)
    dY = O.bf16_round(rng.standard_normal((t, o)).astype(np.float32))
    return X, Wdq, L1, L2, dY


def test_no_dropout_is_the_plain_layer():
    X, Wdq, L1, L2, dY = _case()
    keep = np.ones(X.shape, dtype=bool)
    Y, sT = O.qlora_linear_fwd_dropout(X, Wdq, L1, L2, 0.5, keep, 0.0)
    Y0, sT0 = O.qlora_linear_fwd(X, Wdq, L1, L2, 0.5)
    assert np.array_equal(Y, Y0) and np.array_equal(sT, sT0)
    got = O.qlora_linear_bwd_dropout(dY, X, Wdq, L1, L2, 0.5, keep, 0.0)
    ref = O.qlora_linear_bwd(dY, X, Wdq, L1, L2, 0.5)
    for a, b in zip(got, ref[:3]):
        assert np.array_equal(a, b)


def test_all_dropped_leaves_the_base_product():
    X, Wdq, L1, L2, dY = _case(seed=3)
    keep = np.zeros(X.shape, dtype=bool)
    Y, sT = O.qlora_linear_fwd_dropout(X, Wdq, L1, L2, 0.5, keep, 0.3)
    assert np.array_equal(sT, np.zeros_like(sT))
    assert np.allclose(Y, O._f64(X) @ O._f64(Wdq).T, rtol=0, atol=1e-15)
    dX, dL1, dL2 = O.qlora_linear_bwd_dropout(dY, X, Wdq, L1, L2, 0.5, keep, 0.3)
    assert not dL1.any() and not dL2.any()
    assert np.allclose(dX, O._f64(dY) @ O._f64(Wdq), rtol=0, atol=1e-15)


def test_average_over_masks_is_the_plain_layer():
    # E[M / (1 - p)] = 1 and every output is linear in the mask, so the mean over independent
    # masks converges to the layer without dropout (this fails without the 1/(1-p) factor)
    X, Wdq, L1, L2, dY = _case(t=4, h=64, o=32, r=16, seed=5)
    p, s, n = 0.3, 2.0, 3000
    ref = list(O.qlora_linear_fwd(X, Wdq, L1, L2, s)[:1]) + list(O.qlora_linear_bwd(dY, X, Wdq, L1, L2, s)[:3])
    samples = [[] for _ in ref]
    for seed in range(n):
        keep = O.dropout_keep_mask(X.shape[0], X.shape[1], p, 77_000 + seed)
        Y, _ = O.qlora_linear_fwd_dropout(X, Wdq, L1, L2, s, keep, p)
        dX, dL1, dL2 = O.qlora_linear_bwd_dropout(dY, X, Wdq, L1, L2, s, keep, p)
        for acc, v in zip(samples, (Y, dX, dL1, dL2)):
            acc.append(v)
    for r_, acc in zip(ref, samples):
        a = np.stack(acc)
        mean, se = a.mean(axis=0), a.std(axis=0) / math.sqrt(n)
        z = np.abs(mean - r_) / np.maximum(se, 1e-300)
        moving = se > 0
        assert z[moving].max() < 5.5
        assert np.allclose(mean[~moving], r_[~moving], rtol=0, atol=1e-12)
        # the spread is real: dropout moved these outputs
        assert moving.mean() > 0.5


def test_adjoint_and_bilinearity_for_one_mask():
    X, Wdq, L1, L2, dY = _case(t=7, h=128, o=80, r=16, seed=8)
    p, s = 0.05, 0.25
    keep = O.dropout_keep_mask(7, 128, p, 4242)
    assert (~keep).any()
    Y, sT = O.qlora_linear_fwd_dropout(X, Wdq, L1, L2, s, keep, p)
    dX, dL1, dL2 = O.qlora_linear_bwd_dropout(dY, X, Wdq, L1, L2, s, keep, p)
    X64, dY64 = O._f64(X), O._f64(dY)
    # Y is linear in X for a fixed mask
    lhs, rhs = float((dX * X64).sum()), float((dY64 * Y).sum())
    assert abs(lhs - rhs) <= 1e-12 * (abs(lhs) + 1)
    # Y's adapter term is linear in L1 and in L2 separately
    lora = float((dY64 * (Y - X64 @ O._f64(Wdq).T)).sum())
    assert abs(float((dL1 * O._f64(L1)).sum()) - lora) <= 1e-12 * (abs(lora) + 1)
    assert abs(float((dL2 * O._f64(L2)).sum()) - lora) <= 1e-12 * (abs(lora) + 1)


def test_finite_differences_for_one_mask():
    X, Wdq, L1, L2, dY = _case(t=3, h=64, o=64, r=16, seed=9)
    p, s = 0.2, 0.5
    keep = O.dropout_keep_mask(3, 64, p, 31337)
    X64, L1_64, L2_64, dY64 = (O._f64(a) for a in (X, L1, L2, dY))
    dX, dL1, dL2 = O.qlora_linear_bwd_dropout(dY, X, Wdq, L1, L2, s, keep, p)

    def loss(Xv, L1v, L2v):
        Y, _ = O.qlora_linear_fwd_dropout(Xv, Wdq, L1v, L2v, s, keep, p)
        return float((dY64 * Y).sum())

    eps = 1e-6
    assert (~keep).any() and keep.any()
    for i in range(3):                      # every element of dX, dropped and kept
        for j in range(64):
            E = np.zeros_like(X64); E[i, j] = eps
            fd = (loss(X64 + E, L1_64, L2_64) - loss(X64 - E, L1_64, L2_64)) / (2 * eps)
            assert abs(fd - dX[i, j]) < 1e-7 * (1 + abs(fd))
    rng = np.random.default_rng(0)
    for _ in range(6):
        j = rng.integers(64)
        k, c = rng.integers(64), rng.integers(16)
        E = np.zeros_like(L1_64); E[k, c] = eps
        fd = (loss(X64, L1_64 + E, L2_64) - loss(X64, L1_64 - E, L2_64)) / (2 * eps)
        assert abs(fd - dL1[k, c]) < 1e-7 * (1 + abs(fd))
        E = np.zeros_like(L2_64); E[c, j] = eps
        fd = (loss(X64, L1_64, L2_64 + E) - loss(X64, L1_64, L2_64 - E)) / (2 * eps)
        assert abs(fd - dL2[c, j]) < 1e-7 * (1 + abs(fd))


def test_backward_matches_torch_autograd():
    X, Wdq, L1, L2, dY = _case(t=5, h=64, o=32, r=16, seed=10)
    p, s = 0.1, 0.75
    keep = O.dropout_keep_mask(5, 64, p, 555)
    tX, tL1, tL2 = (torch.tensor(O._f64(a), requires_grad=True) for a in (X, L1, L2))
    tW = torch.tensor(O._f64(Wdq))
    M = torch.tensor(keep, dtype=torch.float64) / (1.0 - float(np.float32(p)))
    Y = tX @ tW.T + s * ((tX * M) @ tL1) @ tL2
    (Y * torch.tensor(O._f64(dY))).sum().backward()
    dX, dL1, dL2 = O.qlora_linear_bwd_dropout(dY, X, Wdq, L1, L2, s, keep, p)
    for got, ref in ((dX, tX.grad), (dL1, tL1.grad), (dL2, tL2.grad)):
        assert np.allclose(got, ref.numpy(), rtol=1e-12, atol=1e-14)


def test_a_draw_equal_to_the_threshold_is_kept():
    """The keep rule is draw >= threshold: find an element whose Philox word has its low 8
    bits zero (so word / 2^32 is exact in fp32), set p to that fraction, and check that the
    threshold equals the word and that the element is kept."""
    seed, t, h = 777, 16, 256
    n = t * h
    ctr = np.zeros((n // 4, 4), np.uint64)
    ctr[:, 0] = np.arange(n // 4, dtype=np.uint64)
    words = O.philox4x32_10(ctr, (seed, 0)).reshape(-1)      # element e takes word e
    hits = np.nonzero(((words & 0xFF) == 0) & (words > 0))[0]
    assert hits.size > 0
    e = int(hits[0])
    w = int(words[e])
    p = float(Fraction(w, 2 ** 32))
    assert float(np.float32(p)) == p and O.dropout_threshold(p) == w
    keep = O.dropout_keep_mask(t, h, p, seed).reshape(-1)
    assert keep[e]
    assert np.array_equal(keep, words.astype(np.int64) >= w)
