"""GPU parity of the LoRA-dropout calls against the CPU oracle ("QLoRA in LLMs" section 12: a
LoRA dropout of 0.05 in the example configuration; read as inverted dropout on the adapter
branch's input).

The keep mask is checked bit for bit (qlora_dropout_apply and the forward's mask bits against the
oracle's own Philox4x32-10 draw); the backward runs with the forward's mask and with a redrawn
one; the products within 2e-2 x RMS of the oracle's fp64 values for the same mask. Because
the adapter term is about 1% of Y and dX for the usual weight and adapter scales, a wrong mask
there would hide under that bound: a zero weight (every code the zero level, scales 0, W' = 0
exactly) leaves Y and dX with nothing but the adapter term, and dX must then be exactly 0 at
every dropped element."""

import numpy as np
import pytest
import torch

from bit_quantized_lora_03_b200 import binding as B
from bit_quantized_lora_03_b200 import inputs
from oracle import nf4_oracle as O

from gpu_util import assert_close_rms, f32, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().view(torch.int16).numpy().astype(np.uint16)


def _tie_p(t: int, h: int, seed: int) -> float:
    """A dropout probability whose threshold equals one of the draws of this (t, h, seed):
    the first word with its low 8 bits zero, over 2^32 (exact in fp32)."""
    n = t * h
    ctr = np.zeros((n // 4, 4), np.uint64)
    ctr[:, 0] = np.arange(n // 4, dtype=np.uint64)
    words = O.philox4x32_10(ctr, (seed, 0)).reshape(-1)
    w = int(words[np.nonzero(((words & 0xFF) == 0) & (words > 0))[0][0]])
    return w / 2.0 ** 32


@pytest.mark.parametrize("t,h,p,seed", [
    (1, 64, 0.05, 0),
    (37, 320, 0.5, 123),
    (256, 4096, 0.05, (1 << 40) + 7),   # seed with a non-zero high half
    (5, 128, 0.0, 9),                   # p = 0 keeps everything
    (64, 640, 0.9, (1 << 64) - 1),
    (3, 64, 1e-12, 4),                  # below 2^-32: threshold 0
    (16, 256, _tie_p(16, 256, 777), 777),  # one draw equals the threshold: that element is kept
])
def test_dropout_mask_bit_exact(t, h, p, seed):
    X = inputs.normal_bf16((t, h), 1.0, inputs._gen(900 + t))
    Xd = B.qlora_dropout_apply(X.cuda(), p, seed)
    assert B.last_status() == 0
    keep = O.dropout_keep_mask(t, h, p, seed)
    ref = np.where(keep, _bits(X), np.uint16(0))
    assert np.array_equal(_bits(Xd), ref)


def _run(li, p, seed, pass_sT=True, pass_mask=True):
    P = B.nf4_quantize(li.Wt.cuda())
    X, L1, L2 = li.X.cuda(), li.L1.cuda(), li.L2.cuda()
    Y, sT, mask = B.qlora_linear_fwd_dropout(X, P, L1, L2, li.s, p, seed, want_mask=True)
    dX, dL1, dL2 = B.qlora_linear_bwd_dropout(li.dY.cuda(), X, P, L1, L2, li.s, p, seed,
                                              sT=sT if pass_sT else None,
                                              mask=mask if pass_mask else None)
    assert B.last_status() == 0
    keep = O.dropout_keep_mask(li.t, li.X.shape[1], p, seed)
    assert np.array_equal(mask.cpu().numpy(), np.packbits(keep.reshape(-1), bitorder="little")), \
        "mask bits"
    return P, Y, sT, dX, dL1, dL2


def _oracle(li, p, seed):
    Wdq = O.nf4_dequantize(O.nf4_quantize(li.Wt.numpy()))
    keep = O.dropout_keep_mask(li.t, li.X.shape[1], p, seed)
    X, L1, L2, dY = f32(li.X), f32(li.L1), f32(li.L2), f32(li.dY)
    Y, sT = O.qlora_linear_fwd_dropout(X, Wdq, L1, L2, li.s, keep, p)
    dX, dL1, dL2 = O.qlora_linear_bwd_dropout(dY, X, Wdq, L1, L2, li.s, keep, p)
    return keep, Y, sT, dX, dL1, dL2


CASES = [
    # t, h, o, r, s, p, seed
    (1, 320, 576, 16, 2.0, 0.05, 1),       # decode GEMV forward
    (9, 320, 576, 16, 2.0, 0.3, 2),        # GEMV with two token groups
    (17, 320, 576, 16, 2.0, 0.05, 3),      # first token count on the GEMM path
    (128, 256, 256, 64, 0.25, 0.5, 4),     # exactly one tile
    (300, 320, 576, 48, 0.5, 0.1, 5),      # ragged M, N, LoRA K
    (257, 640, 320, 80, 1.0, 0.05, 6),     # two LoRA K-steps, ragged
]


@pytest.mark.parametrize("t,h,o,r,s,p,seed", CASES)
def test_dropout_fwd_bwd(t, h, o, r, s, p, seed):
    li = inputs.random_linear(t, h, o, r, s, seed=700 + t + r)
    keep, *ref = _oracle(li, p, seed)
    for pass_sT, pass_mask in ((True, True), (False, False), (True, False)):
        _, *got = _run(li, p, seed, pass_sT, pass_mask)
        for name, g, rf in zip(("Y", "sT", "dX", "dL1", "dL2"), got, ref):
            assert_close_rms(f32(g), rf, name)


def _assert_within_rounding(got, ref, mag, name):
    """Elementwise bound for an output that is a rank-r product through one bf16 intermediate
    and then rounded to bf16 (Y = bf16(sT.L2), dX = bf16(E) with E = bf16(M (.) sU.L1^T) for a
    zero weight): the intermediate's rounding moves each term by at most 2^-8 of its magnitude
    (mag = |intermediate| . |other factor|), the final rounding the result by at most 2^-8 of
    itself, and fp32 accumulation adds far less than the 10% margin."""
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    bound = 2.0 ** -8 * np.abs(ref) + 1.1 * 2.0 ** -8 * mag
    bad = np.abs(got - ref) > bound
    assert not bad.any(), f"{name}: {int(bad.sum())} elements outside the rounding bound"


@pytest.mark.parametrize("t,h,o,r,p", [(5, 256, 320, 16, 0.3), (300, 320, 576, 48, 0.3),
                                       (130, 4096, 256, 64, 0.05)])
def test_zero_weight_isolates_the_adapter_term(t, h, o, r, p):
    li = inputs.random_linear(t, h, o, r, 2.0, seed=800 + t)
    li.Wt.zero_()
    seed = 4000 + t
    keep, Y_ref, sT_ref, dX_ref, dL1_ref, dL2_ref = _oracle(li, p, seed)
    _, Y, sT, dX, dL1, dL2 = _run(li, p, seed, pass_mask=t % 2 == 0)
    for name, g, rf in (("sT", sT, sT_ref), ("dL1", dL1, dL1_ref), ("dL2", dL2, dL2_ref)):
        assert_close_rms(f32(g), rf, name)
    # Y and dX are nothing but the adapter term here, each through one bf16 intermediate
    L1, L2, dY = (f32(a).astype(np.float64) for a in (li.L1, li.L2, li.dY))
    _assert_within_rounding(f32(Y), Y_ref, np.abs(sT_ref) @ np.abs(L2), "Y")
    sU_ref = li.s * O.dropout_scale(p) * (dY @ L2.T)
    _assert_within_rounding(f32(dX), dX_ref, keep * (np.abs(sU_ref) @ np.abs(L1).T), "dX")
    dXb = _bits(dX)
    assert not dXb[~keep].any(), "dX must be exactly 0 where the adapter input was dropped"
    assert (dXb[keep] != 0).mean() > 0.99


def test_p_zero_is_the_plain_layer_bit_for_bit():
    li = inputs.random_linear(200, 320, 576, 32, 0.5, seed=13)
    P = B.nf4_quantize(li.Wt.cuda())
    X, L1, L2, dY = li.X.cuda(), li.L1.cuda(), li.L2.cuda(), li.dY.cuda()
    Y0, sT0 = B.qlora_linear_fwd(X, P, L1, L2, li.s)
    g0 = B.qlora_linear_bwd(dY, X, P, L1, L2, li.s, sT=sT0)
    Y1, sT1, mask = B.qlora_linear_fwd_dropout(X, P, L1, L2, li.s, 0.0, 77, want_mask=True)
    g1 = B.qlora_linear_bwd_dropout(dY, X, P, L1, L2, li.s, 0.0, 77, sT=sT1, mask=mask)
    assert B.last_status() == 0
    assert bool((mask == 255).all())
    for a, b in zip((Y0, sT0, *g0), (Y1, sT1, *g1)):
        assert torch.equal(a, b)


def test_seed_changes_the_mask_and_the_gradients():
    li = inputs.random_linear(256, 256, 256, 16, 1.0, seed=14)
    a = _run(li, 0.1, 1)
    b = _run(li, 0.1, 2)
    assert not torch.equal(a[4], b[4])      # dL1
    c = _run(li, 0.1, 1)
    for x, y in zip(a[1:], c[1:]):           # same seed: same results
        assert torch.equal(x, y)


def test_training_shape_linear_with_dropout():
    """up_proj of the LLaMA-7B layer (h = 4096, o = 11008, r = 64, t = 4096), dropout 0.05:
    the full sT, dL1 and dL2 and 128 seeded rows of Y and dX."""
    li = inputs.training_linear(5)
    p, seed = 0.05, 0x5EED_0005
    _, Y, sT, dX, dL1, dL2 = _run(li, p, seed)
    Wdq = O.nf4_dequantize(O.nf4_quantize(li.Wt.numpy()))
    keep = O.dropout_keep_mask(li.t, 4096, p, seed)
    X, L1, L2, dY = f32(li.X), f32(li.L1), f32(li.L2), f32(li.dY)
    rows = torch.randperm(li.t, generator=torch.Generator().manual_seed(5))[:128].numpy()
    Yr, sTr = O.qlora_linear_fwd_dropout(X[rows], Wdq, L1, L2, li.s, keep[rows], p)
    assert_close_rms(f32(Y)[rows], Yr, "Y rows")
    dXr, _, _ = O.qlora_linear_bwd_dropout(dY[rows], X[rows], Wdq, L1, L2, li.s, keep[rows], p)
    assert_close_rms(f32(dX)[rows], dXr, "dX rows")
    _, sT_ref = O.qlora_linear_fwd_dropout(X, Wdq, L1, L2, li.s, keep, p)
    assert_close_rms(f32(sT), sT_ref, "sT")
    _, dL1_ref, dL2_ref = O.qlora_linear_bwd_dropout(dY, X, Wdq, L1, L2, li.s, keep, p)
    assert_close_rms(f32(dL1), dL1_ref, "dL1")
    assert_close_rms(f32(dL2), dL2_ref, "dL2")
