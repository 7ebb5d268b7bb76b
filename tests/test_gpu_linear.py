"""GPU parity of qlora_linear_fwd / qlora_linear_bwd against the CPU oracle.

The oracle quantizes the same fp32 weight itself and computes Y, sT, dX, dL1, dL2 in fp64;
the bar is max|gpu - oracle| <= 2e-2 * RMS(oracle) per tensor. Shapes cover the decode GEMV
(t <= 16), the tcgen05 GEMM (t > 16) with several tiles and ragged tails in every dimension
(t not a multiple of 128, N not a multiple of 256, r below and above one 64-wide K-step), the
seeded single-linear workload, the decode-shape weights, and one full training-shape linear of
the LLaMA-7B layer with sampled rows of Y and dX and the full adapter gradients."""

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


def _oracle_weight(Wt: torch.Tensor) -> np.ndarray:
    return O.nf4_dequantize(O.nf4_quantize(Wt.numpy()))


def _run_fwd(li: inputs.LinearInputs):
    p = B.nf4_quantize(li.Wt.cuda())
    Y, sT = B.qlora_linear_fwd(li.X.cuda(), p, li.L1.cuda(), li.L2.cuda(), li.s)
    assert B.last_status() == 0
    return p, Y, sT


def _check_fwd(li: inputs.LinearInputs):
    p, Y, sT = _run_fwd(li)
    Wdq = _oracle_weight(li.Wt)
    Y_ref, sT_ref = O.qlora_linear_fwd(f32(li.X), Wdq, f32(li.L1), f32(li.L2), li.s)
    assert_close_rms(f32(Y), Y_ref, "Y")
    assert_close_rms(f32(sT), sT_ref, "sT")
    return p, Y, sT, Wdq


def _check_bwd(li: inputs.LinearInputs, p, sT, Wdq, pass_sT: bool):
    dX, dL1, dL2 = B.qlora_linear_bwd(li.dY.cuda(), li.X.cuda(), p, li.L1.cuda(), li.L2.cuda(),
                                      li.s, sT=sT if pass_sT else None)
    assert B.last_status() == 0
    dX_ref, dL1_ref, dL2_ref, _ = O.qlora_linear_bwd(f32(li.dY), f32(li.X), Wdq, f32(li.L1),
                                                    f32(li.L2), li.s)
    assert_close_rms(f32(dX), dX_ref, "dX")
    assert_close_rms(f32(dL1), dL1_ref, "dL1")
    assert_close_rms(f32(dL2), dL2_ref, "dL2")


def test_single_linear_1024_forward():
    _check_fwd(inputs.single_linear_1024())


@pytest.mark.parametrize("t", [1, 2, 7, 8, 9, 16])
def test_decode_gemv_small(t):
    _check_fwd(inputs.random_linear(t, 320, 576, 16, 2.0, seed=100 + t, with_grad=False))


@pytest.mark.parametrize("t,h,o,r,s", [
    (17, 320, 576, 16, 2.0),        # first token count on the GEMM path
    (128, 256, 256, 64, 0.25),      # exactly one tile
    (300, 320, 576, 48, 0.5),       # ragged M, N, LoRA K (48 < 64)
    (257, 640, 320, 80, 1.0),       # two LoRA K-steps, ragged
    (64, 64, 64, 16, 3.0),          # smallest shapes
])
def test_fwd_bwd_ragged(t, h, o, r, s):
    li = inputs.random_linear(t, h, o, r, s, seed=t * 7 + h + o + r)
    p, Y, sT, Wdq = _check_fwd(li)
    _check_bwd(li, p, sT, Wdq, pass_sT=True)
    _check_bwd(li, p, sT, Wdq, pass_sT=False)


def test_bwd_in_gemv_regime():
    li = inputs.random_linear(5, 256, 320, 16, 2.0, seed=11)
    p, Y, sT, Wdq = _check_fwd(li)
    _check_bwd(li, p, sT, Wdq, pass_sT=True)


def test_s_zero_is_plain_product():
    li = inputs.random_linear(200, 256, 320, 32, 0.0, seed=12)
    p, Y, sT, Wdq = _check_fwd(li)
    assert float(sT.abs().max()) == 0.0


def test_frozen_weight_unchanged_by_backward():
    li = inputs.random_linear(130, 256, 256, 16, 1.0, seed=13)
    p, Y, sT = _run_fwd(li)
    before = [p.codes.clone(), p.absmax_q8.clone(), p.absmax_s2.clone()]
    B.qlora_linear_bwd(li.dY.cuda(), li.X.cuda(), p, li.L1.cuda(), li.L2.cuda(), li.s, sT=sT)
    torch.cuda.synchronize()
    for a, b in zip(before, [p.codes, p.absmax_q8, p.absmax_s2]):
        assert torch.equal(a, b)


@pytest.mark.parametrize("t", [1, 4, 16])
def test_decode_shape_gemv_4096x11008(t):
    name, Wt = inputs.decode_gemv_weights()[0]
    o, h = Wt.shape
    L1, L2 = inputs.decode_gemv_adapters(h, o, 16)
    li = inputs.LinearInputs(name, Wt, inputs.decode_gemv_activations(h, t), L1, L2, 2.0)
    _check_fwd(li)


def test_training_shape_linear_sampled():
    """up_proj of the LLaMA-7B layer (h = 4096, o = 11008, r = 64, t = 4096): full dL1 and
    dL2, and 256 seeded rows of Y and dX (each row depends on one row of X or dY only)."""
    li = inputs.training_linear(5)
    p, Y, sT = _run_fwd(li)
    dX, dL1, dL2 = B.qlora_linear_bwd(li.dY.cuda(), li.X.cuda(), p, li.L1.cuda(), li.L2.cuda(),
                                      li.s, sT=sT)
    assert B.last_status() == 0
    Wdq = _oracle_weight(li.Wt)
    rows = torch.randperm(li.t, generator=torch.Generator().manual_seed(3))[:256].numpy()
    X, dY, L1, L2 = f32(li.X), f32(li.dY), f32(li.L1), f32(li.L2)
    assert_close_rms(f32(Y)[rows], O.qlora_linear_fwd_rows(rows, X, Wdq, L1, L2, li.s), "Y rows")
    assert_close_rms(f32(dX)[rows], O.qlora_linear_bwd_dx_rows(rows, dY, Wdq, L1, L2, li.s),
                     "dX rows")
    _, dL1_ref, dL2_ref, _ = O.qlora_linear_bwd(dY, X, Wdq, L1, L2, li.s)
    assert_close_rms(f32(dL1), dL1_ref, "dL1")
    assert_close_rms(f32(dL2), dL2_ref, "dL2")


@pytest.mark.parametrize("t,ctas", [(1, 1), (5, 3), (12, 1), (16, 2)])
def test_decode_gemv_long_warp_runs(t, ctas):
    """Few CTAs give every warp a long run of units: it crosses row tiles and scale segments
    (h = 64 x 67: 34 units per row, more than one 32-unit segment, the last unit one block)."""
    li = inputs.random_linear(t, 64 * 67, 576, 16, 1.5, seed=500 + t, with_grad=False)
    prev = B.set_gemv_max_ctas(ctas)
    try:
        _check_fwd(li)
    finally:
        B.set_gemv_max_ctas(prev)
