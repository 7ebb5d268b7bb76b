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

from gpu_util import assert_close_rms, f32, oracle_packed_rows, require_gpu

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


@pytest.mark.parametrize("t", [1, 4, 16])
def test_decode_shape_gemv_8192x28672(t):
    """The largest decode weight (o x h = 28672 x 8192, 896 row tiles x 128 blocks) through the
    GEMV at the token counts the bench times: Y on 64 seeded output columns (the oracle
    quantizes only the scale groups that cover those rows of Wt) and all of sT."""
    name, Wt = inputs.decode_gemv_weights()[1]
    o, h = Wt.shape
    L1, L2 = inputs.decode_gemv_adapters(h, o, 16)
    X = inputs.decode_gemv_activations(h, t)
    p = B.nf4_quantize(Wt.cuda())
    Y, sT = B.qlora_linear_fwd(X.cuda(), p, L1.cuda(), L2.cuda(), 2.0)
    assert B.last_status() == 0
    rng = np.random.default_rng(28672 + t)
    cols = np.unique(np.concatenate([[0, 1, o - 1], rng.choice(o, 61, replace=False)]))
    Wdq_J = oracle_packed_rows(Wt.numpy(), cols).astype(np.float64)
    X64, L1_64, L2_64 = f32(X).astype(np.float64), f32(L1).astype(np.float64), f32(L2).astype(np.float64)
    T = X64 @ L1_64
    assert_close_rms(f32(sT), 2.0 * T, "sT")
    Y_ref = X64 @ Wdq_J.T + 2.0 * (T @ L2_64[:, cols])
    assert_close_rms(f32(Y)[:, cols], Y_ref, "Y columns")


@pytest.mark.parametrize("i", [0, 5, 6])
def test_training_shape_linear_sampled(i):
    """A training-shape linear of the LLaMA-7B layer (r = 64, t = 4096): q_proj (4096 x 4096:
    128 CTA-pair tiles, 1.73 waves), up_proj (h = 4096, o = 11008) and down_proj (h = 11008,
    o = 4096). Full dL1 and dL2, and 256 seeded rows of Y and dX (each row depends on one row
    of X or dY only). down_proj's dL1 is 11008 x 64: 86 row tiles of 128, between half and all
    of the 148 SMs, the case the rank-r GEMM plan splits K in two for with two CTAs per SM."""
    li = inputs.training_linear(i)
    if i == 6:
        mtiles = -(-li.h // 128)
        assert 148 // 2 < mtiles < 148
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


@pytest.mark.parametrize("t,ctas,nblk", [(1, 1, 67), (5, 3, 67), (12, 1, 67), (16, 2, 67),
                                         (1, 1, 68), (3, 2, 68), (16, 3, 68)])
def test_decode_gemv_long_warp_runs(t, ctas, nblk):
    """Few CTAs give every warp a long run of units (32 rows x 128 inputs): it crosses row
    tiles and 16-unit scale segments. nblk = 67 blocks per row ends every row with a one-block
    unit and starts rows of 8-bit scales at every byte offset of a 4-byte word; nblk = 68 ends
    on whole units. Second-level groups of 256 blocks begin in the middle of rows."""
    li = inputs.random_linear(t, 64 * nblk, 576, 16, 1.5, seed=500 + t + nblk, with_grad=False)
    prev = B.set_gemv_max_ctas(ctas)
    try:
        _check_fwd(li)
    finally:
        B.set_gemv_max_ctas(prev)


def test_many_tiles_ragged_edges():
    """More 512 x 256 tiles than CTA pairs fit on the GPU at once (81 in the forward and in the
    dX kernel), with a ragged last row block (t = 4396 = 8 x 512 + 300) and ragged last column
    tiles (o = 2176 = 8 x 256 + 128, h = 2112 = 8 x 256 + 64), r = 80 (two LoRA K-steps, the
    second ragged): Y, sT, dX, dL1 and dL2 in full against the oracle, and the same bits when
    the call is repeated on a workspace holding other bytes."""
    t, h, o, r, s = 4396, 2112, 2176, 80, 0.5
    li = inputs.random_linear(t, h, o, r, s, seed=4396)
    dev = torch.device("cuda")
    p = B.nf4_quantize(li.Wt.to(dev))
    X, dY, L1, L2 = (a.to(dev) for a in (li.X, li.dY, li.L1, li.L2))
    Wdq = _oracle_weight(li.Wt)
    Y_ref, sT_ref = O.qlora_linear_fwd(f32(li.X), Wdq, f32(li.L1), f32(li.L2), s)
    dX_ref, dL1_ref, dL2_ref, _ = O.qlora_linear_bwd(f32(li.dY), f32(li.X), Wdq, f32(li.L1),
                                                    f32(li.L2), s)
    outs = []
    for fill in (0xA5, 0x5A):
        wsf = torch.full((B.fwd_workspace_bytes(t, h, o, r),), fill, dtype=torch.uint8, device=dev)
        wsb = torch.full((B.bwd_workspace_bytes(t, h, o, r),), fill, dtype=torch.uint8, device=dev)
        Y, sT = B.qlora_linear_fwd(X, p, L1, L2, s, ws=wsf)
        dX, dL1, dL2 = B.qlora_linear_bwd(dY, X, p, L1, L2, s, sT=sT, ws=wsb)
        torch.cuda.synchronize()
        assert B.last_status() == 0
        assert_close_rms(f32(Y), Y_ref, "Y")
        assert_close_rms(f32(sT), sT_ref, "sT")
        assert_close_rms(f32(dX), dX_ref, "dX")
        assert_close_rms(f32(dL1), dL1_ref, "dL1")
        assert_close_rms(f32(dL2), dL2_ref, "dL2")
        outs.append((Y.clone(), dX.clone(), dL1.clone(), dL2.clone()))
    for a_, b_ in zip(*outs):
        assert torch.equal(a_, b_)
