"""GPU parity of nf4_quantize / nf4_dequantize against the CPU oracle, bit for bit.

Inputs: the seeded workloads (single 1024 x 1024 linear; every linear of a LLaMA-7B-shaped
layer with 1% outliers at +-8 sigma; the decode-shape weights), ragged shapes (partial last
scale group, one block, odd row counts), and the degenerate cases (all-zero blocks and groups,
exactly representable blocks, non-finite weights -> status bit)."""

import numpy as np
import pytest
import torch

from bit_quantized_lora_03_b200 import binding as B
from bit_quantized_lora_03_b200 import inputs
from oracle import nf4_oracle as O

from gpu_util import oracle_packed_rows, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _check_full(Wt: torch.Tensor):
    p = B.nf4_quantize(Wt.cuda())
    deq = B.nf4_dequantize(p)
    assert B.last_status() == 0
    ref = O.nf4_quantize(Wt.numpy())
    assert np.array_equal(p.codes.cpu().numpy(), ref.codes), "packed codes differ"
    assert np.array_equal(p.absmax_q8.cpu().numpy(), ref.absmax_q8), "8-bit scales differ"
    assert np.array_equal(p.absmax_s2.cpu().numpy().view(np.uint32),
                          ref.absmax_s2.view(np.uint32)), "second-level scales differ"
    got = deq.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, O.nf4_dequantize_bits(ref)), "dequantized bf16 differs"


def test_single_linear_1024():
    _check_full(inputs.single_linear_1024().Wt)


@pytest.mark.parametrize("o,h", [(1, 64), (3, 128), (5, 64 * 300), (257, 192), (64, 4096 + 64)])
def test_ragged_shapes(o, h):
    g = torch.Generator().manual_seed(o * 1000 + h)
    _check_full(torch.randn(o, h, generator=g) * 0.02)


@pytest.mark.parametrize("i", range(7))
def test_llama7b_layer_with_outliers(i):
    name, h, o = inputs.LLAMA7B_LINEARS[i]
    _check_full(inputs.weight_f32(o, h, 200 + i, outliers=True))


def test_weights_next_to_thresholds():
    """Blocks whose weights sit within a few ulps of c1 x (each threshold), plus +-c1 itself,
    over block scales from subnormal to 1e3: the quantizer's reciprocal fast path must hand
    every such weight to the IEEE quotient and agree with the oracle bit for bit."""
    mids = O.nf4_midpoints().astype(np.float32)
    rng = np.random.default_rng(7)
    rows = []
    for c1 in np.concatenate([np.float32([1.0, 1e-39, 3e-41, 2.5e-38]),
                              np.exp(rng.uniform(-60, 7, 60)).astype(np.float32)]):
        c1 = np.float32(c1)
        vals = [c1, -c1]
        for m in mids:
            v = np.float32(m * c1)
            for k in range(-3, 4):
                u = v
                for _ in range(abs(k)):
                    u = np.nextafter(u, np.float32(np.inf) if k > 0 else np.float32(-np.inf))
                vals.append(np.clip(u, -c1, c1))
        vals = np.array(vals, np.float32)
        row = np.resize(vals, 64 * ((vals.size + 63) // 64)).astype(np.float32)
        row[::64] = c1   # every block's absmax is exactly c1
        rows.append(np.resize(row, 64 * 4))
    _check_full(torch.from_numpy(np.stack(rows).astype(np.float32)))


def test_decode_weight_4096x11008():
    _check_full(inputs.decode_gemv_weights()[0][1])


def test_degenerate_blocks():
    q = O.nf4_codebook()
    W = torch.zeros(4, 64 * 130)
    W[1, :64] = torch.from_numpy(q[np.arange(64) % 16] * np.float32(0.5))   # representable
    W[2, 64:128] = 1e-30                                                    # tiny block
    W[3, -64:] = -3.0                                                       # one-signed block
    _check_full(W)
    _check_full(torch.zeros(2, 64 * 300))


def test_nonfinite_sets_status_bit():
    W = torch.randn(8, 256) * 0.02
    W[3, 17] = float("nan")
    B.last_status()
    B.nf4_quantize(W.cuda())
    assert B.last_status() & B.QLORA_DEV_NONFINITE
    assert B.last_status() == 0          # reading clears it


def test_sampled_rows_of_the_largest_decode_weight():
    """8192 x 28672 packed on the GPU; 24 rows recomputed by the oracle one by one."""
    Wt = inputs.decode_gemv_weights()[1][1]
    p = B.nf4_quantize(Wt.cuda())
    deq = B.nf4_dequantize(p)
    rows = sorted(set(torch.randint(0, Wt.shape[0], (24,), generator=torch.Generator().manual_seed(5)).tolist()
                      + [0, Wt.shape[0] - 1]))
    ref = oracle_packed_rows(Wt.numpy(), rows)
    got = deq[rows].float().cpu().numpy()
    assert np.array_equal(got.view(np.uint32), ref.astype(np.float32).view(np.uint32))


def _check_codebook(Wt: torch.Tensor, cb: int):
    p = B.nf4_quantize(Wt.cuda(), codebook_id=cb)
    deq = B.nf4_dequantize(p, codebook_id=cb)
    assert B.last_status() == 0
    ref = O.quantize_with(Wt.numpy(), cb)
    assert np.array_equal(p.codes.cpu().numpy(), ref.codes), "packed codes differ"
    assert np.array_equal(p.absmax_q8.cpu().numpy(), ref.absmax_q8), "8-bit scales differ"
    assert np.array_equal(p.absmax_s2.cpu().numpy().view(np.uint32),
                          ref.absmax_s2.view(np.uint32)), "second-level scales differ"
    got = deq.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got.reshape(-1), O.dequantize_bits_with(ref, cb).reshape(-1)), \
        "dequantized bf16 differs"


@pytest.mark.parametrize("cb", [B.CODEBOOK_FP4, B.CODEBOOK_INT4])
def test_other_codebooks_bit_exact(cb):
    """FP4 and INT4 packing, bit for bit: a LLaMA-7B q_proj with 1% outliers, a ragged shape,
    and rows with all-zero blocks (the codebook's own zero code)."""
    _check_codebook(inputs.weight_f32(4096, 4096, 200, outliers=True), cb)
    g = torch.Generator().manual_seed(cb)
    W = torch.randn(257, 192, generator=g) * 0.02
    W[3] = 0.0
    W[10, :64] = 0.0
    _check_codebook(W, cb)


def _check_format(Wt: torch.Tensor, cb: int, fmt: int):
    p = B.nf4_quantize(Wt.cuda(), codebook_id=cb, scale_format=fmt)
    deq = B.nf4_dequantize(p, codebook_id=cb, scale_format=fmt)
    assert B.last_status() == 0
    ref = O.quantize_format(Wt.numpy(), cb, fmt)
    assert np.array_equal(p.codes.cpu().numpy(), ref.codes)
    assert np.array_equal(p.absmax_q8.cpu().numpy(), ref.absmax_q8)
    assert np.array_equal(p.absmax_s2.cpu().numpy().view(np.uint32), ref.absmax_s2.view(np.uint32))
    assert np.array_equal(deq.view(torch.int16).cpu().numpy().view(np.uint16),
                          O.dequantize_bits_format(ref, cb, fmt))


@pytest.mark.parametrize("fmt", [B.SCALES_S8, B.SCALES_E4M3])
@pytest.mark.parametrize("cb", [B.CODEBOOK_NF4, B.CODEBOOK_FP4])
def test_other_scale_formats_bit_exact(cb, fmt):
    """Signed int8 and FP8 E4M3 block scales, bit for bit: a LLaMA-7B q_proj with 1% outliers
    (scales spread over the whole code range, E4M3 subnormals among them), a ragged shape with
    all-zero blocks and a group whose scales are all zero, and blocks of tiny magnitude."""
    _check_format(inputs.weight_f32(4096, 4096, 200, outliers=True), cb, fmt)
    g = torch.Generator().manual_seed(10 + fmt)
    W = torch.randn(257, 192, generator=g) * 0.02
    W[3] = 0.0
    W[10, :64] = 0.0
    W[20:40] *= 1e-5          # block scales far below the group's largest: E4M3 subnormals
    W[160:] = 0.0             # blocks 480 .. 770 zero: second-level group 2 entirely zero
    _check_format(W, cb, fmt)


def test_second_level_ties_round_half_to_even():
    """Block scales with c1 / s2 exactly halfway between two integers (s2 = 2^-8 exactly, c1 =
    (k + 1/2) 2^-8): the 8-bit codes round half to even on the GPU as in the oracle."""
    c1 = [255.0 * 2.0 ** -8] + [(k + 0.5) * 2.0 ** -8 for k in range(255)]
    W = torch.zeros(256, 64)
    W[:, 0] = torch.tensor(c1, dtype=torch.float32)
    W[:, 1] = -0.5 * W[:, 0]
    _check_full(W.reshape(4, 4096))


def test_dequantize_where_the_multiply_order_matters():
    """Packed weights whose (level, q8, s2) make (level * q8) * s2 and level * (q8 * s2) round
    to different bf16 values: the GPU dequantizer gives the second, as the oracle does."""
    q = O.nf4_codebook()
    found = []
    for seed in range(40):
        r = np.random.default_rng(seed)
        s2 = r.uniform(1e-5, 1e-3, 64).astype(np.float32)
        q8 = r.integers(1, 256, (64, 256)).astype(np.float32)
        k = (q8 * s2[:, None]).astype(np.float32)
        exact = (q[None, None, :] * k[..., None]).astype(np.float32)
        other = ((q[None, None, :] * q8[..., None]).astype(np.float32) * s2[:, None, None])
        i, j, c = np.nonzero(O.bf16_bits_rne(exact) != O.bf16_bits_rne(other.astype(np.float32)))
        found += [(s2[a], int(q8[a, b]), int(cc)) for a, b, cc in zip(i, j, c)]
        if len(found) >= 8:
            break
    assert len(found) >= 8
    ng = len(found)
    rng = np.random.default_rng(3)
    codes = rng.integers(0, 16, (ng * 256, 64)).astype(np.uint8)
    q8 = rng.integers(1, 256, ng * 256).astype(np.uint8)
    s2 = np.array([f[0] for f in found], np.float32)
    for g, (_, qq, cc) in enumerate(found):
        q8[g * 256], codes[g * 256] = qq, cc
    ref = O.NF4Packed(O.pack_nibbles(codes.reshape(-1)), q8, s2, ng * 256, 64, None)
    p = B.PackedNF4(ng * 256, 64, "cuda")
    p.codes.copy_(torch.from_numpy(ref.codes))
    p.absmax_q8.copy_(torch.from_numpy(q8))
    p.absmax_s2.copy_(torch.from_numpy(s2))
    got = B.nf4_dequantize(p).view(torch.int16).cpu().numpy().view(np.uint16)
    assert B.last_status() == 0
    assert np.array_equal(got, O.nf4_dequantize_bits(ref))
