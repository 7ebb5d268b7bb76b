"""Plain CPU oracle for the QLoRA NF4 frozen-base linear layer.

TEST INFRASTRUCTURE ONLY. This module is the slow, obviously correct reference that
the CUDA library is checked against. Only the test suite, the smoke check in
``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` may import it. The product
path (the C-ABI library and its Python binding) never imports, calls or links it, and it
shares no code, table or constant generator with that path.

Precision: encodings (codebook, codes, 8-bit scales, dequantized bf16) are computed in the
fp32 arithmetic the method fixes, with every fp32 operation written out; products are
computed in fp64 from the exact inputs.

Sources (web pages on QLoRA, Dettmers et al., arXiv:2305.14314), cited by page title and
section:

* "QLoRA in LLMs" (tensortonic.com): §2 "How Quantization Works" (absmax scale, round,
  multiply back), §3 "How LoRA and Quantization Fit Together" (two codes per byte, a
  16-entry codebook, blocks with a scale each, dequantize to BF16 for compute, base +
  adapter), §4 "One QLoRA Training Step, End to End" (gradients reach the adapters, the
  base is never updated), §5 "NF4" (levels at quantiles of a standard normal), §6 "Double
  Quantization Compresses the Scales" (quantize the block scales; codes unchanged).
* "QLoRA: Efficient Finetuning of Quantized LLMs" (mchromiak.github.io): "The algebra"
  (X is t x h, W is h x o, L1 is h x r, L2 is r x o, scalar s), "1. NormalFloat" (blocks
  with their own scale, BF16 compute), "2. Double quantization" (8-bit first-level scales,
  higher-precision second-level scales; 0.5 -> ~0.127 bits per weight), "A worked memory
  budget for 65 billion weights" (64 weights per block, 256 scales per second-level block).
* "QLoRA: the paper that put large-model fine-tuning on a desk" (goodomens.studio):
  "Idea one: NF4" (each level used equally often), "Idea two: double quantization" (fp32
  scale per 64 weights, re-quantized to 8 bits with a second-level scale per chunk), "The
  core move" (a 4-bit block is dequantized on the fly, used for the matmul, discarded).
* "Chapter 1: What is QLoRA?" (docs.skillversehub.com): "Key Components" (equal number of
  values in each bin).

Readings where the pages are silent (each is also listed in the design notes):

* Codebook construction. The pages fix: quantiles of N(0,1), equal use of every level,
  an exact zero, ends normalised to -1 and +1. The plainest construction with all four:
  8 positive quantiles at probabilities evenly spaced from delta down to (not including)
  1/2, 7 negative ones likewise, the zero, all divided by the largest; delta is the mean of
  the two "centre of the outermost of 15 / of 16 equal-probability bins" probabilities,
  1 - 1/30 and 1 - 1/32. The exact delta is a reading, so the exact 16 values are parity
  unpinned beyond the properties above: no printed table pins them (the pages print none).
* Code choice: nearest level by comparison against fp32 midpoints of adjacent levels; a
  value exactly on a midpoint takes the lower code.
* Second level: unsigned 8-bit absmax codes with step c2/255 (the textbook scheme of
  "QLoRA in LLMs" §2 made unsigned because a block absmax is never negative, §1 on UINT8),
  one fp32 scale per 256 first-level scales; the last group may be partial.
* Layout: the stored matrix is Wt = W' transposed (o x h, row-major, "out x in"); blocks
  of 64 run along h inside one row; element 2j of the flat order sits in the high nibble
  of byte j.
* LoRA: Y = X.W + s.X.L1.L2 with s = alpha / r; backward by the chain rule.
"""

from __future__ import annotations

import math

import numpy as np

BLOCK = 64          # weights per first-level block
GROUP = 256         # first-level scales per second-level scale
ZERO_CODE = 7       # index of the exact-zero level
Q8_MAX = 255        # unsigned 8-bit code range for the first-level scales


# ----------------------------------------------------------------------------------------
# Standard normal quantile, by bisection on the CDF (double precision)
# ----------------------------------------------------------------------------------------

def normal_cdf(x: float) -> float:
    """Phi(x) of the standard normal, from the complementary error function."""
    return 0.5 * math.erfc(-x / math.sqrt(2.0))


def normal_quantile(p: float) -> float:
    """Phi^-1(p) by bisection: the x with Phi(x) = p, to the resolution of a double."""
    if not 0.0 < p < 1.0:
        raise ValueError("p must lie in (0, 1)")
    lo, hi = -40.0, 40.0
    for _ in range(2000):
        mid = 0.5 * (lo + hi)
        if mid == lo or mid == hi:
            break
        if normal_cdf(mid) < p:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


# ----------------------------------------------------------------------------------------
# NF4 codebook ("QLoRA in LLMs" §5; "Idea one: NF4"; "Key Components")
# ----------------------------------------------------------------------------------------

def nf4_tail_probability() -> float:
    """delta: mean of the centre probabilities of the outermost of 15 and of 16 equal bins."""
    return 0.5 * ((1.0 - 1.0 / 30.0) + (1.0 - 1.0 / 32.0))


def nf4_construction_probabilities() -> tuple[list[float], list[float]]:
    """Probabilities at which the positive (8) and negative (7) levels are placed.

    Positive side: delta + i*(1/2 - delta)/8 for i = 0..7 (the point 1/2 itself, i = 8, is
    dropped; the zero level takes its place). Negative side: the same with 7 steps, i = 0..6,
    mirrored (level = -Phi^-1(p)).
    """
    delta = nf4_tail_probability()
    pos = [delta + i * (0.5 - delta) / 8.0 for i in range(8)]
    neg = [delta + i * (0.5 - delta) / 7.0 for i in range(7)]
    return pos, neg


def nf4_codebook_f64() -> np.ndarray:
    """The 16 levels in double precision, ascending, ends exactly -1 and +1, q[7] == 0."""
    pos_p, neg_p = nf4_construction_probabilities()
    pos = [normal_quantile(p) for p in pos_p]
    neg = [-normal_quantile(p) for p in neg_p]
    top = normal_quantile(nf4_tail_probability())
    values = sorted(pos + neg + [0.0])
    return np.array([v / top for v in values], dtype=np.float64)


def nf4_codebook() -> np.ndarray:
    """The 16 NF4 levels rounded to fp32 (the table the method stores and uses)."""
    return nf4_codebook_f64().astype(np.float32)


def nf4_midpoints(levels: np.ndarray | None = None) -> np.ndarray:
    """15 fp32 decision thresholds m[i] = (q[i] + q[i+1]) / 2, summed in double."""
    q = nf4_codebook() if levels is None else np.asarray(levels, dtype=np.float32)
    q64 = q.astype(np.float64)
    return ((q64[:-1] + q64[1:]) / 2.0).astype(np.float32)


# ----------------------------------------------------------------------------------------
# bf16 round-to-nearest-even ("QLoRA in LLMs" §1: BF16 = 8 exponent, 7 fraction bits)
# ----------------------------------------------------------------------------------------

def bf16_bits_rne(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest, ties to even; NaN stays NaN."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    rounded = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        rounded = np.where(nan, ((u >> 16) | 0x40).astype(np.uint16), rounded)
    return rounded


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> the fp32 values they stand for (exact)."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """fp32 values rounded to the nearest bf16 value, returned as fp32."""
    return bf16_bits_to_f32(bf16_bits_rne(x))


# ----------------------------------------------------------------------------------------
# Textbook absmax integer quantization ("QLoRA in LLMs" §2 "Choose a scale, then round")
# ----------------------------------------------------------------------------------------

def absmax_int_quantize(x: np.ndarray, qmax: int, signed: bool):
    """Symmetric absmax quantization of one group to integers in [-qmax, qmax] (or [0, qmax]).

    scale = max|x| / qmax (fp32); code = round-half-even(x / scale), clamped. Returns
    (codes int64, scale fp32). An all-zero group has scale 0 and codes 0.
    """
    x = np.asarray(x, dtype=np.float32)
    absmax = np.float32(np.max(np.abs(x))) if x.size else np.float32(0.0)
    scale = np.float32(absmax / np.float32(qmax))
    if scale == 0.0:
        return np.zeros(x.shape, dtype=np.int64), scale
    codes = np.rint(x / scale).astype(np.int64)
    lo = -qmax if signed else 0
    return np.clip(codes, lo, qmax), scale


def absmax_int_dequantize(codes: np.ndarray, scale: np.float32) -> np.ndarray:
    """Multiply the stored integers back by the group scale (fp32)."""
    return np.asarray(codes, dtype=np.float32) * np.float32(scale)


# ----------------------------------------------------------------------------------------
# NF4 quantizer with double-quantized scales
# ----------------------------------------------------------------------------------------

class NF4Packed:
    """The packed weight: codes (uint8, n/2), absmax_q8 (uint8, n/64), absmax_s2 (fp32)."""

    def __init__(self, codes, absmax_q8, absmax_s2, out_features, in_features, absmax_f32):
        self.codes = codes
        self.absmax_q8 = absmax_q8
        self.absmax_s2 = absmax_s2
        self.out_features = out_features
        self.in_features = in_features
        self.absmax_f32 = absmax_f32       # first-level scales before double quantization


def block_absmax(Wt: np.ndarray) -> np.ndarray:
    """c1[b] = max |w| over block b (64 consecutive weights of the flat row-major order)."""
    w = np.asarray(Wt, dtype=np.float32).reshape(-1, BLOCK)
    return np.max(np.abs(w), axis=1)


def nf4_codes(Wt: np.ndarray, levels: np.ndarray | None = None,
              zero_code: int = ZERO_CODE) -> np.ndarray:
    """Unpacked 4-bit codes (uint8, one per weight) from the exact fp32 block absmax.

    x_hat = w / c1 in fp32 (IEEE, round to nearest); code = number of midpoints strictly
    below x_hat. A block whose absmax is 0 takes the zero level (code `zero_code`) everywhere.
    """
    mid = nf4_midpoints(levels)
    w = np.asarray(Wt, dtype=np.float32).reshape(-1, BLOCK)
    c1 = np.max(np.abs(w), axis=1)
    zero = c1 == 0
    safe = np.where(zero, np.float32(1.0), c1).astype(np.float32)
    xhat = (w / safe[:, None]).astype(np.float32)
    codes = np.zeros(w.shape, dtype=np.uint8)
    for i in range(mid.size):
        codes += (xhat > mid[i]).astype(np.uint8)
    codes[zero, :] = zero_code
    return codes.reshape(-1)


def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    """Two codes per byte: byte j = (code[2j] << 4) | code[2j+1]."""
    c = np.asarray(codes, dtype=np.uint8).reshape(-1, 2)
    return ((c[:, 0] << 4) | c[:, 1]).astype(np.uint8)


def unpack_nibbles(packed: np.ndarray) -> np.ndarray:
    """Inverse of pack_nibbles."""
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.size * 2, dtype=np.uint8)
    out[0::2] = p >> 4
    out[1::2] = p & 0xF
    return out


def double_quantize(c1: np.ndarray):
    """Second-level quantization of the first-level scales.

    Groups of 256 consecutive scales (the last one may be shorter): c2 = max c1,
    s2 = c2 / 255 (fp32), q8 = clamp(round-half-even(c1 / s2), 0, 255). A group whose
    maximum is 0 stores s2 = 0 and q8 = 0.
    """
    c1 = np.asarray(c1, dtype=np.float32)
    nb = c1.size
    ng = (nb + GROUP - 1) // GROUP
    q8 = np.zeros(nb, dtype=np.uint8)
    s2 = np.zeros(ng, dtype=np.float32)
    for g in range(ng):
        seg = c1[g * GROUP:(g + 1) * GROUP]
        c2 = np.float32(np.max(seg))
        scale = np.float32(c2 / np.float32(Q8_MAX))
        s2[g] = scale
        if scale == 0.0:
            continue
        ratio = (seg / scale).astype(np.float32)
        q8[g * GROUP:(g + 1) * GROUP] = np.clip(np.rint(ratio), 0, Q8_MAX).astype(np.uint8)
    return q8, s2


def nf4_quantize(Wt: np.ndarray) -> NF4Packed:
    """Quantize an fp32 weight stored as Wt (o x h, row-major, h % 64 == 0).

    Raises ValueError for non-finite input (the library reports a status instead).
    """
    Wt = np.asarray(Wt, dtype=np.float32)
    if Wt.ndim != 2 or Wt.shape[1] % BLOCK != 0:
        raise ValueError("Wt must be o x h with h a multiple of 64")
    if not np.all(np.isfinite(Wt)):
        raise ValueError("non-finite weight")
    c1 = block_absmax(Wt)
    codes = nf4_codes(Wt)
    q8, s2 = double_quantize(c1)
    return NF4Packed(pack_nibbles(codes), q8, s2, Wt.shape[0], Wt.shape[1], c1)


# ----------------------------------------------------------------------------------------
# Other 4-bit codebooks, for the format comparison the pages draw (NF4 against FP4 and INT4:
# "QLoRA in LLMs" §5 and "Idea one: NF4", goodomens.studio; the textbook absmax integer scheme
# of "QLoRA in LLMs" §2). Same blocks, packing and double-quantized scales; only the 16 levels
# (and the code of the zero level, used for all-zero blocks) differ.
# ----------------------------------------------------------------------------------------

def fp4_codebook() -> np.ndarray:
    """FP4 E2M1: magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6} with both signs, divided by the
    largest (6) so the ends are -1 and +1; -0 and +0 are both kept (16 codes), ascending."""
    mags = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    neg = [-m / 6.0 for m in reversed(mags)]      # -1 ... -0
    pos = [m / 6.0 for m in mags]                 # +0 ... +1
    return np.array(neg + pos, dtype=np.float64).astype(np.float32)


def int4_codebook() -> np.ndarray:
    """Symmetric absmax INT4: k / 7 for k = -8 .. 7 (the textbook absmax scheme with 4-bit
    integers; k = -8 lies below -1 and is never the nearest level of an |x| <= 1)."""
    return np.array([k / 7.0 for k in range(-8, 8)], dtype=np.float64).astype(np.float32)


# codebook id (the ids of the library's codebook calls) -> code of its zero level
CODEBOOK_ZERO_CODE = {0: ZERO_CODE, 1: 7, 2: 8}


def codebook_levels(cb: int) -> np.ndarray:
    return {0: nf4_codebook, 1: fp4_codebook, 2: int4_codebook}[cb]()


def quantize_with(Wt: np.ndarray, cb: int) -> NF4Packed:
    """nf4_quantize with codebook `cb` (0 NF4, 1 FP4, 2 INT4): same blocks, packing and
    double quantization; codes from that codebook's midpoints."""
    Wt = np.asarray(Wt, dtype=np.float32)
    if Wt.ndim != 2 or Wt.shape[1] % BLOCK != 0:
        raise ValueError("Wt must be o x h with h a multiple of 64")
    if not np.all(np.isfinite(Wt)):
        raise ValueError("non-finite weight")
    c1 = block_absmax(Wt)
    codes = nf4_codes(Wt, codebook_levels(cb), CODEBOOK_ZERO_CODE[cb])
    q8, s2 = double_quantize(c1)
    return NF4Packed(pack_nibbles(codes), q8, s2, Wt.shape[0], Wt.shape[1], c1)


def dequantize_bits_with(packed: NF4Packed, cb: int) -> np.ndarray:
    """bf16 bit patterns of bf16(level[code] * (q8 * s2)) with codebook `cb`."""
    return bf16_bits_rne(nf4_dequantize_f32(packed, codebook_levels(cb)))


# ----------------------------------------------------------------------------------------
# Other 8-bit formats for the first-level scales ("QLoRA in LLMs" §1 "FP32, FP16, BF16, and
# FP8": FP8 E4M3 has 4 exponent and 3 fraction bits, and FP8 and INT8 share one byte; §2 "Choose
# a scale, then round": symmetric absmax to the integers -127 .. 127). The second level stays
# one fp32 scale per 256 blocks; only the 8-bit code of each block scale changes:
#   SCALES_U8   (the default) s2 = c2 / 255, q8 = clamp(rint(c1 / s2), 0, 255);
#   SCALES_S8   the textbook signed scheme: s2 = c2 / 127, q8 = clamp(rint(c1 / s2), -127, 127)
#               stored as the two's-complement byte (absmax scales are >= 0, so half the codes
#               go unused: the point of the comparison);
#   SCALES_E4M3 s2 = c2 / 448 (448 = the largest finite E4M3 value), q8 = the E4M3 code of
#               c1 / s2 rounded to nearest even, saturating at 448.
# E4M3 here is the 8-bit float with exponent bias 7, no infinities, and code 0x7F (and 0xFF)
# as NaN, the variant tensor hardware converts to.
# ----------------------------------------------------------------------------------------

SCALES_U8, SCALES_S8, SCALES_E4M3 = 0, 1, 2
E4M3_MAX = 448.0


def e4m3_value(code) -> np.ndarray:
    """Value of E4M3 codes (fp32): sign bit 7, exponent bits 6..3 (bias 7), fraction bits 2..0;
    exponent 0 is subnormal (fraction x 2^-9); exponent 15 with fraction 7 is NaN."""
    c = np.asarray(code, dtype=np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    v = sign * mag
    v = np.where((e == 15) & (m == 7), np.nan, v)
    return v.astype(np.float32)


def e4m3_encode(x) -> np.ndarray:
    """E4M3 code (uint8) of non-negative finite fp32 values: the nearest finite E4M3 value, a tie
    going to the even code (even fraction), values above 448 saturating to 448 (code 0x7E)."""
    x = np.asarray(x, dtype=np.float64)
    if np.any(~np.isfinite(x)) or np.any(x < 0):
        raise ValueError("e4m3_encode takes non-negative finite values")
    vals = e4m3_value(np.arange(0x7F)).astype(np.float64)   # codes 0x00 .. 0x7E, ascending
    hi = np.clip(np.searchsorted(vals, x, side="left"), 0, 0x7E)
    lo = np.clip(hi - 1, 0, 0x7E)
    dlo, dhi = np.abs(x - vals[lo]), np.abs(vals[hi] - x)
    pick = np.where(dlo < dhi, lo, np.where(dhi < dlo, hi, np.where(lo % 2 == 0, lo, hi)))
    return pick.astype(np.uint8)


def double_quantize_with(c1: np.ndarray, fmt: int):
    """Second-level quantization of the block scales in scale format `fmt` (see above);
    groups of 256 blocks as in double_quantize."""
    if fmt == SCALES_U8:
        return double_quantize(c1)
    c1 = np.asarray(c1, dtype=np.float32)
    nb = c1.size
    ng = (nb + GROUP - 1) // GROUP
    q8 = np.zeros(nb, dtype=np.uint8)
    s2 = np.zeros(ng, dtype=np.float32)
    for g in range(ng):
        seg = c1[g * GROUP:(g + 1) * GROUP]
        if fmt == SCALES_S8:
            codes, scale = absmax_int_quantize(seg, 127, signed=True)
            q8[g * GROUP:(g + 1) * GROUP] = codes.astype(np.int8).view(np.uint8)
            s2[g] = scale
        elif fmt == SCALES_E4M3:
            c2 = np.float32(np.max(seg))
            scale = np.float32(c2 / np.float32(E4M3_MAX))
            s2[g] = scale
            if scale == 0.0:
                continue
            q8[g * GROUP:(g + 1) * GROUP] = e4m3_encode((seg / scale).astype(np.float32))
        else:
            raise ValueError("unknown scale format")
    return q8, s2


def scale_code_values(q8: np.ndarray, fmt: int) -> np.ndarray:
    """The number each 8-bit scale code stands for (fp32, exact)."""
    q8 = np.asarray(q8, dtype=np.uint8)
    if fmt == SCALES_U8:
        return q8.astype(np.float32)
    if fmt == SCALES_S8:
        return q8.view(np.int8).astype(np.float32)
    if fmt == SCALES_E4M3:
        return e4m3_value(q8)
    raise ValueError("unknown scale format")


def quantize_format(Wt: np.ndarray, cb: int, fmt: int) -> NF4Packed:
    """quantize_with(Wt, cb) with the block scales in scale format `fmt`; the 4-bit codes do
    not depend on the scale format (they use the exact c1)."""
    p = quantize_with(Wt, cb)
    p.absmax_q8, p.absmax_s2 = double_quantize_with(p.absmax_f32, fmt)
    return p


def dequantize_bits_format(packed: NF4Packed, cb: int, fmt: int) -> np.ndarray:
    """bf16 bit patterns of bf16(level[code] * (value(q8) * s2)), two fp32 multiplies."""
    q = codebook_levels(cb)
    codes = unpack_nibbles(packed.codes).reshape(-1, BLOCK)
    g = np.arange(packed.absmax_q8.size) // GROUP
    k = (scale_code_values(packed.absmax_q8, fmt) *
         np.asarray(packed.absmax_s2, dtype=np.float32)[g]).astype(np.float32)
    w = (q[codes] * k[:, None]).astype(np.float32)
    return bf16_bits_rne(w.reshape(packed.out_features, packed.in_features))


def block_scales(q8: np.ndarray, s2: np.ndarray) -> np.ndarray:
    """Reconstructed first-level scale per block: float(q8[b]) * s2[b // 256] (fp32)."""
    q8 = np.asarray(q8, dtype=np.uint8)
    g = np.arange(q8.size) // GROUP
    return (q8.astype(np.float32) * np.asarray(s2, dtype=np.float32)[g]).astype(np.float32)


def nf4_dequantize_f32(packed: NF4Packed, levels: np.ndarray | None = None) -> np.ndarray:
    """w' before the bf16 rounding: q[code] * (float(q8) * s2), two fp32 multiplies."""
    q = nf4_codebook() if levels is None else np.asarray(levels, dtype=np.float32)
    codes = unpack_nibbles(packed.codes).reshape(-1, BLOCK)
    k = block_scales(packed.absmax_q8, packed.absmax_s2)
    w = (q[codes] * k[:, None]).astype(np.float32)
    return w.reshape(packed.out_features, packed.in_features)


def nf4_dequantize_bits(packed: NF4Packed) -> np.ndarray:
    """The dequantized weight as bf16 bit patterns (uint16, o x h)."""
    return bf16_bits_rne(nf4_dequantize_f32(packed))


def nf4_dequantize(packed: NF4Packed) -> np.ndarray:
    """The dequantized weight W' (stored orientation o x h) as fp32 values of bf16 numbers."""
    return bf16_bits_to_f32(nf4_dequantize_bits(packed))


def dequantize_without_double_quant(codes: np.ndarray, c1: np.ndarray, o: int, h: int):
    """w' with the exact fp32 block absmax (double quantization off), rounded to bf16."""
    q = nf4_codebook()
    c = np.asarray(codes, dtype=np.uint8).reshape(-1, BLOCK)
    w = (q[c] * np.asarray(c1, dtype=np.float32)[:, None]).astype(np.float32)
    return bf16_round(w.reshape(o, h))


# ----------------------------------------------------------------------------------------
# Storage ledger ("A worked memory budget for 65 billion weights"; "2. Double quantization")
# ----------------------------------------------------------------------------------------

def scale_bits_per_weight(double_quant: bool) -> float:
    """Bits of scale metadata per weight: 32/64 without, 8/64 + 32/(64*256) with DQ."""
    if not double_quant:
        return 32.0 / BLOCK
    return 8.0 / BLOCK + 32.0 / (BLOCK * GROUP)


def packed_bytes(n: int) -> int:
    """Bytes of the real packed format for n weights (n % 64 == 0)."""
    nb = n // BLOCK
    return n // 2 + nb + 4 * ((nb + GROUP - 1) // GROUP)


def weight_storage_bytes(n_params: float, bits: float) -> float:
    """Raw storage of n_params values at `bits` bits each (N * b / 8)."""
    return n_params * bits / 8.0


# ----------------------------------------------------------------------------------------
# The adapted linear layer ("The algebra"; "QLoRA in LLMs" §3-§4)
# ----------------------------------------------------------------------------------------

def _f64(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


def qlora_linear_fwd(X, Wdq, L1, L2, s):
    """Y = X.W' + s.(X.L1).L2 in fp64.

    X: t x h; Wdq: the dequantized weight in its stored orientation o x h (so W' = Wdq^T,
    h x o); L1: h x r; L2: r x o. Returns (Y t x o, sT = s.X.L1 t x r), both fp64.
    """
    X, Wt, L1, L2 = _f64(X), _f64(Wdq), _f64(L1), _f64(L2)
    T = X @ L1
    Y = X @ Wt.T + s * (T @ L2)
    return Y, s * T


def qlora_linear_bwd(dY, X, Wdq, L1, L2, s):
    """Gradients of <dY, Y> for Y = X.W' + s.X.L1.L2, in fp64. W' gets none.

    dX = dY.W'^T + s.(dY.L2^T).L1^T; dL1 = s.X^T.(dY.L2^T); dL2 = s.(X.L1)^T.dY.
    Returns (dX t x h, dL1 h x r, dL2 r x o, sU = s.dY.L2^T t x r).
    """
    dY, X, Wt, L1, L2 = _f64(dY), _f64(X), _f64(Wdq), _f64(L1), _f64(L2)
    U = dY @ L2.T
    dX = dY @ Wt + s * (U @ L1.T)
    dL1 = s * (X.T @ U)
    dL2 = s * ((X @ L1).T @ dY)
    return dX, dL1, dL2, s * U


def qlora_linear_fwd_rows(rows, X, Wdq, L1, L2, s):
    """Rows `rows` of Y only (each row of Y depends on the same row of X alone)."""
    rows = np.asarray(rows)
    Y, _ = qlora_linear_fwd(_f64(X)[rows], Wdq, L1, L2, s)
    return Y


def qlora_linear_bwd_dx_rows(rows, dY, Wdq, L1, L2, s):
    """Rows `rows` of dX only (each row of dX depends on the same row of dY alone)."""
    dY, Wt, L1, L2 = _f64(dY)[np.asarray(rows)], _f64(Wdq), _f64(L1), _f64(L2)
    return dY @ Wt + s * ((dY @ L2.T) @ L1.T)


# ----------------------------------------------------------------------------------------
# Adapter merge ("QLoRA in LLMs" §11 "Saving, Loading, and Merging QLoRA Adapters": dequantize
# the base into a wider precision, add the LoRA update, optionally quantize the result again,
# and compare merged with unmerged outputs; "What it added up to", goodomens.studio: merging
# into a 16-bit copy of the base changes the model the adapters compensated for)
# ----------------------------------------------------------------------------------------

def merge_adapters(Wdq, L1, L2, s):
    """The merged weight in the stored orientation (o x h), fp64:
    Wt_m[j][k] = Wdq[j][k] + s * sum_c L2[c][j] * L1[k][c], i.e. W_m = W' + s.L1.L2."""
    Wt, L1, L2 = _f64(Wdq), _f64(L1), _f64(L2)
    return Wt + s * (L2.T @ L1.T)


def merge_error_bound(Wdq, L1, L2, s):
    """Elementwise bound on |fp32 merge - merge_adapters| for an fp32 evaluation that sums the
    r exact bf16 x bf16 products in any order (each partial sum rounded once), scales by s and
    adds W' (two more roundings): (r + 2) * 2^-24 * (|W'| + |s| * sum_c |L2[c][j] L1[k][c]|),
    doubled for margin."""
    Wt, L1, L2 = _f64(Wdq), _f64(L1), _f64(L2)
    r = L1.shape[1]
    mag = np.abs(Wt) + abs(s) * (np.abs(L2).T @ np.abs(L1).T)
    return 2.0 * (r + 2) * 2.0 ** -24 * mag


# ----------------------------------------------------------------------------------------
# Adapter update with a paged optimizer ("QLoRA in LLMs" §4 "Update the adapters" and §7 "Paged
# Optimizers Manage Temporary Memory Spikes"; "Idea three: paged optimizers", goodomens.studio).
# The pages name the optimizer state ("running statistics") but not the rule; the reading is
# AdamW (decoupled weight decay, bias-corrected moments), the optimizer QLoRA pages.
# ----------------------------------------------------------------------------------------

def adamw_step(p, g, m, v, step, lr, beta1, beta2, eps, weight_decay):
    """One AdamW update in fp64; returns (p, m, v) after step `step` (1-based):
    p <- p (1 - lr wd);  m <- b1 m + (1 - b1) g;  v <- b2 v + (1 - b2) g^2;
    p <- p - lr * (m / (1 - b1^t)) / (sqrt(v / (1 - b2^t)) + eps)."""
    p, g, m, v = _f64(p), _f64(g), _f64(m), _f64(v)
    p = p * (1.0 - lr * weight_decay)
    m = beta1 * m + (1.0 - beta1) * g
    v = beta2 * v + (1.0 - beta2) * g * g
    mhat = m / (1.0 - beta1 ** step)
    vhat = v / (1.0 - beta2 ** step)
    return p - lr * mhat / (np.sqrt(vhat) + eps), m, v


# ----------------------------------------------------------------------------------------
# LoRA dropout on the adapter input ("QLoRA in LLMs" §12 "Minimal QLoRA Setup with Hugging
# Face": the example configuration sets a LoRA dropout of 0.05; "What it added up to",
# goodomens.studio, lists dropout among the adapter knobs). The pages do not say where the
# dropout acts; the reading is the adapter branch's input, inverted scaling:
#   Y = X.W' + s.(D(X).L1).L2,   D(X) = X (.) M / (1 - p),
# M a keep mask with P(keep) = 1 - p, drawn by a counter-based generator so that the forward
# and backward passes (and the oracle) draw the same mask without storing it.
# ----------------------------------------------------------------------------------------

# Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3",
# SC'11): a 4 x 32-bit counter is mixed under a 2 x 32-bit key by ten rounds; each round
# multiplies two counter words by fixed odd constants, keeps both halves of the 64-bit
# products and XORs the high halves into the other two words together with the key; the key
# is advanced by two Weyl constants between rounds.
PHILOX_M0, PHILOX_M1 = 0xD2511F53, 0xCD9E8D57
PHILOX_W0, PHILOX_W1 = 0x9E3779B9, 0xBB67AE85
_MASK32 = np.uint64(0xFFFFFFFF)


def philox4x32_10(ctr, key):
    """Philox4x32 with 10 rounds. ctr: (n, 4) uint32 counters; key: (2,) or (n, 2) uint32.
    Returns (n, 4) uint32."""
    c = [np.asarray(ctr, dtype=np.uint64)[:, i].copy() for i in range(4)]
    k = np.broadcast_to(np.asarray(key, dtype=np.uint64), (c[0].shape[0], 2))
    k0, k1 = k[:, 0].copy(), k[:, 1].copy()
    for rnd in range(10):
        if rnd > 0:
            k0 = (k0 + np.uint64(PHILOX_W0)) & _MASK32
            k1 = (k1 + np.uint64(PHILOX_W1)) & _MASK32
        p0 = np.uint64(PHILOX_M0) * c[0]          # exact: both factors < 2^32
        p1 = np.uint64(PHILOX_M1) * c[2]
        hi0, lo0 = p0 >> np.uint64(32), p0 & _MASK32
        hi1, lo1 = p1 >> np.uint64(32), p1 & _MASK32
        c = [hi1 ^ c[1] ^ k0, lo1, hi0 ^ c[3] ^ k1, lo0]
    return np.stack(c, axis=1).astype(np.uint32)


def dropout_threshold(p) -> int:
    """Drop an element when its 32-bit draw is below floor(p * 2^32) (p as fp32, 0 <= p < 1),
    so that P(drop) = threshold / 2^32, within 2^-32 of p."""
    p = float(np.float32(p))
    if not (0.0 <= p < 1.0):
        raise ValueError("dropout probability must lie in [0, 1)")
    return int(np.floor(p * 4294967296.0))


def dropout_keep_mask(t: int, h: int, p, seed: int) -> np.ndarray:
    """Keep mask M (t x h bool) of the adapter input. Element e = i*h + j (row-major) takes
    word e mod 4 of Philox4x32-10 at counter (lo32(e div 4), hi32(e div 4), 0, 0) under key
    (lo32(seed), hi32(seed)); it is kept when that word is >= dropout_threshold(p)."""
    n = t * h
    thr = dropout_threshold(p)
    e = np.arange(n, dtype=np.uint64)
    groups = np.arange((n + 3) // 4, dtype=np.uint64)
    ctr = np.zeros((groups.size, 4), dtype=np.uint64)
    ctr[:, 0] = groups & _MASK32
    ctr[:, 1] = groups >> np.uint64(32)
    seed = int(seed) & 0xFFFFFFFFFFFFFFFF
    words = philox4x32_10(ctr, (seed & 0xFFFFFFFF, seed >> 32))
    draw = words[(e >> np.uint64(2)).astype(np.int64), (e & np.uint64(3)).astype(np.int64)]
    return (draw.astype(np.int64) >= thr).reshape(t, h)


def dropout_scale(p) -> float:
    """1 / (1 - p) in fp64 for the fp32 value of p."""
    return 1.0 / (1.0 - float(np.float32(p)))


def qlora_linear_fwd_dropout(X, Wdq, L1, L2, s, keep, p):
    """Y = X.W' + s.((X (.) M / (1 - p)).L1).L2 in fp64, M = keep.
    Returns (Y t x o, sT = s.(X (.) M / (1 - p)).L1 t x r)."""
    X, Wt, L1, L2 = _f64(X), _f64(Wdq), _f64(L1), _f64(L2)
    Xd = X * np.asarray(keep, dtype=np.float64) * dropout_scale(p)
    T = Xd @ L1
    return X @ Wt.T + s * (T @ L2), s * T


def qlora_linear_bwd_dropout(dY, X, Wdq, L1, L2, s, keep, p):
    """Gradients of <dY, Y> for the dropout forward above, in fp64:
    dX = dY.W'^T + M (.) (s / (1 - p)).(dY.L2^T).L1^T;  dL1 = s.D(X)^T.(dY.L2^T);
    dL2 = s.(D(X).L1)^T.dY. Returns (dX, dL1, dL2)."""
    dY, X, Wt, L1, L2 = _f64(dY), _f64(X), _f64(Wdq), _f64(L1), _f64(L2)
    M = np.asarray(keep, dtype=np.float64) * dropout_scale(p)
    Xd = X * M
    U = dY @ L2.T
    dX = dY @ Wt + M * (s * (U @ L1.T))
    dL1 = s * (Xd.T @ U)
    dL2 = s * ((Xd @ L1).T @ dY)
    return dX, dL1, dL2


def max_err_vs_rms(got, ref) -> tuple[float, float]:
    """(max |got - ref|, RMS(ref)) in fp64: the tolerance test is max <= 2e-2 * RMS."""
    got, ref = _f64(got), _f64(ref)
    return float(np.max(np.abs(got - ref))) if ref.size else 0.0, \
        float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
