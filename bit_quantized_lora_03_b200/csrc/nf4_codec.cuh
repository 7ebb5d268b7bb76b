// NF4 quantizer (with double-quantized block scales) and dequantizer for sm_100a.
//
// Method ("QLoRA in LLMs", tensortonic.com, sections 2, 3, 5, 6; "QLoRA: Efficient Finetuning
// of Quantized LLMs", mchromiak.github.io, "1. NormalFloat" and "2. Double quantization"):
//   block of 64 consecutive weights -> absmax c1 -> x = w / c1 -> nearest of 16 NF4 levels,
//   two 4-bit codes per byte; the c1 of 256 consecutive blocks -> c2 = max c1, s2 = c2 / 255,
//   q8 = round(c1 / s2) (8 bits); dequantized weight w' = bf16(level[code] * (q8 * s2)).
// Both kernels are HBM-bound streams; all fp32 operations that decide an encoding are the
// IEEE round-to-nearest ones the method's definition fixes (__fdiv_rn, __fmul_rn, rint).
#pragma once

#include <cuda_fp8.h>

#include "qlora_common.cuh"

namespace qlora {

// NF4 levels and decision thresholds, passed by value as a kernel parameter.
struct Nf4Table {
  float level[16];
  float mid[16];  // 15 thresholds, mid[15] unused
  int zero_code;  // code of the zero level (all-zero blocks): 7 for NF4
};

constexpr int kBlock = 64;
constexpr int kGroup = 256;

// Nearest-level code of x = w / c1 as the number of thresholds strictly below x, found by a
// four-step binary search over the sorted thresholds in shared memory.
__device__ __forceinline__ uint32_t nf4_code_of(float w, float c1, const float* mids,
                                                uint32_t zero_code = 7u) {
  if (c1 == 0.0f) return zero_code;
  const float x = __fdiv_rn(w, c1);
  uint32_t c = (x > mids[7]) ? 8u : 0u;
  c += (x > mids[c + 3]) ? 4u : 0u;
  c += (x > mids[c + 1]) ? 2u : 0u;
  c += (x > mids[c]) ? 1u : 0u;
  return c;
}

// The same decision without a division in the common case. x' = w * RN(1/c1) is within 2^-22
// of the IEEE quotient x = RN(w / c1) for |w| <= c1 (two roundings of relative size 2^-24
// each, |x| <= 1), so x' and x fall on the same side of every threshold farther than 2^-20
// from x'. The thresholds are found through 128 equal buckets over [-1, 1): bucket b =
// floor((x' + 1) * 64), read from the mantissa of x' + 3 (which lies in [2, 4)); each bucket
// holds the count of thresholds below it and the one threshold inside it (or 4 if none).
// When x' is within 2^-20 of that threshold, the code is decided on the IEEE quotient. The
// host builds the buckets only if every bucket holds at most one threshold and no threshold
// lies within 2^-18 of a bucket edge (so a bucket misread by rounding near an edge still
// gives the same count); otherwise `exact_only` sends every weight to nf4_code_of.
struct Nf4Buckets {
  float thr[128];
  float lo[128];  // counts, as floats
  int exact_only;
};

__device__ __noinline__ uint32_t nf4_code_exact(float w, float c1, const float* mids,
                                               uint32_t zero_code) {
  return nf4_code_of(w, c1, mids, zero_code);
}

// Fast decision; sets `near` when x' is within 2^-20 of the bucket's threshold (the caller
// then decides on the IEEE quotient). The bucket table holds one copy per lane (entry b of
// lane l at 256 b + 8 l: {threshold, count as integer bits}), so lookups never collide on a bank.
__device__ __forceinline__ uint32_t nf4_code_fast(float w, float r, uint32_t lane_tab, bool& near) {
  const float x = __fmul_rn(w, r);
  const float xc = fminf(fmaxf(x, -1.0f), 1.0f - 0x1p-22f);  // then xc + 3 <= 4 - 2^-22 exactly
  const uint32_t b = (__float_as_uint(__fadd_rn(xc, 3.0f)) >> 16) & 127u;
  float thr;
  uint32_t lo;
  asm("ld.shared.v2.b32 {%0, %1}, [%2];" : "=f"(thr), "=r"(lo) : "r"(lane_tab + b * 256u));
  near |= fabsf(__fsub_rn(x, thr)) < 0x1p-20f;
  return lo + (x > thr ? 1u : 0u);
}

// max that propagates NaN (so a block's absmax is NaN or inf exactly when it holds one)
__device__ __forceinline__ float fmax_nan(float a, float b) {
  float d;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
  return d;
}

// Per-block product table: the 16 exact weights bf16(level[c] * k) of one 64-weight block, held
// in registers as byte planes so that byte permutes can select them: lo[q] holds the low
// bytes of entries 4q .. 4q+3, hi[q] their high bytes. Built once per block and stage from the
// fp32 levels (as eight fp32 pairs) with one packed fp32x2 multiply per pair, so each entry is
// the value nf4_dequantize produces; no per-weight shared-memory lookup remains. Used by the
// fused GEMM's producers and by the decode GEMV.
struct ProdTab {
  uint32_t lo[4], hi[4];
};

__device__ __forceinline__ ProdTab build_prod_tab(const uint64_t (&lv2)[8], float k) {
  uint64_t kk;
  asm("mov.b64 %0, {%1, %1};" : "=l"(kk) : "f"(k));
  uint32_t P[8];   // P[i]: entry 2i in the low half, entry 2i+1 in the high half
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(lv2[i]), "l"(kk));
    float ra, rb;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(ra), "=f"(rb) : "l"(r));
    P[i] = pack_bf16x2(ra, rb);
  }
  ProdTab t;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    t.lo[q] = __byte_perm(P[2 * q], P[2 * q + 1], 0x6420);
    t.hi[q] = __byte_perm(P[2 * q], P[2 * q + 1], 0x7531);
  }
  return t;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// Four weights (codes c_n, n = 0..3; sel: nibble n = c_n & 7; m: byte n = 0xFF if c_n & 8) ->
// two bf16x2 words (c_0, c_1) and (c_2, c_3), the first of each pair in the low half.
__device__ __forceinline__ uint2 select4(const ProdTab& t, uint32_t sel, uint32_t m) {
  const uint32_t L = (prmt(t.lo[0], t.lo[1], sel) & ~m) | (prmt(t.lo[2], t.lo[3], sel) & m);
  const uint32_t H = (prmt(t.hi[0], t.hi[1], sel) & ~m) | (prmt(t.hi[2], t.hi[3], sel) & m);
  return make_uint2(prmt(L, H, 0x5140), prmt(L, H, 0x7362));
}

// Eight packed codes (one 32-bit word, element 2j in the high nibble of byte j) -> eight bf16
// weights from the block's product table.
__device__ __forceinline__ uint4 dequant8_tab(uint32_t x, const ProdTab& t) {
  const uint32_t x4 = x << 4;   // byte j: the low nibble (element 2j+1) moved up
  // nibble n = code of element n
  const uint32_t xs = ((x >> 4) & 0x0F0F0F0Fu) | (x4 & 0xF0F0F0F0u);
  const uint32_t s = xs & 0x77777777u;
  // byte n = 0xFF where element n's code has bit 3 set: the sign bit of byte j of x is bit 3 of
  // element 2j, that of byte j of x4 bit 3 of element 2j+1 (prmt's sign-replicating selectors)
  const uint32_t m0 = prmt(x, x4, 0xD9C8u);
  const uint32_t m1 = prmt(x, x4, 0xFBEAu);
  const uint2 a = select4(t, s, m0);
  const uint2 b = select4(t, s >> 16, m1);
  return make_uint4(a.x, a.y, b.x, b.y);
}

// Persistent: CTAs of 512 threads (qz::kCtasPerSm per SM) walk the groups of 256 blocks (16384
// weights, 64 KB of fp32) g = blockIdx.x, blockIdx.x + gridDim.x, ...; thread 0 streams each
// group into a 64 KB shared-memory buffer with bulk copies, kBufs groups ahead, so HBM reads
// overlap arithmetic (the other CTA's, with one buffer). Half-warp h of pass p (0..7) owns
// block 32p + h; each of its lanes reads one float4 of the block from shared memory.
// 8-bit formats of the block scales ("QLoRA in LLMs" section 1: FP8 E4M3 has 4 exponent and 3
// fraction bits; section 2 "Choose a scale, then round": symmetric absmax to -127 .. 127). The
// second level is one fp32 scale s2 per 256 blocks in every format:
//   kScalesU8   s2 = c2 / 255, q8 = clamp(rint(c1 / s2), 0, 255)             (the default)
//   kScalesS8   s2 = c2 / 127, q8 = clamp(rint(c1 / s2), -127, 127) as a two's-complement byte
//   kScalesE4M3 s2 = c2 / 448, q8 = E4M3 code of c1 / s2 (round to nearest even, saturating)
enum ScaleFormat : int { kScalesU8 = 0, kScalesS8 = 1, kScalesE4M3 = 2 };

__host__ __device__ constexpr float scale_format_top(int sfmt) {
  return sfmt == kScalesU8 ? 255.0f : (sfmt == kScalesS8 ? 127.0f : 448.0f);
}

__device__ __forceinline__ uint8_t scale_code(float c1, float s2, int sfmt) {
  if (s2 == 0.0f) return 0;
  const float x = __fdiv_rn(c1, s2);
  if (sfmt == kScalesE4M3)
    return static_cast<uint8_t>(__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3));
  const int lo = sfmt == kScalesS8 ? -127 : 0, hi = sfmt == kScalesS8 ? 127 : 255;
  return static_cast<uint8_t>(min(hi, max(lo, __float2int_rn(x))));
}

// The number an 8-bit scale code stands for (exact in fp32).
__device__ __forceinline__ float scale_code_value(uint8_t q, int sfmt) {
  if (sfmt == kScalesS8) return static_cast<float>(static_cast<int8_t>(q));
  if (sfmt == kScalesE4M3) {
    const __half_raw hr = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(q), __NV_E4M3);
    return __half2float(__half(hr));
  }
  return static_cast<float>(q);
}

namespace qz {
constexpr int kThreads = 512;
constexpr int kGroupBytes = kGroup * kBlock * 4;  // 64 KB
constexpr int kChunk = 16384;                       // bytes per bulk copy
#ifndef QLORA_QZ_BUFS
#define QLORA_QZ_BUFS 1
#endif
// Group buffers per CTA. With one, two CTAs share an SM (98 KB of shared memory each): one
// encodes a group while the other's next group streams in, and 32 warps per SM (not 16)
// hide the latency of the per-weight shuffles and table lookups.
constexpr int kBufs = QLORA_QZ_BUFS;
constexpr int kCtasPerSm = kBufs == 1 ? 2 : 1;
constexpr size_t smem_bytes() { return kBufs * static_cast<size_t>(kGroupBytes) + 64; }
}  // namespace qz

__global__ void __launch_bounds__(qz::kThreads, qz::kCtasPerSm) nf4_quantize_kernel(
    const float* __restrict__ W, uint8_t* __restrict__ codes, uint8_t* __restrict__ q8,
    float* __restrict__ s2, int64_t nblocks, Nf4Table tab, Nf4Buckets bkt, int sfmt) {
  extern __shared__ __align__(128) uint8_t qsm[];
  __shared__ float mids[16];
  __shared__ __align__(16) float2 bk[128 * 32];  // [bucket][lane]
  __shared__ float c1s[kGroup];
  __shared__ float wmax[qz::kThreads / 32];
  __shared__ uint32_t abort_flag;
  float* buf = reinterpret_cast<float*>(qsm);                        // [kBufs][16384]
  uint64_t* full = reinterpret_cast<uint64_t*>(qsm + qz::kBufs * qz::kGroupBytes);
  const int tid = threadIdx.x;
  pdl_launch_dependents();
  if (tid < 16) mids[tid] = tab.mid[tid];
  for (int i = tid; i < 128 * 32; i += qz::kThreads)
    bk[i] = make_float2(bkt.thr[i >> 5], __uint_as_float(static_cast<uint32_t>(bkt.lo[i >> 5])));
  const bool fast = bkt.exact_only == 0;
  const uint32_t zc = static_cast<uint32_t>(tab.zero_code);
  const uint32_t lane_tab = smem_addr(bk) + static_cast<uint32_t>(tid & 31) * 8u;
  const int h32 = tid >> 4, l16 = tid & 15;
  const int64_t ngroups = (nblocks + kGroup - 1) / kGroup;
  bool bad = false;

  auto group_bytes = [&](int64_t g) {
    const int64_t nb = nblocks - g * kGroup < kGroup ? nblocks - g * kGroup : kGroup;
    return static_cast<uint32_t>(nb * kBlock * 4);
  };
  auto issue = [&](int64_t g, int b) {  // thread 0: stream group g into buffer b
    const uint32_t bytes = group_bytes(g);
    mbar_arrive_expect_tx(&full[b], bytes);
    const uint8_t* src = reinterpret_cast<const uint8_t*>(W + g * (kGroup * kBlock));
    uint8_t* dst = reinterpret_cast<uint8_t*>(buf + b * (kGroup * kBlock));
    for (uint32_t off = 0; off < bytes; off += qz::kChunk)
      bulk_load(dst + off, src + off, bytes - off < qz::kChunk ? bytes - off : qz::kChunk, &full[b]);
  };
  // launched with programmatic dependent launch: the set-up above overlaps the kernel before
  // on the stream, whose completion (and memory) this waits for before any global access
  pdl_wait();
  if (tid == 0) {
    abort_flag = 0u;
    for (int b = 0; b < qz::kBufs; ++b) mbar_init(&full[b], 1);
    fence_mbar_init();
    for (int b = 0; b < qz::kBufs; ++b)
      if (blockIdx.x + b * static_cast<int64_t>(gridDim.x) < ngroups)
        issue(blockIdx.x + b * static_cast<int64_t>(gridDim.x), b);
  }
  __syncthreads();

  int it = 0;
  for (int64_t g = blockIdx.x; g < ngroups; g += gridDim.x, ++it) {
    const int b = it % qz::kBufs;
    const int nb = static_cast<int>(group_bytes(g) / (kBlock * 4));
    if (!mbar_wait(&full[b], static_cast<uint32_t>(it / qz::kBufs) & 1u, &abort_flag)) break;
    const float* gb = buf + b * (kGroup * kBlock);
#pragma unroll
    for (int p = 0; p < kGroup / 32; ++p) {
      const int blk = p * 32 + h32;
      float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
      if (blk < nb) x = *reinterpret_cast<const float4*>(gb + blk * kBlock + l16 * 4);
      float a = fmax_nan(fmax_nan(fabsf(x.x), fabsf(x.y)), fmax_nan(fabsf(x.z), fabsf(x.w)));
      a = fmax_nan(a, __shfl_xor_sync(0xffffffffu, a, 8));
      a = fmax_nan(a, __shfl_xor_sync(0xffffffffu, a, 4));
      a = fmax_nan(a, __shfl_xor_sync(0xffffffffu, a, 2));
      a = fmax_nan(a, __shfl_xor_sync(0xffffffffu, a, 1));
      bad |= !(a <= 3.402823466e38f);  // the block holds a NaN or an infinity
      if (blk < nb) {
        if (l16 == 0) c1s[blk] = a;
        uint32_t k0, k1, k2, k3;
        bool near = !(fast && a >= 0x1p-120f);  // RN(1/c1) finite and normal
        if (!near) {
          const float rc = __frcp_rn(a);
          k0 = nf4_code_fast(x.x, rc, lane_tab, near);
          k1 = nf4_code_fast(x.y, rc, lane_tab, near);
          k2 = nf4_code_fast(x.z, rc, lane_tab, near);
          k3 = nf4_code_fast(x.w, rc, lane_tab, near);
        }
        if (near) {  // rare: some weight lies next to a threshold, or c1 is tiny
          k0 = nf4_code_exact(x.x, a, mids, zc);
          k1 = nf4_code_exact(x.y, a, mids, zc);
          k2 = nf4_code_exact(x.z, a, mids, zc);
          k3 = nf4_code_exact(x.w, a, mids, zc);
        }
        const uint32_t packed = ((k0 << 4) | k1) | (((k2 << 4) | k3) << 8);
        *reinterpret_cast<uint16_t*>(codes + g * (kGroup * kBlock / 2) + blk * 32 + l16 * 2) =
            static_cast<uint16_t>(packed);
      }
    }
    __syncthreads();  // every thread is done with buffer b and has written its c1s
    if (tid == 0 && g + qz::kBufs * static_cast<int64_t>(gridDim.x) < ngroups) {
      fence_proxy_async_smem();  // the reads above come before the copy that overwrites b
      issue(g + qz::kBufs * static_cast<int64_t>(gridDim.x), b);
    }
    // second level: c2 = max over the group's block scales; s2 = c2 / top; q8 = code(c1 / s2)
    const float c1 = (tid < nb) ? c1s[tid] : 0.0f;
    float m = c1;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    if ((tid & 31) == 0) wmax[tid >> 5] = m;
    __syncthreads();
    float c2 = wmax[0];
#pragma unroll
    for (int i = 1; i < qz::kThreads / 32; ++i) c2 = fmaxf(c2, wmax[i]);
    const float sc = __fdiv_rn(c2, scale_format_top(sfmt));
    if (tid < nb) q8[g * kGroup + tid] = scale_code(c1, sc, sfmt);
    if (tid == 0) s2[g] = sc;
    __syncthreads();  // c1s and wmax are rewritten by the next group
  }
  if (bad) report(kDevNonfinite);
}

// Dequantize, one warp per chunk of 1024 consecutive weights (16 blocks, always inside one
// group of 256 blocks): each lane loads its 16 code bytes (32 weights, half a block) with one
// coalesced 16-byte load, the next chunk's codes are loaded before this chunk is converted,
// and the lane's 64 bytes of bf16 go into a 2 KB staging buffer that one bulk copy
// (cp.async.bulk, shared -> global) writes out. Two staging buffers per warp alternate, so the
// warp goes on to its next chunk while the last one's copy drains; the stores are whole lines
// and cost the threads nothing after the issue. The lanes of a quarter-warp write their 16-byte
// pieces in a rotated order (lane pairs start at piece 0, 1, 2, 3), so the eight stores of one
// instruction hit eight distinct bank groups. Launched with programmatic dependent launch: the
// CTAs of a dequantization queued behind another kernel are scheduled while it drains and wait
// for it before any global access.
namespace dq {
constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kChunk = 1024;                 // weights per warp per round
constexpr int kStageBytes = kChunk * 2;      // bf16 of one chunk
}  // namespace dq

__global__ void __launch_bounds__(dq::kThreads) nf4_dequantize_kernel(const uint8_t* __restrict__ codes,
                                                                     const uint8_t* __restrict__ q8,
                                                                     const float* __restrict__ s2,
                                                                     uint16_t* __restrict__ out,
                                                                     int64_t n, Nf4Table tab,
                                                                     int sfmt) {
  __shared__ __align__(128) uint8_t stage[dq::kWarps][2][dq::kStageBytes];
  pdl_launch_dependents();
  uint64_t lv2[8];   // the 16 fp32 levels as pairs (2i low, 2i+1 high)
#pragma unroll
  for (int i = 0; i < 8; ++i)
    asm("mov.b64 %0, {%1, %2};" : "=l"(lv2[i]) : "f"(tab.level[2 * i]), "f"(tab.level[2 * i + 1]));
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t nchunks = (n + dq::kChunk - 1) / dq::kChunk;
  const int64_t wstride = static_cast<int64_t>(gridDim.x) * dq::kWarps;
  // this lane's 32 weights of chunk ch: codes and the block scale (two lanes per block)
  auto load = [&](int64_t ch, uint4& cw, float& k) {
    const int64_t e0 = ch * dq::kChunk + lane * 32;
    if (e0 < n) {
      cw = __ldcs(reinterpret_cast<const uint4*>(codes + e0 / 2));
      const int64_t b = e0 >> 6;
      k = __fmul_rn(scale_code_value(__ldg(q8 + b), sfmt), __ldg(s2 + (b >> 8)));
    }
  };
  uint4 cw = make_uint4(0u, 0u, 0u, 0u);
  float k = 0.f;
  int64_t ch = static_cast<int64_t>(blockIdx.x) * dq::kWarps + warp;
  if (ch < nchunks) load(ch, cw, k);
  for (int round = 0; ch < nchunks; ch += wstride, ++round) {
    uint4 ncw = cw;
    float nk = k;
    if (ch + wstride < nchunks) load(ch + wstride, ncw, nk);
    uint8_t* buf = stage[warp][round & 1];
    if (round >= 2) {   // at most one copy (the last round's) may still read its buffer
      if (lane == 0) bulk_wait_group_read<1>();
      __syncwarp();
    }
    const int64_t base = ch * dq::kChunk;
    if (base + lane * 32 < n) {
      // the lane's 32 weights share one block: its 16 exact products, selected by byte permutes
      const ProdTab pt = build_prod_tab(lv2, k);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int q = (j + (lane >> 1)) & 3;   // piece q: weights 8q .. 8q+7 of the lane
        const uint32_t x = q == 0 ? cw.x : (q == 1 ? cw.y : (q == 2 ? cw.z : cw.w));
        *reinterpret_cast<uint4*>(buf + lane * 64 + q * 16) = dequant8_tab(x, pt);
      }
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      const int64_t cnt = n - base < dq::kChunk ? n - base : dq::kChunk;   // a multiple of 64
      bulk_store(out + base, buf, static_cast<uint32_t>(cnt * 2));
      bulk_commit_group();
    }
    cw = ncw;
    k = nk;
  }
  if (lane == 0) bulk_wait_group<0>();   // the output is written before the CTA retires
}

}  // namespace qlora
