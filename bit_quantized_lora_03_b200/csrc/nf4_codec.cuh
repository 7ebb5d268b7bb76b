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

#include "qlora_common.cuh"

namespace qlora {

// NF4 levels and decision thresholds, passed by value as a kernel parameter.
struct Nf4Table {
  float level[16];
  float mid[16];  // 15 thresholds, mid[15] unused
};

constexpr int kBlock = 64;
constexpr int kGroup = 256;

// Nearest-level code of x = w / c1 as the number of thresholds strictly below x, found by a
// four-step binary search over the sorted thresholds in shared memory.
__device__ __forceinline__ uint32_t nf4_code_of(float w, float c1, const float* mids) {
  if (c1 == 0.0f) return 7u;
  const float x = __fdiv_rn(w, c1);
  uint32_t c = (x > mids[7]) ? 8u : 0u;
  c += (x > mids[c + 3]) ? 4u : 0u;
  c += (x > mids[c + 1]) ? 2u : 0u;
  c += (x > mids[c]) ? 1u : 0u;
  return c;
}

// One CTA of 256 threads per group of 256 blocks (16384 weights), grid-stride over groups.
// Half-warp h16 of iteration `it` owns block it*16 + h16; each thread loads one float4.
__global__ void __launch_bounds__(256) nf4_quantize_kernel(const float* __restrict__ W,
                                                           uint8_t* __restrict__ codes,
                                                           uint8_t* __restrict__ q8,
                                                           float* __restrict__ s2,
                                                           int64_t nblocks, Nf4Table tab) {
  __shared__ float mids[16];
  __shared__ float c1s[kGroup];
  __shared__ float wmax[8];
  const int tid = threadIdx.x;
  if (tid < 16) mids[tid] = tab.mid[tid];
  __syncthreads();
  const int h16 = tid >> 4, l16 = tid & 15;
  const int64_t ngroups = (nblocks + kGroup - 1) / kGroup;
  bool bad = false;

  for (int64_t g = blockIdx.x; g < ngroups; g += gridDim.x) {
    const int nb = static_cast<int>((nblocks - g * kGroup < kGroup ? nblocks - g * kGroup : kGroup));
    const float* base = W + g * (kGroup * kBlock);
    float4 v[16];
#pragma unroll
    for (int it = 0; it < 16; ++it) {
      if (it * 16 + h16 < nb)
        v[it] = __ldcs(reinterpret_cast<const float4*>(base + it * 1024 + tid * 4));
      else
        v[it] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int it = 0; it < 16; ++it) {
      const int blk = it * 16 + h16;
      const float4 x = v[it];
      bad |= !(isfinite(x.x) && isfinite(x.y) && isfinite(x.z) && isfinite(x.w));
      float a = fmaxf(fmaxf(fabsf(x.x), fabsf(x.y)), fmaxf(fabsf(x.z), fabsf(x.w)));
      a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 8));
      a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 4));
      a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 2));
      a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
      if (blk < nb) {
        if (l16 == 0) c1s[blk] = a;
        const uint32_t k0 = nf4_code_of(x.x, a, mids), k1 = nf4_code_of(x.y, a, mids);
        const uint32_t k2 = nf4_code_of(x.z, a, mids), k3 = nf4_code_of(x.w, a, mids);
        const uint32_t packed = ((k0 << 4) | k1) | (((k2 << 4) | k3) << 8);
        *reinterpret_cast<uint16_t*>(codes + g * (kGroup * kBlock / 2) + it * 512 + tid * 2) =
            static_cast<uint16_t>(packed);
      }
    }
    __syncthreads();
    // second level: c2 = max over the group's block scales; s2 = c2 / 255; q8 = rint(c1 / s2)
    const float c1 = (tid < nb) ? c1s[tid] : 0.0f;
    float m = c1;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    if ((tid & 31) == 0) wmax[tid >> 5] = m;
    __syncthreads();
    float c2 = wmax[0];
#pragma unroll
    for (int i = 1; i < 8; ++i) c2 = fmaxf(c2, wmax[i]);
    const float sc = __fdiv_rn(c2, 255.0f);
    if (tid < nb) {
      int qv = 0;
      if (sc != 0.0f) qv = min(255, max(0, __float2int_rn(__fdiv_rn(c1, sc))));
      q8[g * kGroup + tid] = static_cast<uint8_t>(qv);
    }
    if (tid == 0) s2[g] = sc;
    __syncthreads();
  }
  if (bad) report(kDevNonfinite);
}

// Dequantize: each work item is 8 weights (4 packed bytes -> 16 bytes of bf16); a thread
// takes 4 items spaced a grid apart so that 4 loads are in flight before any compute, and
// consecutive threads touch consecutive memory (coalesced 4-byte loads, 16-byte stores).
__global__ void __launch_bounds__(256) nf4_dequantize_kernel(const uint8_t* __restrict__ codes,
                                                             const uint8_t* __restrict__ q8,
                                                             const float* __restrict__ s2,
                                                             uint16_t* __restrict__ out,
                                                             int64_t nitems, Nf4Table tab) {
  __shared__ float lv[16];
  if (threadIdx.x < 16) lv[threadIdx.x] = tab.level[threadIdx.x];
  __syncthreads();
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i0 < nitems;
       i0 += 4 * stride) {
    uint32_t w[4];
    float k[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t it = i0 + u * stride;
      if (it < nitems) {
        w[u] = __ldcs(reinterpret_cast<const unsigned int*>(codes) + it);
        const int64_t b = it >> 3;  // 8 items per 64-weight block
        k[u] = __fmul_rn(static_cast<float>(__ldg(q8 + b)), __ldg(s2 + (b >> 8)));
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t it = i0 + u * stride;
      if (it < nitems) {
        const uint32_t x = w[u];
        const float kk = k[u];
        uint4 o;
        o.x = pack_bf16x2(__fmul_rn(lv[(x >> 4) & 15u], kk), __fmul_rn(lv[x & 15u], kk));
        o.y = pack_bf16x2(__fmul_rn(lv[(x >> 12) & 15u], kk), __fmul_rn(lv[(x >> 8) & 15u], kk));
        o.z = pack_bf16x2(__fmul_rn(lv[(x >> 20) & 15u], kk), __fmul_rn(lv[(x >> 16) & 15u], kk));
        o.w = pack_bf16x2(__fmul_rn(lv[(x >> 28) & 15u], kk), __fmul_rn(lv[(x >> 24) & 15u], kk));
        __stcs(reinterpret_cast<uint4*>(out) + it, o);
      }
    }
  }
}

}  // namespace qlora
