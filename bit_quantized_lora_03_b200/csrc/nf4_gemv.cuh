// Fused NF4-dequant GEMV for decode shapes (1..16 tokens) and the small LoRA kernels around it.
//
// Y[n][j] = sum_k X[n][k] * W'[k][j] with W' = Wt^T dequantized on the fly: the packed row of
// Wt is read once from HBM as nibbles, each 64-weight block is turned into bf16 in registers
// (w' = bf16(level * (q8 * s2)), exactly the values nf4_dequantize produces) and fed to the
// tensor cores as the A operand of mma.m16n8k16 with W rows as M and tokens as N. The weight
// never touches shared memory; only the 16 fp32 levels do. ("The core move", goodomens.studio:
// dequantized on the fly, used for the matmul, discarded.)
//
// Work split: a warp owns 64 rows of Wt (4 m16 tiles) and one K slice; the partial sums of the
// K slices meet in an fp32 buffer by atomic adds, and a finalize kernel adds the LoRA term
// sT.L2 and rounds to bf16.
#pragma once

#include "nf4_codec.cuh"

namespace qlora {

struct GemvArgs {
  const uint8_t* codes;
  const uint8_t* q8;
  const float* s2;
  const uint16_t* X;  // t x h bf16
  float* Y32;         // t x o fp32, zeroed by the caller
  int64_t h;
  int64_t o;
  int t;
  int blocks_per_split;  // K slice length in 64-weight blocks
  Nf4Table tab;
};

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// bf16x2 of the two weights in one packed byte: low half = high nibble (the even element).
__device__ __forceinline__ uint32_t deq_byte(uint32_t byte, float k, const float* lv) {
  return pack_bf16x2(__fmul_rn(lv[(byte >> 4) & 15u], k), __fmul_rn(lv[byte & 15u], k));
}

// Fragment mapping (g = lane / 4, q = lane % 4). For block b and mma step s (0..3), lane q
// holds the 4 consecutive k = 64b + 16q + 4s + {0,1,2,3}; they fill its logical k slots
// {2q, 2q+1} (a0/a1, b0) and {2q+8, 2q+9} (a2/a3, b1). Because A and B use the same
// permutation of k, the products are unchanged. A row g of the m16 tile is Wt row base+g.
template <int NT>  // number of n8 token tiles: 1 for t <= 8, 2 for t <= 16
__global__ void __launch_bounds__(128) nf4_gemv_kernel(const GemvArgs args) {
  __shared__ float lv[16];
  if (threadIdx.x < 16) lv[threadIdx.x] = args.tab.level[threadIdx.x];
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, q = lane & 3;
  const int64_t row0 = (static_cast<int64_t>(blockIdx.x) * 4 + warp) * 64;
  if (row0 >= args.o) return;
  const int64_t nblk = args.h / kBlock;
  const int64_t b_begin = static_cast<int64_t>(blockIdx.y) * args.blocks_per_split;
  const int64_t b_end = (b_begin + args.blocks_per_split < nblk) ? b_begin + args.blocks_per_split : nblk;
  const int64_t row_bytes = args.h / 2;

  float acc[4][NT][4];
#pragma unroll
  for (int mt = 0; mt < 4; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[mt][nt][i] = 0.f;

  // token rows this lane feeds into B (zero beyond t)
  const uint16_t* xrow[NT];
  bool xval[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int n = g + 8 * nt;
    xval[nt] = n < args.t;
    xrow[nt] = args.X + static_cast<int64_t>(xval[nt] ? n : 0) * args.h;
  }

  for (int64_t b = b_begin; b < b_end; ++b) {
    uint2 cw[4][2];
    float kv[4][2];
#pragma unroll
    for (int mt = 0; mt < 4; ++mt)
#pragma unroll
      for (int rr = 0; rr < 2; ++rr) {
        const int64_t row = row0 + mt * 16 + g + rr * 8;
        cw[mt][rr] = __ldcs(reinterpret_cast<const uint2*>(args.codes + row * row_bytes + b * 32 +
                                                           q * 8));
        const int64_t qi = row * nblk + b;
        kv[mt][rr] = __fmul_rn(static_cast<float>(__ldg(args.q8 + qi)), __ldg(args.s2 + (qi >> 8)));
      }
    uint2 xb[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int s = 0; s < 4; ++s)
        xb[nt][s] = xval[nt] ? __ldg(reinterpret_cast<const uint2*>(xrow[nt] + b * 64 + q * 16 +
                                                                     s * 4))
                             : make_uint2(0u, 0u);
#pragma unroll
    for (int s = 0; s < 4; ++s) {
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) {
        const uint32_t w0 = (s < 2) ? cw[mt][0].x : cw[mt][0].y;
        const uint32_t w1 = (s < 2) ? cw[mt][1].x : cw[mt][1].y;
        const int sh = (s & 1) * 16;
        const uint32_t a0 = deq_byte((w0 >> sh) & 0xFFu, kv[mt][0], lv);
        const uint32_t a2 = deq_byte((w0 >> (sh + 8)) & 0xFFu, kv[mt][0], lv);
        const uint32_t a1 = deq_byte((w1 >> sh) & 0xFFu, kv[mt][1], lv);
        const uint32_t a3 = deq_byte((w1 >> (sh + 8)) & 0xFFu, kv[mt][1], lv);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
          mma_bf16_16816(acc[mt][nt], a0, a1, a2, a3, xb[nt][s].x, xb[nt][s].y);
      }
    }
  }

  // C fragment: c0 = (row g, token 2q), c1 = (row g, 2q+1), c2 = (row g+8, 2q), c3 = (g+8, 2q+1)
#pragma unroll
  for (int mt = 0; mt < 4; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int n = 8 * nt + 2 * q + (i & 1);
        const int64_t row = row0 + mt * 16 + g + ((i >> 1) * 8);
        if (n < args.t) atomicAdd(args.Y32 + static_cast<int64_t>(n) * args.o + row, acc[mt][nt][i]);
      }
}

// Y[n][j] = bf16( Y32[n][j] + sum_c sT[n][c] * L2[c][j] ) with sT = bf16(s . X.L1): the LoRA
// up-projection folded into the GEMV's output conversion. Grid (ceil(o/256), t).
__global__ void __launch_bounds__(256) gemv_lora_finalize_kernel(
    const float* __restrict__ Y32, const uint16_t* __restrict__ sT, const uint16_t* __restrict__ L2,
    uint16_t* __restrict__ Y, int64_t o, int r) {
  __shared__ float sTs[256];
  const int n = blockIdx.y;
  for (int c = threadIdx.x; c < r; c += blockDim.x)
    sTs[c] = bf16_bits_to_float(sT[static_cast<int64_t>(n) * r + c]);
  __syncthreads();
  const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (j >= o) return;
  float y = Y32[static_cast<int64_t>(n) * o + j];
  for (int c = 0; c < r; ++c)
    y = fmaf(sTs[c], bf16_bits_to_float(L2[static_cast<int64_t>(c) * o + j]), y);
  Y[static_cast<int64_t>(n) * o + j] = __bfloat16_as_ushort(__float2bfloat16_rn(y));
}

}  // namespace qlora
