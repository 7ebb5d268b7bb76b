// tcgen05 (5th-generation tensor core) GEMMs for the training-shape QLoRA linear on sm_100a.
//
// 1) nf4_gemm_kernel<BWD>: the frozen-base product with the NF4 dequantization fused into the
//    producer stage and the LoRA product folded into the same TMEM accumulator:
//       forward  (BWD = false):  Y  = X  . W'   + sT . L2      (M = t, N = o, K = h)
//       backward (BWD = true):   dX = dY . W'^T + sU . L1^T    (M = t, N = h, K = o)
//    ("The algebra", mchromiak.github.io; "QLoRA in LLMs" sections 3-4; "The core move",
//    goodomens.studio: each 4-bit block is dequantized on the fly, used, discarded.)
//    A (X or dY) and the packed codes arrive by TMA; 8 producer warps turn each 64-weight
//    block into bf16 (w' = bf16(level * (q8 * s2)), the exact nf4_dequantize values) and
//    write it straight into the 128-byte-swizzled operand layout the MMA reads: K-major for
//    the forward (rows of Wt are N), MN-major for the backward (rows of Wt are K). A pair of
//    CTAs (a cluster of 2) owns 512 tokens x 256 columns and issues tcgen05.mma.cta_group::2:
//    each CTA dequantizes only its 128 of the 256 columns, and two accumulators per CTA (all
//    512 TMEM columns) make every dequantized tile feed 512 tokens. The r/64 LoRA K-steps
//    (A = sT or sU, B = L2 or L1, both by TMA) run first, then the h/64 (or o/64) weight
//    K-steps. The same 8 warps then drain TMEM to bf16.
//
// 2) tc_gemm_kernel<A_MN, B_MN>: a plain TMA-fed tcgen05 GEMM (both operands by TMA, either
//    major-ness) with split-K and fp32 atomic or bf16 output, for the rank-r products
//    T = X.L1, U = dY.L2^T, dL1 = X^T.sU and dL2^T = dY^T.sT.
//
// Every wait is bounded (qlora::mbar_wait); on expiry the CTA reports QLORA_DEV_TIMEOUT,
// stops issuing, waits for its own copies and MMAs in flight, frees TMEM and returns.
#pragma once

#include "nf4_codec.cuh"

namespace qlora {
namespace tc {

// A CTA pair (thread-block cluster of 2) owns 512 tokens x 256 output columns. One
// tcgen05.mma.cta_group::2 computes 256 tokens x 256 columns: each CTA supplies 128 rows of A
// and 128 of the 256 columns of B from its own shared memory and holds its 128 x 256 fp32
// slice of the accumulator in its own tensor memory. Two such accumulators per CTA (all 512
// TMEM columns) cover the 512 tokens, so each dequantized half-tile feeds 512 tokens.
constexpr int PAIR_M = 512;
constexpr int BN = 256;        // output columns per pair
constexpr int BNH = BN / 2;    // columns of B held (and dequantized) by each CTA
constexpr int BK = 64;         // K per stage: one 128-byte swizzle row of bf16, one NF4 block
constexpr int STAGES = 4;
constexpr int A_HALF = 128 * BK * 2;       // 16 KB: this CTA's 128 rows of one accumulator
constexpr int A_BYTES = 2 * A_HALF;        // 32 KB
constexpr int B_BYTES = BNH * BK * 2;      // 16 KB
constexpr int P_BYTES = BNH * BK / 2;      // 4 KB of packed codes
constexpr int kWorkWarps = 8;              // warps 0-7: dequant producers, then epilogue
constexpr int kTmaWarp = 8;
constexpr int kMmaWarp = 9;                // even CTA: MMA issuer; odd CTA: readiness relay
constexpr int kThreads = 10 * 32;
constexpr int kTmemCols = 512;

constexpr size_t nf4_gemm_smem_bytes() {
  return 1024 /* alignment slack */ + STAGES * (A_BYTES + B_BYTES + P_BYTES) + 256;
}

}  // namespace tc

struct Nf4GemmArgs {
  const uint8_t* q8;
  const float* s2;
  int64_t h;        // in_features: row length of Wt
  int M;            // tokens
  int N;            // output columns: o (forward) or h (backward)
  int num_kb;       // weight K-steps: h/64 (forward) or o/64 (backward)
  int num_lkb;      // LoRA K-steps: ceil(r/64)
  uint16_t* out;    // M x N bf16, row stride N
  Nf4Table tab;
};

// Wait for an mbarrier phase ignoring the abort flag (used only to drain in-flight copies
// after an abort), still bounded by the timeout.
__device__ __forceinline__ void mbar_drain(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > kWaitTimeoutNs) {
      report(kDevTimeout);
      return;
    }
  }
}

// bf16x2 of (a * k, b * k): one packed fp32x2 multiply (IEEE round to nearest per lane, the
// same two products as two separate multiplies), then round-to-nearest-even to bf16.
__device__ __forceinline__ uint32_t scale_pack_bf16x2(float a, float b, uint64_t kk) {
  uint64_t ab, r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(ab) : "f"(a), "f"(b));
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(ab), "l"(kk));
  float ra, rb;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(ra), "=f"(rb) : "l"(r));
  return pack_bf16x2(ra, rb);
}

// Eight packed codes (one 32-bit word, element 2j in the high nibble of byte j) -> eight bf16
// weights level[code] * k. The level table is 16 fp32 in shared memory; the byte offsets
// 4*code of all eight nibbles come from two mask operations and one byte-permute each.
__device__ __forceinline__ uint4 dequant8(uint32_t x, uint64_t kk, const float* lv) {
  const uint32_t hi4 = (x >> 2) & 0x3C3C3C3Cu;   // byte j: 4 * high nibble
  const uint32_t lo4 = (x << 2) & 0x3C3C3C3Cu;   // byte j: 4 * low nibble
  const char* base = reinterpret_cast<const char*>(lv);
  uint32_t w[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t oh = __byte_perm(hi4, 0u, 0x4440u + j);
    const uint32_t ol = __byte_perm(lo4, 0u, 0x4440u + j);
    const float a = *reinterpret_cast<const float*>(base + oh);
    const float b = *reinterpret_cast<const float*>(base + ol);
    w[j] = scale_pack_bf16x2(a, b, kk);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

template <bool kBwd>
__global__ void __launch_bounds__(tc::kThreads, 1)
    nf4_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmP,
                    const __grid_constant__ CUtensorMap tmA2,
                    const __grid_constant__ CUtensorMap tmB2, const Nf4GemmArgs args) {
  using namespace tc;
  extern __shared__ uint8_t smem_raw[];
  __shared__ float lv[16];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + STAGES * A_BYTES;
  uint8_t* sP = sB + STAGES * B_BYTES;
  uint64_t* full_ap = reinterpret_cast<uint64_t*>(sP + STAGES * P_BYTES);
  uint64_t* full_b = full_ap + STAGES;
  uint64_t* peer_ready = full_b + STAGES;   // even CTA: the odd CTA's stage is complete
  uint64_t* empty = peer_ready + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(acc_full + 1);
  volatile uint32_t* abort_flag = tmem_holder + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();             // 0: MMA issuer, 1: its peer
  const int n0 = blockIdx.y * BN;                        // the pair's 256 output columns
  const int nh0 = n0 + static_cast<int>(rank) * BNH;    // this CTA's 128 of them
  const int mrow = (blockIdx.x >> 1) * PAIR_M + static_cast<int>(rank) * 128;  // + a * 256
  const int total = args.num_lkb + args.num_kb;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_ap[s], 1);
      mbar_init(&full_b[s], kWorkWarps * 32);
      mbar_init(&peer_ready[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    *abort_flag = 0u;
    fence_mbar_init();
  }
  if (threadIdx.x < 16) lv[threadIdx.x] = args.tab.level[threadIdx.x];
  if (warp == kMmaWarp) {
    tmem_alloc2(tmem_holder, kTmemCols);
    tmem_relinquish2();
  }
  if (warp == kTmaWarp && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmP);
    tma_prefetch_desc(&tmA2);
    tma_prefetch_desc(&tmB2);
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();   // both CTAs' barriers exist before any cross-CTA arrive
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == kTmaWarp) {
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < total; ++i) {
        const int slot = i % STAGES;
        const uint32_t ph = (i / STAGES) & 1;
        if (!mbar_wait(&empty[slot], ph ^ 1u, abort_flag)) break;
        uint8_t* a_dst = sA + slot * A_BYTES;
        uint8_t* b_dst = sB + slot * B_BYTES;
        if (i < args.num_lkb) {
          mbar_arrive_expect_tx(&full_ap[slot], A_BYTES + B_BYTES);
          tma_load_2d(a_dst, &tmA2, &full_ap[slot], i * BK, mrow);
          tma_load_2d(a_dst + A_HALF, &tmA2, &full_ap[slot], i * BK, mrow + 256);
          if (!kBwd) {
            // L2 (r x o), MN-major B: this CTA's two 64-column atoms, 8 KB apart
            tma_load_2d(b_dst, &tmB2, &full_ap[slot], nh0, i * BK);
            tma_load_2d(b_dst + 8192, &tmB2, &full_ap[slot], nh0 + 64, i * BK);
          } else {
            // L1 (h x r), K-major B: this CTA's 128 rows of 64 ranks
            tma_load_2d(b_dst, &tmB2, &full_ap[slot], i * BK, nh0);
          }
        } else {
          const int kb = i - args.num_lkb;
          mbar_arrive_expect_tx(&full_ap[slot], A_BYTES + P_BYTES);
          tma_load_2d(a_dst, &tmA, &full_ap[slot], kb * BK, mrow);
          tma_load_2d(a_dst + A_HALF, &tmA, &full_ap[slot], kb * BK, mrow + 256);
          if (!kBwd) {
            tma_load_2d(sP + slot * P_BYTES, &tmP, &full_ap[slot], kb * (BK / 2), nh0);
          } else {
            tma_load_2d(sP + slot * P_BYTES, &tmP, &full_ap[slot], nh0 / 2, kb * BK);
            tma_load_2d(sP + slot * P_BYTES + 2048, &tmP, &full_ap[slot], nh0 / 2 + 32, kb * BK);
          }
        }
        issued = i + 1;
      }
      if (*abort_flag) {
        // make sure no copy is still writing this CTA's shared memory before it exits
        for (int j = (issued > STAGES ? issued - STAGES : 0); j < issued; ++j)
          mbar_drain(&full_ap[j % STAGES], (j / STAGES) & 1);
      }
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0 && rank == 0) {
      // M = 256 per instruction (128 rows from each CTA), N = 256 (128 columns from each)
      constexpr uint32_t kIdescMain = idesc_bf16(256, BN, false, kBwd);
      constexpr uint32_t kIdescLora = idesc_bf16(256, BN, false, !kBwd);
      bool any = false;
      for (int i = 0; i < total; ++i) {
        const int slot = i % STAGES;
        const uint32_t ph = (i / STAGES) & 1;
        if (!mbar_wait(&full_ap[slot], ph, abort_flag)) break;
        if (!mbar_wait(&full_b[slot], ph, abort_flag)) break;
        if (!mbar_wait_cluster(&peer_ready[slot], ph, abort_flag)) break;
        tc_fence_after();
        const bool lora = i < args.num_lkb;
        const bool b_mn = lora ? !kBwd : kBwd;
        const uint32_t idesc = lora ? kIdescLora : kIdescMain;
        const uint32_t a_addr = smem_addr(sA + slot * A_BYTES);
        const uint32_t b_addr = smem_addr(sB + slot * B_BYTES);
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          const uint64_t bd = b_mn ? sw128_desc(b_addr + kk * 2048, 8192, 1024)
                                   : sw128_desc(b_addr + kk * 32, 16, 1024);
#pragma unroll
          for (int a = 0; a < 2; ++a) {
            const uint64_t ad = sw128_desc(a_addr + a * A_HALF + kk * 32, 16, 1024);
            umma2_bf16(tmem_base + a * BN, ad, bd, idesc, (i > 0 || kk > 0) ? 1u : 0u);
          }
        }
        umma2_commit_multicast(&empty[slot], 0x3);   // frees the stage in both CTAs
        any = true;
      }
      // completes in both CTAs once every MMA above has finished (also after an abort)
      umma2_commit_multicast(acc_full, 0x3);
      if (*abort_flag && any) mbar_drain(acc_full, 0);
    } else if (lane == 0) {
      // odd CTA: tell the issuer when this CTA's half of each stage is in shared memory
      for (int i = 0; i < total; ++i) {
        const int slot = i % STAGES;
        const uint32_t ph = (i / STAGES) & 1;
        if (!mbar_wait(&full_ap[slot], ph, abort_flag)) break;
        if (!mbar_wait(&full_b[slot], ph, abort_flag)) break;
        mbar_arrive_remote(&peer_ready[slot], 0);
      }
    }
  } else {
    // ---------------- warps 0-7: dequant producers (half a 64-weight block per thread per
    // stage: 128 blocks of this CTA's 128 columns), then the epilogue -----------------------
    const int p = threadIdx.x;       // 0..255
    const int blk = p >> 1, half = p & 1;
    const int64_t nblk_row = args.h / kBlock;
    int64_t qbase, qstep;       // q8 index of this thread's block at weight K-step kb: qbase + kb*qstep
    int out_off, pk_off, swz;
    bool valid;
    if (!kBwd) {
      // block row blk of this CTA's columns is Wt row nh0 + blk; its block kb is K-step kb
      const int64_t j = nh0 + blk;
      valid = j < args.N;
      qbase = j * nblk_row;
      qstep = 1;
      pk_off = blk * 32 + half * 16;
      out_off = (blk >> 3) * 1024 + (blk & 7) * 128;
      swz = blk & 7;
    } else {
      // K row jl of the stage is Wt row kb*64 + jl; local column atom a is blocks nh0/64 + a
      const int jl = blk & 63, a = blk >> 6;
      valid = (nh0 + a * 64) < args.N;
      qbase = static_cast<int64_t>(jl) * nblk_row + (nh0 / 64) + a;
      qstep = 64 * nblk_row;
      pk_off = a * 2048 + jl * 32 + half * 16;
      out_off = a * 8192 + (jl >> 3) * 1024 + (jl & 7) * 128;
      swz = jl & 7;
    }
    // 8-bit scale and second-level scale of this thread's block, fetched two stages ahead
    const int nk = args.num_kb;
    uint32_t q_cur = 0u, q_nxt = 0u;
    float s_cur = 0.f, s_nxt = 0.f;
    if (valid && nk > 0) {
      q_cur = __ldg(args.q8 + qbase);
      s_cur = __ldg(args.s2 + (qbase >> 8));
    }
    if (valid && nk > 1) {
      const int64_t qi = qbase + qstep;
      q_nxt = __ldg(args.q8 + qi);
      s_nxt = __ldg(args.s2 + (qi >> 8));
    }
    bool ok = true;
    for (int i = 0; i < total && ok; ++i) {
      const int slot = i % STAGES;
      const uint32_t ph = (i / STAGES) & 1;
      if (!mbar_wait(&empty[slot], ph ^ 1u, abort_flag)) { ok = false; break; }
      if (i >= args.num_lkb) {
        const int kb = i - args.num_lkb;
        const float k = __fmul_rn(static_cast<float>(q_cur), s_cur);
        q_cur = q_nxt;
        s_cur = s_nxt;
        if (valid && kb + 2 < nk) {
          const int64_t qi = qbase + static_cast<int64_t>(kb + 2) * qstep;
          q_nxt = __ldg(args.q8 + qi);
          s_nxt = __ldg(args.s2 + (qi >> 8));
        }
        if (!mbar_wait(&full_ap[slot], ph, abort_flag)) { ok = false; break; }
        if (valid) {
          uint64_t kk;
          asm("mov.b64 %0, {%1, %1};" : "=l"(kk) : "f"(k));
          const uint4 c = *reinterpret_cast<const uint4*>(sP + slot * P_BYTES + pk_off);
          const uint32_t words[4] = {c.x, c.y, c.z, c.w};
          uint8_t* dst = sB + slot * B_BYTES + out_off;
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int ch = half * 4 + u;   // 16-byte chunk (8 weights) within the 128-byte row
            *reinterpret_cast<uint4*>(dst + ((ch ^ swz) << 4)) = dequant8(words[u], kk, lv);
          }
        }
        fence_proxy_async_smem();
      }
      mbar_arrive(&full_b[slot]);
    }

    // ---------------- epilogue: TMEM -> registers -> bf16 -> global -------------------------
    const bool done = mbar_wait(acc_full, 0, abort_flag);
    tc_fence_after();
    if (done && !*abort_flag) {
      const int acc = warp >> 2, quad = warp & 3;
      const int row = mrow + acc * 256 + quad * 32 + lane;
      const uint32_t lane_addr =
          tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(acc * BN);
      for (int c = 0; c < BN / 16; ++c) {
        if (n0 + c * 16 >= args.N) break;  // N is a multiple of 64: whole chunks only
        uint32_t v[16];
        tmem_ld_16(lane_addr + c * 16, v);
        tmem_ld_wait();
        if (row < args.M) {
          uint4 o0, o1;
          o0.x = pack_bf16x2(__uint_as_float(v[0]), __uint_as_float(v[1]));
          o0.y = pack_bf16x2(__uint_as_float(v[2]), __uint_as_float(v[3]));
          o0.z = pack_bf16x2(__uint_as_float(v[4]), __uint_as_float(v[5]));
          o0.w = pack_bf16x2(__uint_as_float(v[6]), __uint_as_float(v[7]));
          o1.x = pack_bf16x2(__uint_as_float(v[8]), __uint_as_float(v[9]));
          o1.y = pack_bf16x2(__uint_as_float(v[10]), __uint_as_float(v[11]));
          o1.z = pack_bf16x2(__uint_as_float(v[12]), __uint_as_float(v[13]));
          o1.w = pack_bf16x2(__uint_as_float(v[14]), __uint_as_float(v[15]));
          uint4* dst = reinterpret_cast<uint4*>(args.out + static_cast<int64_t>(row) * args.N +
                                                n0 + c * 16);
          dst[0] = o0;
          dst[1] = o1;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();   // no CTA leaves while its peer may still signal it or read its TMEM slice
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc2(tmem_base, kTmemCols);
  }
}

// ------------------------------------------------------------------------------------------
// Plain TMA-fed tcgen05 GEMM for the rank-r products.
// D (M x Ncols) = A (M x K) . B (K x Ncols), Ncols <= 256 (one N tile), split-K over
// blockIdx.z. A_MN / B_MN select MN-major operands (the TMA boxes are 64 x 64 atoms then).
// The pipeline depth is chosen by the host from the B tile size.
// ------------------------------------------------------------------------------------------
namespace tcg {
constexpr int BM = 128, BK = 64, MAX_STAGES = 8;
constexpr int A_BYTES = BM * BK * 2;        // 16 KB
constexpr int kThreads = 6 * 32;            // warps 0-3 epilogue, 4 TMA, 5 MMA
constexpr int kTmaWarp = 4, kMmaWarp = 5;
constexpr int kMaxSmem = 232448 - 1024;     // opt-in maximum per CTA on sm_100, less static smem
// B tile bytes for a given MMA N (BNp, multiple of 16) and major-ness
__host__ __device__ constexpr int b_bytes(int BNp, bool b_mn) {
  return b_mn ? ((BNp + 63) / 64) * 8192 : BNp * 128;
}
__host__ __device__ constexpr int stage_bytes(int BNp, bool b_mn) {
  return A_BYTES + ((b_bytes(BNp, b_mn) + 1023) / 1024) * 1024;
}
constexpr size_t smem_bytes(int stages, int BNp, bool b_mn) {
  return 1024 + static_cast<size_t>(stages) * stage_bytes(BNp, b_mn) + 256;
}
}  // namespace tcg

enum TcOutMode : int {
  kOutAtomicRowMajor = 0,   // out32[m * ld + n] += acc
  kOutAtomicTransposed = 1, // out32[n * ld + m] += acc
  kOutRoundBf16 = 2,        // out32 (m * Ncols + n) += acc; the last CTA of each M tile then
                            // writes bf16(alpha * out32) to out16a (and out16b if set)
};

struct TcGemmArgs {
  int M;
  int Ncols;         // real number of output columns (<= BNp)
  int BNp;           // MMA N: Ncols rounded up to a multiple of 16
  int num_kb;        // ceil(K / 64)
  int kb_per_split;
  int splits;        // gridDim.z
  int stages;
  float alpha;
  int out_mode;
  float* out32;
  int64_t ld;
  uint16_t* out16a;
  uint16_t* out16b;
  unsigned* counters;  // kOutRoundBf16: one per M tile, zeroed by the caller
};

#ifdef QLORA_TRACE
constexpr int kTraceCtas = 8192;
__device__ unsigned long long g_trace[kTraceCtas][8];
__device__ __forceinline__ void trace_stamp(int slot) {
  const unsigned cta = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z);
  if (cta < kTraceCtas) g_trace[cta][slot] = global_timer_ns();
}
#define QLORA_STAMP(i) trace_stamp(i)
#else
#define QLORA_STAMP(i)
#endif

__device__ __forceinline__ void red_add_v4(float* addr, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b),
               "f"(c), "f"(d)
               : "memory");
}

template <bool A_MN, bool B_MN>
__global__ void __launch_bounds__(tcg::kThreads, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const TcGemmArgs args) {
  using namespace tcg;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t last_flag;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int BNp = args.BNp;
  const int STAGES = args.stages;
  const int SB = stage_bytes(BNp, B_MN);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * SB);
  uint64_t* empty = full + MAX_STAGES;
  uint64_t* acc_full = empty + MAX_STAGES;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(acc_full + 1);
  volatile uint32_t* abort_flag = tmem_holder + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * BM;
  const int kb0 = blockIdx.z * args.kb_per_split;
  const int kb1 = min(args.num_kb, kb0 + args.kb_per_split);
  const int nk = kb1 - kb0;
  const uint32_t tmem_cols = BNp <= 32 ? 32u : (BNp <= 64 ? 64u : (BNp <= 128 ? 128u : 256u));
  const int b_atoms = (BNp + 63) / 64;
  const uint32_t bbytes = static_cast<uint32_t>(b_bytes(BNp, B_MN));

  if (threadIdx.x == 0) {
    QLORA_STAMP(0);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    *abort_flag = 0u;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_holder, tmem_cols);
    tmem_relinquish();
  }
  if (warp == kTmaWarp && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  if (threadIdx.x == 0) QLORA_STAMP(1);

  if (warp == kTmaWarp) {
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < nk; ++i) {
        const int slot = i % STAGES;
        const uint32_t ph = (i / STAGES) & 1;
        if (!mbar_wait(&empty[slot], ph ^ 1u, abort_flag)) break;
        const int kb = kb0 + i;
        mbar_arrive_expect_tx(&full[slot], A_BYTES + bbytes);
        uint8_t* a_dst = smem + slot * SB;
        if (!A_MN) {
          tma_load_2d(a_dst, &tmA, &full[slot], kb * BK, m0);
        } else {
          tma_load_2d(a_dst, &tmA, &full[slot], m0, kb * BK);
          tma_load_2d(a_dst + 8192, &tmA, &full[slot], m0 + 64, kb * BK);
        }
        uint8_t* b_dst = a_dst + A_BYTES;
        if (!B_MN) {
          tma_load_2d(b_dst, &tmB, &full[slot], kb * BK, 0);
        } else {
          for (int a = 0; a < b_atoms; ++a)
            tma_load_2d(b_dst + a * 8192, &tmB, &full[slot], a * 64, kb * BK);
        }
        if (i == 0) QLORA_STAMP(2);
        issued = i + 1;
      }
      if (*abort_flag) {
        for (int j = (issued > STAGES ? issued - STAGES : 0); j < issued; ++j)
          mbar_drain(&full[j % STAGES], (j / STAGES) & 1);
      }
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(BM, BNp, A_MN, B_MN);
      bool any = false;
      for (int i = 0; i < nk; ++i) {
        const int slot = i % STAGES;
        const uint32_t ph = (i / STAGES) & 1;
        if (!mbar_wait(&full[slot], ph, abort_flag)) break;
        if (i == 0) QLORA_STAMP(3);
        if (i == nk - 1) QLORA_STAMP(4);
        tc_fence_after();
        const uint32_t a_addr = smem_addr(smem + slot * SB);
        const uint32_t b_addr = a_addr + A_BYTES;
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          const uint64_t ad = A_MN ? sw128_desc(a_addr + kk * 2048, 8192, 1024)
                                   : sw128_desc(a_addr + kk * 32, 16, 1024);
          const uint64_t bd = B_MN ? sw128_desc(b_addr + kk * 2048, 8192, 1024)
                                   : sw128_desc(b_addr + kk * 32, 16, 1024);
          umma_bf16(tmem_base, ad, bd, idesc, (i > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&empty[slot]);
        any = true;
      }
      umma_commit(acc_full);
      if (*abort_flag && any) mbar_drain(acc_full, 0);
    }
  } else {
    // ---------------- epilogue warps 0-3: one accumulator row per thread ------------------
    const bool ok = (nk > 0) && mbar_wait(acc_full, 0, abort_flag);
    if (threadIdx.x == 0) QLORA_STAMP(5);
    tc_fence_after();
    if (ok && !*abort_flag) {
      const int row = m0 + warp * 32 + lane;
      const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(warp * 32) << 16);
      const bool direct_bf16 = args.out_mode == kOutRoundBf16 && args.splits == 1;
      // one accumulator chunk of 16 columns -> the output mode's destination
      auto emit = [&](const uint32_t (&v)[16], int n0) {
        if (row >= args.M || n0 >= args.Ncols) return;  // Ncols is a multiple of 16
        if (args.out_mode == kOutAtomicTransposed) {
#pragma unroll
          for (int e = 0; e < 16; ++e)
            atomicAdd(args.out32 + static_cast<int64_t>(n0 + e) * args.ld + row,
                      __uint_as_float(v[e]));
        } else if (direct_bf16) {
          const float a = args.alpha;
          uint4 o0, o1;
          o0.x = pack_bf16x2(a * __uint_as_float(v[0]), a * __uint_as_float(v[1]));
          o0.y = pack_bf16x2(a * __uint_as_float(v[2]), a * __uint_as_float(v[3]));
          o0.z = pack_bf16x2(a * __uint_as_float(v[4]), a * __uint_as_float(v[5]));
          o0.w = pack_bf16x2(a * __uint_as_float(v[6]), a * __uint_as_float(v[7]));
          o1.x = pack_bf16x2(a * __uint_as_float(v[8]), a * __uint_as_float(v[9]));
          o1.y = pack_bf16x2(a * __uint_as_float(v[10]), a * __uint_as_float(v[11]));
          o1.z = pack_bf16x2(a * __uint_as_float(v[12]), a * __uint_as_float(v[13]));
          o1.w = pack_bf16x2(a * __uint_as_float(v[14]), a * __uint_as_float(v[15]));
          const int64_t off = static_cast<int64_t>(row) * args.Ncols + n0;
          reinterpret_cast<uint4*>(args.out16a + off)[0] = o0;
          reinterpret_cast<uint4*>(args.out16a + off)[1] = o1;
          if (args.out16b) {
            reinterpret_cast<uint4*>(args.out16b + off)[0] = o0;
            reinterpret_cast<uint4*>(args.out16b + off)[1] = o1;
          }
        } else {
          float* dst = args.out32 + static_cast<int64_t>(row) * args.ld + n0;
#pragma unroll
          for (int e = 0; e < 16; e += 4)
            red_add_v4(dst + e, __uint_as_float(v[e]), __uint_as_float(v[e + 1]),
                       __uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
        }
      };
      // up to four 16-column TMEM loads in flight before one wait (the counts are warp-uniform)
      const int nchunks = BNp / 16;
      for (int c = 0; c < nchunks; c += 4) {
        uint32_t v0[16], v1[16], v2[16], v3[16];
        tmem_ld_16(lane_addr + c * 16, v0);
        if (c + 1 < nchunks) tmem_ld_16(lane_addr + (c + 1) * 16, v1);
        if (c + 2 < nchunks) tmem_ld_16(lane_addr + (c + 2) * 16, v2);
        if (c + 3 < nchunks) tmem_ld_16(lane_addr + (c + 3) * 16, v3);
        tmem_ld_wait();
        emit(v0, c * 16);
        if (c + 1 < nchunks) emit(v1, (c + 1) * 16);
        if (c + 2 < nchunks) emit(v2, (c + 2) * 16);
        if (c + 3 < nchunks) emit(v3, (c + 3) * 16);
      }
      // partial sums must be visible device-wide before this CTA is counted as arrived
      if (args.out_mode == kOutRoundBf16 && args.splits > 1) __threadfence();
    }
    if (threadIdx.x == 0) QLORA_STAMP(6);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, tmem_cols);
  }
  // kOutRoundBf16 with split-K: the last CTA of this M tile to finish converts the summed
  // fp32 rows to bf16(alpha * sum). Nobody waits on anybody: earlier CTAs just exit.
  if (args.out_mode == kOutRoundBf16 && args.splits > 1 && nk > 0) {
    if (threadIdx.x == 0) {
      __threadfence();
      const unsigned prev = atomicAdd(args.counters + blockIdx.y, 1u);
      last_flag = (prev == static_cast<unsigned>(args.splits - 1)) ? 1u : 0u;
      __threadfence();
    }
    __syncthreads();
    if (last_flag && warp < 4 && !*abort_flag) {
      const int row = m0 + warp * 32 + lane;
      if (row < args.M) {
        const float* src = args.out32 + static_cast<int64_t>(row) * args.Ncols;
        uint16_t* da = args.out16a + static_cast<int64_t>(row) * args.Ncols;
        uint16_t* db = args.out16b ? args.out16b + static_cast<int64_t>(row) * args.Ncols : nullptr;
        // 64 columns (16 independent 16-byte loads) in flight per round
        for (int n0 = 0; n0 < args.Ncols; n0 += 64) {
          float4 x[16];
#pragma unroll
          for (int u = 0; u < 16; ++u)
            if (n0 + 4 * u < args.Ncols)
              x[u] = __ldcg(reinterpret_cast<const float4*>(src + n0 + 4 * u));
#pragma unroll
          for (int u = 0; u < 16; ++u) {
            if (n0 + 4 * u >= args.Ncols) break;
            uint2 o;
            o.x = pack_bf16x2(args.alpha * x[u].x, args.alpha * x[u].y);
            o.y = pack_bf16x2(args.alpha * x[u].z, args.alpha * x[u].w);
            *reinterpret_cast<uint2*>(da + n0 + 4 * u) = o;
            if (db) *reinterpret_cast<uint2*>(db + n0 + 4 * u) = o;
          }
        }
      }
    }
  }
  if (threadIdx.x == 0) QLORA_STAMP(7);
}

}  // namespace qlora
