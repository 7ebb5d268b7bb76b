// tcgen05 (5th-generation tensor core) fused NF4 GEMM for the training-shape QLoRA linear on
// sm_100a.
//
// nf4_gemm_kernel<BWD>: the frozen-base product with the NF4 dequantization fused into the
//    producer stage and the LoRA product folded into the same TMEM accumulator:
//       forward  (BWD = false):  Y  = X  . W'   + sT . L2      (M = t, N = o, K = h)
//       backward (BWD = true):   dX = dY . W'^T + sU . L1^T    (M = t, N = h, K = o)
//    ("The algebra", mchromiak.github.io; "QLoRA in LLMs" sections 3-4; "The core move",
//    goodomens.studio: each 4-bit block is dequantized on the fly, used, discarded.)
//    A (X or dY) and the packed codes arrive by TMA; 8 producer warps turn each 64-weight
//    block into bf16 (w' = bf16(level * (q8 * s2)), the exact nf4_dequantize values, selected
//    by byte permutes from a 16-entry product table built in registers per block) and
//    write it straight into the 128-byte-swizzled operand layout the MMA reads: K-major for
//    the forward (rows of Wt are N), MN-major for the backward (rows of Wt are K). A pair of
//    CTAs (a cluster of 2) owns 512 tokens x 256 columns and issues tcgen05.mma.cta_group::2:
//    each CTA dequantizes only its 128 of the 256 columns, and two accumulators per CTA (all
//    512 TMEM columns) make every dequantized tile feed 512 tokens. The h/64 (or o/64) weight
//    K-steps run first, then the r/64 LoRA K-steps (A = sT or sU, B = L2 or L1, both by
//    TMA), so that the kernel can start, by programmatic dependent launch, while the kernel
//    that produces sT or sU is still running. The same 8 warps then drain TMEM to bf16.
//
// (tc_gemm.cuh holds the plain tcgen05 GEMM for the rank-r products.)
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
  const uint16_t* addend;  // NULL, or M x N bf16 added to the accumulator before the rounding;
                           // written by the previous kernel on the stream (waited for first)
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

template <bool kBwd>
__global__ void __launch_bounds__(tc::kThreads, 1)
    nf4_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmP,
                    const __grid_constant__ CUtensorMap tmA2,
                    const __grid_constant__ CUtensorMap tmB2,
                    const __grid_constant__ CUtensorMap tmOut, const Nf4GemmArgs args) {
  using namespace tc;
  extern __shared__ uint8_t smem_raw[];
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
  // Grid x walks the column tiles (two CTAs each) and grid y the 512-token row blocks, so the
  // pairs resident at one time share a few row blocks of A (the larger operand) across all
  // column tiles rather than streaming all of A once per wave.
  const int n0 = (blockIdx.x >> 1) * BN;                 // the pair's 256 output columns
  const int nh0 = n0 + static_cast<int>(rank) * BNH;    // this CTA's 128 of them
  const int mrow = blockIdx.y * PAIR_M + static_cast<int>(rank) * 128;  // + a * 256
  const int total = args.num_kb + args.num_lkb;   // weight K-steps, then the LoRA K-steps
  pdl_launch_dependents();

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
  if (warp == kMmaWarp) {
    tmem_alloc2(tmem_holder, kTmemCols);
    tmem_relinquish2();
  }
  if (warp == kTmaWarp && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmP);
    tma_prefetch_desc(&tmA2);
    tma_prefetch_desc(&tmB2);
    tma_prefetch_desc(&tmOut);
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
        if (i >= args.num_kb) {
          // sT / sU come from the kernel launched just before this one, which may still be
          // running (programmatic dependent launch): wait for it before the first LoRA load
          if (i == args.num_kb) pdl_wait();
          const int li = i - args.num_kb;
          mbar_arrive_expect_tx(&full_ap[slot], A_BYTES + B_BYTES);
          tma_load_2d(a_dst, &tmA2, &full_ap[slot], li * BK, mrow);
          tma_load_2d(a_dst + A_HALF, &tmA2, &full_ap[slot], li * BK, mrow + 256);
          if (!kBwd) {
            // L2 (r x o), MN-major B: this CTA's two 64-column atoms, 8 KB apart
            tma_load_2d(b_dst, &tmB2, &full_ap[slot], nh0, li * BK);
            tma_load_2d(b_dst + 8192, &tmB2, &full_ap[slot], nh0 + 64, li * BK);
          } else {
            // L1 (h x r), K-major B: this CTA's 128 rows of 64 ranks
            tma_load_2d(b_dst, &tmB2, &full_ap[slot], li * BK, nh0);
          }
        } else {
          const int kb = i;
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
        const bool lora = i >= args.num_kb;
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
    uint64_t lv2[8];                 // the 16 fp32 levels as pairs (2i low, 2i+1 high)
#pragma unroll
    for (int i = 0; i < 8; ++i)
      asm("mov.b64 %0, {%1, %2};" : "=l"(lv2[i]) : "f"(args.tab.level[2 * i]), "f"(args.tab.level[2 * i + 1]));
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
    // 8-bit scale and second-level scale of this thread's block, fetched kPf stages ahead into
    // a ring of registers; the loop below is unrolled by kPf so that every ring index is a
    // compile-time constant and a load is waited for only when its stage comes up
    constexpr int kPf = 4;
    const int nk = args.num_kb;
    uint32_t qr[kPf];
    float sr[kPf];
#pragma unroll
    for (int j = 0; j < kPf; ++j) {
      qr[j] = 0u;
      sr[j] = 0.f;
      if (valid && j < nk) {
        const int64_t qi = qbase + static_cast<int64_t>(j) * qstep;
        qr[j] = __ldg(args.q8 + qi);
        sr[j] = __ldg(args.s2 + (qi >> 8));
      }
    }
    bool ok = true;
    for (int i0 = 0; i0 < total && ok; i0 += kPf) {
#pragma unroll
      for (int j = 0; j < kPf; ++j) {
        const int i = i0 + j;
        if (i >= total || !ok) break;
        const int slot = i % STAGES;
        const uint32_t ph = (i / STAGES) & 1;
        if (!mbar_wait(&empty[slot], ph ^ 1u, abort_flag)) { ok = false; break; }
        if (i < nk) {
          const float k = __fmul_rn(static_cast<float>(qr[j]), sr[j]);
          if (valid && i + kPf < nk) {
            const int64_t qi = qbase + static_cast<int64_t>(i + kPf) * qstep;
            qr[j] = __ldg(args.q8 + qi);
            sr[j] = __ldg(args.s2 + (qi >> 8));
          }
          if (!mbar_wait(&full_ap[slot], ph, abort_flag)) { ok = false; break; }
          if (valid) {
            const ProdTab tab = build_prod_tab(lv2, k);
            const uint4 c = *reinterpret_cast<const uint4*>(sP + slot * P_BYTES + pk_off);
            const uint32_t words[4] = {c.x, c.y, c.z, c.w};
            uint8_t* dst = sB + slot * B_BYTES + out_off;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int ch = half * 4 + u;   // 16-byte chunk (8 weights) within the 128-byte row
              *reinterpret_cast<uint4*>(dst + ((ch ^ swz) << 4)) = dequant8_tab(words[u], tab);
            }
          }
          fence_proxy_async_smem();
        }
        mbar_arrive(&full_b[slot]);
      }
    }

    // ---------------- epilogue: TMEM -> registers -> bf16 -> shared -> TMA store -------------
    // Warp w drains 32 accumulator rows (TMEM lanes 32 (w mod 4) .., accumulator w / 4) in
    // rounds of 64 columns: four 16-column TMEM loads before one wait, the bf16 row (128 bytes
    // per lane) into a 32 x 64 staging tile, 128-byte swizzled as the output tensor map
    // expects (so the eight lanes of each quarter-warp write eight distinct bank groups), then
    // one TMA store of the tile: whole 128-byte lines instead of 32 scattered row pieces per
    // store instruction. Two staging tiles per warp (8 KB, in the drained stage buffers) let a
    // round's shared-memory writes overlap the previous round's store.
    const bool done = mbar_wait(acc_full, 0, abort_flag);
    tc_fence_after();
    if (done && !*abort_flag) {
      if (args.addend) pdl_wait();
      const int acc = warp >> 2, quad = warp & 3;
      const int row0 = mrow + acc * 256 + quad * 32;
      const int row = row0 + lane;
      const uint32_t lane_addr =
          tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(acc * BN);
      uint8_t* stage_tile = smem + warp * 8192;
      const bool any_row = row0 < args.M;   // warp-uniform: rows past M are not stored
      // N is a multiple of 64, so a round is either wholly inside the output or wholly past it
      for (int c0 = 0; c0 < BN / 16; c0 += 4) {
        if (n0 + c0 * 16 >= args.N) break;
        uint8_t* buf = stage_tile + ((c0 >> 2) & 1) * 4096;
        if (c0 >= 8) {   // the store issued from this tile two rounds ago has read it
          if (lane == 0) bulk_wait_group_read<1>();
          __syncwarp();
        }
        uint32_t vv[4][16];
#pragma unroll
        for (int q = 0; q < 4; ++q) tmem_ld_16(lane_addr + (c0 + q) * 16, vv[q]);
        tmem_ld_wait();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t (&v)[16] = vv[q];
          if (args.addend && row < args.M) {
            const int64_t off = static_cast<int64_t>(row) * args.N + n0 + (c0 + q) * 16;
            const uint4* ad = reinterpret_cast<const uint4*>(args.addend + off);
            const uint4 a0 = ad[0], a1 = ad[1];
            const uint32_t w[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
#pragma unroll
            for (int k = 0; k < 8; ++k) {  // word k: column 2k in the low half, 2k + 1 high
              v[2 * k] = __float_as_uint(__uint_as_float(v[2 * k]) + __uint_as_float(w[k] << 16));
              v[2 * k + 1] = __float_as_uint(__uint_as_float(v[2 * k + 1]) +
                                             __uint_as_float(w[k] & 0xFFFF0000u));
            }
          }
          uint4 o0, o1;
          o0.x = pack_bf16x2(__uint_as_float(v[0]), __uint_as_float(v[1]));
          o0.y = pack_bf16x2(__uint_as_float(v[2]), __uint_as_float(v[3]));
          o0.z = pack_bf16x2(__uint_as_float(v[4]), __uint_as_float(v[5]));
          o0.w = pack_bf16x2(__uint_as_float(v[6]), __uint_as_float(v[7]));
          o1.x = pack_bf16x2(__uint_as_float(v[8]), __uint_as_float(v[9]));
          o1.y = pack_bf16x2(__uint_as_float(v[10]), __uint_as_float(v[11]));
          o1.z = pack_bf16x2(__uint_as_float(v[12]), __uint_as_float(v[13]));
          o1.w = pack_bf16x2(__uint_as_float(v[14]), __uint_as_float(v[15]));
          uint8_t* rowp = buf + lane * 128;
          *reinterpret_cast<uint4*>(rowp + (((2 * q) ^ (lane & 7)) << 4)) = o0;
          *reinterpret_cast<uint4*>(rowp + (((2 * q + 1) ^ (lane & 7)) << 4)) = o1;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && any_row) {
          tma_store_2d(&tmOut, buf, n0 + c0 * 16, row0);
          bulk_commit_group();
        }
      }
      if (lane == 0) bulk_wait_group<0>();   // the output is written before the CTA retires
      __syncwarp();
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();   // no CTA leaves while its peer may still signal it or read its TMEM slice
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc2(tmem_base, kTmemCols);
  }
  // completion stays in stream order even when an abort skipped the wait before the LoRA steps
  if (threadIdx.x == 0) pdl_wait();
}

}  // namespace qlora
