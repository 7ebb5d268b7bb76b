// Plain TMA-fed tcgen05 GEMM for the rank-r products of the QLoRA linear on sm_100a:
// T = X.L1 and U = dY.L2^T (rounded to bf16 sT, sU) and the adapter gradients dL1 = X^T.sU and
// dL2^T = dY^T.sT ("The algebra", mchromiak.github.io; "QLoRA in LLMs" sections 3-4); with
// epilogue variants for the adapter merge (W' + s.L1.L2, "QLoRA in LLMs" section 11) and the
// dropout-masked adapter term of dX (section 12). Both operands by TMA (either major-ness),
// N tiles of up to 256 columns, split-K as one thread-block cluster whose CTAs reduce through
// distributed shared memory.
//
// Every wait is bounded (qlora::mbar_wait); on expiry the CTA reports QLORA_DEV_TIMEOUT,
// stops issuing, waits for its own copies and MMAs in flight, frees TMEM and returns.
#pragma once

#include "nf4_gemm.cuh"

namespace qlora {

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
constexpr int kSmemPerSm = 233472 - 4096;   // shared memory of one SM, less two CTAs' reserve and static arrays
constexpr int kMergeStagingBytes = 4 * 8192;  // the merge epilogue's staging tiles (4 warps)
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
  kOutRowMajor = 0,   // out32[m * ld + n] = acc (fp32)
  kOutTransposed = 1, // out32[n * ld + m] = acc (fp32)
  kOutRoundBf16 = 2,  // out16a[m * Ncols + n] = bf16(alpha * acc) (and out16b if set)
  kOutMergeNF4 = 3,   // out32[m * ld + n] = W'[m][n] + alpha * acc, W' the dequantized NF4
                      // row m (of ld = h weights) of the packed weight in the args
  kOutMaskBf16 = 4,   // out16a[m * Ncols + n] = bf16(M[m][n] * alpha * acc), M the dropout keep
                      // mask: bit (e mod 8) of keep_bits[e / 8], e = m * Ncols + n (no split-K)
};

// Split-K runs as a thread-block cluster of `splits` CTAs along grid z (at most 8): each CTA
// leaves its fp32 partial tile in its own shared memory, and after a cluster barrier rank q
// sums its share of the tile's rows over all ranks through distributed shared memory and
// writes them. No global atomics, no zeroed accumulators, no arrival counters.
// How a launch relates to the kernel before it on the stream (programmatic dependent launch):
enum TcPdl : int {
  kPdlNone = 0,       // launched normally: starts after all earlier work
  kPdlWaitFirst = 1,  // may start early; reads nothing before the previous kernel completes
  kPdlWaitLast = 2,   // may start early and needs nothing from the previous kernel; it still
                      // completes only after it, so completion stays in stream order
};

struct TcGemmArgs {
  int M;
  int Ncols;         // real number of output columns (<= BNp, a multiple of 16)
  int BNp;           // MMA N: Ncols rounded up to a multiple of 16
  int num_kb;        // ceil(K / 64)
  int kb_per_split;
  int splits;        // gridDim.z = cluster size
  int stages;
  float alpha;
  int out_mode;
  float* out32;
  int64_t ld;
  uint16_t* out16a;
  uint16_t* out16b;
  int pdl;           // TcPdl
  // kOutMergeNF4: the packed weight whose dequantized rows are added (Ncols = ld = h)
  const uint8_t* codes;
  const uint8_t* q8;
  const float* s2;
  Nf4Table tab;
  const uint8_t* keep_bits;  // kOutMaskBf16: the keep mask, one bit per element
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

// kMinCtas: CTAs that must fit on one SM at once (bounds the registers per thread); the merge
// runs four small CTAs per SM, the rank-r products one or two large ones.
template <bool A_MN, bool B_MN, int kMinCtas = 1>
__global__ void __launch_bounds__(tcg::kThreads, kMinCtas)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmOut, const TcGemmArgs args) {
  using namespace tcg;
  extern __shared__ uint8_t smem_raw[];
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
  const int nb0 = blockIdx.x * BNp;  // this CTA's first output column (N tiles along grid x)
  const int kb0 = blockIdx.z * args.kb_per_split;
  const int kb1 = min(args.num_kb, kb0 + args.kb_per_split);
  const int nk = kb1 - kb0;
  const uint32_t tmem_cols = BNp <= 32 ? 32u : (BNp <= 64 ? 64u : (BNp <= 128 ? 128u : 256u));
  const int b_atoms = (BNp + 63) / 64;
  const uint32_t bbytes = static_cast<uint32_t>(b_bytes(BNp, B_MN));
  pdl_launch_dependents();

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
      if (args.pdl == kPdlWaitFirst) pdl_wait();  // every global access follows the loads
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
          tma_load_2d(b_dst, &tmB, &full[slot], kb * BK, nb0);
        } else {
          for (int a = 0; a < b_atoms; ++a)
            tma_load_2d(b_dst + a * 8192, &tmB, &full[slot], nb0 + a * 64, kb * BK);
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
    const int rloc = warp * 32 + lane;  // row within the tile
    const int row = m0 + rloc;
    const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(warp * 32) << 16);
    // split-K: the partial tile goes to shared memory (the drained stage buffers), rows of
    // BNp + 4 floats so that eight threads' 16-byte stores cover all 32 banks
    float* part = reinterpret_cast<float*>(smem) + static_cast<size_t>(rloc) * (BNp + 4);
    // one accumulator chunk of 16 columns -> this CTA's destination
    auto emit = [&](const uint32_t (&v)[16], int n0) {
      if (args.splits > 1) {
#pragma unroll
        for (int e = 0; e < 16; e += 4)
          *reinterpret_cast<float4*>(part + n0 + e) =
              make_float4(__uint_as_float(v[e]), __uint_as_float(v[e + 1]),
                          __uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
        return;
      }
      n0 += nb0;
      if (row >= args.M || n0 >= args.Ncols) return;
      if (args.out_mode == kOutTransposed) {
#pragma unroll
        for (int e = 0; e < 16; ++e)
          args.out32[static_cast<int64_t>(n0 + e) * args.ld + row] = __uint_as_float(v[e]);
      } else if (args.out_mode == kOutRoundBf16) {
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
          *reinterpret_cast<float4*>(dst + e) =
              make_float4(__uint_as_float(v[e]), __uint_as_float(v[e + 1]),
                          __uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
      }
    };
    const int nchunks = BNp / 16;
    if (args.out_mode == kOutMaskBf16) {   // uniform over the block: all 128 threads reach
                                           // the named barrier below
      // The tile (128 rows x BNp bf16) is staged in the drained stage buffers, then written
      // row by row by whole warps (512 contiguous bytes per warp store instead of 32 rows x 16
      // bytes). Staging layout: 64-column blocks of 128 rows x 128 bytes, the 16-byte chunk
      // index XORed with (row & 7), so that both the row-wise writes and the column-wise reads
      // of eight consecutive threads hit eight distinct bank groups.
      // After a timeout elsewhere in the CTA the tile is unspecified (the status word says so)
      // but every access stays inside the stage buffers and the output.
      uint8_t* stile = smem;
      const bool go = __all_sync(0xFFFFFFFFu, ok && !*abort_flag);   // tcgen05.ld is warp-wide
      const int rok = row < args.M;
      const int64_t erow = static_cast<int64_t>(row) * args.Ncols;
      for (int c = 0; go && c < nchunks; ++c) {
        uint32_t v[16];
        tmem_ld_16(lane_addr + c * 16, v);
        tmem_ld_wait();
        const int col = nb0 + c * 16;   // a multiple of 16: two bytes of mask bits
        const uint32_t keep = (rok && col < args.Ncols)
            ? *reinterpret_cast<const uint16_t*>(args.keep_bits + (erow + col) / 8) : 0u;
        const float a = args.alpha;
        uint32_t o[8];
#pragma unroll
        for (int k = 0; k < 8; ++k)  // word k: element 2k in the low half, 2k + 1 high
          o[k] = pack_bf16x2(((keep >> (2 * k)) & 1u) ? a * __uint_as_float(v[2 * k]) : 0.f,
                             ((keep >> (2 * k + 1)) & 1u) ? a * __uint_as_float(v[2 * k + 1]) : 0.f);
        const int blk = c >> 2, ch = (c & 3) * 2;   // 64-column block, first 16-byte chunk
        uint8_t* rowp = stile + blk * (128 * 128) + rloc * 128;
        *reinterpret_cast<uint4*>(rowp + (((ch) ^ (rloc & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
        *reinterpret_cast<uint4*>(rowp + (((ch + 1) ^ (rloc & 7)) << 4)) = make_uint4(o[4], o[5], o[6], o[7]);
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");   // the four epilogue warps
      const int chunks_row = BNp / 8;                     // 16-byte chunks per tile row
      const int ncols_here = min(BNp, args.Ncols - nb0);
      for (int rr = warp; go && rr < BM; rr += 4) {
        const int grow = m0 + rr;
        if (grow >= args.M) break;
        for (int q = lane; q < chunks_row; q += 32) {
          if (q * 8 >= ncols_here) break;
          const int blk = q >> 3, ch = q & 7;
          const uint4 val = *reinterpret_cast<const uint4*>(stile + blk * (128 * 128) + rr * 128 +
                                                            ((ch ^ (rr & 7)) << 4));
          *reinterpret_cast<uint4*>(args.out16a + static_cast<int64_t>(grow) * args.Ncols + nb0 + q * 8) = val;
        }
      }
    } else if (ok && !*abort_flag && args.out_mode == kOutMergeNF4 &&
               (kMinCtas == 1 || STAGES * SB < kMergeStagingBytes)) {
      // the merge runs only in its own instantiation (four CTAs per SM), and
      // the staging tiles must lie inside the drained stage buffers: the host plans enough
      // stages, and a launch with fewer reports an error instead of writing past them
      if (lane == 0) report(kDevLaunch);
    } else if (kMinCtas > 1 && ok && !*abort_flag && args.out_mode == kOutMergeNF4 && args.splits == 1) {
      // 32 columns (half an NF4 block of this row) per round: the next round's 16 code bytes
      // and block scale are loaded while this round's two accumulator chunks come out of TMEM.
      // The fp32 row segment (128 bytes per lane) goes into a 32 x 32 staging tile, 128-byte
      // swizzled as the output tensor map expects (the eight lanes of a quarter-warp write
      // eight distinct bank groups), and one TMA store writes it: whole 128-byte lines rather
      // than 32 scattered 16-byte pieces per store instruction. Two 4 KB tiles per warp
      // alternate, so that a round fills one while the store of the round before still reads
      // the other. They lie in the drained stage buffers (8 KB per warp), and the CTA is small
      // (one stage, a 128-column tile in 128 TMEM columns, a register bound), so four CTAs
      // share an SM and one's epilogue overlaps the others' set-up and loads.
      const int64_t rowbase = static_cast<int64_t>(row) * args.ld;
      const bool rok = row < args.M;
      const int row0 = m0 + warp * 32;
      uint8_t* buf = smem + warp * 8192;
      auto load_half = [&](int col, uint4& cw, float& k) {
        if (rok && col < args.Ncols) {
          cw = *reinterpret_cast<const uint4*>(args.codes + (rowbase + col) / 2);
          const int64_t blk = (rowbase + col) / kBlock;
          k = __fmul_rn(static_cast<float>(args.q8[blk]), args.s2[blk / kGroup]);
        }
      };
      uint4 cw = make_uint4(0u, 0u, 0u, 0u);
      float kk = 0.f;
      load_half(nb0, cw, kk);
      uint64_t lv2[8];   // the 16 fp32 levels as pairs (2i low, 2i+1 high)
#pragma unroll
      for (int i = 0; i < 8; ++i)
        asm("mov.b64 %0, {%1, %2};" : "=l"(lv2[i]) : "f"(args.tab.level[2 * i]), "f"(args.tab.level[2 * i + 1]));
      for (int c = 0, round = 0; c < nchunks; c += 2, ++round) {
        const int col0 = nb0 + c * 16;
        if (col0 >= args.Ncols) break;   // Ncols % 64 == 0: whole rounds only
        uint32_t v[2][16];
        tmem_ld_16(lane_addr + c * 16, v[0]);
        tmem_ld_16(lane_addr + (c + 1) * 16, v[1]);
        uint4 ncw = cw;
        float nk = kk;
        if (c + 2 < nchunks) load_half(nb0 + (c + 2) * 16, ncw, nk);
        tmem_ld_wait();
        uint8_t* tile = buf + (round & 1) * 4096;
        if (round >= 2) {   // at most one store (the last round's) may still read its tile
          if (lane == 0) bulk_wait_group_read<1>();
          __syncwarp();
        }
        const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
        uint8_t* rowp = tile + lane * 128;
        // the round's 32 weights share one block: its 16 exact products bf16(level x k),
        // selected by byte permutes
        const ProdTab pt = build_prod_tab(lv2, kk);
#pragma unroll
        for (int w = 0; w < 4; ++w) {          // 8 weights per code word
          const uint4 b = dequant8_tab(words[w], pt);   // element 2j + 1 in the high half
          const uint32_t bw[4] = {b.x, b.y, b.z, b.w};
          float o[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const uint32_t wq = (e & 1) ? (bw[e >> 1] & 0xFFFF0000u) : (bw[e >> 1] << 16);
            o[e] = __fadd_rn(__uint_as_float(wq), __fmul_rn(args.alpha, __uint_as_float(v[w >> 1][(w & 1) * 8 + e])));
          }
          // columns 8w .. 8w+7 of the tile: 16-byte chunks 2w and 2w + 1
          *reinterpret_cast<float4*>(rowp + (((2 * w) ^ (lane & 7)) << 4)) = make_float4(o[0], o[1], o[2], o[3]);
          *reinterpret_cast<float4*>(rowp + (((2 * w + 1) ^ (lane & 7)) << 4)) = make_float4(o[4], o[5], o[6], o[7]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && row0 < args.M) {
          tma_store_2d(&tmOut, tile, col0, row0);
          bulk_commit_group();
        }
        cw = ncw;
        kk = nk;
      }
      if (lane == 0) bulk_wait_group<0>();   // the output is written before the CTA retires
      __syncwarp();
    } else if (ok && !*abort_flag) {
      // up to four 16-column TMEM loads in flight before one wait (the counts are warp-uniform)
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
    } else if (args.splits > 1) {
      uint32_t z[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) z[e] = 0u;
      for (int c = 0; c < nchunks; ++c) emit(z, c * 16);
    }
    if (threadIdx.x == 0) QLORA_STAMP(6);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, tmem_cols);
  }
  if (args.splits > 1) {
    cluster_sync();  // every rank's partial tile is in its shared memory
    const int S = args.splits;
    const int q = static_cast<int>(cluster_ctarank());
    const int r0 = q * BM / S, r1 = (q + 1) * BM / S, nr = r1 - r0;
    const float* part0 = reinterpret_cast<const float*>(smem);
    const int ld_s = BNp + 4;
    const int tile_cols = args.Ncols - nb0 < BNp ? args.Ncols - nb0 : BNp;
    if (!*abort_flag) {
      if (args.out_mode == kOutTransposed) {
        // four adjacent columns per thread (one 16-byte read from each rank); consecutive
        // threads take consecutive rows, so each of the four column stores is coalesced
        const int nq = tile_cols / 4;
        for (int e = threadIdx.x; e < nr * nq; e += kThreads) {
          const int rl = r0 + e % nr, n = 4 * (e / nr);
          float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
          for (int p = 0; p < S; ++p) {
            const float4 v = ld_dsmem_f32x4(part0 + rl * ld_s + n, static_cast<uint32_t>(p));
            sum.x += v.x; sum.y += v.y; sum.z += v.z; sum.w += v.w;
          }
          if (m0 + rl >= args.M || nb0 + n >= args.Ncols) continue;
          float* o = args.out32 + static_cast<int64_t>(nb0 + n) * args.ld + m0 + rl;
          o[0] = sum.x;
          o[args.ld] = sum.y;
          o[2 * args.ld] = sum.z;
          o[3 * args.ld] = sum.w;
        }
      } else {
        const int nq = tile_cols / 4;
        for (int e = threadIdx.x; e < nr * nq; e += kThreads) {
          const int rl = r0 + e / nq, n = 4 * (e % nq);
          float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
          for (int p = 0; p < S; ++p) {
            const float4 v = ld_dsmem_f32x4(part0 + rl * ld_s + n, static_cast<uint32_t>(p));
            sum.x += v.x; sum.y += v.y; sum.z += v.z; sum.w += v.w;
          }
          if (m0 + rl >= args.M || nb0 + n >= args.Ncols) continue;
          if (args.out_mode == kOutRoundBf16) {
            const float a = args.alpha;
            uint2 o;
            o.x = pack_bf16x2(a * sum.x, a * sum.y);
            o.y = pack_bf16x2(a * sum.z, a * sum.w);
            const int64_t off = static_cast<int64_t>(m0 + rl) * args.Ncols + nb0 + n;
            *reinterpret_cast<uint2*>(args.out16a + off) = o;
            if (args.out16b) *reinterpret_cast<uint2*>(args.out16b + off) = o;
          } else {
            *reinterpret_cast<float4*>(args.out32 + static_cast<int64_t>(m0 + rl) * args.ld + nb0 + n) = sum;
          }
        }
      }
    }
    cluster_sync();  // the partial tiles stay in place until every rank has read them
  }
  if (args.pdl == kPdlWaitLast && threadIdx.x == 0) pdl_wait();
  if (threadIdx.x == 0) QLORA_STAMP(7);
}

}  // namespace qlora
