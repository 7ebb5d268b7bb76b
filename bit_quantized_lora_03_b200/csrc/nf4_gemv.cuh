// Fused NF4-dequant GEMV for decode shapes (1..16 tokens) and the LoRA finalize kernel.
//
// Y[n][j] = sum_k X[n][k] * W'[k][j] with W' = Wt^T dequantized on the fly: the packed row of
// Wt is read once from HBM as nibbles, each weight is turned into its exact bf16 value
// (w' = bf16(level * (q8 * s2)), the nf4_dequantize value) in registers and fed to the tensor
// cores as the A operand of mma.m16n8k16 (W rows as M, tokens as N). ("The core move",
// goodomens.studio: dequantized on the fly, used for the matmul, discarded.)
//
// Dequantization of one packed byte (two weights): a byte permute forms the shared-memory
// address of the (level[high nibble], level[low nibble]) fp32 pair directly -- the table sits
// on a 64 KB boundary and holds one copy of the 256 pairs per lane (entry e of lane l at
// 256 e + 8 l), so the permute only drops the code byte into bits 8..15 of this lane's slot
// address and the 32 lanes never collide on a bank -- then one 64-bit shared load, one packed
// fp32x2 multiply by the block scale and one bf16x2 pack. The lookups bound the kernel: every
// weight's fp32 level (4 bytes) comes through the shared-memory pipe.
//
// Work split: one CTA of 16 warps per SM. The work is a list of units -- 32 rows of Wt x 128
// inputs (two 64-weight blocks, 2 KB of codes) -- ordered row tile by row tile, and every warp
// takes an equal contiguous run of it, so the load is balanced to one unit whatever the shape.
// Each warp keeps three units of codes in flight: its lane 0 issues a TMA box load (32 rows x
// 64 bytes) per unit into a three-slot ring of shared memory, so a whole SM has ~96 KB of HBM
// reads outstanding without spending registers on them. The 8-bit block scales of its rows
// arrive in segments of up to 16 units, copied asynchronously one segment ahead; the
// activations come through L1. When the run leaves a row tile, and at its end, the warp adds
// its partial sums to a t x o fp32 buffer (one atomic per output) and the number of units it
// did to the tile's counter; the warp that completes a tile adds the LoRA term sT.L2 to its
// 32 rows and writes them in bf16. sT = bf16(s . X.L1) comes from gemv_lora_down_kernel, one
// cluster of 8 CTAs launched just before, which also zeroes the fp32 buffer and the counters.
#pragma once

#include "nf4_codec.cuh"

namespace qlora {

namespace gv {
// Launch shape (the defaults are the measured best on B200; the macros exist for sweeps)
#ifndef QLORA_GEMV_WARPS
#define QLORA_GEMV_WARPS 16
#endif
#ifndef QLORA_GEMV_DEPTH
#define QLORA_GEMV_DEPTH 3
#endif
#ifndef QLORA_GEMV_SEG
#define QLORA_GEMV_SEG 16
#endif
#ifndef QLORA_GEMV_XAHEAD
#define QLORA_GEMV_XAHEAD 0
#endif
constexpr int kWarps = QLORA_GEMV_WARPS;
constexpr int kThreads = kWarps * 32;
constexpr int kTileRows = 32;                      // rows per unit (two m16 tiles)
constexpr int kUnitK = 128;                        // inputs per unit (two blocks)
constexpr int kUnitBytes = kTileRows * kUnitK / 2; // code bytes per unit (one TMA box)
constexpr int kDepth = QLORA_GEMV_DEPTH;           // units of codes in flight per warp
constexpr bool kXAhead = QLORA_GEMV_XAHEAD != 0;   // activations loaded one unit ahead (t <= 8)
constexpr int kSegUnits = QLORA_GEMV_SEG;          // units per scale segment
// q8 words per row and segment (2 kSegUnits blocks + alignment), rounded up to 2 mod 4,
// which puts the 8 rows of one access (and the word after each) on 16 different banks
constexpr int kSegWords = ((2 * kSegUnits + 6 + 3) / 4 + 1) / 4 * 4 + 2;
constexpr int kSegRowBytes = kSegWords * 4;
constexpr int kSegBytes = kTileRows * kSegRowBytes;
constexpr int kTableBytes = 256 * 32 * 8;          // 64 KB
// per-warp slot: code ring, two scale segments, one mbarrier per ring entry (128-byte multiple)
constexpr int kSlotCodes = 0;
constexpr int kSlotSeg = kDepth * kUnitBytes;
constexpr int kSlotBars = kSlotSeg + 2 * kSegBytes;
constexpr int kSlotBytes = (kSlotBars + kDepth * 8 + 127) / 128 * 128;
// The table must start on a 64 KB boundary of the shared window; warp slots fill the space
// before it and after it. Whatever the window's base, 64 KB + (warps + 1) slots are enough;
// sT (bf16, up to 16 tokens x rank 256) follows them.
constexpr int kMaxTokens = 16;
constexpr int kMaxRank = 256;
constexpr int kDownParts = 8;  // partial sums written by the LoRA-down kernel (one per cluster)
constexpr int kSTBytes = kMaxTokens * kMaxRank * 2;
constexpr size_t slots_end() { return kTableBytes + (kWarps + 1) * static_cast<size_t>(kSlotBytes); }
constexpr size_t smem_bytes() { return slots_end() + kSTBytes; }
static_assert(kSegWords * 4 >= 2 * kSegUnits + 6, "a row segment plus its alignment fits");
static_assert(smem_bytes() <= 232448 - 1024, "fits the opt-in shared memory of one CTA");
}  // namespace gv

struct GemvArgs {
  const uint8_t* codes;
  const uint8_t* q8;
  const float* s2;
  const uint16_t* X;   // t x h bf16
  const float* Tpart;  // gd::kClusters partial sums of X.L1, each t x r fp32
  uint16_t* sT_out;    // t x r bf16 s . X.L1 for the caller (may be null)
  float s;
  const uint16_t* L2;  // r x o bf16
  uint16_t* Y;         // t x o bf16 (output)
  float* Y32;          // t x o fp32, zero on entry
  unsigned* tile_cnt;  // o / 32 unit counters, zero on entry
  int64_t h;
  int64_t o;
  int t;
  int r;
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

__device__ __forceinline__ void cp_async_4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_prev() {  // all groups but the newest landed
  asm volatile("cp.async.wait_group 1;" ::: "memory");
}
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

// bf16x2 of the two weights of byte j of `w` (low half = high nibble = the even element):
// (level[hi] * k, level[lo] * k) from this lane's pair table, packed fp32x2 multiply, RNE.
// lane_slot = table address + 8 * lane, table address a multiple of 65536.
#ifndef QLORA_GEMV_MUL2
#define QLORA_GEMV_MUL2 1
#endif
template <int J>
__device__ __forceinline__ uint32_t gemv_deq_byte(uint32_t w, uint32_t lane_slot, uint64_t kk) {
  const uint32_t addr = __byte_perm(w, lane_slot, 0x7604u | (J << 4));
  uint32_t out;  // bf16x2 (RNE), the first weight in the low half
#if QLORA_GEMV_MUL2
  uint64_t pair, prod;  // fp32x2 (level[hi], level[lo]) and its product with (k, k)
  asm("ld.shared.b64 %0, [%1];" : "=l"(pair) : "r"(addr));  // the table is read-only here
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(prod) : "l"(pair), "l"(kk));
  asm("{\n\t.reg .b32 lo, hi;\n\tmov.b64 {lo, hi}, %1;\n\tcvt.rn.bf16x2.f32 %0, hi, lo;\n\t}"
      : "=r"(out)
      : "l"(prod));
#else
  float lh, ll;
  asm("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(lh), "=f"(ll) : "r"(addr));
  const float k = __uint_as_float(static_cast<uint32_t>(kk));
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(out) : "f"(__fmul_rn(ll, k)), "f"(__fmul_rn(lh, k)));
#endif
  return out;
}

// Lane (g = lane / 4, q = lane % 4) holds, for each m16 tile, rows g and g + 8: the 32 weights
// 32q .. 32q + 31 of the unit (16 bytes per row; q < 2 lies in the unit's first block, q >= 2
// in its second). A unit's codes sit in its ring entry as 32 rows x 64 bytes.
struct GemvCodes {
  uint4 cw[2][2];
};

__device__ __forceinline__ void gemv_read_codes(GemvCodes& d, uint32_t entry, int g, int q) {
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int rr = 0; rr < 2; ++rr)
      d.cw[mt][rr] = lds128(entry + (mt * 16 + rr * 8 + g) * 64 + q * 16);
}

// The activations of a unit for this lane's 32 inputs (zero where the token or the block does
// not exist, so nothing past a row of X is read).
template <int NT>
__device__ __forceinline__ void gemv_load_x(uint4 (&xb)[NT][4], const GemvArgs& a, int64_t unit,
                                            int g, int q, bool kvalid) {
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int n = g + 8 * nt;
    const uint16_t* xr = a.X + static_cast<int64_t>(n < a.t ? n : 0) * a.h + unit * gv::kUnitK + q * 32;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      xb[nt][j] = (n < a.t && kvalid) ? __ldg(reinterpret_cast<const uint4*>(xr + j * 8))
                                      : make_uint4(0u, 0u, 0u, 0u);
  }
}

// Step s (0..7) of a unit: lane q's inputs 32q + 4s + {0,1,2,3} take the fragment's k slots
// {2q, 2q+1} (a0/a1, b0) and {2q+8, 2q+9} (a2/a3, b1): bytes 2s and 2s+1 of its 16 code
// bytes. A and B use the same permutation of k, so the products are unchanged.
template <int S, int NT>
__device__ __forceinline__ void gemv_step(const GemvCodes& d, const uint4 (&xb)[NT][4],
                                          const uint64_t (&kk)[2][2], float (&acc)[2][NT][4],
                                          uint32_t lane_slot) {
  constexpr int J0 = (2 * S) & 3, J1 = (2 * S + 1) & 3, W = S >> 1;
#pragma unroll
  for (int mt = 0; mt < 2; ++mt) {
    const uint4 c0 = d.cw[mt][0], c1 = d.cw[mt][1];
    const uint32_t w0 = W == 0 ? c0.x : W == 1 ? c0.y : W == 2 ? c0.z : c0.w;
    const uint32_t w1 = W == 0 ? c1.x : W == 1 ? c1.y : W == 2 ? c1.z : c1.w;
    const uint32_t a0 = gemv_deq_byte<J0>(w0, lane_slot, kk[mt][0]);
    const uint32_t a2 = gemv_deq_byte<J1>(w0, lane_slot, kk[mt][0]);
    const uint32_t a1 = gemv_deq_byte<J0>(w1, lane_slot, kk[mt][1]);
    const uint32_t a3 = gemv_deq_byte<J1>(w1, lane_slot, kk[mt][1]);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const uint4 x = xb[nt][W];
      const uint32_t b0 = (S & 1) ? x.z : x.x, b1 = (S & 1) ? x.w : x.y;
      mma_bf16_16816(acc[mt][nt], a0, a1, a2, a3, b0, b1);
    }
  }
}

template <int NT>
__device__ __forceinline__ void gemv_compute(const GemvCodes& d, const uint4 (&xb)[NT][4],
                                             const uint64_t (&kk)[2][2], float (&acc)[2][NT][4],
                                             uint32_t lane_slot) {
  gemv_step<0, NT>(d, xb, kk, acc, lane_slot);
  gemv_step<1, NT>(d, xb, kk, acc, lane_slot);
  gemv_step<2, NT>(d, xb, kk, acc, lane_slot);
  gemv_step<3, NT>(d, xb, kk, acc, lane_slot);
  gemv_step<4, NT>(d, xb, kk, acc, lane_slot);
  gemv_step<5, NT>(d, xb, kk, acc, lane_slot);
  gemv_step<6, NT>(d, xb, kk, acc, lane_slot);
  gemv_step<7, NT>(d, xb, kk, acc, lane_slot);
}

// A run of units inside one row tile whose scales share a staging buffer.
struct GemvSeg {
  int64_t tile;  // row tile (32 rows)
  int u0, u1;    // units [u0, u1) of the tile; empty when u0 == u1
};

__device__ __forceinline__ GemvSeg gemv_seg_at(int64_t f, int64_t f_end, int64_t upt) {
  GemvSeg sg;
  if (f >= f_end) {
    sg.tile = 0;
    sg.u0 = sg.u1 = 0;
    return sg;
  }
  sg.tile = f / upt;
  const int64_t u0 = f - sg.tile * upt;
  int64_t u1 = u0 + gv::kSegUnits;
  if (u1 > upt) u1 = upt;
  if (u1 > f_end - sg.tile * upt) u1 = f_end - sg.tile * upt;
  sg.u0 = static_cast<int>(u0);
  sg.u1 = static_cast<int>(u1);
  return sg;
}

// Copy the q8 bytes of a segment (32 rows x blocks [2 u0, 2 u1)) into a staging buffer as
// 4-byte words starting at the word that holds the row's first block. Every word read lies
// inside the q8 array: rows start at multiples of nblk, and o * nblk is a multiple of 4.
__device__ __forceinline__ void gemv_stage_q8(uint32_t dst, const GemvArgs& a, const GemvSeg& sg,
                                              int64_t nblk, int lane) {
  if (sg.u0 == sg.u1) return;
  const int64_t b0 = 2 * static_cast<int64_t>(sg.u0);
  const int64_t b1 = 2 * static_cast<int64_t>(sg.u1) < nblk ? 2 * static_cast<int64_t>(sg.u1) : nblk;
  for (int e = lane; e < gv::kTileRows * gv::kSegWords; e += 32) {
    const int r = e / gv::kSegWords, wd = e - r * gv::kSegWords;
    const int64_t rb = (sg.tile * gv::kTileRows + r) * nblk;
    const int64_t src = ((rb + b0) & ~int64_t(3)) + 4 * wd;
    if (src < ((rb + b1 + 3) & ~int64_t(3)))
      cp_async_4(dst + r * gv::kSegRowBytes + 4 * wd, a.q8 + src);
  }
}

// Partial sums of a row tile -> Y32. C fragment: c0 = (row g, token 2q), c1 = (row g, 2q+1),
// c2 = (row g+8, 2q), c3 = (row g+8, 2q+1) of each m16 tile and token tile.
template <int NT>
__device__ __forceinline__ void gemv_flush(float (&acc)[2][NT][4], const GemvArgs& a,
                                           int64_t tile, int g, int q) {
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int n = 8 * nt + 2 * q + (i & 1);
        const int64_t row = tile * gv::kTileRows + mt * 16 + g + (i >> 1) * 8;
        if (n < a.t) atomicAdd(a.Y32 + static_cast<int64_t>(n) * a.o + row, acc[mt][nt][i]);
        acc[mt][nt][i] = 0.f;
      }
}

// The last warp to add to a row tile finishes it: Y[n][row] = bf16(Y32[n][row] + sum_c
// sT[n][c] L2[c][row]) for its 32 rows, lane = row. The fp32 sums of the other warps are read
// from L2 after the counter showed them all done (each adder fenced before counting).
template <int NT>
__device__ __forceinline__ void gemv_finish_tile(const GemvArgs& a, const uint16_t* sts,
                                                 int64_t tile, int lane) {
  const int64_t row = tile * gv::kTileRows + lane;
  float y[NT * 8];
#pragma unroll
  for (int n = 0; n < NT * 8; ++n)
    y[n] = n < a.t ? __ldcg(a.Y32 + static_cast<int64_t>(n) * a.o + row) : 0.f;
  for (int c0 = 0; c0 < a.r; c0 += 8) {  // r % 16 == 0: eight loads in flight per lane
    float l2[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
      l2[j] = bf16_bits_to_float(__ldg(a.L2 + static_cast<int64_t>(c0 + j) * a.o + row));
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int n = 0; n < NT * 8; ++n)
        if (n < a.t) y[n] = fmaf(bf16_bits_to_float(sts[n * gv::kMaxRank + c0 + j]), l2[j], y[n]);
  }
#pragma unroll
  for (int n = 0; n < NT * 8; ++n)
    if (n < a.t)
      a.Y[static_cast<int64_t>(n) * a.o + row] = __bfloat16_as_ushort(__float2bfloat16_rn(y[n]));
}

template <int NT>  // NT: n8 token tiles (1 for t <= 8, 2 for t <= 16)
__global__ void __launch_bounds__(gv::kThreads, 1)
    nf4_gemv_kernel(const GemvArgs args, const __grid_constant__ CUtensorMap map_codes) {
  using namespace gv;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ uint32_t abort_flag;
  uint32_t dyn_bytes;
  asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn_bytes));
  const uint32_t sbase = smem_addr(smem);
  const uint32_t tab = (sbase + 65535u) & ~65535u;
  const uint32_t first = (sbase + 127u) & ~127u;
  const uint32_t before = tab > first ? (tab - first) / kSlotBytes : 0u;  // slots before the table

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, q = lane & 3;
  auto slot_of = [&](uint32_t w) {
    return w < before ? first + w * kSlotBytes : tab + kTableBytes + (w - before) * kSlotBytes;
  };
  const uint32_t slot = slot_of(static_cast<uint32_t>(warp));
  // the last warp's slot ends last; the test is the same in every thread of the CTA
  if (sbase + slots_end() + kSTBytes > sbase + dyn_bytes || slot_of(kWarps - 1) + kSlotBytes > sbase + slots_end() ||
      tab + kTableBytes > sbase + slots_end()) {
    if (threadIdx.x == 0) report(kDevLaunch);  // launched with too little shared memory
    return;
  }
  float2* table = reinterpret_cast<float2*>(smem + (tab - sbase));  // [256 byte values][32 lanes]
  uint16_t* sts = reinterpret_cast<uint16_t*>(smem + slots_end());   // [token][kMaxRank]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (slot - sbase) + kSlotBars);

  const int64_t nblk = args.h / kBlock;
  const int64_t upt = (nblk + 1) >> 1;  // units per row tile (the last may hold one block)
  const int64_t units = (args.o / kTileRows) * upt;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * kWarps;
  const int64_t wid = static_cast<int64_t>(blockIdx.x) * kWarps + warp;
  const int64_t f_begin = units * wid / nwarps, f_end = units * (wid + 1) / nwarps;
  const int64_t nrun = f_end - f_begin;

  // codes: lane 0 fills the ring with the run's first kDepth units
  int64_t p_tile = f_begin / upt, p_u = f_begin - p_tile * upt;  // next unit to request
  if (lane == 0 && nrun > 0) {
    for (int i = 0; i < kDepth; ++i) mbar_init(&bars[i], 1);
    fence_mbar_init();
    tma_prefetch_desc(&map_codes);
    for (int i = 0; i < kDepth && i < nrun; ++i) {
      mbar_arrive_expect_tx(&bars[i], kUnitBytes);
      tma_load_2d(smem + (slot - sbase) + kSlotCodes + i * kUnitBytes, &map_codes, &bars[i],
                  static_cast<int32_t>(p_u * 64), static_cast<int32_t>(p_tile * kTileRows));
      if (++p_u == upt) { p_u = 0; ++p_tile; }
    }
  }
  // scale segments: the first two go in flight
  const uint32_t seg_base = slot + kSlotSeg;
  GemvSeg cur = gemv_seg_at(f_begin, f_end, upt);
  GemvSeg nxt = gemv_seg_at(cur.tile * upt + cur.u1, f_end, upt);
  gemv_stage_q8(seg_base, args, cur, nblk, lane);
  cp_async_commit();
  gemv_stage_q8(seg_base + kSegBytes, args, nxt, nblk, lane);
  cp_async_commit();

  uint4 xc[NT][4], xn[NT][4];
  if (NT == 1 && kXAhead && nrun > 0) gemv_load_x<NT>(xc, args, cur.u0, g, q, 2 * cur.u0 + (q >> 1) < nblk);

  if (threadIdx.x == 0) abort_flag = 0u;
  for (int i = threadIdx.x; i < 256 * 32; i += kThreads) {
    const int e = i >> 5;
    table[i] = make_float2(args.tab.level[e >> 4], args.tab.level[e & 15]);
  }
  // sT = bf16(s . X.L1) from the LoRA-down kernel's partial sums (launched just before this
  // kernel, which may start early: wait for its completion and memory first)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  for (int i = threadIdx.x; i < args.t * args.r; i += kThreads) {
    float v = 0.f;
#pragma unroll
    for (int p = 0; p < kDownParts; ++p) v += __ldcg(args.Tpart + p * args.t * args.r + i);
    const uint16_t b = __bfloat16_as_ushort(__float2bfloat16_rn(args.s * v));
    sts[(i / args.r) * kMaxRank + i % args.r] = b;
    if (blockIdx.x == 0 && args.sT_out) args.sT_out[i] = b;
  }
  __syncthreads();
  if (nrun <= 0) return;

  const uint32_t lane_slot = tab + static_cast<uint32_t>(lane) * 8u;
  float acc[2][NT][4];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[mt][nt][i] = 0.f;

  int cb = 0;
  int tile_units = 0;  // units of the current row tile done by this warp
  int i = 0;        // position in the run
  int e = 0;        // its ring entry, i % kDepth
  uint32_t ph = 0;  // the entry's fill parity, (i / kDepth) & 1
  cp_async_wait_prev();
  __syncwarp();
  while (true) {
    // byte offset of block 2 u0 of each of this lane's rows within the staged segment
    const uint32_t qs = seg_base + cb * kSegBytes;
    int qoff[2][2];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int rr = 0; rr < 2; ++rr) {
        const int r = mt * 16 + rr * 8 + g;
        const int64_t rb = (cur.tile * kTileRows + r) * nblk + 2 * static_cast<int64_t>(cur.u0);
        qoff[mt][rr] = r * kSegRowBytes + static_cast<int>(rb & 3) - 2 * cur.u0;
      }
    const int64_t row0 = cur.tile * kTileRows;
    for (int u = cur.u0; u < cur.u1; ++u) {
      if (!mbar_wait(&bars[e], ph, &abort_flag)) return;
      GemvCodes cc;
      gemv_read_codes(cc, slot + kSlotCodes + e * kUnitBytes, g, q);
      __syncwarp();  // every lane has read the entry before it is refilled
      if (lane == 0 && i + kDepth < nrun) {
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(&bars[e], kUnitBytes);
        tma_load_2d(smem + (slot - sbase) + kSlotCodes + e * kUnitBytes, &map_codes, &bars[e],
                    static_cast<int32_t>(p_u * 64), static_cast<int32_t>(p_tile * kTileRows));
        if (++p_u == upt) { p_u = 0; ++p_tile; }
      }
      const int bl = 2 * u + (q >> 1);  // this lane's block within the row
      const bool bv = bl < nblk;
      if (NT == 1 && kXAhead) {
        // the next unit's activations (the next unit may open the next segment)
        const int nu = u + 1 < cur.u1 ? u + 1 : (nxt.u0 < nxt.u1 ? nxt.u0 : -1);
        if (nu >= 0) gemv_load_x<NT>(xn, args, nu, g, q, 2 * nu + (q >> 1) < nblk);
      } else {
        gemv_load_x<NT>(xc, args, u, g, q, bv);
      }
      uint64_t kk[2][2];
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
          float k = 0.f;
          if (bv) {
            const int64_t qi = (row0 + mt * 16 + rr * 8 + g) * nblk + bl;
            uint32_t q8;
            asm volatile("ld.shared.u8 %0, [%1];" : "=r"(q8) : "r"(qs + qoff[mt][rr] + bl));
            k = __fmul_rn(static_cast<float>(q8), __ldg(args.s2 + (qi >> 8)));
          }
          asm("mov.b64 %0, {%1, %1};" : "=l"(kk[mt][rr]) : "f"(k));
        }
      gemv_compute<NT>(cc, xc, kk, acc, lane_slot);
      ++i;
      if (++e == kDepth) {
        e = 0;
        ph ^= 1u;
      }
      if (NT == 1 && kXAhead) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int j = 0; j < 4; ++j) xc[nt][j] = xn[nt][j];
      }
    }
    tile_units += cur.u1 - cur.u0;
    if (nxt.u0 == nxt.u1 || nxt.tile != cur.tile) {
      // add the tile's sums, then count its units; the warp that completes the tile
      // finishes it (the fence makes this warp's sums visible before its count)
      gemv_flush<NT>(acc, args, cur.tile, g, q);
      __threadfence();
      __syncwarp();
      unsigned before_me = 0;
      if (lane == 0) before_me = atomicAdd(args.tile_cnt + cur.tile, static_cast<unsigned>(tile_units));
      before_me = __shfl_sync(0xffffffffu, before_me, 0);
      if (before_me + tile_units == upt) {
        __threadfence();
        gemv_finish_tile<NT>(args, sts, cur.tile, lane);
      }
      tile_units = 0;
    }
    if (nxt.u0 == nxt.u1) break;
    // move to the next segment; its buffer's copies were issued one segment ago
    cur = nxt;
    cb ^= 1;
    nxt = gemv_seg_at(cur.tile * upt + cur.u1, f_end, upt);
    __syncwarp();  // every lane is done reading the buffer about to be refilled
    gemv_stage_q8(seg_base + (cb ^ 1) * kSegBytes, args, nxt, nblk, lane);
    cp_async_commit();
    cp_async_wait_prev();
    __syncwarp();
  }
}

// T = X.L1 for the decode path (t <= 16) as partial sums: 8 clusters of 8 CTAs; CTA q of
// cluster p sums its share of the inputs k into an fp32 t x r partial in shared memory (thread
// = column pair x a stride of k, four rows in flight), and the cluster's CTA 0 adds its eight
// CTAs' partials over distributed shared memory and writes partial p. The GEMV adds the 8
// partials, scales by s and rounds once to bf16 (the tensor-core path's sT up to summation
// order). The grid also zeroes the GEMV's fp32 output sums and tile counters.
namespace gd {
constexpr int kClusterCtas = 8;
constexpr int kClusters = gv::kDownParts;
constexpr int kCtas = kClusterCtas * kClusters;
constexpr int kThreads = 256;
constexpr size_t smem_bytes(int t, int r) {
  return (static_cast<size_t>(2 * kThreads) * t + static_cast<size_t>(t) * r) * 4;
}
}  // namespace gd

__global__ void __cluster_dims__(gd::kClusterCtas, 1, 1) __launch_bounds__(gd::kThreads)
    gemv_lora_down_kernel(const uint16_t* __restrict__ X, const uint16_t* __restrict__ L1,
                          float* Tpart, float* Y32, unsigned* tile_cnt, int64_t h, int64_t o,
                          int t, int r) {
  extern __shared__ __align__(16) float dsm[];
  const int tid = threadIdx.x;
  const uint32_t rank = cluster_ctarank();
  const int cluster = blockIdx.x / gd::kClusterCtas;
  // the GEMV launched after this kernel may be scheduled now (it waits for this grid's
  // completion before reading anything written here)
  asm volatile("griddepcontrol.launch_dependents;");

  // zero the GEMV's accumulators (t x o floats, o / 32 counters)
  {
    const int64_t gt = static_cast<int64_t>(blockIdx.x) * gd::kThreads + tid;
    const int64_t gn = static_cast<int64_t>(gd::kCtas) * gd::kThreads;
    float4* y4 = reinterpret_cast<float4*>(Y32);
    for (int64_t i = gt; i < static_cast<int64_t>(t) * o / 4; i += gn) y4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int64_t i = gt; i < o / 32; i += gn) tile_cnt[i] = 0u;
  }

  const int ncp = r / 2;                // column pairs
  const int nkg = gd::kThreads / ncp;   // k strides (r <= 256, r % 16 == 0: exact)
  const int cp = tid % ncp, kg = tid / ncp;
  // this CTA's inputs: an even share of the 2-row pairs
  const int64_t pairs = h / 2;
  const int64_t p0 = pairs * blockIdx.x / gd::kCtas, p1 = pairs * (blockIdx.x + 1) / gd::kCtas;
  float acc[16][2];
#pragma unroll
  for (int n = 0; n < 16; ++n) acc[n][0] = acc[n][1] = 0.f;
  for (int64_t pb = p0 + kg; pb < p1; pb += 4 * nkg) {
    uint32_t la[4], lb[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t pr = pb + u * nkg;
      const int64_t k = 2 * (pr < p1 ? pr : p0);
      la[u] = __ldg(reinterpret_cast<const uint32_t*>(L1 + k * r) + cp);
      lb[u] = __ldg(reinterpret_cast<const uint32_t*>(L1 + (k + 1) * r) + cp);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t pr = pb + u * nkg;
      if (pr >= p1) break;
      const int64_t k = 2 * pr;
      const float a0 = bf16_bits_to_float(la[u] & 0xffffu), a1 = bf16_bits_to_float(la[u] >> 16);
      const float b0 = bf16_bits_to_float(lb[u] & 0xffffu), b1 = bf16_bits_to_float(lb[u] >> 16);
#pragma unroll
      for (int n = 0; n < 16; ++n) {
        if (n < t) {
          const uint32_t xv = __ldg(reinterpret_cast<const uint32_t*>(X + static_cast<int64_t>(n) * h + k));
          const float x0 = bf16_bits_to_float(xv & 0xffffu), x1 = bf16_bits_to_float(xv >> 16);
          acc[n][0] = fmaf(x1, b0, fmaf(x0, a0, acc[n][0]));
          acc[n][1] = fmaf(x1, b1, fmaf(x0, a1, acc[n][1]));
        }
      }
    }
  }
  // [kg][n][c] partials -> this CTA's t x r sums
  float* red = dsm;
  float* part = dsm + static_cast<size_t>(2 * gd::kThreads) * t;
#pragma unroll
  for (int n = 0; n < 16; ++n)
    if (n < t) {
      red[(kg * t + n) * r + 2 * cp] = acc[n][0];
      red[(kg * t + n) * r + 2 * cp + 1] = acc[n][1];
    }
  __syncthreads();
  for (int i = tid; i < t * r; i += gd::kThreads) {
    float v = 0.f;
    for (int j = 0; j < nkg; ++j) v += red[j * t * r + i];
    part[i] = v;
  }
  cluster_sync();
  if (rank == 0) {
    for (int i = tid; i < t * r; i += gd::kThreads) {
      float v = 0.f;
#pragma unroll
      for (uint32_t q = 0; q < gd::kClusterCtas; ++q) v += ld_dsmem_f32(part + i, q);
      Tpart[static_cast<int64_t>(cluster) * t * r + i] = v;
    }
  }
  cluster_sync();  // the partials stay in place until the cluster's CTA 0 has read them
}

}  // namespace qlora
