// LoRA dropout on the adapter input ("QLoRA in LLMs" section 12, "Minimal QLoRA Setup with
// Hugging Face": the example configuration trains with a LoRA dropout of 0.05). Read as
// inverted dropout on the input of the adapter branch only:
//   Y = X.W' + s.((X (.) M / (1 - p)).L1).L2,
// M a keep mask drawn from a counter-based generator, so that the forward, the backward and
// any other pass over the same (seed, element) draw the same bit without storing a mask.
//
// Generator: Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As Easy as
// 1, 2, 3", SC'11). Element e = i*h + j of the t x h input takes word e mod 4 of the generator
// at counter (lo32(e / 4), hi32(e / 4), 0, 0) under key (lo32(seed), hi32(seed)); it is kept
// when that word is >= thr = floor(p * 2^32).
#pragma once

#include <cstdint>

namespace qlora {

struct DropoutKey {
  uint32_t k0, k1;  // the seed's low and high halves
  uint32_t thr;     // drop when the draw is below this (0: keep everything)
};

// The ten round keys of one seed: round r uses (k0 + r W0, k1 + r W1) mod 2^32, the Weyl
// increments added between rounds. Computed once per thread, not once per generator call.
struct PhiloxRoundKeys {
  uint32_t k0[10], k1[10];
};

__device__ __forceinline__ PhiloxRoundKeys philox_round_keys(const DropoutKey& key) {
  constexpr uint32_t kW0 = 0x9E3779B9u, kW1 = 0xBB67AE85u;
  PhiloxRoundKeys rk;
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    rk.k0[r] = key.k0 + static_cast<uint32_t>(r) * kW0;
    rk.k1[r] = key.k1 + static_cast<uint32_t>(r) * kW1;
  }
  return rk;
}

// Ten rounds: two 32x32 -> 64-bit products of counter words with fixed odd multipliers; the
// high halves are XORed with the other two counter words and the round key.
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, const PhiloxRoundKeys& rk) {
  constexpr uint32_t kM0 = 0xD2511F53u, kM1 = 0xCD9E8D57u;
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint64_t p0 = static_cast<uint64_t>(kM0) * c.x;
    const uint64_t p1 = static_cast<uint64_t>(kM1) * c.z;
    c = make_uint4(static_cast<uint32_t>(p1 >> 32) ^ c.y ^ rk.k0[r], static_cast<uint32_t>(p1),
                   static_cast<uint32_t>(p0 >> 32) ^ c.w ^ rk.k1[r], static_cast<uint32_t>(p0));
  }
  return c;
}

// Keep bits of elements 4g .. 4g+3: bit k is element 4g + k.
__device__ __forceinline__ uint32_t dropout_keep4(uint64_t g, const PhiloxRoundKeys& rk,
                                                  uint32_t thr) {
  const uint4 w = philox4x32_10(
      make_uint4(static_cast<uint32_t>(g), static_cast<uint32_t>(g >> 32), 0u, 0u), rk);
  return static_cast<uint32_t>(w.x >= thr) | (static_cast<uint32_t>(w.y >= thr) << 1) |
         (static_cast<uint32_t>(w.z >= thr) << 2) | (static_cast<uint32_t>(w.w >= thr) << 3);
}

// A 32-bit word holding bf16 elements 2k (low half) and 2k + 1 (high half): keep bits k2, k2+1
// of `keep` select which halves survive.
__device__ __forceinline__ uint32_t keep_halves(uint32_t keep, int k2) {
  return ((keep >> k2) & 1u ? 0x0000FFFFu : 0u) | ((keep >> (k2 + 1)) & 1u ? 0xFFFF0000u : 0u);
}

// Xd = X (.) M over n8 groups of 8 bf16 (n = 8 n8 elements, row-major t x h, so the element
// index is the flat index). The keep bits of group i (bit k = element 8i + k) are either drawn
// (two generator calls per group) and, when `bits` is given, stored as byte i; or, with
// kFromBits, read from byte i of `bits` (a mask an earlier pass drew). Dropped elements become
// +0. Grid-stride with four groups per thread in flight (their loads issued before any
// generator call), so that enough bytes are in flight to cover the memory latency.
constexpr int kDropUnroll = 4;

// X and Xd may be the same buffer: each 16-byte group is read and written by one thread.
template <bool kFromBits>
__global__ void __launch_bounds__(256) dropout_apply_kernel(const uint4* X, uint4* Xd,
                                                            uint8_t* __restrict__ bits,
                                                            int64_t n8, DropoutKey key) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const PhiloxRoundKeys rk = philox_round_keys(key);
  for (int64_t base = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; base < n8;
       base += kDropUnroll * stride) {
    uint4 x[kDropUnroll];
    uint32_t kb[kDropUnroll];
#pragma unroll
    for (int u = 0; u < kDropUnroll; ++u) {
      const int64_t i = base + u * stride;
      if (i < n8) {
        x[u] = X[i];
        if (kFromBits) kb[u] = bits[i];
      }
    }
#pragma unroll
    for (int u = 0; u < kDropUnroll; ++u) {
      const int64_t i = base + u * stride;
      if (i >= n8) continue;
      uint32_t keep;
      if (kFromBits) {
        keep = kb[u];
      } else {
        keep = dropout_keep4(2 * static_cast<uint64_t>(i), rk, key.thr) |
               (dropout_keep4(2 * static_cast<uint64_t>(i) + 1, rk, key.thr) << 4);
        if (bits) bits[i] = static_cast<uint8_t>(keep);
      }
      uint4 v = x[u];
      v.x &= keep_halves(keep, 0);
      v.y &= keep_halves(keep, 2);
      v.z &= keep_halves(keep, 4);
      v.w &= keep_halves(keep, 6);
      Xd[i] = v;
    }
  }
}

}  // namespace qlora
