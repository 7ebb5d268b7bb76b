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

// Ten rounds: two 32x32 -> 64-bit products of counter words with fixed odd multipliers; the
// high halves are XORed with the other two counter words and the key; the key advances by two
// Weyl increments between rounds.
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
  constexpr uint32_t kM0 = 0xD2511F53u, kM1 = 0xCD9E8D57u;
  constexpr uint32_t kW0 = 0x9E3779B9u, kW1 = 0xBB67AE85u;
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r > 0) {
      k0 += kW0;
      k1 += kW1;
    }
    const uint32_t lo0 = kM0 * c.x, hi0 = __umulhi(kM0, c.x);
    const uint32_t lo1 = kM1 * c.z, hi1 = __umulhi(kM1, c.z);
    c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
  }
  return c;
}

struct DropoutKey {
  uint32_t k0, k1;  // the seed's low and high halves
  uint32_t thr;     // drop when the draw is below this (0: keep everything)
};

// Keep bits of elements 4g .. 4g+3: bit k is element 4g + k.
__device__ __forceinline__ uint32_t dropout_keep4(uint64_t g, const DropoutKey& key) {
  const uint4 w = philox4x32_10(
      make_uint4(static_cast<uint32_t>(g), static_cast<uint32_t>(g >> 32), 0u, 0u), key.k0, key.k1);
  return static_cast<uint32_t>(w.x >= key.thr) | (static_cast<uint32_t>(w.y >= key.thr) << 1) |
         (static_cast<uint32_t>(w.z >= key.thr) << 2) | (static_cast<uint32_t>(w.w >= key.thr) << 3);
}

// A 32-bit word holding bf16 elements 2k (low half) and 2k + 1 (high half): keep bits k2, k2+1
// of `keep` select which halves survive.
__device__ __forceinline__ uint32_t keep_halves(uint32_t keep, int k2) {
  return ((keep >> k2) & 1u ? 0x0000FFFFu : 0u) | ((keep >> (k2 + 1)) & 1u ? 0xFFFF0000u : 0u);
}

// Xd = X (.) M over n8 groups of 8 bf16 (n = 8 n8 elements, row-major t x h, so the element
// index is the flat index): one 16-byte load, two generator calls, one 16-byte store per group,
// and, when `bits` is given, the group's 8 keep bits as one byte (bit k = element 8i + k).
// Dropped elements become +0. Grid-stride with four groups per thread in flight (their loads
// issued before any generator call), so that enough bytes are in flight to cover the memory
// latency; the kernel is bound by HBM (2 + 2 bytes/element, + 1/8 for the bits).
constexpr int kDropUnroll = 4;

__device__ __forceinline__ uint4 dropout_group(uint4 x, int64_t i, const DropoutKey& key,
                                               uint8_t* bits) {
  const uint32_t keep = dropout_keep4(2 * static_cast<uint64_t>(i), key) |
                        (dropout_keep4(2 * static_cast<uint64_t>(i) + 1, key) << 4);
  x.x &= keep_halves(keep, 0);
  x.y &= keep_halves(keep, 2);
  x.z &= keep_halves(keep, 4);
  x.w &= keep_halves(keep, 6);
  if (bits) bits[i] = static_cast<uint8_t>(keep);
  return x;
}

__global__ void __launch_bounds__(256) dropout_apply_kernel(const uint4* __restrict__ X,
                                                            uint4* __restrict__ Xd,
                                                            uint8_t* __restrict__ bits,
                                                            int64_t n8, DropoutKey key) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t base = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; base < n8;
       base += kDropUnroll * stride) {
    uint4 x[kDropUnroll];
#pragma unroll
    for (int u = 0; u < kDropUnroll; ++u) {
      const int64_t i = base + u * stride;
      if (i < n8) x[u] = X[i];
    }
#pragma unroll
    for (int u = 0; u < kDropUnroll; ++u) {
      const int64_t i = base + u * stride;
      if (i < n8) Xd[i] = dropout_group(x[u], i, key, bits);
    }
  }
}

}  // namespace qlora
