// Adapter update: one fused AdamW step over an fp32 parameter vector ("QLoRA in LLMs" section 4
// "Update the adapters": the base stays fixed, the adapters change; section 7 and "Idea three:
// paged optimizers", goodomens.studio: the optimizer state may live in unified memory and move
// between CPU and GPU memory). The pages name the state ("running statistics") but not the
// rule; the rule here is AdamW with decoupled weight decay and bias-corrected moments:
//   p <- p (1 - lr wd);  m <- b1 m + (1 - b1) g;  v <- b2 v + (1 - b2) g^2;
//   p <- p - (lr / (1 - b1^t)) m / (sqrt(v) / sqrt(1 - b2^t) + eps)
// and the bf16 copy of p the next forward reads. HBM-bound: 16 B read + 12 B written (+2 B
// bf16) per parameter; four parameters per thread and item, grid-stride over items.
#pragma once

#include "qlora_common.cuh"

namespace qlora {

struct AdamwArgs {
  float* p;
  uint16_t* p16;  // may be null
  const float* g;
  float* m;
  float* v;
  int64_t n4;     // parameters / 4
  float lr, beta1, beta2, eps, wd;
  float step_size;   // lr / (1 - b1^t)
  float inv_sqrt_bc2;  // 1 / sqrt(1 - b2^t)
};

struct AdamwHyper {
  float lr, beta1, beta2, eps, wd;
  float step_size;     // lr / (1 - b1^t)
  float inv_sqrt_bc2;  // 1 / sqrt(1 - b2^t)
};

// One item: four parameters of one tensor.
__device__ __forceinline__ void adamw_item(float* P, uint16_t* P16, const float* G, float* M,
                                           float* V, int64_t i, const AdamwHyper& a) {
  float4 p = reinterpret_cast<const float4*>(P)[i];
  const float4 g = __ldcs(reinterpret_cast<const float4*>(G) + i);
  float4 m = reinterpret_cast<const float4*>(M)[i];
  float4 v = reinterpret_cast<const float4*>(V)[i];
  float* pp = &p.x;
  const float* gg = &g.x;
  float* mm = &m.x;
  float* vv = &v.x;
  const float decay = 1.0f - a.lr * a.wd;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    mm[e] = fmaf(a.beta1, mm[e], (1.0f - a.beta1) * gg[e]);
    vv[e] = fmaf(a.beta2, vv[e], (1.0f - a.beta2) * gg[e] * gg[e]);
    const float denom = sqrtf(vv[e]) * a.inv_sqrt_bc2 + a.eps;
    pp[e] = pp[e] * decay - a.step_size * mm[e] / denom;
  }
  reinterpret_cast<float4*>(P)[i] = p;
  reinterpret_cast<float4*>(M)[i] = m;
  reinterpret_cast<float4*>(V)[i] = v;
  if (P16) reinterpret_cast<uint2*>(P16)[i] = make_uint2(pack_bf16x2(p.x, p.y), pack_bf16x2(p.z, p.w));
}

__device__ __forceinline__ AdamwHyper adamw_hyper(const AdamwArgs& a) {
  return AdamwHyper{a.lr, a.beta1, a.beta2, a.eps, a.wd, a.step_size, a.inv_sqrt_bc2};
}

__global__ void __launch_bounds__(256) adamw_kernel(const AdamwArgs a) {
  const AdamwHyper hy = adamw_hyper(a);
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < a.n4; i += stride)
    adamw_item(a.p, a.p16, a.g, a.m, a.v, i, hy);
}

// Several tensors (the adapters of a model) in one launch: the items of all tensors form one
// list, tensor k owning items [first4[k], first4[k + 1]); a thread finds an item's tensor by
// binary search. Per parameter the arithmetic is adamw_kernel's, so results are identical.
constexpr int kAdamwMaxTensors = 64;

struct AdamwMultiArgs {
  float* p[kAdamwMaxTensors];
  uint16_t* p16[kAdamwMaxTensors];
  const float* g[kAdamwMaxTensors];
  float* m[kAdamwMaxTensors];
  float* v[kAdamwMaxTensors];
  int64_t first4[kAdamwMaxTensors + 1];
  int ntensors;
  AdamwHyper hy;
};

__global__ void __launch_bounds__(256) adamw_multi_kernel(const __grid_constant__ AdamwMultiArgs a) {
  const int64_t total = a.first4[a.ntensors];
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride) {
    int lo = 0, hi = a.ntensors - 1;  // the last k with first4[k] <= i
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (a.first4[mid] <= i) lo = mid; else hi = mid - 1;
    }
    adamw_item(a.p[lo], a.p16[lo], a.g[lo], a.m[lo], a.v[lo], i - a.first4[lo], a.hy);
  }
}

}  // namespace qlora
