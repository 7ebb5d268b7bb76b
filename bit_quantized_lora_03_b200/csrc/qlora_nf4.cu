// libqlora_nf4: host implementation of the C ABI declared in include/qlora_nf4.h.
//
// Validates every argument on the host before any CUDA call, derives the NF4 codebook, builds
// TMA tensor maps (cuTensorMapEncodeTiled through the runtime's driver entry point, so the
// library does not link libcuda), and launches the hand-written sm_100a kernels of csrc/ on
// the caller's stream. It never allocates device memory: scratch comes from the caller.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include "qlora_nf4.h"

#include "nf4_codec.cuh"
#include "nf4_gemm.cuh"
#include "tc_gemm.cuh"
#include "adamw.cuh"
#include "dropout.cuh"
#include "nf4_gemv.cuh"

using namespace qlora;

namespace {

constexpr int kMergeCtasPerSm = 4;   // the adapter merge's CTAs per SM (one register bound)
std::atomic<int> g_gemv_max_ctas{0};  // cap on the decode GEMV's CTAs (0 = one per SM)

// ------------------------------------------------------------------------------------------
// NF4 codebook ("QLoRA in LLMs" section 5; "Idea one: NF4" on goodomens.studio; "Key
// Components" on docs.skillversehub.com): 16 levels at standard-normal quantiles, an exact
// zero, ends normalised to -1 and +1. Eight positive levels at probabilities evenly spaced
// from delta towards 1/2 (1/2 itself excluded), seven negative ones likewise, plus zero, all
// divided by the largest; delta = ((1 - 1/30) + (1 - 1/32)) / 2. Computed here in double
// with a safeguarded Newton iteration on Phi(x) = p and rounded once to fp32.
// ------------------------------------------------------------------------------------------
double normal_cdf(double x) { return 0.5 * std::erfc(-x / std::sqrt(2.0)); }

double normal_pdf(double x) { return std::exp(-0.5 * x * x) / std::sqrt(2.0 * 3.14159265358979323846); }

double normal_quantile(double p) {
  double lo = -40.0, hi = 40.0, x = 0.0;
  for (int it = 0; it < 500; ++it) {
    const double f = normal_cdf(x) - p;
    if (f < 0.0) lo = x; else hi = x;
    const double d = normal_pdf(x);
    double xn = d > 0.0 ? x - f / d : 0.5 * (lo + hi);
    if (!(xn > lo && xn < hi)) xn = 0.5 * (lo + hi);
    if (xn == x) break;
    x = xn;
  }
  return x;
}

struct Codebook {
  float level[16];
  float mid[15];
  int zero_code;  // the code of the zero level (all-zero blocks)
};

Codebook finish(const double (&v)[16], int zero_code) {
  Codebook c{};
  for (int i = 0; i < 16; ++i) c.level[i] = static_cast<float>(v[i]);
  for (int i = 0; i < 15; ++i)
    c.mid[i] = static_cast<float>((static_cast<double>(c.level[i]) +
                                   static_cast<double>(c.level[i + 1])) / 2.0);
  c.zero_code = zero_code;
  return c;
}

// Codebook ids: 0 NF4 (above); 1 FP4 E2M1, magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6} with both
// signs over 6 (both zeros kept); 2 absmax INT4, k / 7 for k = -8 .. 7 (the textbook absmax
// integer scheme, "QLoRA in LLMs" section 2). Same blocks, packing and scales; the pages set
// NF4 against these two ("QLoRA in LLMs" section 5; "Idea one: NF4", goodomens.studio).
constexpr int kCodebooks = 3;

const Codebook& codebook(int id = 0) {
  static const Codebook cbs[kCodebooks] = {
      [] {
        const double delta = 0.5 * ((1.0 - 1.0 / 30.0) + (1.0 - 1.0 / 32.0));
        std::vector<double> v;
        for (int i = 0; i < 8; ++i) v.push_back(normal_quantile(delta + i * (0.5 - delta) / 8.0));
        for (int i = 0; i < 7; ++i) v.push_back(-normal_quantile(delta + i * (0.5 - delta) / 7.0));
        v.push_back(0.0);
        std::sort(v.begin(), v.end());
        const double top = normal_quantile(delta);
        double w[16];
        for (int i = 0; i < 16; ++i) w[i] = v[i] / top;
        return finish(w, 7);
      }(),
      [] {
        const double mags[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
        double w[16];
        for (int i = 0; i < 8; ++i) {
          w[i] = -mags[7 - i] / 6.0;  // -1 ... -0
          w[8 + i] = mags[i] / 6.0;   // +0 ... +1
        }
        return finish(w, 7);
      }(),
      [] {
        double w[16];
        for (int k = -8; k < 8; ++k) w[k + 8] = k / 7.0;
        return finish(w, 8);
      }()};
  return cbs[id];
}

Nf4Table device_table(int id = 0) {
  Nf4Table t{};
  const Codebook& cb = codebook(id);
  for (int i = 0; i < 16; ++i) t.level[i] = cb.level[i];
  for (int i = 0; i < 15; ++i) t.mid[i] = cb.mid[i];
  t.mid[15] = 2.0f;
  t.zero_code = cb.zero_code;
  return t;
}

// Buckets of the quantizer's fast decision (see nf4_code_fast): bucket b covers
// [-1 + b/64, -1 + (b+1)/64); fp32 arithmetic on these edges is exact.
Nf4Buckets device_buckets(int id = 0) {
  Nf4Buckets bk{};
  const Codebook& cb = codebook(id);
  int bad = 0;
  for (int b = 0; b < 128; ++b) {
    const float lo = -1.0f + static_cast<float>(b) / 64.0f, hi = lo + 1.0f / 64.0f;
    int n = 0;
    while (n < 15 && cb.mid[n] < lo) ++n;
    bk.lo[b] = static_cast<float>(n);
    bk.thr[b] = (n < 15 && cb.mid[n] < hi) ? cb.mid[n] : 4.0f;
    if (n + 1 < 15 && cb.mid[n + 1] < hi) bad = 1;  // two thresholds in one bucket
  }
  for (int i = 0; i < 15; ++i) {  // no threshold within 2^-18 of a bucket edge
    const double u = (static_cast<double>(cb.mid[i]) + 1.0) * 64.0;
    if (std::fabs(u - std::nearbyint(u)) / 64.0 < std::ldexp(1.0, -18)) bad = 1;
  }
  bk.exact_only = bad;
  return bk;
}

// ------------------------------------------------------------------------------------------
// device checks, kernel attributes
// ------------------------------------------------------------------------------------------
constexpr int kMaxDevices = 64;

struct DeviceInfo {
  std::once_flag once;
  int ok = 0;        // 1 = sm_100 device ready
  int sms = 148;
  // CTAs per SM that fit at once (occupancy calculator) for grid-stride kernels whose grids are
  // one wave of these: a CTA that could only start after others finished would leave SMs idle
  int dq_ctas = 1;           // nf4_dequantize_kernel
  int adamw_ctas = 1;        // adamw_kernel, 256 threads
  int adamw_multi_ctas = 1;  // adamw_multi_kernel, 256 threads
};
DeviceInfo g_dev[kMaxDevices];

int current_device(int* dev_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return QLORA_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return QLORA_ERR_UNSUPPORTED_DEVICE;
  DeviceInfo& d = g_dev[dev];
  std::call_once(d.once, [&] {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      d.ok = -1;
      return;
    }
    if (major != 10 || minor != 0) {
      d.ok = -2;
      return;
    }
    d.sms = sms;
    bool fine = true;
    fine &= cudaFuncSetAttribute(nf4_gemm_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(tc::nf4_gemm_smem_bytes())) == cudaSuccess;
    fine &= cudaFuncSetAttribute(nf4_gemm_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(tc::nf4_gemm_smem_bytes())) == cudaSuccess;
    fine &= cudaFuncSetAttribute(nf4_quantize_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(qz::smem_bytes())) == cudaSuccess;
    fine &= cudaFuncSetAttribute(gemv_lora_down_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(gd::smem_bytes(16, 256))) == cudaSuccess;
    fine &= cudaFuncSetAttribute(nf4_gemv_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(gv::smem_bytes())) == cudaSuccess;
    fine &= cudaFuncSetAttribute(nf4_gemv_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(gv::smem_bytes())) == cudaSuccess;
    fine &= cudaFuncSetAttribute(tc_gemm_kernel<true, false>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 tcg::kMaxSmem) == cudaSuccess;
    fine &= cudaFuncSetAttribute(tc_gemm_kernel<false, false>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 tcg::kMaxSmem) == cudaSuccess;
    fine &= cudaFuncSetAttribute(tc_gemm_kernel<false, true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 tcg::kMaxSmem) == cudaSuccess;
    fine &= cudaFuncSetAttribute(tc_gemm_kernel<true, true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 tcg::kMaxSmem) == cudaSuccess;
    fine &= cudaFuncSetAttribute(tc_gemm_kernel<true, false, kMergeCtasPerSm>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 tcg::kMaxSmem) == cudaSuccess;
    int n = 0;
    fine &= cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, nf4_dequantize_kernel, dq::kThreads, 0) == cudaSuccess;
    d.dq_ctas = std::max(1, n);
    n = 0;
    fine &= cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, adamw_kernel, 256, 0) == cudaSuccess;
    d.adamw_ctas = std::max(1, n);
    n = 0;
    fine &= cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, adamw_multi_kernel, 256, 0) == cudaSuccess;
    d.adamw_multi_ctas = std::max(1, n);
    if (!fine) cudaGetLastError();
    d.ok = fine ? 1 : -1;
  });
  *dev_out = dev;
  if (d.ok == 1) return QLORA_OK;
  return d.ok == -2 ? QLORA_ERR_UNSUPPORTED_DEVICE : QLORA_ERR_CUDA;
}

int sm_count(int dev) { return g_dev[dev].sms; }
const DeviceInfo& device_info(int dev) { return g_dev[dev]; }

int launch_status() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

// ------------------------------------------------------------------------------------------
// kernel timing: CUDA events around each launch while a profile is open
// ------------------------------------------------------------------------------------------
namespace prof {
enum Kind {
  kQuant = 0, kDequant, kGemv, kGemvLoraDown, kTcGemm, kGemmFwd, kGemmBwd, kDropout, kKinds
};
const char* const kNames[kKinds] = {
    "nf4_quantize_kernel", "nf4_dequantize_kernel", "nf4_gemv_kernel",
    "gemv_lora_down_kernel", "tc_gemm_kernel",
    "nf4_gemm_kernel<fwd>", "nf4_gemm_kernel<bwd>", "dropout_apply_kernel"};
static_assert(kKinds == QLORA_KERNEL_KINDS, "kernel kinds");

struct State {
  std::mutex mu;
  std::atomic<bool> on{false};
  bool overflow = false;
  std::vector<cudaEvent_t> events;  // two per record
  std::vector<int> kinds;
  int capacity = 0;
  int n = 0;
};
State g;

// Records a start event now and a stop event when it goes out of scope (after the launch).
struct Scope {
  int idx = -1;
  cudaStream_t st;
  Scope(int kind, cudaStream_t s) : st(s) {
    if (!g.on.load(std::memory_order_relaxed)) return;
    std::lock_guard<std::mutex> lock(g.mu);
    if (!g.on.load()) return;
    if (g.n >= g.capacity) {
      g.overflow = true;
      return;
    }
    idx = g.n++;
    g.kinds[idx] = kind;
    cudaEventRecord(g.events[2 * idx], st);
  }
  ~Scope() {
    if (idx >= 0) cudaEventRecord(g.events[2 * idx + 1], st);
  }
};
}  // namespace prof

// ------------------------------------------------------------------------------------------
// TMA tensor maps
// ------------------------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess) {
      cudaGetLastError();
      return static_cast<EncodeTiledFn>(nullptr);
    }
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// 2-D map over a row-major matrix: `inner` contiguous elements per row, `outer` rows,
// `row_bytes` between rows; box = box_inner x box_outer elements.
bool make_map_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t inner,
                 uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                 bool swizzle128) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE,
                        swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool map_bf16(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint32_t box_cols,
              uint32_t box_rows) {
  return make_map_2d(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, cols, rows, cols * 2, box_cols,
                     box_rows, true);
}

// ------------------------------------------------------------------------------------------
// argument checks
// ------------------------------------------------------------------------------------------
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr int64_t kMaxDim = int64_t(1) << 31;

int check_weight(const nf4_weight* q) {
  if (!q || !q->codes || !q->absmax_q8 || !q->absmax_s2) return QLORA_ERR_INVALID_ARG;
  if (q->out_features < 1 || q->in_features < 64 || q->in_features % 64 != 0)
    return QLORA_ERR_BAD_SHAPE;
  if (q->out_features >= kMaxDim || q->in_features >= kMaxDim) return QLORA_ERR_BAD_SHAPE;
  const int64_t n = q->out_features * q->in_features;
  if (n / q->in_features != q->out_features || n > (int64_t(1) << 46)) return QLORA_ERR_BAD_SHAPE;
  if (!aligned16(q->codes) || !aligned16(q->absmax_q8) || !aligned16(q->absmax_s2))
    return QLORA_ERR_MISALIGNED;
  return QLORA_OK;
}

int check_linear_shape(int64_t t, int64_t h, int64_t o, int64_t r) {
  if (t < 1 || r < 16 || r > 256 || r % 16 != 0) return QLORA_ERR_INVALID_ARG;
  if (h < 64 || h % 64 != 0 || o < 64 || o % 64 != 0) return QLORA_ERR_BAD_SHAPE;
  if (t >= kMaxDim || h >= kMaxDim || o >= kMaxDim) return QLORA_ERR_BAD_SHAPE;
  return QLORA_OK;
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// workspace region of one rank-r down projection: t x r bf16 (sT or sU), 256-byte aligned
size_t lora_region_bytes(int64_t t, int64_t r) { return align256(static_cast<size_t>(t) * r * 2); }

// decode path (t <= 16): partial sums of X.L1 (gv::kDownParts x t x r fp32), the GEMV's fp32
// t x o sums, its o / 32 tile counters
struct GemvWs {
  float* Tpart;
  float* Y32;
  unsigned* cnt;
};
size_t gemv_ws_bytes(int64_t t, int64_t o, int64_t r) {
  return align256(static_cast<size_t>(gv::kDownParts) * t * r * 4) +
         align256(static_cast<size_t>(t) * o * 4) + align256(static_cast<size_t>(o / 32) * 4);
}
GemvWs carve_gemv(void* base, int64_t t, int64_t o, int64_t r) {
  uint8_t* b = reinterpret_cast<uint8_t*>(base);
  GemvWs w;
  w.Tpart = reinterpret_cast<float*>(b);
  b += align256(static_cast<size_t>(gv::kDownParts) * t * r * 4);
  w.Y32 = reinterpret_cast<float*>(b);
  b += align256(static_cast<size_t>(t) * o * 4);
  w.cnt = reinterpret_cast<unsigned*>(b);
  return w;
}

constexpr int64_t kGemvMaxTokens = 16;

// ------------------------------------------------------------------------------------------
// launch helpers
// ------------------------------------------------------------------------------------------
constexpr int kMaxTcSplits = 8;

struct TcPlan {
  int stages, splits, kb_per_split, num_kb, mtiles, BNp;
  size_t smem;
};

// These products stream one large operand (X or dY, read once from HBM) through a small
// accumulator. One wave of one CTA per SM, each with the deepest pipeline that fits (up to 8
// stages), keeps HBM busy; split-K only as far as needed to give every SM a CTA, so the fixed
// per-CTA costs (set-up, epilogue, the final rounding) are paid as few times as possible.
TcPlan plan_tc(int64_t M, int64_t ncols, int64_t K, bool b_mn, int sms) {
  TcPlan p{};
  p.BNp = static_cast<int>(std::min<int64_t>(256, (ncols + 15) / 16 * 16));  // N > 256: N tiles
  p.num_kb = static_cast<int>((K + 63) / 64);
  p.mtiles = static_cast<int>((M + 127) / 128);
  int stages = tcg::MAX_STAGES;
  while (stages > 2 && tcg::smem_bytes(stages, p.BNp, b_mn) > static_cast<size_t>(tcg::kMaxSmem))
    --stages;
  p.stages = stages;
  p.smem = tcg::smem_bytes(stages, p.BNp, b_mn);
  int splits = std::max(1, sms / p.mtiles);
  splits = std::min(splits, std::max(1, p.num_kb / 4));
  splits = std::min(splits, kMaxTcSplits);  // split-K is one cluster (portable size)
  // Between sms/2 and sms row tiles (e.g. 86 for an 11008-row output) one CTA per tile leaves
  // SMs idle: split K in two and halve the pipeline so that two CTAs fit on an SM.
  if (splits == 1 && p.mtiles < sms && p.num_kb >= 8) {
    int st2 = stages;
    while (st2 > 2 && 2 * tcg::smem_bytes(st2, p.BNp, b_mn) > static_cast<size_t>(tcg::kSmemPerSm)) --st2;
    if (2 * tcg::smem_bytes(st2, p.BNp, b_mn) <= static_cast<size_t>(tcg::kSmemPerSm)) {
      splits = 2;
      p.stages = st2;
      p.smem = tcg::smem_bytes(st2, p.BNp, b_mn);
    }
  }
#ifdef QLORA_TUNING
  if (const char* e = std::getenv("QLORA_TC_WAVE")) splits = std::max(1, (std::atoi(e) * sms) / p.mtiles);
  if (const char* e = std::getenv("QLORA_TC_MINKB")) splits = std::min(splits, std::max(1, p.num_kb / std::atoi(e)));
  if (const char* e = std::getenv("QLORA_TC_STAGES")) {
    p.stages = std::atoi(e);
    p.smem = tcg::smem_bytes(p.stages, p.BNp, b_mn);
  }
#endif
  // the split-K partial tile (128 rows of BNp + 4 floats) reuses the drained stage buffers
  if (static_cast<size_t>(tcg::BM) * (p.BNp + 4) * 4 >
      static_cast<size_t>(p.stages) * tcg::stage_bytes(p.BNp, b_mn))
    splits = 1;
  p.kb_per_split = (p.num_kb + splits - 1) / splits;
  p.splits = (p.num_kb + p.kb_per_split - 1) / p.kb_per_split;
  // no more stages than K-steps per CTA (a short K leaves room for more CTAs per SM)
  if (p.stages > std::max(2, p.kb_per_split)) {
    p.stages = std::max(2, p.kb_per_split);
    p.smem = tcg::smem_bytes(p.stages, p.BNp, b_mn);
  }
  return p;
}

template <bool A_MN, bool B_MN, int kMinCtas = 1>
int launch_tc_gemm(const CUtensorMap& mA, const CUtensorMap& mB, int64_t M, int64_t ncols,
                   const TcPlan& pl, float alpha, int mode, float* out32, int64_t ld,
                   uint16_t* o16a, uint16_t* o16b, int pdl, cudaStream_t st,
                   const nf4_weight* merge_w = nullptr, const uint8_t* keep_bits = nullptr,
                   const CUtensorMap* mOut = nullptr) {
  TcGemmArgs a{};
  a.M = static_cast<int>(M);
  a.Ncols = static_cast<int>(ncols);
  a.BNp = pl.BNp;
  a.num_kb = pl.num_kb;
  a.kb_per_split = pl.kb_per_split;
  a.splits = pl.splits;
  a.stages = pl.stages;
  a.alpha = alpha;
  a.out_mode = mode;
  a.out32 = out32;
  a.ld = ld;
  a.out16a = o16a;
  a.out16b = o16b;
  a.pdl = pdl;
  if (merge_w) {
    a.codes = merge_w->codes;
    a.q8 = merge_w->absmax_q8;
    a.s2 = merge_w->absmax_s2;
    a.tab = device_table();
  }
  a.keep_bits = keep_bits;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((ncols + pl.BNp - 1) / pl.BNp), static_cast<unsigned>(pl.mtiles),
                     static_cast<unsigned>(pl.splits));
  cfg.blockDim = dim3(tcg::kThreads, 1, 1);
  cfg.dynamicSmemBytes = pl.smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;  // the split-K CTAs of a tile: one cluster
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = static_cast<unsigned>(pl.splits);
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl == kPdlNone ? 1 : 2;
  cudaError_t e;
  {
    prof::Scope ps(prof::kTcGemm, st);
    // the output map is used by the merge epilogue only; the others get A's map as filler
    e = cudaLaunchKernelEx(&cfg, tc_gemm_kernel<A_MN, B_MN, kMinCtas>, mA, mB, mOut ? *mOut : mA, a);
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    return QLORA_ERR_CUDA;
  }
  return launch_status();
}

struct LoraWs {
  uint16_t* b16;  // t x r bf16
};

LoraWs carve_lora(void* base, int64_t, int64_t) {
  LoraWs w;
  w.b16 = reinterpret_cast<uint16_t*>(base);
  return w;
}

// The fused NF4 GEMM runs as clusters of 2 CTAs (cta_group::2): grid x = 2 CTAs per 256-column
// tile, grid y = 512-token row blocks.
template <bool kBwd>
int launch_nf4_gemm(const CUtensorMap& mA, const CUtensorMap& mP, const CUtensorMap& mA2,
                    const CUtensorMap& mB2, const Nf4GemmArgs& ga, int64_t t, int64_t ncols,
                    cudaStream_t st, int prof_kind) {
  // the output (t x ncols bf16) as 32-row x 64-column boxes for the epilogue's TMA stores
  CUtensorMap mOut;
  if (!map_bf16(&mOut, ga.out, static_cast<uint64_t>(ncols), static_cast<uint64_t>(t), 64, 32))
    return QLORA_ERR_CUDA;
  if ((t + tc::PAIR_M - 1) / tc::PAIR_M > 65535) return QLORA_ERR_BAD_SHAPE;  // grid y limit
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * ((ncols + tc::BN - 1) / tc::BN)),
                     static_cast<unsigned>((t + tc::PAIR_M - 1) / tc::PAIR_M), 1);
  cfg.blockDim = dim3(tc::kThreads, 1, 1);
  cfg.dynamicSmemBytes = tc::nf4_gemm_smem_bytes();
  cfg.stream = st;
  // always launched right after the kernel that produces its LoRA operand (sT or sU): it
  // may start early and waits for that kernel before its LoRA K-steps
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaError_t e;
  {
    prof::Scope ps(prof_kind, st);
    e = cudaLaunchKernelEx(&cfg, nf4_gemm_kernel<kBwd>, mA, mP, mA2, mB2, mOut, ga);
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    return QLORA_ERR_CUDA;
  }
  return launch_status();
}

// out16 = bf16(s . A.B) (and out16b if given) for a rank-r down projection: A is t x K
// (K-major), B given by its map (ncols = r). One launch; split-K CTAs of a tile form one
// cluster and reduce through distributed shared memory.
template <bool B_MN>
int lora_down(const CUtensorMap& mA, const CUtensorMap& mB, int64_t t, int64_t K, int64_t r,
              float s, uint16_t* out16, uint16_t* out16b, int sms, cudaStream_t st) {
  TcPlan pl = plan_tc(t, r, K, B_MN, sms);
#ifdef QLORA_TUNING
  if (const char* e = std::getenv("QLORA_RB_SPLITS")) {
    int sp = std::max(1, std::min({pl.num_kb, kMaxTcSplits, std::atoi(e)}));
    pl.kb_per_split = (pl.num_kb + sp - 1) / sp;
    pl.splits = (pl.num_kb + pl.kb_per_split - 1) / pl.kb_per_split;
  }
#endif
  return launch_tc_gemm<false, B_MN>(mA, mB, t, r, pl, s, kOutRoundBf16, nullptr, r, out16,
                                     out16b, kPdlNone, st);
}

// ------------------------------------------------------------------------------------------
// the adapted linear layer
// ------------------------------------------------------------------------------------------
// Dropout on the adapter input: key of the generator and the drop threshold floor(p * 2^32).
DropoutKey dropout_key(float p, uint64_t seed) {
  DropoutKey k{};
  k.k0 = static_cast<uint32_t>(seed);
  k.k1 = static_cast<uint32_t>(seed >> 32);
  k.thr = static_cast<uint32_t>(std::floor(static_cast<double>(p) * 4294967296.0));
  return k;
}

bool valid_dropout_p(float p) { return std::isfinite(p) && p >= 0.0f && p < 1.0f; }

// X (.) M, t x h bf16
size_t dropout_region_bytes(int64_t t, int64_t h) { return align256(static_cast<size_t>(t) * h * 2); }
// the keep mask as bits, t x h / 8 bytes
size_t keep_bits_bytes(int64_t t, int64_t h) { return align256(static_cast<size_t>(t) * h / 8); }

// Xd = X (.) M; the keep bits are drawn (and stored into `bits` if given) or, with from_bits,
// read from `bits`.
int launch_dropout_apply(const uint16_t* X, int64_t n, uint16_t* Xd, uint8_t* bits, bool from_bits,
                         const DropoutKey& key, int dev, cudaStream_t st) {
  const int64_t n8 = n / 8;
  const int64_t per_block = 256 * kDropUnroll;
  // up to 8 CTAs per SM: more than fit at once (5 or 6), measured ~3% faster than one wave
  const int64_t blocks = std::max<int64_t>(
      1, std::min<int64_t>((n8 + per_block - 1) / per_block, static_cast<int64_t>(sm_count(dev)) * 8));
  {
    prof::Scope ps(prof::kDropout, st);
    const auto kern = from_bits ? dropout_apply_kernel<true> : dropout_apply_kernel<false>;
    kern<<<static_cast<unsigned>(blocks), 256, 0, st>>>(
        reinterpret_cast<const uint4*>(X), reinterpret_cast<uint4*>(Xd), bits, n8, key);
  }
  return launch_status();
}

int check_fwd_args(const uint16_t* X, int64_t t, const nf4_weight* W, const uint16_t* L1,
                   const uint16_t* L2, int64_t r, float s, const uint16_t* Y, const uint16_t* sT_out,
                   const void* workspace) {
  if (!X || !L1 || !L2 || !Y) return QLORA_ERR_INVALID_ARG;
  if (!std::isfinite(s)) return QLORA_ERR_INVALID_ARG;
  int rc = check_weight(W);
  if (rc) return rc;
  if ((rc = check_linear_shape(t, W->in_features, W->out_features, r))) return rc;
  if (!aligned16(X) || !aligned16(L1) || !aligned16(L2) || !aligned16(Y) ||
      (sT_out && !aligned16(sT_out)) || (workspace && !aligned16(workspace)))
    return QLORA_ERR_MISALIGNED;
  return QLORA_OK;
}

int check_bwd_args(const uint16_t* dY, const uint16_t* X, int64_t t, const nf4_weight* W,
                   const uint16_t* L1, const uint16_t* L2, int64_t r, float s,
                   const uint16_t* sT_saved, const uint16_t* dX, const float* dL1, const float* dL2,
                   const void* workspace) {
  if (!dY || !X || !L1 || !L2 || !dX || !dL1 || !dL2) return QLORA_ERR_INVALID_ARG;
  if (!std::isfinite(s)) return QLORA_ERR_INVALID_ARG;
  int rc = check_weight(W);
  if (rc) return rc;
  if ((rc = check_linear_shape(t, W->in_features, W->out_features, r))) return rc;
  if (!aligned16(dY) || !aligned16(X) || !aligned16(L1) || !aligned16(L2) || !aligned16(dX) ||
      !aligned16(dL1) || !aligned16(dL2) || (sT_saved && !aligned16(sT_saved)) ||
      (workspace && !aligned16(workspace)))
    return QLORA_ERR_MISALIGNED;
  return QLORA_OK;
}

// Y = X.W' + bf16(s . Xl.L1).L2. Xl is the adapter branch's input: X itself, or X with the
// dropout mask applied (s then carries the 1 / (1 - p)). Arguments already checked.
int fwd_core(const uint16_t* X, const uint16_t* Xl, int64_t t, const nf4_weight* W,
             const uint16_t* L1, const uint16_t* L2, int64_t r, float s, uint16_t* Y,
             uint16_t* sT_out, void* workspace, cudaStream_t st) {
  int dev, rc;
  if ((rc = current_device(&dev))) return rc;
  const int64_t h = W->in_features, o = W->out_features;
  const int sms = sm_count(dev);
  if (t <= kGemvMaxTokens) {
    // partial sums of Xl.L1 (+ zeroed sums and counters), then the GEMV, which forms
    // sT = bf16(s . Xl.L1) and finishes Y
    GemvWs gw = carve_gemv(workspace, t, o, r);
    // codes as 32-row x 64-byte boxes (one unit each); encoded before the first launch, so
    // that the GEMV's launch follows the LoRA-down kernel's at once and can start under it
    CUtensorMap mC;
    if (!make_map_2d(&mC, CU_TENSOR_MAP_DATA_TYPE_UINT8, W->codes, h / 2, o, h / 2, 64,
                     gv::kTileRows, false))
      return QLORA_ERR_CUDA;
    {
      prof::Scope ps(prof::kGemvLoraDown, st);
      gemv_lora_down_kernel<<<gd::kCtas, gd::kThreads, gd::smem_bytes(static_cast<int>(t), static_cast<int>(r)), st>>>(
          Xl, L1, gw.Tpart, gw.Y32, gw.cnt, h, o, static_cast<int>(t), static_cast<int>(r));
    }
    if ((rc = launch_status())) return rc;
    GemvArgs ga{};
    ga.codes = W->codes;
    ga.q8 = W->absmax_q8;
    ga.s2 = W->absmax_s2;
    ga.X = X;
    ga.Tpart = gw.Tpart;
    ga.sT_out = sT_out;
    ga.s = s;
    ga.L2 = L2;
    ga.Y = Y;
    ga.Y32 = gw.Y32;
    ga.tile_cnt = gw.cnt;
    ga.h = h;
    ga.o = o;
    ga.t = static_cast<int>(t);
    ga.r = static_cast<int>(r);
    ga.tab = device_table();
    // one CTA of 16 warps per SM (fewer when there are fewer units than warps, or capped)
    const int64_t units = (o / gv::kTileRows) * ((h / 64 + 1) / 2);
    int64_t ctas = std::min<int64_t>(sms, (units + gv::kWarps - 1) / gv::kWarps);
    const int cap = g_gemv_max_ctas.load(std::memory_order_relaxed);
    if (cap > 0) ctas = std::min<int64_t>(ctas, cap);
    dim3 grid(static_cast<unsigned>(ctas));
    {
      // programmatic dependent launch: the GEMV's CTAs may start (table, first code loads)
      // while the LoRA-down kernel runs; they wait for its results before using them
      prof::Scope ps(prof::kGemv, st);
      cudaLaunchConfig_t cfg{};
      cfg.gridDim = grid;
      cfg.blockDim = dim3(gv::kThreads);
      cfg.dynamicSmemBytes = gv::smem_bytes();
      cfg.stream = st;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      attr[0].val.programmaticStreamSerializationAllowed = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      const cudaError_t e = t <= 8 ? cudaLaunchKernelEx(&cfg, nf4_gemv_kernel<1>, ga, mC)
                                   : cudaLaunchKernelEx(&cfg, nf4_gemv_kernel<2>, ga, mC);
      if (e != cudaSuccess) return QLORA_ERR_CUDA;
    }
    return launch_status();
  }

  LoraWs ws = carve_lora(workspace, t, r);

  // T = Xl . L1 (t x r), then sT = bf16(s . T)
  CUtensorMap mXl, mL1;
  if (!map_bf16(&mXl, Xl, h, t, 64, 128) || !map_bf16(&mL1, L1, r, h, 64, 64)) return QLORA_ERR_CUDA;
  uint16_t* sT = ws.b16;
  if ((rc = lora_down<true>(mXl, mL1, t, h, r, s, sT, sT_out, sms, st))) return rc;

  // Y = X . W' + sT . L2
  CUtensorMap mA, mP, mA2, mB2;
  if (!map_bf16(&mA, X, h, t, 64, 128) ||
      !make_map_2d(&mP, CU_TENSOR_MAP_DATA_TYPE_UINT8, W->codes, h / 2, o, h / 2, 32, tc::BNH, false) ||
      !map_bf16(&mA2, sT, r, t, 64, 128) || !map_bf16(&mB2, L2, o, r, 64, 64))
    return QLORA_ERR_CUDA;
  Nf4GemmArgs ga{};
  ga.q8 = W->absmax_q8;
  ga.s2 = W->absmax_s2;
  ga.h = h;
  ga.M = static_cast<int>(t);
  ga.N = static_cast<int>(o);
  ga.num_kb = static_cast<int>(h / 64);
  ga.num_lkb = static_cast<int>((r + 63) / 64);
  ga.out = Y;
  ga.tab = device_table();
  return launch_nf4_gemm<false>(mA, mP, mA2, mB2, ga, t, o, st, prof::kGemmFwd);
}

// dX = dY.W'^T + M (.) (sU.L1^T), dL1 = Xl^T.sU, dL2 = sT^T.dY with sU = bf16(s . dY.L2^T) and
// sT = bf16(s . Xl.L1) (or the forward's copy). Without dropout (keep_bits == NULL) Xl = X, M
// is all ones and the LoRA term of dX is a K-step of the fused kernel. With dropout Xl = X (.) M
// (computed into `xd`, t x h bf16, by the caller, with the mask as bits in keep_bits: bit
// e mod 8 of byte e / 8), s carries the 1 / (1 - p), and the masked term
// E = bf16(M (.) sU.L1^T) is made after dL1 has consumed Xl, into the same buffer; the fused
// kernel adds E to its fp32 accumulator before its one rounding to bf16. Arguments already
// checked.
int bwd_core(const uint16_t* dY, const uint16_t* Xl, int64_t t, const nf4_weight* W,
             const uint16_t* L1, const uint16_t* L2, int64_t r, float s,
             const uint16_t* sT_saved, uint16_t* dX, float* dL1, float* dL2, void* workspace,
             cudaStream_t st, const uint8_t* keep_bits, uint16_t* xd) {
  int dev, rc;
  if ((rc = current_device(&dev))) return rc;
  const int64_t h = W->in_features, o = W->out_features;
  const int sms = sm_count(dev);
  LoraWs wsU = carve_lora(workspace, t, r);
  LoraWs wsT = carve_lora(reinterpret_cast<uint8_t*>(workspace) + lora_region_bytes(t, r), t, r);

  // sU = bf16(s . dY . L2^T): A = dY (t x o, K-major), B[k=j][n=c] = L2[c][j] (K-major)
  CUtensorMap mdY, mL2k;
  if (!map_bf16(&mdY, dY, o, t, 64, 128) ||
      !map_bf16(&mL2k, L2, o, r, 64, static_cast<uint32_t>((r + 15) / 16 * 16)))
    return QLORA_ERR_CUDA;
  uint16_t* sU = wsU.b16;
  if ((rc = lora_down<false>(mdY, mL2k, t, o, r, s, sU, nullptr, sms, st))) return rc;

  // sT = bf16(s . Xl . L1) unless the forward's copy was passed in
  const uint16_t* sT = sT_saved;
  if (!sT) {
    CUtensorMap mXl, mL1;
    if (!map_bf16(&mXl, Xl, h, t, 64, 128) || !map_bf16(&mL1, L1, r, h, 64, 64)) return QLORA_ERR_CUDA;
    if ((rc = lora_down<true>(mXl, mL1, t, h, r, s, wsT.b16, nullptr, sms, st))) return rc;
    sT = wsT.b16;
  }

  // Launch order U [, sT], dL1, [E,] dX, dL2, each after the first by programmatic dependent
  // launch: dL1 waits for sU; E waits for dL1 (it overwrites dL1's input); the fused dX kernel
  // streams dY and W' while the kernel before it runs and waits for it (hence for sU, and for E)
  // before its LoRA K-step or its epilogue; dL2 needs nothing made in this call unless sT was
  // recomputed, so it can fill the SMs the dX kernel's last wave leaves idle.
  // dL1 = Xl^T . sU (h x r) and dL2^T = dY^T . sT (o x r), reductions over the t tokens
  CUtensorMap mXmn, msU, mdYmn, msT;
  if (!map_bf16(&mXmn, Xl, h, t, 64, 64) || !map_bf16(&msU, sU, r, t, 64, 64) ||
      !map_bf16(&mdYmn, dY, o, t, 64, 64) || !map_bf16(&msT, sT, r, t, 64, 64))
    return QLORA_ERR_CUDA;
  const TcPlan p1 = plan_tc(h, r, t, true, sms);
  if ((rc = launch_tc_gemm<true, true>(mXmn, msU, h, r, p1, 1.0f, kOutRowMajor, dL1, r,
                                       nullptr, nullptr, kPdlWaitFirst, st)))
    return rc;

  const uint16_t* E = nullptr;
  if (keep_bits) {
    // E = bf16(M (.) sU . L1^T), t x h: a K = r product (one CTA per 128 x BNp tile, no
    // split-K) whose epilogue applies the keep bits
    TcPlan pm = plan_tc(t, h, r, false, sms);
    pm.splits = 1;
    pm.kb_per_split = pm.num_kb;
    pm.stages = std::max(2, std::min(pm.stages, pm.num_kb));
    pm.smem = tcg::smem_bytes(pm.stages, pm.BNp, false);
    CUtensorMap mU, mL1k;
    if (!map_bf16(&mU, sU, r, t, 64, 128) || !map_bf16(&mL1k, L1, r, h, 64, static_cast<uint32_t>(pm.BNp)))
      return QLORA_ERR_CUDA;
    if ((rc = launch_tc_gemm<false, false>(mU, mL1k, t, h, pm, 1.0f, kOutMaskBf16, nullptr, h, xd,
                                           nullptr, kPdlWaitFirst, st, nullptr, keep_bits)))
      return rc;
    E = xd;
  }

  // dX = dY . W'^T + sU . L1^T (one accumulator), or dY . W'^T + E
  {
    CUtensorMap mA, mP, mA2, mB2;
    if (!map_bf16(&mA, dY, o, t, 64, 128) ||
        !make_map_2d(&mP, CU_TENSOR_MAP_DATA_TYPE_UINT8, W->codes, h / 2, o, h / 2, 32, 64, false) ||
        !map_bf16(&mA2, sU, r, t, 64, 128) || !map_bf16(&mB2, L1, r, h, 64, tc::BNH))
      return QLORA_ERR_CUDA;
    Nf4GemmArgs ga{};
    ga.q8 = W->absmax_q8;
    ga.s2 = W->absmax_s2;
    ga.h = h;
    ga.M = static_cast<int>(t);
    ga.N = static_cast<int>(h);
    ga.num_kb = static_cast<int>(o / 64);
    ga.num_lkb = E ? 0 : static_cast<int>((r + 63) / 64);
    ga.out = dX;
    ga.tab = device_table();
    ga.addend = E;
    if ((rc = launch_nf4_gemm<true>(mA, mP, mA2, mB2, ga, t, h, st, prof::kGemmBwd))) return rc;
  }

  const TcPlan p2 = plan_tc(o, r, t, true, sms);
  return launch_tc_gemm<true, true>(mdYmn, msT, o, r, p2, 1.0f, kOutTransposed, dL2, o, nullptr,
                                    nullptr, sT_saved ? kPdlWaitLast : kPdlWaitFirst, st);
}

}  // namespace

// ==========================================================================================
// C ABI
// ==========================================================================================
extern "C" {

int qlora_nf4_codebook(float* levels, float* midpoints) {
  if (!levels) return QLORA_ERR_INVALID_ARG;
  const Codebook& cb = codebook();
  std::memcpy(levels, cb.level, sizeof(cb.level));
  if (midpoints) std::memcpy(midpoints, cb.mid, sizeof(cb.mid));
  return QLORA_OK;
}

// W_m = W' + s.L1.L2 in the stored orientation ("QLoRA in LLMs" section 11: dequantize the
// base into a wider precision and add the LoRA update): Wt_m (o x h fp32) = Wt' + s.L2^T.L1^T,
// one tcgen05 product with K = r (A = L2 read MN-major, B = L1 read K-major, 128 x 256 output
// tiles), the dequantized rows added in the epilogue.
int qlora_merge_adapters(const nf4_weight* W, const uint16_t* L1, const uint16_t* L2, int64_t r,
                         float s, float* Wt_merged, qlora_stream_t stream) {
  if (!L1 || !L2 || !Wt_merged) return QLORA_ERR_INVALID_ARG;
  if (!std::isfinite(s)) return QLORA_ERR_INVALID_ARG;
  int rc = check_weight(W);
  if (rc) return rc;
  const int64_t h = W->in_features, o = W->out_features;
  if ((rc = check_linear_shape(1, h, o, r))) return rc;
  if (!aligned16(L1) || !aligned16(L2) || !aligned16(Wt_merged)) return QLORA_ERR_MISALIGNED;
  int dev;
  if ((rc = current_device(&dev))) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  CUtensorMap mA, mB, mOut;
  TcPlan pl = plan_tc(o, h, r, false, sm_count(dev));
  pl.splits = 1;   // the merge epilogue needs the whole K (= r) in one CTA
  pl.kb_per_split = pl.num_kb;
  // 128-column tiles: 128 TMEM columns per CTA, so that kMergeCtasPerSm CTAs fit on an SM
  pl.BNp = static_cast<int>(std::min<int64_t>(128, (h + 15) / 16 * 16));
  // one stage per K-step (a short K needs no more; a small CTA lets four share an SM), but
  // the staging tiles (4 warps x 8 KB) live in the drained stage buffers: keep enough stages
  pl.stages = std::min(pl.num_kb, tcg::MAX_STAGES);
  while (static_cast<size_t>(pl.stages) * tcg::stage_bytes(pl.BNp, false) < tcg::kMergeStagingBytes &&
         pl.stages < tcg::MAX_STAGES)
    ++pl.stages;
  pl.smem = tcg::smem_bytes(pl.stages, pl.BNp, false);
  if (static_cast<size_t>(pl.stages) * tcg::stage_bytes(pl.BNp, false) < tcg::kMergeStagingBytes)
    return QLORA_ERR_BAD_SHAPE;
  if (!map_bf16(&mA, L2, o, r, 64, 64) || !map_bf16(&mB, L1, r, h, 64, static_cast<uint32_t>(pl.BNp)) ||
      !make_map_2d(&mOut, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, Wt_merged, h, o, h * 4, 32, 32, true))
    return QLORA_ERR_CUDA;
  return launch_tc_gemm<true, false, kMergeCtasPerSm>(mA, mB, o, h, pl, s, kOutMergeNF4, Wt_merged,
                                                      h, nullptr, nullptr, kPdlNone, st, W, nullptr,
                                                      &mOut);
}

// Bring a buffer in unified (managed) memory to this device before a kernel touches it, as a
// paged optimizer's state returns when the optimizer needs it; plain device memory is left as
// it is. Pure hints: a failed query or prefetch changes nothing but speed.
void prefetch_if_managed(const void* ptr, size_t bytes, int dev, cudaStream_t st) {
  cudaPointerAttributes at{};
  if (cudaPointerGetAttributes(&at, ptr) != cudaSuccess) {
    cudaGetLastError();
    return;
  }
  if (at.type == cudaMemoryTypeManaged && cudaMemPrefetchAsync(ptr, bytes, dev, st) != cudaSuccess)
    cudaGetLastError();
}

int qlora_adamw_step(float* param, uint16_t* param_bf16, const float* grad, float* m, float* v,
                     int64_t n, float lr, float beta1, float beta2, float eps, float weight_decay,
                     int64_t step, unsigned flags, qlora_stream_t stream) {
  if (!param || !grad || !m || !v || n <= 0 || n % 4 != 0 || step < 1) return QLORA_ERR_INVALID_ARG;
  if (!std::isfinite(lr) || !std::isfinite(eps) || !std::isfinite(weight_decay) || eps <= 0.f ||
      !(beta1 >= 0.f && beta1 < 1.f) || !(beta2 >= 0.f && beta2 < 1.f))
    return QLORA_ERR_INVALID_ARG;
  if (!aligned16(param) || !aligned16(grad) || !aligned16(m) || !aligned16(v) ||
      (param_bf16 && (reinterpret_cast<uintptr_t>(param_bf16) & 7u)))
    return QLORA_ERR_MISALIGNED;
  int dev, rc;
  if ((rc = current_device(&dev))) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (flags & ~static_cast<unsigned>(QLORA_ADAMW_PREFETCH)) return QLORA_ERR_INVALID_ARG;
  if (flags & QLORA_ADAMW_PREFETCH) {
    const size_t bytes = static_cast<size_t>(n) * 4;
    prefetch_if_managed(m, bytes, dev, st);
    prefetch_if_managed(v, bytes, dev, st);
    prefetch_if_managed(param, bytes, dev, st);
    prefetch_if_managed(grad, bytes, dev, st);
  }
  AdamwArgs a{};
  a.p = param;
  a.p16 = param_bf16;
  a.g = grad;
  a.m = m;
  a.v = v;
  a.n4 = n / 4;
  a.lr = lr;
  a.beta1 = beta1;
  a.beta2 = beta2;
  a.eps = eps;
  a.wd = weight_decay;
  a.step_size = static_cast<float>(lr / (1.0 - std::pow(static_cast<double>(beta1), static_cast<double>(step))));
  a.inv_sqrt_bc2 = static_cast<float>(1.0 / std::sqrt(1.0 - std::pow(static_cast<double>(beta2), static_cast<double>(step))));
  const int64_t want = (a.n4 + 255) / 256;
  const int grid = static_cast<int>(std::max<int64_t>(
      1, std::min<int64_t>(want, int64_t(sm_count(dev)) * device_info(dev).adamw_ctas)));
  adamw_kernel<<<grid, 256, 0, st>>>(a);
  return launch_status();
}

int qlora_adamw_step_multi(int ntensors, float* const* params, uint16_t* const* params_bf16,
                           const float* const* grads, float* const* m, float* const* v,
                           const int64_t* counts, float lr, float beta1, float beta2, float eps,
                           float weight_decay, int64_t step, unsigned flags, qlora_stream_t stream) {
  if (ntensors < 1 || ntensors > kAdamwMaxTensors || !params || !grads || !m || !v || !counts ||
      step < 1)
    return QLORA_ERR_INVALID_ARG;
  if (!std::isfinite(lr) || !std::isfinite(eps) || !std::isfinite(weight_decay) || eps <= 0.f ||
      !(beta1 >= 0.f && beta1 < 1.f) || !(beta2 >= 0.f && beta2 < 1.f))
    return QLORA_ERR_INVALID_ARG;
  if (flags & ~static_cast<unsigned>(QLORA_ADAMW_PREFETCH)) return QLORA_ERR_INVALID_ARG;
  AdamwMultiArgs a{};
  a.ntensors = ntensors;
  a.first4[0] = 0;
  for (int k = 0; k < ntensors; ++k) {
    if (!params[k] || !grads[k] || !m[k] || !v[k] || counts[k] <= 0 || counts[k] % 4 != 0)
      return QLORA_ERR_INVALID_ARG;
    uint16_t* p16 = params_bf16 ? params_bf16[k] : nullptr;
    if (!aligned16(params[k]) || !aligned16(grads[k]) || !aligned16(m[k]) || !aligned16(v[k]) ||
        (p16 && (reinterpret_cast<uintptr_t>(p16) & 7u)))
      return QLORA_ERR_MISALIGNED;
    a.p[k] = params[k];
    a.p16[k] = p16;
    a.g[k] = grads[k];
    a.m[k] = m[k];
    a.v[k] = v[k];
    a.first4[k + 1] = a.first4[k] + counts[k] / 4;
  }
  int dev, rc;
  if ((rc = current_device(&dev))) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (flags & QLORA_ADAMW_PREFETCH) {
    for (int k = 0; k < ntensors; ++k) {
      const size_t bytes = static_cast<size_t>(counts[k]) * 4;
      prefetch_if_managed(m[k], bytes, dev, st);
      prefetch_if_managed(v[k], bytes, dev, st);
      prefetch_if_managed(params[k], bytes, dev, st);
      prefetch_if_managed(grads[k], bytes, dev, st);
    }
  }
  a.hy.lr = lr;
  a.hy.beta1 = beta1;
  a.hy.beta2 = beta2;
  a.hy.eps = eps;
  a.hy.wd = weight_decay;
  a.hy.step_size = static_cast<float>(lr / (1.0 - std::pow(static_cast<double>(beta1), static_cast<double>(step))));
  a.hy.inv_sqrt_bc2 = static_cast<float>(1.0 / std::sqrt(1.0 - std::pow(static_cast<double>(beta2), static_cast<double>(step))));
  const int64_t want = (a.first4[ntensors] + 255) / 256;
  const int grid = static_cast<int>(std::max<int64_t>(
      1, std::min<int64_t>(want, int64_t(sm_count(dev)) * device_info(dev).adamw_multi_ctas)));
  adamw_multi_kernel<<<grid, 256, 0, st>>>(a);
  return launch_status();
}

// One thread waits on an mbarrier that no arrival will ever complete; the bounded wait gives
// up after limit_ns, raises its CTA's abort flag and reports kDevTimeout. Nothing faults.
__global__ void wait_timeout_selftest_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ uint32_t abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0u;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) (void)mbar_wait(&bar, 0u, &abort_flag, limit_ns);
}

int qlora_selftest_wait_timeout(int64_t limit_ns, qlora_stream_t stream) {
  if (limit_ns < 1000 || limit_ns > static_cast<int64_t>(kWaitTimeoutNs)) return QLORA_ERR_INVALID_ARG;
  int dev, rc;
  if ((rc = current_device(&dev))) return rc;
  wait_timeout_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<uint64_t>(limit_ns));
  return launch_status();
}

int qlora_set_gemv_max_ctas(int n) {
  return g_gemv_max_ctas.exchange(n > 0 ? n : 0);
}

const char* qlora_status_string(int status) {
  switch (status) {
    case QLORA_OK: return "QLORA_OK";
    case QLORA_ERR_INVALID_ARG: return "QLORA_ERR_INVALID_ARG: null pointer or invalid argument";
    case QLORA_ERR_BAD_SHAPE: return "QLORA_ERR_BAD_SHAPE: unsupported shape";
    case QLORA_ERR_MISALIGNED: return "QLORA_ERR_MISALIGNED: pointer not 16-byte aligned";
    case QLORA_ERR_WORKSPACE: return "QLORA_ERR_WORKSPACE: workspace missing or too small";
    case QLORA_ERR_CUDA: return "QLORA_ERR_CUDA: CUDA runtime or launch error";
    case QLORA_ERR_UNSUPPORTED_DEVICE: return "QLORA_ERR_UNSUPPORTED_DEVICE: not an sm_100 GPU";
    case QLORA_ERR_SCRATCH_LIMIT:
      return "QLORA_ERR_SCRATCH_LIMIT: shape needs more than the static scratch holds";
    case QLORA_DEV_NONFINITE: return "QLORA_DEV_NONFINITE: non-finite weight";
    case QLORA_DEV_TIMEOUT: return "QLORA_DEV_TIMEOUT: a kernel wait timed out";
    case QLORA_DEV_NONFINITE | QLORA_DEV_TIMEOUT:
      return "QLORA_DEV_NONFINITE|QLORA_DEV_TIMEOUT";
    default: return "unknown status";
  }
}

size_t qlora_fwd_workspace_bytes(int64_t t, int64_t h, int64_t o, int64_t r) {
  if (check_linear_shape(t, h, o, r) != QLORA_OK) return 0;
  if (t <= kGemvMaxTokens) return gemv_ws_bytes(t, o, r);
  return lora_region_bytes(t, r);
}

size_t qlora_bwd_workspace_bytes(int64_t t, int64_t h, int64_t o, int64_t r) {
  if (check_linear_shape(t, h, o, r) != QLORA_OK) return 0;
  return 2 * lora_region_bytes(t, r);
}

int qlora_profile_begin(int capacity) {
  if (capacity < 1 || capacity > (1 << 20)) return QLORA_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(prof::g.mu);
  while (static_cast<int>(prof::g.events.size()) < 2 * capacity) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) {
      cudaGetLastError();
      return QLORA_ERR_CUDA;
    }
    prof::g.events.push_back(e);
  }
  if (static_cast<int>(prof::g.kinds.size()) < capacity) prof::g.kinds.resize(capacity);
  prof::g.capacity = capacity;
  prof::g.n = 0;
  prof::g.overflow = false;
  prof::g.on.store(true);
  return QLORA_OK;
}

int qlora_profile_end(double* ms, int64_t* launches, int nkinds) {
  std::lock_guard<std::mutex> lock(prof::g.mu);
  prof::g.on.store(false);
  if (ms) for (int k = 0; k < nkinds; ++k) ms[k] = 0.0;
  if (launches) for (int k = 0; k < nkinds; ++k) launches[k] = 0;
  for (int i = 0; i < prof::g.n; ++i) {
    if (cudaEventSynchronize(prof::g.events[2 * i + 1]) != cudaSuccess) {
      cudaGetLastError();
      return QLORA_ERR_CUDA;
    }
    float t = 0.f;
    if (cudaEventElapsedTime(&t, prof::g.events[2 * i], prof::g.events[2 * i + 1]) != cudaSuccess) {
      cudaGetLastError();
      return QLORA_ERR_CUDA;
    }
    const int k = prof::g.kinds[i];
    if (k < nkinds) {
      if (ms) ms[k] += t;
      if (launches) launches[k] += 1;
    }
  }
  if (prof::g.overflow) return QLORA_ERR_INVALID_ARG;
  return prof::g.n;
}

const char* qlora_kernel_name(int kind) {
  if (kind < 0 || kind >= prof::kKinds) return "unknown";
  return prof::kNames[kind];
}

int qlora_get_last_status(qlora_stream_t stream) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return QLORA_ERR_CUDA;
  }
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return QLORA_ERR_CUDA;
  }
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(v)) != cudaSuccess ||
      cudaMemcpyToSymbol(g_status, &zero, sizeof(zero)) != cudaSuccess) {
    cudaGetLastError();
    return QLORA_ERR_CUDA;
  }
  return static_cast<int>(v);
}

int qlora_quantize_format(const float* Wt, const nf4_weight* q, int codebook_id, int scale_format,
                          qlora_stream_t stream) {
  if (!Wt) return QLORA_ERR_INVALID_ARG;
  if (codebook_id < 0 || codebook_id >= kCodebooks) return QLORA_ERR_INVALID_ARG;
  if (scale_format < kScalesU8 || scale_format > kScalesE4M3) return QLORA_ERR_INVALID_ARG;
  int rc = check_weight(q);
  if (rc) return rc;
  if (!aligned16(Wt)) return QLORA_ERR_MISALIGNED;
  int dev;
  if ((rc = current_device(&dev))) return rc;
  const int64_t nblocks = q->out_features * q->in_features / 64;
  const int64_t ngroups = (nblocks + 255) / 256;
  const int grid = static_cast<int>(std::min<int64_t>(ngroups, int64_t(sm_count(dev)) * qz::kCtasPerSm));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(qz::kThreads, 1, 1);
  cfg.dynamicSmemBytes = qz::smem_bytes();
  cfg.stream = reinterpret_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e;
  {
    prof::Scope ps(prof::kQuant, reinterpret_cast<cudaStream_t>(stream));
    e = cudaLaunchKernelEx(&cfg, nf4_quantize_kernel, Wt, q->codes, q->absmax_q8, q->absmax_s2,
                           nblocks, device_table(codebook_id), device_buckets(codebook_id),
                           scale_format);
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    return QLORA_ERR_CUDA;
  }
  return launch_status();
}

int qlora_dequantize_format(const nf4_weight* q, int codebook_id, int scale_format, uint16_t* Wt_out,
                            qlora_stream_t stream) {
  if (!Wt_out) return QLORA_ERR_INVALID_ARG;
  if (codebook_id < 0 || codebook_id >= kCodebooks) return QLORA_ERR_INVALID_ARG;
  if (scale_format < kScalesU8 || scale_format > kScalesE4M3) return QLORA_ERR_INVALID_ARG;
  int rc = check_weight(q);
  if (rc) return rc;
  if (!aligned16(Wt_out)) return QLORA_ERR_MISALIGNED;
  int dev;
  if ((rc = current_device(&dev))) return rc;
  const int64_t n = q->out_features * q->in_features;   // a multiple of 64
  const int64_t want = (n + dq::kChunk * dq::kWarps - 1) / (dq::kChunk * dq::kWarps);
  const int grid = static_cast<int>(
      std::min<int64_t>(want, int64_t(sm_count(dev)) * device_info(dev).dq_ctas));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(std::max(grid, 1)), 1, 1);
  cfg.blockDim = dim3(dq::kThreads, 1, 1);
  cfg.stream = reinterpret_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e;
  {
    prof::Scope ps(prof::kDequant, reinterpret_cast<cudaStream_t>(stream));
    e = cudaLaunchKernelEx(&cfg, nf4_dequantize_kernel, q->codes, q->absmax_q8, q->absmax_s2,
                           Wt_out, n, device_table(codebook_id), scale_format);
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    return QLORA_ERR_CUDA;
  }
  return launch_status();
}

int qlora_quantize_codebook(const float* Wt, const nf4_weight* q, int codebook_id,
                            qlora_stream_t stream) {
  return qlora_quantize_format(Wt, q, codebook_id, kScalesU8, stream);
}

int qlora_dequantize_codebook(const nf4_weight* q, int codebook_id, uint16_t* Wt_out,
                              qlora_stream_t stream) {
  return qlora_dequantize_format(q, codebook_id, kScalesU8, Wt_out, stream);
}

int nf4_quantize(const float* Wt, const nf4_weight* q, qlora_stream_t stream) {
  return qlora_quantize_codebook(Wt, q, 0, stream);
}

int nf4_dequantize(const nf4_weight* q, uint16_t* Wt_out, qlora_stream_t stream) {
  return qlora_dequantize_codebook(q, 0, Wt_out, stream);
}

int qlora_codebook(int codebook_id, float* levels, float* midpoints) {
  if (!levels || codebook_id < 0 || codebook_id >= kCodebooks) return QLORA_ERR_INVALID_ARG;
  const Codebook& cb = codebook(codebook_id);
  std::memcpy(levels, cb.level, sizeof(cb.level));
  if (midpoints) std::memcpy(midpoints, cb.mid, sizeof(cb.mid));
  return QLORA_OK;
}

int qlora_linear_fwd(const uint16_t* X, int64_t t, const nf4_weight* W, const uint16_t* L1,
                     const uint16_t* L2, int64_t r, float s, uint16_t* Y, uint16_t* sT_out,
                     void* workspace, size_t ws_bytes, qlora_stream_t stream) {
  int rc = check_fwd_args(X, t, W, L1, L2, r, s, Y, sT_out, workspace);
  if (rc) return rc;
  if (!workspace || ws_bytes < qlora_fwd_workspace_bytes(t, W->in_features, W->out_features, r))
    return QLORA_ERR_WORKSPACE;
  return fwd_core(X, X, t, W, L1, L2, r, s, Y, sT_out, workspace, reinterpret_cast<cudaStream_t>(stream));
}

int qlora_linear_bwd(const uint16_t* dY, const uint16_t* X, int64_t t, const nf4_weight* W,
                     const uint16_t* L1, const uint16_t* L2, int64_t r, float s,
                     const uint16_t* sT_saved, uint16_t* dX, float* dL1, float* dL2,
                     void* workspace, size_t ws_bytes, qlora_stream_t stream) {
  int rc = check_bwd_args(dY, X, t, W, L1, L2, r, s, sT_saved, dX, dL1, dL2, workspace);
  if (rc) return rc;
  if (!workspace || ws_bytes < qlora_bwd_workspace_bytes(t, W->in_features, W->out_features, r))
    return QLORA_ERR_WORKSPACE;
  return bwd_core(dY, X, t, W, L1, L2, r, s, sT_saved, dX, dL1, dL2, workspace,
                  reinterpret_cast<cudaStream_t>(stream), nullptr, nullptr);
}

size_t qlora_fwd_dropout_workspace_bytes(int64_t t, int64_t h, int64_t o, int64_t r) {
  const size_t base = qlora_fwd_workspace_bytes(t, h, o, r);
  return base ? dropout_region_bytes(t, h) + base : 0;
}

size_t qlora_bwd_dropout_workspace_bytes(int64_t t, int64_t h, int64_t o, int64_t r) {
  const size_t base = qlora_bwd_workspace_bytes(t, h, o, r);
  return base ? dropout_region_bytes(t, h) + keep_bits_bytes(t, h) + base : 0;
}

int qlora_dropout_apply(const uint16_t* X, int64_t t, int64_t h, float p, uint64_t seed,
                        uint16_t* Xd, qlora_stream_t stream) {
  if (!X || !Xd || !valid_dropout_p(p)) return QLORA_ERR_INVALID_ARG;
  if (t < 1 || h < 64 || h % 64 != 0 || t >= kMaxDim || h >= kMaxDim) return QLORA_ERR_BAD_SHAPE;
  if (!aligned16(X) || !aligned16(Xd)) return QLORA_ERR_MISALIGNED;
  const uintptr_t a = reinterpret_cast<uintptr_t>(X), b = reinterpret_cast<uintptr_t>(Xd);
  const uintptr_t bytes = static_cast<uintptr_t>(t) * static_cast<uintptr_t>(h) * 2u;
  if (a != b && a < b + bytes && b < a + bytes) return QLORA_ERR_INVALID_ARG;  // partial overlap
  int dev, rc;
  if ((rc = current_device(&dev))) return rc;
  return launch_dropout_apply(X, t * h, Xd, nullptr, false, dropout_key(p, seed), dev,
                              reinterpret_cast<cudaStream_t>(stream));
}

int qlora_linear_fwd_dropout(const uint16_t* X, int64_t t, const nf4_weight* W, const uint16_t* L1,
                             const uint16_t* L2, int64_t r, float s, float p, uint64_t seed,
                             uint16_t* Y, uint16_t* sT_out, uint8_t* mask_out, void* workspace,
                             size_t ws_bytes, qlora_stream_t stream) {
  int rc = check_fwd_args(X, t, W, L1, L2, r, s, Y, sT_out, workspace);
  if (rc) return rc;
  if (!valid_dropout_p(p)) return QLORA_ERR_INVALID_ARG;
  const float s_eff = s / (1.0f - p);
  if (!std::isfinite(s_eff)) return QLORA_ERR_INVALID_ARG;
  if (mask_out && !aligned16(mask_out)) return QLORA_ERR_MISALIGNED;
  const int64_t h = W->in_features;
  if (!workspace || ws_bytes < qlora_fwd_dropout_workspace_bytes(t, h, W->out_features, r))
    return QLORA_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint16_t* Xd = reinterpret_cast<uint16_t*>(workspace);
  void* rest = reinterpret_cast<uint8_t*>(workspace) + dropout_region_bytes(t, h);
  const DropoutKey key = dropout_key(p, seed);
  if (key.thr == 0) {
    if (mask_out && cudaMemsetAsync(mask_out, 0xFF, static_cast<size_t>(t) * h / 8, st) != cudaSuccess) {
      cudaGetLastError();
      return QLORA_ERR_CUDA;
    }
    return fwd_core(X, X, t, W, L1, L2, r, s, Y, sT_out, rest, st);
  }
  int dev;
  if ((rc = current_device(&dev))) return rc;
  if ((rc = launch_dropout_apply(X, t * h, Xd, mask_out, false, key, dev, st))) return rc;
  return fwd_core(X, Xd, t, W, L1, L2, r, s_eff, Y, sT_out, rest, st);
}

int qlora_linear_bwd_dropout(const uint16_t* dY, const uint16_t* X, int64_t t, const nf4_weight* W,
                             const uint16_t* L1, const uint16_t* L2, int64_t r, float s, float p,
                             uint64_t seed, const uint16_t* sT_saved, const uint8_t* mask_saved,
                             uint16_t* dX, float* dL1, float* dL2, void* workspace, size_t ws_bytes,
                             qlora_stream_t stream) {
  int rc = check_bwd_args(dY, X, t, W, L1, L2, r, s, sT_saved, dX, dL1, dL2, workspace);
  if (rc) return rc;
  if (!valid_dropout_p(p)) return QLORA_ERR_INVALID_ARG;
  const float s_eff = s / (1.0f - p);
  if (!std::isfinite(s_eff)) return QLORA_ERR_INVALID_ARG;
  if (mask_saved && !aligned16(mask_saved)) return QLORA_ERR_MISALIGNED;
  const int64_t h = W->in_features;
  if (!workspace || ws_bytes < qlora_bwd_dropout_workspace_bytes(t, h, W->out_features, r))
    return QLORA_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* b = reinterpret_cast<uint8_t*>(workspace);
  uint16_t* Xd = reinterpret_cast<uint16_t*>(b);
  uint8_t* bits = b + dropout_region_bytes(t, h);
  void* rest = bits + keep_bits_bytes(t, h);
  const DropoutKey key = dropout_key(p, seed);
  if (key.thr == 0)
    return bwd_core(dY, X, t, W, L1, L2, r, s, sT_saved, dX, dL1, dL2, rest, st, nullptr, nullptr);
  int dev;
  if ((rc = current_device(&dev))) return rc;
  // the forward's mask when given (no generator calls), else drawn again from (p, seed)
  uint8_t* mask = mask_saved ? const_cast<uint8_t*>(mask_saved) : bits;
  if ((rc = launch_dropout_apply(X, t * h, Xd, mask, mask_saved != nullptr, key, dev, st)))
    return rc;
  return bwd_core(dY, Xd, t, W, L1, L2, r, s_eff, sT_saved, dX, dL1, dL2, rest, st, mask, Xd);
}

}  // extern "C"

// ==========================================================================================
// Allocation-free forward: the caller's workspace replaced by a scratch array in the library's
// own device image. The forward itself is qlora_linear_fwd, unchanged.
// ==========================================================================================
namespace {

// One copy per device that loads the library, alive until the process exits.
static __device__ __align__(256) unsigned char g_static_scratch[QLORA_STATIC_SCRATCH_BYTES];

// Device address of g_static_scratch per device, cached only once a lookup has succeeded, so
// that a failed lookup (a transient error, or a first call made during a stream capture) is
// retried by the next call instead of being remembered.
std::atomic<void*> g_scratch_ptr[kMaxDevices];
std::mutex g_scratch_mu;

// In host code the name g_static_scratch is only a host-side stand-in, not a device address:
// the address a kernel may use is looked up per device, with that device current.
int static_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return QLORA_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return QLORA_ERR_UNSUPPORTED_DEVICE;
  void* p = g_scratch_ptr[dev].load(std::memory_order_acquire);
  if (!p) {
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    p = g_scratch_ptr[dev].load(std::memory_order_relaxed);
    if (!p) {
      if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) {
        cudaGetLastError();
        return QLORA_ERR_CUDA;
      }
      g_scratch_ptr[dev].store(p, std::memory_order_release);
    }
  }
  *out = p;
  return QLORA_OK;
}

}  // namespace

extern "C" int qlora_linear_fwd_noalloc(const uint16_t* X, int64_t t, const nf4_weight* W,
                                        const uint16_t* L1, const uint16_t* L2, int64_t r, float s,
                                        uint16_t* Y, uint16_t* sT_out, qlora_stream_t stream) {
  if (!W) return QLORA_ERR_INVALID_ARG;
  const size_t need = qlora_fwd_workspace_bytes(t, W->in_features, W->out_features, r);
  if (need > QLORA_STATIC_SCRATCH_BYTES) return QLORA_ERR_SCRATCH_LIMIT;
  void* scratch = nullptr;
  if (need != 0) {  // need == 0: invalid shape, let the forward's own checks report it
    const int rc = static_scratch(&scratch);
    if (rc != QLORA_OK) return rc;
  }
  return qlora_linear_fwd(X, t, W, L1, L2, r, s, Y, sT_out, scratch,
                          scratch ? static_cast<size_t>(QLORA_STATIC_SCRATCH_BYTES) : 0, stream);
}

#ifdef QLORA_TRACE
extern "C" QLORA_API int qlora_trace_read(void* host, size_t bytes) {
  if (bytes > sizeof(g_trace)) bytes = sizeof(g_trace);
  return cudaMemcpyFromSymbol(host, g_trace, bytes) == cudaSuccess ? 0 : -5;
}
extern "C" QLORA_API int qlora_trace_clear() {
  static unsigned long long zero[kTraceCtas][8];
  return cudaMemcpyToSymbol(g_trace, zero, sizeof(zero)) == cudaSuccess ? 0 : -5;
}
#endif
