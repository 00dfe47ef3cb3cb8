// flce.cu - the C ABI (include/flce.h) of the sm_100a fused LM-head projection
// + cross-entropy, its auxiliary kernels and the host-side planning.
//
// Forward  (nemo_automodel.components.models.inkling2.loss,
//           Inkling2FusedLinearCrossEntropy: BF16 x BF16 -> FP32, softcap and
//           CE in FP32, rows >= unpadded_vocab never enter the softmax):
//   [cast]  FP32 head rows [0, V) -> BF16 (only for an FP32 head)
//   K1      tensor-core GEMM hidden . W^T, epilogue: softcap, per-tile
//           (max, sum exp) and the label's logit  -> partials [V/256][N]
//   K2      merge partials per token -> lse, token loss, block sums
//   K2b     deterministic final sum -> loss (/ num_label_tokens, or mean)
// Backward (nemo_automodel.components.loss.chunked_ce,
//           _ChunkedCrossEntropySum.backward: recompute instead of storing):
//   prep    per-token gradient scale s_n, lse * log2(e), zero tile counters
//   per vocabulary chunk c = [v0, v0 + Vc), G double-buffered (G[c % 2]):
//     K3    GEMM hidden . W[chunk]^T, epilogue: G = s_n (softmax - onehot) dcap
//           -> BF16 G[N, Vc] (bounded chunk buffer, never [N, V])
//     K5    GEMM G . W[chunk]  -> dhidden, FP32 accumulation across chunks,
//           BF16 on the last chunk
//     K4    GEMM G^T . hidden  -> dW[chunk] (head dtype)
//   launched as K3(0), then one grouped launch per chunk {K5(c), K4(c),
//   K3(c+1)} whose CTAs take tiles dynamically, long K5 tiles first, so no
//   launch ends on a partial wave of long tiles
//   zero    dW rows [V, Vp)
// Every GEMM above runs on the CTA-pair kernel of gemm_sm100_pair.cuh (256 x
// 256 tiles, tcgen05 cta_group::2); the epilogues are in epilogues.cuh.
// Cross entropy on given logits (chunked_ce page) is at the end of this file,
// its row kernels in chunked_ce.cuh; the forward without allocation at the end.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <atomic>
#include <mutex>
#include <vector>

#include <nvtx3/nvToolsExt.h>  // header-only; ranges cost a pointer test unless a tool attaches

#include "flce.h"
#include "epilogues.cuh"
#include "gemm_sm100.cuh"
#include "gemm_sm100_pair.cuh"
#include "chunked_ce.cuh"

namespace flce {

__device__ unsigned int g_device_error;  // per-device sticky error word (kDevErr*)

constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;  // 2 s per pipeline wait
constexpr int kMergeRows = 32;                         // token rows per merge block
constexpr int kMergeWarps = 16;
constexpr int kFinalThreads = 256;
constexpr int64_t kMaxDim = (int64_t(1) << 31) - 1024;  // TMA coordinates are int32
constexpr size_t kAlign = 1024;
constexpr size_t kChunkBudgetBytes = size_t(1) << 30;  // default cap on each G buffer
constexpr int64_t kMinChunk = 4096;

// Contractions run on CTA pairs: 256 x 256 tiles, tcgen05 cta_group::2.
constexpr int kTileRows = kPairBM;   // output rows per tile
constexpr int kBBoxRows = kBN / 2;   // K-major B rows loaded per CTA (half of the tile's)

// ------------------------------------------------------------------ kernels

// FP32 -> BF16 (round to nearest even), 8 elements per step.
__global__ void cast_f32_to_bf16_kernel(const float4* __restrict__ src, uint4* __restrict__ dst,
                                        int64_t n8) {
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n8;
       i += int64_t(gridDim.x) * blockDim.x) {
    const float4 a = src[2 * i], b = src[2 * i + 1];
    uint4 w;
    w.x = pack_bf16x2(a.x, a.y);
    w.y = pack_bf16x2(a.z, a.w);
    w.z = pack_bf16x2(b.x, b.y);
    w.w = pack_bf16x2(b.z, b.w);
    dst[i] = w;
  }
}

__global__ void zero16_kernel(uint4* __restrict__ dst, int64_t n16) {
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n16;
       i += int64_t(gridDim.x) * blockDim.x)
    dst[i] = make_uint4(0, 0, 0, 0);
}

// K2: merge the per-tile partials of 32 token rows (16 warps split the tiles),
// then per token: lse, token loss, label check (mask: optional, 0 = ignore the
// token); per block: loss and count sums.  Also finishes the cross entropy on
// given logits, whose row segments leave partials in the same layout.
__global__ void __launch_bounds__(kMergeRows* kMergeWarps)
    lse_merge_kernel(const float* __restrict__ part_m, const float* __restrict__ part_s,
                     int v_tiles, int64_t n_tokens, const float* __restrict__ label_logit,
                     const int64_t* __restrict__ labels, const uint8_t* __restrict__ mask,
                     int64_t vocab, int64_t ignore_index,
                     float* __restrict__ lse_out, float* __restrict__ token_loss,
                     double* __restrict__ blk_loss, int* __restrict__ blk_cnt,
                     unsigned* __restrict__ err) {
  __shared__ float sm_m[kMergeWarps][kMergeRows];
  __shared__ float sm_s[kMergeWarps][kMergeRows];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t n = int64_t(blockIdx.x) * kMergeRows + lane;
  float M = -INFINITY, S = 0.0f;
  if (n < n_tokens) {
#pragma unroll 4
    for (int t = warp; t < v_tiles; t += kMergeWarps) {
      const float m = part_m[int64_t(t) * n_tokens + n];
      const float s = part_s[int64_t(t) * n_tokens + n];
      if (m == -INFINITY) continue;  // an empty partial (or one of only -inf logits)
      const float mn = fmaxf(M, m);
      S = S * exp2f(M - mn) + s * exp2f(m - mn);
      M = mn;
    }
  }
  sm_m[warp][lane] = M;
  sm_s[warp][lane] = S;
  __syncthreads();
  if (warp != 0) return;
  float Mt = -INFINITY, St = 0.0f;
#pragma unroll
  for (int w = 0; w < kMergeWarps; ++w) {
    const float m = sm_m[w][lane], s = sm_s[w][lane];
    if (m == -INFINITY) continue;
    const float mn = fmaxf(Mt, m);
    St = St * exp2f(Mt - mn) + s * exp2f(m - mn);
    Mt = mn;
  }
  double loss = 0.0;
  int cnt = 0;
  if (n < n_tokens) {
    const float lse = (Mt + log2f(St)) * 0.6931471805599453f;
    const int64_t y = labels[n];
    bool valid = y != ignore_index && (mask == nullptr || mask[n] != 0);
    if (valid && (y < 0 || y >= vocab)) {
      atomicOr(err, kDevErrBadLabel);
      valid = false;
    }
    const float l = valid ? lse - label_logit[n] : 0.0f;
    lse_out[n] = lse;
    if (token_loss) token_loss[n] = l;
    loss = l;
    cnt = valid ? 1 : 0;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    loss += __shfl_down_sync(0xffffffffu, loss, o);
    cnt += __shfl_down_sync(0xffffffffu, cnt, o);
  }
  if (lane == 0) {
    blk_loss[blockIdx.x] = loss;
    blk_cnt[blockIdx.x] = cnt;
  }
}

// K2b: fixed-order sum of the block partials -> loss[0].
__global__ void __launch_bounds__(kFinalThreads)
    loss_finalize_kernel(const double* __restrict__ blk_loss, const int* __restrict__ blk_cnt,
                         int nblk, int reduction, int64_t num_label_tokens,
                         float* __restrict__ loss) {
  __shared__ double sl[kFinalThreads];
  __shared__ long long sc[kFinalThreads];
  double l = 0.0;
  long long c = 0;
  for (int i = threadIdx.x; i < nblk; i += kFinalThreads) {
    l += blk_loss[i];
    c += blk_cnt[i];
  }
  sl[threadIdx.x] = l;
  sc[threadIdx.x] = c;
  __syncthreads();
  for (int s = kFinalThreads / 2; s > 0; s >>= 1) {
    if (threadIdx.x < s) {
      sl[threadIdx.x] += sl[threadIdx.x + s];
      sc[threadIdx.x] += sc[threadIdx.x + s];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    double total = sl[0];
    if (reduction == FLCE_SUM) {
      if (num_label_tokens > 0) total /= double(num_label_tokens);
    } else if (reduction == FLCE_MEAN) {
      total = sc[0] > 0 ? total / double(sc[0]) : double(NAN);
    }
    loss[0] = float(total);
  }
}

// Backward prep (one block): valid-label count, per-token gradient scale
// s_n = d loss / d token loss (0 for ignored / invalid labels), lse * log2(e).
__global__ void __launch_bounds__(1024)
    bwd_prep_kernel(const int64_t* __restrict__ labels, const uint8_t* __restrict__ mask,
                    int64_t n_tokens, int64_t vocab,
                    int64_t ignore_index, int reduction, int64_t num_label_tokens,
                    const float* __restrict__ grad_loss, const float* __restrict__ lse,
                    float* __restrict__ lse2, float* __restrict__ scale,
                    unsigned* __restrict__ counters, int n_counters,
                    unsigned* __restrict__ err) {
  __shared__ int warp_cnt[32];
  for (int i = threadIdx.x; i < n_counters; i += blockDim.x) counters[i] = 0u;
  int cnt = 0;
  bool bad = false;
  for (int64_t n = threadIdx.x; n < n_tokens; n += blockDim.x) {
    const int64_t y = labels[n];
    if (y == ignore_index || (mask != nullptr && mask[n] == 0)) continue;
    if (y < 0 || y >= vocab) {
      bad = true;
      continue;
    }
    ++cnt;
  }
  if (bad) atomicOr(err, kDevErrBadLabel);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_down_sync(0xffffffffu, cnt, o);
  if ((threadIdx.x & 31) == 0) warp_cnt[threadIdx.x >> 5] = cnt;
  __syncthreads();
  int total = 0;
  for (int w = 0; w < int(blockDim.x >> 5); ++w) total += warp_cnt[w];
  float base = 0.0f;
  if (reduction == FLCE_SUM) {
    base = grad_loss[0];
    if (num_label_tokens > 0) base = float(double(base) / double(num_label_tokens));
  } else if (reduction == FLCE_MEAN) {
    base = total > 0 ? float(double(grad_loss[0]) / double(total)) : 0.0f;
  }
  for (int64_t n = threadIdx.x; n < n_tokens; n += blockDim.x) {
    const int64_t y = labels[n];
    const bool valid = y != ignore_index && (mask == nullptr || mask[n] != 0) && y >= 0 &&
                       y < vocab;
    const float g = reduction == FLCE_NONE ? grad_loss[n] : base;
    scale[n] = valid ? g : 0.0f;
    lse2[n] = lse[n] * kLog2e;
  }
}

// A wait on a barrier that nothing arrives on: exercises the bounded-wait path.
__global__ void wait_timeout_selftest_kernel(unsigned* err, uint64_t timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ PipeCtl ctl;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    ctl.abort = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    wait_phase(smem_u32(&bar), 0, &ctl, err, timeout_ns);
  }
  __syncthreads();
}

// ------------------------------------------------------------------ host side

struct DeviceInfo {
  bool init = false;
  unsigned long long ctx_id = 0;  // driver id of the context the cached addresses belong to
  int status = FLCE_OK;
  int num_sms = 0;
  int max_pairs = 0;  // CTA pairs of the pair GEMM that fit at once (0 = not yet queried)
  int ce_blocks[4] = {};  // resident CTAs per SM of the CE kernels (0 = not yet queried)
  unsigned* err = nullptr;
};

static std::mutex g_mutex;
static DeviceInfo g_dev[64];
static PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

// Id of the calling thread's current CUDA context, 0 when it has none (for
// instance right after cudaDeviceReset, until the runtime creates a new one),
// kContextUnknown when the driver cannot tell.  Device addresses looked up in
// one context (the error word, the no-allocation scratch array) are stale in
// the next, so they are cached with this id and looked up again when it
// changes; with kContextUnknown the cache is kept.
constexpr unsigned long long kContextUnknown = ~0ull;

static unsigned long long current_context_id() {
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* fn = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(fn);
    fn = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(fn);
  });
  if (get_current == nullptr || get_id == nullptr) return kContextUnknown;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS) return kContextUnknown;
  if (ctx == nullptr) return 0;
  unsigned long long id = 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return kContextUnknown;
  return id;
}

// True when addresses cached in context `cached` must be looked up again.
static bool context_changed(unsigned long long now, unsigned long long cached) {
  return now != kContextUnknown && (now == 0 || now != cached);
}

static int device_info(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return FLCE_ERR_CUDA;
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceInfo& d = g_dev[dev];
  if (d.init && context_changed(ctx, d.ctx_id)) d.init = false;  // a new context: look up again
  if (!d.init) {
    d.init = true;
    d.status = FLCE_OK;
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      d.status = FLCE_ERR_CUDA;
    } else if (major != 10 || minor != 0) {
      d.status = FLCE_ERR_UNSUPPORTED;  // built for sm_100a only
    } else if (cudaGetSymbolAddress(reinterpret_cast<void**>(&d.err), g_device_error) !=
               cudaSuccess) {
      d.status = FLCE_ERR_CUDA;
    }
    if (d.status == FLCE_OK && g_encode == nullptr) {
      cudaDriverEntryPointQueryResult q;
      void* fn = nullptr;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
              cudaSuccess ||
          q != cudaDriverEntryPointSuccess || fn == nullptr)
        d.status = FLCE_ERR_CUDA;
      else
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    // The lookups above made the runtime create the context if it had none.
    d.ctx_id = current_context_id();
  }
  if (d.status != FLCE_OK) {
    d.init = false;  // retry next call (e.g. after the caller fixed the device)
    return d.status;
  }
  *out = &d;
  return FLCE_OK;
}

// ------------------------------------------------------------------ launch accounting
// Every kernel launch is counted; while profiling is on, each launch is also
// bracketed by CUDA events on its stream so a benchmark can report per-kernel
// device time and algorithmic work without a profiler attached.

enum KernelFamily {
  KF_CAST = 0, KF_ZERO, KF_GEMM_FWD, KF_MERGE, KF_FINAL, KF_BWD_PREP, KF_GEMM_GRAD, KF_GEMM_DW,
  KF_GEMM_DH, KF_SELFTEST_GEMM, KF_SELFTEST_WAIT, KF_GEMM_BWD, KF_CE_FWD, KF_CE_BWD, KF_COUNT
};
static const char* const kFamilyNames[KF_COUNT] = {
    "cast_f32_bf16", "zero_rows",     "gemm_fwd_lse", "lse_merge",
    "loss_finalize", "bwd_prep",      "gemm_bwd_grad", "gemm_bwd_dw",
    "gemm_bwd_dh",   "selftest_gemm", "selftest_wait", "gemm_bwd_fused",
    "ce_logits_fwd", "ce_logits_bwd"};

struct ProfRecord {
  int family;
  int device;
  cudaEvent_t start, stop;
  double flops, bytes;
};

static std::atomic<unsigned long long> g_launches{0};
static std::mutex g_prof_mutex;
static bool g_prof_on = false;
static std::vector<ProfRecord> g_prof_records;
static std::vector<cudaEvent_t> g_event_pool[64];

static cudaEvent_t take_event(int dev) {
  if (!g_event_pool[dev].empty()) {
    cudaEvent_t e = g_event_pool[dev].back();
    g_event_pool[dev].pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

// An NVTX range over a host-side scope (an entry point, one launch), so a
// profiler's timeline and its kernel filters can attribute GPU work.
class NvtxRange {
 public:
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

class LaunchScope {
 public:
  LaunchScope(int family, double flops, double bytes, cudaStream_t st)
      : st_(st), range_(kFamilyNames[family]) {
    g_launches.fetch_add(1, std::memory_order_relaxed);
    std::lock_guard<std::mutex> lock(g_prof_mutex);
    if (!g_prof_on) return;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return;
    rec_.family = family;
    rec_.device = dev;
    rec_.flops = flops;
    rec_.bytes = bytes;
    rec_.start = take_event(dev);
    rec_.stop = take_event(dev);
    if (rec_.start && rec_.stop && cudaEventRecord(rec_.start, st_) == cudaSuccess) active_ = true;
  }
  ~LaunchScope() {
    if (!active_) return;
    std::lock_guard<std::mutex> lock(g_prof_mutex);
    if (cudaEventRecord(rec_.stop, st_) == cudaSuccess) g_prof_records.push_back(rec_);
  }

 private:
  cudaStream_t st_;
  NvtxRange range_;
  ProfRecord rec_{};
  bool active_ = false;
};

// 2-D BF16 (or FP32) tensor map, 128-byte swizzle, zero fill outside [inner, outer).
static bool make_tmap(CUtensorMap* tm, const void* base, uint64_t inner, uint64_t outer,
                      uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                      bool f32 = false) {
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = g_encode(tm, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                      : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                              2, const_cast<void*>(base),
                              dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// K-major operand [outer rows][inner K]: one box of 64 K x `rows` rows.
static bool tmap_kmajor(CUtensorMap* tm, const void* base, int64_t k, int64_t rows,
                        int64_t ld_elems, int box_rows) {
  return make_tmap(tm, base, uint64_t(k), uint64_t(rows), uint64_t(ld_elems) * 2, 64,
                   uint32_t(box_rows));
}
// MN-major operand [outer K rows][inner MN]: boxes of 64 MN x 64 K.
static bool tmap_mnmajor(CUtensorMap* tm, const void* base, int64_t mn, int64_t k,
                         int64_t ld_elems) {
  return make_tmap(tm, base, uint64_t(mn), uint64_t(k), uint64_t(ld_elems) * 2, 64, 64);
}
// FP32 B operands for the in-kernel conversion (128-byte rows of 32 values):
// K-major [rows][K] as boxes of 32 K x 128 rows, MN-major [K rows][MN] as boxes
// of 32 MN x 64 K rows.
static bool tmap_kmajor_f32(CUtensorMap* tm, const void* base, int64_t k, int64_t rows,
                            int64_t ld_elems) {
  return make_tmap(tm, base, uint64_t(k), uint64_t(rows), uint64_t(ld_elems) * 4, 32, 128, true);
}
static bool tmap_mnmajor_f32(CUtensorMap* tm, const void* base, int64_t mn, int64_t k,
                             int64_t ld_elems) {
  return make_tmap(tm, base, uint64_t(mn), uint64_t(k), uint64_t(ld_elems) * 4, 32, 64, true);
}

static int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }
static size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// Tile order.  When all of one operand fits in L2 it is kept there (loaded
// with evict_last) and the other streams from HBM once.  Otherwise tiles are
// taken in groups of g rows (or columns) of tiles, the group's index running
// fastest, and g and the orientation are chosen by a model of the HBM bytes
// the operand panels cost:
//   - the grouped operand is read once if the group's panels fit in L2 (and
//     they are then kept with evict_last when the group lasts two waves or
//     more, so later waves find them), else once per wave of the group;
//   - the other operand is read once per group (its panel is shared by the
//     group's g tiles, which run side by side), or once per wave when a wave
//     spans several groups.
// A wave is `pairs` tiles (the resident CTA pairs).
constexpr int64_t kL2ResidentBytes = int64_t(40) << 20;  // a whole operand kept in L2
constexpr int64_t kL2GroupBytes = int64_t(60) << 20;     // one group's panels kept in L2

struct RasterPlan {
  TileRaster raster;
  int a_keep, b_keep;
};

// Modelled HBM bytes of the operand panels for groups of g tiles along the
// grouped operand (tiles_g of them, panel_g bytes each) against tiles_o tiles
// of the other operand (panel_o bytes each).
static double raster_bytes(int64_t tiles_g, int64_t tiles_o, double panel_g, double panel_o,
                           int64_t g, double pairs, bool* keep) {
  const double all_g = panel_g * double(tiles_g), all_o = panel_o * double(tiles_o);
  const double waves_total = double(tiles_g) * double(tiles_o) / pairs;
  const double waves_group = double(g) * double(tiles_o) / pairs;
  const bool fits = double(g) * panel_g <= double(kL2GroupBytes);
  *keep = fits && waves_group >= 2.0;
  const double bytes_g = all_g * (fits ? 1.0 : std::max(1.0, waves_group));
  const double groups = double(cdiv(tiles_g, g));
  const double bytes_o = all_o * std::min(groups, std::max(1.0, waves_total));
  return bytes_g + bytes_o;
}

static RasterPlan make_raster(int64_t m, int64_t n, int64_t k, int pairs) {
  RasterPlan plan{};
  TileRaster& r = plan.raster;
  r.m_tiles = int(cdiv(m, kTileRows));
  r.n_tiles = int(cdiv(n, kBN));
  const int64_t kk = std::max<int64_t>(k, 1);
  const int64_t a_panel = int64_t(kTileRows) * kk * 2, b_panel = int64_t(kBN) * kk * 2;
  const int64_t a_all = a_panel * r.m_tiles, b_all = b_panel * r.n_tiles;
  if (a_all <= kL2ResidentBytes && a_all <= b_all) {
    r.n_fast = 0;
    r.group = r.m_tiles;
    plan.a_keep = 1;
    return plan;
  }
  if (b_all <= kL2ResidentBytes) {
    r.n_fast = 1;
    r.group = r.n_tiles;
    plan.b_keep = 1;
    return plan;
  }
  const double p = double(std::max(pairs, 1));
  double best = -1.0;
  for (int fast = 0; fast < 2; ++fast) {
    const int64_t tg = fast ? r.n_tiles : r.m_tiles, to = fast ? r.m_tiles : r.n_tiles;
    const double pg = double(fast ? b_panel : a_panel), po = double(fast ? a_panel : b_panel);
    for (int64_t g = 1; g <= tg; ++g) {
      bool keep = false;
      const double bytes = raster_bytes(tg, to, pg, po, g, p, &keep);
      if (best < 0.0 || bytes < best * (1.0 - 1e-9)) {
        best = bytes;
        r.n_fast = fast;
        r.group = int(g);
        plan.a_keep = !fast && keep ? 1 : 0;
        plan.b_keep = fast && keep ? 1 : 0;
      }
    }
  }
  return plan;
}

static GemmProblem make_problem(int64_t m, int64_t n, int64_t k, bool a_mn, bool b_mn, int epi,
                                int pairs) {
  GemmProblem p{};
  p.m = m;
  p.n = n;
  p.k = k;
  p.a_mn = a_mn;
  p.b_mn = b_mn;
  p.epi = epi;
  p.num_kb = int(cdiv(k, kBK));
  const RasterPlan rp = make_raster(m, n, k, pairs);
  p.raster = rp.raster;
  p.a_keep = rp.a_keep;
  p.b_keep = rp.b_keep;
  p.tiles = (m > 0 && n > 0) ? int64_t(p.raster.m_tiles) * p.raster.n_tiles : 0;
  return p;
}

// One persistent launch over up to kMaxProblems problems; tiles taken from
// `counter` (zeroed beforehand) when given, else round robin.
// Problem i runs with configuration Ci (its slot is fixed even when it has no
// tiles, so the compile-time configuration always matches).
template <int kKinds, class C0, class C1 = NoProblem, class C2 = NoProblem>
static int launch_group(const GemmProblem* probs, const CUtensorMap* maps_a,
                        const CUtensorMap* maps_b, int count, const EpiSet<kKinds>& ep,
                        unsigned* counter, DeviceInfo& dev, cudaStream_t st, int family,
                        double flops, double bytes) {
  GemmMaps maps;
  GemmGroup g{};
  int64_t total = 0;
  for (int i = 0; i < count; ++i) {
    g.prob[i] = probs[i];
    g.prob[i].tile_begin = total;
    total += probs[i].tiles;
    maps.a[i] = maps_a[i];
    maps.b[i] = maps_b[i];
  }
  g.num_problems = count;
  if (total == 0) return FLCE_OK;
  if (total >= (int64_t(1) << 31)) return FLCE_ERR_UNSUPPORTED;  // the tile counter is 32-bit
  g.total_tiles = total;
  g.tile_counter = counter;
  g.err = dev.err;
  g.timeout_ns = kDefaultTimeoutNs;
  using Layout = PairLayoutOf<C0, C1, C2>;
  auto kern = tc_gemm_pair_kernel<EpiSet<kKinds>, C0, C1, C2>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           int(Layout::kSmemBytes)) != cudaSuccess)
    return FLCE_ERR_CUDA;
  // Pairs that can be resident at once (clusters need two SMs of one GPC);
  // queried once per device: every instantiation takes the same shared memory,
  // which limits it to one CTA per SM whatever its thread count.
  int max_pairs = dev.max_pairs;
  if (max_pairs == 0) {
    cudaLaunchConfig_t q = {};
    q.gridDim = dim3(2 * (dev.num_sms / 2), 1, 1);
    q.blockDim = dim3(Layout::kBlockThreads, 1, 1);
    q.dynamicSmemBytes = Layout::kSmemBytes;
    cudaLaunchAttribute qa[1];
    qa[0].id = cudaLaunchAttributeClusterDimension;
    qa[0].val.clusterDim.x = 2;
    qa[0].val.clusterDim.y = 1;
    qa[0].val.clusterDim.z = 1;
    q.attrs = qa;
    q.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &q) != cudaSuccess || n <= 0)
      n = dev.num_sms / 2;
    max_pairs = std::min(n, dev.num_sms / 2);
    std::lock_guard<std::mutex> lock(g_mutex);
    dev.max_pairs = max_pairs;
  }
  const int pairs = int(std::min<int64_t>(max_pairs, total));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cfg.blockDim = dim3(Layout::kBlockThreads, 1, 1);
  cfg.dynamicSmemBytes = Layout::kSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  // Programmatic dependent launch: the kernel's set-up may overlap the tail of
  // the previous kernel in the stream; it waits (griddepcontrol.wait) before
  // reading or writing anything else.
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  LaunchScope scope(family, flops, bytes, st);
  if (cudaLaunchKernelEx(&cfg, kern, maps, g, ep) != cudaSuccess) return FLCE_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? FLCE_OK : FLCE_ERR_CUDA;
}

static int launch_zero(void* p, size_t bytes, const DeviceInfo& dev, cudaStream_t st) {
  if (bytes == 0) return FLCE_OK;
  const int64_t n16 = int64_t(bytes / 16);
  const int grid = int(std::min<int64_t>(int64_t(dev.num_sms) * 8, cdiv(n16, 256)));
  LaunchScope scope(KF_ZERO, 0.0, double(bytes), st);
  zero16_kernel<<<std::max(grid, 1), 256, 0, st>>>(static_cast<uint4*>(p), n16);
  return cudaGetLastError() == cudaSuccess ? FLCE_OK : FLCE_ERR_CUDA;
}

static int launch_cast(const float* src, __nv_bfloat16* dst, int64_t elems,
                       const DeviceInfo& dev, cudaStream_t st) {
  const int64_t n8 = elems / 8;
  if (n8 == 0) return FLCE_OK;
  const int grid = int(std::min<int64_t>(int64_t(dev.num_sms) * 8, cdiv(n8, 256)));
  LaunchScope scope(KF_CAST, 0.0, double(elems) * 6.0, st);
  cast_f32_to_bf16_kernel<<<grid, 256, 0, st>>>(reinterpret_cast<const float4*>(src),
                                                reinterpret_cast<uint4*>(dst), n8);
  return cudaGetLastError() == cudaSuccess ? FLCE_OK : FLCE_ERR_CUDA;
}

// ---------------------------------------------------------------- planning

struct Shape {
  int64_t n, h, vp, v;
  int w_dtype;
  int fused_cast;  // 1: an FP32 head is rounded inside the GEMMs; no BF16 copy
};

struct FwdPlan {
  int64_t v_tiles, nblk;
  size_t off_pm, off_ps, off_zl, off_bl, off_bc, off_cnt, off_wb, total;
};

struct BwdPlan {
  int64_t vc;  // vocabulary chunk width (multiple of 256)
  int64_t n_counters;
  size_t off_lse2, off_scale, off_cnt, off_dh32, off_wb, off_g, fixed, total;
};

// Both plans put the BF16 copy of an FP32 head at offset 0, so a backward
// given the forward's workspace finds the copy the forward wrote there
// (flce_backward_ex with FLCE_BWD_HEAD_COPY_VALID).
static size_t head_copy_bytes(const Shape& s) {
  return s.w_dtype == FLCE_F32 && !s.fused_cast ? align_up(size_t(s.v) * s.h * 2) : 0;
}

static FwdPlan plan_forward(const Shape& s) {
  FwdPlan p{};
  p.v_tiles = cdiv(s.v, kBN);
  p.nblk = cdiv(s.n, kMergeRows);
  p.off_wb = 0;
  size_t o = head_copy_bytes(s);
  p.off_pm = o;  o = align_up(o + size_t(p.v_tiles) * s.n * 4);
  p.off_ps = o;  o = align_up(o + size_t(p.v_tiles) * s.n * 4);
  p.off_zl = o;  o = align_up(o + size_t(s.n) * 4);
  p.off_bl = o;  o = align_up(o + size_t(p.nblk) * 8);
  p.off_bc = o;  o = align_up(o + size_t(p.nblk) * 4);
  p.off_cnt = o; o = align_up(o + 4);  // the projection GEMM's tile counter
  p.total = std::max(o, kAlign);  // never zero, so N = 0 still has a valid buffer
  return p;
}

static int64_t default_chunk(const Shape& s) {
  const int64_t cap = cdiv(cdiv(s.v, 5), kBN) * kBN;  // at most a fifth of the vocabulary
  int64_t budget = int64_t(kChunkBudgetBytes / (2 * size_t(std::max<int64_t>(s.n, 1))));
  budget = budget / kBN * kBN;
  return std::max<int64_t>(kBN, std::min(cap, std::max(kMinChunk, budget)));
}

static BwdPlan plan_backward(const Shape& s, int64_t vc) {
  BwdPlan p{};
  p.vc = vc;
  p.off_wb = 0;
  size_t o = head_copy_bytes(s);
  p.off_lse2 = o;  o = align_up(o + size_t(s.n) * 4);
  p.off_scale = o; o = align_up(o + size_t(s.n) * 4);
  p.n_counters = cdiv(s.v, kBN) + 2;  // one per launch at the narrowest chunking
  p.off_cnt = o;   o = align_up(o + size_t(p.n_counters) * 4);
  p.off_dh32 = o;  o = align_up(o + size_t(s.n) * s.h * 4);
  p.fixed = o;
  p.off_g = o;     o = align_up(o + 2 * size_t(s.n) * vc * 2);  // two chunk buffers
  p.total = o;
  return p;
}

static bool shape_ok(int64_t n, int64_t h, int64_t vp, int64_t v, int w_dtype) {
  if (n < 0 || h <= 0 || vp <= 0) return false;
  if (h % 8 != 0) return false;
  if (v <= 0 || v > vp) return false;
  if (n > kMaxDim || h > kMaxDim || vp > kMaxDim) return false;
  if (w_dtype != FLCE_BF16 && w_dtype != FLCE_F32) return false;
  return true;
}

static bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

static int check_common(const void* hidden, const void* weight, int w_dtype,
                        const int64_t* labels, int64_t n, int64_t h, int64_t vp, int64_t v,
                        float softcap, int reduction, int64_t num_label_tokens) {
  if (!shape_ok(n, h, vp, v, w_dtype)) return FLCE_ERR_INVALID_ARG;
  if (!(softcap >= 0.0f) || !std::isfinite(softcap)) return FLCE_ERR_INVALID_ARG;
  if (reduction != FLCE_SUM && reduction != FLCE_MEAN && reduction != FLCE_NONE)
    return FLCE_ERR_INVALID_ARG;
  if (num_label_tokens > 0 && reduction != FLCE_SUM) return FLCE_ERR_INVALID_ARG;
  if (weight == nullptr || !aligned(weight, 16)) return FLCE_ERR_INVALID_ARG;
  if (n > 0) {
    if (hidden == nullptr || labels == nullptr) return FLCE_ERR_INVALID_ARG;
    if (!aligned(hidden, 16) || !aligned(labels, 8)) return FLCE_ERR_INVALID_ARG;
  }
  return FLCE_OK;
}

}  // namespace flce

using namespace flce;

// ====================================================================== C ABI

extern "C" size_t flce_workspace_size_ex(int64_t n, int64_t h, int64_t vp, int64_t unpadded,
                                         int w_dtype, unsigned int flags) {
  const int64_t v = unpadded <= 0 ? vp : unpadded;
  if (!shape_ok(n, h, vp, v, w_dtype) || (flags & ~FLCE_FUSED_HEAD_CAST) != 0u) return 0;
  const Shape s{n, h, vp, v, w_dtype, (flags & FLCE_FUSED_HEAD_CAST) ? 1 : 0};
  return std::max(plan_forward(s).total, plan_backward(s, default_chunk(s)).total);
}

extern "C" size_t flce_workspace_size(int64_t n, int64_t h, int64_t vp, int64_t unpadded,
                                      int w_dtype) {
  return flce_workspace_size_ex(n, h, vp, unpadded, w_dtype, 0u);
}

extern "C" size_t flce_workspace_min_size_ex(int64_t n, int64_t h, int64_t vp, int64_t unpadded,
                                             int w_dtype, unsigned int flags) {
  const int64_t v = unpadded <= 0 ? vp : unpadded;
  if (!shape_ok(n, h, vp, v, w_dtype) || (flags & ~FLCE_FUSED_HEAD_CAST) != 0u) return 0;
  const Shape s{n, h, vp, v, w_dtype, (flags & FLCE_FUSED_HEAD_CAST) ? 1 : 0};
  return std::max(plan_forward(s).total, plan_backward(s, kBN).total);
}

extern "C" size_t flce_workspace_min_size(int64_t n, int64_t h, int64_t vp, int64_t unpadded,
                                          int w_dtype) {
  return flce_workspace_min_size_ex(n, h, vp, unpadded, w_dtype, 0u);
}

extern "C" double flce_flops_fwd_bwd(int64_t n, int64_t h, int64_t v) {
  return 8.0 * double(n) * double(v) * double(h);
}

extern "C" const char* flce_status_string(int status) {
  switch (status) {
    case FLCE_OK: return "ok";
    case FLCE_ERR_INVALID_ARG: return "invalid argument";
    case FLCE_ERR_WORKSPACE: return "workspace missing or too small";
    case FLCE_ERR_UNSUPPORTED: return "unsupported device or size (needs sm_100)";
    case FLCE_ERR_CUDA: return "CUDA runtime error";
    case FLCE_ERR_BAD_LABEL: return "label outside [0, unpadded_vocab) that is not ignore_index";
    case FLCE_ERR_TIMEOUT: return "a pipeline wait timed out";
    default: return "unknown status";
  }
}

extern "C" int flce_forward_ex(const void* hidden, const void* weight, int w_dtype,
                               const int64_t* labels, int64_t n, int64_t h, int64_t vp,
                               int64_t unpadded, int64_t ignore_index, float softcap,
                               int reduction, int64_t num_label_tokens, float* loss, float* lse,
                               void* workspace, size_t ws_bytes, unsigned int flags,
                               flce_stream_t stream) {
  NvtxRange range("flce_forward");
  const int64_t v = unpadded <= 0 ? vp : unpadded;
  if ((flags & ~FLCE_FUSED_HEAD_CAST) != 0u) return FLCE_ERR_INVALID_ARG;
  const bool fused = (flags & FLCE_FUSED_HEAD_CAST) != 0u && w_dtype == FLCE_F32;
  int st = check_common(hidden, weight, w_dtype, labels, n, h, vp, v, softcap, reduction,
                        num_label_tokens);
  if (st != FLCE_OK) return st;
  if ((n > 0 || reduction != FLCE_NONE) && (loss == nullptr || !aligned(loss, 4)))
    return FLCE_ERR_INVALID_ARG;
  if (n > 0 && (lse == nullptr || !aligned(lse, 4))) return FLCE_ERR_INVALID_ARG;
  const Shape s{n, h, vp, v, w_dtype, fused ? 1 : 0};
  const FwdPlan p = plan_forward(s);
  if (workspace == nullptr || !aligned(workspace, 16) || ws_bytes < p.total)
    return FLCE_ERR_WORKSPACE;
  DeviceInfo* dev = nullptr;
  if ((st = device_info(&dev)) != FLCE_OK) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  double* blk_loss = reinterpret_cast<double*>(ws + p.off_bl);
  int* blk_cnt = reinterpret_cast<int*>(ws + p.off_bc);

  if (n == 0) {
    if (reduction == FLCE_NONE) return FLCE_OK;
    LaunchScope scope(KF_FINAL, 0.0, 4.0, cs);
    loss_finalize_kernel<<<1, kFinalThreads, 0, cs>>>(blk_loss, blk_cnt, 0, reduction,
                                                      num_label_tokens, loss);
    return cudaGetLastError() == cudaSuccess ? FLCE_OK : FLCE_ERR_CUDA;
  }

  const void* wb = weight;
  if (w_dtype == FLCE_F32 && !fused) {
    wb = ws + p.off_wb;
    if ((st = launch_cast(static_cast<const float*>(weight),
                          reinterpret_cast<__nv_bfloat16*>(ws + p.off_wb), v * h, *dev, cs)) !=
        FLCE_OK)
      return st;
  }

  CUtensorMap ta, tb;
  if (!tmap_kmajor(&ta, hidden, h, n, h, kBM) ||
      !(fused ? tmap_kmajor_f32(&tb, weight, h, v, h) : tmap_kmajor(&tb, wb, h, v, h, kBBoxRows)))
    return FLCE_ERR_CUDA;
  const GemmProblem prob = make_problem(n, v, h, false, false, kEpiForward, dev->num_sms / 2);
  EpiSet<kEpiSetForward> es{};
  EpiForward::Params& ep = es.fwd;
  ep.labels = labels;
  ep.n_tokens = n;
  ep.vocab = v;
  ep.softcap = softcap;
  ep.softcap_k = softcap > 0.0f ? 2.0f * kLog2e / softcap : 0.0f;
  ep.part_m = reinterpret_cast<float*>(ws + p.off_pm);
  ep.part_s = reinterpret_cast<float*>(ws + p.off_ps);
  ep.label_logit = reinterpret_cast<float*>(ws + p.off_zl);
  const double fwd_flops = 2.0 * double(n) * double(v) * double(h);
  const double fwd_bytes = 2.0 * (double(n) + double(v)) * double(h) + 8.0 * double(p.v_tiles) * n;
  // Tiles are taken from a counter (zeroed here, in stream order), so pairs that
  // run slower take fewer tiles and the launch does not wait on the slowest one.
  unsigned* counter = reinterpret_cast<unsigned*>(ws + p.off_cnt);
  if (cudaMemsetAsync(counter, 0, sizeof(unsigned), cs) != cudaSuccess) return FLCE_ERR_CUDA;
  st = fused ? launch_group<kEpiSetForward, ProblemCfg<false, false, kEpiForward, true>>(
                   &prob, &ta, &tb, 1, es, counter, *dev, cs, KF_GEMM_FWD, fwd_flops,
                   fwd_bytes + 2.0 * double(v) * double(h))
             : launch_group<kEpiSetForward, ProblemCfg<false, false, kEpiForward>>(
                   &prob, &ta, &tb, 1, es, counter, *dev, cs, KF_GEMM_FWD, fwd_flops,
                   fwd_bytes);
  if (st != FLCE_OK) return st;
  {
    LaunchScope scope(KF_MERGE, 0.0, 8.0 * double(p.v_tiles) * n + 24.0 * n, cs);
    lse_merge_kernel<<<int(p.nblk), kMergeRows * kMergeWarps, 0, cs>>>(
        ep.part_m, ep.part_s, int(p.v_tiles), n, ep.label_logit, labels, nullptr, v,
        ignore_index, lse, reduction == FLCE_NONE ? loss : nullptr, blk_loss, blk_cnt, dev->err);
  }
  if (cudaGetLastError() != cudaSuccess) return FLCE_ERR_CUDA;
  if (reduction != FLCE_NONE) {
    LaunchScope scope(KF_FINAL, 0.0, 12.0 * double(p.nblk), cs);
    loss_finalize_kernel<<<1, kFinalThreads, 0, cs>>>(blk_loss, blk_cnt, int(p.nblk), reduction,
                                                      num_label_tokens, loss);
    if (cudaGetLastError() != cudaSuccess) return FLCE_ERR_CUDA;
  }
  return FLCE_OK;
}

extern "C" int flce_forward(const void* hidden, const void* weight, int w_dtype,
                            const int64_t* labels, int64_t n, int64_t h, int64_t vp,
                            int64_t unpadded, int64_t ignore_index, float softcap, int reduction,
                            int64_t num_label_tokens, float* loss, float* lse, void* workspace,
                            size_t ws_bytes, flce_stream_t stream) {
  return flce_forward_ex(hidden, weight, w_dtype, labels, n, h, vp, unpadded, ignore_index,
                         softcap, reduction, num_label_tokens, loss, lse, workspace, ws_bytes, 0u,
                         stream);
}

extern "C" int flce_backward_ex(const void* hidden, const void* weight, int w_dtype,
                                const int64_t* labels, int64_t n, int64_t h, int64_t vp,
                                int64_t unpadded, int64_t ignore_index, float softcap,
                                int reduction, int64_t num_label_tokens, const float* grad_loss,
                                const float* lse, void* dhidden, void* dweight, void* workspace,
                                size_t ws_bytes, unsigned int flags, flce_stream_t stream) {
  NvtxRange range("flce_backward");
  const int64_t v = unpadded <= 0 ? vp : unpadded;
  int st = check_common(hidden, weight, w_dtype, labels, n, h, vp, v, softcap, reduction,
                        num_label_tokens);
  if (st != FLCE_OK) return st;
  if ((flags & ~(FLCE_BWD_HEAD_COPY_VALID | FLCE_FUSED_HEAD_CAST)) != 0u ||
      (flags & (FLCE_BWD_HEAD_COPY_VALID | FLCE_FUSED_HEAD_CAST)) ==
          (FLCE_BWD_HEAD_COPY_VALID | FLCE_FUSED_HEAD_CAST))
    return FLCE_ERR_INVALID_ARG;
  const bool fused = (flags & FLCE_FUSED_HEAD_CAST) != 0u && w_dtype == FLCE_F32;
  if (dweight == nullptr || !aligned(dweight, 16)) return FLCE_ERR_INVALID_ARG;
  if (n > 0) {
    if (grad_loss == nullptr || lse == nullptr || dhidden == nullptr) return FLCE_ERR_INVALID_ARG;
    if (!aligned(grad_loss, 4) || !aligned(lse, 4) || !aligned(dhidden, 16))
      return FLCE_ERR_INVALID_ARG;
  }
  const Shape s{n, h, vp, v, w_dtype, fused ? 1 : 0};
  const BwdPlan p0 = plan_backward(s, kBN);
  if (workspace == nullptr || !aligned(workspace, 16) || ws_bytes < p0.total)
    return FLCE_ERR_WORKSPACE;
  // Widest chunk that fits the workspace, up to the default.
  int64_t vc = default_chunk(s);
  if (n > 0) {
    // two chunk buffers of n x vc BF16
    const int64_t fit = int64_t((ws_bytes - p0.fixed) / (4 * size_t(n))) / kBN * kBN;
    vc = std::max<int64_t>(kBN, std::min(vc, fit));
  }
  const BwdPlan p = plan_backward(s, vc);
  if (ws_bytes < p.total) return FLCE_ERR_WORKSPACE;
  DeviceInfo* dev = nullptr;
  if ((st = device_info(&dev)) != FLCE_OK) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const size_t wsz = w_dtype == FLCE_F32 ? 4 : 2;

  // Rows the softmax never sees get exactly zero gradient; with no tokens, all rows.
  const int64_t zero_from = n == 0 ? 0 : v;
  if ((st = launch_zero(static_cast<uint8_t*>(dweight) + size_t(zero_from) * h * wsz,
                        size_t(vp - zero_from) * h * wsz, *dev, cs)) != FLCE_OK)
    return st;
  if (n == 0) return FLCE_OK;

  const void* wb = weight;
  if (w_dtype == FLCE_F32 && !fused) {
    wb = ws + p.off_wb;
    // The caller vouches that the copy at offset 0 still holds bf16(weight[:V])
    // (written by flce_forward on this workspace and unchanged since).
    if ((flags & FLCE_BWD_HEAD_COPY_VALID) == 0u &&
        (st = launch_cast(static_cast<const float*>(weight),
                          reinterpret_cast<__nv_bfloat16*>(ws + p.off_wb), v * h, *dev, cs)) !=
            FLCE_OK)
      return st;
  }
  float* lse2 = reinterpret_cast<float*>(ws + p.off_lse2);
  float* scale = reinterpret_cast<float*>(ws + p.off_scale);
  float* dh32 = reinterpret_cast<float*>(ws + p.off_dh32);
  unsigned* counters = reinterpret_cast<unsigned*>(ws + p.off_cnt);
  __nv_bfloat16* gbufs[2] = {reinterpret_cast<__nv_bfloat16*>(ws + p.off_g),
                             reinterpret_cast<__nv_bfloat16*>(ws + p.off_g) + size_t(n) * vc};
  // The chunk buffers' rows are vc x 2 bytes apart (vc % 256 == 0), so both
  // buffers take 32-byte stores when the first starts 32-byte aligned.
  const int g_v8 = aligned(gbufs[0], 32) ? 1 : 0;
  {
    LaunchScope prep_scope(KF_BWD_PREP, 0.0, 24.0 * double(n), cs);
    bwd_prep_kernel<<<1, 1024, 0, cs>>>(labels, nullptr, n, v, ignore_index, reduction,
                                        num_label_tokens,
                                        grad_loss, lse, lse2, scale, counters,
                                        int(p.n_counters), dev->err);
  }
  if (cudaGetLastError() != cudaSuccess) return FLCE_ERR_CUDA;

  CUtensorMap t_hid_k, t_w_k, t_hid_mn, t_w_mn;
  if (!tmap_kmajor(&t_hid_k, hidden, h, n, h, kBM) || !tmap_mnmajor(&t_hid_mn, hidden, h, n, h))
    return FLCE_ERR_CUDA;
  if (fused ? !tmap_kmajor_f32(&t_w_k, weight, h, v, h) || !tmap_mnmajor_f32(&t_w_mn, weight, h, v, h)
            : !tmap_kmajor(&t_w_k, wb, h, v, h, kBBoxRows) || !tmap_mnmajor(&t_w_mn, wb, h, v, h))
    return FLCE_ERR_CUDA;

  // The head's GEMMs (recompute: B = W K-major; dhidden: B = W MN-major) take
  // it as FP32 and round it in the kernel when `fused`.
  using CfgDw = ProblemCfg<true, true, kEpiStoreRows>;
  auto launch_grad = [&](const GemmProblem* pr, const CUtensorMap* ma, const CUtensorMap* mb,
                         const EpiSet<kEpiSetBackward>& es, unsigned* cnt, double fl,
                         double by) {
    return fused ? launch_group<kEpiSetBackward, ProblemCfg<false, false, kEpiGrad, true>>(
                       pr, ma, mb, 1, es, cnt, *dev, cs, KF_GEMM_GRAD, fl, by)
                 : launch_group<kEpiSetBackward, ProblemCfg<false, false, kEpiGrad>>(
                       pr, ma, mb, 1, es, cnt, *dev, cs, KF_GEMM_GRAD, fl, by);
  };
  auto launch_fused_bwd = [&](const GemmProblem* pr, const CUtensorMap* ma,
                              const CUtensorMap* mb, int count,
                              const EpiSet<kEpiSetBackward>& es, unsigned* cnt, double fl,
                              double by) {
    return fused ? launch_group<kEpiSetBackward, ProblemCfg<false, true, kEpiAccumRows, true>,
                                CfgDw, ProblemCfg<false, false, kEpiGrad, true>>(
                       pr, ma, mb, count, es, cnt, *dev, cs, KF_GEMM_BWD, fl, by)
                 : launch_group<kEpiSetBackward, ProblemCfg<false, true, kEpiAccumRows>, CfgDw,
                                ProblemCfg<false, false, kEpiGrad>>(
                       pr, ma, mb, count, es, cnt, *dev, cs, KF_GEMM_BWD, fl, by);
  };
  const double w_extra = fused ? 2.0 : 0.0;  // FP32 head bytes beyond the BF16 ones
  const int64_t chunks = cdiv(v, vc);
  auto chunk_v0 = [&](int64_t c) { return c * vc; };
  auto chunk_width = [&](int64_t c) { return std::min(vc, v - c * vc); };
  auto chunk_gcols = [&](int64_t c) { return cdiv(chunk_width(c), kBN) * kBN; };
  const float softcap_k = softcap > 0.0f ? 2.0f * kLog2e / softcap : 0.0f;

  // K3 for chunk c: problem, maps and epilogue parameters.
  auto grad_problem = [&](int64_t c, GemmProblem* pr, CUtensorMap* ma, CUtensorMap* mb,
                          EpiGrad::Params* ep) {
    *pr = make_problem(n, chunk_width(c), h, false, false, kEpiGrad, dev->num_sms / 2);
    pr->b_mn_off = int(chunk_v0(c));
    *ma = t_hid_k;
    *mb = t_w_k;
    ep->labels = labels;
    ep->n_tokens = n;
    ep->vocab = v;
    ep->v0 = chunk_v0(c);
    ep->softcap = softcap;
    ep->softcap_k = softcap_k;
    ep->lse2 = lse2;
    ep->scale = scale;
    ep->g = gbufs[c & 1];
    ep->ldg = vc;
    ep->v8 = g_v8;
  };
  auto grad_flops = [&](int64_t c) { return 2.0 * double(n) * double(chunk_width(c)) * double(h); };
  auto grad_bytes = [&](int64_t c) {
    return 2.0 * (double(n) + double(chunk_width(c))) * double(h) +
           w_extra * double(chunk_width(c)) * double(h) + 2.0 * double(n) * double(chunk_gcols(c));
  };

  {  // K3 of the first chunk on its own
    GemmProblem pr;
    CUtensorMap ma, mb;
    EpiSet<kEpiSetBackward> es{};
    grad_problem(0, &pr, &ma, &mb, &es.grad);
    if ((st = launch_grad(&pr, &ma, &mb, es, &counters[0], grad_flops(0), grad_bytes(0))) !=
        FLCE_OK)
      return st;
  }
  for (int64_t c = 0; c < chunks; ++c) {
    const int64_t v0 = chunk_v0(c), width = chunk_width(c), gcols = chunk_gcols(c);
    __nv_bfloat16* gbuf = gbufs[c & 1];
    CUtensorMap t_g_mn, t_g_k;
    if (!tmap_mnmajor(&t_g_mn, gbuf, gcols, n, vc) || !tmap_kmajor(&t_g_k, gbuf, gcols, n, vc, kBM))
      return FLCE_ERR_CUDA;
    GemmProblem pr[3];
    CUtensorMap ma[3], mb[3];
    EpiSet<kEpiSetBackward> es{};
    int count = 0;
    double flops = 0.0, bytes = 0.0;
    // K5: dhidden (+)= G . W[v0 : v0 + width]  (contraction over the chunk; long tiles first)
    pr[count] = make_problem(n, h, gcols, false, true, kEpiAccumRows, dev->num_sms / 2);
    pr[count].b_k_off = int(v0);
    ma[count] = t_g_k;
    mb[count] = t_w_mn;
    es.accum.acc32 = dh32;
    es.accum.out = static_cast<__nv_bfloat16*>(dhidden);
    es.accum.ld = h;
    es.accum.rows = n;
    es.accum.cols = h;
    es.accum.mode = chunks == 1 ? 3 : (c == 0 ? 0 : (c == chunks - 1 ? 2 : 1));
    es.accum.v8 = aligned(dh32, 32) ? 1 : 0;  // rows are H x 4 bytes apart, H % 8 == 0
    {
      const double rmw = es.accum.mode == 0 ? 4.0 : (es.accum.mode == 1 ? 8.0 : (es.accum.mode == 2 ? 6.0 : 2.0));
      flops += 2.0 * double(n) * double(width) * double(h);
      bytes += 2.0 * double(n) * gcols + (2.0 + w_extra) * double(width) * h +
               rmw * double(n) * h;
    }
    ++count;
    // K4: dW[v0 : v0 + width] = G^T . hidden  (contraction over tokens)
    pr[count] = make_problem(width, h, n, true, true, kEpiStoreRows, dev->num_sms / 2);
    ma[count] = t_g_mn;
    mb[count] = t_hid_mn;
    es.store.out = static_cast<uint8_t*>(dweight) + size_t(v0) * h * wsz;
    es.store.ldo = h;
    es.store.rows = width;
    es.store.cols = h;
    es.store.f32 = w_dtype == FLCE_F32;
    es.store.v8 = aligned(es.store.out, 32) && (size_t(h) * wsz) % 32 == 0 ? 1 : 0;
    flops += 2.0 * double(n) * double(width) * double(h);
    bytes += 2.0 * double(n) * (double(gcols) + double(h)) + double(wsz) * width * h;
    ++count;
    // K3 of the next chunk into the other G buffer
    if (c + 1 < chunks) {
      grad_problem(c + 1, &pr[count], &ma[count], &mb[count], &es.grad);
      flops += grad_flops(c + 1);
      bytes += grad_bytes(c + 1);
      ++count;
    }
    if ((st = launch_fused_bwd(pr, ma, mb, count, es, &counters[c + 1], flops, bytes)) !=
        FLCE_OK)
      return st;
  }
  return FLCE_OK;
}

extern "C" int flce_backward(const void* hidden, const void* weight, int w_dtype,
                             const int64_t* labels, int64_t n, int64_t h, int64_t vp,
                             int64_t unpadded, int64_t ignore_index, float softcap,
                             int reduction, int64_t num_label_tokens, const float* grad_loss,
                             const float* lse, void* dhidden, void* dweight, void* workspace,
                             size_t ws_bytes, flce_stream_t stream) {
  return flce_backward_ex(hidden, weight, w_dtype, labels, n, h, vp, unpadded, ignore_index,
                          softcap, reduction, num_label_tokens, grad_loss, lse, dhidden, dweight,
                          workspace, ws_bytes, 0u, stream);
}

extern "C" int flce_get_error(flce_stream_t stream) {
  DeviceInfo* dev = nullptr;
  int st = device_info(&dev);
  if (st != FLCE_OK) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  unsigned host = 0;
  if (cudaMemcpyAsync(&host, dev->err, sizeof(unsigned), cudaMemcpyDeviceToHost, cs) !=
          cudaSuccess ||
      cudaMemsetAsync(dev->err, 0, sizeof(unsigned), cs) != cudaSuccess ||
      cudaStreamSynchronize(cs) != cudaSuccess)
    return FLCE_ERR_CUDA;
  if (host & kDevErrTimeout) return FLCE_ERR_TIMEOUT;
  if (host & kDevErrBadLabel) return FLCE_ERR_BAD_LABEL;
  return FLCE_OK;
}

extern "C" int flce_selftest_gemm(const void* a, const void* b, float* d, int64_t m, int64_t n,
                                  int64_t k, int a_mn, int b_mn, flce_stream_t stream) {
  if (a == nullptr || b == nullptr || d == nullptr || m <= 0 || n <= 0 || k <= 0)
    return FLCE_ERR_INVALID_ARG;
  if (m > kMaxDim || n > kMaxDim || k > kMaxDim) return FLCE_ERR_INVALID_ARG;
  if (n % 8 != 0 || (a_mn ? m % 8 : k % 8) != 0 || (b_mn ? n % 8 : k % 8) != 0)
    return FLCE_ERR_INVALID_ARG;
  if (!aligned(a, 16) || !aligned(b, 16) || !aligned(d, 16)) return FLCE_ERR_INVALID_ARG;
  DeviceInfo* dev = nullptr;
  int st = device_info(&dev);
  if (st != FLCE_OK) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  CUtensorMap ta, tb;
  const bool ok_a = a_mn ? tmap_mnmajor(&ta, a, m, k, m) : tmap_kmajor(&ta, a, k, m, k, kBM);
  const bool ok_b = b_mn ? tmap_mnmajor(&tb, b, n, k, n) : tmap_kmajor(&tb, b, k, n, k, kBBoxRows);
  if (!ok_a || !ok_b) return FLCE_ERR_CUDA;
  const GemmProblem prob = make_problem(m, n, k, a_mn != 0, b_mn != 0, kEpiStoreRows,
                                        dev->num_sms / 2);
  EpiSet<kEpiSetStore> es{};
  EpiStoreRows::Params& ep = es.store;
  ep.out = d;
  ep.ldo = n;
  ep.rows = m;
  ep.cols = n;
  ep.f32 = 1;
  ep.v8 = aligned(d, 32) ? 1 : 0;  // rows are n x 4 bytes apart, n % 8 == 0
  const double fl = 2.0 * double(m) * double(n) * double(k);
  const double by = 2.0 * (double(m) + double(n)) * double(k) + 4.0 * double(m) * n;
  const int f = KF_SELFTEST_GEMM;
  if (!a_mn && !b_mn)
    return launch_group<kEpiSetStore, ProblemCfg<false, false, kEpiStoreRows>>(
        &prob, &ta, &tb, 1, es, nullptr, *dev, cs, f, fl, by);
  if (!a_mn && b_mn)
    return launch_group<kEpiSetStore, ProblemCfg<false, true, kEpiStoreRows>>(
        &prob, &ta, &tb, 1, es, nullptr, *dev, cs, f, fl, by);
  if (a_mn && !b_mn)
    return launch_group<kEpiSetStore, ProblemCfg<true, false, kEpiStoreRows>>(
        &prob, &ta, &tb, 1, es, nullptr, *dev, cs, f, fl, by);
  return launch_group<kEpiSetStore, ProblemCfg<true, true, kEpiStoreRows>>(
      &prob, &ta, &tb, 1, es, nullptr, *dev, cs, f, fl, by);
}

extern "C" int flce_selftest_wait_timeout(unsigned int timeout_us, flce_stream_t stream) {
  if (timeout_us == 0 || timeout_us > 2000000u) return FLCE_ERR_INVALID_ARG;
  DeviceInfo* dev = nullptr;
  int st = device_info(&dev);
  if (st != FLCE_OK) return st;
  LaunchScope scope(KF_SELFTEST_WAIT, 0.0, 0.0, static_cast<cudaStream_t>(stream));
  wait_timeout_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      dev->err, uint64_t(timeout_us) * 1000ull);
  return cudaGetLastError() == cudaSuccess ? FLCE_OK : FLCE_ERR_CUDA;
}

extern "C" unsigned long long flce_launch_count(void) {
  return g_launches.load(std::memory_order_relaxed);
}

extern "C" int flce_profile_start(void) {
  std::lock_guard<std::mutex> lock(g_prof_mutex);
  if (g_prof_on) return FLCE_ERR_INVALID_ARG;
  g_prof_on = true;
  return FLCE_OK;
}

extern "C" int flce_profile_stop(flce_kernel_stat* stats, int capacity, int* count) {
  std::vector<ProfRecord> recs;
  {
    std::lock_guard<std::mutex> lock(g_prof_mutex);
    if (!g_prof_on) return FLCE_ERR_INVALID_ARG;
    g_prof_on = false;
    recs.swap(g_prof_records);
  }
  double ms[KF_COUNT] = {0}, fl[KF_COUNT] = {0}, by[KF_COUNT] = {0};
  int64_t nl[KF_COUNT] = {0};
  int status = FLCE_OK;
  for (const ProfRecord& r : recs) {
    float t = 0.0f;
    if (cudaEventSynchronize(r.stop) != cudaSuccess ||
        cudaEventElapsedTime(&t, r.start, r.stop) != cudaSuccess)
      status = FLCE_ERR_CUDA;
    ms[r.family] += t;
    fl[r.family] += r.flops;
    by[r.family] += r.bytes;
    nl[r.family] += 1;
  }
  {
    std::lock_guard<std::mutex> lock(g_prof_mutex);
    for (const ProfRecord& r : recs) {
      g_event_pool[r.device].push_back(r.start);
      g_event_pool[r.device].push_back(r.stop);
    }
  }
  int k = 0;
  for (int f = 0; f < KF_COUNT; ++f) {
    if (nl[f] == 0) continue;
    if (stats != nullptr && k < capacity) {
      std::memset(&stats[k], 0, sizeof(flce_kernel_stat));
      std::strncpy(stats[k].name, kFamilyNames[f], sizeof(stats[k].name) - 1);
      stats[k].launches = nl[f];
      stats[k].total_ms = ms[f];
      stats[k].flops = fl[f];
      stats[k].bytes = by[f];
    }
    ++k;
  }
  if (count) *count = k;
  return status;
}

// ================================================== forward without allocation
//
// For callers that cannot hand this library any device memory of their own
// beyond inputs and outputs: for example a plugin running inside another
// framework whose allocator owns the whole device and offers no scratch API,
// or a service that forbids device allocations after start-up because one
// that fails mid-run cannot be recovered.  The forward's scratch (per-tile
// logsumexp partials, the label logits and the loss block sums) then lives in
// a fixed array in this library's own device memory instead of a workspace.

namespace flce {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB on every device
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];
static std::mutex g_noalloc_mutex;
static void* g_noalloc_addr[64];  // device address of g_noalloc_scratch, per device
static unsigned long long g_noalloc_ctx[64];  // context that address belongs to

}  // namespace flce

extern "C" int flce_forward_noalloc(const void* hidden, const void* weight, int w_dtype,
                                    const int64_t* labels, int64_t n, int64_t h, int64_t vp,
                                    int64_t unpadded, int64_t ignore_index, float softcap,
                                    int reduction, int64_t num_label_tokens, float* loss,
                                    float* lse, flce_stream_t stream) {
  NvtxRange range("flce_forward_noalloc");
  const int64_t v = unpadded <= 0 ? vp : unpadded;
  if (!shape_ok(n, h, vp, v, w_dtype)) return FLCE_ERR_INVALID_ARG;
  // An FP32 head is rounded inside the GEMM (no BF16 copy), so the scratch is
  // the same as for a BF16 head; it must fit the fixed array, which nothing
  // here can grow.
  const unsigned flags = w_dtype == FLCE_F32 ? FLCE_FUSED_HEAD_CAST : 0u;
  if (plan_forward(Shape{n, h, vp, v, w_dtype, flags != 0u ? 1 : 0}).total > kNoAllocScratchBytes)
    return FLCE_ERR_WORKSPACE;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return FLCE_ERR_CUDA;
  void* scratch = nullptr;
  {
    // First call on a device (or in a new context on it, e.g. after
    // cudaDeviceReset): look up where the array lives.  In host code the
    // array's name is only a host-side stand-in, never a device address, so
    // the kernels get this looked-up pointer instead.
    const unsigned long long ctx = current_context_id();
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (g_noalloc_addr[dev] == nullptr || context_changed(ctx, g_noalloc_ctx[dev])) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
        return FLCE_ERR_CUDA;
      g_noalloc_addr[dev] = p;
      g_noalloc_ctx[dev] = current_context_id();
    }
    scratch = g_noalloc_addr[dev];
  }
  // Same kernels, same results as flce_forward; every scratch byte the
  // forward reads is written earlier in the same call, so the array's stale
  // contents from a previous call never need clearing.
  return flce_forward_ex(hidden, weight, w_dtype, labels, n, h, vp, unpadded, ignore_index,
                         softcap, reduction, num_label_tokens, loss, lse, scratch,
                         kNoAllocScratchBytes, flags, stream);
}

// ===================================== cross entropy on given logits (chunked_ce)

namespace flce {

struct CePlan {
  size_t off_pm, off_ps, off_zl, off_bl, off_bc, off_lse2, off_scale, total;
  int64_t nblk;
};

// Workspace: per-segment partials for up to kCeMaxSplits segments per row,
// the label logits, the merge blocks' loss sums and the backward's per-token
// lse * log2 e and gradient scale.
static CePlan plan_ce(int64_t n) {
  CePlan p{};
  p.nblk = cdiv(n, kMergeRows);
  size_t o = 0;
  p.off_pm = o;    o = align_up(o + size_t(n) * kCeMaxSplits * 4);
  p.off_ps = o;    o = align_up(o + size_t(n) * kCeMaxSplits * 4);
  p.off_zl = o;    o = align_up(o + size_t(n) * 4);
  p.off_bl = o;    o = align_up(o + size_t(p.nblk) * 8);
  p.off_bc = o;    o = align_up(o + size_t(p.nblk) * 4);
  p.off_lse2 = o;  o = align_up(o + size_t(n) * 4);
  p.off_scale = o; o = align_up(o + size_t(n) * 4);
  p.total = std::max(o, kAlign);
  return p;
}

static int check_ce(const void* logits, int dtype, const int64_t* labels, int64_t n, int64_t v,
                    int64_t ld, int reduction, int64_t num_label_tokens) {
  if (n < 0 || v <= 0 || ld < v || n > kMaxDim || ld > (int64_t(1) << 40) / std::max<int64_t>(n, 1))
    return FLCE_ERR_INVALID_ARG;
  if (dtype != FLCE_BF16 && dtype != FLCE_F32) return FLCE_ERR_INVALID_ARG;
  if (reduction != FLCE_SUM && reduction != FLCE_MEAN && reduction != FLCE_NONE)
    return FLCE_ERR_INVALID_ARG;
  if (num_label_tokens > 0 && reduction != FLCE_SUM) return FLCE_ERR_INVALID_ARG;
  if (n > 0) {
    if (logits == nullptr || labels == nullptr) return FLCE_ERR_INVALID_ARG;
    if (!aligned(logits, 16) || !aligned(labels, 8)) return FLCE_ERR_INVALID_ARG;
  }
  return FLCE_OK;
}

// Launch shape of a CE kernel: whole rows per CTA (grid-stride, up to 16
// CTAs per SM, the hardware scheduler fills slots as CTAs finish).  When the
// rows are fewer than the resident CTA slots (queried once per device and
// kernel), rows are cut into segments of at least kCeMinSegment elements so
// every slot gets work; longer units keep each CTA's load pipeline full.
struct CeLaunch {
  int grid, splits;
};

template <typename Kernel>
static CeLaunch ce_launch(DeviceInfo& dev, int which, Kernel kern, int smem, int64_t n,
                          int64_t v) {
  int per_sm = dev.ce_blocks[which];
  if (per_sm == 0) {  // first launch of this kernel on this device
    if (smem > 0 &&
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
            cudaSuccess)
      return CeLaunch{0, 0};
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kCeThreads, smem) !=
            cudaSuccess ||
        per_sm <= 0)
      per_sm = 1;
    std::lock_guard<std::mutex> lock(g_mutex);
    dev.ce_blocks[which] = per_sm;
  }
  const int64_t slots = int64_t(per_sm) * dev.num_sms;
  CeLaunch l;
  l.splits = 1;
  if (n < slots)
    l.splits = int(std::max<int64_t>(
        1, std::min<int64_t>({kCeMaxSplits, slots / std::max<int64_t>(n, 1), v / kCeMinSegment})));
  l.grid = int(std::min<int64_t>(n * l.splits, int64_t(dev.num_sms) * 16));
  return l;
}

}  // namespace flce

extern "C" size_t flce_ce_workspace_size(int64_t n_tokens) {
  if (n_tokens < 0) return 0;
  return plan_ce(n_tokens).total;
}

extern "C" int flce_ce_forward(const void* logits, int dtype, const int64_t* labels,
                               const uint8_t* mask, int64_t n, int64_t v, int64_t ld,
                               int64_t ignore_index, int reduction, int64_t num_label_tokens,
                               float* loss, float* lse, void* workspace, size_t ws_bytes,
                               flce_stream_t stream) {
  NvtxRange range("flce_ce_forward");
  int st = check_ce(logits, dtype, labels, n, v, ld, reduction, num_label_tokens);
  if (st != FLCE_OK) return st;
  if ((n > 0 || reduction != FLCE_NONE) && (loss == nullptr || !aligned(loss, 4)))
    return FLCE_ERR_INVALID_ARG;
  if (n > 0 && (lse == nullptr || !aligned(lse, 4))) return FLCE_ERR_INVALID_ARG;
  const CePlan p = plan_ce(n);
  if (workspace == nullptr || !aligned(workspace, 16) || ws_bytes < p.total)
    return FLCE_ERR_WORKSPACE;
  DeviceInfo* dev = nullptr;
  if ((st = device_info(&dev)) != FLCE_OK) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* part_m = reinterpret_cast<float*>(ws + p.off_pm);
  float* part_s = reinterpret_cast<float*>(ws + p.off_ps);
  float* label_logit = reinterpret_cast<float*>(ws + p.off_zl);
  double* blk_loss = reinterpret_cast<double*>(ws + p.off_bl);
  int* blk_cnt = reinterpret_cast<int*>(ws + p.off_bc);
  if (n > 0) {
    const size_t esz = dtype == FLCE_F32 ? 4 : 2;
    CeLaunch l;
    {
      LaunchScope scope(KF_CE_FWD, 0.0, double(n) * double(v) * esz + 24.0 * double(n), cs);
      if (dtype == FLCE_BF16) {
        auto kern = ce_partials_kernel<__nv_bfloat16>;
        l = ce_launch(*dev, 0, kern, 0, n, v);
        if (l.grid == 0) return FLCE_ERR_CUDA;
        kern<<<l.grid, kCeThreads, 0, cs>>>(
            static_cast<const __nv_bfloat16*>(logits), ld, labels, mask, n, v, ignore_index,
            l.splits, part_m, part_s, label_logit);
      } else {
        auto kern = ce_partials_kernel<float>;
        l = ce_launch(*dev, 1, kern, 0, n, v);
        if (l.grid == 0) return FLCE_ERR_CUDA;
        kern<<<l.grid, kCeThreads, 0, cs>>>(
            static_cast<const float*>(logits), ld, labels, mask, n, v, ignore_index, l.splits,
            part_m, part_s, label_logit);
      }
    }
    if (cudaGetLastError() != cudaSuccess) return FLCE_ERR_CUDA;
    LaunchScope scope(KF_MERGE, 0.0, 8.0 * double(l.splits) * double(n) + 24.0 * double(n), cs);
    lse_merge_kernel<<<int(p.nblk), kMergeRows * kMergeWarps, 0, cs>>>(
        part_m, part_s, l.splits, n, label_logit, labels, mask, v, ignore_index, lse,
        reduction == FLCE_NONE ? loss : nullptr, blk_loss, blk_cnt, dev->err);
    if (cudaGetLastError() != cudaSuccess) return FLCE_ERR_CUDA;
  }
  if (reduction != FLCE_NONE) {
    LaunchScope scope(KF_FINAL, 0.0, 12.0 * double(p.nblk), cs);
    loss_finalize_kernel<<<1, kFinalThreads, 0, cs>>>(blk_loss, blk_cnt, int(p.nblk), reduction,
                                                      num_label_tokens, loss);
    if (cudaGetLastError() != cudaSuccess) return FLCE_ERR_CUDA;
  }
  return FLCE_OK;
}

extern "C" int flce_ce_backward(const void* logits, int dtype, const int64_t* labels,
                                const uint8_t* mask, int64_t n, int64_t v, int64_t ld,
                                int64_t ignore_index, int reduction, int64_t num_label_tokens,
                                const float* grad_loss, const float* lse, void* dlogits,
                                void* workspace, size_t ws_bytes, flce_stream_t stream) {
  NvtxRange range("flce_ce_backward");
  int st = check_ce(logits, dtype, labels, n, v, ld, reduction, num_label_tokens);
  if (st != FLCE_OK) return st;
  if (n > 0) {
    if (grad_loss == nullptr || lse == nullptr || dlogits == nullptr) return FLCE_ERR_INVALID_ARG;
    if (!aligned(grad_loss, 4) || !aligned(lse, 4) || !aligned(dlogits, 16))
      return FLCE_ERR_INVALID_ARG;
  }
  const CePlan p = plan_ce(n);
  if (workspace == nullptr || !aligned(workspace, 16) || ws_bytes < p.total)
    return FLCE_ERR_WORKSPACE;
  if (n == 0) return FLCE_OK;
  DeviceInfo* dev = nullptr;
  if ((st = device_info(&dev)) != FLCE_OK) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* lse2 = reinterpret_cast<float*>(ws + p.off_lse2);
  float* scale = reinterpret_cast<float*>(ws + p.off_scale);
  {
    LaunchScope scope(KF_BWD_PREP, 0.0, 24.0 * double(n), cs);
    bwd_prep_kernel<<<1, 1024, 0, cs>>>(labels, mask, n, v, ignore_index, reduction,
                                        num_label_tokens, grad_loss, lse, lse2, scale, nullptr, 0,
                                        dev->err);
  }
  if (cudaGetLastError() != cudaSuccess) return FLCE_ERR_CUDA;
  const size_t esz = dtype == FLCE_F32 ? 4 : 2;
  LaunchScope scope(KF_CE_BWD, 0.0, 2.0 * double(n) * double(v) * esz + 16.0 * double(n), cs);
  if (dtype == FLCE_BF16) {
    auto kern = ce_backward_kernel<__nv_bfloat16>;
    const CeLaunch l = ce_launch(*dev, 2, kern, kCeRingBytes, n, v);
    if (l.grid == 0) return FLCE_ERR_CUDA;
    kern<<<l.grid, kCeThreads, kCeRingBytes, cs>>>(
        static_cast<const __nv_bfloat16*>(logits), ld, labels, n, v, l.splits, lse2, scale,
        static_cast<__nv_bfloat16*>(dlogits));
  } else {
    auto kern = ce_backward_kernel<float>;
    const CeLaunch l = ce_launch(*dev, 3, kern, kCeRingBytes, n, v);
    if (l.grid == 0) return FLCE_ERR_CUDA;
    kern<<<l.grid, kCeThreads, kCeRingBytes, cs>>>(static_cast<const float*>(logits), ld, labels,
                                                   n, v, l.splits, lse2, scale,
                                                   static_cast<float*>(dlogits));
  }
  return cudaGetLastError() == cudaSuccess ? FLCE_OK : FLCE_ERR_CUDA;
}
