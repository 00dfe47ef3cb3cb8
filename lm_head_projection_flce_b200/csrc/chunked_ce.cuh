// chunked_ce.cuh - cross entropy on given logits ("nemo_automodel.components.
// loss.chunked_ce": ChunkedCrossEntropy.forward, _ChunkedCrossEntropySum
// forward / backward).  Logits [N, V] (BF16 or FP32, row stride ld) are read
// once by the forward and once more by the backward, which writes the logits
// gradient in the logits' dtype; nothing is upcast into an FP32 copy.
//
// Work is cut into units (token row n, segment p of `splits` equal pieces of
// the row; one segment per row unless the rows are too few to fill the GPU).
// The forward keeps the next batch of 16-byte loads in registers while it
// folds the current one (it also runs one exponential per element and needs
// the occupancy); the backward streams each thread's vectors through a
// private ring of shared-memory slots with cp.async, so several batches per
// thread are in flight without holding registers.  The forward writes a
// base-2 (max, sum of exponentials) pair per unit, in the [splits, N] layout
// the projection forward uses for its per-tile partials, and the same merge
// kernel finishes both.
#pragma once

#include <cuda_bf16.h>

#include "epilogues.cuh"

namespace flce {

constexpr int kCeThreads = 256;
constexpr int kCeBatch = 4;          // 16-byte vectors per thread per batch
constexpr int kCeStages = 4;         // backward: batches per thread in the ring (3 in flight)
constexpr int kCeRingBytes = kCeStages * kCeBatch * kCeThreads * 16;  // 64 KB per CTA
constexpr int kCeMaxSplits = 16;     // segments per row at most (sizes the workspace)
constexpr int64_t kCeMinSegment = 32768;  // elements per segment at least

template <typename T>
struct CeVec;
template <>
struct CeVec<__nv_bfloat16> {
  static constexpr int kN = 8;  // elements per 16-byte vector
  static __device__ __forceinline__ float2 pair(uint32_t u) {  // bf16x2 -> float2, exact
    return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
  }
  static __device__ __forceinline__ void unpack(const uint4& w, float (&x)[8]) {
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = pair(u[i]);
      x[2 * i] = f.x;
      x[2 * i + 1] = f.y;
    }
  }
  // Largest element of the batch (packed BF16 max: exact, NaN ignored like fmaxf).
  template <int U>
  static __device__ __forceinline__ float vmax(const uint4 (&r)[U]) {
    __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&r[0].x);
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const uint32_t w[4] = {r[u].x, r[u].y, r[u].z, r[u].w};
#pragma unroll
      for (int i = 0; i < 4; ++i) a = __hmax2(a, *reinterpret_cast<const __nv_bfloat162*>(&w[i]));
    }
    const float2 f = __bfloat1622float2(a);
    return fmaxf(f.x, f.y);
  }
  // acc += 2^(x * log2 e - m) over the vector, two lanes at a time.
  static __device__ __forceinline__ void acc_exp(const uint4& r, float2 negm, float2& acc) {
    const uint32_t u[4] = {r.x, r.y, r.z, r.w};
    const float2 l2e = make_float2(kLog2e, kLog2e);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 t = __ffma2_rn(pair(u[i]), l2e, negm);
      acc = __fadd2_rn(acc, make_float2(fast_exp2(t.x), fast_exp2(t.y)));
    }
  }
  static __device__ __forceinline__ void store(__nv_bfloat16* p, const float (&x)[8]) {
    uint4 w;
    w.x = pack_bf16x2(x[0], x[1]);
    w.y = pack_bf16x2(x[2], x[3]);
    w.z = pack_bf16x2(x[4], x[5]);
    w.w = pack_bf16x2(x[6], x[7]);
    *reinterpret_cast<uint4*>(p) = w;
  }
  static __device__ __forceinline__ float one(const __nv_bfloat16* p) { return __bfloat162float(*p); }
  static __device__ __forceinline__ void put(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }
};
template <>
struct CeVec<float> {
  static constexpr int kN = 4;
  static __device__ __forceinline__ void unpack(const uint4& w, float (&x)[4]) {
    x[0] = __uint_as_float(w.x);
    x[1] = __uint_as_float(w.y);
    x[2] = __uint_as_float(w.z);
    x[3] = __uint_as_float(w.w);
  }
  template <int U>
  static __device__ __forceinline__ float vmax(const uint4 (&r)[U]) {
    float a = __uint_as_float(r[0].x);
#pragma unroll
    for (int u = 0; u < U; ++u)
      a = fmaxf(fmaxf(a, fmaxf(__uint_as_float(r[u].x), __uint_as_float(r[u].y))),
                fmaxf(__uint_as_float(r[u].z), __uint_as_float(r[u].w)));
    return a;
  }
  static __device__ __forceinline__ void acc_exp(const uint4& r, float2 negm, float2& acc) {
    const float2 l2e = make_float2(kLog2e, kLog2e);
    const float2 t0 = __ffma2_rn(make_float2(__uint_as_float(r.x), __uint_as_float(r.y)), l2e, negm);
    const float2 t1 = __ffma2_rn(make_float2(__uint_as_float(r.z), __uint_as_float(r.w)), l2e, negm);
    acc = __fadd2_rn(acc, make_float2(fast_exp2(t0.x), fast_exp2(t0.y)));
    acc = __fadd2_rn(acc, make_float2(fast_exp2(t1.x), fast_exp2(t1.y)));
  }
  static __device__ __forceinline__ void store(float* p, const float (&x)[4]) {
    *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
  }
  static __device__ __forceinline__ float one(const float* p) { return *p; }
  static __device__ __forceinline__ void put(float* p, float x) { *p = x; }
};

// Running (max, sum 2^(u - max)) of base-2 scaled logits u; merge of two pairs.
__device__ __forceinline__ void ms_merge(float& m, float& s, float m2, float s2) {
  const float mn = fmaxf(m, m2);
  if (mn == -INFINITY) return;
  s = s * fast_exp2(m - mn) + s2 * fast_exp2(m2 - mn);
  m = mn;
}

// Elements [0, head) scalar, [head, head + nvec*N) in vectors, then the tail.
template <typename T>
__device__ __forceinline__ void ce_row_split(const T* row, int64_t v, int64_t& head, int64_t& nvec) {
  const uintptr_t a = reinterpret_cast<uintptr_t>(row);
  head = static_cast<int64_t>(((16 - (a & 15)) & 15) / sizeof(T));
  if (head > v) head = v;
  nvec = (v - head) / CeVec<T>::kN;
}

// Vectors [j0, j1) of segment p (of `splits`) of a row with nvec vectors.
__device__ __forceinline__ void ce_segment(int64_t nvec, int p, int splits, int64_t& j0,
                                           int64_t& j1) {
  const int64_t per = (nvec + splits - 1) / splits;
  j0 = min(nvec, int64_t(p) * per);
  j1 = min(nvec, j0 + per);
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// This thread's vectors of [j0, j1) (every kCeThreads-th, from j0 + tid) in
// batches of kCeBatch, copied into the thread's own kCeStages slots of `ring`
// (so no other thread touches them and no CTA barrier is needed) while the
// batch kCeStages - 1 behind is used.  full(r, j) gets a whole batch whose
// first vector is j, part(v, j) the vectors of a short last batch.  A stage
// is refilled one iteration after it was read, once its values were used.
template <typename Full, typename Part>
__device__ __forceinline__ void ce_stream(const uint4* __restrict__ body, int64_t j0, int64_t j1,
                                          const uint4* ring, Full&& full, Part&& part) {
  constexpr int U = kCeBatch, S = kCeStages;
  const int tid = threadIdx.x;
  const int64_t first = j0 + tid;
  const int cnt = first < j1 ? int((j1 - first + kCeThreads - 1) / kCeThreads) : 0;
  const int nb = (cnt + U - 1) / U;
  const uint32_t ring_sh = smem_u32(ring);
  auto slot = [&](int stage, int u) { return (stage * U + u) * kCeThreads + tid; };
  auto issue = [&](int b) {
    if (b < nb) {
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (b * U + u < cnt)
          cp_async16(ring_sh + 16u * slot(b % S, u), body + first + int64_t(b * U + u) * kCeThreads);
    }
    cp_async_commit();  // empty groups keep the group count uniform
  };
#pragma unroll
  for (int b = 0; b < S - 1; ++b) issue(b);
  for (int b = 0; b < nb; ++b) {
    issue(b + S - 1);
    cp_async_wait<S - 1>();  // batch b has landed
    const int st = b % S;
    const int64_t jb = first + int64_t(b * U) * kCeThreads;
    if ((b + 1) * U <= cnt) {
      uint4 r[U];
#pragma unroll
      for (int u = 0; u < U; ++u) r[u] = ring[slot(st, u)];
      full(r, jb);
    } else {
      for (int u = 0; b * U + u < cnt; ++u) part(ring[slot(st, u)], jb + int64_t(u) * kCeThreads);
    }
  }
}

// Fold a batch of U vectors into the running base-2 (m, s): one rescale per
// batch, then 2^(x log2 e - m) summed in two lanes.
template <typename T, int U>
__device__ __forceinline__ void ce_fold(const uint4 (&r)[U], float& m, float2& s) {
  const float vm = CeVec<T>::template vmax<U>(r) * kLog2e;
  if (vm == -INFINITY) return;
  if (vm > m) {
    const float f = fast_exp2(m - vm);
    s.x *= f;
    s.y *= f;
    m = vm;
  }
  const float2 negm = make_float2(-m, -m);
  float2 a0 = make_float2(0.0f, 0.0f), a1 = a0;
#pragma unroll
  for (int u = 0; u < U; u += 2) {
    CeVec<T>::acc_exp(r[u], negm, a0);
    if (u + 1 < U) CeVec<T>::acc_exp(r[u + 1], negm, a1);
  }
  s = __fadd2_rn(s, __fadd2_rn(a0, a1));
}

// Forward, pass 1: unit u = n * splits + p reduces segment p of row n (the
// scalar head goes with p = 0, the scalar tail with p = splits - 1) to a
// base-2 (max, sum) pair at [p, n] of part_m / part_s; p = 0 also stores the
// label's logit (0 for ignored, masked or out-of-range labels; the merge
// kernel flags the latter).
template <typename T>
__global__ void __launch_bounds__(kCeThreads)
    ce_partials_kernel(const T* __restrict__ logits, int64_t ld, const int64_t* __restrict__ labels,
                       const uint8_t* __restrict__ mask, int64_t n_tokens, int64_t vocab,
                       int64_t ignore_index, int splits, float* __restrict__ part_m,
                       float* __restrict__ part_s, float* __restrict__ label_logit) {
  constexpr int VN = CeVec<T>::kN;
  constexpr int U = kCeBatch;
  constexpr int64_t kStep = int64_t(U) * kCeThreads;
  __shared__ float sm_m[kCeThreads / 32], sm_s[kCeThreads / 32];
  const int tid = threadIdx.x;
  const int64_t units = n_tokens * splits;
  for (int64_t unit = blockIdx.x; unit < units; unit += gridDim.x) {
    const int64_t n = unit / splits;
    const int p = int(unit - n * splits);
    const T* row = logits + n * ld;
    int64_t head, nvec, j0, j1;
    ce_row_split(row, vocab, head, nvec);
    ce_segment(nvec, p, splits, j0, j1);
    float m = -INFINITY, s1 = 0.0f;
    if (p == 0)
      for (int64_t i = tid; i < head; i += kCeThreads) ms_merge(m, s1, CeVec<T>::one(row + i) * kLog2e, 1.0f);
    if (p == splits - 1)
      for (int64_t i = head + nvec * VN + tid; i < vocab; i += kCeThreads)
        ms_merge(m, s1, CeVec<T>::one(row + i) * kLog2e, 1.0f);
    float2 s = make_float2(s1, 0.0f);
    // Registers, not the shared-memory ring: this pass is bound by the
    // exponentials as much as by HBM and needs the higher occupancy.  The
    // next batch's loads are issued before the current batch is folded.
    const uint4* body = reinterpret_cast<const uint4*>(row + head);
    int64_t j = j0 + tid;
    if (j + (U - 1) * kCeThreads < j1) {
      uint4 cur[U];
#pragma unroll
      for (int u = 0; u < U; ++u) cur[u] = body[j + u * kCeThreads];
      for (;;) {
        const int64_t jn = j + kStep;
        const bool more = jn + (U - 1) * kCeThreads < j1;
        uint4 nxt[U];
        if (more) {
#pragma unroll
          for (int u = 0; u < U; ++u) nxt[u] = body[jn + u * kCeThreads];
        }
        ce_fold<T, U>(cur, m, s);
        j = jn;
        if (!more) break;
#pragma unroll
        for (int u = 0; u < U; ++u) cur[u] = nxt[u];
      }
    }
    for (; j < j1; j += kCeThreads) {
      const uint4 one[1] = {body[j]};
      ce_fold<T, 1>(one, m, s);
    }
    float sum = s.x + s.y;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
      const float s2 = __shfl_xor_sync(0xffffffffu, sum, o);
      ms_merge(m, sum, m2, s2);
    }
    if ((tid & 31) == 0) {
      sm_m[tid >> 5] = m;
      sm_s[tid >> 5] = sum;
    }
    __syncthreads();
    if (tid == 0) {
      float M = -INFINITY, S = 0.0f;
      for (int w = 0; w < kCeThreads / 32; ++w) ms_merge(M, S, sm_m[w], sm_s[w]);
      part_m[int64_t(p) * n_tokens + n] = M;
      part_s[int64_t(p) * n_tokens + n] = S;
      if (p == 0) {
        const int64_t y = labels[n];
        const bool take = y != ignore_index && (mask == nullptr || mask[n] != 0) && y >= 0 &&
                          y < vocab;
        label_logit[n] = take ? CeVec<T>::one(row + y) : 0.0f;
      }
    }
    __syncthreads();
  }
}

// dlogits[n, v] = s_n * (exp(z - lse_n) - [v == y_n]), in the logits' dtype,
// over the same (row, segment) units as the forward.
template <typename T>
__global__ void __launch_bounds__(kCeThreads)
    ce_backward_kernel(const T* __restrict__ logits, int64_t ld, const int64_t* __restrict__ labels,
                       int64_t n_tokens, int64_t vocab, int splits, const float* __restrict__ lse2,
                       const float* __restrict__ scale, T* __restrict__ dlogits) {
  constexpr int VN = CeVec<T>::kN;
  extern __shared__ __align__(16) uint4 ce_ring[];  // kCeRingBytes
  const int64_t units = n_tokens * splits;
  for (int64_t unit = blockIdx.x; unit < units; unit += gridDim.x) {
    const int64_t n = unit / splits;
    const int p = int(unit - n * splits);
    const T* row = logits + n * ld;
    T* out = dlogits + n * ld;
    const float l2 = lse2[n];
    const float sc = scale[n];
    const int64_t y = labels[n];
    int64_t head, nvec, j0, j1;
    ce_row_split(row, vocab, head, nvec);
    ce_segment(nvec, p, splits, j0, j1);
    auto grad = [&](float z, int64_t col) {
      return sc * (fast_exp2(z * kLog2e - l2) - (col == y ? 1.0f : 0.0f));
    };
    if (p == 0)
      for (int64_t i = threadIdx.x; i < head; i += kCeThreads)
        CeVec<T>::put(out + i, grad(CeVec<T>::one(row + i), i));
    if (p == splits - 1)
      for (int64_t i = head + nvec * VN + threadIdx.x; i < vocab; i += kCeThreads)
        CeVec<T>::put(out + i, grad(CeVec<T>::one(row + i), i));
    const uint4* body = reinterpret_cast<const uint4*>(row + head);
    T* obody = out + head;
    auto emit = [&](const uint4& w, int64_t j) {
      float x[VN];
      CeVec<T>::unpack(w, x);
      const int64_t c0 = head + j * VN;
#pragma unroll
      for (int e = 0; e < VN; ++e) x[e] = grad(x[e], c0 + e);
      CeVec<T>::store(obody + j * VN, x);
    };
    ce_stream(
        body, j0, j1, ce_ring,
        [&](const uint4 (&r)[kCeBatch], int64_t j) {
#pragma unroll
          for (int u = 0; u < kCeBatch; ++u) emit(r[u], j + int64_t(u) * kCeThreads);
        },
        emit);
  }
}

}  // namespace flce
