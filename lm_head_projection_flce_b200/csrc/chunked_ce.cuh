// chunked_ce.cuh - cross entropy on given logits ("nemo_automodel.components.
// loss.chunked_ce": ChunkedCrossEntropy.forward, _ChunkedCrossEntropySum
// forward / backward).  Logits [N, V] (BF16 or FP32, row stride ld) are read
// once by the forward and once more by the backward, which writes the logits
// gradient in the logits' dtype; nothing is upcast into an FP32 copy.  One CTA
// per token row streams the row with 16-byte loads (scalar head and tail for
// rows that do not start on a 16-byte boundary), keeps a running base-2
// (max, sum of exponentials) in registers and merges the 256 threads' pairs.
#pragma once

#include <cuda_bf16.h>

#include "epilogues.cuh"

namespace flce {

constexpr int kCeThreads = 256;

template <typename T>
struct CeVec;
template <>
struct CeVec<__nv_bfloat16> {
  static constexpr int kN = 8;  // elements per 16-byte vector
  static __device__ __forceinline__ void load(const __nv_bfloat16* p, float (&x)[8]) {
    const uint4 w = *reinterpret_cast<const uint4*>(p);
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u[i]));
      x[2 * i] = f.x;
      x[2 * i + 1] = f.y;
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
  static __device__ __forceinline__ void load(const float* p, float (&x)[4]) {
    const float4 w = *reinterpret_cast<const float4*>(p);
    x[0] = w.x;
    x[1] = w.y;
    x[2] = w.z;
    x[3] = w.w;
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

template <typename T>
__global__ void __launch_bounds__(kCeThreads)
    ce_forward_kernel(const T* __restrict__ logits, int64_t ld, const int64_t* __restrict__ labels,
                      const uint8_t* __restrict__ mask, int64_t n_tokens, int64_t vocab,
                      int64_t ignore_index, float* __restrict__ lse_out,
                      float* __restrict__ token_loss, double* __restrict__ row_loss,
                      int* __restrict__ row_cnt, unsigned* __restrict__ err) {
  constexpr int VN = CeVec<T>::kN;
  __shared__ float sm_m[kCeThreads / 32], sm_s[kCeThreads / 32];
  for (int64_t n = blockIdx.x; n < n_tokens; n += gridDim.x) {
    const T* row = logits + n * ld;
    int64_t head, nvec;
    ce_row_split(row, vocab, head, nvec);
    float m = -INFINITY, s = 0.0f;
    for (int64_t i = threadIdx.x; i < head; i += kCeThreads)
      ms_merge(m, s, CeVec<T>::one(row + i) * kLog2e, 1.0f);
    const T* body = row + head;
    // Four independent 16-byte loads in flight per thread, then one rescale.
    constexpr int U = 4;
    int64_t j = threadIdx.x;
    for (; j + (U - 1) * kCeThreads < nvec; j += U * kCeThreads) {
      float x[U][VN];
#pragma unroll
      for (int u = 0; u < U; ++u) CeVec<T>::load(body + (j + u * kCeThreads) * VN, x[u]);
      float vm = -INFINITY;
#pragma unroll
      for (int u = 0; u < U; ++u)
#pragma unroll
        for (int e = 0; e < VN; ++e) {
          x[u][e] *= kLog2e;
          vm = fmaxf(vm, x[u][e]);
        }
      if (vm == -INFINITY) continue;
      if (vm > m) {
        s = s * fast_exp2(m - vm);
        m = vm;
      }
      float acc = 0.0f;
#pragma unroll
      for (int u = 0; u < U; ++u)
#pragma unroll
        for (int e = 0; e < VN; ++e) acc += fast_exp2(x[u][e] - m);
      s += acc;
    }
    for (; j < nvec; j += kCeThreads) {
      float x[VN];
      CeVec<T>::load(body + j * VN, x);
      float vm = -INFINITY;
#pragma unroll
      for (int e = 0; e < VN; ++e) {
        x[e] *= kLog2e;
        vm = fmaxf(vm, x[e]);
      }
      if (vm == -INFINITY) continue;
      if (vm > m) {
        s = s * fast_exp2(m - vm);
        m = vm;
      }
#pragma unroll
      for (int e = 0; e < VN; ++e) s += fast_exp2(x[e] - m);
    }
    for (int64_t i = head + nvec * VN + threadIdx.x; i < vocab; i += kCeThreads)
      ms_merge(m, s, CeVec<T>::one(row + i) * kLog2e, 1.0f);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
      const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
      ms_merge(m, s, m2, s2);
    }
    if ((threadIdx.x & 31) == 0) {
      sm_m[threadIdx.x >> 5] = m;
      sm_s[threadIdx.x >> 5] = s;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      float M = -INFINITY, S = 0.0f;
      for (int w = 0; w < kCeThreads / 32; ++w) ms_merge(M, S, sm_m[w], sm_s[w]);
      const float lse = (M + log2f(S)) * 0.6931471805599453f;
      const int64_t y = labels[n];
      bool valid = y != ignore_index && (mask == nullptr || mask[n] != 0);
      if (valid && (y < 0 || y >= vocab)) {
        atomicOr(err, kDevErrBadLabel);
        valid = false;
      }
      const float l = valid ? lse - CeVec<T>::one(row + y) : 0.0f;
      lse_out[n] = lse;
      if (token_loss) token_loss[n] = l;
      row_loss[n] = l;
      row_cnt[n] = valid ? 1 : 0;
    }
    __syncthreads();
  }
}

// dlogits[n, v] = s_n * (exp(z - lse_n) - [v == y_n]), in the logits' dtype.
template <typename T>
__global__ void __launch_bounds__(kCeThreads)
    ce_backward_kernel(const T* __restrict__ logits, int64_t ld, const int64_t* __restrict__ labels,
                       int64_t n_tokens, int64_t vocab, const float* __restrict__ lse2,
                       const float* __restrict__ scale, T* __restrict__ dlogits) {
  constexpr int VN = CeVec<T>::kN;
  for (int64_t n = blockIdx.x; n < n_tokens; n += gridDim.x) {
    const T* row = logits + n * ld;
    T* out = dlogits + n * ld;
    const float l2 = lse2[n];
    const float sc = scale[n];
    const int64_t y = labels[n];
    int64_t head, nvec;
    ce_row_split(row, vocab, head, nvec);
    auto grad = [&](float z, int64_t col) {
      return sc * (fast_exp2(z * kLog2e - l2) - (col == y ? 1.0f : 0.0f));
    };
    for (int64_t i = threadIdx.x; i < head; i += kCeThreads)
      CeVec<T>::put(out + i, grad(CeVec<T>::one(row + i), i));
    const T* body = row + head;
    T* obody = out + head;
#pragma unroll 2
    for (int64_t j = threadIdx.x; j < nvec; j += kCeThreads) {
      float x[VN];
      CeVec<T>::load(body + j * VN, x);
      const int64_t c0 = head + j * VN;
#pragma unroll
      for (int e = 0; e < VN; ++e) x[e] = grad(x[e], c0 + e);
      CeVec<T>::store(obody + j * VN, x);
    }
    for (int64_t i = head + nvec * VN + threadIdx.x; i < vocab; i += kCeThreads)
      CeVec<T>::put(out + i, grad(CeVec<T>::one(row + i), i));
  }
}

}  // namespace flce
