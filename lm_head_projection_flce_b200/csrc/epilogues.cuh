// epilogues.cuh - per-tile epilogues of the tensor-core GEMM.  Each runs on
// one epilogue thread that owns accumulator row `row` (0..127) of tile
// (mt, nt) and reads its 256 FP32 columns from tensor memory 32 at a time.
// tcgen05.ld is warp-collective, so rows past the problem edge still load and
// only skip their stores.
#pragma once

#include <cuda_bf16.h>

#include "gemm_sm100.cuh"

namespace flce {

constexpr float kLog2e = 1.4426950408889634f;

// Softcap c*tanh(z/c) from tanh(x) = 1 - 2/(exp(2x) + 1), on two columns at
// once with packed FP32 arithmetic: zc = c - 2c r with r = 1/(2^(z k) + 1),
// k = 2*log2(e)/c.  r is returned for the derivative
// d(c*tanh(z/c))/dz = 1 - tanh^2 = 4r(1-r), which stays finite at both ends
// (r -> 0 and r -> 1).  c2 = (c, c), m2c = (-2c, -2c), k2 = (k, k).
__device__ __forceinline__ float2 softcap_pair(float2 z, float2 c2, float2 m2c, float2 k2,
                                               float2& r) {
  const float2 t = __fmul2_rn(z, k2);
  const float2 e = __fadd2_rn(make_float2(fast_exp2(t.x), fast_exp2(t.y)), make_float2(1.0f, 1.0f));
  r = make_float2(fast_rcp(e.x), fast_rcp(e.y));
  return __ffma2_rn(r, m2c, c2);  // c - 2c r
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);  // round to nearest even
  return *reinterpret_cast<uint32_t*>(&h);
}

// 32 FP32 values rounded to BF16 and stored at `out` (64 bytes): two 32-byte
// stores when `v8` (out 32-byte aligned), else four 16-byte ones.
__device__ __forceinline__ void store_bf16x32(uint4* out, const float (&v)[32], bool v8) {
  if (v8) {
#pragma unroll
    for (int q = 0; q < 2; ++q)
      st_global_v8(out + 2 * q, pack_bf16x2(v[16 * q + 0], v[16 * q + 1]),
                   pack_bf16x2(v[16 * q + 2], v[16 * q + 3]),
                   pack_bf16x2(v[16 * q + 4], v[16 * q + 5]),
                   pack_bf16x2(v[16 * q + 6], v[16 * q + 7]),
                   pack_bf16x2(v[16 * q + 8], v[16 * q + 9]),
                   pack_bf16x2(v[16 * q + 10], v[16 * q + 11]),
                   pack_bf16x2(v[16 * q + 12], v[16 * q + 13]),
                   pack_bf16x2(v[16 * q + 14], v[16 * q + 15]));
  } else {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint4 w;
      w.x = pack_bf16x2(v[8 * q + 0], v[8 * q + 1]);
      w.y = pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
      w.z = pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
      w.w = pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
      out[q] = w;
    }
  }
}

// -------------------------------------------------------------------------
// Forward: logits tile -> per-row partial (max, sum of exponentials) over the
// tile's live vocabulary columns, plus the label's capped logit.
//   Rows are tokens (A = hidden), columns are head rows (B = W).  Partials are
//   in base 2: m = max_v zc*log2(e), s = sum_v 2^(zc*log2(e) - m).
// -------------------------------------------------------------------------
struct EpiForward {
  struct Params {
    const int64_t* labels;
    int64_t n_tokens;
    int64_t vocab;        // unpadded V: columns >= V never enter the softmax
    float softcap;        // 0 = off
    float softcap_k;      // 2*log2(e)/softcap
    float* part_m;        // [v_tiles][n_tokens]
    float* part_s;        // [v_tiles][n_tokens]
    float* label_logit;   // [n_tokens]: zc at the label (written by the tile holding it)
  };

  static __device__ __forceinline__ void tile(const Params& p, uint32_t taddr, int mt, int nt,
                                              int row) {
    const int64_t n = static_cast<int64_t>(mt) * kBM + row;
    const bool live = n < p.n_tokens;
    const int64_t vbase = static_cast<int64_t>(nt) * kBN;
    const int64_t y = live ? p.labels[n] : -1;
    const int64_t ylocal = y - vbase;
    const int ncols = static_cast<int>(min(static_cast<int64_t>(kBN), p.vocab - vbase));
    float m = -INFINITY, s = 0.0f, zl = 0.0f;
    const bool capped = p.softcap > 0.0f;
    const float2 l2e = make_float2(kLog2e, kLog2e);
#pragma unroll 1
    for (int c0 = 0; c0 < kBN; c0 += 32) {
      float v[32];
      tmem_load_32cols(taddr + c0, v);
      if (capped) {
        const float2 c2 = make_float2(p.softcap, p.softcap);
        const float2 m2c = make_float2(-2.0f * p.softcap, -2.0f * p.softcap);
        const float2 k2 = make_float2(p.softcap_k, p.softcap_k);
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          float2 r;
          const float2 zc = softcap_pair(make_float2(v[j], v[j + 1]), c2, m2c, k2, r);
          v[j] = zc.x;
          v[j + 1] = zc.y;
        }
      }
      if (ylocal >= c0 && ylocal < c0 + 32) {
        // Pick column ylocal - c0 with a select tree on its bits (no local-memory indexing).
        const int jl = static_cast<int>(ylocal - c0);
        float t16[16], t8[8], t4[4], t2[2];
#pragma unroll
        for (int j = 0; j < 16; ++j) t16[j] = (jl & 16) ? v[j + 16] : v[j];
#pragma unroll
        for (int j = 0; j < 8; ++j) t8[j] = (jl & 8) ? t16[j + 8] : t16[j];
#pragma unroll
        for (int j = 0; j < 4; ++j) t4[j] = (jl & 4) ? t8[j + 4] : t8[j];
#pragma unroll
        for (int j = 0; j < 2; ++j) t2[j] = (jl & 2) ? t4[j + 2] : t4[j];
        zl = (jl & 1) ? t2[1] : t2[0];
      }
      if (c0 + 32 > ncols) {  // only in the vocabulary's last tile
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (c0 + j >= ncols) v[j] = -INFINITY;
      }
      // max on the raw values (log2 e > 0 keeps the order), then
      // 2^(z log2 e - mn) with the scale folded into one packed FMA per pair.
      float c[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) c[j] = fmaxf(v[j], v[j + 16]);
#pragma unroll
      for (int w = 8; w > 0; w >>= 1)
#pragma unroll
        for (int j = 0; j < w; ++j) c[j] = fmaxf(c[j], c[j + w]);
      const float mn = fmaxf(m, c[0] * kLog2e);
      if (mn != -INFINITY) {
        const float2 nm = make_float2(-mn, -mn);
        float2 a0 = make_float2(0.0f, 0.0f), a1 = a0;
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
          const float2 t0 = __ffma2_rn(make_float2(v[j], v[j + 1]), l2e, nm);
          const float2 t1 = __ffma2_rn(make_float2(v[j + 2], v[j + 3]), l2e, nm);
          a0 = __fadd2_rn(a0, make_float2(fast_exp2(t0.x), fast_exp2(t0.y)));
          a1 = __fadd2_rn(a1, make_float2(fast_exp2(t1.x), fast_exp2(t1.y)));
        }
        const float2 a = __fadd2_rn(a0, a1);
        s = s * fast_exp2(m - mn) + (a.x + a.y);
        m = mn;
      }
    }
    if (live) {
      p.part_m[static_cast<int64_t>(nt) * p.n_tokens + n] = m;
      p.part_s[static_cast<int64_t>(nt) * p.n_tokens + n] = s;
      if (ylocal >= 0 && ylocal < ncols) p.label_logit[n] = zl;
    }
  }
};

// -------------------------------------------------------------------------
// Backward recompute: logits tile -> gradient of the loss w.r.t. the logits,
//   G[n, v] = s_n * (softmax(zc)[n, v] - [v == y_n]) * dzc/dz,   0 for v >= V,
// rounded to BF16 and stored to the chunk buffer G[n, v - v0].
// -------------------------------------------------------------------------
struct EpiGrad {
  struct Params {
    const int64_t* labels;
    int64_t n_tokens;
    int64_t vocab;       // unpadded V
    int64_t v0;          // vocabulary index of GEMM column 0 (chunk start)
    float softcap;
    float softcap_k;
    const float* lse2;   // [n_tokens] logsumexp * log2(e)
    const float* scale;  // [n_tokens] d loss / d token loss (0 if ignored)
    __nv_bfloat16* g;    // [n_tokens][ldg]
    int64_t ldg;
    int v8;              // 1: g and its rows are 32-byte aligned (32-byte stores)
  };

  static __device__ __forceinline__ void tile(const Params& p, uint32_t taddr, int mt, int nt,
                                              int row) {
    const int64_t n = static_cast<int64_t>(mt) * kBM + row;
    const bool live = n < p.n_tokens;
    const int64_t vbase = p.v0 + static_cast<int64_t>(nt) * kBN;
    const int64_t y = live ? p.labels[n] : -1;
    const int64_t ylocal = y - vbase;
    const float l2 = live ? p.lse2[n] : 0.0f;
    const float sc = live ? p.scale[n] : 0.0f;
    const int ncols = static_cast<int>(min(static_cast<int64_t>(kBN), p.vocab - vbase));
    uint4* out = reinterpret_cast<uint4*>(p.g + (live ? n : 0) * p.ldg + static_cast<int64_t>(nt) * kBN);
    const bool capped = p.softcap > 0.0f;
    const float2 l2e = make_float2(kLog2e, kLog2e), nl2 = make_float2(-l2, -l2),
                 sc2 = make_float2(sc, sc);
#pragma unroll 1
    for (int c0 = 0; c0 < kBN; c0 += 32) {
      float v[32];
      tmem_load_32cols(taddr + c0, v);
      if (!capped) {
        // sc * 2^(z log2 e - lse log2 e), two columns per packed FMA / multiply
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          const float2 t = __ffma2_rn(make_float2(v[j], v[j + 1]), l2e, nl2);
          const float2 g = __fmul2_rn(make_float2(fast_exp2(t.x), fast_exp2(t.y)), sc2);
          v[j] = g.x;
          v[j + 1] = g.y;
        }
        if (ylocal >= c0 && ylocal < c0 + 32) {  // the label's column: - sc
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (c0 + j == ylocal) v[j] -= sc;
        }
      } else {
        // (2^(zc log2 e - lse log2 e) - onehot) * sc * 4r(1 - r), two columns at a time
        const float2 c2 = make_float2(p.softcap, p.softcap);
        const float2 m2c = make_float2(-2.0f * p.softcap, -2.0f * p.softcap);
        const float2 k2 = make_float2(p.softcap_k, p.softcap_k);
        const float2 four = make_float2(4.0f, 4.0f);
        auto pair = [&](int j, bool label) {
          float2 r;
          const float2 zc = softcap_pair(make_float2(v[j], v[j + 1]), c2, m2c, k2, r);
          const float2 q = __fmul2_rn(r, four);
          const float2 dsc = __fmul2_rn(__ffma2_rn(make_float2(-q.x, -q.y), r, q), sc2);
          const float2 t = __ffma2_rn(zc, l2e, nl2);
          float2 pr = make_float2(fast_exp2(t.x), fast_exp2(t.y));
          if (label) {
            if (c0 + j == ylocal) pr.x -= 1.0f;
            if (c0 + j + 1 == ylocal) pr.y -= 1.0f;
          }
          const float2 g = __fmul2_rn(pr, dsc);
          v[j] = g.x;
          v[j + 1] = g.y;
        };
        if (ylocal >= c0 && ylocal < c0 + 32) {
#pragma unroll
          for (int j = 0; j < 32; j += 2) pair(j, true);
        } else {
#pragma unroll
          for (int j = 0; j < 32; j += 2) pair(j, false);
        }
      }
      if (c0 + 32 > ncols) {  // only in the vocabulary's last tile
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (c0 + j >= ncols) v[j] = 0.0f;
      }
      if (live) store_bf16x32(out + c0 / 8, v, p.v8 != 0);
    }
  }
};

// -------------------------------------------------------------------------
// Plain store of D rows (dW chunk rows, or the self-test GEMM's output):
// row r of the tile goes to out[(row0 + r) * ldo + col], as BF16 or FP32.
// `cols` is a multiple of 8.
// -------------------------------------------------------------------------
struct EpiStoreRows {
  struct Params {
    void* out;
    int64_t ldo;
    int64_t rows;
    int64_t cols;
    int f32;
    int v8;      // 1: out and its rows are 32-byte aligned (32-byte stores)
  };

  static __device__ __forceinline__ void tile(const Params& p, uint32_t taddr, int mt, int nt,
                                              int row) {
    const int64_t r = static_cast<int64_t>(mt) * kBM + row;
    const bool live = r < p.rows;
    const int64_t h0 = static_cast<int64_t>(nt) * kBN;
#pragma unroll 1
    for (int c0 = 0; c0 < kBN; c0 += 32) {
      float v[32];
      tmem_load_32cols(taddr + c0, v);
      if (!live) continue;
      if (p.v8 && h0 + c0 + 32 <= p.cols) {  // all 32 columns in range
        if (p.f32) {
          float* o = static_cast<float*>(p.out) + r * p.ldo + h0 + c0;
#pragma unroll
          for (int q = 0; q < 4; ++q)
            st_global_v8(o + 8 * q, __float_as_uint(v[8 * q + 0]), __float_as_uint(v[8 * q + 1]),
                         __float_as_uint(v[8 * q + 2]), __float_as_uint(v[8 * q + 3]),
                         __float_as_uint(v[8 * q + 4]), __float_as_uint(v[8 * q + 5]),
                         __float_as_uint(v[8 * q + 6]), __float_as_uint(v[8 * q + 7]));
        } else {
          store_bf16x32(reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + r * p.ldo +
                                                 h0 + c0),
                        v, true);
        }
        continue;
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int64_t h = h0 + c0 + 8 * q;
        if (h >= p.cols) break;
        if (p.f32) {
          float4* o = reinterpret_cast<float4*>(static_cast<float*>(p.out) + r * p.ldo + h);
          o[0] = make_float4(v[8 * q + 0], v[8 * q + 1], v[8 * q + 2], v[8 * q + 3]);
          o[1] = make_float4(v[8 * q + 4], v[8 * q + 5], v[8 * q + 6], v[8 * q + 7]);
        } else {
          uint4 w;
          w.x = pack_bf16x2(v[8 * q + 0], v[8 * q + 1]);
          w.y = pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
          w.z = pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
          w.w = pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
          *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + r * p.ldo + h) = w;
        }
      }
    }
  }
};

// -------------------------------------------------------------------------
// dhidden accumulation over vocabulary chunks, exclusive per tile:
//   mode 0 (first chunk)  acc32  = D
//   mode 1 (middle)       acc32 += D
//   mode 2 (last)         out    = bf16(acc32 + D)
//   mode 3 (only chunk)   out    = bf16(D)
// -------------------------------------------------------------------------
struct EpiAccumRows {
  struct Params {
    float* acc32;          // [rows][ld]
    __nv_bfloat16* out;    // [rows][ld]
    int64_t ld;
    int64_t rows;
    int64_t cols;          // multiple of 8
    int mode;
    int v8;                // 1: acc32 and its rows are 32-byte aligned (32-byte accesses)
  };

  static __device__ __forceinline__ void tile(const Params& p, uint32_t taddr, int mt, int nt,
                                              int row) {
    const int64_t r = static_cast<int64_t>(mt) * kBM + row;
    const bool live = r < p.rows;
    const int64_t h0 = static_cast<int64_t>(nt) * kBN;
#pragma unroll 1
    for (int c0 = 0; c0 < kBN; c0 += 32) {
      float v[32];
      tmem_load_32cols(taddr + c0, v);
      if (!live) continue;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int64_t h = h0 + c0 + 8 * q;
        if (h >= p.cols) break;
        float* a = p.acc32 + r * p.ld + h;
        float x[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) x[i] = v[8 * q + i];
        if (p.mode == 1 || p.mode == 2) {
          if (p.v8) {
            float y[8];
            ld_global_v8(a, y);
#pragma unroll
            for (int i = 0; i < 8; ++i) x[i] += y[i];
          } else {
            const float4 a0 = reinterpret_cast<const float4*>(a)[0];
            const float4 a1 = reinterpret_cast<const float4*>(a)[1];
            x[0] += a0.x; x[1] += a0.y; x[2] += a0.z; x[3] += a0.w;
            x[4] += a1.x; x[5] += a1.y; x[6] += a1.z; x[7] += a1.w;
          }
        }
        if (p.mode <= 1) {
          if (p.v8) {
            st_global_v8(a, __float_as_uint(x[0]), __float_as_uint(x[1]), __float_as_uint(x[2]),
                         __float_as_uint(x[3]), __float_as_uint(x[4]), __float_as_uint(x[5]),
                         __float_as_uint(x[6]), __float_as_uint(x[7]));
          } else {
            reinterpret_cast<float4*>(a)[0] = make_float4(x[0], x[1], x[2], x[3]);
            reinterpret_cast<float4*>(a)[1] = make_float4(x[4], x[5], x[6], x[7]);
          }
        } else {
          uint4 w;
          w.x = pack_bf16x2(x[0], x[1]);
          w.y = pack_bf16x2(x[2], x[3]);
          w.z = pack_bf16x2(x[4], x[5]);
          w.w = pack_bf16x2(x[6], x[7]);
          *reinterpret_cast<uint4*>(p.out + r * p.ld + h) = w;
        }
      }
    }
  }
};

}  // namespace flce

namespace flce {

// The epilogues a grouped launch may run, selected per problem at run time.
// kKinds is a bit mask of the EpiKind values compiled into the kernel.
template <int kKinds>
struct EpiSet {
  EpiForward::Params fwd;
  EpiGrad::Params grad;
  EpiStoreRows::Params store;
  EpiAccumRows::Params accum;

  static __device__ __forceinline__ void dispatch(int kind, const EpiSet& e, uint32_t taddr,
                                                  int mt, int nt, int row) {
    if ((kKinds & (1 << kEpiForward)) && kind == kEpiForward)
      EpiForward::tile(e.fwd, taddr, mt, nt, row);
    else if ((kKinds & (1 << kEpiGrad)) && kind == kEpiGrad)
      EpiGrad::tile(e.grad, taddr, mt, nt, row);
    else if ((kKinds & (1 << kEpiStoreRows)) && kind == kEpiStoreRows)
      EpiStoreRows::tile(e.store, taddr, mt, nt, row);
    else if ((kKinds & (1 << kEpiAccumRows)) && kind == kEpiAccumRows)
      EpiAccumRows::tile(e.accum, taddr, mt, nt, row);
  }
};

constexpr int kEpiSetForward = 1 << kEpiForward;
constexpr int kEpiSetBackward = (1 << kEpiGrad) | (1 << kEpiStoreRows) | (1 << kEpiAccumRows);
constexpr int kEpiSetStore = 1 << kEpiStoreRows;

}  // namespace flce
