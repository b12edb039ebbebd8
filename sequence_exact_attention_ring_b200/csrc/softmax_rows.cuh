// Row-wise pieces of the online softmax shared by the fused kernels. A softmax
// thread owns one query row, or one half of its key columns; its scores for a
// block of keys sit in registers as raw fp32 bits loaded from tensor memory.
//
// The update follows the RingAttention deep-architecture article (techknowgenie),
// section 3: m_new = max(m_old, rowmax S), alpha = exp(m_old - m_new),
// P = exp(S - m_new), l = l*alpha + rowsum P, O = O*alpha + P V, in base 2 with
// scale*log2(e) folded in, and with the reference maximum moved only when the
// block maximum exceeds it by more than kRescaleLog2. The tensor-core kernels first
// exponentiate a block against the current reference and keep the result when every
// row sum stays <= 2^20 (finite); only then do they take the block maximum.
#pragma once

#include <math.h>
#include <stdint.h>

#include "sm100_ptx.cuh"

namespace ringattn {

constexpr float kRescaleLog2 = 8.0f;

// Number of keys of the block starting at key kb0 that are visible (keys < lim), in [0, N].
template <int N>
__device__ __forceinline__ int visible_keys(int64_t kb0, int64_t lim) {
  const int64_t v = lim - kb0;
  return v <= 0 ? 0 : (v >= N ? N : (int)v);
}

// Masks block-local keys c >= cut to -inf (a no-op when cut == N).
template <int N>
__device__ __forceinline__ void mask_scores(uint32_t (&sr)[N], int cut) {
  if (cut < N) {
#pragma unroll
    for (int c = 0; c < N; ++c) sr[c] = c < cut ? sr[c] : 0xff800000u;  // -inf
  }
}

// Maximum of N raw scores (N a multiple of 16): independent chains of three-input max.
template <int N>
__device__ __forceinline__ float raw_rowmax(const uint32_t (&sr)[N]) {
  constexpr int kChains = N / 16;
  float mx[kChains];
#pragma unroll
  for (int ch = 0; ch < kChains; ++ch) {
    const uint32_t* v = &sr[ch * 16];
    float m = fmax3(__uint_as_float(v[0]), __uint_as_float(v[1]), __uint_as_float(v[2]));
#pragma unroll
    for (int e = 3; e < 15; e += 2) m = fmax3(m, __uint_as_float(v[e]), __uint_as_float(v[e + 1]));
    mx[ch] = fmaxf(m, __uint_as_float(v[15]));
  }
  float r = mx[0];
#pragma unroll
  for (int ch = 1; ch + 1 < kChains; ch += 2) r = fmax3(r, mx[ch], mx[ch + 1]);
  if (kChains % 2 == 0) r = fmaxf(r, mx[kChains - 1]);
  return r;
}

// p = 2^(s*scale_log2 - m) for N raw scores; packs P to bf16 pairs and returns
// the fp32 row sum. Of every 8 column pairs, kEmu take 2^x from the FMA-pipe
// polynomial and the rest from MUFU ex2.
template <int N, int kEmu>
__device__ __forceinline__ float exp_pack(const uint32_t (&sr)[N], float scale_log2, float m_sub,
                                          uint32_t (&pk)[N / 2]) {
  const uint64_t c2 = f2_splat(scale_log2);
  const uint64_t negm = f2_splat(-m_sub);
  uint64_t acc[4] = {0, 0, 0, 0};
#pragma unroll
  for (int c = 0; c < N; c += 2) {
    const uint64_t xy = f2_fma(f2_pack(sr[c], sr[c + 1]), c2, negm);
    uint64_t pp;
    if ((c / 2) % 8 < kEmu) {
      pp = exp2_poly2(xy);
    } else {
      float x0, x1;
      f2_unpack(xy, x0, x1);
      pp = f2_pack(__float_as_uint(ex2_approx(x0)), __float_as_uint(ex2_approx(x1)));
    }
    acc[(c / 2) % 4] = f2_add(acc[(c / 2) % 4], pp);
    float p0, p1;
    f2_unpack(pp, p0, p1);
    pk[c / 2] = pack_bf16x2(p0, p1);
  }
  const uint64_t t = f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3]));
  float t0, t1;
  f2_unpack(t, t0, t1);
  return t0 + t1;
}

// The same result as exp_pack, written in three phases over all N scores: every
// exponent argument first (packed FMA), then every 2^x back to back, then the bf16
// packing and the row sum. The exponentials of a thread are independent, so the
// phases give the scheduler long runs of independent special-function operations
// instead of short dependent chains per column pair. Of every 8 column pairs, kEmu
// take 2^x from the FMA-pipe polynomial (interleaved with the MUFU operations).
template <int N, int kEmu>
__device__ __forceinline__ float exp_pack_phased(uint32_t (&sr)[N], float scale_log2, float m_sub,
                                                 uint32_t (&pk)[N / 2]) {
  const uint64_t c2 = f2_splat(scale_log2);
  const uint64_t negm = f2_splat(-m_sub);
#pragma unroll
  for (int c = 0; c < N; c += 2) {
    const uint64_t xy = f2_fma(f2_pack(sr[c], sr[c + 1]), c2, negm);
    float x0, x1;
    f2_unpack(xy, x0, x1);
    sr[c] = __float_as_uint(x0);
    sr[c + 1] = __float_as_uint(x1);
  }
#pragma unroll
  for (int c = 0; c < N; c += 2) {
    if ((c / 2) % 8 < kEmu) {
      float p0, p1;
      f2_unpack(exp2_poly2(f2_pack(sr[c], sr[c + 1])), p0, p1);
      sr[c] = __float_as_uint(p0);
      sr[c + 1] = __float_as_uint(p1);
    } else {
      sr[c] = __float_as_uint(ex2_approx(__uint_as_float(sr[c])));
      sr[c + 1] = __float_as_uint(ex2_approx(__uint_as_float(sr[c + 1])));
    }
  }
  uint64_t acc[4] = {0, 0, 0, 0};
#pragma unroll
  for (int c = 0; c < N; c += 2) {
    acc[(c / 2) % 4] = f2_add(acc[(c / 2) % 4], f2_pack(sr[c], sr[c + 1]));
    pk[c / 2] = pack_bf16x2(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1]));
  }
  const uint64_t t = f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3]));
  float t0, t1;
  f2_unpack(t, t0, t1);
  return t0 + t1;
}

// Multiplies kCols accumulator columns of this warp's 32 rows in tensor memory by
// each lane's alpha (1 for rows that keep their reference maximum).
template <int kCols>
__device__ __forceinline__ void rescale_o(uint32_t tO, float alpha) {
#pragma unroll 1
  for (int c = 0; c < kCols / 32; ++c) {
    uint32_t o[32];
    tmem_ld32(tO + c * 32, o);
    tmem_wait_ld();
#pragma unroll
    for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
    tmem_st32(tO + c * 32, o);
  }
  tmem_wait_st();
}

// Final O / l of kCols accumulator columns of one row, written to columns
// [col0, col0 + kCols) of an output row of row_stride elements: bf16 (natural token
// order) or fp32 partial (shard order). All lanes execute the tensor-memory loads;
// only rows that exist are stored.
template <int kCols>
__device__ __forceinline__ void store_row_cols(uint32_t tO, bool have_acc, bool row_ok, float inv_l, bool partial,
                                               void* out, int64_t out_row, int row_stride, int col0) {
#pragma unroll 1
  for (int c = 0; c < kCols / 32; ++c) {
    uint32_t o[32];
    if (have_acc) {
      tmem_ld32(tO + c * 32, o);
      tmem_wait_ld();
    }
    if (!row_ok) continue;
    const int64_t base = out_row * row_stride + col0 + c * 32;
    if (partial) {
      float* dst = reinterpret_cast<float*>(out) + base;
#pragma unroll
      for (int e = 0; e < 32; e += 4) {
        float4 v4;
        v4.x = have_acc ? __uint_as_float(o[e]) * inv_l : 0.f;
        v4.y = have_acc ? __uint_as_float(o[e + 1]) * inv_l : 0.f;
        v4.z = have_acc ? __uint_as_float(o[e + 2]) * inv_l : 0.f;
        v4.w = have_acc ? __uint_as_float(o[e + 3]) * inv_l : 0.f;
        *reinterpret_cast<float4*>(dst + e) = v4;
      }
    } else {
      uint32_t* dst = reinterpret_cast<uint32_t*>(reinterpret_cast<uint16_t*>(out) + base);
#pragma unroll
      for (int e = 0; e < 32; e += 8) {
        uint4 v4;
        v4.x = pack_bf16x2(__uint_as_float(o[e]) * inv_l, __uint_as_float(o[e + 1]) * inv_l);
        v4.y = pack_bf16x2(__uint_as_float(o[e + 2]) * inv_l, __uint_as_float(o[e + 3]) * inv_l);
        v4.z = pack_bf16x2(__uint_as_float(o[e + 4]) * inv_l, __uint_as_float(o[e + 5]) * inv_l);
        v4.w = pack_bf16x2(__uint_as_float(o[e + 6]) * inv_l, __uint_as_float(o[e + 7]) * inv_l);
        *reinterpret_cast<uint4*>(dst + e / 2) = v4;
      }
    }
  }
}

// Final O / l of a whole row of D columns.
template <int D>
__device__ __forceinline__ void store_row(uint32_t tO, bool have_acc, bool row_ok, float inv_l, bool partial,
                                          void* out, int64_t out_row) {
  store_row_cols<D>(tO, have_acc, row_ok, inv_l, partial, out, out_row, D, 0);
}

// Weights of a running normalised state (lse_a) and of a new normalised partial
// (lse_s) in their merge: the online-softmax rescale of the RingAttention
// deep-architecture article (techknowgenie), section 3, applied to states whose l is
// already divided out. lse = ln(e^lse_a + e^lse_s); an empty side (-inf) gets weight
// 0; both empty give lse = -inf and weights 0.
__device__ __forceinline__ void fold_weights(float lse_a, float lse_s, float& wa, float& ws, float& lse) {
  wa = 0.f;
  ws = 0.f;
  lse = -INFINITY;
  if (lse_a != -INFINITY || lse_s != -INFINITY) {
    const float mx = fmaxf(lse_a, lse_s);
    const float ea = expf(lse_a - mx);
    const float es = expf(lse_s - mx);
    const float sum = ea + es;
    lse = mx + logf(sum);
    wa = ea / sum;
    ws = es / sum;
  }
}

// Folds one row's result of a ring step into the running state (shard-local row
// `row`): o = wa * acc_o + ws * (O / l), lse = ln(e^lse_acc + e^lse_step). On the
// first step the state is this step's row; on the last step the merged row goes to
// `out` (bf16) and `lse_out` instead of the state. A row this step adds nothing to
// (lse_step = -inf) leaves the state untouched. All lanes execute the tensor-memory
// loads; only rows that exist are read and written.
template <int D>
__device__ __forceinline__ void fold_row(uint32_t tO, bool have_acc, bool row_ok, float inv_l, float lse_step,
                                         bool first, bool last, float* acc_o, float* acc_lse, void* out,
                                         float* lse_out, int64_t row) {
  const float lse_a = (first || !row_ok) ? -INFINITY : acc_lse[row];
  float wa, ws, lse;
  fold_weights(lse_a, lse_step, wa, ws, lse);
  const bool write = row_ok && (first || last || lse_step != -INFINITY);
  const float wsl = ws * inv_l;
#pragma unroll 1
  for (int c = 0; c < D / 32; ++c) {
    uint32_t o[32];
    if (have_acc) {
      tmem_ld32(tO + c * 32, o);
      tmem_wait_ld();
    }
    if (!write) continue;
    const int64_t base = row * D + c * 32;
    float v[32];
#pragma unroll
    for (int e = 0; e < 32; e += 4) {
      const float4 a4 = first ? make_float4(0.f, 0.f, 0.f, 0.f) : *reinterpret_cast<const float4*>(acc_o + base + e);
      v[e] = wa * a4.x + (have_acc ? wsl * __uint_as_float(o[e]) : 0.f);
      v[e + 1] = wa * a4.y + (have_acc ? wsl * __uint_as_float(o[e + 1]) : 0.f);
      v[e + 2] = wa * a4.z + (have_acc ? wsl * __uint_as_float(o[e + 2]) : 0.f);
      v[e + 3] = wa * a4.w + (have_acc ? wsl * __uint_as_float(o[e + 3]) : 0.f);
    }
    if (last) {
      uint32_t* dst = reinterpret_cast<uint32_t*>(reinterpret_cast<uint16_t*>(out) + base);
#pragma unroll
      for (int e = 0; e < 32; e += 8) {
        uint4 v4;
        v4.x = pack_bf16x2(v[e], v[e + 1]);
        v4.y = pack_bf16x2(v[e + 2], v[e + 3]);
        v4.z = pack_bf16x2(v[e + 4], v[e + 5]);
        v4.w = pack_bf16x2(v[e + 6], v[e + 7]);
        *reinterpret_cast<uint4*>(dst + e / 2) = v4;
      }
    } else {
#pragma unroll
      for (int e = 0; e < 32; e += 4)
        *reinterpret_cast<float4*>(acc_o + base + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
    }
  }
  if (write) {
    if (last)
      lse_out[row] = lse;
    else
      acc_lse[row] = lse;
  }
}

}  // namespace ringattn
