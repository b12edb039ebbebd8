// Merge of normalised partial attention results (HBM-bound, vectorised).
//
// A partial k covers a subset of the keys of a row and holds O_k = (its softmax
// weights) * V and lse_k = ln(sum of its exponentials). The online-softmax rescale
// of the RingAttention deep-architecture article (techknowgenie), section 3
// (alpha = exp(m_old - m_new), beta = exp(m_block - m_new)) applied to such
// normalised states gives
//     lse = lse_max + ln sum_k exp(lse_k - lse_max),   O = sum_k exp(lse_k - lse) O_k.
// Empty partials (lse_k = -inf) get weight 0; an all-empty row yields O = 0, lse = -inf.
//
// Each thread owns 8 consecutive columns of one row: two 16-byte fp32 loads per
// partial, one 16-byte bf16 store (or two fp32 stores) per row chunk. When there are
// few rows and many partials (decode), merge_wide_kernel splits the partials of a row
// across a block instead.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "ringattn_internal.h"

namespace ringattn {
namespace merge {

constexpr int kThreads = 256;
constexpr int kVec = 8;

template <bool kBf16Out>
__global__ void __launch_bounds__(kThreads) merge_kernel(const float* __restrict__ o_parts,
                                                         const float* __restrict__ lse_parts, int n_parts,
                                                         int64_t rows, int D, void* __restrict__ out,
                                                         float* __restrict__ lse_out) {
  const int tpr = D / kVec;  // threads per row
  const int rows_per_block = kThreads / tpr;
  const int64_t row = (int64_t)blockIdx.x * rows_per_block + threadIdx.x / tpr;
  const int col = (threadIdx.x % tpr) * kVec;
  if (threadIdx.x >= rows_per_block * tpr || row >= rows) return;

  float mx = -INFINITY;
  for (int k = 0; k < n_parts; ++k) mx = fmaxf(mx, __ldg(lse_parts + (int64_t)k * rows + row));
  float acc[kVec];
#pragma unroll
  for (int e = 0; e < kVec; ++e) acc[e] = 0.f;
  float lse_v = -INFINITY;
  if (mx != -INFINITY) {
    float tot = 0.f;
    for (int k = 0; k < n_parts; ++k) {
      const float lk = __ldg(lse_parts + (int64_t)k * rows + row);
      if (lk == -INFINITY) continue;
      const float wk = expf(lk - mx);
      tot += wk;
      const float4* src = reinterpret_cast<const float4*>(o_parts + ((int64_t)k * rows + row) * D + col);
      const float4 x0 = __ldg(src);
      const float4 x1 = __ldg(src + 1);
      acc[0] = fmaf(wk, x0.x, acc[0]);
      acc[1] = fmaf(wk, x0.y, acc[1]);
      acc[2] = fmaf(wk, x0.z, acc[2]);
      acc[3] = fmaf(wk, x0.w, acc[3]);
      acc[4] = fmaf(wk, x1.x, acc[4]);
      acc[5] = fmaf(wk, x1.y, acc[5]);
      acc[6] = fmaf(wk, x1.z, acc[6]);
      acc[7] = fmaf(wk, x1.w, acc[7]);
    }
    const float inv = 1.f / tot;
#pragma unroll
    for (int e = 0; e < kVec; ++e) acc[e] *= inv;
    lse_v = mx + logf(tot);
  }
  if (kBf16Out) {
    __nv_bfloat162 h[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) h[e] = __floats2bfloat162_rn(acc[2 * e], acc[2 * e + 1]);
    *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(out) + row * D + col) =
        *reinterpret_cast<const uint4*>(h);
  } else {
    float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(out) + row * D + col);
    dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
  }
  if (threadIdx.x % tpr == 0) lse_out[row] = lse_v;
}

// The same merge for few rows with many partials (a decode step: B*Hq rows, hundreds
// of split-KV parts). One block per row; its threads form groups of D/8, group g
// folds parts g, g + groups, ... with its own running maximum (rescaling its sum and
// accumulator when the maximum grows), and group 0 combines the groups' states by the
// same rescale.
template <bool kBf16Out>
__global__ void __launch_bounds__(kThreads) merge_wide_kernel(const float* __restrict__ o_parts,
                                                              const float* __restrict__ lse_parts, int n_parts,
                                                              int64_t rows, int D, void* __restrict__ out,
                                                              float* __restrict__ lse_out) {
  __shared__ float s_m[kThreads];
  __shared__ float s_t[kThreads];
  __shared__ float s_acc[kThreads * kVec];
  const int tpr = D / kVec;
  const int groups = kThreads / tpr;
  const int g = threadIdx.x / tpr;
  const int col = (threadIdx.x % tpr) * kVec;
  const int64_t row = blockIdx.x;
  float m = -INFINITY, tot = 0.f, acc[kVec];
#pragma unroll
  for (int e = 0; e < kVec; ++e) acc[e] = 0.f;
  if (g < groups) {
    for (int k = g; k < n_parts; k += groups) {
      const float lk = __ldg(lse_parts + (int64_t)k * rows + row);
      if (lk == -INFINITY) continue;
      if (lk > m) {
        const float sc = (m == -INFINITY) ? 0.f : expf(m - lk);
        tot *= sc;
#pragma unroll
        for (int e = 0; e < kVec; ++e) acc[e] *= sc;
        m = lk;
      }
      const float wk = expf(lk - m);
      tot += wk;
      const float4* src = reinterpret_cast<const float4*>(o_parts + ((int64_t)k * rows + row) * D + col);
      const float4 x0 = __ldg(src);
      const float4 x1 = __ldg(src + 1);
      acc[0] = fmaf(wk, x0.x, acc[0]);
      acc[1] = fmaf(wk, x0.y, acc[1]);
      acc[2] = fmaf(wk, x0.z, acc[2]);
      acc[3] = fmaf(wk, x0.w, acc[3]);
      acc[4] = fmaf(wk, x1.x, acc[4]);
      acc[5] = fmaf(wk, x1.y, acc[5]);
      acc[6] = fmaf(wk, x1.z, acc[6]);
      acc[7] = fmaf(wk, x1.w, acc[7]);
    }
  }
  s_m[threadIdx.x] = m;
  s_t[threadIdx.x] = tot;
#pragma unroll
  for (int e = 0; e < kVec; ++e) s_acc[threadIdx.x * kVec + e] = acc[e];
  __syncthreads();
  if (g != 0) return;
  const int lane_col = threadIdx.x;  // group 0: thread index == column slot
  float M = -INFINITY;
  for (int x = 0; x < groups; ++x) M = fmaxf(M, s_m[x * tpr + lane_col]);
  float res[kVec];
#pragma unroll
  for (int e = 0; e < kVec; ++e) res[e] = 0.f;
  float lse_v = -INFINITY;
  if (M != -INFINITY) {
    float T = 0.f;
    for (int x = 0; x < groups; ++x) {
      const int t = x * tpr + lane_col;
      if (s_m[t] == -INFINITY) continue;
      const float w = expf(s_m[t] - M);
      T += w * s_t[t];
#pragma unroll
      for (int e = 0; e < kVec; ++e) res[e] = fmaf(w, s_acc[t * kVec + e], res[e]);
    }
    const float inv = 1.f / T;
#pragma unroll
    for (int e = 0; e < kVec; ++e) res[e] *= inv;
    lse_v = M + logf(T);
  }
  if (kBf16Out) {
    __nv_bfloat162 h[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) h[e] = __floats2bfloat162_rn(res[2 * e], res[2 * e + 1]);
    *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(out) + row * D + col) =
        *reinterpret_cast<const uint4*>(h);
  } else {
    float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(out) + row * D + col);
    dst[0] = make_float4(res[0], res[1], res[2], res[3]);
    dst[1] = make_float4(res[4], res[5], res[6], res[7]);
  }
  if (lane_col == 0) lse_out[row] = lse_v;
}

}  // namespace merge

int launch_merge(const float* o_parts, const float* lse_parts, int n_parts, int64_t rows, int D, void* out,
                 float* lse_out, int out_dtype, cudaStream_t stream) {
  if (rows == 0) return RING_ATTN_OK;
  const int tpr = D / merge::kVec;
  // few rows, many parts: one block per row, the parts split across its threads
  if (rows * tpr < 148 * merge::kThreads && n_parts >= 16 && rows <= 0x7fffffff) {
    if (out_dtype == RING_ATTN_DTYPE_BF16)
      merge::merge_wide_kernel<true><<<(unsigned)rows, merge::kThreads, 0, stream>>>(o_parts, lse_parts, n_parts,
                                                                                      rows, D, out, lse_out);
    else
      merge::merge_wide_kernel<false><<<(unsigned)rows, merge::kThreads, 0, stream>>>(o_parts, lse_parts, n_parts,
                                                                                       rows, D, out, lse_out);
    return cudaGetLastError() == cudaSuccess ? RING_ATTN_OK : RING_ATTN_ECUDA;
  }
  const int rows_per_block = merge::kThreads / tpr;
  const int64_t blocks = (rows + rows_per_block - 1) / rows_per_block;
  if (blocks > 0x7fffffff) return RING_ATTN_EINVAL;
  if (out_dtype == RING_ATTN_DTYPE_BF16)
    merge::merge_kernel<true><<<(unsigned)blocks, merge::kThreads, 0, stream>>>(o_parts, lse_parts, n_parts, rows,
                                                                                 D, out, lse_out);
  else
    merge::merge_kernel<false><<<(unsigned)blocks, merge::kThreads, 0, stream>>>(o_parts, lse_parts, n_parts,
                                                                                  rows, D, out, lse_out);
  return cudaGetLastError() == cudaSuccess ? RING_ATTN_OK : RING_ATTN_ECUDA;
}

}  // namespace ringattn
