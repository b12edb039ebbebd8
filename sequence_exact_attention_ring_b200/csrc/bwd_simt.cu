// CUDA-core backward pass (fp32 math; fp32 or bf16 inputs; D = 64 or 128; any layout).
//
// The same computation and schedule as the tensor-core backward (RingAttention
// deep-architecture article, techknowgenie, section "activation checkpointing and
// memory recomputation": K/V travel the reverse ring while the map is recomputed from
// the saved statistics), for every shape those kernels do not take: fp32 inputs, head
// dim 64, zigzag shards whose chunks are not whole 128-row tiles. Gradients are the
// chain rule through the forward definition:
//     P = exp(S - lse), dV = P^T dO, dP = dO V^T, Delta = rowsum(dO * O),
//     dS = P * (dP - Delta), dQ = scale dS K, dK = scale dS^T Q.
// Nothing is rounded below fp32 before the output (exp2f, not the approximate unit),
// which is what the fp32 workload's tolerance needs.
//
// dK/dV: one CTA per 32-key tile of a KV shard (the key rows stay in registers); it
//        meets the query rows that see it in 32-row steps, staged in shared memory.
// dQ:    one CTA per 32-row query tile (the rows stay in registers); it walks 32-key
//        tiles in backward-ring order, staged in shared memory.
// 256 threads: 8 per row, each holding D / 8 dims; dot products close with three
// butterfly shuffles inside each group of 8 lanes.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "ring_schedule.h"
#include "ringattn_internal.h"

namespace ringattn {
namespace bwdsimt {

constexpr int TK = 32;
constexpr int TQ = 32;
constexpr int kThreads = 256;

template <typename T>
__device__ __forceinline__ float ld(const T* p);
template <>
__device__ __forceinline__ float ld<float>(const float* p) { return *p; }
template <>
__device__ __forceinline__ float ld<__nv_bfloat16>(const __nv_bfloat16* p) { return __bfloat162float(*p); }

template <typename T>
__device__ __forceinline__ void st(T* p, float x);
template <>
__device__ __forceinline__ void st<float>(float* p, float x) { *p = x; }
template <>
__device__ __forceinline__ void st<__nv_bfloat16>(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

__device__ __forceinline__ float group8_sum(float x) {
  x += __shfl_xor_sync(0xffffffffu, x, 1);
  x += __shfl_xor_sync(0xffffffffu, x, 2);
  x += __shfl_xor_sync(0xffffffffu, x, 4);
  return x;
}

// One warp per padded shard-local query row: lse2 = lse * log2(e), delta = <dO_t, O_t>;
// rows past the shard get +inf and 0 (the layout of the tensor-core path).
template <typename T, int D>
__global__ void __launch_bounds__(256) prep_kernel(const T* __restrict__ out, const T* __restrict__ dout,
                                                   const float* __restrict__ lse, float* __restrict__ lse2,
                                                   float* __restrict__ delta, RingGeom g, int64_t sq_pad,
                                                   int64_t rows) {
  const int64_t row = (int64_t)blockIdx.x * 8 + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (row >= rows) return;
  const int64_t per_bh = (int64_t)g.P * sq_pad;
  const int64_t bh = row / per_bh;
  const int i = (int)((row % per_bh) / sq_pad);
  const int64_t a = row % sq_pad;
  if (a >= g.Sq) {
    if (lane == 0) {
      lse2[row] = INFINITY;
      delta[row] = 0.f;
    }
    return;
  }
  const int64_t t = token_of(g, i, a);
  const int64_t base = (bh * g.S + t) * D;
  float acc = 0.f;
#pragma unroll
  for (int d = lane; d < D; d += 32) acc = fmaf(ld<T>(out + base + d), ld<T>(dout + base + d), acc);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) {
    lse2[row] = lse[bh * g.S + t] * 1.4426950408889634f;
    delta[row] = acc;
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads) dkdv_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                        const T* __restrict__ v, const T* __restrict__ dout,
                                                        const float* __restrict__ lse2,
                                                        const float* __restrict__ delta, T* __restrict__ dk,
                                                        T* __restrict__ dv, RingGeom g, int64_t sq_pad, float scale,
                                                        float scale_log2) {
  constexpr int NE = D / 8;
  __shared__ float Qs[TQ][D + 1];
  __shared__ float Ds[TQ][D + 1];
  __shared__ float Ls[TQ], Dl[TQ];
  __shared__ int64_t Tok[TQ];
  const KvUnit U = decode_kv_unit(g, TK, blockIdx.x);
  const int rep = g.Hq / g.Hkv;
  const int r = threadIdx.x / 8, sub = threadIdx.x % 8;
  const int64_t bk = (int64_t)U.kt * TK + r;
  const bool key_ok = bk < g.Sq;
  const int64_t u = key_ok ? token_of(g, U.j, bk) : 0;
  const int bh_kv = U.b * g.Hkv + U.g;
  float kr[NE], vr[NE], dkr[NE], dvr[NE];
#pragma unroll
  for (int e = 0; e < NE; ++e) {
    const int64_t off = ((int64_t)bh_kv * g.S + u) * D + sub + 8 * e;
    kr[e] = key_ok ? ld<T>(k + off) : 0.f;
    vr[e] = key_ok ? ld<T>(v + off) : 0.f;
    dkr[e] = dvr[e] = 0.f;
  }
  for (QWalk w = qwalk_begin(g, U, TQ, TK); qwalk_valid(w); qwalk_next(g, w, TQ)) {
    const int bh_q = U.b * g.Hq + U.g * rep + w.hr;
    const int64_t a0 = (int64_t)w.qt * TQ;
    __syncthreads();
    for (int x = threadIdx.x; x < TQ * D; x += kThreads) {
      const int c = x / D, d = x % D;
      const int64_t a = a0 + c;
      const bool ok = a < g.Sq;
      const int64_t off = ((int64_t)bh_q * g.S + (ok ? token_of(g, w.i, a) : 0)) * D + d;
      Qs[c][d] = ok ? ld<T>(q + off) : 0.f;
      Ds[c][d] = ok ? ld<T>(dout + off) : 0.f;
    }
    if (threadIdx.x < TQ) {
      const int c = threadIdx.x;
      const int64_t a = a0 + c;
      const int64_t stat = ((int64_t)bh_q * g.P + w.i) * sq_pad + a;  // a < sq_pad: padded to 128 rows
      Ls[c] = lse2[stat];
      Dl[c] = delta[stat];
      Tok[c] = a < g.Sq ? token_of(g, w.i, a) : -1;
    }
    __syncthreads();
#pragma unroll 2
    for (int c = 0; c < TQ; ++c) {
      float sp = 0.f, dpp = 0.f;
#pragma unroll
      for (int e = 0; e < NE; ++e) {
        sp = fmaf(kr[e], Qs[c][sub + 8 * e], sp);
        dpp = fmaf(vr[e], Ds[c][sub + 8 * e], dpp);
      }
      sp = group8_sum(sp);
      dpp = group8_sum(dpp);
      const bool allowed = key_ok && Tok[c] >= 0 && (!g.causal || u <= Tok[c]);
      const float p = allowed ? exp2f(fmaf(sp, scale_log2, -Ls[c])) : 0.f;
      const float ds = p * (dpp - Dl[c]);
#pragma unroll
      for (int e = 0; e < NE; ++e) {
        dvr[e] = fmaf(p, Ds[c][sub + 8 * e], dvr[e]);
        dkr[e] = fmaf(ds, Qs[c][sub + 8 * e], dkr[e]);
      }
    }
  }
  if (key_ok) {
#pragma unroll
    for (int e = 0; e < NE; ++e) {
      const int64_t off = ((int64_t)bh_kv * g.S + u) * D + sub + 8 * e;
      st<T>(dk + off, dkr[e] * scale);
      st<T>(dv + off, dvr[e]);
    }
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads) dq_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                      const T* __restrict__ v, const T* __restrict__ dout,
                                                      const float* __restrict__ lse2, const float* __restrict__ delta,
                                                      T* __restrict__ dq, RingGeom g, int64_t sq_pad, float scale,
                                                      float scale_log2) {
  constexpr int NE = D / 8;
  __shared__ float Ks[TK][D + 1];
  __shared__ float Vs[TK][D + 1];
  const Unit U = decode_unit(g, TQ, -1, blockIdx.x);
  const int64_t a0 = (int64_t)U.tb * TQ;
  const int64_t a_hi = (a0 + TQ - 1 < g.Sq - 1) ? a0 + TQ - 1 : g.Sq - 1;
  const int bh_q = U.b * g.Hq + U.h;
  const int bh_kv = U.b * g.Hkv + U.h / (g.Hq / g.Hkv);
  const int r = threadIdx.x / 8, sub = threadIdx.x % 8;
  const int64_t a = a0 + r;
  const bool row_ok = a < g.Sq;
  const int64_t t = row_ok ? token_of(g, U.i, a) : 0;
  const int64_t stat = ((int64_t)bh_q * g.P + U.i) * sq_pad + a;
  const float row_lse2 = lse2[stat];
  const float row_delta = delta[stat];
  float qr[NE], dor[NE], dqr[NE];
#pragma unroll
  for (int e = 0; e < NE; ++e) {
    const int64_t off = ((int64_t)bh_q * g.S + t) * D + sub + 8 * e;
    qr[e] = row_ok ? ld<T>(q + off) : 0.f;
    dor[e] = row_ok ? ld<T>(dout + off) : 0.f;
    dqr[e] = 0.f;
  }
  for (TileWalk w = walk_begin_rev(g, U.i, a_hi, TK, launch_anchor(g, -1)); walk_valid(w); walk_next(g, w, a_hi, TK)) {
    __syncthreads();
    for (int x = threadIdx.x; x < TK * D; x += kThreads) {
      const int c = x / D, d = x % D;
      const int64_t bb = (int64_t)w.kb * TK + c;
      const bool ok = bb < g.Sq;
      const int64_t off = ((int64_t)bh_kv * g.S + (ok ? token_of(g, w.j, bb) : 0)) * D + d;
      Ks[c][d] = ok ? ld<T>(k + off) : 0.f;
      Vs[c][d] = ok ? ld<T>(v + off) : 0.f;
    }
    __syncthreads();
    const int64_t lim = row_ok ? key_limit(g, U.i, w.j, a) : 0;
#pragma unroll 2
    for (int c = 0; c < TK; ++c) {
      float sp = 0.f, dpp = 0.f;
#pragma unroll
      for (int e = 0; e < NE; ++e) {
        sp = fmaf(qr[e], Ks[c][sub + 8 * e], sp);
        dpp = fmaf(dor[e], Vs[c][sub + 8 * e], dpp);
      }
      sp = group8_sum(sp);
      dpp = group8_sum(dpp);
      const bool allowed = (int64_t)w.kb * TK + c < lim;
      const float p = allowed ? exp2f(fmaf(sp, scale_log2, -row_lse2)) : 0.f;
      const float ds = p * (dpp - row_delta);
#pragma unroll
      for (int e = 0; e < NE; ++e) dqr[e] = fmaf(ds, Ks[c][sub + 8 * e], dqr[e]);
    }
  }
  if (row_ok) {
#pragma unroll
    for (int e = 0; e < NE; ++e) st<T>(dq + ((int64_t)bh_q * g.S + t) * D + sub + 8 * e, dqr[e] * scale);
  }
}

template <typename T, int D>
static int launch(const void* q, const void* k, const void* v, const void* out, const float* lse, const void* dout,
                  void* dq, void* dk, void* dv, const RingGeom& g, float scale, float* stats, cudaStream_t stream) {
  const int64_t sq_pad = bwd_sq_pad(g);
  const int64_t rows = (int64_t)g.B * g.Hq * g.P * sq_pad;
  float* lse2 = stats;
  float* delta = stats + rows;
  const int64_t prep_blocks = (rows + 7) / 8;
  const int64_t kv_units = num_kv_units(g, TK);
  const int64_t q_units = num_units(g, TQ, -1);
  if (prep_blocks > 0x7fffffff || kv_units > 0x7fffffff || q_units > 0x7fffffff) return RING_ATTN_EINVAL;
  const float scale_log2 = scale * 1.4426950408889634f;
  prep_kernel<T, D><<<(unsigned)prep_blocks, 256, 0, stream>>>(static_cast<const T*>(out), static_cast<const T*>(dout),
                                                               lse, lse2, delta, g, sq_pad, rows);
  dkdv_kernel<T, D><<<(unsigned)kv_units, kThreads, 0, stream>>>(
      static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v), static_cast<const T*>(dout), lse2,
      delta, static_cast<T*>(dk), static_cast<T*>(dv), g, sq_pad, scale, scale_log2);
  dq_kernel<T, D><<<(unsigned)q_units, kThreads, 0, stream>>>(
      static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v), static_cast<const T*>(dout), lse2,
      delta, static_cast<T*>(dq), g, sq_pad, scale, scale_log2);
  return cudaGetLastError() == cudaSuccess ? RING_ATTN_OK : RING_ATTN_ECUDA;
}

}  // namespace bwdsimt

int launch_bwd_simt(const void* q, const void* k, const void* v, const void* out, const float* lse, const void* dout,
                    void* dq, void* dk, void* dv, const RingGeom& g, float scale, int dtype, float* stats,
                    cudaStream_t stream) {
  using namespace bwdsimt;
  if (dtype == RING_ATTN_DTYPE_FP32) {
    if (g.D == 128) return launch<float, 128>(q, k, v, out, lse, dout, dq, dk, dv, g, scale, stats, stream);
    if (g.D == 64) return launch<float, 64>(q, k, v, out, lse, dout, dq, dk, dv, g, scale, stats, stream);
  } else {
    if (g.D == 128) return launch<__nv_bfloat16, 128>(q, k, v, out, lse, dout, dq, dk, dv, g, scale, stats, stream);
    if (g.D == 64) return launch<__nv_bfloat16, 64>(q, k, v, out, lse, dout, dq, dk, dv, g, scale, stats, stream);
  }
  return RING_ATTN_EUNSUPPORTED;
}

}  // namespace ringattn
