// fp32-accumulating CUDA-core ring-attention forward (fp32 or bf16 inputs).
//
// It runs the same unit schedule and masks as the tensor-core kernel and follows
// the code form of the RingAttention deep-architecture article (techknowgenie),
// section 5 listing: per KV block, m_new = max(m, rowmax S), alpha = exp(m - m_new),
// P = exp(S - m_new), l = l*alpha + rowsum P, O = O*alpha + P V, final O / l.
// Everything stays fp32 (P is not rounded), which is what the fp32 workload's
// 1e-5 tolerance needs; tf32 tensor cores cannot meet it.
//
// CTA = 64 query rows of one shard of one head, 256 threads; 4 threads per row.
// KV tiles of 32 keys are staged in shared memory as fp32.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "ring_schedule.h"
#include "ringattn_internal.h"

namespace ringattn {
namespace simt {

constexpr int BQ = 64;
constexpr int BK = 32;
constexpr int kThreads = 256;

template <int D>
struct Smem {
  static constexpr int kQStride = D + 4;
  static constexpr int kKStride = D + 1;
  static constexpr int kPStride = BK + 1;
  static constexpr int kBytes = (BQ * kQStride + BK * kKStride + BK * D + BQ * kPStride) * 4;
};

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ void store_out(T* p, float x);
template <>
__device__ __forceinline__ void store_out<float>(float* p, float x) { *p = x; }
template <>
__device__ __forceinline__ void store_out<__nv_bfloat16>(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

struct Params {
  RingGeom g;
  void* out;
  float* lse;
  float scale;
  int s_begin, s_end, q_shard_only;
  FwdOut fo;
};

// Row of local index a of shard i in a [B, H, ., D] input: the whole sequence in token
// order, or (local) a single shard in shard-local order.
__device__ __forceinline__ int64_t input_row(const RingGeom& g, bool local, int bh, int i, int64_t a) {
  return local ? (int64_t)bh * g.Sq + a : (int64_t)bh * g.S + token_of(g, i, a);
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads) ring_fwd_simt_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                                 const T* __restrict__ v, const Params p) {
  using L = Smem<D>;
  extern __shared__ float sm[];
  float* Qs = sm;
  float* Ks = Qs + BQ * L::kQStride;
  float* Vs = Ks + BK * L::kKStride;
  float* Ps = Vs + BK * D;

  const RingGeom& g = p.g;
  const Unit U = decode_unit(g, BQ, p.q_shard_only, blockIdx.x);
  const int64_t a0 = (int64_t)U.tb * BQ;
  const int64_t a_hi = (a0 + BQ - 1 < g.Sq - 1) ? a0 + BQ - 1 : g.Sq - 1;
  const int bh_q = U.b * g.Hq + U.h;
  const int bh_kv = U.b * g.Hkv + U.h / (g.Hq / g.Hkv);
  const int tid = threadIdx.x;
  const int rr = tid / 4;   // query row within the tile
  const int sub = tid % 4;  // which quarter of the keys / columns
  const int64_t a = a0 + rr;

  for (int e = tid; e < BQ * D; e += kThreads) {
    const int r = e / D, d = e % D;
    const int64_t aa = a0 + r;
    float val = 0.f;
    if (aa < g.Sq) val = to_f32<T>(q[input_row(g, p.fo.local, bh_q, U.i, aa) * D + d]);
    Qs[r * L::kQStride + d] = val;
  }

  constexpr int NC = D / 4;  // output columns per thread: sub + 4*e
  float o[NC];
#pragma unroll
  for (int e = 0; e < NC; ++e) o[e] = 0.f;
  float m = -INFINITY, l = 0.f;

  TileWalk w = walk_begin(g, U.i, a_hi, BK, p.s_begin, p.s_end, launch_anchor(g, p.q_shard_only));
  for (; walk_valid(w); walk_next(g, w, a_hi, BK)) {
    __syncthreads();
    for (int e = tid; e < BK * D; e += kThreads) {
      const int c = e / D, d = e % D;
      const int64_t b = (int64_t)w.kb * BK + c;
      float kv = 0.f, vv = 0.f;
      if (b < g.Sq) {
        const int64_t off = input_row(g, p.fo.local, bh_kv, w.j, b) * D + d;
        kv = to_f32<T>(k[off]);
        vv = to_f32<T>(v[off]);
      }
      Ks[c * L::kKStride + d] = kv;
      Vs[c * D + d] = vv;
    }
    __syncthreads();

    float x[BK / 4];
#pragma unroll
    for (int t = 0; t < BK / 4; ++t) x[t] = 0.f;
    for (int d = 0; d < D; ++d) {
      const float qd = Qs[rr * L::kQStride + d];
#pragma unroll
      for (int t = 0; t < BK / 4; ++t) x[t] = fmaf(qd, Ks[(sub + 4 * t) * L::kKStride + d], x[t]);
    }
    const int64_t lim = key_limit(g, U.i, w.j, a);
    float mblk = -INFINITY;
#pragma unroll
    for (int t = 0; t < BK / 4; ++t) {
      const int64_t b = (int64_t)w.kb * BK + sub + 4 * t;
      x[t] = (b < lim) ? x[t] * p.scale : -INFINITY;
      mblk = fmaxf(mblk, x[t]);
    }
    mblk = fmaxf(mblk, __shfl_xor_sync(0xffffffffu, mblk, 1));
    mblk = fmaxf(mblk, __shfl_xor_sync(0xffffffffu, mblk, 2));
    const float m_new = fmaxf(m, mblk);
    const float alpha = (m == -INFINITY) ? 0.f : expf(m - m_new);
    const float msub = (m_new == -INFINITY) ? 0.f : m_new;
    float rs = 0.f;
#pragma unroll
    for (int t = 0; t < BK / 4; ++t) {
      const float pe = expf(x[t] - msub);
      rs += pe;
      Ps[rr * L::kPStride + sub + 4 * t] = pe;
    }
    rs += __shfl_xor_sync(0xffffffffu, rs, 1);
    rs += __shfl_xor_sync(0xffffffffu, rs, 2);
    l = l * alpha + rs;
    m = m_new;
#pragma unroll
    for (int e = 0; e < NC; ++e) o[e] *= alpha;
    __syncthreads();
    for (int c = 0; c < BK; ++c) {
      const float pc = Ps[rr * L::kPStride + c];
#pragma unroll
      for (int e = 0; e < NC; ++e) o[e] = fmaf(pc, Vs[c * D + sub + 4 * e], o[e]);
    }
  }

  if (a >= g.Sq) return;
  const bool empty = !(l > 0.f);
  const float inv_l = empty ? 0.f : 1.f / l;
  const float lse_v = empty ? -INFINITY : m + logf(l);
  if (p.fo.kind == kOutFold) {
    // fold this step's row into the running state (weights as in fold_weights of the
    // tensor-core kernels: lse = ln(e^lse_acc + e^lse_step))
    const int64_t row = (int64_t)bh_q * g.Sq + a;
    const float lse_a = p.fo.first ? -INFINITY : p.fo.acc_lse[row];
    float wa = 0.f, ws = 0.f, lse_n = -INFINITY;
    if (lse_a != -INFINITY || lse_v != -INFINITY) {
      const float mx = fmaxf(lse_a, lse_v);
      const float ea = expf(lse_a - mx), es = expf(lse_v - mx);
      lse_n = mx + logf(ea + es);
      wa = ea / (ea + es);
      ws = es / (ea + es);
    }
    if (!(p.fo.first || p.fo.last || lse_v != -INFINITY)) return;  // nothing to add: state unchanged
    float* acc = p.fo.acc_o + row * D;
    T* dst = reinterpret_cast<T*>(p.out) + row * D;
#pragma unroll
    for (int e = 0; e < NC; ++e) {
      const float prev = p.fo.first ? 0.f : acc[sub + 4 * e];
      const float val = wa * prev + ws * (o[e] * inv_l);
      if (p.fo.last)
        store_out<T>(dst + sub + 4 * e, val);
      else
        acc[sub + 4 * e] = val;
    }
    if (sub == 0) {
      if (p.fo.last)
        p.lse[row] = lse_n;
      else
        p.fo.acc_lse[row] = lse_n;
    }
  } else if (p.fo.kind == kOutPartial) {
    float* dst = reinterpret_cast<float*>(p.out) + ((int64_t)bh_q * g.Sq + a) * D;
#pragma unroll
    for (int e = 0; e < NC; ++e) dst[sub + 4 * e] = o[e] * inv_l;
    if (sub == 0) p.lse[(int64_t)bh_q * g.Sq + a] = lse_v;
  } else {
    const int64_t tok = token_of(g, U.i, a);
    T* dst = reinterpret_cast<T*>(p.out) + ((int64_t)bh_q * g.S + tok) * D;
#pragma unroll
    for (int e = 0; e < NC; ++e) store_out<T>(dst + sub + 4 * e, o[e] * inv_l);
    if (sub == 0) p.lse[(int64_t)bh_q * g.S + tok] = lse_v;
  }
}

template <typename T, int D>
static int launch_t(const void* q, const void* k, const void* v, const Params& p, cudaStream_t stream) {
  const int smem = Smem<D>::kBytes;
  if (cudaFuncSetAttribute(ring_fwd_simt_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess)
    return RING_ATTN_ECUDA;
  const int64_t units = num_units(p.g, BQ, p.q_shard_only);
  if (units == 0) return RING_ATTN_OK;
  ring_fwd_simt_kernel<T, D><<<(unsigned)units, kThreads, smem, stream>>>(
      static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v), p);
  return cudaGetLastError() == cudaSuccess ? RING_ATTN_OK : RING_ATTN_ECUDA;
}

}  // namespace simt

int launch_fwd_simt(const void* q, const void* k, const void* v, void* out, float* lse, const RingGeom& g,
                    float scale, int dtype, int s_begin, int s_end, int q_shard_only, const FwdOut& fo,
                    cudaStream_t stream) {
  simt::Params p;
  p.g = g;
  p.out = out;
  p.lse = lse;
  p.scale = scale;
  p.s_begin = s_begin;
  p.s_end = s_end;
  p.q_shard_only = q_shard_only;
  p.fo = fo;
  if (dtype == RING_ATTN_DTYPE_FP32) {
    if (g.D == 64) return simt::launch_t<float, 64>(q, k, v, p, stream);
    if (g.D == 128) return simt::launch_t<float, 128>(q, k, v, p, stream);
  } else {
    if (g.D == 64) return simt::launch_t<__nv_bfloat16, 64>(q, k, v, p, stream);
    if (g.D == 128) return simt::launch_t<__nv_bfloat16, 128>(q, k, v, p, stream);
  }
  return RING_ATTN_EUNSUPPORTED;
}

}  // namespace ringattn
