// Long-context decode against a sharded KV cache on sm_100a (bf16, D = 128).
//
// A decode step has one new query row per head, placed after every cached key, so
// it attends to all S keys (RingAttention newsletter, cmlonder, section "code and
// integration map": after a million-token prefill, each generated token reads the
// whole KV cache). The cache keeps the ring's sharding (contiguous, striped or
// zigzag shards of S/P tokens). The work is bound by reading K and V once, so it is
// split across SMs: each CTA takes one chunk of one shard for one (batch, kv head)
// and every query head of its GQA group, and writes a normalised partial (O, lse);
// ring_attn_merge then combines the P * chunks partials with the online-softmax
// rescale (RingAttention deep-architecture article, techknowgenie, section 3).
//
// Per CTA: one producer warp streams 128-key K and V tiles with TMA (the shard
// maps, 128-byte swizzle) through a 3-stage ring; eight consumer warps then
//   1. score: thread (half, r) forms the dot products of key r of the tile with
//      every query head of the group over one half of the head dim (q in shared
//      memory, read as a broadcast; the swizzle makes the lanes' reads of 32
//      different key rows conflict-free);
//   2. warps 0-3 add the halves, take the tile maximum per head, move the reference
//      maximum only when it grows by more than 8 (log2 units; every consumer then
//      rescales its O and l), and write p = 2^(s - m) to shared memory;
//   3. accumulate: thread (half, d) adds p_key * V[key][d] over its half of the
//      tile's keys into output column d of every head; the halves are summed once
//      at the end of the chunk.
// The consumer warps meet on a named barrier (they always take the same path: only
// one thread waits on the tile's mbarrier, with the watchdog, and broadcasts the
// outcome).
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "ring_schedule.h"
#include "ringattn_internal.h"
#include "sm100_ptx.cuh"

namespace ringattn {
namespace dec {

constexpr int D = 128;
constexpr int TK = 128;                   // keys per tile
constexpr int BOXW = 64;
constexpr int kBoxBytes = TK * BOXW * 2;  // 16 KiB
constexpr int kTileBytes = TK * D * 2;    // 32 KiB
constexpr int kStages = 3;
constexpr int kStageBytes = 2 * kTileBytes;  // K then V
constexpr int kMaxRep = 16;
constexpr int kConsumers = 256;  // 8 warps: two halves of the head dim (scores) or of the keys (P V)
constexpr int kThreads = kConsumers + 32;
constexpr int kProducerWarp = kConsumers / 32;
constexpr int kOffQ = kStages * kStageBytes;              // fp32 [rep][D]
constexpr int kOffP = kOffQ + kMaxRep * D * 4;            // fp32 [rep][TK]
constexpr int kOffPart = kOffP + kMaxRep * TK * 4;        // fp32 [2][rep][TK] partial dots / partial O
constexpr int kOffRed = kOffPart + 2 * kMaxRep * TK * 4;  // fp32 [2][4 warps][rep]
constexpr int kOffBar = kOffRed + 2 * 4 * kMaxRep * 4;    // full[kStages], empty[kStages]
constexpr int kOffMisc = kOffBar + 2 * kStages * 8;
constexpr int kSmemBytes = kOffMisc + 64 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget");
constexpr float kRescaleLog2 = 8.0f;

struct Params {
  RingGeom g;
  const uint16_t* q;  // [B, Hq, D] bf16
  float* o_parts;     // [n_parts][B*Hq][D]
  float* lse_parts;   // [n_parts][B*Hq]
  int chunk_keys;     // keys per chunk (multiple of TK)
  int chunks;         // chunks per shard
  float scale_log2;
  int* status;
  uint64_t watchdog_ns;
};

__device__ __forceinline__ void consumers_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kConsumers) : "memory"); }

__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > limit_ns) return;
  }
}

// Byte offset of the 8-element chunk holding column d of row r in a 128-byte-swizzled
// tile staged as two 64-column boxes.
__device__ __forceinline__ int swz(int r, int d) {
  return (d / BOXW) * kBoxBytes + r * 128 + ((((d % BOXW) / 8) ^ (r & 7)) * 16);
}

__device__ __forceinline__ float bf16_lo(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t x) { return __uint_as_float(x & 0xffff0000u); }

// REP: query heads per kv head (the GQA group size), a compile-time constant so that
// every per-head loop is unrolled exactly.
template <int REP>
__global__ void __launch_bounds__(kThreads, 1)
    decode_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* qs = reinterpret_cast<float*>(smem + kOffQ);
  float* ps = reinterpret_cast<float*>(smem + kOffP);
  float* part = reinterpret_cast<float*>(smem + kOffPart);
  float* red = reinterpret_cast<float*>(smem + kOffRed);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* empty = full + kStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc);
  volatile int* go = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
  const int tid = threadIdx.x;
  const int warp = tid / 32, lane = tid % 32;
  const RingGeom& g = p.g;

  // unit: chunk fastest, then shard, then (b, kv head)
  int64_t u = blockIdx.x;
  const int c = (int)(u % p.chunks);
  u /= p.chunks;
  const int j = (int)(u % g.P);
  u /= g.P;
  const int kvh = (int)(u % g.Hkv);
  const int b = (int)(u / g.Hkv);
  const int bh_kv = b * g.Hkv + kvh;
  const int64_t k0 = (int64_t)c * p.chunk_keys;
  const int64_t k1 = (k0 + p.chunk_keys < g.Sq) ? k0 + p.chunk_keys : g.Sq;
  const int ntiles = (int)((k1 - k0 + TK - 1) / TK);

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumers / 32);
    }
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  __syncthreads();
  const Watchdog wd{abort_flag, p.status, p.watchdog_ns};

  if (warp == kProducerWarp) {
    if (lane == 0) {
      // ------------------------------------------------------------------ producer
      bool ok = true;
      int n = 0;
      for (; n < ntiles && ok; ++n) {
        const int s = n % kStages;
        if (!(ok = mbar_wait_backoff<false>(&empty[s], ((uint32_t)(n / kStages) & 1) ^ 1, wd, 64))) break;
        int c1, c2;
        shard_map_coords(g, j, k0 + (int64_t)n * TK, c1, c2);
        uint8_t* dst = smem + s * kStageBytes;
        mbar_arrive_expect_tx(&full[s], kStageBytes);
        for (int bx = 0; bx < 2; ++bx) {
          tma_load_4d(dst + bx * kBoxBytes, &tm_k, &full[s], bx * BOXW, c1, c2, bh_kv);
          tma_load_4d(dst + kTileBytes + bx * kBoxBytes, &tm_v, &full[s], bx * BOXW, c1, c2, bh_kv);
        }
      }
      if (!ok) {
        for (int m = (n > kStages ? n - kStages : 0); m < n; ++m)
          drain_wait(&full[m % kStages], (uint32_t)(m / kStages) & 1, p.watchdog_ns);
      }
    }
    return;
  }

  // ---------------------------------------------------------------------- consumers
  const int half = tid / TK;  // scores: half of the head dim; P V: half of the tile's keys
  const int r = tid % TK;     // scores: key row of the tile; P V: output column
  for (int x = tid; x < REP * D; x += kConsumers) {
    const int h = x / D, d = x % D;
    qs[h * D + d] = bf16_lo(p.q[((int64_t)(b * g.Hq + kvh * REP + h)) * D + d]);
  }
  float o[REP], m_ref[REP], l[REP], sc[REP];
#pragma unroll
  for (int h = 0; h < REP; ++h) {
    o[h] = 0.f;
    m_ref[h] = -INFINITY;
    l[h] = 0.f;
  }
  bool ok = true;
  for (int n = 0; n < ntiles; ++n) {
    const int s = n % kStages;
    if (tid == 0) *go = mbar_wait(&full[s], (uint32_t)(n / kStages) & 1, wd) ? 1 : 0;
    consumers_sync();
    if (!*go) {
      ok = false;
      break;
    }
    const uint8_t* Ks = smem + s * kStageBytes;
    const uint8_t* Vs = Ks + kTileBytes;
    const bool valid = k0 + (int64_t)n * TK + r < k1;
    // 1. partial scores over this thread's half of the head dim
    {
      float a0[REP], a1[REP];
#pragma unroll
      for (int h = 0; h < REP; ++h) a0[h] = a1[h] = 0.f;
#pragma unroll
      for (int dd = 0; dd < D / 2; dd += 8) {
        const int d = half * (D / 2) + dd;
        const uint4 kk = *reinterpret_cast<const uint4*>(Ks + swz(r, d));
#pragma unroll
        for (int h = 0; h < REP; ++h) {
          const float4 q0 = *reinterpret_cast<const float4*>(qs + h * D + d);
          const float4 q1 = *reinterpret_cast<const float4*>(qs + h * D + d + 4);
          a0[h] = fmaf(bf16_lo(kk.x), q0.x, fmaf(bf16_hi(kk.x), q0.y, fmaf(bf16_lo(kk.y), q0.z, fmaf(bf16_hi(kk.y), q0.w, a0[h]))));
          a1[h] = fmaf(bf16_lo(kk.z), q1.x, fmaf(bf16_hi(kk.z), q1.y, fmaf(bf16_lo(kk.w), q1.z, fmaf(bf16_hi(kk.w), q1.w, a1[h]))));
        }
      }
#pragma unroll
      for (int h = 0; h < REP; ++h) part[(half * REP + h) * TK + r] = a0[h] + a1[h];
    }
    consumers_sync();
    // 2. tile maximum per head (warps 0-3 hold the 128 keys)
    if (half == 0) {
#pragma unroll
      for (int h = 0; h < REP; ++h) {
        sc[h] = valid ? (part[h * TK + r] + part[(REP + h) * TK + r]) * p.scale_log2 : -INFINITY;
        float mx = sc[h];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        if (lane == 0) red[warp * kMaxRep + h] = mx;
      }
    }
    consumers_sync();
    // every consumer moves the reference maximum the same way; warps 0-3 write p
#pragma unroll
    for (int h = 0; h < REP; ++h) {
      const float mt = fmaxf(fmaxf(red[h], red[kMaxRep + h]), fmaxf(red[2 * kMaxRep + h], red[3 * kMaxRep + h]));
      if (n == 0) {
        m_ref[h] = mt;
      } else if (mt > m_ref[h] + kRescaleLog2) {
        const float alpha = ex2_approx(m_ref[h] - mt);
        o[h] *= alpha;
        l[h] *= alpha;
        m_ref[h] = mt;
      }
      if (half == 0) {
        const float pe = valid ? ex2_approx(sc[h] - m_ref[h]) : 0.f;
        ps[h * TK + r] = pe;
        float sum = pe;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
        if (lane == 0) red[4 * kMaxRep + warp * kMaxRep + h] = sum;
      }
    }
    consumers_sync();
    // 3. O += P V: column r, keys [64 half, 64 half + 64) of the tile
#pragma unroll
    for (int h = 0; h < REP; ++h)
      l[h] += (red[4 * kMaxRep + h] + red[5 * kMaxRep + h]) + (red[6 * kMaxRep + h] + red[7 * kMaxRep + h]);
    {
      float b0[REP], b1[REP];
#pragma unroll
      for (int h = 0; h < REP; ++h) b0[h] = b1[h] = 0.f;
      const int key0 = half * (TK / 2);
#pragma unroll 4
      for (int kk = 0; kk < TK / 2; kk += 4) {
        const int key = key0 + kk;
        float vv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
          vv[e] = bf16_lo(*reinterpret_cast<const uint16_t*>(Vs + swz(key + e, r) + (r % 8) * 2));
#pragma unroll
        for (int h = 0; h < REP; ++h) {
          const float4 pp = *reinterpret_cast<const float4*>(ps + h * TK + key);
          b0[h] = fmaf(pp.x, vv[0], fmaf(pp.y, vv[1], b0[h]));
          b1[h] = fmaf(pp.z, vv[2], fmaf(pp.w, vv[3], b1[h]));
        }
      }
#pragma unroll
      for (int h = 0; h < REP; ++h) o[h] += b0[h] + b1[h];
    }
    consumers_sync();  // every consumer is done with this stage and with ps, part, red
    if (lane == 0) mbar_arrive(&empty[s]);
  }
  if (!ok) return;
  // the two key halves' partial O, then the normalised partial of this chunk
  if (half == 1) {
#pragma unroll
    for (int h = 0; h < REP; ++h) part[h * TK + r] = o[h];
  }
  consumers_sync();
  if (half == 0) {
    const int pidx = j * p.chunks + c;
    const int64_t rows = (int64_t)g.B * g.Hq;
#pragma unroll
    for (int h = 0; h < REP; ++h) {
      const int64_t row = (int64_t)b * g.Hq + kvh * REP + h;
      const float ot = o[h] + part[h * TK + r];
      const bool empty_part = !(l[h] > 0.f);  // cannot happen for a chunk with a key; kept exact anyway
      p.o_parts[((int64_t)pidx * rows + row) * D + r] = empty_part ? 0.f : ot / l[h];
      if (r == 0)
        p.lse_parts[(int64_t)pidx * rows + row] =
            empty_part ? -INFINITY : (m_ref[h] + log2f(l[h])) * 0.69314718055994530942f;
    }
  }
}

}  // namespace dec

// Chunking of every shard: enough CTAs for about 16 waves on 148 SMs, at most one
// chunk per 128-key tile and at most 1024 partials in all (the merge kernel's
// limit). Returns the tiles per chunk; *chunks gets the chunks per shard (each with
// at least one key).
int decode_chunking(const RingGeom& g, int* chunks) {
  const int64_t tiles = (g.Sq + dec::TK - 1) / dec::TK;
  const int64_t per = (int64_t)g.B * g.Hkv * g.P;
  const int64_t want = (16 * 148 + per - 1) / per;
  int64_t cap = tiles < 1024 / g.P ? tiles : 1024 / g.P;
  if (cap < 1) cap = 1;
  const int64_t n = want < 1 ? 1 : (want > cap ? cap : want);
  const int64_t chunk_tiles = (tiles + n - 1) / n;
  *chunks = (int)((tiles + chunk_tiles - 1) / chunk_tiles);
  return (int)chunk_tiles;
}

int64_t decode_parts(const RingGeom& g) {
  int chunks = 1;
  decode_chunking(g, &chunks);
  return (int64_t)g.P * chunks;
}

int launch_decode_sm100(const void* q, const void* k, const void* v, void* out, float* lse, const RingGeom& g,
                        float scale, float* o_parts, float* lse_parts, int* status, uint64_t watchdog_ns,
                        cudaStream_t stream) {
  using namespace dec;
  if (g.D != D) return RING_ATTN_EUNSUPPORTED;
  int chunks = 1;
  const int chunk_tiles = decode_chunking(g, &chunks);
  if ((int64_t)g.P * chunks > 1024) return RING_ATTN_EUNSUPPORTED;
  CUtensorMap mk, mv;
  int rc;
  if ((rc = encode_shard_map(&mk, k, g, g.Hkv, D, TK)) != 0) return rc;
  if ((rc = encode_shard_map(&mv, v, g, g.Hkv, D, TK)) != 0) return rc;
  Params p;
  p.g = g;
  p.q = static_cast<const uint16_t*>(q);
  p.o_parts = o_parts;
  p.lse_parts = lse_parts;
  p.chunk_keys = chunk_tiles * TK;
  p.chunks = chunks;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.status = status;
  p.watchdog_ns = watchdog_ns;
  const int64_t grid = (int64_t)g.B * g.Hkv * g.P * chunks;
  if (grid > 0x7fffffff) return RING_ATTN_EINVAL;
  void (*kern)(CUtensorMap, CUtensorMap, Params) = nullptr;
  switch (g.Hq / g.Hkv) {
    case 1: kern = decode_kernel<1>; break;
    case 2: kern = decode_kernel<2>; break;
    case 3: kern = decode_kernel<3>; break;
    case 4: kern = decode_kernel<4>; break;
    case 5: kern = decode_kernel<5>; break;
    case 6: kern = decode_kernel<6>; break;
    case 7: kern = decode_kernel<7>; break;
    case 8: kern = decode_kernel<8>; break;
    case 16: kern = decode_kernel<16>; break;
    default: return RING_ATTN_EUNSUPPORTED;
  }
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) != cudaSuccess)
    return RING_ATTN_ECUDA;
  kern<<<(unsigned)grid, kThreads, kSmemBytes, stream>>>(mk, mv, p);
  if (cudaGetLastError() != cudaSuccess) return RING_ATTN_ECUDA;
  return launch_merge(o_parts, lse_parts, g.P * chunks, (int64_t)g.B * g.Hq, D, out, lse, RING_ATTN_DTYPE_BF16,
                      stream);
}

}  // namespace ringattn
