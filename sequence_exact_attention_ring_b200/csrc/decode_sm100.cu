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
// Per CTA, the blockwise online softmax of the forward kernels with a 128-row query
// tile of which only the group's REP rows are real (the others are never read):
//   warp 0  softmax and epilogue: TMEM lanes 0..31 = query heads of the group
//   warp 1  TMA producer: 128-key K and V tiles through a 3-stage ring
//   warp 2  TMEM owner and MMA issuer: S = Q K^T with Q in tensor memory as the A
//           operand (so only the K tile is read from shared memory), O += P V with P
//           in tensor memory
// Tensor memory: S double-buffered [0,128) and [128,256), O [256,384), Q [384,448).
// S of tile n + 1 is computed while the softmax works on tile n; the tensor work per
// tile (about 1000 clocks) stays under the time HBM needs to deliver the tile, for
// any group size up to 32.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "ring_schedule.h"
#include "ringattn_internal.h"
#include "sm100_ptx.cuh"
#include "softmax_rows.cuh"

namespace ringattn {
namespace dec {

constexpr int D = 128;
constexpr int TK = 128;                   // keys per tile
constexpr int BOXW = 64;
constexpr int kBoxBytes = TK * BOXW * 2;  // 16 KiB
constexpr int kTileBytes = TK * D * 2;    // 32 KiB
constexpr int kStages = 3;
constexpr int kStageBytes = 2 * kTileBytes;  // K then V
constexpr int kMaxRep = 32;
constexpr int kThreads = 128;
constexpr int kSoftmaxWarp = 0, kProducerWarp = 1, kMmaWarp = 2;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 256;
constexpr uint32_t kColQ = 384;
constexpr uint32_t kIdescQK = idesc_bf16_f32(128, TK, 0, 0);
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, 0, 1);
enum Bar { kQReady = 0, kSFull = 1, kPReady = 3, kPvDone = 5, kODone = 6, kDrain = 7, kFull = 8 };
constexpr int kNumBars = kFull + 2 * kStages;
constexpr int kOffBar = kStages * kStageBytes;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmemBytes = kOffMisc + 64 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget");

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

__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > limit_ns) return;
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    decode_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* full = &bars[kFull];
  uint64_t* empty = &bars[kFull + kStages];
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 8);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const RingGeom& g = p.g;
  const int rep = g.Hq / g.Hkv;

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
  const int ntiles = (int)((k1 - k0 + TK - 1) / TK);  // >= 1 for every launched chunk

  if (threadIdx.x == 0) {
    mbar_init(&bars[kQReady], 1);
    for (int x = 0; x < 2; ++x) {
      mbar_init(&bars[kSFull + x], 1);
      mbar_init(&bars[kPReady + x], 1);
    }
    mbar_init(&bars[kPvDone], 1);
    mbar_init(&bars[kODone], 1);
    mbar_init(&bars[kDrain], 1);
    for (int s = 0; s < 2 * kStages; ++s) mbar_init(&bars[kFull + s], 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Watchdog wd{abort_flag, p.status, p.watchdog_ns};

  if (warp == kProducerWarp) {
    if (lane == 0) {
      // ------------------------------------------------------------------ producer
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
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
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer
    const bool issuer = elect_one_sync();
    const uint32_t sbase = smem_u32(smem);
    auto all = [&](bool r) { return __all_sync(0xffffffffu, r); };
    // S_b = Q K_n^T into buffer n % 2 once tile n has landed
    auto issue_s = [&](int n) -> bool {
      const int s = n % kStages;
      if (!all(mbar_wait(&full[s], (uint32_t)(n / kStages) & 1, wd))) return false;
      tc_fence_after();
      const uint64_t dk = smem_desc_sw128(sbase + s * kStageBytes, 0, 1024);
      const uint32_t d = tmem + (uint32_t)(128 * (n & 1));
#pragma unroll
      for (int k = 0; k < D / 16; ++k)
        if (issuer)
          mma_ts(d, tmem + kColQ + 8 * k, dk + (uint64_t)((((k / 4) * kBoxBytes) + (k % 4) * 32) >> 4), kIdescQK,
                 k > 0);
      if (issuer) mma_commit(&bars[kSFull + (n & 1)]);
      return true;
    };
    bool ok = all(mbar_wait(&bars[kQReady], 0, wd));
    if (ok) {
      tc_fence_after();
      ok = issue_s(0);
    }
    if (ok && ntiles > 1) ok = issue_s(1);
    for (int n = 0; ok && n < ntiles; ++n) {
      const int s = n % kStages;
      if (!(ok = all(mbar_wait(&bars[kPReady + (n & 1)], (uint32_t)((n >> 1) & 1), wd)))) break;
      tc_fence_after();
      // O += P V: P in the first 64 columns of S_b, V as the MN-major B operand
      const uint64_t dv = smem_desc_sw128(sbase + s * kStageBytes + kTileBytes, kBoxBytes, 1024);
      const uint32_t pa = tmem + (uint32_t)(128 * (n & 1));
#pragma unroll
      for (int k = 0; k < TK / 16; ++k)
        if (issuer) mma_ts(tmem + kColO, pa + 8 * k, dv + (uint64_t)((k * 16 * 128) >> 4), kIdescPV, !(n == 0 && k == 0));
      if (issuer) {
        mma_commit(&bars[kPvDone]);
        mma_commit(&empty[s]);
      }
      if (n + 2 < ntiles && !(ok = issue_s(n + 2))) break;
    }
    if (issuer) {
      mma_commit(&bars[kODone]);
      mma_commit(&bars[kDrain]);
    }
    drain_wait(&bars[kDrain], 0, p.watchdog_ns);
  } else if (warp == kSoftmaxWarp) {
    // ------------------------------------------------------------- softmax + epilogue
    const int h = lane;                  // query head of the group (row of the tile)
    const bool live = h < rep;
    {
      // Q rows into tensor memory as bf16 pairs (dims 2c, 2c + 1 in column c), zeros
      // for the rows past the group; rows 32..127 are never read back
      uint32_t x[32];
      const uint16_t* src = p.q + ((int64_t)(b * g.Hq + kvh * rep + (live ? h : 0))) * D;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) {
          const uint4 v4 = live ? *reinterpret_cast<const uint4*>(src + 64 * half + 8 * cc) : make_uint4(0, 0, 0, 0);
          x[4 * cc] = v4.x;
          x[4 * cc + 1] = v4.y;
          x[4 * cc + 2] = v4.z;
          x[4 * cc + 3] = v4.w;
        }
        tmem_st32(tmem + kColQ + 32 * half, x);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[kQReady]);
    }
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int n = 0; n < ntiles; ++n) {
      const int bb = n & 1;
      if (!(ok = mbar_wait(&bars[kSFull + bb], (uint32_t)((n >> 1) & 1), wd))) break;
      tc_fence_after();
      const uint32_t tS = tmem + (uint32_t)(128 * bb);
      uint32_t sr[TK];
#pragma unroll
      for (int cc = 0; cc < TK / 32; ++cc) tmem_ld32(tS + cc * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[cc * 32]));
      tmem_wait_ld();
      const int cut = live ? visible_keys<TK>(k0 + (int64_t)n * TK, k1) : 0;  // keys past the chunk are out
      mask_scores<TK>(sr, cut);
      const float mblk = cut == 0 ? -INFINITY : raw_rowmax<TK>(sr) * p.scale_log2;
      float alpha = 1.f;
      bool resc = false;
      if (n == 0) {
        m_ref = mblk;
      } else if (mblk > m_ref + kRescaleLog2) {
        alpha = (m_ref == -INFINITY) ? 0.f : ex2_approx(m_ref - mblk);
        l *= alpha;
        m_ref = mblk;
        resc = true;
      }
      if (__any_sync(0xffffffffu, resc)) {
        // S of this tile was issued before P V of the previous one: O must hold every
        // product issued so far before it is rescaled
        if (n > 0 && !(ok = mbar_wait(&bars[kPvDone], (uint32_t)((n - 1) & 1), wd))) break;
        tc_fence_after();
        rescale_o<D>(tmem + kColO, alpha);
      }
      uint32_t pk[TK / 2];
      if (cut == 0) {
#pragma unroll
        for (int cc = 0; cc < TK / 2; ++cc) pk[cc] = 0u;
      } else {
        l += exp_pack<TK, 0>(sr, p.scale_log2, (m_ref == -INFINITY) ? 0.f : m_ref, pk);
      }
#pragma unroll
      for (int cc = 0; cc < TK / 64; ++cc) tmem_st32(tS + cc * 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[cc * 32]));
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[kPReady + bb]);
    }
    if (ok && mbar_wait(&bars[kODone], 0, wd)) {
      tc_fence_after();
      const int part = j * p.chunks + c;
      const int64_t rows = (int64_t)g.B * g.Hq;
      const int64_t row = (int64_t)b * g.Hq + kvh * rep + (live ? h : 0);
      const bool empty_part = !(l > 0.f);  // cannot happen for a chunk with a key; kept exact anyway
      const float inv_l = empty_part ? 0.f : 1.f / l;
      float* dst = p.o_parts + ((int64_t)part * rows + row) * D;
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t o[32];
        tmem_ld32(tmem + kColO + cc * 32, o);
        tmem_wait_ld();
        if (live) {
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(dst + cc * 32 + e) =
                make_float4(__uint_as_float(o[e]) * inv_l, __uint_as_float(o[e + 1]) * inv_l,
                            __uint_as_float(o[e + 2]) * inv_l, __uint_as_float(o[e + 3]) * inv_l);
        }
      }
      if (live)
        p.lse_parts[(int64_t)part * rows + row] =
            empty_part ? -INFINITY : (m_ref + log2f(l)) * 0.69314718055994530942f;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
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
  if (g.D != D || g.Hq / g.Hkv > kMaxRep) return RING_ATTN_EUNSUPPORTED;
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
  if (cudaFuncSetAttribute(decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) != cudaSuccess)
    return RING_ATTN_ECUDA;
  decode_kernel<<<(unsigned)grid, kThreads, kSmemBytes, stream>>>(mk, mv, p);
  if (cudaGetLastError() != cudaSuccess) return RING_ATTN_ECUDA;
  return launch_merge(o_parts, lse_parts, g.P * chunks, (int64_t)g.B * g.Hq, D, out, lse, RING_ATTN_DTYPE_BF16,
                      stream);
}

}  // namespace ringattn
