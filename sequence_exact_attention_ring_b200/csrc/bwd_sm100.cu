// Backward pass of exact ring attention for sm_100a (B200), D = 128, bf16 inputs.
//
// Method (RingAttention deep-architecture article, techknowgenie, section
// "activation checkpointing and memory recomputation"): the forward keeps only the
// queries and the row statistics; the backward lets the K/V blocks travel the ring
// in the opposite direction and recomputes the attention map where they meet the
// queries. The statistics are kept as lse = m + ln l, one number per row. With
// S = scale Q K^T on the causal mask (global token order), the gradients of
// O = softmax(S) V against dO are the chain rule through that definition:
//     P = exp(S - lse),  dV = P^T dO,  dP = dO V^T,  Delta = rowsum(dO * O),
//     dS = P * (dP - Delta),  dQ = scale dS K,  dK = scale dS^T Q.
//
// Three kernels, all on one stream:
//   bwd_prep_kernel    Delta and lse * log2(e) per query row, written in shard-local
//                      order and padded to whole 128-row tiles (+inf / 0 padding), so
//                      a query tile's statistics are 512 contiguous bytes.
//   bwd_dkdv_kernel    one CTA per K/V tile (b, kv head, shard j, 128 keys). As the
//                      tile travels the backward ring it meets query shard (j - s) mod P
//                      at step s; the CTA visits, 64 rows at a time, every query row (of
//                      every query head of the GQA group) that sees it:
//                          S^T = K Q^T, dP^T = V dO^T        (SS MMAs into TMEM)
//                          P^T, dS^T per key row              (8 warps, registers)
//                          dV += P^T dO, dK += dS^T Q         (A operands from TMEM)
//                      and writes dK, dV once, without atomics.
//   bwd_dq_kernel      one CTA per 128-row query tile; it walks the keys, 64 at a time,
//                      in backward-ring order (shard (i + s) mod P at step s):
//                          S = Q K^T, dP = dO V^T, then P, dS per query row,
//                          dQ += dS K                         (A operand from TMEM)
// Both keep two TMEM buffers of the 64-column score and dP tiles, so the tensor cores
// compute step n + 1 (and finish step n - 1's accumulation) while the elementwise
// warps work on step n.
// The streamed operands of a step (dK/dV: the Q and dO steps and their statistics; dQ:
// the K and V steps) share one shared-memory ring slot behind one barrier: every
// barrier wait costs the MMA warp on the order of a hundred clocks, during which the
// tensor pipe, which queues only a few instructions, drains.
// Splitting dQ from dK/dV recomputes S and dP once more (7 instead of 5 GEMMs) and
// in exchange needs no atomic accumulation anywhere.
//
// Tensor memory (512 columns): score buffers [0,64) and [64,128), dP buffers [128,192)
// and [192,256), accumulators from 256 (the dQ kernel keeps Q and dO at 384 and 448). Eight elementwise warps split each 64-column
// tile: warp w owns TMEM lanes 32 (w % 4) .. +31 and columns 32 (w / 4) .. +31 of it;
// it writes its 32 bf16 P (or dS) values packed into the first 16 of those columns,
// which it has already read, so no warp overwrites a value another warp still needs.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "ring_schedule.h"
#include "ringattn_internal.h"
#include "sm100_ptx.cuh"
#include "softmax_rows.cuh"

namespace ringattn {
namespace bwd {

constexpr int D = 128;
constexpr int BT = 128;                    // rows of every tile (keys or queries)
constexpr int BOXW = 64;                   // bf16 per TMA box row (128 bytes, 128B swizzle)
constexpr int kBoxBytes = BT * BOXW * 2;   // 16 KiB
constexpr int kTileBytes = BT * D * 2;     // 32 KiB
constexpr int kSmemLimit = 232448;
constexpr int kThreads = 384;              // 8 elementwise warps, producer, MMA, 2 idle
constexpr int kEwWarps = 8;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr uint32_t kProducerSleepNs = 64;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColAcc = 256;
constexpr uint32_t kIdescTS = idesc_bf16_f32(BT, D, 0, 1);   // B MN-major (rows of the K dim)

__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > limit_ns) return;
  }
}

// K-major operand descriptor of a 128-row tile staged as two 64-column boxes; K
// step k (16 columns) sits in box k/4 at byte 32 (k%4) of each 128-byte row.
__device__ __forceinline__ uint64_t kmajor_step(uint64_t base, int k) {
  return base + (uint64_t)((((k / 4) * kBoxBytes) + (k % 4) * 32) >> 4);
}
// MN-major operand (rows of the tile run along K): K step k covers rows 16k..16k+15.
__device__ __forceinline__ uint64_t mnmajor_step(uint64_t base, int k) {
  return base + (uint64_t)((k * 16 * 128) >> 4);
}

// ----------------------------------------------------------------------- prep
// One warp per padded shard-local query row (bh, i, a): lse2 = lse * log2(e) and
// delta = <dO_t, O_t> in fp32 for t = token_of(i, a); rows a >= Sq get +inf and 0.
// local_i >= 0: out, dout and lse hold only query shard local_i, in shard-local order,
// and the statistics are laid out for that one shard ([B*Hq][1][sq_pad]).
__global__ void __launch_bounds__(256) bwd_prep_kernel(const uint16_t* __restrict__ out,
                                                       const uint16_t* __restrict__ dout,
                                                       const float* __restrict__ lse, float* __restrict__ lse2,
                                                       float* __restrict__ delta, RingGeom g, int64_t sq_pad,
                                                       int64_t rows, int local_i) {
  const int64_t row = (int64_t)blockIdx.x * 8 + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (row >= rows) return;
  const int64_t per_bh = (int64_t)(local_i >= 0 ? 1 : g.P) * sq_pad;
  const int64_t bh = row / per_bh;
  const int i = local_i >= 0 ? local_i : (int)((row % per_bh) / sq_pad);
  const int64_t a = row % sq_pad;
  if (a >= g.Sq) {
    if (lane == 0) {
      lse2[row] = INFINITY;
      delta[row] = 0.f;
    }
    return;
  }
  const int64_t t = token_of(g, i, a);
  const int64_t in_row = local_i >= 0 ? bh * g.Sq + a : bh * g.S + t;
  const int64_t base = in_row * g.D;
  float acc = 0.f;
  for (int d = lane * 4; d < g.D; d += 128) {
    const uint2 o = *reinterpret_cast<const uint2*>(out + base + d);
    const uint2 x = *reinterpret_cast<const uint2*>(dout + base + d);
    acc += __uint_as_float(o.x << 16) * __uint_as_float(x.x << 16);
    acc += __uint_as_float(o.x & 0xffff0000u) * __uint_as_float(x.x & 0xffff0000u);
    acc += __uint_as_float(o.y << 16) * __uint_as_float(x.y << 16);
    acc += __uint_as_float(o.y & 0xffff0000u) * __uint_as_float(x.y & 0xffff0000u);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) {
    lse2[row] = lse[in_row] * 1.4426950408889634f;
    delta[row] = acc;
  }
}

struct Params {
  RingGeom g;
  const void* q;       // bf16 [B,Hq,S,D] (read directly by the dQ kernel)
  const void* dout;    // bf16 [B,Hq,S,D]
  const float* lse2;   // [B*Hq][P][sq_pad]
  const float* delta;  // [B*Hq][P][sq_pad]
  int64_t sq_pad;
  void* out0;          // dK (dk/dv pass) or dQ (dq pass), bf16 [B,H,S,D]
  void* out1;          // dV (dk/dv pass)
  float scale;
  float scale_log2;
  int* status;
  uint64_t watchdog_ns;
  // One step of a ring spread over devices (step = 1): q, dout, k and v are single-shard
  // buffers in shard-local order and the statistics cover that one query shard; the dK/dV
  // pass meets only query shard q_only, the dQ pass units are query shard q_only's and
  // walk only KV shard kv_only; the epilogues fold into fp32 accumulators acc0 (dK or dQ)
  // and acc1 (dV), started on `first`, and on `last` write the bf16 results to out0/out1.
  int step;
  int q_only, kv_only;
  int first, last;
  float* acc0;
  float* acc1;
};

// Statistics row of local query row a of shard i, and the memory row of the same query
// row in q / dout (whole sequence in token order, or one shard in shard-local order).
__device__ __forceinline__ int64_t stat_row(const Params& p, int bh, int i, int64_t a) {
  return ((int64_t)bh * (p.step ? 1 : p.g.P) + (p.step ? 0 : i)) * p.sq_pad + a;
}
__device__ __forceinline__ int64_t input_row(const Params& p, int bh, int i, int64_t a) {
  return p.step ? (int64_t)bh * p.g.Sq + a : (int64_t)bh * p.g.S + token_of(p.g, i, a);
}

// Ring-step epilogue for kCols columns of one row (row stride D): acc = (first ? 0 : acc)
// + mul * T, with T read from tensor memory; on the last step the sum goes to `out` in
// bf16 instead. A row this step adds nothing to keeps its accumulator. All lanes execute
// the tensor-memory loads; only rows that exist are read and written.
template <int kCols>
__device__ __forceinline__ void fold_cols(uint32_t tA, bool have, bool row_ok, float mul, bool first, bool last,
                                          float* acc, void* out, int64_t row, int col0) {
#pragma unroll 1
  for (int c = 0; c < kCols / 32; ++c) {
    uint32_t o[32];
    if (have) {
      tmem_ld32(tA + c * 32, o);
      tmem_wait_ld();
    }
    if (!row_ok || (!have && !first && !last)) continue;
    const int64_t base = row * D + col0 + c * 32;
    float v[32];
#pragma unroll
    for (int e = 0; e < 32; e += 4) {
      const float4 a4 = first ? make_float4(0.f, 0.f, 0.f, 0.f) : *reinterpret_cast<const float4*>(acc + base + e);
      v[e] = a4.x + (have ? mul * __uint_as_float(o[e]) : 0.f);
      v[e + 1] = a4.y + (have ? mul * __uint_as_float(o[e + 1]) : 0.f);
      v[e + 2] = a4.z + (have ? mul * __uint_as_float(o[e + 2]) : 0.f);
      v[e + 3] = a4.w + (have ? mul * __uint_as_float(o[e + 3]) : 0.f);
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
        *reinterpret_cast<float4*>(acc + base + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
    }
  }
}

// P and dS for 32 columns (raw fp32 bits of s and dP), on packed column pairs (f32x2
// arithmetic): x = s * scale_log2 - lse2,
// P = 2^x, dS = P * (dP - Delta). kPerCol: the statistics belong to the columns (read in
// pairs from shared memory); otherwise one row value for all columns. The per-column mask
// selects run only when a column of the chunk lies outside [cmin, cmax).
template <bool kPerCol>
__device__ __forceinline__ void p_ds_chunk_packed(const uint32_t (&s)[32], const uint32_t (&dp)[32],
                                                  const float* lse2c, const float* deltac, float row_lse2,
                                                  float row_delta, float scale_log2, int c0, int cmin, int cmax,
                                                  uint32_t* pp, uint32_t* pds) {
  const uint64_t c2 = f2_splat(scale_log2);
  const uint64_t l2r = f2_splat(row_lse2);
  const uint64_t dlr = f2_splat(row_delta);
  const bool whole = c0 >= cmin && c0 + 32 <= cmax;
#pragma unroll
  for (int e = 0; e < 32; e += 2) {
    uint64_t l2 = l2r, dl = dlr;
    if (kPerCol) {
      const float2 lv = *reinterpret_cast<const float2*>(lse2c + e);
      const float2 dv = *reinterpret_cast<const float2*>(deltac + e);
      l2 = f2_pack(__float_as_uint(lv.x), __float_as_uint(lv.y));
      dl = f2_pack(__float_as_uint(dv.x), __float_as_uint(dv.y));
    }
    float x0, x1;
    f2_unpack(f2_sub(f2_mul(f2_pack(s[e], s[e + 1]), c2), l2), x0, x1);
    float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
    if (!whole) {
      p0 = (c0 + e >= cmin && c0 + e < cmax) ? p0 : 0.f;
      p1 = (c0 + e + 1 >= cmin && c0 + e + 1 < cmax) ? p1 : 0.f;
    }
    const uint64_t pv = f2_pack(__float_as_uint(p0), __float_as_uint(p1));
    float d0, d1;
    f2_unpack(f2_mul(pv, f2_sub(f2_pack(dp[e], dp[e + 1]), dl)), d0, d1);
    pp[e / 2] = pack_bf16x2(p0, p1);
    pds[e / 2] = pack_bf16x2(d0, d1);
  }
}

constexpr int TS = 64;                          // rows of a streamed step (query rows or keys)
constexpr int kStepBoxBytes = TS * BOXW * 2;    // 8 KiB
constexpr int kStepTileBytes = TS * D * 2;      // 16 KiB
constexpr int kStepStatBytes = TS * 4;          // 256 B
constexpr uint32_t kIdescSS64 = idesc_bf16_f32(BT, TS, 0, 0);  // M = 128, N = 64, both K-major
// TMEM columns of double buffer b: the score tile (transposed in the dK/dV kernel) and the dP tile
__device__ __forceinline__ uint32_t col_s(int b) { return (uint32_t)(64 * b); }
__device__ __forceinline__ uint32_t col_dp(int b) { return (uint32_t)(128 + 64 * b); }
// K step k of a 64-row K-major operand staged as two 64-column boxes of 8 KiB
__device__ __forceinline__ uint64_t kmajor64_step(uint64_t base, int k) {
  return base + (uint64_t)((((k / 4) * kStepBoxBytes) + (k % 4) * 32) >> 4);
}
// TMEM column of K step k (16 rows of the K dim) of a packed bf16 operand over 64 K
// rows written by the two column halves (32 rows each, 16 packed columns each)
__device__ __forceinline__ uint32_t packed64_step_col(int k) { return (uint32_t)((k / 2) * 32 + (k % 2) * 8); }

// Shared memory of the dK/dV kernel: K and V tiles, then a ring of query-side slots,
// each one step's 64-row Q tile, its dO tile and their statistics (lse, Delta) behind
// one barrier (one wait per step for the MMA warp).
constexpr int kA_OffK = 0;
constexpr int kA_OffV = kTileBytes;
constexpr int kA_OffRing = 2 * kTileBytes;
constexpr int kA_SlotDO = kStepTileBytes;
constexpr int kA_SlotLse = 2 * kStepTileBytes;
constexpr int kA_SlotDelta = kA_SlotLse + kStepStatBytes;
constexpr int kA_SlotFill = 2 * kStepTileBytes + 2 * kStepStatBytes;
constexpr int kA_SlotBytes = ((kA_SlotFill + 1023) / 1024) * 1024;
constexpr int kA_SlotsFit = (kSmemLimit - 1024 - 64 - 512 - kA_OffRing) / kA_SlotBytes;
constexpr int kA_Slots = kA_SlotsFit < 4 ? kA_SlotsFit : 4;
constexpr int kA_OffBar = kA_OffRing + kA_Slots * kA_SlotBytes;
enum BarA { kA_KVFull = 0, kA_STFull = 1, kA_PReady = 3, kA_Done = 5, kA_Drain = 6, kA_Ring = 7 };
constexpr int kA_NumBars = kA_Ring + 2 * kA_Slots;
constexpr int kA_OffMisc = kA_OffBar + kA_NumBars * 8;
constexpr int kA_SmemBytes = kA_OffMisc + 64 + 1024;
static_assert(kA_Slots >= 3, "steps n, n + 1 and n + 2 are held at once");
static_assert(kA_SmemBytes <= kSmemLimit, "shared memory budget");

// dK/dV: one CTA per 128-key tile; query rows arrive in steps of 64. TMEM holds two
// buffers of (S^T 64 columns, dP^T 64 columns) and the dV, dK accumulators, so the
// products of step n + 1 run while the elementwise warps work on step n.
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                    const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kA_OffBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kA_OffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kA_OffMisc + 8);
  uint64_t* full = &bars[kA_Ring];
  uint64_t* empty = &bars[kA_Ring + kA_Slots];
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const RingGeom& g = p.g;

  if (threadIdx.x == 0) {
    mbar_init(&bars[kA_KVFull], 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars[kA_STFull + b], 1);
      mbar_init(&bars[kA_PReady + b], kEwWarps);
    }
    mbar_init(&bars[kA_Done], 1);
    mbar_init(&bars[kA_Drain], 1);
    for (int s = 0; s < 2 * kA_Slots; ++s) mbar_init(&bars[kA_Ring + s], 1);
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
  const KvUnit U = p.step ? decode_kv_unit_shard(g, BT, blockIdx.x, p.kv_only) : decode_kv_unit(g, BT, blockIdx.x);
  const int bh_kv = U.b * g.Hkv + U.g;
  const int rep = g.Hq / g.Hkv;
  const int q_only = p.step ? p.q_only : -1;
  const int64_t N = qwalk_count(g, U, TS, BT, q_only);  // query steps met (x2 loads each)
  auto slot_of = [&](int64_t m) { return (int)(m % kA_Slots); };
  auto phase_of = [&](int64_t m) { return (uint32_t)((m / kA_Slots) & 1); };

  if (warp == kProducerWarp) {
    if (lane == 0 && N > 0) {
      // ------------------------------------------------------------------ producer
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_do);
      int c1, c2;
      tile_coords(g, p.step != 0, U.j, (int64_t)U.kt * BT, c1, c2);
      mbar_arrive_expect_tx(&bars[kA_KVFull], 2 * kTileBytes);
      for (int bx = 0; bx < 2; ++bx) {
        tma_load_4d(smem + kA_OffK + bx * kBoxBytes, &tm_k, &bars[kA_KVFull], bx * BOXW, c1, c2, bh_kv);
        tma_load_4d(smem + kA_OffV + bx * kBoxBytes, &tm_v, &bars[kA_KVFull], bx * BOXW, c1, c2, bh_kv);
      }
      int64_t m = 0;  // steps loaded
      bool ok = true;
      for (QWalk w = qwalk_begin(g, U, TS, BT, q_only); qwalk_valid(w) && ok; qwalk_next(g, w, TS), ++m) {
        const int bh_q = U.b * g.Hq + U.g * rep + w.hr;
        const int64_t a0 = (int64_t)w.qt * TS;
        tile_coords(g, p.step != 0, w.i, a0, c1, c2);
        const int64_t stat = stat_row(p, bh_q, w.i, a0);
        const int slot = slot_of(m);
        if (!(ok = mbar_wait_backoff<false>(&empty[slot], phase_of(m) ^ 1, wd, kProducerSleepNs))) break;
        uint8_t* dst = smem + kA_OffRing + slot * kA_SlotBytes;
        mbar_arrive_expect_tx(&full[slot], kA_SlotFill);
        for (int bx = 0; bx < 2; ++bx)
          tma_load_4d(dst + bx * kStepBoxBytes, &tm_q, &full[slot], bx * BOXW, c1, c2, bh_q);
        for (int bx = 0; bx < 2; ++bx)
          tma_load_4d(dst + kA_SlotDO + bx * kStepBoxBytes, &tm_do, &full[slot], bx * BOXW, c1, c2, bh_q);
        bulk_load(dst + kA_SlotLse, p.lse2 + stat, kStepStatBytes, &full[slot]);
        bulk_load(dst + kA_SlotDelta, p.delta + stat, kStepStatBytes, &full[slot]);
      }
      if (!ok) {
        // wind down: this CTA's own copies must land before its shared memory goes away
        drain_wait(&bars[kA_KVFull], 0, p.watchdog_ns);
        for (int64_t x = (m > kA_Slots ? m - kA_Slots : 0); x < m; ++x)
          drain_wait(&full[slot_of(x)], phase_of(x), p.watchdog_ns);
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer
    const bool issuer = elect_one_sync();
    const uint32_t sbase = smem_u32(smem);
    const uint64_t dK = smem_desc_sw128(sbase + kA_OffK, 0, 1024);
    const uint64_t dV = smem_desc_sw128(sbase + kA_OffV, 0, 1024);
    auto all = [&](bool r) { return __all_sync(0xffffffffu, r); };
    auto slot_addr = [&](int64_t n) { return sbase + kA_OffRing + slot_of(n) * kA_SlotBytes; };
    // S^T = K Q^T and dP^T = V dO^T of step n into buffer n % 2
    auto issue_st = [&](int64_t n) -> bool {
      if (!all(mbar_wait(&full[slot_of(n)], phase_of(n), wd))) return false;
      tc_fence_after();
      const int b = (int)(n & 1);
      const uint64_t bq = smem_desc_sw128(slot_addr(n), 0, 1024);
      const uint64_t bd = smem_desc_sw128(slot_addr(n) + kA_SlotDO, 0, 1024);
#pragma unroll
      for (int k = 0; k < D / 16; ++k)
        if (issuer) mma_ss(tmem + col_s(b), kmajor_step(dK, k), kmajor64_step(bq, k), kIdescSS64, k > 0);
#pragma unroll
      for (int k = 0; k < D / 16; ++k)
        if (issuer) mma_ss(tmem + col_dp(b), kmajor_step(dV, k), kmajor64_step(bd, k), kIdescSS64, k > 0);
      if (issuer) mma_commit(&bars[kA_STFull + b]);
      return true;
    };
    bool ok = N > 0 && all(mbar_wait(&bars[kA_KVFull], 0, wd));
    if (ok) ok = issue_st(0);
    if (ok && N > 1) ok = issue_st(1);
    for (int64_t n = 0; ok && n < N; ++n) {
      const int b = (int)(n & 1);
      if (!(ok = all(mbar_wait(&bars[kA_PReady + b], (uint32_t)((n >> 1) & 1), wd)))) break;
      tc_fence_after();
      const uint64_t mq = smem_desc_sw128(slot_addr(n), kStepBoxBytes, 1024);
      const uint64_t md = smem_desc_sw128(slot_addr(n) + kA_SlotDO, kStepBoxBytes, 1024);
#pragma unroll
      for (int k = 0; k < TS / 16; ++k)  // dV += P^T dO
        if (issuer) mma_ts(tmem + kColAcc, tmem + col_s(b) + packed64_step_col(k), mnmajor_step(md, k), kIdescTS,
                           !(n == 0 && k == 0));
#pragma unroll
      for (int k = 0; k < TS / 16; ++k)  // dK += dS^T Q
        if (issuer) mma_ts(tmem + kColAcc + D, tmem + col_dp(b) + packed64_step_col(k), mnmajor_step(mq, k), kIdescTS,
                           !(n == 0 && k == 0));
      if (issuer) mma_commit(&empty[slot_of(n)]);
      // buffer b is free for step n + 2 once these products have read its P and dS
      if (n + 2 < N && !(ok = issue_st(n + 2))) break;
    }
    if (issuer) {
      mma_commit(&bars[kA_Done]);
      mma_commit(&bars[kA_Drain]);
    }
    drain_wait(&bars[kA_Drain], 0, p.watchdog_ns);
  } else if (warp < kEwWarps) {
    // ------------------------------------------------------------- elementwise + epilogue
    // warp = 4 hh + wq: TMEM lanes 32 wq (key rows), query columns 32 hh .. 32 hh + 31 of a step
    const int wq = warp % 4, hh = warp / 4;
    const int r = wq * 32 + lane;
    const int64_t bk = (int64_t)U.kt * BT + r;  // key row of shard j
    const int64_t u = token_of(g, U.j, bk);
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    int64_t n = 0;
    bool ok = true;
    int row_i = -1;    // query shard of the cached first visible row
    int64_t row0 = 0;  // first row of shard row_i whose token is >= u
    for (QWalk w = qwalk_begin(g, U, TS, BT, q_only); qwalk_valid(w); qwalk_next(g, w, TS), ++n) {
      const int b = (int)(n & 1);
      const int sl = slot_of(n);
      if (!(ok = mbar_wait(&bars[kA_STFull + b], (uint32_t)((n >> 1) & 1), wd))) break;
      // the statistics came with the tiles: wait on their barrier too (already complete)
      if (!(ok = mbar_wait(&full[sl], phase_of(n), wd))) break;
      tc_fence_after();
      const float* lse2c = reinterpret_cast<const float*>(smem + kA_OffRing + sl * kA_SlotBytes + kA_SlotLse);
      const float* deltac = reinterpret_cast<const float*>(smem + kA_OffRing + sl * kA_SlotBytes + kA_SlotDelta);
      if (w.i != row_i) {
        row_i = w.i;
        row0 = g.causal ? first_row_at_or_after(g, w.i, u) : 0;
      }
      const int64_t cm = row0 - (int64_t)w.qt * TS;
      const int cmin = cm < 0 ? 0 : (cm > TS ? TS : (int)cm);
      uint32_t sv[32], dpv[32], pp[16], pds[16];
      tmem_ld32(tmem + lane_off + col_s(b) + 32 * hh, sv);
      tmem_ld32(tmem + lane_off + col_dp(b) + 32 * hh, dpv);
      tmem_wait_ld();
      p_ds_chunk_packed<true>(sv, dpv, lse2c + 32 * hh, deltac + 32 * hh, 0.f, 0.f, p.scale_log2, 32 * hh, cmin,
                              TS, pp, pds);
      // the packed columns overlap only this warp's own, already loaded fp32 columns
      tmem_st16(tmem + lane_off + col_s(b) + 32 * hh, pp);
      tmem_st16(tmem + lane_off + col_dp(b) + 32 * hh, pds);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[kA_PReady + b]);
    }
    const bool have = n > 0 && ok && mbar_wait(&bars[kA_Done], 0, wd);
    if (have || n == 0) {
      tc_fence_after();
      const bool row_ok = bk < g.Sq;
      const uint32_t tAcc = tmem + lane_off + kColAcc + hh * 64;
      if (p.step) {
        const int64_t acc_row = (int64_t)bh_kv * g.Sq + bk;  // shard-local
        fold_cols<64>(tAcc, n > 0, row_ok, 1.f, p.first, p.last, p.acc1, p.out1, acc_row, hh * 64);         // dV
        fold_cols<64>(tAcc + D, n > 0, row_ok, p.scale, p.first, p.last, p.acc0, p.out0, acc_row, hh * 64);  // dK
      } else {
        const int64_t out_row = (int64_t)bh_kv * g.S + (row_ok ? u : 0);
        store_row_cols<64>(tAcc, n > 0, row_ok, 1.f, false, p.out1, out_row, D, hh * 64);         // dV
        store_row_cols<64>(tAcc + D, n > 0, row_ok, p.scale, false, p.out0, out_row, D, hh * 64);  // dK
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Shared memory of the dQ kernel: a ring of 64-key slots only, each the K step followed
// by the V step, behind one barrier (one wait per step for the MMA warp); Q and dO sit
// in tensor memory as the A operands of their products.
constexpr int kB_OffRing = 0;
constexpr int kB_SlotBytes = 2 * kStepTileBytes;
constexpr int kB_SlotsFit = (kSmemLimit - 1024 - 64 - 512 - kB_OffRing) / kB_SlotBytes;
constexpr int kB_Slots = kB_SlotsFit < 6 ? kB_SlotsFit : 6;
constexpr int kB_OffBar = kB_OffRing + kB_Slots * kB_SlotBytes;
constexpr uint32_t kColQ = 384;   // Q tile, bf16 pairs: 64 columns
constexpr uint32_t kColDO = 448;  // dO tile, bf16 pairs: 64 columns
// kB_QReady: the eight elementwise warps have written Q and dO into tensor memory
enum BarB { kB_QReady = 0, kB_SFull = 1, kB_PReady = 3, kB_Done = 5, kB_Drain = 6, kB_Ring = 7 };
constexpr int kB_NumBars = kB_Ring + 2 * kB_Slots;
constexpr int kB_OffMisc = kB_OffBar + kB_NumBars * 8;
constexpr int kB_SmemBytes = kB_OffMisc + 64 + 1024;
static_assert(kB_Slots >= 3, "steps n, n + 1 and n + 2 are held at once");
static_assert(kB_SmemBytes <= kSmemLimit, "shared memory budget");

// dQ: one CTA per 128-row query tile; keys arrive in steps of 64 along the backward
// ring. TMEM holds two buffers of (S 64 columns, dP 64 columns), the dQ accumulator,
// and Q and dO as packed bf16 pairs: S = Q K^T and dP = dO V^T then take A from
// tensor memory and read only the 64-key step from shared memory.
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                  const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                  const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kB_OffBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kB_OffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kB_OffMisc + 8);
  uint64_t* full = &bars[kB_Ring];
  uint64_t* empty = &bars[kB_Ring + kB_Slots];
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const RingGeom& g = p.g;

  if (threadIdx.x == 0) {
    mbar_init(&bars[kB_QReady], kEwWarps);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars[kB_SFull + b], 1);
      mbar_init(&bars[kB_PReady + b], kEwWarps);
    }
    mbar_init(&bars[kB_Done], 1);
    mbar_init(&bars[kB_Drain], 1);
    for (int s = 0; s < 2 * kB_Slots; ++s) mbar_init(&bars[kB_Ring + s], 1);
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
  const Unit U = decode_unit(g, BT, p.step ? p.q_only : -1, blockIdx.x);
  const int64_t a0 = (int64_t)U.tb * BT;
  const int64_t a_hi = (a0 + BT - 1 < g.Sq - 1) ? a0 + BT - 1 : g.Sq - 1;
  const int bh_q = U.b * g.Hq + U.h;
  const int bh_kv = U.b * g.Hkv + U.h / (g.Hq / g.Hkv);
  // the backward ring meets KV shard (i + s) mod P at step s: all steps, or in a ring step
  // the one that meets kv_only (counted from the query shard itself)
  const int anchor = p.step ? -1 : launch_anchor(g, -1);
  const int s_lo = p.step ? (p.kv_only - U.i + g.P) % g.P : 0;
  const int s_hi = p.step ? s_lo + 1 : g.P;
  const int64_t N = p.step ? kv_tiles_for(g, U.i, p.kv_only, a_hi, TS)
                           : unit_tile_count(g, U.i, a_hi, TS, 0, g.P);  // the same steps in either ring direction
  auto slot_of = [&](int64_t m) { return (int)(m % kB_Slots); };
  auto phase_of = [&](int64_t m) { return (uint32_t)((m / kB_Slots) & 1); };

  if (warp == kProducerWarp) {
    if (lane == 0 && N > 0) {
      // ------------------------------------------------------------------ producer
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      int c1, c2;
      int64_t m = 0;  // steps loaded
      bool ok = true;
      for (TileWalk w = walk_begin_rev(g, U.i, a_hi, TS, anchor, s_lo, s_hi); walk_valid(w) && ok;
           walk_next(g, w, a_hi, TS), ++m) {
        tile_coords(g, p.step != 0, w.j, (int64_t)w.kb * TS, c1, c2);
        const int slot = slot_of(m);
        if (!(ok = mbar_wait_backoff<false>(&empty[slot], phase_of(m) ^ 1, wd, kProducerSleepNs))) break;
        uint8_t* dst = smem + kB_OffRing + slot * kB_SlotBytes;
        mbar_arrive_expect_tx(&full[slot], kB_SlotBytes);
        for (int bx = 0; bx < 2; ++bx)
          tma_load_4d(dst + bx * kStepBoxBytes, &tm_k, &full[slot], bx * BOXW, c1, c2, bh_kv);
        for (int bx = 0; bx < 2; ++bx)
          tma_load_4d(dst + kStepTileBytes + bx * kStepBoxBytes, &tm_v, &full[slot], bx * BOXW, c1, c2, bh_kv);
      }
      if (!ok) {
        for (int64_t x = (m > kB_Slots ? m - kB_Slots : 0); x < m; ++x)
          drain_wait(&full[slot_of(x)], phase_of(x), p.watchdog_ns);
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer
    const bool issuer = elect_one_sync();
    const uint32_t sbase = smem_u32(smem);
    auto all = [&](bool r) { return __all_sync(0xffffffffu, r); };
    auto slot_addr = [&](int64_t n) { return sbase + kB_OffRing + slot_of(n) * kB_SlotBytes; };
    // S = Q K^T and dP = dO V^T of step n into buffer n % 2
    auto issue_sd = [&](int64_t n) -> bool {
      if (!all(mbar_wait(&full[slot_of(n)], phase_of(n), wd))) return false;
      tc_fence_after();
      const int b = (int)(n & 1);
      const uint64_t bk = smem_desc_sw128(slot_addr(n), 0, 1024);
      const uint64_t bv = smem_desc_sw128(slot_addr(n) + kStepTileBytes, 0, 1024);
#pragma unroll
      for (int k = 0; k < D / 16; ++k)  // K step k: dims 16k..16k+15 = packed columns 8k..8k+7
        if (issuer) mma_ts(tmem + col_s(b), tmem + kColQ + 8 * k, kmajor64_step(bk, k), kIdescSS64, k > 0);
#pragma unroll
      for (int k = 0; k < D / 16; ++k)
        if (issuer) mma_ts(tmem + col_dp(b), tmem + kColDO + 8 * k, kmajor64_step(bv, k), kIdescSS64, k > 0);
      if (issuer) mma_commit(&bars[kB_SFull + b]);
      return true;
    };
    bool ok = N > 0 && all(mbar_wait(&bars[kB_QReady], 0, wd));
    if (ok) {
      tc_fence_after();
      ok = issue_sd(0);
    }
    if (ok && N > 1) ok = issue_sd(1);
    for (int64_t n = 0; ok && n < N; ++n) {
      const int b = (int)(n & 1);
      if (!(ok = all(mbar_wait(&bars[kB_PReady + b], (uint32_t)((n >> 1) & 1), wd)))) break;
      tc_fence_after();
      const uint64_t mk = smem_desc_sw128(slot_addr(n), kStepBoxBytes, 1024);
#pragma unroll
      for (int k = 0; k < TS / 16; ++k)  // dQ += dS K
        if (issuer) mma_ts(tmem + kColAcc, tmem + col_s(b) + packed64_step_col(k), mnmajor_step(mk, k), kIdescTS,
                           !(n == 0 && k == 0));
      if (issuer) mma_commit(&empty[slot_of(n)]);  // K (dQ) and V (dP) of step n are read
      if (n + 2 < N && !(ok = issue_sd(n + 2))) break;
    }
    if (issuer) {
      mma_commit(&bars[kB_Done]);
      mma_commit(&bars[kB_Drain]);
    }
    drain_wait(&bars[kB_Drain], 0, p.watchdog_ns);
  } else if (warp < kEwWarps) {
    // ------------------------------------------------------------- elementwise + epilogue
    // warp = 4 hh + wq: TMEM lanes 32 wq (query rows), keys 32 hh .. 32 hh + 31 of a step
    const int wq = warp % 4, hh = warp / 4;
    const int r = wq * 32 + lane;
    const int64_t a = a0 + r;
    const int64_t stat = stat_row(p, bh_q, U.i, a);  // a < sq_pad always
    const float row_lse2 = p.lse2[stat];
    const float row_delta = p.delta[stat];
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    if (N > 0) {
      // this thread's row, dims 64 hh .. 64 hh + 63, as 32 bf16 pairs (the memory order);
      // rows past the shard are zeros
      const bool row_ok = a < g.Sq;
      const int64_t base = (row_ok ? input_row(p, bh_q, U.i, a) : 0) * D + 64 * hh;
      uint32_t x[32];
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const uint16_t* src = static_cast<const uint16_t*>(t == 0 ? p.q : p.dout) + base;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 v4 = row_ok ? *reinterpret_cast<const uint4*>(src + 8 * c) : make_uint4(0, 0, 0, 0);
          x[4 * c] = v4.x;
          x[4 * c + 1] = v4.y;
          x[4 * c + 2] = v4.z;
          x[4 * c + 3] = v4.w;
        }
        tmem_st32(tmem + lane_off + (t == 0 ? kColQ : kColDO) + 32 * hh, x);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[kB_QReady]);
    }
    int64_t n = 0;
    bool ok = true;
    for (TileWalk w = walk_begin_rev(g, U.i, a_hi, TS, anchor, s_lo, s_hi); walk_valid(w);
         walk_next(g, w, a_hi, TS), ++n) {
      const int b = (int)(n & 1);
      if (!(ok = mbar_wait(&bars[kB_SFull + b], (uint32_t)((n >> 1) & 1), wd))) break;
      tc_fence_after();
      const int cut = visible_keys<TS>((int64_t)w.kb * TS, key_limit(g, U.i, w.j, a));
      uint32_t sv[32], dpv[32], pp[16], pds[16];
      tmem_ld32(tmem + lane_off + col_s(b) + 32 * hh, sv);
      tmem_ld32(tmem + lane_off + col_dp(b) + 32 * hh, dpv);
      tmem_wait_ld();
      p_ds_chunk_packed<false>(sv, dpv, nullptr, nullptr, row_lse2, row_delta, p.scale_log2, 32 * hh, 0, cut, pp,
                               pds);
      tmem_st16(tmem + lane_off + col_s(b) + 32 * hh, pds);  // only dS feeds the dQ MMA
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[kB_PReady + b]);
    }
    const bool have = n > 0 && ok && mbar_wait(&bars[kB_Done], 0, wd);
    if (have || n == 0) {
      tc_fence_after();
      const bool row_ok = a < g.Sq;
      if (p.step) {
        fold_cols<64>(tmem + lane_off + kColAcc + hh * 64, n > 0, row_ok, p.scale, p.first, p.last, p.acc0, p.out0,
                      (int64_t)bh_q * g.Sq + a, hh * 64);
      } else {
        const int64_t out_row = (int64_t)bh_q * g.S + (row_ok ? token_of(g, U.i, a) : 0);
        store_row_cols<64>(tmem + lane_off + kColAcc + hh * 64, n > 0, row_ok, p.scale, false, p.out0, out_row, D,
                           hh * 64);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace bwd

int64_t bwd_sq_pad(const RingGeom& g) { return (g.Sq + bwd::BT - 1) / bwd::BT * bwd::BT; }

namespace {

bwd::Params base_params(const RingGeom& g, const void* q, const void* dout, float* stats, int64_t stat_rows,
                        float scale, int* status, uint64_t watchdog_ns) {
  bwd::Params p;
  p.g = g;
  p.q = q;
  p.dout = dout;
  p.lse2 = stats;
  p.delta = stats + stat_rows;
  p.sq_pad = bwd_sq_pad(g);
  p.out0 = nullptr;
  p.out1 = nullptr;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.status = status;
  p.watchdog_ns = watchdog_ns;
  p.step = 0;
  p.q_only = -1;
  p.kv_only = -1;
  p.first = 0;
  p.last = 0;
  p.acc0 = nullptr;
  p.acc1 = nullptr;
  return p;
}

int set_smem() {
  using namespace bwd;
  if (cudaFuncSetAttribute(bwd_dkdv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kA_SmemBytes) !=
          cudaSuccess ||
      cudaFuncSetAttribute(bwd_dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kB_SmemBytes) != cudaSuccess)
    return RING_ATTN_ECUDA;
  return RING_ATTN_OK;
}

int launch_prep(const void* out, const float* lse, const void* dout, const RingGeom& g, float* stats, int64_t rows,
                int local_i, cudaStream_t stream) {
  const int64_t prep_blocks = (rows + 7) / 8;
  if (prep_blocks > 0x7fffffff) return RING_ATTN_EINVAL;
  if (prep_blocks == 0) return RING_ATTN_OK;
  bwd::bwd_prep_kernel<<<(unsigned)prep_blocks, 256, 0, stream>>>(static_cast<const uint16_t*>(out),
                                                                    static_cast<const uint16_t*>(dout), lse, stats,
                                                                    stats + rows, g, bwd_sq_pad(g), rows, local_i);
  return cudaGetLastError() == cudaSuccess ? RING_ATTN_OK : RING_ATTN_ECUDA;
}

}  // namespace

int launch_bwd_sm100(const void* q, const void* k, const void* v, const void* out, const float* lse,
                     const void* dout, void* dq, void* dk, void* dv, const RingGeom& g, float scale, float* stats,
                     int* status, uint64_t watchdog_ns, cudaStream_t stream) {
  using namespace bwd;
  if (g.D != D) return RING_ATTN_EUNSUPPORTED;
  const int64_t rows = (int64_t)g.B * g.Hq * g.P * bwd_sq_pad(g);
  int rc = launch_prep(out, lse, dout, g, stats, rows, -1, stream);
  if (rc) return rc;
  // 128-row boxes for the stationary tiles, 64-row boxes for the streamed steps
  CUtensorMap mq, mdo, mk, mv, mq64, mdo64, mk64, mv64;
  if ((rc = encode_shard_map(&mq, q, g, g.Hq, D, BT)) != 0) return rc;
  if ((rc = encode_shard_map(&mdo, dout, g, g.Hq, D, BT)) != 0) return rc;
  if ((rc = encode_shard_map(&mk, k, g, g.Hkv, D, BT)) != 0) return rc;
  if ((rc = encode_shard_map(&mv, v, g, g.Hkv, D, BT)) != 0) return rc;
  if ((rc = encode_shard_map(&mq64, q, g, g.Hq, D, TS)) != 0) return rc;
  if ((rc = encode_shard_map(&mdo64, dout, g, g.Hq, D, TS)) != 0) return rc;
  if ((rc = encode_shard_map(&mk64, k, g, g.Hkv, D, TS)) != 0) return rc;
  if ((rc = encode_shard_map(&mv64, v, g, g.Hkv, D, TS)) != 0) return rc;
  Params p = base_params(g, q, dout, stats, rows, scale, status, watchdog_ns);
  if ((rc = set_smem())) return rc;
  const int64_t kv_units = num_kv_units(g, BT);
  const int64_t q_units = num_units(g, BT, -1);
  if (kv_units > 0x7fffffff || q_units > 0x7fffffff) return RING_ATTN_EINVAL;
  p.out0 = dk;
  p.out1 = dv;
  bwd_dkdv_kernel<<<(unsigned)kv_units, kThreads, kA_SmemBytes, stream>>>(mq64, mdo64, mk, mv, p);
  if (cudaGetLastError() != cudaSuccess) return RING_ATTN_ECUDA;
  p.out0 = dq;
  p.out1 = nullptr;
  bwd_dq_kernel<<<(unsigned)q_units, kThreads, kB_SmemBytes, stream>>>(mq, mdo, mk64, mv64, p);
  return cudaGetLastError() == cudaSuccess ? RING_ATTN_OK : RING_ATTN_ECUDA;
}

int64_t bwd_ring_stat_rows(const RingGeom& g) { return (int64_t)g.B * g.Hq * bwd_sq_pad(g); }

int launch_bwd_ring_prep(const void* out, const float* lse, const void* dout, const RingGeom& g, int q_index,
                         float* stats, cudaStream_t stream) {
  if (g.D != bwd::D) return RING_ATTN_EUNSUPPORTED;
  return launch_prep(out, lse, dout, g, stats, bwd_ring_stat_rows(g), q_index, stream);
}

int launch_bwd_ring_step_sm100(const void* q, const void* dout, const void* k, const void* v, float* dq_acc,
                               float* dk_acc, float* dv_acc, void* dq, void* dk, void* dv, const RingGeom& g,
                               int q_index, int kv_index, float scale, int parts, int first, int last, float* stats,
                               int* status, uint64_t watchdog_ns, cudaStream_t stream) {
  using namespace bwd;
  if (g.D != D) return RING_ATTN_EUNSUPPORTED;
  const int64_t rows = bwd_ring_stat_rows(g);
  // single-shard buffers in shard-local order: a 4-D view of one shard of P = 1
  CUtensorMap mq, mdo, mk, mv, mq64, mdo64, mk64, mv64;
  int rc;
  if ((rc = encode_input_map(&mq, q, g, true, g.Hq, D, BT)) != 0) return rc;
  if ((rc = encode_input_map(&mdo, dout, g, true, g.Hq, D, BT)) != 0) return rc;
  if ((rc = encode_input_map(&mk, k, g, true, g.Hkv, D, BT)) != 0) return rc;
  if ((rc = encode_input_map(&mv, v, g, true, g.Hkv, D, BT)) != 0) return rc;
  if ((rc = encode_input_map(&mq64, q, g, true, g.Hq, D, TS)) != 0) return rc;
  if ((rc = encode_input_map(&mdo64, dout, g, true, g.Hq, D, TS)) != 0) return rc;
  if ((rc = encode_input_map(&mk64, k, g, true, g.Hkv, D, TS)) != 0) return rc;
  if ((rc = encode_input_map(&mv64, v, g, true, g.Hkv, D, TS)) != 0) return rc;
  Params p = base_params(g, q, dout, stats, rows, scale, status, watchdog_ns);
  p.step = 1;
  p.q_only = q_index;
  p.kv_only = kv_index;
  p.first = first;
  p.last = last;
  if ((rc = set_smem())) return rc;
  if (parts & RING_ATTN_BWD_PART_KV) {
    const int64_t kv_units = num_kv_units_shard(g, BT);
    if (kv_units > 0x7fffffff) return RING_ATTN_EINVAL;
    p.out0 = dk;
    p.out1 = dv;
    p.acc0 = dk_acc;
    p.acc1 = dv_acc;
    bwd_dkdv_kernel<<<(unsigned)kv_units, kThreads, kA_SmemBytes, stream>>>(mq64, mdo64, mk, mv, p);
    if (cudaGetLastError() != cudaSuccess) return RING_ATTN_ECUDA;
  }
  if (parts & RING_ATTN_BWD_PART_Q) {
    const int64_t q_units = num_units(g, BT, q_index);
    if (q_units > 0x7fffffff) return RING_ATTN_EINVAL;
    p.out0 = dq;
    p.out1 = nullptr;
    p.acc0 = dq_acc;
    p.acc1 = nullptr;
    bwd_dq_kernel<<<(unsigned)q_units, kThreads, kB_SmemBytes, stream>>>(mq, mdo, mk64, mv64, p);
    if (cudaGetLastError() != cudaSuccess) return RING_ATTN_ECUDA;
  }
  return RING_ATTN_OK;
}

}  // namespace ringattn
