// Fused ring-attention forward on CTA pairs (sm_100a, cta_group::2 MMAs), D = 128.
//
// Same method and roles as fwd_sm100.cu (RingAttention deep-architecture article,
// techknowgenie, sections 2, 3, 5 and 7: query shard i folds KV shard (i - s) mod P
// at ring step s with the online-softmax rescale, causal mask on global token
// order, contiguous or striped shards). The difference is the unit of work: a
// cluster of two CTAs on two SMs owns 512 query rows and shares every K/V tile.
//
//   * An M=256 MMA spans both CTAs: rows 0-127 come from CTA 0's shared memory and
//     land in CTA 0's tensor memory, rows 128-255 likewise in CTA 1. The B operand
//     is split along N: for S = Q K^T each CTA stages 64 of the tile's 128 keys;
//     for O += P V each CTA stages 64 of the 128 head-dim columns of V. Each SM
//     therefore loads half of every K/V tile (32 KiB instead of 64 KiB), which is
//     the load the per-SM TMA path can sustain at the tensor cores' rate.
//   * CTA r, query tile q holds rows a0 + 256 q + 128 r of the unit (q = 0, 1).
//   * Only the leader (rank 0) issues MMAs. Both CTAs' TMA loads complete on the
//     leader's "full" barriers (the leader arms them for both halves); every commit
//     is multicast to the barrier at the same offset in both CTAs (S ready, slot
//     empty, O done). Softmax warps of both CTAs arrive on the leader's P-ready
//     barriers (one arrival per warp).
//   * No TMA load uses multicast.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "ring_schedule.h"
#include "ringattn_internal.h"
#include "sm100_ptx.cuh"
#include "softmax_rows.cuh"

namespace ringattn {
namespace sm100x2 {

constexpr int D = 128;
constexpr int BM = 128;            // query rows per tile per CTA (TMEM lanes)
constexpr int BN = 128;            // keys per KV tile
constexpr int NQ = 2;              // query tiles per CTA
constexpr int kCtas = 2;
constexpr int BQ = BM * NQ * kCtas;  // query rows per unit (cluster)
constexpr int BOXW = 64;
constexpr int kThreads = 384;
constexpr int kLaunchRegs = 168;
constexpr int kRegsSoftmax = 208;
constexpr int kRegsOther = 88;
static_assert(2 * kRegsSoftmax + kRegsOther <= 3 * kLaunchRegs, "register split exceeds the launch pool");
constexpr int kProducerWarp = 8;
constexpr uint64_t kCopyGraceNs = 2000000;  // after a watchdog abort, see the producer
constexpr uint32_t kProducerSleepNs = 64;  // the producer polls slots this often (other back-offs measured neutral)
constexpr int kMmaWarp = 9;
// Of every 8 column pairs of a score row, this many take 2^x from the FMA-pipe
// polynomial (exp2_poly2) and the rest from the MUFU ex2 unit (the exponentials are
// evaluated in phases, exp_pack_phased). On the 1M-token causal workload, with the
// speculative exponentials below: 1 of 8 measured 1015 TFLOP/s, 2 of 8 1003, 3 of 8 988,
// 4 of 8 938 (one box, 1462 MHz).
constexpr int kEmuPairsPer8 = 1;
constexpr float kSpecMaxSum = 1048576.0f;  // 2^20: the speculative exponentials' row-sum limit
constexpr uint16_t kPairMask = 0x3;

constexpr int kSmemLimit = 232448;
constexpr int kQTileBytes = BM * D * 2;     // 32 KiB: 128 rows x 128 dims (2 boxes of 64 dims)
constexpr int kQBoxBytes = BM * BOXW * 2;   // 16 KiB
constexpr int kHalfBytes = 16384;           // K half: 64 keys x 128 dims; V half: 128 keys x 64 dims
constexpr int kKBoxBytes = 64 * BOXW * 2;   // 8 KiB: 64 keys x 64 dims
constexpr int kOffQ = 0;
constexpr int kOffKV = NQ * kQTileBytes;
constexpr int kSlotsFit = (kSmemLimit - 1024 - 512 - kOffKV) / kHalfBytes;
constexpr int kSlots = kSlotsFit < 10 ? kSlotsFit : 10;
constexpr int kOffBar = kOffKV + kSlots * kHalfBytes;
enum Bar { kQFull = 0, kSFull = 1, kPReady = 3, kODone = 5, kDrain = 7, kRing = 8 };
constexpr int kNumBars = kRing + 2 * kSlots;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmemBytes = kOffMisc + 64 + 1024;
static_assert(kSlots >= 4, "need at least four K/V half slots");
static_assert(kSmemBytes <= kSmemLimit, "shared memory budget");

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;
constexpr uint32_t kColO = 2 * BN;
constexpr uint32_t kIdescQK = idesc_bf16_f32(2 * BM, BN, 0, 0);  // M = 256 across the pair
constexpr uint32_t kIdescPV = idesc_bf16_f32(2 * BM, D, 0, 1);

struct Params {
  RingGeom g;
  void* out;      // see FwdOut: final, per-step partial or (last fold step) shard-local bf16
  float* lse;
  int* status;
  float scale_log2;
  int s_begin, s_end;
  int q_shard_only;
  FwdOut fo;
  uint64_t watchdog_ns;
};

__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait_cluster(bar, parity)) {
    if (global_timer_ns() - t0 > limit_ns) return;
  }
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    ring_fwd_sm100_2sm_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                              const __grid_constant__ CUtensorMap tm_v, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 8);
  uint64_t* full = &bars[kRing];
  uint64_t* empty = &bars[kRing + kSlots];

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const RingGeom& g = p.g;

  if (threadIdx.x == 0) {
    mbar_init(&bars[kQFull], 1);
    for (int q = 0; q < NQ; ++q) {
      mbar_init(&bars[kSFull + q], 1);
      mbar_init(&bars[kPReady + q], kCtas * BM / 32);  // one arrival per softmax warp of each CTA
      mbar_init(&bars[kODone + q], 1);
    }
    mbar_init(&bars[kDrain], 1);
    for (int s = 0; s < 2 * kSlots; ++s) mbar_init(&bars[kRing + s], 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc_2sm(tmem_slot, kTmemCols);
    tmem_relinquish_2sm();
  }
  if (warp == kProducerWarp && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers are initialised before any cross-CTA signal
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const Watchdog wd{abort_flag, p.status, p.watchdog_ns};
  const Unit U = decode_unit(g, BQ, p.q_shard_only, blockIdx.x / kCtas);
  const int64_t a0 = (int64_t)U.tb * BQ;
  const int64_t a_hi = (a0 + BQ - 1 < g.Sq - 1) ? a0 + BQ - 1 : g.Sq - 1;
  const int bh_q = U.b * g.Hq + U.h;
  const int bh_kv = U.b * g.Hkv + U.h / (g.Hq / g.Hkv);

  if (warp >= 8) {
    regs_decrease<kRegsOther>();
    if (warp == kProducerWarp && lane == 0) {
      // ---------------------------------------------------------------- producer (both CTAs)
      const uint32_t leader_q = mapa_shared(smem_u32(&bars[kQFull]), 0);
      int n = 0;
      // a unit with no KV tile (a fully masked single ring step) loads nothing at all,
      // so no copy can still be in flight when the CTA exits
      const bool any = unit_tile_count(g, U.i, a_hi, BN, p.s_begin, p.s_end) > 0;
      bool ok = any;
      if (ok && leader) mbar_arrive_expect_tx(&bars[kQFull], kCtas * NQ * kQTileBytes);
      for (int q = 0; q < NQ && ok; ++q) {
        const int row = (int)(a0 + 256 * q + 128 * rank);
        int c1, c2;
        tile_coords(g, p.fo.local, U.i, row, c1, c2);
        for (int bx = 0; bx < 2; ++bx) {
          uint8_t* dst = smem + kOffQ + q * kQTileBytes + bx * kQBoxBytes;
          tma_load_4d_2sm(dst, &tm_q, leader_q, bx * BOXW, c1, c2, bh_q);
        }
      }
      for (TileWalk w = walk_begin(g, U.i, a_hi, BN, p.s_begin, p.s_end, launch_anchor(g, p.q_shard_only));
           walk_valid(w) && ok; walk_next(g, w, a_hi, BN)) {
        for (int kv = 0; kv < 2; ++kv, ++n) {
          const int slot = n % kSlots;
          const uint32_t ph = (uint32_t)(n / kSlots) & 1;
          if (!(ok = mbar_wait_backoff<true>(&empty[slot], ph ^ 1, wd, kProducerSleepNs))) break;
          if (leader) mbar_arrive_expect_tx(&full[slot], kCtas * kHalfBytes);
          const uint32_t leader_full = mapa_shared(smem_u32(&full[slot]), 0);
          uint8_t* dst = smem + kOffKV + slot * kHalfBytes;
          if (kv == 0) {
            // K half: keys [64 r, 64 r + 64) of the tile, all 128 dims (two 64-dim boxes)
            int c1, c2;
            tile_coords(g, p.fo.local, w.j, w.kb * BN + 64 * (int)rank, c1, c2);
            for (int bx = 0; bx < 2; ++bx)
              tma_load_4d_2sm(dst + bx * kKBoxBytes, &tm_k, leader_full, bx * BOXW, c1, c2, bh_kv);
          } else {
            // V half: all 128 keys of the tile, dims [64 r, 64 r + 64)
            int c1, c2;
            tile_coords(g, p.fo.local, w.j, w.kb * BN, c1, c2);
            tma_load_4d_2sm(dst, &tm_v, leader_full, 64 * (int)rank, c1, c2, bh_kv);
          }
        }
      }
      if (!ok && any) {
        // wind down: this CTA's own copies must land before its shared memory goes away.
        // Their bytes are counted on the leader's barriers, and mbarrier waits take only
        // barriers of the waiting CTA, so the producer gives them a fixed grace period
        // (a 16 KiB tile copy completes in microseconds; the grace is about 1000 times that).
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < kCopyGraceNs) {
        }
      }
    } else if (warp == kMmaWarp && leader) {
      // ---------------------------------------------------------------- MMA issuer (leader only)
      // The whole warp runs this loop and waits on the barriers; one elected lane
      // issues each tcgen05 instruction. Descriptor bases are built once; every MMA
      // then adds a compile-time offset (address >> 4) to the start-address field.
      const int64_t N = unit_tile_count(g, U.i, a_hi, BN, p.s_begin, p.s_end);
      const uint32_t sbase = smem_u32(smem);
      const uint64_t dq0 = smem_desc_sw128(sbase + kOffQ, 0, 1024);
      const uint64_t dk0 = smem_desc_sw128(sbase + kOffKV, 0, 1024);
      const uint64_t dv0 = smem_desc_sw128(sbase + kOffKV, kHalfBytes, 1024);
      const bool issuer = elect_one_sync();
      auto issue_s = [&](int q, int slot) {
        const uint64_t dq = dq0 + (uint64_t)((q * kQTileBytes) >> 4);
        const uint64_t dk = dk0 + (uint64_t)((slot * kHalfBytes) >> 4);
        const uint32_t d = tmem + kColS + q * BN;
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
          if (issuer)
            mma_ss_2sm(d, dq + (((k / 4) * kQBoxBytes + (k % 4) * 32) >> 4),
                       dk + (((k / 4) * kKBoxBytes + (k % 4) * 32) >> 4), kIdescQK, k > 0);
      };
      auto issue_pv = [&](int q, int slot, bool first) {
        const uint64_t dv = dv0 + (uint64_t)((slot * kHalfBytes) >> 4);
        const uint32_t d = tmem + kColO + q * D;
        const uint32_t pa = tmem + kColS + q * BN;
#pragma unroll
        for (int k = 0; k < BN / 16; ++k)
          if (issuer) mma_ts_2sm(d, pa + k * 8, dv + ((k * 16 * 128) >> 4), kIdescPV, !(first && k == 0));
      };
      auto commit = [&](uint64_t* bar) {
        if (issuer) mma_commit_2sm(bar, kPairMask);
      };
      // every lane polls; the warp proceeds only if all lanes saw the phase complete
      auto wait_all = [&](bool r) { return __all_sync(0xffffffffu, r); };
      auto kslot = [&](int64_t n) { return (int)((2 * n) % kSlots); };
      auto kphase = [&](int64_t n) { return (uint32_t)(((2 * n) / kSlots) & 1); };
      auto vslot = [&](int64_t n) { return (int)((2 * n + 1) % kSlots); };
      auto vphase = [&](int64_t n) { return (uint32_t)(((2 * n + 1) / kSlots) & 1); };
      bool ok = N > 0 && wait_all(mbar_wait_cluster(&bars[kQFull], 0, wd));
      if (ok) ok = wait_all(mbar_wait_cluster(&full[kslot(0)], kphase(0), wd));
      if (ok) {
        tc_fence_after();
        issue_s(0, kslot(0));
        commit(&bars[kSFull + 0]);
        issue_s(1, kslot(0));
        commit(&bars[kSFull + 1]);
        commit(&empty[kslot(0)]);
      }
      for (int64_t n = 0; ok && n < N; ++n) {
        const bool more = n + 1 < N;
        if (!(ok = wait_all(mbar_wait_cluster(&full[vslot(n)], vphase(n), wd)))) break;
        if (!(ok = wait_all(mbar_wait_cluster(&bars[kPReady + 0], (uint32_t)(n & 1), wd)))) break;
        tc_fence_after();
        issue_pv(0, vslot(n), n == 0);
        if (more) {
          if (!(ok = wait_all(mbar_wait_cluster(&full[kslot(n + 1)], kphase(n + 1), wd)))) break;
          tc_fence_after();
          issue_s(0, kslot(n + 1));
          commit(&bars[kSFull + 0]);
        } else {
          commit(&bars[kODone + 0]);
        }
        if (!(ok = wait_all(mbar_wait_cluster(&bars[kPReady + 1], (uint32_t)(n & 1), wd)))) break;
        tc_fence_after();
        issue_pv(1, vslot(n), n == 0);
        commit(&empty[vslot(n)]);
        if (more) {
          issue_s(1, kslot(n + 1));
          commit(&bars[kSFull + 1]);
          commit(&empty[kslot(n + 1)]);
        } else {
          commit(&bars[kODone + 1]);
        }
      }
      // both CTAs learn when every pair MMA has finished (before TMEM is released)
      commit(&bars[kDrain]);
      drain_wait(&bars[kDrain], 0, p.watchdog_ns);
    } else if (warp == kMmaWarp && lane == 0) {
      drain_wait(&bars[kDrain], 0, p.watchdog_ns);
    }
  } else {
    regs_increase<kRegsSoftmax>();
    // -------------------------------------------------------------------- softmax (both CTAs)
    const int q = warp / 4;
    const int wq = warp % 4;
    const int r = wq * 32 + lane;
    const int64_t a = a0 + 256 * q + 128 * (int64_t)rank + r;  // local query index in shard U.i
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t tS = tmem + lane_off + kColS + q * BN;
    const uint32_t tO = tmem + lane_off + kColO + q * D;
    const uint32_t leader_p = mapa_shared(smem_u32(&bars[kPReady + q]), 0);
    const float NEG_INF = -INFINITY;
    float m_ref = NEG_INF;
    float l = 0.f;
    int n = 0;
    bool ok = true;
    TileWalk w = walk_begin(g, U.i, a_hi, BN, p.s_begin, p.s_end, launch_anchor(g, p.q_shard_only));
    for (; walk_valid(w); walk_next(g, w, a_hi, BN), ++n) {
      if (!(ok = mbar_wait_cluster(&bars[kSFull + q], (uint32_t)(n & 1), wd))) break;
      tc_fence_after();
      uint32_t sr[BN];
#pragma unroll
      for (int c = 0; c < BN / 32; ++c) tmem_ld32(tS + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
      tmem_wait_ld();
      const int cut = visible_keys<BN>((int64_t)w.kb * BN, key_limit(g, U.i, w.j, a));
      mask_scores<BN>(sr, cut);
      // a block no row of this warp can see contributes nothing: P = 0, state unchanged
      const bool warp_empty = __all_sync(0xffffffffu, cut == 0);
      uint32_t pk[BN / 2];
      if (warp_empty) {
#pragma unroll
        for (int c = 0; c < BN / 2; ++c) pk[c] = 0u;
      } else {
        float lb = 0.f;
        // Exponentials against the current reference maximum first. The reference moves
        // only when a block's scores rise well above it, and O/l and lse do not depend on
        // it, so a block whose row sums stay <= kSpecMaxSum (every P <= 2^20, finite) is
        // kept as is. Otherwise (and for the first block) the warp reloads the scores,
        // takes the block maximum and follows the rescale rule below.
        bool fast = __all_sync(0xffffffffu, m_ref != NEG_INF);
        if (fast) {
          lb = exp_pack_phased<BN, kEmuPairsPer8>(sr, p.scale_log2, m_ref, pk);
          fast = __all_sync(0xffffffffu, lb <= kSpecMaxSum);
        }
        if (!fast) {
#pragma unroll
          for (int c = 0; c < BN / 32; ++c)
            tmem_ld32(tS + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
          tmem_wait_ld();
          mask_scores<BN>(sr, cut);
          const float mblk = raw_rowmax<BN>(sr) * p.scale_log2;
          float alpha = 1.f;
          bool resc = false;
          if (mblk > m_ref + kRescaleLog2) {
            // (m_ref = -inf: nothing has been accumulated yet, alpha = 0 keeps l and O at 0)
            alpha = (m_ref == NEG_INF) ? 0.f : ex2_approx(m_ref - mblk);
            l *= alpha;
            m_ref = mblk;
            resc = true;
          }
          // S ready for tile n implies PV(n-1) of this query tile completed: O is stable
          if (__any_sync(0xffffffffu, resc)) rescale_o<D>(tO, alpha);
          lb = exp_pack_phased<BN, kEmuPairsPer8>(sr, p.scale_log2, (m_ref == NEG_INF) ? 0.f : m_ref, pk);
        }
        l += lb;
      }
#pragma unroll
      for (int c = 0; c < BN / 64; ++c) tmem_st32(tS + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[c * 32]));
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(leader_p);
    }
    const bool have = (n > 0) && ok && mbar_wait_cluster(&bars[kODone + q], 0, wd);
    if (have || n == 0) {
      tc_fence_after();
      const bool row_ok = a < g.Sq;
      const bool empty_row = !(l > 0.f);
      const float inv_l = empty_row ? 0.f : 1.f / l;
      const float lse_v = empty_row ? NEG_INF : (m_ref + log2f(l)) * 0.69314718055994530942f;
      if (p.fo.kind == kOutFold) {
        fold_row<D>(tO, n > 0, row_ok, inv_l, lse_v, p.fo.first, p.fo.last, p.fo.acc_o, p.fo.acc_lse, p.out, p.lse,
                    (int64_t)bh_q * g.Sq + a);
      } else {
        const bool partial = p.fo.kind == kOutPartial;
        const int64_t out_row = partial ? (int64_t)bh_q * g.Sq + a : (int64_t)bh_q * g.S + token_of(g, U.i, a);
        store_row<D>(tO, n > 0, row_ok, inv_l, partial, p.out, out_row);
        if (row_ok) p.lse[out_row] = lse_v;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the leader's MMAs read this CTA's shared and tensor memory until here
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc_2sm(tmem, kTmemCols);
  }
}

}  // namespace sm100x2

int launch_fwd_sm100_2sm(const void* q, const void* k, const void* v, void* out, float* lse, const RingGeom& g,
                         float scale, int s_begin, int s_end, int q_shard_only, const FwdOut& fo, int* status,
                         uint64_t watchdog_ns, cudaStream_t stream) {
  using namespace sm100x2;
  if (g.D != D) return RING_ATTN_EUNSUPPORTED;
  CUtensorMap mq, mk, mv;
  int rc;
  const bool local = fo.local != 0;
  if ((rc = encode_input_map(&mq, q, g, local, g.Hq, D, BM)) != 0) return rc;
  if ((rc = encode_input_map(&mk, k, g, local, g.Hkv, D, 64)) != 0) return rc;
  if ((rc = encode_input_map(&mv, v, g, local, g.Hkv, D, BN)) != 0) return rc;
  Params p;
  p.g = g;
  p.out = out;
  p.lse = lse;
  p.status = status;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.s_begin = s_begin;
  p.s_end = s_end;
  p.q_shard_only = q_shard_only;
  p.fo = fo;
  p.watchdog_ns = watchdog_ns;
  if (cudaFuncSetAttribute(ring_fwd_sm100_2sm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) !=
      cudaSuccess)
    return RING_ATTN_ECUDA;
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, ring_fwd_sm100_2sm_kernel) != cudaSuccess) return RING_ATTN_ECUDA;
  if (fa.numRegs * kThreads < 128 * (2 * kRegsSoftmax + kRegsOther)) return RING_ATTN_EUNSUPPORTED;
  const int64_t units = num_units(g, BQ, q_shard_only);
  if (units == 0) return RING_ATTN_OK;
  if (units * kCtas > 0x7fffffff) return RING_ATTN_EINVAL;
  ring_fwd_sm100_2sm_kernel<<<(unsigned)(units * kCtas), kThreads, kSmemBytes, stream>>>(mq, mk, mv, p);
  return cudaGetLastError() == cudaSuccess ? RING_ATTN_OK : RING_ATTN_ECUDA;
}

}  // namespace ringattn
