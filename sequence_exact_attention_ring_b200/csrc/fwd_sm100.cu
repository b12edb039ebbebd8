// Fused ring-attention forward for sm_100a (B200): TMA-staged tiles, tcgen05 MMAs
// with fp32 accumulators in tensor memory, warp-specialised roles.
//
// Method (RingAttention deep-architecture article, techknowgenie):
//   section 2: query shard i stays; at ring step s it folds KV shard (i - s) mod P.
//   section 3 equations / section 5 listing: per block, S = Q K^T * scale,
//     m_new = max(m_old, rowmax S), alpha = exp(m_old - m_new), P = exp(S - m_new),
//     l = l*alpha + rowsum P, O = O*alpha + P V; finally O / l.
//   section 7: causal mask on global token order, contiguous or striped shards.
// FlashAttention video summary (aitrends), chapters on tiling and online softmax:
//   query tiles outside, key/value tiles inside, the score tile never leaves chip.
//
// One CTA = one work unit: two 128-row query tiles (rows a0..a0+255 of shard i of
// head h) that share every K/V tile. The CTA walks the unit's KV tiles in ring
// order (step s = 0..P-1, KV shard j = (i-s) mod P, tiles 0..n_j-1 of shard j).
//
// Roles (384 threads = 3 warpgroups):
//   warps 0-3  softmax for query tile 0 (one row per thread, TMEM lanes 0..127)
//   warps 4-7  softmax for query tile 1
//   warp 8     TMA producer: Q once, then K and V tiles through one shared ring of
//              shared-memory slots (K(n) and V(n) alternate), plus L2 prefetch of
//              the tiles a few steps further along the walk
//   warp 9     TMEM owner; lane 0 issues every tcgen05.mma and commit
//   warps 10-11 idle (they complete the third warpgroup for the register split)
// Registers: launched at 168 per thread; the softmax warpgroups grow to 208 and
// the third warpgroup shrinks to 88 (2*208 + 88 = 3*168).
// Tensor memory (512 columns): S0 [0,128) S1 [128,256) O0 [256,256+D) O1 [256+D,256+2D).
// P (bf16) overwrites the first 64 columns of its S tile and feeds the PV MMA
// directly from TMEM. The S MMAs read both operands from shared memory (8 KiB per
// 128x128x16 step, the whole 128 B/clock shared-memory port at full tensor rate),
// which is what bounds this single-SM variant; the CTA-pair kernel halves it.
//
// Differences from the pages' listing (same result up to rounding):
//   * exponentials are base 2 with log2(e) folded into the scale;
//   * the running maximum used for the exponent is only moved when the block
//     maximum exceeds it by more than 8 (log2 units); then O and l are rescaled.
//     A block is first exponentiated against the current maximum and kept when its
//     row sums stay <= 2^20 (every P <= 2^20, finite); otherwise, and for a row's
//     first block, the block maximum is taken and the rule above applies. The
//     final O/l and lse are invariant to the reference maximum;
//   * P is rounded to bf16 before P V (as the listing does with `.to(v.dtype)`),
//     l sums the unrounded fp32 P.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "ring_schedule.h"
#include "ringattn_internal.h"
#include "sm100_ptx.cuh"
#include "softmax_rows.cuh"

namespace ringattn {
namespace sm100 {

constexpr int BM = 128;          // query rows per tile (TMEM lanes)
constexpr int BN = 128;          // keys per KV tile
constexpr int NQ = 2;            // query tiles per CTA
constexpr int BQ = BM * NQ;      // query rows per unit
constexpr int kSmemLimit = 232448;  // 227 KiB of dynamic shared memory per CTA
constexpr int BOXW = 64;         // bf16 elements per TMA box row (128 bytes, 128B swizzle)
constexpr int kThreads = 384;
constexpr int kLaunchRegs = 168;     // 65536 / 384 rounded down to a multiple of 8
constexpr int kRegsSoftmax = 208;    // per thread, warpgroups 0 and 1
constexpr int kRegsOther = 88;       // per thread, warpgroup 2
static_assert(2 * kRegsSoftmax + kRegsOther <= 3 * kLaunchRegs, "register split exceeds the launch pool");
constexpr int kProducerWarp = 8;
constexpr uint32_t kProducerSleepNs = 64;  // the producer polls slots this often (other back-offs measured neutral)
constexpr int kMmaWarp = 9;
// Of every 8 column pairs of a score row, this many take 2^x from the FMA-pipe
// polynomial (exp2_poly2) and the rest from the MUFU ex2 unit, which the tensor
// cores would otherwise wait on (both run at 16 results/clock/SM for this shape).
// At D = 64 the share did not pay (576-588 against 591 TFLOP/s), so it is 0 here.
constexpr int kEmuPairsPer8 = 0;
constexpr float kSpecMaxSum = 1048576.0f;  // 2^20: the speculative exponentials' row-sum limit

template <int D>
struct Cfg {
  static constexpr int kBoxes = D / BOXW;
  static constexpr int kBoxBytes = BM * BOXW * 2;       // 16 KiB
  static constexpr int kTileBytes = BM * D * 2;         // Q, K or V tile
  static constexpr int kOffQ = 0;
  static constexpr int kOffKV = NQ * kTileBytes;
  // as many K/V slots as fit next to the two Q tiles (5 for D=128, capped at 8)
  static constexpr int kSlotsFit = (kSmemLimit - 1024 - 512 - kOffKV) / kTileBytes;
  static constexpr int kSlots = kSlotsFit < 8 ? kSlotsFit : 8;
  static constexpr int kOffBar = kOffKV + kSlots * kTileBytes;
  static constexpr int kNumBars = 8 + 2 * kSlots;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 64 + 1024;  // + alignment slack
  static_assert(kSlots >= 3, "need at least three K/V slots");
  static_assert(kSmemBytes <= kSmemLimit, "shared memory budget");
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS = 0;                 // + q*BN
  static constexpr uint32_t kColO = 2 * BN;            // + q*D
  static constexpr uint32_t kIdescQK = idesc_bf16_f32(BM, BN, 0, 0);
  static constexpr uint32_t kIdescPV = idesc_bf16_f32(BM, D, 0, 1);
};

struct Params {
  RingGeom g;
  void* out;           // final: bf16 [B,Hq,S,D]; partial: fp32 [B,Hq,Sq,D]; last fold step: bf16 [B,Hq,Sq,D]
  float* lse;          // final: [B,Hq,S];      partial, fold: [B,Hq,Sq]
  int* status;         // workspace status word
  float scale_log2;    // scale * log2(e)
  int s_begin, s_end;  // ring steps folded by every unit
  int q_shard_only;    // -1: all query shards
  FwdOut fo;           // output mode and input layout
  uint64_t watchdog_ns;
};

// Barrier slots: Q full, S ready x2, P ready x2, O done x2, drain, then the K/V
// ring's full[kSlots] and empty[kSlots]. Load m of a unit is K(m/2) for even m and
// V(m/2) for odd m; it uses slot m % kSlots with phase (m / kSlots) & 1.
enum Bar { kQFull = 0, kSFull = 1, kPReady = 3, kODone = 5, kDrain = 7, kRing = 8 };

// Bounded wait that ignores the abort flag: used only to drain in-flight work.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > limit_ns) return;
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    ring_fwd_sm100_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const Params p) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 8);
  uint64_t* full = &bars[kRing];
  uint64_t* empty = &bars[kRing + C::kSlots];

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const RingGeom& g = p.g;

  if (threadIdx.x == 0) {
    mbar_init(&bars[kQFull], 1);
    for (int q = 0; q < NQ; ++q) {
      mbar_init(&bars[kSFull + q], 1);
      mbar_init(&bars[kPReady + q], BM / 32);  // one arrival per softmax warp
      mbar_init(&bars[kODone + q], 1);
    }
    mbar_init(&bars[kDrain], 1);
    for (int s = 0; s < 2 * C::kSlots; ++s) mbar_init(&bars[kRing + s], 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  if (warp == kProducerWarp && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const Watchdog wd{abort_flag, p.status, p.watchdog_ns};
  const Unit U = decode_unit(g, BQ, p.q_shard_only, blockIdx.x);
  const int64_t a0 = (int64_t)U.tb * BQ;
  const int64_t a_hi = (a0 + BQ - 1 < g.Sq - 1) ? a0 + BQ - 1 : g.Sq - 1;
  const int bh_q = U.b * g.Hq + U.h;
  const int bh_kv = U.b * g.Hkv + U.h / (g.Hq / g.Hkv);
  const int64_t N = unit_tile_count(g, U.i, a_hi, BN, p.s_begin, p.s_end);

  if (warp >= 8) {
    regs_decrease<kRegsOther>();
    if (warp == kProducerWarp && lane == 0) {
      // ---------------------------------------------------------------- producer
      int n = 0;
      bool ok = true;
      // a unit with no KV tile (a fully masked single ring step) loads nothing at all,
      // so no copy can still be in flight when the CTA exits
      if (N > 0) {
        mbar_arrive_expect_tx(&bars[kQFull], NQ * C::kTileBytes);
        for (int q = 0; q < NQ; ++q) {
          int c1, c2;
          tile_coords(g, p.fo.local, U.i, a0 + q * BM, c1, c2);
          for (int bx = 0; bx < C::kBoxes; ++bx) {
            uint8_t* dst = smem + C::kOffQ + q * C::kTileBytes + bx * C::kBoxBytes;
            tma_load_4d(dst, &tm_q, &bars[kQFull], bx * BOXW, c1, c2, bh_q);
          }
        }
      }
      for (TileWalk w = walk_begin(g, U.i, a_hi, BN, p.s_begin, p.s_end, launch_anchor(g, p.q_shard_only));
           walk_valid(w); walk_next(g, w, a_hi, BN)) {
        int c1, c2;
        tile_coords(g, p.fo.local, w.j, w.kb * BN, c1, c2);
        for (int kv = 0; kv < 2 && ok; ++kv, ++n) {
          const int slot = n % C::kSlots;
          const uint32_t ph = (uint32_t)(n / C::kSlots) & 1;
          if (!(ok = mbar_wait_backoff<false>(&empty[slot], ph ^ 1, wd, kProducerSleepNs))) break;
          mbar_arrive_expect_tx(&full[slot], C::kTileBytes);
          const void* tm = kv == 0 ? static_cast<const void*>(&tm_k) : static_cast<const void*>(&tm_v);
          for (int bx = 0; bx < C::kBoxes; ++bx) {
            uint8_t* dst = smem + C::kOffKV + slot * C::kTileBytes + bx * C::kBoxBytes;
            tma_load_4d(dst, tm, &full[slot], bx * BOXW, c1, c2, bh_kv);
          }
        }
        if (!ok) break;
      }
      if (!ok) {
        // wind down: let this CTA's own copies land before the shared memory goes away
        drain_wait(&bars[kQFull], 0, p.watchdog_ns);
        for (int m = (n > C::kSlots ? n - C::kSlots : 0); m < n; ++m)
          drain_wait(&full[m % C::kSlots], (uint32_t)(m / C::kSlots) & 1, p.watchdog_ns);
      }
    } else if (warp == kMmaWarp && lane == 0) {
      // ---------------------------------------------------------------- MMA issuer
      const uint32_t sbase = smem_u32(smem);
      // Descriptor bases are built once; every MMA then only adds a compile-time
      // offset (address >> 4) to the start-address field, keeping the issuing thread
      // lean while it shares its scheduler with the softmax warps.
      const uint64_t dq0 = smem_desc_sw128(sbase + C::kOffQ, 0, 1024);
      const uint64_t dk0 = smem_desc_sw128(sbase + C::kOffKV, 0, 1024);
      const uint64_t dv0 = smem_desc_sw128(sbase + C::kOffKV, C::kBoxBytes, 1024);
      auto issue_s = [&](int q, int slot) {
        const uint64_t dq = dq0 + (uint64_t)((q * C::kTileBytes) >> 4);
        const uint64_t dk = dk0 + (uint64_t)((slot * C::kTileBytes) >> 4);
        const uint32_t d = tmem + C::kColS + q * BN;
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = ((k / 4) * C::kBoxBytes + (k % 4) * 32) >> 4;
          mma_ss(d, dq + off, dk + off, C::kIdescQK, k > 0);
        }
      };
      auto issue_pv = [&](int q, int slot, bool first) {
        const uint64_t dv = dv0 + (uint64_t)((slot * C::kTileBytes) >> 4);
        const uint32_t d = tmem + C::kColO + q * D;
        const uint32_t pa = tmem + C::kColS + q * BN;
#pragma unroll
        for (int k = 0; k < BN / 16; ++k) mma_ts(d, pa + k * 8, dv + ((k * 16 * 128) >> 4), C::kIdescPV, !(first && k == 0));
      };
      auto kslot = [&](int64_t n) { return (int)((2 * n) % C::kSlots); };
      auto kphase = [&](int64_t n) { return (uint32_t)(((2 * n) / C::kSlots) & 1); };
      auto vslot = [&](int64_t n) { return (int)((2 * n + 1) % C::kSlots); };
      auto vphase = [&](int64_t n) { return (uint32_t)(((2 * n + 1) / C::kSlots) & 1); };
      bool ok = N > 0 && mbar_wait(&bars[kQFull], 0, wd);
      if (ok) ok = mbar_wait(&full[kslot(0)], kphase(0), wd);
      if (ok) {
        tc_fence_after();
        issue_s(0, kslot(0));
        mma_commit(&bars[kSFull + 0]);
        issue_s(1, kslot(0));
        mma_commit(&bars[kSFull + 1]);
        mma_commit(&empty[kslot(0)]);
      }
      // Issue order per KV tile n: PV0(n), S0(n+1), PV1(n), S1(n+1). A commit after
      // S0(n+1) implies PV0(n) has completed, so softmax 0 may rescale O0 as soon as
      // it sees S0(n+1); each softmax overlaps the other tile's PV and S MMAs.
      for (int64_t n = 0; ok && n < N; ++n) {
        const bool more = n + 1 < N;
        if (!(ok = mbar_wait(&full[vslot(n)], vphase(n), wd))) break;
        if (!(ok = mbar_wait(&bars[kPReady + 0], (uint32_t)(n & 1), wd))) break;
        tc_fence_after();
        issue_pv(0, vslot(n), n == 0);
        if (more) {
          if (!(ok = mbar_wait(&full[kslot(n + 1)], kphase(n + 1), wd))) break;
          tc_fence_after();
          issue_s(0, kslot(n + 1));
          mma_commit(&bars[kSFull + 0]);
        } else {
          mma_commit(&bars[kODone + 0]);
        }
        if (!(ok = mbar_wait(&bars[kPReady + 1], (uint32_t)(n & 1), wd))) break;
        tc_fence_after();
        issue_pv(1, vslot(n), n == 0);
        mma_commit(&empty[vslot(n)]);
        if (more) {
          issue_s(1, kslot(n + 1));
          mma_commit(&bars[kSFull + 1]);
          mma_commit(&empty[kslot(n + 1)]);
        } else {
          mma_commit(&bars[kODone + 1]);
        }
      }
      // every MMA this thread issued must finish before TMEM is released
      mma_commit(&bars[kDrain]);
      drain_wait(&bars[kDrain], 0, p.watchdog_ns);
    }
  } else {
    regs_increase<kRegsSoftmax>();
    // -------------------------------------------------------------------- softmax
    const int q = warp / 4;
    const int wq = warp % 4;
    const int r = wq * 32 + lane;
    const int64_t a = a0 + q * BM + r;  // local query index in shard U.i
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t tS = tmem + lane_off + C::kColS + q * BN;
    const uint32_t tO = tmem + lane_off + C::kColO + q * D;
    const float NEG_INF = -INFINITY;
    float m_ref = NEG_INF;
    float l = 0.f;
    int n = 0;
    bool ok = true;
    TileWalk w = walk_begin(g, U.i, a_hi, BN, p.s_begin, p.s_end, launch_anchor(g, p.q_shard_only));
    for (; walk_valid(w); walk_next(g, w, a_hi, BN), ++n) {
      if (!(ok = mbar_wait(&bars[kSFull + q], (uint32_t)(n & 1), wd))) break;
      tc_fence_after();
      uint32_t sr[BN];
#pragma unroll
      for (int c = 0; c < BN / 32; ++c) tmem_ld32(tS + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
      tmem_wait_ld();
      // mask on the raw scores (scale > 0 keeps the order): keys b >= lim are out
      const int cut = visible_keys<BN>((int64_t)w.kb * BN, key_limit(g, U.i, w.j, a));
      mask_scores<BN>(sr, cut);
      // a block no row of this warp can see contributes nothing: P = 0, state unchanged
      const bool warp_empty = __all_sync(0xffffffffu, cut == 0);
      uint32_t pk[BN / 2];
      if (warp_empty) {
#pragma unroll
        for (int c = 0; c < BN / 2; ++c) pk[c] = 0u;
      } else {
        // Exponentials against the current reference maximum first (O/l and lse do not
        // depend on it); a block whose row sums stay <= kSpecMaxSum (every P <= 2^20,
        // finite) is kept. Otherwise, and for the first block, the warp reloads the
        // scores, takes the block maximum and follows the rescale rule.
        float lb = 0.f;
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
      if (lane == 0) mbar_arrive(&bars[kPReady + q]);
    }
    const bool have = (n > 0) && ok && mbar_wait(&bars[kODone + q], 0, wd);
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
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ------------------------------------------------------------------------------ host
template <int D>
static int launch_impl(const void* q, const void* k, const void* v, void* out, float* lse, const RingGeom& g,
                       float scale, int s_begin, int s_end, int q_shard_only, const FwdOut& fo, int* status,
                       uint64_t watchdog_ns, cudaStream_t stream) {
  using C = Cfg<D>;
  CUtensorMap mq, mk, mv;
  int rc;
  const bool local = fo.local != 0;
  if ((rc = encode_input_map(&mq, q, g, local, g.Hq, D, BM)) != 0) return rc;
  if ((rc = encode_input_map(&mk, k, g, local, g.Hkv, D, BN)) != 0) return rc;
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
  if (cudaFuncSetAttribute(ring_fwd_sm100_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           C::kSmemBytes) != cudaSuccess)
    return RING_ATTN_ECUDA;
  // The register split reallocates the block's launch pool (threads x registers at
  // launch); refuse to launch if the compiled kernel was given fewer registers than
  // the split needs, instead of letting setmaxnreg.inc wait forever.
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, ring_fwd_sm100_kernel<D>) != cudaSuccess) return RING_ATTN_ECUDA;
  if (fa.numRegs * kThreads < 128 * (2 * kRegsSoftmax + kRegsOther)) return RING_ATTN_EUNSUPPORTED;
  const int64_t units = num_units(g, BQ, q_shard_only);
  if (units == 0) return RING_ATTN_OK;
  ring_fwd_sm100_kernel<D><<<(unsigned)units, kThreads, C::kSmemBytes, stream>>>(mq, mk, mv, p);
  return cudaGetLastError() == cudaSuccess ? RING_ATTN_OK : RING_ATTN_ECUDA;
}

}  // namespace sm100

int launch_fwd_sm100(const void* q, const void* k, const void* v, void* out, float* lse, const RingGeom& g,
                     float scale, int s_begin, int s_end, int q_shard_only, const FwdOut& fo, int* status,
                     uint64_t watchdog_ns, cudaStream_t stream) {
  if (g.D == 128)
    return sm100::launch_impl<128>(q, k, v, out, lse, g, scale, s_begin, s_end, q_shard_only, fo, status,
                                   watchdog_ns, stream);
  if (g.D == 64)
    return sm100::launch_impl<64>(q, k, v, out, lse, g, scale, s_begin, s_end, q_shard_only, fo, status,
                                  watchdog_ns, stream);
  return RING_ATTN_EUNSUPPORTED;
}

int64_t fwd_sm100_units(const RingGeom& g, int q_shard_only) { return num_units(g, sm100::BQ, q_shard_only); }

}  // namespace ringattn
