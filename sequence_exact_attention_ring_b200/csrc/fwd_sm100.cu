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
//   warp 8     TMA producer: Q once, then K and V tiles into 2-stage rings
//   warp 9     TMEM owner; lane 0 issues every tcgen05.mma and commit
//   warps 10-11 idle (they complete the third warpgroup for the register split)
// Registers: launched at 168 per thread; the softmax warpgroups grow to 208 and
// the third warpgroup shrinks to 88 (2*208 + 88 = 3*168).
// Tensor memory (512 columns): S0 [0,128) S1 [128,256) O0 [256,256+D) O1 [256+D,256+2D).
// P (bf16) overwrites the first 64 columns of its S tile and feeds the PV MMA
// directly from TMEM.
//
// Differences from the pages' listing (same result up to rounding):
//   * exponentials are base 2 with log2(e) folded into the scale;
//   * the running maximum used for the exponent is only moved when the block
//     maximum exceeds it by more than 8 (log2 units); then O and l are rescaled.
//     Otherwise exponents stay <= 2^8, exact in fp32 and bf16 range. The final O/l
//     and lse are invariant to the reference maximum;
//   * P is rounded to bf16 before P V (as the listing does with `.to(v.dtype)`),
//     l sums the unrounded fp32 P.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "ring_schedule.h"
#include "ringattn_internal.h"
#include "sm100_ptx.cuh"

namespace ringattn {
namespace sm100 {

constexpr int BM = 128;          // query rows per tile (TMEM lanes)
constexpr int BN = 128;          // keys per KV tile
constexpr int NQ = 2;            // query tiles per CTA
constexpr int BQ = BM * NQ;      // query rows per unit
constexpr int STAGES = 2;        // K and V ring depth
constexpr int BOXW = 64;         // bf16 elements per TMA box row (128 bytes, 128B swizzle)
constexpr int kThreads = 384;
constexpr int kLaunchRegs = 168;     // 65536 / 384 rounded down to a multiple of 8
constexpr int kRegsSoftmax = 208;    // per thread, warpgroups 0 and 1
constexpr int kRegsOther = 88;       // per thread, warpgroup 2
static_assert(2 * kRegsSoftmax + kRegsOther <= 3 * kLaunchRegs, "register split exceeds the launch pool");
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
// Of every 8 column pairs of a score row, this many take 2^x from the FMA-pipe
// polynomial (exp2_poly2) and the rest from the MUFU ex2 unit, which the tensor
// cores would otherwise wait on (both run at 16 results/clock/SM for this shape).
constexpr int kEmuPairsPer8 = 2;

template <int D>
struct Cfg {
  static constexpr int kBoxes = D / BOXW;
  static constexpr int kBoxBytes = BM * BOXW * 2;       // 16 KiB
  static constexpr int kTileBytes = BM * D * 2;         // Q, K or V tile
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = NQ * kTileBytes;
  static constexpr int kOffV = kOffK + STAGES * kTileBytes;
  static constexpr int kOffBar = kOffV + STAGES * kTileBytes;
  static constexpr int kNumBars = 16;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 64 + 1024;  // + alignment slack
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS = 0;                 // + q*BN
  static constexpr uint32_t kColO = 2 * BN;            // + q*D
  static constexpr uint32_t kIdescQK = idesc_bf16_f32(BM, BN, 0, 0);
  static constexpr uint32_t kIdescPV = idesc_bf16_f32(BM, D, 0, 1);
};

struct Params {
  RingGeom g;
  void* out;           // final: bf16 [B,Hq,S,D]; partial: fp32 [B,Hq,Sq,D]
  float* lse;          // final: [B,Hq,S];      partial: [B,Hq,Sq]
  int* status;         // workspace status word
  float scale_log2;    // scale * log2(e)
  int s_begin, s_end;  // ring steps folded by every unit
  int q_shard_only;    // -1: all query shards
  int partial;         // 1: write the normalised per-step partial (fp32, local order)
  uint64_t watchdog_ns;
};

enum Bar { kQFull = 0, kKFull = 1, kKEmpty = 3, kVFull = 5, kVEmpty = 7, kSFull = 9, kPReady = 11,
           kODone = 13, kDrain = 15 };

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

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const RingGeom& g = p.g;

  if (threadIdx.x == 0) {
    mbar_init(&bars[kQFull], 1);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&bars[kKFull + s], 1);
      mbar_init(&bars[kKEmpty + s], 1);
      mbar_init(&bars[kVFull + s], 1);
      mbar_init(&bars[kVEmpty + s], 1);
    }
    for (int q = 0; q < NQ; ++q) {
      mbar_init(&bars[kSFull + q], 1);
      mbar_init(&bars[kPReady + q], BM);
      mbar_init(&bars[kODone + q], 1);
    }
    mbar_init(&bars[kDrain], 1);
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
  const bool striped = g.layout == kStriped;

  if (warp >= 8) {
    regs_decrease<kRegsOther>();
  if (warp == kProducerWarp) {
    if (lane == 0) {
      // ---------------------------------------------------------------- producer
      int n = 0;
      bool ok = true;
      mbar_arrive_expect_tx(&bars[kQFull], NQ * C::kTileBytes);
      for (int q = 0; q < NQ; ++q) {
        const int row = (int)(a0 + q * BM);
        for (int bx = 0; bx < C::kBoxes; ++bx) {
          uint8_t* dst = smem + C::kOffQ + q * C::kTileBytes + bx * C::kBoxBytes;
          if (striped)
            tma_load_4d(dst, &tm_q, &bars[kQFull], bx * BOXW, U.i, row, bh_q);
          else
            tma_load_4d(dst, &tm_q, &bars[kQFull], bx * BOXW, row, U.i, bh_q);
        }
      }
      TileWalk w = walk_begin(g, U.i, a_hi, BN, p.s_begin, p.s_end);
      for (; walk_valid(w); walk_next(g, w, a_hi, BN), ++n) {
        const int slot = n % STAGES;
        const uint32_t ph = (n / STAGES) & 1;
        const int krow = w.kb * BN;
        if (!(ok = mbar_wait(&bars[kKEmpty + slot], ph ^ 1, wd))) break;
        mbar_arrive_expect_tx(&bars[kKFull + slot], C::kTileBytes);
        for (int bx = 0; bx < C::kBoxes; ++bx) {
          uint8_t* dst = smem + C::kOffK + slot * C::kTileBytes + bx * C::kBoxBytes;
          if (striped)
            tma_load_4d(dst, &tm_k, &bars[kKFull + slot], bx * BOXW, w.j, krow, bh_kv);
          else
            tma_load_4d(dst, &tm_k, &bars[kKFull + slot], bx * BOXW, krow, w.j, bh_kv);
        }
        if (!(ok = mbar_wait(&bars[kVEmpty + slot], ph ^ 1, wd))) {
          ++n;  // the K load of this tile is in flight
          break;
        }
        mbar_arrive_expect_tx(&bars[kVFull + slot], C::kTileBytes);
        for (int bx = 0; bx < C::kBoxes; ++bx) {
          uint8_t* dst = smem + C::kOffV + slot * C::kTileBytes + bx * C::kBoxBytes;
          if (striped)
            tma_load_4d(dst, &tm_v, &bars[kVFull + slot], bx * BOXW, w.j, krow, bh_kv);
          else
            tma_load_4d(dst, &tm_v, &bars[kVFull + slot], bx * BOXW, krow, w.j, bh_kv);
        }
      }
      if (!ok) {
        // wind down: let this CTA's own copies land before the shared memory goes away
        drain_wait(&bars[kQFull], 0, p.watchdog_ns);
        for (int m = (n > STAGES ? n - STAGES : 0); m < n; ++m) {
          drain_wait(&bars[kKFull + m % STAGES], (m / STAGES) & 1, p.watchdog_ns);
          drain_wait(&bars[kVFull + m % STAGES], (m / STAGES) & 1, p.watchdog_ns);
        }
      }
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      // ---------------------------------------------------------------- MMA issuer
      const int64_t N = unit_tile_count(g, U.i, a_hi, BN, p.s_begin, p.s_end);
      const uint32_t sbase = smem_u32(smem);
      auto issue_s = [&](int q, int slot) {
        const uint32_t qa = sbase + C::kOffQ + q * C::kTileBytes;
        const uint32_t ka = sbase + C::kOffK + slot * C::kTileBytes;
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = (k / 4) * C::kBoxBytes + (k % 4) * 32;
          mma_ss(tmem + C::kColS + q * BN, smem_desc_sw128(qa + off, 0, 1024), smem_desc_sw128(ka + off, 0, 1024),
                 C::kIdescQK, k > 0);
        }
      };
      auto issue_pv = [&](int q, int slot, bool first) {
        const uint32_t va = sbase + C::kOffV + slot * C::kTileBytes;
#pragma unroll
        for (int k = 0; k < BN / 16; ++k) {
          mma_ts(tmem + C::kColO + q * D, tmem + C::kColS + q * BN + k * 8,
                 smem_desc_sw128(va + k * 16 * 128, C::kBoxBytes, 1024), C::kIdescPV, !(first && k == 0));
        }
      };
      bool ok = N > 0 && mbar_wait(&bars[kQFull], 0, wd);
      if (ok) ok = mbar_wait(&bars[kKFull], 0, wd);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        mma_commit(&bars[kSFull + 0]);
        issue_s(1, 0);
        mma_commit(&bars[kSFull + 1]);
        mma_commit(&bars[kKEmpty + 0]);
      }
      for (int64_t n = 0; ok && n < N; ++n) {
        const int slot = (int)(n % STAGES);
        const uint32_t ph = (uint32_t)((n / STAGES) & 1);
        const int ns = (int)((n + 1) % STAGES);
        const uint32_t nph = (uint32_t)(((n + 1) / STAGES) & 1);
        const bool more = n + 1 < N;
        if (!(ok = mbar_wait(&bars[kVFull + slot], ph, wd))) break;
        if (!(ok = mbar_wait(&bars[kPReady + 0], (uint32_t)(n & 1), wd))) break;
        tc_fence_after();
        issue_pv(0, slot, n == 0);
        if (more) {
          if (!(ok = mbar_wait(&bars[kKFull + ns], nph, wd))) break;
          tc_fence_after();
          issue_s(0, ns);
          mma_commit(&bars[kSFull + 0]);
        } else {
          mma_commit(&bars[kODone + 0]);
        }
        if (!(ok = mbar_wait(&bars[kPReady + 1], (uint32_t)(n & 1), wd))) break;
        tc_fence_after();
        issue_pv(1, slot, n == 0);
        mma_commit(&bars[kVEmpty + slot]);
        if (more) {
          issue_s(1, ns);
          mma_commit(&bars[kSFull + 1]);
          mma_commit(&bars[kKEmpty + ns]);
        } else {
          mma_commit(&bars[kODone + 1]);
        }
      }
      // every MMA this thread issued must finish before TMEM is released
      mma_commit(&bars[kDrain]);
      drain_wait(&bars[kDrain], 0, p.watchdog_ns);
    }
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
    TileWalk w = walk_begin(g, U.i, a_hi, BN, p.s_begin, p.s_end);
    for (; walk_valid(w); walk_next(g, w, a_hi, BN), ++n) {
      if (!(ok = mbar_wait(&bars[kSFull + q], (uint32_t)(n & 1), wd))) break;
      tc_fence_after();
      uint32_t sr[BN];
#pragma unroll
      for (int c = 0; c < BN / 32; ++c) tmem_ld32(tS + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
      tmem_wait_ld();
      // mask on the raw scores (scale > 0 keeps the order): keys b >= lim are out
      const int64_t lim = key_limit(g, U.i, w.j, a);
      const int64_t kb0 = (int64_t)w.kb * BN;
      if (kb0 + BN > lim) {
#pragma unroll
        for (int c = 0; c < BN; ++c)
          if (kb0 + c >= lim) sr[c] = 0xff800000u;  // -inf
      }
      // row max: 8 independent chains of three-input max, then combine
      float mx[8];
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {
        const uint32_t* v = &sr[ch * 16];
        float m8 = fmax3(__uint_as_float(v[0]), __uint_as_float(v[1]), __uint_as_float(v[2]));
#pragma unroll
        for (int e = 3; e < 15; e += 2) m8 = fmax3(m8, __uint_as_float(v[e]), __uint_as_float(v[e + 1]));
        mx[ch] = fmaxf(m8, __uint_as_float(v[15]));
      }
      const float mraw = fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
      const float mblk = mraw * p.scale_log2;
      float alpha = 1.f;
      bool resc = false;
      if (n == 0) {
        m_ref = mblk;
      } else if (mblk > m_ref + kRescaleThreshold) {
        alpha = (m_ref == NEG_INF) ? 0.f : ex2_approx(m_ref - mblk);
        l *= alpha;
        m_ref = mblk;
        resc = true;
      }
      if (__any_sync(0xffffffffu, resc)) {
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + c * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(tO + c * 32, o);
        }
        tmem_wait_st();
      }
      // p = 2^(s*scale*log2e - m): one packed FMA per two scores, then ex2
      const uint64_t c2 = f2_splat(p.scale_log2);
      const uint64_t negm = f2_splat((m_ref == NEG_INF) ? 0.f : -m_ref);
      uint64_t acc[4] = {0, 0, 0, 0};
      uint32_t pk[BN / 2];
#pragma unroll
      for (int c = 0; c < BN; c += 2) {
        const uint64_t xy = f2_fma(f2_pack(sr[c], sr[c + 1]), c2, negm);
        uint64_t pp;
        if ((c / 2) % 8 < kEmuPairsPer8) {
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
      {
        const uint64_t t = f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3]));
        float t0, t1;
        f2_unpack(t, t0, t1);
        l += t0 + t1;
      }
#pragma unroll
      for (int c = 0; c < BN / 64; ++c) tmem_st32(tS + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[c * 32]));
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars[kPReady + q]);
    }
    const bool have = (n > 0) && ok && mbar_wait(&bars[kODone + q], 0, wd);
    if (have || n == 0) {
      tc_fence_after();
      const bool row_ok = a < g.Sq;
      const bool empty = !(l > 0.f);
      const float inv_l = empty ? 0.f : 1.f / l;
      const float lse_v = empty ? NEG_INF : (m_ref + log2f(l)) * 0.69314718055994530942f;
      const int64_t tok = token_of(g, U.i, a);
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        if (n > 0) {
          tmem_ld32(tO + c * 32, o);
          tmem_wait_ld();
        }
        if (!row_ok) continue;
        if (p.partial) {
          float* dst = reinterpret_cast<float*>(p.out) + ((int64_t)bh_q * g.Sq + a) * D + c * 32;
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            float4 v4;
            v4.x = (n > 0) ? __uint_as_float(o[e]) * inv_l : 0.f;
            v4.y = (n > 0) ? __uint_as_float(o[e + 1]) * inv_l : 0.f;
            v4.z = (n > 0) ? __uint_as_float(o[e + 2]) * inv_l : 0.f;
            v4.w = (n > 0) ? __uint_as_float(o[e + 3]) * inv_l : 0.f;
            *reinterpret_cast<float4*>(dst + e) = v4;
          }
        } else {
          uint32_t* dst = reinterpret_cast<uint32_t*>(reinterpret_cast<uint16_t*>(p.out) +
                                                      ((int64_t)bh_q * g.S + tok) * D + c * 32);
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
      if (row_ok) {
        if (p.partial)
          p.lse[(int64_t)bh_q * g.Sq + a] = lse_v;
        else
          p.lse[(int64_t)bh_q * g.S + tok] = lse_v;
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
static PFN_encodeTiled get_encode_fn() {
  static PFN_encodeTiled fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult qres;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &qres) == cudaSuccess &&
        qres == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_encodeTiled>(ptr);
  }
  return fn;
}

// 4-D view (D, local, shard, batch*heads) of a [B, H, S, D] bf16 tensor whose
// sequence axis is split into P shards: contiguous shards are consecutive token
// ranges, striped shards interleave with stride P. Dimensions are listed
// innermost first so the strides grow; the kernel swaps the two middle
// coordinates for the striped layout.
static int encode_shard_map(CUtensorMap* map, const void* base, const RingGeom& g, int heads, int D) {
  PFN_encodeTiled enc = get_encode_fn();
  if (!enc) return RING_ATTN_ECUDA;
  cuuint64_t dims[4];
  cuuint64_t strides[3];
  cuuint32_t box[4];
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const uint64_t row = (uint64_t)D * 2;
  if (g.layout == kStriped) {
    dims[0] = D; dims[1] = g.P; dims[2] = g.Sq; dims[3] = (uint64_t)g.B * heads;
    strides[0] = row; strides[1] = row * g.P; strides[2] = row * g.S;
    box[0] = BOXW; box[1] = 1; box[2] = BM; box[3] = 1;
  } else {
    dims[0] = D; dims[1] = g.Sq; dims[2] = g.P; dims[3] = (uint64_t)g.B * heads;
    strides[0] = row; strides[1] = row * g.Sq; strides[2] = row * g.S;
    box[0] = BOXW; box[1] = BM; box[2] = 1; box[3] = 1;
  }
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? RING_ATTN_OK : RING_ATTN_ECUDA;
}

template <int D>
static int launch_impl(const void* q, const void* k, const void* v, void* out, float* lse, const RingGeom& g,
                       float scale, int s_begin, int s_end, int q_shard_only, int partial, int* status,
                       uint64_t watchdog_ns, cudaStream_t stream) {
  using C = Cfg<D>;
  CUtensorMap mq, mk, mv;
  int rc;
  if ((rc = encode_shard_map(&mq, q, g, g.Hq, D)) != 0) return rc;
  if ((rc = encode_shard_map(&mk, k, g, g.Hkv, D)) != 0) return rc;
  if ((rc = encode_shard_map(&mv, v, g, g.Hkv, D)) != 0) return rc;
  Params p;
  p.g = g;
  p.out = out;
  p.lse = lse;
  p.status = status;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.s_begin = s_begin;
  p.s_end = s_end;
  p.q_shard_only = q_shard_only;
  p.partial = partial;
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
                     float scale, int s_begin, int s_end, int q_shard_only, int partial, int* status,
                     uint64_t watchdog_ns, cudaStream_t stream) {
  if (g.D == 128)
    return sm100::launch_impl<128>(q, k, v, out, lse, g, scale, s_begin, s_end, q_shard_only, partial, status,
                                   watchdog_ns, stream);
  if (g.D == 64)
    return sm100::launch_impl<64>(q, k, v, out, lse, g, scale, s_begin, s_end, q_shard_only, partial, status,
                                  watchdog_ns, stream);
  return RING_ATTN_EUNSUPPORTED;
}

int64_t fwd_sm100_units(const RingGeom& g, int q_shard_only) { return num_units(g, sm100::BQ, q_shard_only); }

}  // namespace ringattn
