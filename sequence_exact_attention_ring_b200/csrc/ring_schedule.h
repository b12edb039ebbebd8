// Ring geometry and schedule shared by the host scheduler and every kernel.
//
// RingAttention deep-architecture article (techknowgenie):
//   section 2 "core principle": the sequence of S tokens is cut into P shards of
//     Sq = S/P tokens; query shard i never moves, and at ring step s it meets the
//     KV shard (i - s) mod P (blocks travel to the next device, arrive from the
//     previous one; step 0 is the device's own block, per the section 5 listing).
//   section 7 "causal attention with striped attention": under a causal mask
//     token t sees only tokens u <= t (inclusive diagonal); the striped layout
//     deals tokens round-robin, token t on shard t mod P.
// RingAttention newsletter (cmlonder), section "claim and reality": striped or
//   zigzag schedules balance the causal ring. Zigzag is named there without a
//   definition; the reading used here cuts the sequence into 2P chunks of
//   C = S/(2P) tokens and gives shard i chunks i and 2P-1-i, in that order.
//
// On one GPU the ring becomes the order in which a work unit visits KV tiles.
// Everything here is plain integer arithmetic, compiled for both host and device
// so the CPU tests check the exact code the kernels run.
#pragma once

#include <stdint.h>

#if defined(__CUDACC__)
#define RA_HD __host__ __device__ __forceinline__
#else
#define RA_HD inline
#endif

namespace ringattn {

enum Layout : int { kContiguous = 0, kStriped = 1, kZigzag = 2 };

struct RingGeom {
  int B, Hq, Hkv;
  int64_t S;
  int D, P;
  int causal;   // 0 | 1
  int layout;   // kContiguous | kStriped | kZigzag
  int64_t Sq;   // S / P
};

// Global token of local index a in shard i.
//   contiguous: shard i = tokens [i*Sq, (i+1)*Sq); striped: token a*P + i;
//   zigzag: a < C is token i*C + a, a >= C is token (2P-1-i)*C + (a - C).
RA_HD int64_t token_of(const RingGeom& g, int i, int64_t a) {
  if (g.layout == kStriped) return a * g.P + i;
  if (g.layout == kZigzag) {
    const int64_t C = g.Sq / 2;
    return a < C ? (int64_t)i * C + a : (int64_t)(2 * g.P - 1 - i) * C + (a - C);
  }
  return (int64_t)i * g.Sq + a;
}

// Coordinates (dim 1, dim 2) of local row a of shard i in the layout's 4-D tensor
// map; dim 0 is the head dimension and dim 3 batch*heads (see encode_shard_map).
// Rows past the end of a shard land outside the map and are zero-filled by TMA.
RA_HD void shard_map_coords(const RingGeom& g, int i, int64_t a, int& c1, int& c2) {
  if (g.layout == kStriped) {
    c1 = i;
    c2 = (int)a;
  } else if (g.layout == kZigzag) {
    const int64_t C = g.Sq / 2;
    c1 = (int)(a < C ? a : a - C);
    c2 = a < C ? i : 2 * g.P - 1 - i;
  } else {
    c1 = (int)a;
    c2 = i;
  }
}

// Tensor-map coordinates of local row a of shard i: in the sharded view of the whole
// sequence (shard_map_coords), or, when the tensor holds only that one shard in
// shard-local order (a device of a multi-GPU ring holds one query shard and one KV
// shard at a time), row a of that buffer.
RA_HD void tile_coords(const RingGeom& g, bool local, int i, int64_t a, int& c1, int& c2) {
  if (local) {
    c1 = (int)a;
    c2 = 0;
  } else {
    shard_map_coords(g, i, a, c1, c2);
  }
}

// KV shard met by query shard i at ring step s (0 <= s < P).
RA_HD int ring_kv_shard(int i, int s, int P) { return (i - s + P) % P; }

// Ring step at which query shard i meets KV shard j.
RA_HD int ring_step_of(int i, int j, int P) { return (i - j + P) % P; }

// Keys of shard j visible to the query with local index a in shard i are exactly
// the local indices b < key_limit(g, i, j, a) (always further capped at Sq).
//   contiguous causal: j < i all keys; j == i keys b <= a; j > i none.
//   striped causal: token b*P+j <= a*P+i  <=>  b < a, or b == a and j <= i.
//   zigzag causal: shard j's tokens rise with b (its first chunk precedes its
//     second), so the visible keys are those of each chunk up to token t.
RA_HD int64_t key_limit(const RingGeom& g, int i, int j, int64_t a) {
  int64_t lim;
  if (!g.causal) {
    lim = g.Sq;
  } else if (g.layout == kContiguous) {
    lim = (j < i) ? g.Sq : (j == i ? a + 1 : 0);
  } else if (g.layout == kZigzag) {
    const int64_t C = g.Sq / 2;
    const int64_t t = token_of(g, i, a);
    int64_t lo = t - (int64_t)j * C + 1;
    int64_t hi = t - (int64_t)(2 * g.P - 1 - j) * C + 1;
    lo = lo < 0 ? 0 : (lo > C ? C : lo);
    hi = hi < 0 ? 0 : (hi > C ? C : hi);
    lim = lo + hi;
  } else {
    lim = (j <= i) ? a + 1 : a;
  }
  return lim < g.Sq ? lim : g.Sq;
}

// Number of TK-key tiles of shard j that the query rows [.., a_hi] of shard i
// must visit (key_limit is non-decreasing in a, so the last row decides).
RA_HD int kv_tiles_for(const RingGeom& g, int i, int j, int64_t a_hi, int TK) {
  int64_t lim = key_limit(g, i, j, a_hi);
  return (int)((lim + TK - 1) / TK);
}

// Work units. A unit is (b, h, q shard i, block of BQ query rows tb), folding
// ring steps [s_begin, s_end). A grid runs its units roughly in index order:
//   contiguous causal: cost grows with i*nkt + (rows of tb), so units are numbered
//     longest first by the combined index c = i*nblk + tb, descending;
//   striped causal and every non-causal layout ("block-major"): tb descending (a
//     block's cost grows with its local index), inside a tb by (b, kv head, i, head in
//     the GQA group). The units of one (b, kv head, tb) have the same number of key
//     tiles in every shard (within one tile at the diagonal), so for long sequences
//     (launch_anchor) they all walk the ring from the same shard and read the same K/V
//     tiles at about the same time: L2 serves the re-reads of every query shard and
//     head of the group;
//   zigzag causal, long sequences (grouped_order: one (b, kv head)'s K and V take
//     >= 32 MiB in bf16, so the K/V of the heads in flight no longer fits in L2): a
//     shard's tile counts depend on the query shard here, so units are grouped by
//     (b, kv head, query shard i), each group's blocks longest first (tb descending),
//     the query heads of a GQA group innermost; a group walks the same ring sequence
//     of KV shards and starts together;
//   zigzag causal, shorter sequences with whole blocks per chunk: the 2P chunks from
//     the last to the first (cost grows with the block's global position).
struct Unit {
  int b, h, i, tb;
};

RA_HD int64_t num_row_blocks(const RingGeom& g, int BQ) { return (g.Sq + BQ - 1) / BQ; }

RA_HD int64_t num_units(const RingGeom& g, int BQ, int q_shard_only) {
  int64_t shards = q_shard_only >= 0 ? 1 : g.P;
  return (int64_t)g.B * g.Hq * shards * num_row_blocks(g, BQ);
}

// K and V of one (b, kv head) take 4*S*D bytes in bf16; at >= 32 MiB the grouped
// launch orders are used (see above).
RA_HD bool grouped_order(const RingGeom& g) { return g.S * (int64_t)g.D >= ((int64_t)1 << 23); }

RA_HD Unit decode_unit(const RingGeom& g, int BQ, int q_shard_only, int64_t u) {
  const int64_t nblk = num_row_blocks(g, BQ);
  const int rep = g.Hq / g.Hkv;
  Unit r;
  if (q_shard_only >= 0) {
    // a single query shard (one literal ring step): (tb desc, b, head)
    const int64_t bh_n = (int64_t)g.B * g.Hq;
    r.tb = (int)(nblk - 1 - u / bh_n);
    int64_t bh = u % bh_n;
    r.b = (int)(bh / g.Hq);
    r.h = (int)(bh % g.Hq);
    r.i = q_shard_only;
    return r;
  }
  if (g.causal && g.layout == kContiguous) {
    const int64_t bh_n = (int64_t)g.B * g.Hq;
    const int64_t c = (int64_t)g.P * nblk - 1 - u / bh_n;
    int64_t bh = u % bh_n;
    r.i = (int)(c / nblk);
    r.tb = (int)(c % nblk);
    int64_t bg = bh / rep;  // (b, kv head) outer, GQA group member inner
    r.b = (int)(bg / g.Hkv);
    r.h = (int)((bg % g.Hkv) * rep + bh % rep);
    return r;
  }
  if (g.causal && g.layout == kZigzag && grouped_order(g)) {
    int64_t x = u;  // (((b*Hkv + kvh)*P + i)*nblk + (nblk-1-tb))*rep + hr
    const int hr = (int)(x % rep);
    x /= rep;
    r.tb = (int)(nblk - 1 - x % nblk);
    x /= nblk;
    r.i = (int)(x % g.P);
    x /= g.P;
    const int kvh = (int)(x % g.Hkv);
    r.b = (int)(x / g.Hkv);
    r.h = kvh * rep + hr;
    return r;
  }
  if (g.causal && g.layout == kZigzag && (g.Sq / 2) % BQ == 0) {
    const int64_t bh_n = (int64_t)g.B * g.Hq;
    const int64_t nbc = nblk / 2;  // blocks per chunk
    const int64_t pos = (int64_t)g.P * nblk - 1 - u / bh_n;
    const int c = (int)(pos / nbc);
    r.i = c < g.P ? c : 2 * g.P - 1 - c;
    r.tb = (int)((c < g.P ? 0 : nbc) + pos % nbc);
    int64_t bh = u % bh_n;
    int64_t bg = bh / rep;
    r.b = (int)(bg / g.Hkv);
    r.h = (int)((bg % g.Hkv) * rep + bh % rep);
    return r;
  }
  const int64_t per_tb = (int64_t)g.B * g.Hq * g.P;
  r.tb = (int)(nblk - 1 - u / per_tb);
  int64_t x = u % per_tb;  // ((b*Hkv + kvh)*P + i)*rep + hr
  const int hr = (int)(x % rep);
  x /= rep;
  r.i = (int)(x % g.P);
  x /= g.P;
  const int kvh = (int)(x % g.Hkv);
  r.b = (int)(x / g.Hkv);
  r.h = kvh * rep + hr;
  return r;
}

// Total KV tiles a unit visits over ring steps [s_begin, s_end).
RA_HD int64_t unit_tile_count(const RingGeom& g, int i, int64_t a_hi, int TK, int s_begin, int s_end) {
  int64_t n = 0;
  for (int s = s_begin; s < s_end; ++s) n += kv_tiles_for(g, i, ring_kv_shard(i, s, g.P), a_hi, TK);
  return n;
}

// The shard a full launch's walks count the ring from. In the literal ring, query shard
// i holds its own KV shard at step 0 (anchor i, the default, -1). On one GPU the fold
// does not depend on where a query shard's ring starts (exact up to rounding), so for
// long block-major launches every unit counts the ring from the last shard instead:
// units of one (b, kv head, tb) then read the same KV shard at the same time. Single
// ring steps (q_shard_only >= 0) keep the literal step.
RA_HD int launch_anchor(const RingGeom& g, int q_shard_only) {
  const bool block_major = g.layout == kStriped || !g.causal;
  return (q_shard_only < 0 && block_major && grouped_order(g)) ? g.P - 1 : -1;
}

// Incremental walk over the (ring step, kv tile) sequence of one unit; every role
// of a kernel advances an identical copy, so they agree on every tile.
struct TileWalk {
  int s, s_end, j, kb, nkb;
  int i, P;
  int rev;     // 1: the backward ring, KV shard (anchor + s) mod P at step s
  int anchor;  // step s holds KV shard (anchor - s) mod P (forward ring)
};

RA_HD void walk_skip_empty(const RingGeom& g, TileWalk& w, int64_t a_hi, int TK) {
  while (w.s < w.s_end) {
    w.j = w.rev ? (w.anchor + w.s) % g.P : ring_kv_shard(w.anchor, w.s, g.P);
    w.nkb = kv_tiles_for(g, w.i, w.j, a_hi, TK);
    if (w.nkb > 0) return;
    ++w.s;
  }
}

RA_HD TileWalk walk_begin(const RingGeom& g, int i, int64_t a_hi, int TK, int s_begin, int s_end,
                          int anchor = -1) {
  TileWalk w;
  w.s = s_begin; w.s_end = s_end; w.i = i; w.P = g.P; w.kb = 0; w.j = 0; w.nkb = 0; w.rev = 0;
  w.anchor = anchor < 0 ? i : anchor;
  walk_skip_empty(g, w, a_hi, TK);
  return w;
}

// The same walk over the backward ring (RingAttention deep-architecture article,
// techknowgenie, section "activation checkpointing and memory recomputation": KV
// blocks travel the ring in the opposite direction), so query shard i meets KV
// shard (i + s) mod P at step s (counted from `anchor` instead of i when given).
RA_HD TileWalk walk_begin_rev(const RingGeom& g, int i, int64_t a_hi, int TK, int anchor = -1, int s_begin = 0,
                              int s_end = -1) {
  TileWalk w;
  w.s = s_begin; w.s_end = s_end < 0 ? g.P : s_end; w.i = i; w.P = g.P; w.kb = 0; w.j = 0; w.nkb = 0; w.rev = 1;
  w.anchor = anchor < 0 ? i : anchor;
  walk_skip_empty(g, w, a_hi, TK);
  return w;
}

RA_HD bool walk_valid(const TileWalk& w) { return w.s < w.s_end; }

RA_HD void walk_next(const RingGeom& g, TileWalk& w, int64_t a_hi, int TK) {
  if (++w.kb < w.nkb) return;
  w.kb = 0;
  ++w.s;
  walk_skip_empty(g, w, a_hi, TK);
}

// ---------------------------------------------------------------- backward, K/V side
// The dK/dV pass gives each CTA one KV tile (b, kv head g, KV shard j, tile kt of
// TK keys) and lets it meet every query tile that can see it, the way a KV block
// meets the query shards as it travels the backward ring: at step s it sits with
// query shard (j - s) mod P. Inside a shard, query rows see a key exactly when
// their token is not below the key's (causal), and tokens rise with the local index.

// First local row of shard i whose token is >= u (Sq if none): binary search on the
// monotone token map.
RA_HD int64_t first_row_at_or_after(const RingGeom& g, int i, int64_t u) {
  int64_t lo = 0, hi = g.Sq;
  while (lo < hi) {
    const int64_t mid = (lo + hi) / 2;
    if (token_of(g, i, mid) >= u) hi = mid; else lo = mid + 1;
  }
  return lo;
}

struct KvUnit {
  int b, g, j, kt;
};

RA_HD int64_t num_kv_tiles(const RingGeom& g, int TK) { return (g.Sq + TK - 1) / TK; }

RA_HD int64_t num_kv_units(const RingGeom& g, int TK) { return (int64_t)g.B * g.Hkv * g.P * num_kv_tiles(g, TK); }

// A KV tile's work grows as its first token falls. Contiguous causal: shard j,
// then tile (the earliest tiles of the sequence first, longest first); zigzag
// causal with whole tiles per chunk: chunk 0..2P-1, then tile (longest first);
// otherwise, for long sequences (grouped_order): shard j, then tile ascending, so
// the concurrently running tiles of one shard walk the same ring sequence of query
// shards and share Q and dO through L2; for shorter ones: tile, then shard (longest
// first). (b, kv head) is innermost.
RA_HD KvUnit decode_kv_unit(const RingGeom& g, int TK, int64_t u) {
  const int64_t nkt = num_kv_tiles(g, TK);
  const int64_t bg_n = (int64_t)g.B * g.Hkv;
  const int64_t pos = u / bg_n;
  const int64_t bg = u % bg_n;
  KvUnit r;
  r.b = (int)(bg / g.Hkv);
  r.g = (int)(bg % g.Hkv);
  if (g.causal && g.layout == kContiguous) {
    r.j = (int)(pos / nkt);
    r.kt = (int)(pos % nkt);
  } else if (g.causal && g.layout == kZigzag && (g.Sq / 2) % TK == 0) {
    const int64_t tpc = nkt / 2;  // tiles per chunk
    const int c = (int)(pos / tpc);
    r.j = c < g.P ? c : 2 * g.P - 1 - c;
    r.kt = (int)((c < g.P ? 0 : tpc) + pos % tpc);
  } else if (grouped_order(g)) {
    r.j = (int)(pos / nkt);
    r.kt = (int)(pos % nkt);
  } else {
    r.kt = (int)(pos / g.P);
    r.j = (int)(pos % g.P);
  }
  return r;
}

// The KV units of one shard j only (one step of a ring spread over devices: the device
// holds one KV shard): (b, kv head) innermost, tiles in index order (longest first
// under a causal mask).
RA_HD int64_t num_kv_units_shard(const RingGeom& g, int TK) { return (int64_t)g.B * g.Hkv * num_kv_tiles(g, TK); }

RA_HD KvUnit decode_kv_unit_shard(const RingGeom& g, int TK, int64_t u, int j) {
  const int64_t bg_n = (int64_t)g.B * g.Hkv;
  KvUnit r;
  r.kt = (int)(u / bg_n);
  const int64_t bg = u % bg_n;
  r.b = (int)(bg / g.Hkv);
  r.g = (int)(bg % g.Hkv);
  r.j = j;
  return r;
}

// Walk over (query head of the group, ring step, query tile) for one KV tile.
struct QWalk {
  int hr, rep;  // query head hr of the GQA group
  int s, i;     // ring step and the query shard met there
  int qt, nqt;  // current query tile and the shard's tile count
  int qt0;      // first query tile of shard i that sees the KV tile
  int j;
  int64_t u_min;   // smallest key token of the tile
  int s_lo, s_hi;  // the ring steps walked: [0, P), or the one step that meets a single query shard
};

RA_HD void qwalk_skip_empty(const RingGeom& g, QWalk& w, int TQ) {
  while (w.hr < w.rep) {
    while (w.s < w.s_hi) {
      w.i = (w.j - w.s + g.P) % g.P;
      const int64_t a0 = g.causal ? first_row_at_or_after(g, w.i, w.u_min) : 0;
      if (a0 < g.Sq) {
        w.qt0 = (int)(a0 / TQ);
        w.qt = w.qt0;
        return;
      }
      ++w.s;
    }
    w.s = w.s_lo;
    ++w.hr;
  }
}

// q_only >= 0 restricts the walk to the one ring step at which the KV tile meets query
// shard q_only (one step of a ring spread over devices).
RA_HD QWalk qwalk_begin(const RingGeom& g, const KvUnit& U, int TQ, int TK, int q_only = -1) {
  QWalk w;
  w.s_lo = q_only < 0 ? 0 : (U.j - q_only + g.P) % g.P;
  w.s_hi = q_only < 0 ? g.P : w.s_lo + 1;
  w.hr = 0; w.rep = g.Hq / g.Hkv; w.s = w.s_lo; w.i = U.j; w.j = U.j;
  w.nqt = (int)((g.Sq + TQ - 1) / TQ);
  w.qt = 0; w.qt0 = 0;
  w.u_min = token_of(g, U.j, (int64_t)U.kt * TK);
  qwalk_skip_empty(g, w, TQ);
  return w;
}

RA_HD bool qwalk_valid(const QWalk& w) { return w.hr < w.rep; }

RA_HD void qwalk_next(const RingGeom& g, QWalk& w, int TQ) {
  if (++w.qt < w.nqt) return;
  ++w.s;
  qwalk_skip_empty(g, w, TQ);
}

// Causal mask inside one (query tile, KV tile) block of the dK/dV pass: the key of
// token u is visible to the tile's query columns c >= the returned value (query
// rows a0 + c of shard i); 0 when not causal.
RA_HD int bwd_first_visible_col(const RingGeom& g, int i, int64_t a0, int64_t u, int TQ) {
  if (!g.causal) return 0;
  const int64_t c = first_row_at_or_after(g, i, u) - a0;
  return c < 0 ? 0 : (c > TQ ? TQ : (int)c);
}

// Query tiles one KV unit meets: per shard, the tiles from the first that sees the
// KV tile's smallest token to the end, for every query head of the group.
RA_HD int64_t qwalk_count(const RingGeom& g, const KvUnit& U, int TQ, int TK, int q_only = -1) {
  const int64_t nqt = (g.Sq + TQ - 1) / TQ;
  const int64_t u_min = token_of(g, U.j, (int64_t)U.kt * TK);
  int64_t n = 0;
  for (int i = 0; i < g.P; ++i) {
    if (q_only >= 0 && i != q_only) continue;
    const int64_t a0 = g.causal ? first_row_at_or_after(g, i, u_min) : 0;
    if (a0 < g.Sq) n += nqt - a0 / TQ;
  }
  return n * (g.Hq / g.Hkv);
}

}  // namespace ringattn
