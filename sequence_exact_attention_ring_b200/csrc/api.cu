// C ABI of libringattn.so: argument validation, dispatch, status word, test hooks.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "ringattn.h"
#include "ring_schedule.h"
#include "ringattn_internal.h"
#include "sm100_ptx.cuh"

using namespace ringattn;

namespace {

constexpr int kVersion = 100;  // 0.1.0

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_geom(int B, int Hq, int Hkv, int64_t S, int D, int P, int causal, int layout, int dtype, RingGeom* g) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || S <= 0 || D <= 0 || P <= 0) return RING_ATTN_EINVAL;
  if (S % P != 0 || Hq % Hkv != 0) return RING_ATTN_EINVAL;
  if (causal != 0 && causal != 1) return RING_ATTN_EINVAL;
  if (layout != RING_ATTN_LAYOUT_CONTIGUOUS && layout != RING_ATTN_LAYOUT_STRIPED &&
      layout != RING_ATTN_LAYOUT_ZIGZAG)
    return RING_ATTN_EINVAL;
  if (layout == RING_ATTN_LAYOUT_ZIGZAG && S % (2 * (int64_t)P) != 0) return RING_ATTN_EINVAL;
  if (dtype != RING_ATTN_DTYPE_FP32 && dtype != RING_ATTN_DTYPE_BF16) return RING_ATTN_EINVAL;
  if ((int64_t)B * Hq > (1 << 24) || S > ((int64_t)1 << 31)) return RING_ATTN_EINVAL;
  if (D != 64 && D != 128) return RING_ATTN_EUNSUPPORTED;
  g->B = B;
  g->Hq = Hq;
  g->Hkv = Hkv;
  g->S = S;
  g->D = D;
  g->P = P;
  g->causal = causal;
  g->layout = layout;
  g->Sq = S / P;
  return RING_ATTN_OK;
}

// sm_100 family check for the tensor-core path, cached per device ordinal.
bool device_is_sm100() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  static int cache[64];  // 0 unknown, 1 yes, 2 no
  if (dev < 0 || dev >= 64) return false;
  if (cache[dev] == 0) {
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    cache[dev] = (major == 10 && minor == 0) ? 1 : 2;
  }
  return cache[dev] == 1;
}

uint64_t watchdog_ns() {
  static uint64_t ns = 0;
  if (ns == 0) {
    uint64_t ms = 2000;
    const char* e = getenv("RING_ATTN_WATCHDOG_MS");
    if (e && atoi(e) > 0) ms = (uint64_t)atoi(e);
    ns = ms * 1000000ull;
  }
  return ns;
}

// The tensor-core kernels load 128-row tiles with TMA; under zigzag a tile must not
// cross from a shard's first chunk into its second, so chunks are whole tiles.
bool tcgen05_layout_ok(const RingGeom& g) { return g.layout != kZigzag || (g.Sq / 2) % 128 == 0; }

int resolve_algo(int algo, int dtype, const RingGeom& g) {
  if (algo == RING_ATTN_ALGO_AUTO)
    return dtype == RING_ATTN_DTYPE_BF16 && tcgen05_layout_ok(g) ? RING_ATTN_ALGO_TCGEN05 : RING_ATTN_ALGO_SIMT;
  return algo;
}

int check_algo(int algo, int dtype, const RingGeom& g) {
  if (algo != RING_ATTN_ALGO_SIMT && algo != RING_ATTN_ALGO_TCGEN05 && algo != RING_ATTN_ALGO_TCGEN05_1SM)
    return RING_ATTN_EINVAL;
  if (algo != RING_ATTN_ALGO_SIMT && (dtype != RING_ATTN_DTYPE_BF16 || !tcgen05_layout_ok(g) || !device_is_sm100()))
    return RING_ATTN_EUNSUPPORTED;
  return RING_ATTN_OK;
}

int reset_status(void* workspace, cudaStream_t stream) {
  return cudaMemsetAsync(workspace, 0, sizeof(int), stream) == cudaSuccess ? RING_ATTN_OK : RING_ATTN_ECUDA;
}

// Launch one ring-attention pass for the given ring-step range and output mode.
int run_fwd(const void* q, const void* k, const void* v, void* out, float* lse, const RingGeom& g, float scale,
            int dtype, int algo, int s_begin, int s_end, int q_shard_only, const FwdOut& fo, void* workspace,
            cudaStream_t stream) {
  int rc = reset_status(workspace, stream);
  if (rc) return rc;
  if (algo == RING_ATTN_ALGO_TCGEN05 && g.D == 128)
    return launch_fwd_sm100_2sm(q, k, v, out, lse, g, scale, s_begin, s_end, q_shard_only, fo,
                                static_cast<int*>(workspace), watchdog_ns(), stream);
  if (algo == RING_ATTN_ALGO_TCGEN05 || algo == RING_ATTN_ALGO_TCGEN05_1SM)
    return launch_fwd_sm100(q, k, v, out, lse, g, scale, s_begin, s_end, q_shard_only, fo,
                            static_cast<int*>(workspace), watchdog_ns(), stream);
  return launch_fwd_simt(q, k, v, out, lse, g, scale, dtype, s_begin, s_end, q_shard_only, fo, stream);
}

FwdOut out_mode(int kind) {
  FwdOut fo;
  fo.kind = kind;
  fo.local = 0;
  fo.first = 0;
  fo.last = 0;
  fo.acc_o = nullptr;
  fo.acc_lse = nullptr;
  return fo;
}

}  // namespace

extern "C" {

int ring_attn_version(void) { return kVersion; }

const char* ring_attn_strerror(int code) {
  switch (code) {
    case RING_ATTN_OK: return "success";
    case RING_ATTN_EINVAL: return "invalid argument";
    case RING_ATTN_EALIGN: return "pointer not 16-byte aligned";
    case RING_ATTN_EUNSUPPORTED: return "unsupported configuration (head dim, dtype or device)";
    case RING_ATTN_EWORKSPACE: return "workspace missing or too small";
    case RING_ATTN_ECUDA: return "CUDA call failed";
    case RING_ATTN_ETIMEOUT: return "device wait exceeded its watchdog limit";
    default: return "unknown error";
  }
}

size_t ring_attn_fwd_workspace_bytes(int B, int Hq, int Hkv, int64_t S, int D, int P, int causal, int layout,
                                     int dtype) {
  RingGeom g;
  if (check_geom(B, Hq, Hkv, S, D, P, causal, layout, dtype, &g) != RING_ATTN_OK) return 0;
  return kWorkspaceHeaderBytes;
}

int ring_attn_fwd_algo(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq, int Hkv,
                       int64_t S, int D, int P, int causal, int layout, float scale, int dtype, void* workspace,
                       size_t workspace_bytes, void* stream, int algo) {
  RingGeom g;
  int rc = check_geom(B, Hq, Hkv, S, D, P, causal, layout, dtype, &g);
  if (rc) return rc;
  if (!q || !k || !v || !out || !lse) return RING_ATTN_EINVAL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse))
    return RING_ATTN_EALIGN;
  if (!workspace || workspace_bytes < kWorkspaceHeaderBytes || !aligned16(workspace)) return RING_ATTN_EWORKSPACE;
  if (!(scale > 0.f) || !isfinite(scale)) return RING_ATTN_EINVAL;
  algo = resolve_algo(algo, dtype, g);
  if ((rc = check_algo(algo, dtype, g))) return rc;
  return run_fwd(q, k, v, out, lse, g, scale, dtype, algo, 0, P, -1, out_mode(kOutFinal), workspace,
                 static_cast<cudaStream_t>(stream));
}

int ring_attn_fwd(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq, int Hkv,
                  int64_t S, int D, int P, int causal, int layout, float scale, int dtype, void* workspace,
                  size_t workspace_bytes, void* stream) {
  return ring_attn_fwd_algo(q, k, v, out, lse, B, Hq, Hkv, S, D, P, causal, layout, scale, dtype, workspace,
                            workspace_bytes, stream, RING_ATTN_ALGO_AUTO);
}

int ring_attn_fwd_step(const void* q, const void* k, const void* v, float* o_part, float* lse_part, int B, int Hq,
                       int Hkv, int64_t S, int D, int P, int q_shard, int kv_shard, int causal, int layout,
                       float scale, int dtype, int algo, void* workspace, size_t workspace_bytes, void* stream) {
  RingGeom g;
  int rc = check_geom(B, Hq, Hkv, S, D, P, causal, layout, dtype, &g);
  if (rc) return rc;
  if (q_shard < 0 || q_shard >= P || kv_shard < 0 || kv_shard >= P) return RING_ATTN_EINVAL;
  if (!q || !k || !v || !o_part || !lse_part) return RING_ATTN_EINVAL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o_part) || !aligned16(lse_part))
    return RING_ATTN_EALIGN;
  if (!workspace || workspace_bytes < kWorkspaceHeaderBytes || !aligned16(workspace)) return RING_ATTN_EWORKSPACE;
  if (!(scale > 0.f) || !isfinite(scale)) return RING_ATTN_EINVAL;
  algo = resolve_algo(algo, dtype, g);
  if ((rc = check_algo(algo, dtype, g))) return rc;
  const int s = ring_step_of(q_shard, kv_shard, P);
  return run_fwd(q, k, v, o_part, lse_part, g, scale, dtype, algo, s, s + 1, q_shard, out_mode(kOutPartial), workspace,
                 static_cast<cudaStream_t>(stream));
}

int ring_attn_fwd_ring_step(const void* q_shard, const void* k_shard, const void* v_shard, float* o_acc,
                            float* lse_acc, void* out, float* lse_out, int B, int Hq, int Hkv, int64_t S, int D,
                            int P, int q_index, int kv_index, int causal, int layout, float scale, int dtype,
                            int flags, void* workspace, size_t workspace_bytes, void* stream) {
  RingGeom g;
  int rc = check_geom(B, Hq, Hkv, S, D, P, causal, layout, dtype, &g);
  if (rc) return rc;
  if (q_index < 0 || q_index >= P || kv_index < 0 || kv_index >= P) return RING_ATTN_EINVAL;
  if (flags & ~(RING_ATTN_STEP_FIRST | RING_ATTN_STEP_LAST)) return RING_ATTN_EINVAL;
  const bool first = (flags & RING_ATTN_STEP_FIRST) != 0;
  const bool last = (flags & RING_ATTN_STEP_LAST) != 0;
  const bool need_acc = !(first && last);
  if (!q_shard || !k_shard || !v_shard) return RING_ATTN_EINVAL;
  if (need_acc && (!o_acc || !lse_acc)) return RING_ATTN_EINVAL;
  if (last && (!out || !lse_out)) return RING_ATTN_EINVAL;
  if (!aligned16(q_shard) || !aligned16(k_shard) || !aligned16(v_shard)) return RING_ATTN_EALIGN;
  if (need_acc && (!aligned16(o_acc) || !aligned16(lse_acc))) return RING_ATTN_EALIGN;
  if (last && (!aligned16(out) || !aligned16(lse_out))) return RING_ATTN_EALIGN;
  if (!workspace || workspace_bytes < kWorkspaceHeaderBytes || !aligned16(workspace)) return RING_ATTN_EWORKSPACE;
  if (!(scale > 0.f) || !isfinite(scale)) return RING_ATTN_EINVAL;
  // shard-local buffers carry no chunk boundary inside a tile, so every layout tiles
  int algo = dtype == RING_ATTN_DTYPE_BF16 ? RING_ATTN_ALGO_TCGEN05 : RING_ATTN_ALGO_SIMT;
  if (algo == RING_ATTN_ALGO_TCGEN05 && !device_is_sm100()) return RING_ATTN_EUNSUPPORTED;
  // a block no query row can see (contiguous causal, kv_index > q_index) adds nothing;
  // only a first or last step still has the state to initialise or to write out
  if (key_limit(g, q_index, kv_index, g.Sq - 1) == 0 && !first && !last) return RING_ATTN_OK;
  FwdOut fo = out_mode(kOutFold);
  fo.local = 1;
  fo.first = first;
  fo.last = last;
  fo.acc_o = o_acc;
  fo.acc_lse = lse_acc;
  const int s = ring_step_of(q_index, kv_index, P);
  return run_fwd(q_shard, k_shard, v_shard, out, lse_out, g, scale, dtype, algo, s, s + 1, q_index, fo, workspace,
                 static_cast<cudaStream_t>(stream));
}

int ring_attn_merge(const float* o_parts, const float* lse_parts, int n_parts, int64_t rows, int D, void* out,
                    float* lse_out, int out_dtype, void* stream) {
  if (!o_parts || !lse_parts || !out || !lse_out) return RING_ATTN_EINVAL;
  if (n_parts < 1 || n_parts > 1024 || rows < 0 || D <= 0 || D % 8 != 0 || D > 256) return RING_ATTN_EINVAL;
  if (out_dtype != RING_ATTN_DTYPE_FP32 && out_dtype != RING_ATTN_DTYPE_BF16) return RING_ATTN_EINVAL;
  if (!aligned16(o_parts) || !aligned16(out) || !aligned16(lse_parts) || !aligned16(lse_out)) return RING_ATTN_EALIGN;
  return launch_merge(o_parts, lse_parts, n_parts, rows, D, out, lse_out, out_dtype,
                      static_cast<cudaStream_t>(stream));
}

size_t ring_attn_bwd_workspace_bytes(int B, int Hq, int Hkv, int64_t S, int D, int P, int causal, int layout,
                                     int dtype) {
  RingGeom g;
  if (check_geom(B, Hq, Hkv, S, D, P, causal, layout, dtype, &g) != RING_ATTN_OK) return 0;
  return kWorkspaceHeaderBytes + 2 * sizeof(float) * (size_t)B * Hq * P * (size_t)bwd_sq_pad(g);
}

int ring_attn_bwd(const void* q, const void* k, const void* v, const void* out, const float* lse, const void* dout,
                  void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int64_t S, int D, int P, int causal,
                  int layout, float scale, int dtype, void* workspace, size_t workspace_bytes, void* stream) {
  RingGeom g;
  int rc = check_geom(B, Hq, Hkv, S, D, P, causal, layout, dtype, &g);
  if (rc) return rc;
  if (!q || !k || !v || !out || !lse || !dout || !dq || !dk || !dv) return RING_ATTN_EINVAL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse) || !aligned16(dout) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return RING_ATTN_EALIGN;
  const size_t need = ring_attn_bwd_workspace_bytes(B, Hq, Hkv, S, D, P, causal, layout, dtype);
  if (!workspace || workspace_bytes < need || !aligned16(workspace)) return RING_ATTN_EWORKSPACE;
  if (!(scale > 0.f) || !isfinite(scale)) return RING_ATTN_EINVAL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((rc = reset_status(workspace, st))) return rc;
  float* stats = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kWorkspaceHeaderBytes);
  // bf16 with D = 128 runs on the tensor-core kernels; every other shape (fp32, D = 64,
  // zigzag chunks that are not whole 128-row tiles) on the CUDA-core kernels
  if (dtype == RING_ATTN_DTYPE_BF16 && D == 128 && tcgen05_layout_ok(g) && device_is_sm100())
    return launch_bwd_sm100(q, k, v, out, lse, dout, dq, dk, dv, g, scale, stats, static_cast<int*>(workspace),
                            watchdog_ns(), st);
  return launch_bwd_simt(q, k, v, out, lse, dout, dq, dk, dv, g, scale, dtype, stats, st);
}

size_t ring_attn_bwd_ring_workspace_bytes(int B, int Hq, int Hkv, int64_t S, int D, int P, int causal, int layout,
                                          int dtype) {
  RingGeom g;
  if (check_geom(B, Hq, Hkv, S, D, P, causal, layout, dtype, &g) != RING_ATTN_OK) return 0;
  return kWorkspaceHeaderBytes + 2 * sizeof(float) * (size_t)bwd_ring_stat_rows(g);
}

namespace {
int check_bwd_ring(int B, int Hq, int Hkv, int64_t S, int D, int P, int q_index, int causal, int layout, int dtype,
                   void* workspace, size_t workspace_bytes, RingGeom* g) {
  int rc = check_geom(B, Hq, Hkv, S, D, P, causal, layout, dtype, g);
  if (rc) return rc;
  if (q_index < 0 || q_index >= P) return RING_ATTN_EINVAL;
  const size_t need = ring_attn_bwd_ring_workspace_bytes(B, Hq, Hkv, S, D, P, causal, layout, dtype);
  if (!workspace || workspace_bytes < need || !aligned16(workspace)) return RING_ATTN_EWORKSPACE;
  if (dtype != RING_ATTN_DTYPE_BF16 || D != 128 || !device_is_sm100()) return RING_ATTN_EUNSUPPORTED;
  return RING_ATTN_OK;
}
}  // namespace

int ring_attn_bwd_ring_prep(const void* out_shard, const float* lse_shard, const void* dout_shard, int B, int Hq,
                            int Hkv, int64_t S, int D, int P, int q_index, int causal, int layout, int dtype,
                            void* workspace, size_t workspace_bytes, void* stream) {
  if (!out_shard || !lse_shard || !dout_shard) return RING_ATTN_EINVAL;
  RingGeom g;
  int rc = check_bwd_ring(B, Hq, Hkv, S, D, P, q_index, causal, layout, dtype, workspace, workspace_bytes, &g);
  if (rc) return rc;
  if (!aligned16(out_shard) || !aligned16(lse_shard) || !aligned16(dout_shard)) return RING_ATTN_EALIGN;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((rc = reset_status(workspace, st))) return rc;
  float* stats = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kWorkspaceHeaderBytes);
  return launch_bwd_ring_prep(out_shard, lse_shard, dout_shard, g, q_index, stats, st);
}

int ring_attn_bwd_ring_step(const void* q_shard, const void* dout_shard, const void* k_shard, const void* v_shard,
                            float* dq_acc, float* dk_acc, float* dv_acc, void* dq, void* dk, void* dv, int B, int Hq,
                            int Hkv, int64_t S, int D, int P, int q_index, int kv_index, int causal, int layout,
                            float scale, int dtype, int parts, int flags, void* workspace, size_t workspace_bytes,
                            void* stream) {
  RingGeom g;
  int rc = check_geom(B, Hq, Hkv, S, D, P, causal, layout, dtype, &g);
  if (rc) return rc;
  if (kv_index < 0 || kv_index >= P) return RING_ATTN_EINVAL;
  if (parts < 1 || parts > (RING_ATTN_BWD_PART_KV | RING_ATTN_BWD_PART_Q)) return RING_ATTN_EINVAL;
  if (flags & ~(RING_ATTN_STEP_FIRST | RING_ATTN_STEP_LAST)) return RING_ATTN_EINVAL;
  const bool first = (flags & RING_ATTN_STEP_FIRST) != 0;
  const bool last = (flags & RING_ATTN_STEP_LAST) != 0;
  const bool need_acc = !(first && last);
  const bool kv = (parts & RING_ATTN_BWD_PART_KV) != 0;
  const bool qp = (parts & RING_ATTN_BWD_PART_Q) != 0;
  if (!q_shard || !dout_shard || !k_shard || !v_shard) return RING_ATTN_EINVAL;
  if (kv && ((need_acc && (!dk_acc || !dv_acc)) || (last && (!dk || !dv)))) return RING_ATTN_EINVAL;
  if (qp && ((need_acc && !dq_acc) || (last && !dq))) return RING_ATTN_EINVAL;
  if (!aligned16(q_shard) || !aligned16(dout_shard) || !aligned16(k_shard) || !aligned16(v_shard))
    return RING_ATTN_EALIGN;
  if ((dk_acc && !aligned16(dk_acc)) || (dv_acc && !aligned16(dv_acc)) || (dq_acc && !aligned16(dq_acc)) ||
      (dq && !aligned16(dq)) || (dk && !aligned16(dk)) || (dv && !aligned16(dv)))
    return RING_ATTN_EALIGN;
  if (!(scale > 0.f) || !isfinite(scale)) return RING_ATTN_EINVAL;
  if ((rc = check_bwd_ring(B, Hq, Hkv, S, D, P, q_index, causal, layout, dtype, workspace, workspace_bytes, &g)))
    return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((rc = reset_status(workspace, st))) return rc;
  float* stats = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kWorkspaceHeaderBytes);
  return launch_bwd_ring_step_sm100(q_shard, dout_shard, k_shard, v_shard, dq_acc, dk_acc, dv_acc, dq, dk, dv, g,
                                    q_index, kv_index, scale, parts, first, last, stats, static_cast<int*>(workspace),
                                    watchdog_ns(), st);
}

size_t ring_attn_decode_workspace_bytes(int B, int Hq, int Hkv, int64_t S, int D, int P, int layout, int dtype) {
  RingGeom g;
  if (check_geom(B, Hq, Hkv, S, D, P, 0, layout, dtype, &g) != RING_ATTN_OK) return 0;
  const size_t rows = (size_t)B * Hq;
  return kWorkspaceHeaderBytes + sizeof(float) * (size_t)decode_parts(g) * rows * (size_t)(D + 1);
}

int ring_attn_decode(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq, int Hkv,
                     int64_t S, int D, int P, int layout, float scale, int dtype, void* workspace,
                     size_t workspace_bytes, void* stream) {
  RingGeom g;
  int rc = check_geom(B, Hq, Hkv, S, D, P, 0, layout, dtype, &g);
  if (rc) return rc;
  if (!q || !k || !v || !out || !lse) return RING_ATTN_EINVAL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse)) return RING_ATTN_EALIGN;
  const size_t need = ring_attn_decode_workspace_bytes(B, Hq, Hkv, S, D, P, layout, dtype);
  if (!workspace || workspace_bytes < need || !aligned16(workspace)) return RING_ATTN_EWORKSPACE;
  if (!(scale > 0.f) || !isfinite(scale)) return RING_ATTN_EINVAL;
  if (dtype != RING_ATTN_DTYPE_BF16 || D != 128 || Hq / Hkv > 32 || !tcgen05_layout_ok(g) || !device_is_sm100())
    return RING_ATTN_EUNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((rc = reset_status(workspace, st))) return rc;
  float* o_parts = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kWorkspaceHeaderBytes);
  float* lse_parts = o_parts + (size_t)decode_parts(g) * B * Hq * D;
  return launch_decode_sm100(q, k, v, out, lse, g, scale, o_parts, lse_parts, static_cast<int*>(workspace),
                             watchdog_ns(), st);
}

int ring_attn_status(const void* workspace, void* stream) {
  if (!workspace) return RING_ATTN_EINVAL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return RING_ATTN_ECUDA;
  int status = 0;
  if (cudaMemcpy(&status, workspace, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return RING_ATTN_ECUDA;
  return status;
}

int64_t ring_attn_debug_bwd_visit_counts(int64_t S, int P, int causal, int layout, int pass, int32_t* counts) {
  RingGeom g;
  int rc = check_geom(1, 1, 1, S, 128, P, causal, layout, RING_ATTN_DTYPE_BF16, &g);
  if (rc) return rc;
  if (!counts || S > 4096 || (pass != 0 && pass != 1)) return RING_ATTN_EINVAL;
  const int T = 128;   // stationary tile rows (keys of the dK/dV pass, queries of the dQ pass)
  const int TS = 64;   // rows of a streamed step
  int64_t visits = 0;
  if (pass == 0) {
    // dK/dV pass: every KV unit, every query step it meets, the kernel's column rule
    for (int64_t uu = 0; uu < num_kv_units(g, T); ++uu) {
      const KvUnit U = decode_kv_unit(g, T, uu);
      for (QWalk w = qwalk_begin(g, U, TS, T); qwalk_valid(w); qwalk_next(g, w, TS)) {
        ++visits;
        for (int r = 0; r < T; ++r) {
          const int64_t b = (int64_t)U.kt * T + r;
          if (b >= g.Sq) continue;
          const int64_t u = token_of(g, U.j, b);
          const int cmin = bwd_first_visible_col(g, w.i, (int64_t)w.qt * TS, u, TS);
          for (int c = cmin; c < TS; ++c) {
            const int64_t a = (int64_t)w.qt * TS + c;
            if (a < g.Sq) counts[token_of(g, w.i, a) * S + u] += 1;
          }
        }
      }
    }
  } else {
    // dQ pass: every query unit, its backward-ring walk in key steps, the key limit per row
    for (int64_t uu = 0; uu < num_units(g, T, -1); ++uu) {
      const Unit U = decode_unit(g, T, -1, uu);
      const int64_t a0 = (int64_t)U.tb * T;
      const int64_t a_hi = (a0 + T - 1 < g.Sq - 1) ? a0 + T - 1 : g.Sq - 1;
      for (TileWalk w = walk_begin_rev(g, U.i, a_hi, TS, launch_anchor(g, -1)); walk_valid(w);
           walk_next(g, w, a_hi, TS)) {
        ++visits;
        for (int r = 0; r < T && a0 + r < g.Sq; ++r) {
          const int64_t a = a0 + r;
          const int64_t lim = key_limit(g, U.i, w.j, a);
          for (int c = 0; c < TS; ++c) {
            const int64_t b = (int64_t)w.kb * TS + c;
            if (b < lim) counts[token_of(g, U.i, a) * S + token_of(g, w.j, b)] += 1;
          }
        }
      }
    }
  }
  return visits;
}

int64_t ring_attn_debug_visit_counts(int64_t S, int P, int causal, int layout, int tile_q, int tile_k,
                                     int32_t* counts) {
  RingGeom g;
  int rc = check_geom(1, 1, 1, S, 64, P, causal, layout, RING_ATTN_DTYPE_BF16, &g);
  if (rc) return rc;
  if (!counts || tile_q <= 0 || tile_k <= 0 || S > 4096) return RING_ATTN_EINVAL;
  int64_t tiles = 0;
  const int64_t units = num_units(g, tile_q, -1);
  for (int64_t u = 0; u < units; ++u) {
    const Unit U = decode_unit(g, tile_q, -1, u);
    const int64_t a0 = (int64_t)U.tb * tile_q;
    const int64_t a_hi = (a0 + tile_q - 1 < g.Sq - 1) ? a0 + tile_q - 1 : g.Sq - 1;
    for (TileWalk w = walk_begin(g, U.i, a_hi, tile_k, 0, P, launch_anchor(g, -1)); walk_valid(w);
         walk_next(g, w, a_hi, tile_k)) {
      ++tiles;
      for (int64_t a = a0; a < a0 + tile_q && a < g.Sq; ++a) {
        const int64_t lim = key_limit(g, U.i, w.j, a);
        for (int c = 0; c < tile_k; ++c) {
          const int64_t b = (int64_t)w.kb * tile_k + c;
          if (b < lim) counts[token_of(g, U.i, a) * S + token_of(g, w.j, b)] += 1;
        }
      }
    }
  }
  return tiles;
}

int ring_attn_debug_decode_units(int B, int Hq, int Hkv, int64_t S, int P, int causal, int layout, int tile_q,
                                 int32_t* units_out, int64_t max_units) {
  RingGeom g;
  int rc = check_geom(B, Hq, Hkv, S, 64, P, causal, layout, RING_ATTN_DTYPE_BF16, &g);
  if (rc) return rc;
  if (tile_q <= 0) return RING_ATTN_EINVAL;
  const int64_t n = num_units(g, tile_q, -1);
  if (!units_out || n > max_units) return RING_ATTN_EINVAL;
  for (int64_t u = 0; u < n; ++u) {
    const Unit U = decode_unit(g, tile_q, -1, u);
    const int64_t a0 = (int64_t)U.tb * tile_q;
    const int64_t a_hi = (a0 + tile_q - 1 < g.Sq - 1) ? a0 + tile_q - 1 : g.Sq - 1;
    units_out[5 * u + 0] = U.b;
    units_out[5 * u + 1] = U.h;
    units_out[5 * u + 2] = U.i;
    units_out[5 * u + 3] = U.tb;
    units_out[5 * u + 4] = (int32_t)unit_tile_count(g, U.i, a_hi, 128, 0, P);
  }
  return (int)n;
}

int64_t ring_attn_debug_unit_walk(int B, int Hq, int Hkv, int64_t S, int P, int causal, int layout, int tile_q,
                                  int tile_k, int64_t unit, int32_t* pairs_out, int64_t max_pairs) {
  RingGeom g;
  int rc = check_geom(B, Hq, Hkv, S, 64, P, causal, layout, RING_ATTN_DTYPE_BF16, &g);
  if (rc) return rc;
  if (tile_q <= 0 || tile_k <= 0 || !pairs_out || unit < 0 || unit >= num_units(g, tile_q, -1))
    return RING_ATTN_EINVAL;
  const Unit U = decode_unit(g, tile_q, -1, unit);
  const int64_t a0 = (int64_t)U.tb * tile_q;
  const int64_t a_hi = (a0 + tile_q - 1 < g.Sq - 1) ? a0 + tile_q - 1 : g.Sq - 1;
  int64_t n = 0;
  for (TileWalk w = walk_begin(g, U.i, a_hi, tile_k, 0, P, launch_anchor(g, -1)); walk_valid(w);
       walk_next(g, w, a_hi, tile_k), ++n) {
    if (n >= max_pairs) return RING_ATTN_EINVAL;
    pairs_out[2 * n] = w.j;
    pairs_out[2 * n + 1] = w.kb;
  }
  return n;
}

int ring_attn_debug_schedule_info(int B, int Hq, int Hkv, int64_t S, int D, int P, int causal, int layout,
                                  int64_t* info) {
  RingGeom g;
  int rc = check_geom(B, Hq, Hkv, S, D, P, causal, layout, RING_ATTN_DTYPE_BF16, &g);
  if (rc) return rc;
  if (!info) return RING_ATTN_EINVAL;
  const int BQ = 256, BN = 128;
  const int64_t units = num_units(g, BQ, -1);
  int64_t total = 0, partial = 0, longest = 0, first = 0, last = 0;
  for (int64_t u = 0; u < units; ++u) {
    const Unit U = decode_unit(g, BQ, -1, u);
    const int64_t a0 = (int64_t)U.tb * BQ;
    const int64_t a_hi = (a0 + BQ - 1 < g.Sq - 1) ? a0 + BQ - 1 : g.Sq - 1;
    int64_t n = 0;
    for (TileWalk w = walk_begin(g, U.i, a_hi, BN, 0, P, launch_anchor(g, -1)); walk_valid(w);
         walk_next(g, w, a_hi, BN)) {
      ++n;
      if ((int64_t)w.kb * BN + BN > key_limit(g, U.i, w.j, a0)) ++partial;
    }
    total += n;
    if (n > longest) longest = n;
    if (u == 0) first = n;
    last = n;
  }
  info[0] = units;
  info[1] = total;
  info[2] = partial;
  info[3] = longest;
  info[4] = first;
  info[5] = last;
  return RING_ATTN_OK;
}

int ring_attn_debug_exp2(const float* x, float* y, int64_t n, void* stream) {
  if (!x || !y || n < 0 || (n & 1)) return RING_ATTN_EINVAL;
  if (!aligned16(x) || !aligned16(y)) return RING_ATTN_EALIGN;
  return launch_exp2_probe(x, y, n, static_cast<cudaStream_t>(stream));
}

int ring_attn_debug_watchdog(int timeout_us, void* workspace, size_t workspace_bytes, void* stream) {
  if (timeout_us <= 0 || timeout_us > 10000000) return RING_ATTN_EINVAL;
  if (!workspace || workspace_bytes < kWorkspaceHeaderBytes) return RING_ATTN_EWORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int rc = reset_status(workspace, s);
  if (rc) return rc;
  return launch_watchdog_probe(timeout_us, static_cast<int*>(workspace), s);
}

}  // extern "C"

// ---------------------------------------------------------------- watchdog probe
namespace ringattn {

__global__ void watchdog_probe_kernel(int* status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbarrier_init();
  }
  __syncthreads();
  const Watchdog wd{&abort_flag, status, limit_ns};
  // nobody arrives on `bar`: the bounded wait must give up and report
  (void)mbar_wait(&bar, 0, wd);
  __syncthreads();
}

__global__ void exp2_probe_kernel(const float* __restrict__ x, float* __restrict__ y, int64_t n) {
  for (int64_t i = 2 * ((int64_t)blockIdx.x * blockDim.x + threadIdx.x); i < n;
       i += 2 * (int64_t)gridDim.x * blockDim.x) {
    const uint64_t r = exp2_poly2(f2_pack(__float_as_uint(x[i]), __float_as_uint(x[i + 1])));
    float a, b;
    f2_unpack(r, a, b);
    y[i] = a;
    y[i + 1] = b;
  }
}

int launch_exp2_probe(const float* x, float* y, int64_t n, cudaStream_t stream) {
  if (n == 0) return RING_ATTN_OK;
  exp2_probe_kernel<<<148, 256, 0, stream>>>(x, y, n);
  return cudaGetLastError() == cudaSuccess ? RING_ATTN_OK : RING_ATTN_ECUDA;
}

int launch_watchdog_probe(int timeout_us, int* status, cudaStream_t stream) {
  watchdog_probe_kernel<<<1, 32, 0, stream>>>(status, (uint64_t)timeout_us * 1000ull);
  return cudaGetLastError() == cudaSuccess ? RING_ATTN_OK : RING_ATTN_ECUDA;
}

}  // namespace ringattn
