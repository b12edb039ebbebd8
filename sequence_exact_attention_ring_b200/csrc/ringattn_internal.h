// Internal declarations shared by the C-ABI layer and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ringattn.h"
#include "ring_schedule.h"

namespace ringattn {

typedef CUresult (*PFN_encodeTiled)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                    const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                    CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// TMA map of a sharded [B, H, S, D] bf16 tensor (box: 64 elements x box_rows tokens).
int encode_shard_map(CUtensorMap* map, const void* base, const RingGeom& g, int heads, int D, int box_rows);
// The same for a single-shard buffer [B, H, Sq, D] in shard-local order when `local`
// (coordinates from tile_coords), else encode_shard_map.
int encode_input_map(CUtensorMap* map, const void* base, const RingGeom& g, bool local, int heads, int D,
                     int box_rows);

// Status word layout at the start of the caller's workspace.
constexpr size_t kWorkspaceHeaderBytes = 256;

// How a forward launch reads its inputs and writes its result.
//   kOutFinal    out in the input dtype [B,Hq,S,D] and lse [B,Hq,S], natural token order
//   kOutPartial  the normalised per-step partial: fp32 [B,Hq,Sq,D] and lse [B,Hq,Sq],
//                shard-local order
//   kOutFold     the step's normalised partial folded into a running state (acc_o fp32
//                [B,Hq,Sq,D], acc_lse [B,Hq,Sq], shard-local order):
//                    lse = ln(e^lse_acc + e^lse_step),
//                    o   = e^(lse_acc - lse) o_acc + e^(lse_step - lse) o_step.
//                `first`: the state starts from this step (acc is only written);
//                `last`: the merged rows go to out (input dtype) and lse instead of acc.
// local: q is one query shard and k, v one KV shard, each a [B, H, Sq, D] buffer in
// shard-local order (as one device of a multi-GPU ring holds them), instead of the
// whole sequence in natural token order.
enum { kOutFinal = 0, kOutPartial = 1, kOutFold = 2 };
struct FwdOut {
  int kind;
  int local;
  int first, last;
  float* acc_o;
  float* acc_lse;
};

// Fused tcgen05 kernel (bf16), single CTAs, D = 64 or 128.
int launch_fwd_sm100(const void* q, const void* k, const void* v, void* out, float* lse, const RingGeom& g,
                     float scale, int s_begin, int s_end, int q_shard_only, const FwdOut& fo, int* status,
                     uint64_t watchdog_ns, cudaStream_t stream);
int64_t fwd_sm100_units(const RingGeom& g, int q_shard_only);

// The same computation on CTA pairs (cta_group::2 MMAs, D = 128 only): each CTA of
// a pair stages half of every K and V tile.
int launch_fwd_sm100_2sm(const void* q, const void* k, const void* v, void* out, float* lse, const RingGeom& g,
                         float scale, int s_begin, int s_end, int q_shard_only, const FwdOut& fo, int* status,
                         uint64_t watchdog_ns, cudaStream_t stream);

// fp32-accumulating SIMT kernel (fp32 or bf16 inputs), same schedule and output modes.
int launch_fwd_simt(const void* q, const void* k, const void* v, void* out, float* lse, const RingGeom& g,
                    float scale, int dtype, int s_begin, int s_end, int q_shard_only, const FwdOut& fo,
                    cudaStream_t stream);

// Backward pass (bf16, D = 128): the Delta / lse prep kernel, then the dK/dV and dQ
// tcgen05 kernels. `stats` holds 2 * B*Hq*P*bwd_sq_pad(g) floats.
int64_t bwd_sq_pad(const RingGeom& g);
int launch_bwd_sm100(const void* q, const void* k, const void* v, const void* out, const float* lse,
                     const void* dout, void* dq, void* dk, void* dv, const RingGeom& g, float scale, float* stats,
                     int* status, uint64_t watchdog_ns, cudaStream_t stream);

// One step of the backward ring spread over devices (bf16, D = 128), on shard-local
// buffers: the statistics of query shard q_index (launch_bwd_ring_prep, into `stats`:
// 2 * bwd_ring_stat_rows(g) floats), then per step the dK/dV part (KV shard kv_index's
// gradients from query shard q_index, folded into dk_acc/dv_acc) and/or the dQ part
// (query shard q_index's gradient from KV shard kv_index, folded into dq_acc); on the
// last step the bf16 results go to dq/dk/dv.
int64_t bwd_ring_stat_rows(const RingGeom& g);
int launch_bwd_ring_prep(const void* out, const float* lse, const void* dout, const RingGeom& g, int q_index,
                         float* stats, cudaStream_t stream);
int launch_bwd_ring_step_sm100(const void* q, const void* dout, const void* k, const void* v, float* dq_acc,
                               float* dk_acc, float* dv_acc, void* dq, void* dk, void* dv, const RingGeom& g,
                               int q_index, int kv_index, float scale, int parts, int first, int last, float* stats,
                               int* status, uint64_t watchdog_ns, cudaStream_t stream);

// Decode (one query row per head against the whole sharded cache, bf16, D = 128):
// split-KV partials into o_parts [decode_parts(g)][B*Hq][D] and lse_parts, then the
// merge kernel writes out [B*Hq][D] bf16 and lse [B*Hq].
int64_t decode_parts(const RingGeom& g);
int launch_decode_sm100(const void* q, const void* k, const void* v, void* out, float* lse, const RingGeom& g,
                        float scale, float* o_parts, float* lse_parts, int* status, uint64_t watchdog_ns,
                        cudaStream_t stream);

// CUDA-core backward for the shapes the tensor-core kernels do not take (fp32 or
// bf16, D = 64 or 128, any layout); same statistics layout in `stats`.
int launch_bwd_simt(const void* q, const void* k, const void* v, const void* out, const float* lse, const void* dout,
                    void* dq, void* dk, void* dv, const RingGeom& g, float scale, int dtype, float* stats,
                    cudaStream_t stream);

int launch_merge(const float* o_parts, const float* lse_parts, int n_parts, int64_t rows, int D, void* out,
                 float* lse_out, int out_dtype, cudaStream_t stream);

int launch_watchdog_probe(int timeout_us, int* status, cudaStream_t stream);
int launch_exp2_probe(const float* x, float* y, int64_t n, cudaStream_t stream);

}  // namespace ringattn
