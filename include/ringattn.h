/*
 * ringattn.h - C ABI of libringattn.so: exact ring attention on one B200 (sm_100a).
 *
 * What is computed. RingAttention (deep-architecture article on techknowgenie,
 * section 3 "rigorous derivation of blockwise online softmax") cuts a sequence of
 * S tokens into P shards of Sq = S/P tokens. Query shard i stays put; at ring step
 * s = 0..P-1 it meets KV shard j = (i - s) mod P (section 2 "core principle";
 * section 5 listing starts from the device's own block). Each block is folded into
 * a running row state (m, l, O) by
 *     S = Q_i K_j^T * scale,  m_new = max(m, rowmax S),  alpha = exp(m - m_new),
 *     P = exp(S - m_new),     l = l*alpha + rowsum P,    O = O*alpha + P V_j,
 * and the result is O / l. This equals ordinary softmax attention exactly (same
 * section), so the output does not depend on P or on the layout; both select the
 * order of the work. Causal masking (section 7 "causal attention with striped
 * attention") lets query token t see keys u <= t (inclusive diagonal). Layout
 * CONTIGUOUS puts tokens [i*Sq, (i+1)*Sq) on shard i; STRIPED puts token t on
 * shard t mod P. ZIGZAG (named as a causal load balancer by the RingAttention
 * newsletter on cmlonder, section "claim and reality", without a definition) is
 * read as: cut the sequence into 2P chunks of C = S/(2P) tokens and give shard i
 * chunks i and 2P-1-i, so every shard folds the same causal work.
 *
 * Tensor layout (all row-major, contiguous, natural token order for every layout):
 *     q, out : [B, Hq,  S, D]      k, v : [B, Hkv, S, D]      lse : [B, Hq, S] fp32
 * Query head h reads KV head h / (Hq/Hkv) (grouped-query attention when Hkv < Hq).
 * lse = m + ln(l): natural log-sum-exp of the scaled scores of each row.
 *
 * Ownership. The caller allocates and frees every buffer (device memory unless
 * stated). The library allocates no device memory and keeps no state between
 * calls. All compute entry points are asynchronous on `stream` (a cudaStream_t
 * passed as void*; NULL = legacy default stream); they return after enqueueing.
 *
 * Errors. Every entry point returns 0 on success or a negative RING_ATTN_E* code.
 * On an argument error nothing is enqueued and no output is touched. A kernel
 * whose internal wait exceeds its watchdog limit stops early, writes
 * RING_ATTN_ETIMEOUT into the status word at the start of the workspace and
 * leaves the outputs undefined; ring_attn_status() reports it.
 */
#ifndef RINGATTN_H_
#define RINGATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define RING_ATTN_OK 0
#define RING_ATTN_EINVAL (-1)       /* null pointer, non-positive size or scale, S % P != 0 (S % 2P != 0 for zigzag), Hq % Hkv != 0, bad enum */
#define RING_ATTN_EALIGN (-2)       /* a tensor pointer is not 16-byte aligned */
#define RING_ATTN_EUNSUPPORTED (-3) /* D not in {64, 128}, or no sm_100 device for the tensor-core path */
#define RING_ATTN_EWORKSPACE (-4)   /* workspace null or smaller than ring_attn_fwd_workspace_bytes() */
#define RING_ATTN_ECUDA (-5)        /* a CUDA runtime/driver call failed (launch, tensor-map encode) */
#define RING_ATTN_ETIMEOUT (-6)     /* a device-side wait hit its watchdog limit */

#define RING_ATTN_LAYOUT_CONTIGUOUS 0
#define RING_ATTN_LAYOUT_STRIPED 1
#define RING_ATTN_LAYOUT_ZIGZAG 2 /* needs S % (2P) == 0; the tensor-core kernels also need (S/(2P)) % 128 == 0 */

#define RING_ATTN_DTYPE_FP32 0
#define RING_ATTN_DTYPE_BF16 1

#define RING_ATTN_ALGO_AUTO 0    /* bf16 -> tensor-core kernel, fp32 -> SIMT kernel */
#define RING_ATTN_ALGO_SIMT 1    /* fp32-accumulating CUDA-core kernel (fp32 or bf16 inputs) */
#define RING_ATTN_ALGO_TCGEN05 2 /* sm_100a tcgen05/TMEM/TMA kernel (bf16 inputs only); D=128 runs on
                                    CTA pairs (cta_group::2), D=64 on single CTAs */
#define RING_ATTN_ALGO_TCGEN05_1SM 3 /* the single-CTA tcgen05 kernel for every D (bf16 inputs only) */

/* Library version (major*10000 + minor*100 + patch). */
int ring_attn_version(void);

/* Text for an error code; never NULL. */
const char* ring_attn_strerror(int code);

/*
 * Bytes of device workspace ring_attn_fwd needs for these arguments (>= 256:
 * the first 4 bytes are the status word). Returns 0 for invalid arguments.
 */
size_t ring_attn_fwd_workspace_bytes(int B, int Hq, int Hkv, int64_t S, int D, int P,
                                     int causal, int layout, int dtype);

/*
 * Exact attention over P ring shards: out = softmax(q k^T * scale, causal mask) v
 * and lse, folding KV shards in ring order for every query shard.
 *   q, k, v   device pointers, dtype `dtype`, shapes above, 16-byte aligned
 *   out       device pointer [B,Hq,S,D] in `dtype` (bf16 rounded to nearest even)
 *   lse       device pointer [B,Hq,S] fp32
 *   S % P == 0, Hq % Hkv == 0, D in {64, 128}; causal 0|1; layout RING_ATTN_LAYOUT_*
 *             (AUTO runs zigzag shapes the tensor-core kernels cannot tile on the SIMT kernel)
 *   scale     score scale, finite and > 0 (the pages use 1/sqrt(D))
 *   workspace device scratch of >= ring_attn_fwd_workspace_bytes() bytes
 * q/k/v must not alias out/lse.
 */
int ring_attn_fwd(const void* q, const void* k, const void* v, void* out, float* lse,
                  int B, int Hq, int Hkv, int64_t S, int D, int P,
                  int causal, int layout, float scale, int dtype,
                  void* workspace, size_t workspace_bytes, void* stream);

/* ring_attn_fwd with an explicit kernel choice (RING_ATTN_ALGO_*). */
int ring_attn_fwd_algo(const void* q, const void* k, const void* v, void* out, float* lse,
                       int B, int Hq, int Hkv, int64_t S, int D, int P,
                       int causal, int layout, float scale, int dtype,
                       void* workspace, size_t workspace_bytes, void* stream, int algo);

/*
 * One literal ring step: query shard i against KV shard j (any 0 <= i, j < P),
 * as device i computes it at ring step (i - j) mod P. Writes the step's
 * normalised partial in the shard's local order:
 *   o_part   device [B, Hq, Sq, D] fp32 = softmax over the block's allowed keys, times V_j
 *   lse_part device [B, Hq, Sq]    fp32, -inf for rows with no allowed key (then o_part row = 0)
 * Merging the P steps of shard i with ring_attn_merge gives rows of ring_attn_fwd.
 * Same argument rules as ring_attn_fwd; uses `workspace` for its status word.
 */
int ring_attn_fwd_step(const void* q, const void* k, const void* v, float* o_part, float* lse_part,
                       int B, int Hq, int Hkv, int64_t S, int D, int P, int q_shard, int kv_shard,
                       int causal, int layout, float scale, int dtype, int algo,
                       void* workspace, size_t workspace_bytes, void* stream);

/*
 * One step of a ring spread over devices, on shard-local buffers, folded into a
 * running state. This is what one device of the pages' ring runs at each step
 * (RingAttention deep-architecture article, techknowgenie, section 2 "core
 * principle": a device keeps its query shard while KV shards pass around the ring;
 * section 5 listing: per step the block is folded into the running (m, l, O), and the
 * output is produced after the last step). The state between steps is kept
 * normalised, (o, lse) with l divided out, and each step's block result is folded in
 * with the section 3 rescale:
 *     lse = ln(e^lse_acc + e^lse_step),  o = e^(lse_acc - lse) o_acc + e^(lse_step - lse) o_step.
 *   q_shard   device [B, Hq,  Sq, D]  query shard q_index, rows in shard-local order
 *   k_shard,  device [B, Hkv, Sq, D]  KV shard kv_index, shard-local order (Sq = S/P)
 *   v_shard
 *   o_acc     device [B, Hq, Sq, D] fp32  running state, shard-local order
 *   lse_acc   device [B, Hq, Sq]    fp32
 *   out       device [B, Hq, Sq, D] in dtype, written only by a LAST step
 *   lse_out   device [B, Hq, Sq]    fp32,     written only by a LAST step
 *   flags     RING_ATTN_STEP_FIRST: the state starts from this step (o_acc/lse_acc
 *             are written, not read). RING_ATTN_STEP_LAST: the merged rows go to
 *             out/lse_out and the state is left as it was. FIRST|LAST: out is this
 *             step alone, and o_acc/lse_acc may be NULL.
 * S, P, layout and causal describe the whole ring (shard map and causal mask on
 * global tokens, as in ring_attn_fwd); q_index/kv_index in [0, P). Every layout
 * runs on the tensor cores here (bf16; fp32 runs on the CUDA-core kernel). A step
 * whose block no query row can see (contiguous causal with kv_index > q_index) and
 * that is neither FIRST nor LAST enqueues nothing. Outputs must not alias inputs
 * or the state. Same argument, workspace and watchdog rules as ring_attn_fwd.
 */
#define RING_ATTN_STEP_FIRST 1
#define RING_ATTN_STEP_LAST 2
int ring_attn_fwd_ring_step(const void* q_shard, const void* k_shard, const void* v_shard,
                            float* o_acc, float* lse_acc, void* out, float* lse_out,
                            int B, int Hq, int Hkv, int64_t S, int D, int P, int q_index, int kv_index,
                            int causal, int layout, float scale, int dtype, int flags,
                            void* workspace, size_t workspace_bytes, void* stream);

/*
 * Combine n normalised partials of the same rows (the online-softmax rescale of
 * section 3 applied to states whose l is already divided out):
 *   lse = lse_max + ln sum_k exp(lse_k - lse_max),  out = sum_k exp(lse_k - lse) * o_k
 *   o_parts   device [n_parts, rows, D] fp32     lse_parts device [n_parts, rows] fp32
 *   out       device [rows, D] in out_dtype      lse_out   device [rows] fp32
 * A part with lse_k = -inf is empty and its o_k is ignored; if all parts are
 * empty the row gets out = 0, lse = -inf. D % 8 == 0, D <= 256. Outputs must
 * not alias inputs. 1 <= n_parts <= 1024.
 */
int ring_attn_merge(const float* o_parts, const float* lse_parts, int n_parts, int64_t rows, int D,
                    void* out, float* lse_out, int out_dtype, void* stream);

/*
 * Bytes of device workspace ring_attn_bwd needs: the 256-byte status header plus two
 * fp32 arrays of B*Hq*P*ceil(S/P / 128)*128 values (per-row statistics in shard order).
 * Returns 0 for invalid arguments.
 */
size_t ring_attn_bwd_workspace_bytes(int B, int Hq, int Hkv, int64_t S, int D, int P,
                                     int causal, int layout, int dtype);

/*
 * Backward pass of ring_attn_fwd (RingAttention deep-architecture article, section
 * "activation checkpointing and memory recomputation": only Q and the row statistics
 * are kept, and K/V travel the ring in the opposite direction while the attention map
 * is recomputed). Given the forward's out and lse and the output gradient dout, it
 * writes the gradients of out with respect to q, k and v:
 *   P = exp(scale q k^T - lse) on the mask,  dv = P^T dout,  dP = dout v^T,
 *   Delta = rowsum(dout * out),  dS = P * (dP - Delta),
 *   dq = scale dS k,  dk = scale dS^T q   (GQA: dk, dv sum over the group's heads).
 *   q, out, dout, dq : device [B,Hq,S,D] in dtype    k, v, dk, dv : device [B,Hkv,S,D] in dtype
 *   lse              : device [B,Hq,S] fp32 as returned by ring_attn_fwd
 *   workspace        : >= ring_attn_bwd_workspace_bytes(); first word is the status word
 * bf16 with D = 128 runs on the tcgen05 kernels (zigzag: when (S/(2P)) % 128 == 0);
 * every other dtype/D/layout the forward accepts runs on fp32 CUDA-core kernels.
 * Outputs must not alias inputs. Same argument and watchdog rules as ring_attn_fwd.
 */
int ring_attn_bwd(const void* q, const void* k, const void* v, const void* out, const float* lse,
                  const void* dout, void* dq, void* dk, void* dv,
                  int B, int Hq, int Hkv, int64_t S, int D, int P,
                  int causal, int layout, float scale, int dtype,
                  void* workspace, size_t workspace_bytes, void* stream);

/*
 * The backward pass as one device of a ring spread over devices runs it (RingAttention
 * deep-architecture article, techknowgenie, section "activation checkpointing and
 * memory recomputation": each device keeps its query shard, dO and the row statistics;
 * the K/V shards travel the ring in the reverse direction, each carrying its dK/dV
 * accumulators, and the attention map is recomputed where they meet). At step s the
 * device holding query shard i holds KV shard j = (i + s) mod P. The gradients are the
 * ones ring_attn_bwd computes; every buffer is one shard in shard-local order:
 *   q_shard, out_shard, dout_shard, dq, dq_acc : [B, Hq,  Sq, D]   (dq_acc fp32, others bf16)
 *   k_shard, v_shard, dk, dv, dk_acc, dv_acc   : [B, Hkv, Sq, D]   (acc fp32, others bf16)
 *   lse_shard                                  : [B, Hq,  Sq] fp32, as ring_attn_fwd_ring_step wrote it
 * ring_attn_bwd_ring_prep computes query shard q_index's row statistics (Delta and lse
 * in base 2) into `workspace`, once per backward pass; every step of that pass then
 * uses the same workspace. ring_attn_bwd_ring_step runs the parts asked for:
 *   RING_ATTN_BWD_PART_KV  KV shard kv_index's dK/dV contributions from query shard
 *                          q_index, folded into dk_acc/dv_acc (they travel with the shard)
 *   RING_ATTN_BWD_PART_Q   query shard q_index's dQ contribution from KV shard kv_index,
 *                          folded into dq_acc
 * (calling the two parts separately lets the dK/dV accumulators leave for the next
 * device while the dQ part runs). flags: RING_ATTN_STEP_FIRST starts the accumulators
 * of the parts run (they are written, not read); RING_ATTN_STEP_LAST writes the summed
 * gradients in bf16 to dq / dk, dv instead. In a ring both hold at the same steps: the
 * shard's journey and the device's steps both start at s = 0 and end at s = P - 1.
 * Supported: bf16, D = 128, an sm_100 device; otherwise RING_ATTN_EUNSUPPORTED.
 */
#define RING_ATTN_BWD_PART_KV 1
#define RING_ATTN_BWD_PART_Q 2
size_t ring_attn_bwd_ring_workspace_bytes(int B, int Hq, int Hkv, int64_t S, int D, int P,
                                          int causal, int layout, int dtype);
int ring_attn_bwd_ring_prep(const void* out_shard, const float* lse_shard, const void* dout_shard,
                            int B, int Hq, int Hkv, int64_t S, int D, int P, int q_index,
                            int causal, int layout, int dtype,
                            void* workspace, size_t workspace_bytes, void* stream);
int ring_attn_bwd_ring_step(const void* q_shard, const void* dout_shard, const void* k_shard, const void* v_shard,
                            float* dq_acc, float* dk_acc, float* dv_acc, void* dq, void* dk, void* dv,
                            int B, int Hq, int Hkv, int64_t S, int D, int P, int q_index, int kv_index,
                            int causal, int layout, float scale, int dtype, int parts, int flags,
                            void* workspace, size_t workspace_bytes, void* stream);

/*
 * Bytes of device workspace ring_attn_decode needs: the status header plus the
 * split-KV partials (at most 1024 per row). Returns 0 for invalid arguments.
 */
size_t ring_attn_decode_workspace_bytes(int B, int Hq, int Hkv, int64_t S, int D, int P, int layout, int dtype);

/*
 * One decode step against a KV cache of S tokens kept in P ring shards (layout as in
 * ring_attn_fwd). Each head has one new query row whose position follows every cached
 * key, so it attends to all S keys (no mask): out = softmax(scale q k^T) v, and lse.
 * (After a million-token prefill, each new token reads the whole cache: RingAttention
 * newsletter, cmlonder, section "code and integration map".) The cache is read once,
 * split across SMs by shard and chunk, and the normalised partials are combined by
 * the merge of ring_attn_merge.
 *   q   : device [B, Hq, D] bf16          k, v : device [B, Hkv, S, D] bf16
 *   out : device [B, Hq, D] bf16          lse  : device [B, Hq] fp32
 * Supported: bf16, D = 128, Hq/Hkv <= 32, an sm_100 device (zigzag needs
 * (S/(2P)) % 128 == 0); otherwise RING_ATTN_EUNSUPPORTED. S % P == 0.
 */
int ring_attn_decode(const void* q, const void* k, const void* v, void* out, float* lse,
                     int B, int Hq, int Hkv, int64_t S, int D, int P, int layout, float scale, int dtype,
                     void* workspace, size_t workspace_bytes, void* stream);

/*
 * Synchronise `stream` and read the status word at the start of `workspace`
 * (written by the last compute call that used it): 0, or RING_ATTN_ETIMEOUT.
 * Returns RING_ATTN_ECUDA if the stream reports an error.
 */
int ring_attn_status(const void* workspace, void* stream);

/*
 * ring_attn_fwd without a caller workspace. The method described by the pages has no
 * counterpart; this is a library convenience. It is for callers that cannot allocate
 * device memory: a plain C/C++ host that links only this library and has no device
 * allocator of its own, or a process whose device memory is planned up front and
 * which treats any later allocation as an error.
 *
 * The scratch (status word included) is a static __device__ array of this library,
 * RING_ATTN_NOALLOC_SCRATCH_BYTES bytes per device. Neither the call nor its one-time
 * setup calls cudaMalloc, cudaFree or any other allocating routine.
 *   Arguments q ... dtype, stream: as ring_attn_fwd.
 *   scratch_out  optional host pointer (may be NULL). On success it receives the
 *                device address of this device's scratch. Pass that address to
 *                ring_attn_status() to read the status word of the last call.
 * Setup: the first call in each CUDA context (the device's primary context, or a
 * context the caller made current with the driver API) looks up the array's
 * device address in that context (cudaGetSymbolAddress) and caches it under the
 * context's unique id, so a context created after cudaDeviceReset gets a fresh
 * lookup. Make that first call before any stream capture in that context.
 * Errors: as ring_attn_fwd (the same code for the same bad argument). If these
 * arguments need more workspace than the array holds, it returns
 * RING_ATTN_EWORKSPACE and enqueues nothing. If the address lookup fails, it
 * returns RING_ATTN_ECUDA.
 * Concurrency: every call on a device shares one scratch array. Calls that overlap
 * on the device (different streams, or host threads without ordering) race on the
 * status word. Order them on one stream, or use ring_attn_fwd with separate
 * workspaces.
 */
#define RING_ATTN_NOALLOC_SCRATCH_BYTES 4096
int ring_attn_fwd_noalloc(const void* q, const void* k, const void* v, void* out, float* lse,
                          int B, int Hq, int Hkv, int64_t S, int D, int P,
                          int causal, int layout, float scale, int dtype,
                          void* stream, void** scratch_out);

/* ---- test hooks ------------------------------------------------------------ */

/*
 * Host only, no GPU. Walks the exact schedule and per-element masks of one pass of
 * ring_attn_bwd (pass 0: the dK/dV kernel's 128-key units and the 64-row query steps
 * each meets; pass 1: the dQ kernel's 128-row query units and their backward-ring walk
 * in 64-key steps) and adds 1 to counts[t*S + u] for every (query token t, key token u) pair
 * it lets into the gradient. counts: host S*S int32 zeroed by the caller, S <= 4096.
 * Returns the number of tile visits, or a negative error code.
 */
int64_t ring_attn_debug_bwd_visit_counts(int64_t S, int P, int causal, int layout, int pass, int32_t* counts);

/*
 * Host only, no GPU. Walks the exact unit/tile schedule and per-element masks the
 * kernels use (tile sizes tile_q x tile_k, any positive values) and adds 1 to
 * counts[t*S + u] for every (query token t, key token u) pair the schedule lets
 * into the softmax. counts is host memory of S*S int32, zeroed by the caller.
 * S <= 4096. Returns the number of visited tiles (>= 0) or an error code.
 */
int64_t ring_attn_debug_visit_counts(int64_t S, int P, int causal, int layout,
                                     int tile_q, int tile_k, int32_t* counts);

/*
 * Host only. Writes the fused kernel's work units in launch order for query
 * blocks of tile_q rows: 5 int32 per unit (b, h, q_shard, row_block, kv tiles of
 * 128 keys the unit visits). Returns the unit count, or an error code
 * (RING_ATTN_EINVAL if it exceeds max_units).
 */
int ring_attn_debug_decode_units(int B, int Hq, int Hkv, int64_t S, int P, int causal, int layout, int tile_q,
                                 int32_t* units_out, int64_t max_units);

/*
 * Host only. The (kv_shard, kv_tile) sequence, in visiting order, of work unit
 * `unit` (launch order, query blocks of tile_q rows, key tiles of tile_k keys):
 * 2 int32 per visited tile into pairs_out. Returns the tile count or an error
 * code (RING_ATTN_EINVAL if it exceeds max_pairs or unit is out of range).
 */
int64_t ring_attn_debug_unit_walk(int B, int Hq, int Hkv, int64_t S, int P, int causal, int layout, int tile_q,
                                  int tile_k, int64_t unit, int32_t* pairs_out, int64_t max_pairs);

/*
 * Host only. Fills info[0..5] for the fused-kernel grid of these arguments:
 * number of units, total KV tiles visited, KV tiles with a partial mask, longest
 * unit in tiles, first unit's tiles, last unit's tiles. Returns 0 or an error code.
 */
int ring_attn_debug_schedule_info(int B, int Hq, int Hkv, int64_t S, int D, int P,
                                  int causal, int layout, int64_t* info);

/*
 * Device test of the fused kernel's software 2^x (FMA-pipe polynomial used for a
 * fraction of the softmax exponentials): y[i] = 2^x[i] for i < n, n even, device
 * pointers, 16-byte aligned. Relative error <= 1.02e-4 for -126 <= x <= 127;
 * x <= -127 (including -inf) gives exactly 0.
 */
int ring_attn_debug_exp2(const float* x, float* y, int64_t n, void* stream);

/*
 * Launches one CTA that waits on an mbarrier nobody arrives on, with a watchdog
 * limit of timeout_us microseconds; the wait gives up, the kernel records
 * RING_ATTN_ETIMEOUT in the workspace status word and returns. Exercises the
 * bounded-wait path without faulting or hanging the GPU.
 */
int ring_attn_debug_watchdog(int timeout_us, void* workspace, size_t workspace_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* RINGATTN_H_ */
