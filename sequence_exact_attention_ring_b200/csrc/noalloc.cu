// ring_attn_fwd_noalloc: the fused forward with its scratch in a file-scope device array.
//
// ring_attn_fwd takes a caller-provided workspace (its first word is the kernel's
// status word, reset to 0 before every launch and set to RING_ATTN_ETIMEOUT if a
// device-side wait gives up). Some callers cannot provide one:
//   * a plain C or C++ host that links only this library has no device allocator of
//     its own and would need cudaMalloc just for a few hundred bytes;
//   * a process that reserves all of its device memory up front (a serving loop
//     with a fixed memory plan) treats any allocation after start-up as an error.
// This entry point serves them: the scratch is a static __device__ array of this
// library's module, so neither the call nor its setup allocates device memory.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "ringattn.h"

namespace {

static_assert(RING_ATTN_NOALLOC_SCRATCH_BYTES % 256 == 0, "scratch size");
static __device__ __align__(256) unsigned char g_noalloc_scratch[RING_ATTN_NOALLOC_SCRATCH_BYTES];

// The array's device address belongs to the module loaded into one CUDA context: a
// context created with the driver API loads its own copy, and cudaDeviceReset
// destroys the primary context (the next one may place the array elsewhere). So the
// address is cached per context, keyed by the context's unique id (cuCtxGetId),
// and looked up again whenever the current context is one not seen before.
typedef CUresult (*PFN_ctxGetCurrent)(CUcontext*);
typedef CUresult (*PFN_ctxGetId)(CUcontext, unsigned long long*);

constexpr int kCacheEntries = 64;
struct CacheEntry {
  unsigned long long ctx_id;
  void* ptr;
};
std::mutex g_setup_mutex;
CacheEntry g_cache[kCacheEntries];
int g_cache_next = 0;  // round-robin replacement once the table is full

bool current_context_id(unsigned long long* id) {
  static PFN_ctxGetCurrent get_current = nullptr;
  static PFN_ctxGetId get_id = nullptr;
  if (!get_current || !get_id) {
    void* a = nullptr;
    void* b = nullptr;
    cudaDriverEntryPointQueryResult qa, qb;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &a, cudaEnableDefault, &qa) != cudaSuccess ||
        qa != cudaDriverEntryPointSuccess ||
        cudaGetDriverEntryPoint("cuCtxGetId", &b, cudaEnableDefault, &qb) != cudaSuccess ||
        qb != cudaDriverEntryPointSuccess)
      return false;
    get_current = reinterpret_cast<PFN_ctxGetCurrent>(a);
    get_id = reinterpret_cast<PFN_ctxGetId>(b);
  }
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of the scratch array in the current context, looked up once per
// context (with that context current). Returns NULL if the lookup fails.
void* scratch_for_current_context(int* rc) {
  unsigned long long id = 0;
  if (!current_context_id(&id)) {
    // no context is current yet: the runtime's first call on this thread creates the
    // current device's primary context and makes it current
    void* probe = nullptr;
    if (cudaGetSymbolAddress(&probe, g_noalloc_scratch) != cudaSuccess || !current_context_id(&id)) {
      *rc = RING_ATTN_ECUDA;
      return nullptr;
    }
  }
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  for (int e = 0; e < kCacheEntries; ++e) {
    if (g_cache[e].ptr != nullptr && g_cache[e].ctx_id == id) {
      *rc = RING_ATTN_OK;
      return g_cache[e].ptr;
    }
  }
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) {
    *rc = RING_ATTN_ECUDA;
    return nullptr;
  }
  g_cache[g_cache_next] = CacheEntry{id, ptr};
  g_cache_next = (g_cache_next + 1) % kCacheEntries;
  *rc = RING_ATTN_OK;
  return ptr;
}

}  // namespace

extern "C" int ring_attn_fwd_noalloc(const void* q, const void* k, const void* v, void* out, float* lse, int B,
                                     int Hq, int Hkv, int64_t S, int D, int P, int causal, int layout, float scale,
                                     int dtype, void* stream, void** scratch_out) {
  const size_t need = ring_attn_fwd_workspace_bytes(B, Hq, Hkv, S, D, P, causal, layout, dtype);
  if (need == 0) {
    // the shape arguments are invalid or unsupported: ring_attn_fwd returns the same
    // code as for any caller (its shape check comes before anything is enqueued)
    return ring_attn_fwd(q, k, v, out, lse, B, Hq, Hkv, S, D, P, causal, layout, scale, dtype, nullptr, 0, stream);
  }
  if (need > RING_ATTN_NOALLOC_SCRATCH_BYTES) return RING_ATTN_EWORKSPACE;
  int rc = RING_ATTN_OK;
  void* scratch = scratch_for_current_context(&rc);
  if (!scratch) return rc;
  if (scratch_out) *scratch_out = scratch;
  // ring_attn_fwd validates the remaining arguments and zeroes the status word on
  // `stream` (cudaMemsetAsync, no allocation) before its kernel starts.
  return ring_attn_fwd(q, k, v, out, lse, B, Hq, Hkv, S, D, P, causal, layout, scale, dtype, scratch,
                       RING_ATTN_NOALLOC_SCRATCH_BYTES, stream);
}
