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
#include <cuda_runtime.h>

#include <mutex>

#include "ringattn.h"

namespace {

static_assert(RING_ATTN_NOALLOC_SCRATCH_BYTES % 256 == 0, "scratch size");
static __device__ __align__(256) unsigned char g_noalloc_scratch[RING_ATTN_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices];  // device address of g_noalloc_scratch, per device ordinal

// Device address of the scratch array on the current device, looked up once per device
// (with that device current). Returns NULL if the lookup fails.
void* scratch_for_current_device(int* rc) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    *rc = RING_ATTN_ECUDA;
    return nullptr;
  }
  if (dev < 0 || dev >= kMaxDevices) {
    *rc = RING_ATTN_EUNSUPPORTED;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) {
      *rc = RING_ATTN_ECUDA;
      return nullptr;
    }
    g_scratch_ptr[dev] = ptr;
  }
  *rc = RING_ATTN_OK;
  return g_scratch_ptr[dev];
}

}  // namespace

extern "C" int ring_attn_fwd_noalloc(const void* q, const void* k, const void* v, void* out, float* lse, int B,
                                     int Hq, int Hkv, int64_t S, int D, int P, int causal, int layout, float scale,
                                     int dtype, void* stream, void** scratch_out) {
  const size_t need = ring_attn_fwd_workspace_bytes(B, Hq, Hkv, S, D, P, causal, layout, dtype);
  if (need == 0) return RING_ATTN_EINVAL;
  if (need > RING_ATTN_NOALLOC_SCRATCH_BYTES) return RING_ATTN_EWORKSPACE;
  int rc = RING_ATTN_OK;
  void* scratch = scratch_for_current_device(&rc);
  if (!scratch) return rc;
  if (scratch_out) *scratch_out = scratch;
  // ring_attn_fwd validates the remaining arguments and zeroes the status word on
  // `stream` (cudaMemsetAsync, no allocation) before its kernel starts.
  return ring_attn_fwd(q, k, v, out, lse, B, Hq, Hkv, S, D, P, causal, layout, scale, dtype, scratch,
                       RING_ATTN_NOALLOC_SCRATCH_BYTES, stream);
}
