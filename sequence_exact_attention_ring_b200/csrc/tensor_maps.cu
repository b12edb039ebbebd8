// Host-side TMA tensor maps over sharded [B, H, S, D] bf16 tensors.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ring_schedule.h"
#include "ringattn_internal.h"

namespace ringattn {

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

// 4-D view of a [B, H, S, D] bf16 tensor whose sequence axis is split into P
// shards, dimensions listed innermost first so the strides grow:
//   contiguous (D, local, shard, batch*heads): shards are consecutive token ranges;
//   striped    (D, shard, local, batch*heads): shards interleave with stride P;
//   zigzag     (D, offset, chunk, batch*heads): 2P chunks of Sq/2 tokens.
// shard_map_coords gives a row's (dim 1, dim 2). Box: 64 elements (128 bytes,
// 128-byte swizzle) by `box_rows` consecutive tokens.
int encode_shard_map(CUtensorMap* map, const void* base, const RingGeom& g, int heads, int D, int box_rows) {
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
    box[0] = 64; box[1] = 1; box[2] = box_rows; box[3] = 1;
  } else if (g.layout == kZigzag) {
    const uint64_t C = (uint64_t)g.Sq / 2;
    dims[0] = D; dims[1] = C; dims[2] = 2 * (uint64_t)g.P; dims[3] = (uint64_t)g.B * heads;
    strides[0] = row; strides[1] = row * C; strides[2] = row * g.S;
    box[0] = 64; box[1] = box_rows; box[2] = 1; box[3] = 1;
  } else {
    dims[0] = D; dims[1] = g.Sq; dims[2] = g.P; dims[3] = (uint64_t)g.B * heads;
    strides[0] = row; strides[1] = row * g.Sq; strides[2] = row * g.S;
    box[0] = 64; box[1] = box_rows; box[2] = 1; box[3] = 1;
  }
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? RING_ATTN_OK : RING_ATTN_ECUDA;
}

int encode_input_map(CUtensorMap* map, const void* base, const RingGeom& g, bool local, int heads, int D,
                     int box_rows) {
  if (!local) return encode_shard_map(map, base, g, heads, D, box_rows);
  // one shard in local order is a contiguous sequence of Sq rows (one shard of P = 1)
  RingGeom one = g;
  one.layout = kContiguous;
  one.S = g.Sq;
  one.P = 1;
  return encode_shard_map(map, base, one, heads, D, box_rows);
}

}  // namespace ringattn
