// kda_items.cuh — dispatch order of the fp32 chunk-local work items (forward and backward).
#pragma once

#include "kda_common.cuh"

namespace kda {

// ---------------------------------------------------------------------------------------------
// Chunk-local work items (chunk c, head h) are dispatched with the head index fastest (grid x =
// head, y and z = chunk): the blocks resident at one time then cover whole token rows ([H, d],
// contiguous in the [tokens, H, d] layout) of a few consecutive chunks instead of one piece per
// row. Chunks beyond 65535 continue in z. (The tensor-core chunk-local kernel keeps the chunk
// index fastest: its A-matrix mode follows the head's decay, so with the heads fastest every SM
// runs several modes at once, and its prefill with raw gates measured 18 % slower that way.)
// ---------------------------------------------------------------------------------------------
struct ChunkItem {
  int c, h;
};
__device__ __forceinline__ ChunkItem chunk_item() {
  return ChunkItem{(int)(blockIdx.z * gridDim.y + blockIdx.y), (int)blockIdx.x};
}
inline dim3 item_grid(int max_chunks, int H) {  // max_chunks > 0
  const int cy = max_chunks < 65535 ? max_chunks : 65535;
  return dim3((unsigned)H, (unsigned)cy, (unsigned)ceil_div(max_chunks, cy));
}

}  // namespace kda
