// sel.cuh -- the selected blocks of one (sequence, group) as a list of key chunks.
//
// The selected branch attends to the tokens tau <= t of the blocks chosen by top-n
// (selection branch, top168.com article on VideoNSA, section "一、革命性的三重注意机制").
// The decode branch kernel streams those tokens in fixed-size chunks; build_chunk_list
// turns a block list into the chunk start positions it has to visit.
#pragma once
#include "warp_attn.cuh"

namespace nsa {

// Compact the valid `ck`-key chunks of a selection list (ascending block indices, -1
// padded) into `out` (shared, >= top_n * sel_len / ck entries); returns the count. A chunk
// is valid if it starts at or before t.
__device__ __forceinline__ int build_chunk_list(const int32_t* __restrict__ blocks, int top_n, int sel_len, int t,
                                                int* out, int lane, int ck = kChunkKeys) {
  const int per = sel_len / ck;
  int count = 0;
  for (int base = 0; base < per * top_n; base += 32) {
    const int ci = base + lane;
    int start = -1;
    if (ci < per * top_n) {
      const int j = blocks[ci / per];
      const int s = j * sel_len + (ci % per) * ck;
      if (j >= 0 && s <= t) start = s;
    }
    const uint32_t m = __ballot_sync(0xffffffffu, start >= 0);
    if (start >= 0) out[count + __popc(m & ((1u << lane) - 1u))] = start;
    count += __popc(m);
  }
  __syncwarp();
  return count;
}

}  // namespace nsa
