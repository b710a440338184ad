// topn.cuh -- selection branch, step 2: per (token, KV group), keep the top-n blocks.
//
// The selection branch scores all video blocks and keeps only the most important ones
// (top168.com article on VideoNSA, section "一、革命性的三重注意机制", selection
// branch). This library always keeps block 0 and the two blocks nearest the query
// (t/l' and t/l' - 1, the "local" blocks), then the best top_n - |forced| remaining blocks
// j <= t/l' ordered by score (descending) and block index (ascending) on ties. The
// result is written ascending and padded with -1.
//
// One warp per (row, group). The row's candidate scores are staged in shared memory;
// each lane keeps the best of its strided subset as a 64-bit key
// (score bits << 32 | ~j): scores are >= 0, so unsigned comparison of the float bits
// orders them, and the complemented index makes the lower block win a tie. Each round
// takes the warp-wide maximum key, removes it, and the owning lane rescans its subset.
#pragma once
#include <cstdint>
#include "sm100.cuh"

namespace nsa {

constexpr int kTopnWarps = 4;

__device__ __forceinline__ unsigned long long warp_max_u64(unsigned long long x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long y = __shfl_xor_sync(0xffffffffu, x, o);
    x = y > x ? y : x;
  }
  return x;
}

// Warp-cooperative top-n of one (row, group). `sc` (shared, >= jt+1 floats) holds the
// candidate scores of blocks 0..jt; `bits` (shared, >= jt/32+1 words) receives the
// selection bitmap. Writes top_n entries to dst (and dst2 if non-null).
__device__ __forceinline__ void warp_topn(float* sc, uint32_t* bits, const float* __restrict__ src, int jt,
                                          int top_n, int32_t* __restrict__ dst, int32_t* __restrict__ dst2,
                                          int lane) {
  const int nwords = jt / 32 + 1;
  for (int w = lane; w < nwords; w += 32) bits[w] = 0u;
  __syncwarp();
  // forced blocks are marked selected and kept out of the candidate set (score -1)
  for (int j = lane; j <= jt; j += 32) {
    const bool forced = (j == 0) || (j == jt) || (j == jt - 1);
    sc[j] = forced ? -1.f : src[j];
    if (forced) atomicOr(&bits[j >> 5], 1u << (j & 31));
  }
  __syncwarp();
  const int nf = 1 + (jt >= 1 ? 1 : 0) + (jt >= 2 ? 1 : 0);
  const int k = min(top_n - nf, jt + 1 - nf);
  auto local_best = [&]() -> unsigned long long {
    unsigned long long best = 0ull;
    for (int j = lane; j <= jt; j += 32) {
      const float x = sc[j];
      if (x >= 0.f) {
        const unsigned long long key =
            (static_cast<unsigned long long>(__float_as_uint(x)) << 32) | (0xFFFFFFFFu - static_cast<uint32_t>(j));
        best = key > best ? key : best;
      }
    }
    return best;
  };
  unsigned long long mine = local_best();
  for (int round = 0; round < k; ++round) {
    const unsigned long long win = warp_max_u64(mine);
    if (win == 0ull) break;
    const int j = static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(win & 0xFFFFFFFFull));
    if ((j & 31) == lane) {
      sc[j] = -1.f;
      bits[j >> 5] |= 1u << (j & 31);
      mine = local_best();
    }
    __syncwarp();
  }
  // emit the selected set in ascending order, then -1 padding
  int pos = 0;
  for (int w = 0; w < nwords; ++w) {
    const uint32_t word = bits[w];
    const bool set = (word >> lane) & 1u;
    const int p = pos + __popc(word & ((1u << lane) - 1u));
    if (set && p < top_n) {
      dst[p] = w * 32 + lane;
      if (dst2) dst2[p] = w * 32 + lane;
    }
    pos += __popc(word);
  }
  for (int p = pos + lane; p < top_n; p += 32) {
    dst[p] = -1;
    if (dst2) dst2[p] = -1;
  }
  __syncwarp();
}

// scores: [nitems][nsel] fp32 (item = row * hkv + g); idx / idx_copy: [nitems][top_n].
// Row position t = row (prefill rows are token positions).
__global__ void __launch_bounds__(kTopnWarps * 32) topn_kernel(const float* __restrict__ scores, int nitems, int hkv,
                                                                int nsel, int sel_len, int top_n,
                                                                int32_t* __restrict__ idx,
                                                                int32_t* __restrict__ idx_copy) {
  extern __shared__ float tsm[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwords = (nsel + 31) / 32;
  float* sc = tsm + static_cast<size_t>(warp) * (nsel + nwords);
  uint32_t* bits = reinterpret_cast<uint32_t*>(sc + nsel);
  for (int item = blockIdx.x * kTopnWarps + warp; item < nitems; item += gridDim.x * kTopnWarps) {
    const int t = item / hkv;
    const int jt = t / sel_len;
    if (jt >= nsel) {  // cannot happen for valid arguments; never index past the row
      if (lane == 0) record_error(kErrBadIndex);
      continue;
    }
    warp_topn(sc, bits, scores + static_cast<size_t>(item) * nsel, jt, top_n, idx + static_cast<size_t>(item) * top_n,
              idx_copy ? idx_copy + static_cast<size_t>(item) * top_n : nullptr, lane);
  }
}

}  // namespace nsa
