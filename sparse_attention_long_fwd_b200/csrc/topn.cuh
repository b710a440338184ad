// topn.cuh -- selection branch, step 2: per (token, KV group), keep the top-n blocks.
//
// The selection branch scores all video blocks and keeps only the most important ones
// (top168.com article on VideoNSA, section "一、革命性的三重注意机制", selection
// branch). This library always keeps block 0 and the two blocks nearest the query
// (t/l' and t/l' - 1, the "local" blocks), then the best top_n - |forced| remaining blocks
// j <= t/l' ordered by score (descending) and block index (ascending) on ties. The
// result is written ascending and padded with -1.
//
// One warp per (row, group); see warp_topn for the selection itself.
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

// Warp-cooperative top-n of one (row, group). `sc` (shared, >= jt+1 floats) receives the
// candidate scores of blocks 0..jt; `bits` (shared, >= jt/32+1 words) the selection
// bitmap; `list` (shared, >= jt+1 ints) is scratch. Writes top_n entries to dst (and dst2
// if non-null).
//
// Keys are (score bits << 32 | ~j), unique per block. Each lane first keeps the two
// largest keys of its strided subset; the k-th largest of those 64 keys is a lower bound
// on the k-th largest key overall (they are a subset of all keys), so only candidates at
// or above it can be selected. Those survivors -- usually about k of them -- are
// compacted and the exact top-k is taken from them by rounds of warp-wide maxima.
__device__ __forceinline__ unsigned long long cand_key(float x, int j) {
  return x >= 0.f ? (static_cast<unsigned long long>(__float_as_uint(x)) << 32) |
                        (0xFFFFFFFFu - static_cast<uint32_t>(j))
                  : 0ull;
}

__device__ __forceinline__ void warp_topn(float* sc, uint32_t* bits, int* list, const float* __restrict__ src,
                                          int jt, int top_n, int32_t* __restrict__ dst,
                                          int32_t* __restrict__ dst2, int lane) {
  const int nwords = jt / 32 + 1;
  for (int w = lane; w < nwords; w += 32) bits[w] = 0u;
  __syncwarp();
  // stage the candidate scores, 8 independent loads per lane in flight; forced blocks are
  // marked selected and kept out of the candidate set (score -1)
  for (int base = 0; base <= jt; base += 256) {
    float v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int j = base + u * 32 + lane;
      v[u] = j <= jt ? src[j] : -1.f;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int j = base + u * 32 + lane;
      if (j <= jt) sc[j] = (j == 0 || j == jt || j == jt - 1) ? -1.f : v[u];
    }
  }
  if (lane == 0) {
    bits[0] |= 1u;
    if (jt >= 1) bits[jt >> 5] |= 1u << (jt & 31);
    if (jt >= 2) bits[(jt - 1) >> 5] |= 1u << ((jt - 1) & 31);
  }
  __syncwarp();
  const int nf = 1 + (jt >= 1 ? 1 : 0) + (jt >= 2 ? 1 : 0);
  const int k = min(top_n - nf, jt + 1 - nf);
  if (k > 0) {
    // 1. the two largest keys of this lane's subset
    unsigned long long k1 = 0ull, k2 = 0ull;
    for (int j = lane; j <= jt; j += 32) {
      const unsigned long long key = cand_key(sc[j], j);
      if (key > k1) {
        k2 = k1;
        k1 = key;
      } else if (key > k2) {
        k2 = key;
      }
    }
    // 2. threshold = k-th largest of the 64 lane-top-2 keys (0 if fewer exist)
    unsigned long long thr = 0ull;
    {
      unsigned long long a = k1, b2 = k2;
      for (int round = 0; round < k && round < 64; ++round) {
        const unsigned long long w = warp_max_u64(a);
        thr = w;
        if (w == 0ull) break;
        if (a == w) {
          a = b2;
          b2 = 0ull;
        }
      }
      if (k > 64) thr = 0ull;
    }
    // 3. compact the survivors (keys >= threshold)
    int nsurv = 0;
    for (int base = 0; base <= jt; base += 32) {
      const int j = base + lane;
      const unsigned long long key = j <= jt ? cand_key(sc[j], j) : 0ull;
      const bool keep = key != 0ull && key >= thr;
      const uint32_t m = __ballot_sync(0xffffffffu, keep);
      if (keep) list[nsurv + __popc(m & ((1u << lane) - 1u))] = j;
      nsurv += __popc(m);
    }
    __syncwarp();
    // 4. exact top-k among the survivors
    auto local_best = [&]() -> unsigned long long {
      unsigned long long best = 0ull;
      for (int i = lane; i < nsurv; i += 32) {
        const int j = list[i];
        const unsigned long long key = cand_key(sc[j], j);
        best = key > best ? key : best;
      }
      return best;
    };
    unsigned long long mine = local_best();
    for (int round = 0; round < k; ++round) {
      const unsigned long long win = warp_max_u64(mine);
      if (win == 0ull) break;
      const int j = static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(win & 0xFFFFFFFFull));
      if (win == mine) {
        sc[j] = -1.f;
        bits[j >> 5] |= 1u << (j & 31);
        mine = local_best();
      }
      __syncwarp();
    }
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

// Register-resident variant for rows with at most 32 * PL candidate blocks (jt < 32 * PL)
// and top_n <= 32 (the selected set is held one block per lane, then sorted):
// lane l holds blocks l, l + 32, ... as 32-bit keys (score bits + 1 for a candidate, so a
// zero score stays selectable; 0 for none); key order is score order because scores are
// non-negative. Warp-wide maxima are single __reduce_max_sync instructions.
//   1. each lane's two half-slice maxima: the k-th largest of those 64 keys is a lower
//      bound on the k-th largest key overall (they are distinct blocks of the row);
//   2. candidates at or above that bound are compacted to `list` (block indices; the first
//      64 are kept, `list` holds 64 ints);
//   3. k rounds take the largest key among them, the smallest block index on ties (from the
//      list when at most 64 survived, else by scanning the candidates again).
template <int PL>
__device__ __forceinline__ void warp_topn_regs(int* list, const float* __restrict__ src, int jt, int top_n,
                                               int32_t* __restrict__ dst, int32_t* __restrict__ dst2, int lane) {
  float v[PL];
#pragma unroll
  for (int u = 0; u < PL; ++u) {
    const int j = lane + 32 * u;
    v[u] = j <= jt ? src[j] : -1.f;
  }
  uint32_t key[PL];
#pragma unroll
  for (int u = 0; u < PL; ++u) {
    const int j = lane + 32 * u;
    const bool forced = j == 0 || j == jt || j == jt - 1;
    key[u] = (j <= jt && !forced && v[u] >= 0.f) ? __float_as_uint(v[u]) + 1u : 0u;
  }
  // the selected blocks, one per lane (INT_MAX: none): forced blocks in lanes 0..nf-1
  const int nf = 1 + (jt >= 1 ? 1 : 0) + (jt >= 2 ? 1 : 0);
  int mine = lane == 0 ? 0 : (lane == 1 && jt >= 1) ? jt : (lane == 2 && jt >= 2) ? jt - 1 : 0x7fffffff;
  const int k = min(top_n - nf, jt + 1 - nf);
  if (k > 0) {
    // 1. lower bound: k-th largest of the 64 half-slice maxima (0 when fewer exist)
    uint32_t a = 0u, b = 0u;
#pragma unroll
    for (int u = 0; u < PL; ++u) {
      if (u < PL / 2) a = max(a, key[u]);
      else b = max(b, key[u]);
    }
    uint32_t thr = 0u;
    if (k <= 64) {
      for (int round = 0; round < k; ++round) {
        const uint32_t w = __reduce_max_sync(0xffffffffu, max(a, b));
        thr = w;
        if (w == 0u) break;
        // remove one instance of w: the lowest lane holding it, its first slot
        const uint32_t holders = __ballot_sync(0xffffffffu, a == w || b == w);
        if (lane == __ffs(holders) - 1) {
          if (a == w) a = 0u; else b = 0u;
        }
      }
    }
    // 2. compact the candidates with key >= thr (block indices, in lane-slot order)
    static_assert(PL <= 64, "candidate bits");
    uint32_t cand = 0u, cand_hi = 0u;  // bit u (u - 32): block lane + 32u is a candidate
#pragma unroll
    for (int u = 0; u < PL; ++u) {
      if (key[u] != 0u && key[u] >= thr) {
        if (u < 32) cand |= 1u << (u & 31);
        else cand_hi |= 1u << (u & 31);
      }
    }
    const int cnt = __popc(cand) + __popc(cand_hi);
    int off = cnt;  // inclusive scan over lanes
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, off, o);
      if (lane >= o) off += y;
    }
    const int nsurv = __shfl_sync(0xffffffffu, off, 31);
    off -= cnt;
#pragma unroll
    for (int u = 0; u < PL; ++u) {
      const bool c = u < 32 ? ((cand >> (u & 31)) & 1u) : ((cand_hi >> (u & 31)) & 1u);
      if (c) {
        if (off < 64) list[off] = lane + 32 * u;  // the exact pass below needs only 64
        ++off;
      }
    }
    __syncwarp();
    // 3. exact top-k among them: largest key, smallest block index on ties; the winner of
    //    round r goes to lane nf + r
    if (nsurv <= 64) {
      const int j0 = lane < nsurv ? list[lane] : -1, j1 = lane + 32 < nsurv ? list[lane + 32] : -1;
      // the keys again from the (cached) scores of the compacted blocks
      uint32_t q0 = j0 >= 0 ? __float_as_uint(src[j0]) + 1u : 0u;
      uint32_t q1 = j1 >= 0 ? __float_as_uint(src[j1]) + 1u : 0u;
      for (int round = 0; round < k; ++round) {
        const uint32_t w = __reduce_max_sync(0xffffffffu, max(q0, q1));
        if (w == 0u) break;
        const uint32_t c0 = q0 == w ? static_cast<uint32_t>(j0) : 0xFFFFFFFFu;
        const uint32_t c1 = q1 == w ? static_cast<uint32_t>(j1) : 0xFFFFFFFFu;
        const uint32_t jw = __reduce_min_sync(0xffffffffu, min(c0, c1));
        if (static_cast<uint32_t>(j0) == jw) q0 = 0u;
        if (static_cast<uint32_t>(j1) == jw) q1 = 0u;
        if (lane == nf + round) mine = static_cast<int>(jw);
      }
    } else {
      // many ties at the bound (rare): rounds over the candidate bits, the keys read again
      // from the row (the list holds only the first 64 candidates)
      for (int round = 0; round < k; ++round) {
        uint32_t best = 0u, bj = 0xFFFFFFFFu;
        for (int u = 0; u < PL; ++u) {  // slots in block order: the first maximum has the lowest index
          const bool c = u < 32 ? ((cand >> (u & 31)) & 1u) : ((cand_hi >> (u & 31)) & 1u);
          if (c) {
            const float x = src[lane + 32 * u];
            const uint32_t kx = __float_as_uint(x) + 1u;
            if (kx > best) {
              best = kx;
              bj = static_cast<uint32_t>(lane + 32 * u);
            }
          }
        }
        const uint32_t w = __reduce_max_sync(0xffffffffu, best);
        if (w == 0u) break;
        const uint32_t jw = __reduce_min_sync(0xffffffffu, best == w ? bj : 0xFFFFFFFFu);
        if (static_cast<int>(jw & 31u) == lane) {  // taken: clear its candidate bit
          const int u = static_cast<int>(jw >> 5);
          if (u < 32) cand &= ~(1u << u);
          else cand_hi &= ~(1u << (u - 32));
        }
        if (lane == nf + round) mine = static_cast<int>(jw);
      }
    }
  }
  // ascending order: bitonic sort of the 32 lanes' values (empty lanes sort last)
#pragma unroll
  for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      const int other = __shfl_xor_sync(0xffffffffu, mine, stride);
      const bool up = (lane & size) == 0;           // this block sorts ascending
      const bool low = (lane & stride) == 0;        // this lane keeps the smaller value
      mine = (low == up) ? min(mine, other) : max(mine, other);
    }
  }
  if (lane < top_n) {
    const int out = mine == 0x7fffffff ? -1 : mine;
    dst[lane] = out;
    if (dst2) dst2[lane] = out;
  }
  __syncwarp();
}

// scores: [nitems][stride] fp32 (item = row * hkv + g; stride >= nsel); idx / idx_copy:
// [nitems][top_n].
// Row position t = row (prefill rows are token positions); in a packed batch (vinfo, see
// AttnArgs) t is the row's position in its own sequence's video stream.
// One warp per (row, group). kRegsOnly: every row has fewer than 2,048 candidate blocks and
// top_n <= 32 (checked by the host), so only the register path runs and each warp needs just
// the 64-entry candidate list in shared memory; otherwise each warp also has the score row,
// the list and the bitmap of the shared-memory path.
template <bool kRegsOnly, bool kPacked = false>
__global__ void __launch_bounds__(kTopnWarps * 32) topn_kernel(const float* __restrict__ scores, int nitems, int hkv,
                                                                int nsel, int stride, int sel_len, int top_n,
                                                                int32_t* __restrict__ idx,
                                                                int32_t* __restrict__ idx_copy,
                                                                const int4* __restrict__ vinfo) {
  extern __shared__ float tsm[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwords = (nsel + 31) / 32;
  float* sc = tsm + static_cast<size_t>(warp) * (kRegsOnly ? 64 : 2 * nsel + nwords);
  int* list = kRegsOnly ? reinterpret_cast<int*>(sc) : reinterpret_cast<int*>(sc + nsel);
  uint32_t* bits = reinterpret_cast<uint32_t*>(list + nsel);
  for (int item = blockIdx.x * kTopnWarps + warp; item < nitems; item += gridDim.x * kTopnWarps) {
    const int row = item / hkv;
    const int t = kPacked ? row - vinfo[row].x : row;
    const int jt = t / sel_len;
    if (jt >= nsel || (kRegsOnly && (top_n > 32 || jt >= 32 * 64))) {
      // cannot happen for valid arguments; never index past the row
      if (lane == 0) record_error(kErrBadIndex);
      continue;
    }
    const float* src = scores + static_cast<size_t>(item) * stride;
    int32_t* d = idx + static_cast<size_t>(item) * top_n;
    int32_t* d2 = idx_copy ? idx_copy + static_cast<size_t>(item) * top_n : nullptr;
    if (!kRegsOnly && (top_n > 32 || jt >= 32 * 64)) warp_topn(sc, bits, list, src, jt, top_n, d, d2, lane);
    else if (jt < 32 * 4) warp_topn_regs<4>(list, src, jt, top_n, d, d2, lane);
    else if (jt < 32 * 16) warp_topn_regs<16>(list, src, jt, top_n, d, d2, lane);
    else if (jt < 32 * 32) warp_topn_regs<32>(list, src, jt, top_n, d, d2, lane);
    else warp_topn_regs<64>(list, src, jt, top_n, d, d2, lane);
  }
}

}  // namespace nsa
