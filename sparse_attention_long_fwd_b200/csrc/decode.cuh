// decode.cuh -- single-query NSA decode against a KV cache and a compressed cache.
//
// Per sequence b (query at t = L_b - 1) and KV group g the same three branches as the
// prefill are evaluated for one token (top168.com article on VideoNSA, section
// "一、革命性的三重注意机制"). With one query the work is a stream over the caches, so it
// is HBM-bound and split four ways:
//   dec_cmp_kernel      split-K over the compressed cache: each CTA attends to a slice of
//                       the visible blocks, keeps its base-2 logits for the scoring step
//                       and writes a partial (max, sum, unnormalised output) per head;
//   dec_select_kernel   merges the partials into o_cmp and the row log-sum-exp, turns
//                       the stored logits into selection-block scores summed over the
//                       group, and picks the top-n blocks (topn.cuh);
//   dec_branch_kernel   the selected-block and the sliding-window branches, one CTA per
//                       (sequence, group, branch), four warps splitting the key chunks;
//   dec_combine_kernel  out = g_cmp*o_cmp + g_sel*o_sel + g_win*o_win.
#pragma once
#include "sel.cuh"
#include "topn.cuh"

namespace nsa {

constexpr int kDecWarps = 4;

// Sequence length of b, clamped to [1, lmax]; an out-of-range value is recorded in the
// device error word instead of being used to index the caches.
__device__ __forceinline__ int seq_len_checked(const int32_t* seq_lens, int b, int lmax) {
  const int L = seq_lens[b];
  if (L < 1 || L > lmax) {
    record_error(kErrBadIndex);
    return L < 1 ? 1 : lmax;
  }
  return L;
}

struct DecArgs {
  int batch, lmax, hq, hkv, G, d;
  int ncmax;            // Ncmp(Lmax): compressed rows per sequence
  int nsplit;           // CTAs per (sequence, group) in dec_cmp_kernel
  int cmp_len, cmp_stride, sel_len, top_n, window, nsel_max;
  float sl2;            // softmax scale * log2(e)
  float* logits;        // [B][hkv][G][ncmax] base-2 scaled logits of the compressed branch
  float* part;          // [B][hkv][nsplit][G][2 + D] (m, l, o[D])
  float* o_cmp;         // [B][hq][D]
  float* lse;           // [B][hq] natural log
  float* scores;        // [B][hkv][nsel_max]
  int32_t* sel_idx;     // [B][hkv][top_n]
  float* o_sel;         // [B][hq][D]
  float* o_win;         // [B][hq][D]
};

template <int D>
struct DecSmem {
  WarpChunkBuf<D, kChunkKeys, 2> buf[kDecWarps];
  WarpPartial<D> part[kDecWarps];
  int chunk_start[kDecWarps][128];
};

// Merge the four warps' partial states of rows < G; returns through the callback
// f(row, m, l, o_ptr_scaled...) -- written inline at the two call sites below.
template <int D>
__device__ __forceinline__ void merge_rows(const WarpPartial<D>* parts, int nparts, int G, int row, float& M,
                                           float& L, float* wts) {
  M = -INFINITY;
  for (int w = 0; w < nparts; ++w) M = fmaxf(M, parts[w].m[row]);
  L = 0.f;
  for (int w = 0; w < nparts; ++w) {
    wts[w] = (M == -INFINITY) ? 0.f : ex2_approx(parts[w].m[row] - M);
    L += parts[w].l[row] * wts[w];
  }
}

template <int D>
__global__ void __launch_bounds__(kDecWarps * 32) dec_cmp_kernel(const __nv_bfloat16* __restrict__ q,
                                                                 const __nv_bfloat16* __restrict__ kcmp,
                                                                 const __nv_bfloat16* __restrict__ vcmp,
                                                                 const int32_t* __restrict__ seq_lens,
                                                                 const DecArgs a) {
  extern __shared__ uint8_t dec_smem_raw[];
  DecSmem<D>& sm = *reinterpret_cast<DecSmem<D>*>((reinterpret_cast<uintptr_t>(dec_smem_raw) + 127) & ~uintptr_t(127));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bg = blockIdx.y, b = bg / a.hkv, g = bg % a.hkv, split = blockIdx.x;
  const int L = seq_len_checked(seq_lens, b, a.lmax);
  const int nc = (L >= a.cmp_len) ? (L - a.cmp_len) / a.cmp_stride + 1 : 0;
  const int per = ((a.ncmax + a.nsplit - 1) / a.nsplit + kDecWarps * kChunkKeys - 1) / (kDecWarps * kChunkKeys) *
                  (kDecWarps * kChunkKeys);
  const int i0 = split * per;
  const int i1 = min(i0 + per, nc);
  const int wper = per / kDecWarps;
  const int w0 = i0 + warp * wper;
  const int w1 = min(w0 + wper, i1);
  uint32_t qa[D / 16][4];
  load_q_frags<D>(qa, q + (static_cast<size_t>(b) * a.hq + g * a.G) * D, a.G, lane);
  const size_t rs = static_cast<size_t>(a.hkv) * D;
  const __nv_bfloat16* kb = kcmp + static_cast<size_t>(b) * a.ncmax * rs + static_cast<size_t>(g) * D;
  const __nv_bfloat16* vb = vcmp + static_cast<size_t>(b) * a.ncmax * rs + static_cast<size_t>(g) * D;
  float* lg = a.logits + static_cast<size_t>(bg) * a.G * a.ncmax;
  auto& buf = sm.buf[warp];
  WarpAttnState<D> st;
  state_init(st);
  const int nch = w1 > w0 ? (w1 - w0 + kChunkKeys - 1) / kChunkKeys : 0;
  if (nch > 0) {
    load_chunk<D>(buf, 0, kb, vb, rs, w0, w1, lane);
    cp_async_commit();
  }
  for (int ci = 0; ci < nch; ++ci) {
    if (ci + 1 < nch) {
      load_chunk<D>(buf, (ci + 1) & 1, kb, vb, rs, w0 + (ci + 1) * kChunkKeys, w1, lane);
      cp_async_commit();
      cp_async_wait_1();
    } else {
      cp_async_wait_0();
    }
    __syncwarp();
    attend_chunk<D>(st, qa, buf, ci & 1, w0 + ci * kChunkKeys, w0, w1, a.sl2, lane, lg, a.ncmax, 0, a.G);
    __syncwarp();
  }
  state_reduce_l(st);
  state_store(st, sm.part[warp], lane);
  __syncthreads();
  float* dst = a.part + (static_cast<size_t>(bg) * a.nsplit + split) * a.G * (2 + D);
  for (int row = warp; row < a.G; row += kDecWarps) {
    float M, Lsum, wts[kDecWarps];
    merge_rows<D>(sm.part, kDecWarps, a.G, row, M, Lsum, wts);
    float* pr = dst + static_cast<size_t>(row) * (2 + D);
    if (lane == 0) {
      pr[0] = M;
      pr[1] = Lsum;
    }
    for (int c = lane; c < D; c += 32) {
      float acc = 0.f;
      for (int w = 0; w < kDecWarps; ++w) acc += sm.part[w].o[row][c] * wts[w];
      pr[2 + c] = acc;
    }
  }
}

// One CTA (256 threads) per (sequence, group).
template <int D>
__global__ void __launch_bounds__(256) dec_select_kernel(const int32_t* __restrict__ seq_lens, const DecArgs a,
                                                         int32_t* __restrict__ out_sel_idx) {
  extern __shared__ float ds_smem[];
  float* sc = ds_smem;                                        // [nsel_max]
  int* list = reinterpret_cast<int*>(sc + a.nsel_max);        // [nsel_max]
  uint32_t* bits = reinterpret_cast<uint32_t*>(list + a.nsel_max);  // [nsel_max/32 + 1]
  float* lse2 = reinterpret_cast<float*>(bits + a.nsel_max / 32 + 1);  // [G]
  const int bg = blockIdx.x, b = bg / a.hkv, g = bg % a.hkv;
  const int tid = threadIdx.x;
  const int L = seq_len_checked(seq_lens, b, a.lmax);
  const int t = L - 1;
  const int nc = (L >= a.cmp_len) ? (L - a.cmp_len) / a.cmp_stride + 1 : 0;
  const int jt = t / a.sel_len;
  const float* part = a.part + static_cast<size_t>(bg) * a.nsplit * a.G * (2 + D);
  // ---- merge split partials: o_cmp and the base-2 log-sum-exp per head
  for (int row = tid / 32; row < a.G; row += 8) {
    float M = -INFINITY;
    for (int s = 0; s < a.nsplit; ++s) M = fmaxf(M, part[(static_cast<size_t>(s) * a.G + row) * (2 + D)]);
    float Lsum = 0.f;
    for (int s = 0; s < a.nsplit; ++s) {
      const float* pr = part + (static_cast<size_t>(s) * a.G + row) * (2 + D);
      if (M != -INFINITY) Lsum += pr[1] * ex2_approx(pr[0] - M);
    }
    const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
    const int h = g * a.G + row;
    for (int c = tid % 32; c < D; c += 32) {
      float acc = 0.f;
      for (int s = 0; s < a.nsplit; ++s) {
        const float* pr = part + (static_cast<size_t>(s) * a.G + row) * (2 + D);
        if (M != -INFINITY) acc += pr[2 + c] * ex2_approx(pr[0] - M);
      }
      a.o_cmp[(static_cast<size_t>(b) * a.hq + h) * D + c] = acc * inv;
    }
    if (tid % 32 == 0) {
      lse2[row] = Lsum > 0.f ? M + __log2f(Lsum) : INFINITY;
      a.lse[static_cast<size_t>(b) * a.hq + h] = Lsum > 0.f ? (M + __log2f(Lsum)) * 0.69314718055994530942f : -INFINITY;
    }
  }
  __syncthreads();
  // ---- selection-block scores: compressed block i covers tokens [16i, 16i+32);
  // block j gets half of blocks 4j-1 and 4j+3 and all of 4j..4j+2.
  const float* lg = a.logits + static_cast<size_t>(bg) * a.G * a.ncmax;
  for (int j = tid; j <= jt; j += blockDim.x) {
    float acc = 0.f;
    for (int row = 0; row < a.G; ++row) {
      const float* lr = lg + static_cast<size_t>(row) * a.ncmax;
      const float l2 = lse2[row];
      auto p = [&](int i) -> float { return (i >= 0 && i < nc) ? ex2_approx(lr[i] - l2) : 0.f; };
      acc += 0.5f * p(4 * j - 1) + p(4 * j) + p(4 * j + 1) + p(4 * j + 2) + 0.5f * p(4 * j + 3);
    }
    sc[j] = acc;
    a.scores[static_cast<size_t>(bg) * a.nsel_max + j] = acc;
  }
  __syncthreads();
  if (tid < 32) {
    int32_t* d = a.sel_idx + static_cast<size_t>(bg) * a.top_n;
    int32_t* d2 = out_sel_idx ? out_sel_idx + static_cast<size_t>(bg) * a.top_n : nullptr;
    if (a.top_n > 32 || jt >= 32 * 64) warp_topn(sc, bits, list, sc, jt, a.top_n, d, d2, tid);
    else if (jt < 32 * 4) warp_topn_regs<4>(list, sc, jt, a.top_n, d, d2, tid);
    else if (jt < 32 * 16) warp_topn_regs<16>(list, sc, jt, a.top_n, d, d2, tid);
    else if (jt < 32 * 32) warp_topn_regs<32>(list, sc, jt, a.top_n, d, d2, tid);
    else warp_topn_regs<64>(list, sc, jt, a.top_n, d, d2, tid);
  }
}

// grid (B*hkv, 2): blockIdx.y = 0 -> selected blocks, 1 -> sliding window.
template <int D>
__global__ void __launch_bounds__(kDecWarps * 32) dec_branch_kernel(const __nv_bfloat16* __restrict__ q,
                                                                    const __nv_bfloat16* __restrict__ kcache,
                                                                    const __nv_bfloat16* __restrict__ vcache,
                                                                    const int32_t* __restrict__ seq_lens,
                                                                    const DecArgs a) {
  extern __shared__ uint8_t dec_smem_raw[];
  DecSmem<D>& sm = *reinterpret_cast<DecSmem<D>*>((reinterpret_cast<uintptr_t>(dec_smem_raw) + 127) & ~uintptr_t(127));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bg = blockIdx.x, b = bg / a.hkv, g = bg % a.hkv;
  const bool is_win = blockIdx.y == 1;
  const int L = seq_len_checked(seq_lens, b, a.lmax);
  const int t = L - 1;
  // chunk list (shared by the four warps; warp w takes chunks w, w+4, ...)
  int* list = sm.chunk_start[0];
  int nch;
  if (warp == 0) {
    if (is_win) {
      const int w0 = max(0, t - a.window + 1);
      nch = (t + 1 - w0 + kChunkKeys - 1) / kChunkKeys;
      if (nch > 128) nch = 128;  // window <= 4096 is validated on the host
      for (int ci = lane; ci < nch; ci += 32) list[ci] = w0 + ci * kChunkKeys;
      __syncwarp();
    } else {
      nch = build_chunk_list(a.sel_idx + static_cast<size_t>(bg) * a.top_n, a.top_n, a.sel_len, t, list, lane);
    }
    if (lane == 0) sm.chunk_start[1][0] = nch;
  }
  __syncthreads();
  nch = sm.chunk_start[1][0];
  const int key_lo = is_win ? max(0, t - a.window + 1) : 0;
  uint32_t qa[D / 16][4];
  load_q_frags<D>(qa, q + (static_cast<size_t>(b) * a.hq + g * a.G) * D, a.G, lane);
  const size_t rs = static_cast<size_t>(a.hkv) * D;
  const __nv_bfloat16* kb = kcache + static_cast<size_t>(b) * a.lmax * rs + static_cast<size_t>(g) * D;
  const __nv_bfloat16* vb = vcache + static_cast<size_t>(b) * a.lmax * rs + static_cast<size_t>(g) * D;
  auto& buf = sm.buf[warp];
  WarpAttnState<D> st;
  state_init(st);
  const int my = nch > warp ? (nch - warp + kDecWarps - 1) / kDecWarps : 0;
  if (my > 0) {
    load_chunk<D>(buf, 0, kb, vb, rs, list[warp], t + 1, lane);
    cp_async_commit();
  }
  for (int x = 0; x < my; ++x) {
    const int ci = warp + x * kDecWarps;
    if (x + 1 < my) {
      load_chunk<D>(buf, (x + 1) & 1, kb, vb, rs, list[ci + kDecWarps], t + 1, lane);
      cp_async_commit();
      cp_async_wait_1();
    } else {
      cp_async_wait_0();
    }
    __syncwarp();
    attend_chunk<D>(st, qa, buf, x & 1, list[ci], key_lo, t + 1, a.sl2, lane);
    __syncwarp();
  }
  state_reduce_l(st);
  state_store(st, sm.part[warp], lane);
  __syncthreads();
  float* dst = (is_win ? a.o_win : a.o_sel) + (static_cast<size_t>(b) * a.hq + g * a.G) * D;
  for (int row = warp; row < a.G; row += kDecWarps) {
    float M, Lsum, wts[kDecWarps];
    merge_rows<D>(sm.part, kDecWarps, a.G, row, M, Lsum, wts);
    const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
    for (int c = lane; c < D; c += 32) {
      float acc = 0.f;
      for (int w = 0; w < kDecWarps; ++w) acc += sm.part[w].o[row][c] * wts[w];
      dst[static_cast<size_t>(row) * D + c] = acc * inv;
    }
  }
}

__global__ void __launch_bounds__(256) dec_combine_kernel(const float* __restrict__ gates, const float* __restrict__ o_cmp,
                                                          const float* __restrict__ o_sel,
                                                          const float* __restrict__ o_win, void* __restrict__ out,
                                                          int out_f32, int rows, int d) {
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= static_cast<long long>(rows) * d) return;
  const long long row = i / d;
  const float v = gates[row * 3 + 0] * o_cmp[i] + gates[row * 3 + 1] * o_sel[i] + gates[row * 3 + 2] * o_win[i];
  if (out_f32)
    static_cast<float*>(out)[i] = v;
  else
    static_cast<__nv_bfloat16*>(out)[i] = __float2bfloat16_rn(v);
}

}  // namespace nsa
