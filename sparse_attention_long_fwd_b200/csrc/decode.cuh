// decode.cuh -- single-query NSA decode against a KV cache and a compressed cache.
//
// Per sequence b (query at t = L_b - 1) and KV group g the same three branches as the
// prefill are evaluated for one token (top168.com article on VideoNSA, section
// "一、革命性的三重注意机制"). With one query the work is a stream over the caches, so it
// is HBM-bound and split four ways:
//   dec_cmp_kernel      split-K over the compressed cache: each CTA attends to a slice of
//                       the visible blocks, keeps its base-2 logits for the scoring step
//                       and writes a partial (max, sum, unnormalised output) per head; one
//                       more CTA per (sequence, group) runs the sliding-window branch, which
//                       needs no selection, beside the compressed stream;
//   dec_select_kernel   merges the partials into o_cmp and the row log-sum-exp, turns
//                       the stored logits into selection-block scores summed over the
//                       group, and picks the top-n blocks (topn.cuh);
//   dec_branch_kernel   the selected-block branch, one CTA per (sequence, group), four
//                       warps splitting the key chunks, then the gated combine
//                       out = g_cmp*o_cmp + g_sel*o_sel + g_win*o_win of the group's heads.
#pragma once
#include "sel.cuh"
#include "topn.cuh"

namespace nsa {

constexpr int kDecWarps = 4;
// Cache keys per chunk and chunks in flight per warp: 16-key chunks in a 3-stage ring keep
// two chunks loading while one is used, in 24 KB per warp (d = 128), so two CTAs fit an SM.
constexpr int kDecChunk = 16;
constexpr int kDecStages = 3;

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
  int lstride;          // floats between logit rows: ncmax rounded up to 4 (16-byte rows)
  float* logits;        // [B][hkv][G][lstride] base-2 scaled logits of the compressed branch
  float* part;          // [B][hkv][nsplit][G][2 + D] (m, l, o[D])
  float* o_cmp;         // [B][hq][D]
  float* lse;           // [B][hq] natural log
  float* scores;        // [B][hkv][nsel_max]
  int32_t* sel_idx;     // [B][hkv][top_n]
  float* o_win;         // [B][hq][D]
  const float* gates;   // [B][hq][3]
  void* out;            // [B][hq][D]
  int out_f32;
};

template <int D>
struct DecSmem {
  union {
    WarpChunkBuf<D, kDecChunk, kDecStages> buf[kDecWarps];
    WarpPartial<D> part[kDecWarps];  // after the last chunk: the warps' partial states
  };
  int chunk_start[512];  // chunk list of the branch kernel (flat)
};
static_assert(sizeof(WarpPartial<128>) * kDecWarps <= sizeof(WarpChunkBuf<128, kDecChunk, kDecStages>) * kDecWarps,
              "partials alias the chunk ring");

// Stream `nch` chunks through the warp's ring (kDecStages - 1 in flight), calling
// use(stage, ci) on each in order; load(stage, ci) issues chunk ci's cp.async copies.
template <typename Load, typename Use>
__device__ __forceinline__ void dec_stream(int nch, Load&& load, Use&& use) {
#pragma unroll
  for (int c = 0; c < kDecStages - 1; ++c) {
    if (c < nch) load(c, c);
    cp_async_commit();
  }
  for (int ci = 0; ci < nch; ++ci) {
    const int cn = ci + kDecStages - 1;
    if (cn < nch) load(cn % kDecStages, cn);
    cp_async_commit();  // (possibly empty: keeps the group count uniform)
    asm volatile("cp.async.wait_group %0;" ::"n"(kDecStages - 1) : "memory");
    __syncwarp();
    use(ci % kDecStages, ci);
    __syncwarp();
  }
}

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

// Programmatic dependent launch: a kernel lets the next one in the stream be launched
// while it runs (its CTAs then wait, resident, in grid_dependency_wait until this grid has
// finished and its writes are visible), so the launch gap between the decode's kernels is
// hidden.
__device__ __forceinline__ void grid_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// One (sequence, group)'s selected-block (is_win false) or sliding-window (is_win true)
// branch: the four warps split the key chunks, then merge; each normalised output value
// goes to f(row, c, value) for the lane's columns c.
template <int D, typename F>
__device__ __forceinline__ void dec_branch_body(DecSmem<D>& sm, const __nv_bfloat16* __restrict__ q,
                                                const __nv_bfloat16* __restrict__ kcache,
                                                const __nv_bfloat16* __restrict__ vcache, const DecArgs& a, int b,
                                                int g, int L, bool is_win, F&& f) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bg = b * a.hkv + g;
  const int t = L - 1;
  // chunk list (shared by the four warps; warp w takes chunks w, w+4, ...); its last entry
  // holds the count
  int* list = sm.chunk_start;
  int nch;
  if (warp == 0) {
    if (is_win) {
      const int w0 = max(0, t - a.window + 1);
      nch = (t + 1 - w0 + kDecChunk - 1) / kDecChunk;
      if (nch > 511) nch = 511;  // window <= 4096 is validated on the host
      for (int ci = lane; ci < nch; ci += 32) list[ci] = w0 + ci * kDecChunk;
      __syncwarp();
    } else {
      // (top_n * sel_len / kDecChunk <= 511 entries for the validated sizes)
      nch = build_chunk_list(a.sel_idx + static_cast<size_t>(bg) * a.top_n, a.top_n, a.sel_len, t, list, lane,
                             kDecChunk);
    }
    if (lane == 0) sm.chunk_start[511] = nch;
  }
  __syncthreads();
  nch = sm.chunk_start[511];
  const int key_lo = is_win ? max(0, t - a.window + 1) : 0;
  uint32_t qa[D / 16][4];
  load_q_frags<D>(qa, q + (static_cast<size_t>(b) * a.hq + g * a.G) * D, a.G, lane);
  const size_t rs = static_cast<size_t>(a.hkv) * D;
  const __nv_bfloat16* kb = kcache + static_cast<size_t>(b) * a.lmax * rs + static_cast<size_t>(g) * D;
  const __nv_bfloat16* vb = vcache + static_cast<size_t>(b) * a.lmax * rs + static_cast<size_t>(g) * D;
  auto& buf = sm.buf[warp];
  const uint64_t pol = l2_evict_first_policy();  // the cache rows are read once per step
  WarpAttnState<D> st;
  state_init(st);
  const int my = nch > warp ? (nch - warp + kDecWarps - 1) / kDecWarps : 0;
  dec_stream(
      my,
      [&](int stg, int x) { load_chunk<D>(buf, stg, kb, vb, rs, list[warp + x * kDecWarps], t + 1, lane, pol); },
      [&](int stg, int x) { attend_chunk<D>(st, qa, buf, stg, list[warp + x * kDecWarps], key_lo, t + 1, a.sl2, lane); });
  state_reduce_l(st);
  cp_async_wait_0();
  __syncthreads();  // every warp is done with the ring: the partials take its place
  state_store(st, sm.part[warp], lane);
  __syncthreads();
  for (int row = warp; row < a.G; row += kDecWarps) {
    float M, Lsum, wts[kDecWarps];
    merge_rows<D>(sm.part, kDecWarps, a.G, row, M, Lsum, wts);
    const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
    // (unrolled: the callback's global loads for all of the lane's columns go out together)
#pragma unroll
    for (int c = lane; c < D; c += 32) {
      float acc = 0.f;
#pragma unroll
      for (int w = 0; w < kDecWarps; ++w) acc += sm.part[w].o[row][c] * wts[w];
      f(row, c, acc * inv);
    }
  }
}

template <int D>
__global__ void __launch_bounds__(kDecWarps * 32) dec_cmp_kernel(const __nv_bfloat16* __restrict__ q,
                                                                 const __nv_bfloat16* __restrict__ kcmp,
                                                                 const __nv_bfloat16* __restrict__ vcmp,
                                                                 const __nv_bfloat16* __restrict__ kcache,
                                                                 const __nv_bfloat16* __restrict__ vcache,
                                                                 const int32_t* __restrict__ seq_lens,
                                                                 const DecArgs a) {
  extern __shared__ uint8_t dec_smem_raw[];
  DecSmem<D>& sm = *reinterpret_cast<DecSmem<D>*>((reinterpret_cast<uintptr_t>(dec_smem_raw) + 127) & ~uintptr_t(127));
  grid_launch_dependents();  // dec_select_kernel may take free slots and wait there
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bg = blockIdx.y, b = bg / a.hkv, g = bg % a.hkv, split = blockIdx.x;
  const int L = seq_len_checked(seq_lens, b, a.lmax);
  if (split == a.nsplit) {  // the window branch of (sequence, group)
    float* dst = a.o_win + (static_cast<size_t>(b) * a.hq + g * a.G) * D;
    dec_branch_body<D>(sm, q, kcache, vcache, a, b, g, L, true,
                       [&](int row, int c, float v) { dst[static_cast<size_t>(row) * D + c] = v; });
    return;
  }
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
  float* lg = a.logits + static_cast<size_t>(bg) * a.G * a.lstride;
  auto& buf = sm.buf[warp];
  // the compressed cache is read once per step: its lines go first, so the logits and partials
  // this grid writes are still in L2 for dec_select_kernel
  const uint64_t pol = l2_evict_first_policy();
  WarpAttnState<D> st;
  state_init(st);
  const int nch = w1 > w0 ? (w1 - w0 + kDecChunk - 1) / kDecChunk : 0;
  dec_stream(
      nch, [&](int stg, int ci) { load_chunk<D>(buf, stg, kb, vb, rs, w0 + ci * kDecChunk, w1, lane, pol); },
      [&](int stg, int ci) {
        attend_chunk<D>(st, qa, buf, stg, w0 + ci * kDecChunk, w0, w1, a.sl2, lane, lg, a.lstride, 0, a.G);
      });
  state_reduce_l(st);
  cp_async_wait_0();
  __syncthreads();  // every warp is done with the ring: the partials take its place
  state_store(st, sm.part[warp], lane);
  __syncthreads();
  float* dst = a.part + (static_cast<size_t>(bg) * a.nsplit + split) * a.G * (2 + D);
  const uint64_t keep = l2_evict_last_policy();  // dec_select_kernel reads the partials back
  for (int row = warp; row < a.G; row += kDecWarps) {
    float M, Lsum, wts[kDecWarps];
    merge_rows<D>(sm.part, kDecWarps, a.G, row, M, Lsum, wts);
    float* pr = dst + static_cast<size_t>(row) * (2 + D);
    if (lane == 0) {
      st_f32_hint(pr, M, keep);
      st_f32_hint(pr + 1, Lsum, keep);
    }
#pragma unroll
    for (int c = lane; c < D; c += 32) {
      float acc = 0.f;
#pragma unroll
      for (int w = 0; w < kDecWarps; ++w) acc += sm.part[w].o[row][c] * wts[w];
      st_f32_hint(pr + 2 + c, acc, keep);
    }
  }
}

// One CTA (256 threads) per (sequence, group); two CTAs per SM, so the 64 x 4 (sequence,
// group) pairs of a full batch run as one wave on 148 SMs.
template <int D>
__global__ void __launch_bounds__(256, 2) dec_select_kernel(const int32_t* __restrict__ seq_lens, const DecArgs a,
                                                         int32_t* __restrict__ out_sel_idx) {
  grid_dependency_wait();  // dec_cmp_kernel's partials and logits
  grid_launch_dependents();
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
  // ---- merge split partials: o_cmp and the base-2 log-sum-exp per head. A warp per head
  // row: lane s holds split s (and s + 32), so the (max, sum) loads go out together, and the
  // output columns' loads are unrolled over the splits.
  const int lane = tid & 31;
  for (int row = tid / 32; row < a.G; row += 8) {
    auto ml = [&](int s, int k) -> float {
      return s < a.nsplit ? part[(static_cast<size_t>(s) * a.G + row) * (2 + D) + k] : (k == 0 ? -INFINITY : 0.f);
    };
    const float m0 = ml(lane, 0), l0 = ml(lane, 1), m1 = ml(lane + 32, 0), l1 = ml(lane + 32, 1);
    float M = fmaxf(m0, m1);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    const float w0 = (M == -INFINITY || m0 == -INFINITY) ? 0.f : ex2_approx(m0 - M);
    const float w1 = (M == -INFINITY || m1 == -INFINITY) ? 0.f : ex2_approx(m1 - M);
    float Lsum = l0 * w0 + l1 * w1;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) Lsum += __shfl_xor_sync(0xffffffffu, Lsum, o);
    const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
    const int h = g * a.G + row;
    constexpr int kPer = D / 32;
    float acc[kPer];
#pragma unroll
    for (int k = 0; k < kPer; ++k) acc[k] = 0.f;
    // (the split loop unrolled 16-wide: its loads go out together)
    for (int s0 = 0; s0 < a.nsplit; s0 += 16) {
#pragma unroll
      for (int s = s0; s < s0 + 16; ++s) {
        const float w = __shfl_sync(0xffffffffu, s < 32 ? w0 : w1, s & 31);
        if (s < a.nsplit) {
          const float* pr = part + (static_cast<size_t>(s) * a.G + row) * (2 + D) + 2;
#pragma unroll
          for (int k = 0; k < kPer; ++k) acc[k] += w * pr[lane + 32 * k];
        }
      }
    }
#pragma unroll
    for (int k = 0; k < kPer; ++k) a.o_cmp[(static_cast<size_t>(b) * a.hq + h) * D + lane + 32 * k] = acc[k] * inv;
    if (lane == 0) {
      lse2[row] = Lsum > 0.f ? M + __log2f(Lsum) : INFINITY;
      a.lse[static_cast<size_t>(b) * a.hq + h] = Lsum > 0.f ? (M + __log2f(Lsum)) * 0.69314718055994530942f : -INFINITY;
    }
  }
  __syncthreads();
  // ---- selection-block scores: compressed block i covers tokens [16i, 16i+32);
  // block j gets half of blocks 4j-1 and 4j+3 and all of 4j..4j+2. Thread tid takes the 8
  // blocks j0 .. j0+7 (j0 = 8 tid + 2048 pass): per head row it needs compressed blocks
  // 4 j0 - 1 .. 4 j0 + 31, read as 8 aligned float4 and one scalar, and the next row's loads
  // are issued before this row is binned, so a row costs about one load latency.
  {
    const float* lg = a.logits + static_cast<size_t>(bg) * a.G * a.lstride;
    for (int j0 = 8 * tid; j0 <= jt; j0 += 8 * 256) {  // (uniform trip count per warp is not needed)
      const int i0 = 4 * j0;  // first of the 32 aligned values
      float4 cur[8], nxt[8];
      float hcur = 0.f, hnxt = 0.f;
      auto load = [&](int row, float4 (&v)[8], float& halo) {
        const float* lr = lg + static_cast<size_t>(row) * a.lstride;
#pragma unroll
        for (int k = 0; k < 8; ++k)
          v[k] = (i0 + 4 * k < nc) ? *reinterpret_cast<const float4*>(lr + i0 + 4 * k)
                                   : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
        halo = (i0 >= 1 && i0 - 1 < nc) ? lr[i0 - 1] : -INFINITY;
      };
      float acc[8];
#pragma unroll
      for (int b2 = 0; b2 < 8; ++b2) acc[b2] = 0.f;
      load(0, cur, hcur);
      for (int row = 0; row < a.G; ++row) {
        if (row + 1 < a.G) load(row + 1, nxt, hnxt);
        const float l2 = lse2[row];
        float p[33];
        p[0] = i0 >= 1 && i0 - 1 < nc ? ex2_approx(hcur - l2) : 0.f;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float x[4] = {cur[k].x, cur[k].y, cur[k].z, cur[k].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) p[1 + 4 * k + e] = (i0 + 4 * k + e < nc) ? ex2_approx(x[e] - l2) : 0.f;
        }
#pragma unroll
        for (int b2 = 0; b2 < 8; ++b2)
          acc[b2] += 0.5f * p[4 * b2] + p[4 * b2 + 1] + p[4 * b2 + 2] + p[4 * b2 + 3] + 0.5f * p[4 * b2 + 4];
#pragma unroll
        for (int k = 0; k < 8; ++k) cur[k] = nxt[k];
        hcur = hnxt;
      }
#pragma unroll
      for (int b2 = 0; b2 < 8; ++b2) {
        const int j = j0 + b2;
        if (j <= jt) {
          sc[j] = acc[b2];
          a.scores[static_cast<size_t>(bg) * a.nsel_max + j] = acc[b2];
        }
      }
    }
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

// One CTA per (sequence, group): the selected-block branch, then the gated combine of the
// group's heads (o_cmp from dec_select_kernel, o_win from dec_cmp_kernel's window CTAs).
template <int D>
__global__ void __launch_bounds__(kDecWarps * 32) dec_branch_kernel(const __nv_bfloat16* __restrict__ q,
                                                                    const __nv_bfloat16* __restrict__ kcache,
                                                                    const __nv_bfloat16* __restrict__ vcache,
                                                                    const int32_t* __restrict__ seq_lens,
                                                                    const DecArgs a) {
  extern __shared__ uint8_t dec_smem_raw[];
  DecSmem<D>& sm = *reinterpret_cast<DecSmem<D>*>((reinterpret_cast<uintptr_t>(dec_smem_raw) + 127) & ~uintptr_t(127));
  const int bg = blockIdx.x, b = bg / a.hkv, g = bg % a.hkv;
  grid_dependency_wait();  // dec_select_kernel's selection and o_cmp (and, before it, o_win)
  const int L = seq_len_checked(seq_lens, b, a.lmax);
  const size_t row0 = static_cast<size_t>(b) * a.hq + g * a.G;
  dec_branch_body<D>(sm, q, kcache, vcache, a, b, g, L, false, [&](int row, int c, float v) {
    const size_t r = row0 + row;
    const size_t e = r * D + c;
    const float o = __ldg(a.gates + r * 3 + 0) * __ldcg(a.o_cmp + e) + __ldg(a.gates + r * 3 + 1) * v +
                    __ldg(a.gates + r * 3 + 2) * __ldcg(a.o_win + e);
    if (a.out_f32)
      static_cast<float*>(a.out)[e] = o;
    else
      static_cast<__nv_bfloat16*>(a.out)[e] = __float2bfloat16_rn(o);
  });
}

}  // namespace nsa
