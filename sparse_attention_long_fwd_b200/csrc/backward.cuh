// backward.cuh -- gradients of the NSA prefill: dq, dk, dv and the gates' gradient.
//
// The pages train the model end to end (shd-paper.top page "VideoNSA: Native Sparse
// Attention Scales Video Understanding", abstract); this is the backward of the forward in
// this library, with the selection held constant (block indices carry no gradient) and the
// compressed keys' gradient returned to their tokens with the compression's weights. For a
// row (token t, head h) and a branch b with gate g_b:
//   P = softmax(scale K_b q), o_b = P V_b;  d g_b = <dO, o_b>
//   dS_j = g_b P_j (<dO, v_j> - <dO, o_b>);  dq += scale sum_j dS_j k_j
//   dk_j += scale dS_j q;  dv_j += g_b P_j dO
// Text rows (t >= n_video) are one dense branch with gate 1.
//
// Three passes, all on warp-level mma.sync tiles (m16n8k16, bf16 in, fp32 accumulate):
//   bwd_row_kernel   one warp per (two adjacent tokens, group) when a group has at most
//                    8 heads (else one token): the heads are the rows of a 16-row tile.
//                    Per branch: pass A streams the keys once for each row's log-sum-exp
//                    and o_b, giving <dO, o_b> (the gate gradient); pass B streams them
//                    again for dS and dq += dS K. Writes dq, the gate gradient and
//                    (lse, <dO, o_b>) per (row, branch) for the next pass. Given the
//                    forward's saved log-sum-exp and output of the compressed branch,
//                    that branch skips pass A.
//   bwd_key_kernel   one warp per (branch, 16-key tile, group, segment of the rows that
//                    attend those keys): S^T = K Q^T and dP^T = V dO^T for 16 rows at a
//                    time, then dv += P^T dO and dk += dS^T Q in registers; the sums are
//                    added to dk / dv (or to the compressed keys' gradient) once per item.
//                    The selected branch takes its rows from the (group, block) buckets.
//   pool_bwd_kernel  the compressed keys' gradient back to the tokens of each block.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "warp_attn.cuh"

namespace nsa {

constexpr int kBwdChunk = 16;     // keys per chunk (row pass) and rows per chunk (key pass)
constexpr int kBwdWarps = 4;      // warps per CTA in both passes
constexpr int kBwdSegCmp = 1024;  // tokens per item of the compressed branch's key pass
constexpr int kBwdSegSel = 256;   // bucket entries per item of the selected branch's key pass
constexpr int kBwdSegDense = 1024;

enum BwdBranch { kBwdCmp = 0, kBwdSel = 1, kBwdWin = 2, kBwdDense = 3 };

struct BwdArgs {
  int N, nv, hq, hkv, G, ncmp, nsel, top_n, cmp_len, cmp_stride, sel_len, window;
  float scale, sl2;
  const __nv_bfloat16* q;     // [N][hq][D]
  const __nv_bfloat16* k;     // [N][hkv][D]
  const __nv_bfloat16* v;
  const __nv_bfloat16* kc;    // [ncmp][hkv][D] compressed keys and values of the forward
  const __nv_bfloat16* vc;
  const __nv_bfloat16* dout;  // [N][hq][D]
  const float* gates;         // [N][hq][3]
  const int32_t* sel_idx;     // [nv][hkv][top_n], ascending, -1 padded
  float2* stats;              // [N][hq][3]: (log2-sum-exp of the scaled base-2 logits, <dO, o_b>)
  float* dq;                  // [N][hq][D]
  float* dk;                  // [N][hkv][D], zeroed by the host
  float* dv;
  float* dkc;                 // [ncmp][hkv][D], zeroed by the host
  float* dvc;
  float* dgates;              // [N][hq][3]
  const int* ent_off;         // selected-branch buckets: [hkv*nsel + 1] entry offsets
  const int* seg_off;         // [hkv*nsel + 1] segment offsets (ceil(count / kBwdSegSel))
  const int* list;            // bucketed entries t * 64 + slot
  const float* fwd_lse;       // [nv][hq] the forward's compressed-branch log-sum-exp (natural log),
  const __half* fwd_ocmp;     // [nv][hq][D] and its output, or both null: pass A recomputes them
  int cmp_rows_done;          // 1: the video rows' compressed-branch dq, statistics and gate gradient
                              // are already written; the row pass adds the other branches to dq
  // kept by the forward (nsa_params_t.keep_branch_stats), else null
  const float* fwd_lse_sel;   // [nv][hq] natural log
  const __half* fwd_osel;     // [nv][hq][D]
  const float* fwd_lse_win;   // [nv][hq] natural log
  const __half* fwd_owin;     // [nv][hq][D]
  int video_rows_done;        // 1: the tensor-core kernels write every video row; the row pass
                              // takes the text rows only
  const int* row_of;          // [nv][hkv][top_n] first partial row of each (token, group, slot)
  __half* dq_part;            // [part rows][D] the selected branch's dq per (row, block), fp16
  float2* part_scale;         // [part rows] the factor of each 64-column half of a partial row
};

// ---------------------------------------------------------------- row pass
// A warp's 16 MMA rows: thread rows lane/4 (half 0) and lane/4 + 8 (half 1). With G <= 8 a
// warp takes two adjacent tokens of the same kind (half 0: token A's heads, half 1: token
// B's), so 2G of the 16 rows do work; with G > 8 it takes one token (half 1: heads 8..G-1).
// Keys are masked per half: adjacent tokens differ in their last compressed block, their
// window and their selection, and attend the union with their own ranges.

struct ChunkDesc {
  int start, row_end;  // keys start .. start+15 are loaded where < row_end
  int lo[2], hi[2];    // key range of each half
};

// Streams `nch` chunks of keys from (kb, vb) through the warp's two-stage ring.
template <int D, class Desc, class Use>
__device__ __forceinline__ void bwd_stream(WarpChunkBuf<D, kBwdChunk, 2>& buf, const __nv_bfloat16* kb,
                                           const __nv_bfloat16* vb, size_t stride, int nch, Desc desc, Use use,
                                           int lane) {
  if (nch <= 0) return;
  {
    const ChunkDesc d0 = desc(0);
    load_chunk<D, kBwdChunk, 2>(buf, 0, kb, vb, stride, d0.start, d0.row_end, lane);
  }
  cp_async_commit();
  for (int c = 0; c < nch; ++c) {
    if (c + 1 < nch) {
      const ChunkDesc dn = desc(c + 1);
      load_chunk<D, kBwdChunk, 2>(buf, (c + 1) & 1, kb, vb, stride, dn.start, dn.row_end, lane);
    }
    cp_async_commit();
    cp_async_wait_1();
    __syncwarp();
    use(c & 1, desc(c));
    __syncwarp();  // every lane is done with this stage before it is refilled
  }
  cp_async_wait_0();
}

// A fragments of the 16 rows: half 0 from row pointer p0, half 1 from p1 (null: zero).
template <int D>
__device__ __forceinline__ void bwd_load_frags(uint32_t (&a)[D / 16][4], const __nv_bfloat16* p0,
                                               const __nv_bfloat16* p1, int lane) {
  const int c = 2 * (lane & 3);
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks) {
    const int col = ks * 16 + c;
    a[ks][0] = p0 ? *reinterpret_cast<const uint32_t*>(p0 + col) : 0u;
    a[ks][1] = p1 ? *reinterpret_cast<const uint32_t*>(p1 + col) : 0u;
    a[ks][2] = p0 ? *reinterpret_cast<const uint32_t*>(p0 + col + 8) : 0u;
    a[ks][3] = p1 ? *reinterpret_cast<const uint32_t*>(p1 + col + 8) : 0u;
  }
}

// Pass A on one chunk: online softmax over the chunk's keys (per-half ranges), O += P V.
template <int D>
__device__ __forceinline__ void bwd_attend_chunk(WarpAttnState<D>& s, const uint32_t (&qa)[D / 16][4],
                                                 const WarpChunkBuf<D, kBwdChunk, 2>& buf, int st,
                                                 const ChunkDesc& cd, float sl2, int lane) {
  constexpr int NT = kBwdChunk / 8;
  const uint32_t kaddr = smem_u32(&buf.kv[st][0][0]);
  const uint32_t vaddr = smem_u32(&buf.kv[st][1][0]);
  float sc[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
    for (int ks = 0; ks < D / 16; ks += 2) {
      const int row = nt * 8 + (lane & 7);
      const int unit = ks * 2 + (lane >> 3);
      uint32_t b0, b1, b2, b3;
      ldsm_x4(kaddr + (row * D + swz_unit(row, unit) * 8) * 2, b0, b1, b2, b3);
      mma_bf16_16816(sc[nt], qa[ks], b0, b1);
      mma_bf16_16816(sc[nt], qa[ks + 1], b2, b3);
    }
  }
  float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int r = e >> 1;
      const int key = cd.start + nt * 8 + 2 * (lane & 3) + (e & 1);
      const float z = (key >= cd.lo[r] && key < cd.hi[r]) ? sc[nt][e] * sl2 : -INFINITY;
      sc[nt][e] = z;
      mx[r] = fmaxf(mx[r], z);
    }
  }
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
    mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
  }
  float alpha[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const float mnew = fmaxf(s.m[r], mx[r]);
    alpha[r] = (mnew == -INFINITY) ? 1.f : ex2_approx(s.m[r] - mnew);
    s.m[r] = mnew;
  }
  s.l[0] *= alpha[0];
  s.l[1] *= alpha[1];
  uint32_t pa[4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    float p[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float mr = s.m[e >> 1];
      p[e] = (mr == -INFINITY) ? 0.f : ex2_approx(sc[nt][e] - mr);
    }
    s.l[0] += p[0] + p[1];
    s.l[1] += p[2] + p[3];
    pa[nt * 2 + 0] = pack_bf16x2(p[0], p[1]);
    pa[nt * 2 + 1] = pack_bf16x2(p[2], p[3]);
  }
#pragma unroll
  for (int n = 0; n < D / 8; ++n) {
    s.o[n][0] *= alpha[0];
    s.o[n][1] *= alpha[0];
    s.o[n][2] *= alpha[1];
    s.o[n][3] *= alpha[1];
  }
#pragma unroll
  for (int n = 0; n < D / 8; n += 2) {
    const int row = (lane & 7) + ((lane >> 3) & 1) * 8;
    const int unit = n + (lane >> 4);
    uint32_t b0, b1, b2, b3;
    ldsm_x4_t(vaddr + (row * D + swz_unit(row, unit) * 8) * 2, b0, b1, b2, b3);
    mma_bf16_16816(s.o[n], pa, b0, b1);
    mma_bf16_16816(s.o[n + 1], pa, b2, b3);
  }
}

// Pass B on one chunk: S = Q K^T, dP = dO V^T, dS = gs * P * (dP - dg), dq += dS K.
template <int D>
__device__ __forceinline__ void bwd_dq_chunk(float (&dq)[D / 8][4], const uint32_t (&qa)[D / 16][4],
                                             const uint32_t (&da)[D / 16][4],
                                             const WarpChunkBuf<D, kBwdChunk, 2>& buf, int st, const ChunkDesc& cd,
                                             float sl2, const float (&lse2)[2], const float (&dg)[2],
                                             const float (&gs)[2], int lane) {
  constexpr int NT = kBwdChunk / 8;
  const uint32_t kaddr = smem_u32(&buf.kv[st][0][0]);
  const uint32_t vaddr = smem_u32(&buf.kv[st][1][0]);
  float sc[NT][4], dp[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) sc[nt][e] = dp[nt][e] = 0.f;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
    for (int ks = 0; ks < D / 16; ks += 2) {
      const int row = nt * 8 + (lane & 7);
      const int unit = ks * 2 + (lane >> 3);
      const uint32_t off = (row * D + swz_unit(row, unit) * 8) * 2;
      uint32_t b0, b1, b2, b3;
      ldsm_x4(kaddr + off, b0, b1, b2, b3);
      mma_bf16_16816(sc[nt], qa[ks], b0, b1);
      mma_bf16_16816(sc[nt], qa[ks + 1], b2, b3);
      ldsm_x4(vaddr + off, b0, b1, b2, b3);
      mma_bf16_16816(dp[nt], da[ks], b0, b1);
      mma_bf16_16816(dp[nt], da[ks + 1], b2, b3);
    }
  }
  uint32_t sa[4];  // dS as the A operand of one 16-key k-step
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    float ds[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int r = e >> 1;
      const int key = cd.start + nt * 8 + 2 * (lane & 3) + (e & 1);
      const bool ok = key >= cd.lo[r] && key < cd.hi[r] && lse2[r] != -INFINITY;
      const float p = ok ? ex2_approx(sc[nt][e] * sl2 - lse2[r]) : 0.f;
      ds[e] = gs[r] * p * (dp[nt][e] - dg[r]);
    }
    sa[nt * 2 + 0] = pack_bf16x2(ds[0], ds[1]);
    sa[nt * 2 + 1] = pack_bf16x2(ds[2], ds[3]);
  }
#pragma unroll
  for (int n = 0; n < D / 8; n += 2) {
    const int row = (lane & 7) + ((lane >> 3) & 1) * 8;
    const int unit = n + (lane >> 4);
    uint32_t b0, b1, b2, b3;
    ldsm_x4_t(kaddr + (row * D + swz_unit(row, unit) * 8) * 2, b0, b1, b2, b3);
    mma_bf16_16816(dq[n], sa, b0, b1);
    mma_bf16_16816(dq[n + 1], sa, b2, b3);
  }
}

// <dO, o / l> of the two rows this thread holds (half r from dO row pointer p[r]), reduced
// over the quad.
template <int D>
__device__ __forceinline__ void bwd_row_dot(const WarpAttnState<D>& s, const __nv_bfloat16* const (&p)[2],
                                            int lane, float (&dg)[2]) {
  const int c = 2 * (lane & 3);
  float part[2] = {0.f, 0.f};
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    if (p[r] == nullptr) continue;
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
      const float2 d = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p[r] + n * 8 + c));
      part[r] += s.o[n][2 * r] * d.x + s.o[n][2 * r + 1] * d.y;
    }
  }
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    part[r] += __shfl_xor_sync(0xffffffffu, part[r], 1);
    part[r] += __shfl_xor_sync(0xffffffffu, part[r], 2);
    dg[r] = s.l[r] > 0.f ? part[r] / s.l[r] : 0.f;
  }
}

template <int D>
struct BwdRowSmem {
  WarpChunkBuf<D, kBwdChunk, 2> buf;
  int2 blocks[128];  // the union of the tokens' selected blocks: (block, mask of the halves)
};

template <int D>
__global__ void __launch_bounds__(32 * kBwdWarps) bwd_row_kernel(const BwdArgs a) {
  extern __shared__ __align__(128) uint8_t bwd_row_smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto& sm = reinterpret_cast<BwdRowSmem<D>*>(bwd_row_smem)[warp];
  const int G = a.G;
  const int tpw = G <= 8 ? 2 : 1;  // tokens per warp
  const int nv_items = (a.nv + tpw - 1) / tpw;
  const int nt_items = (a.N - a.nv + tpw - 1) / tpw;
  const long long item = static_cast<long long>(blockIdx.x) * kBwdWarps + warp;
  if (item >= static_cast<long long>(nv_items + nt_items) * a.hkv) return;  // warp-uniform, no CTA barrier follows
  const int g = static_cast<int>(item % a.hkv);
  const int pi = static_cast<int>(item / a.hkv);
  const bool video = pi < nv_items;
  if (video && a.video_rows_done) return;  // warp-uniform
  const int t_end = video ? a.nv : a.N;
  const int tA = video ? pi * tpw : a.nv + (pi - nv_items) * tpw;
  const int h0 = g * G;
  const int r0 = lane >> 2;
  // the two halves: token, head and validity
  int tok[2], head[2];
  bool ok[2];
  if (tpw == 2) {
    tok[0] = tA;
    tok[1] = tA + 1;
    head[0] = head[1] = r0;
    ok[0] = r0 < G;
    ok[1] = r0 < G && tA + 1 < t_end;
  } else {
    tok[0] = tok[1] = tA;
    head[0] = r0;
    head[1] = r0 + 8;
    ok[0] = r0 < G;
    ok[1] = r0 + 8 < G;
  }
  const bool has_b = tpw == 2 ? (tA + 1 < t_end) : true;  // warp-uniform: half 1 exists at all
  const int tB = tpw == 2 ? (has_b ? tA + 1 : tA) : tA;   // the later token of the warp
  const __nv_bfloat16* qp[2];
  const __nv_bfloat16* dp[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const size_t row = (static_cast<size_t>(tok[r]) * a.hq + h0 + head[r]) * D;
    qp[r] = ok[r] ? a.q + row : nullptr;
    dp[r] = ok[r] ? a.dout + row : nullptr;
  }
  const size_t kv_stride = static_cast<size_t>(a.hkv) * D;
  uint32_t qa[D / 16][4];
  bwd_load_frags<D>(qa, qp[0], qp[1], lane);
  float dq[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n) dq[n][0] = dq[n][1] = dq[n][2] = dq[n][3] = 0.f;
  const int nb = video ? 3 : 1;
  // token of each half for the key ranges (a missing token B takes A's ranges, masked off by gs = 0)
  const int tk[2] = {tok[0], tpw == 2 ? tB : tok[1]};
  int nblk = 0;
  if (video) {
    // the union of the tokens' selected blocks, ascending, with the halves that chose each
    if (lane == 0) {
      const int32_t* sa_ = a.sel_idx + (static_cast<size_t>(tk[0]) * a.hkv + g) * a.top_n;
      const int32_t* sb_ = a.sel_idx + (static_cast<size_t>(tk[1]) * a.hkv + g) * a.top_n;
      int ia = 0, ib = 0;
      while (true) {
        const int ja = ia < a.top_n ? sa_[ia] : -1;
        const int jb = ib < a.top_n ? sb_[ib] : -1;
        if (ja < 0 && jb < 0) break;
        int j, mask;
        if (jb < 0 || (ja >= 0 && ja < jb)) {
          j = ja;
          mask = 1;
          ++ia;
        } else if (ja < 0 || jb < ja) {
          j = jb;
          mask = 2;
          ++ib;
        } else {
          j = ja;
          mask = 3;
          ++ia;
          ++ib;
        }
        sm.blocks[nblk++] = make_int2(j, mask);
      }
    }
    nblk = __shfl_sync(0xffffffffu, nblk, 0);
    __syncwarp();
  }
  const int per_block = a.sel_len / kBwdChunk;
  const int b0 = video && a.cmp_rows_done ? 1 : 0;
  for (int b = b0; b < nb; ++b) {
    const int br = video ? b : static_cast<int>(kBwdDense);
    const __nv_bfloat16* kb = (br == kBwdCmp) ? a.kc + g * D : a.k + g * D;
    const __nv_bfloat16* vb = (br == kBwdCmp) ? a.vc + g * D : a.v + g * D;
    int lo[2], hi[2], nch = 0;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int t = tk[r];
      if (br == kBwdCmp) {
        lo[r] = 0;
        hi[r] = t >= a.cmp_len - 1 ? min((t - a.cmp_len + 1) / a.cmp_stride + 1, a.ncmp) : 0;
      } else if (br == kBwdWin) {
        lo[r] = max(0, t - a.window + 1);
        hi[r] = t + 1;
      } else {
        lo[r] = 0;
        hi[r] = t + 1;
      }
    }
    const int range_lo = min(lo[0], lo[1]), range_hi = max(hi[0], hi[1]);
    if (br == kBwdSel) nch = nblk * per_block;
    else nch = range_hi > range_lo ? (range_hi - range_lo + kBwdChunk - 1) / kBwdChunk : 0;
    auto desc = [&](int c) -> ChunkDesc {
      ChunkDesc d;
      if (br == kBwdSel) {
        const int2 e = sm.blocks[c / per_block];
        d.start = e.x * a.sel_len + (c % per_block) * kBwdChunk;
        d.row_end = d.start;
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int end = min(e.x * a.sel_len + a.sel_len, tk[r] + 1);
          const bool mine = (e.y >> r) & 1;
          d.lo[r] = d.start;
          d.hi[r] = mine ? end : d.start;
          d.row_end = max(d.row_end, d.hi[r]);
        }
      } else {
        d.start = range_lo + c * kBwdChunk;
        d.row_end = range_hi;
        d.lo[0] = lo[0];
        d.lo[1] = lo[1];
        d.hi[0] = hi[0];
        d.hi[1] = hi[1];
      }
      return d;
    };
    float lse2[2], dg[2], gs[2];
    if (br == kBwdCmp && a.fwd_lse != nullptr) {
      // the forward's statistics: lse2 = lse / ln 2, <dO, o_cmp> from its fp16 output
      const int c = 2 * (lane & 3);
      float part[2] = {0.f, 0.f};
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        lse2[r] = -INFINITY;
        if (!ok[r]) continue;
        const size_t row = static_cast<size_t>(tok[r]) * a.hq + h0 + head[r];
        lse2[r] = a.fwd_lse[row] * 1.4426950408889634f;
        const __half* o = a.fwd_ocmp + row * D + c;
#pragma unroll
        for (int n = 0; n < D / 8; ++n) {
          const float2 ov = __half22float2(*reinterpret_cast<const __half2*>(o + n * 8));
          const float2 dv = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(dp[r] + n * 8 + c));
          part[r] += ov.x * dv.x + ov.y * dv.y;
        }
      }
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        part[r] += __shfl_xor_sync(0xffffffffu, part[r], 1);
        part[r] += __shfl_xor_sync(0xffffffffu, part[r], 2);
        dg[r] = part[r];
      }
    } else {
      // pass A: log-sum-exp and o_b
      WarpAttnState<D> st;
      state_init<D>(st);
      bwd_stream<D>(sm.buf, kb, vb, kv_stride, nch, desc,
                    [&](int stg, const ChunkDesc& cd) { bwd_attend_chunk<D>(st, qa, sm.buf, stg, cd, a.sl2, lane); },
                    lane);
      state_reduce_l<D>(st);
#pragma unroll
      for (int r = 0; r < 2; ++r) lse2[r] = st.l[r] > 0.f ? st.m[r] + __log2f(st.l[r]) : -INFINITY;
      bwd_row_dot<D>(st, dp, lane, dg);
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const size_t o = (static_cast<size_t>(tok[r]) * a.hq + h0 + head[r]) * 3;
      const float gate = ok[r] ? (video ? a.gates[o + b] : 1.f) : 0.f;
      gs[r] = gate * a.scale;
      if ((lane & 3) == 0 && ok[r]) {
        a.stats[o + b] = make_float2(lse2[r], dg[r]);
        a.dgates[o + b] = video ? dg[r] : 0.f;
        if (!video) {
          a.dgates[o + 1] = 0.f;
          a.dgates[o + 2] = 0.f;
        }
      }
    }
    // pass B: dS and dq
    uint32_t da[D / 16][4];
    bwd_load_frags<D>(da, dp[0], dp[1], lane);
    bwd_stream<D>(sm.buf, kb, vb, kv_stride, nch, desc,
                  [&](int stg, const ChunkDesc& cd) {
                    bwd_dq_chunk<D>(dq, qa, da, sm.buf, stg, cd, a.sl2, lse2, dg, gs, lane);
                  },
                  lane);
  }
  const int c = 2 * (lane & 3);
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    if (!ok[r]) continue;
    float* dst = a.dq + (static_cast<size_t>(tok[r]) * a.hq + h0 + head[r]) * D + c;
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
      float2 acc = make_float2(dq[n][2 * r], dq[n][2 * r + 1]);
      if (b0 == 1) {
        const float2 prev = *reinterpret_cast<const float2*>(dst + n * 8);
        acc.x += prev.x;
        acc.y += prev.y;
      }
      *reinterpret_cast<float2*>(dst + n * 8) = acc;
    }
  }
}

// ---------------------------------------------------------------- key pass

template <int D>
struct BwdKeySmem {
  alignas(128) __nv_bfloat16 kt[kBwdChunk * D];  // the item's 16 keys (swizzled rows)
  alignas(128) __nv_bfloat16 vt[kBwdChunk * D];
  alignas(128) __nv_bfloat16 qr[2][kBwdChunk * D];  // 16 gathered (token, head) rows of q
  alignas(128) __nv_bfloat16 dr[2][kBwdChunk * D];  // ... and of dO
  float lse[2][kBwdChunk], dg[2][kBwdChunk], gs[2][kBwdChunk];
  int tok[2][kBwdChunk];
};

template <int D, int BR>
__global__ void __launch_bounds__(32 * kBwdWarps, 2) bwd_key_kernel(const BwdArgs a, long long n_items) {
  extern __shared__ __align__(128) uint8_t bwd_key_smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto& sm = reinterpret_cast<BwdKeySmem<D>*>(bwd_key_smem)[warp];
  const long long item = static_cast<long long>(blockIdx.x) * kBwdWarps + warp;
  if (item >= n_items) return;  // warp-uniform; no CTA-wide barrier follows
  const int G = a.G;
  // ---- the item: its group, 16 keys and the tokens whose rows attend them
  int g = 0, key0 = 0, nkeys = 0, tok_lo = 0, ntok = 0, ent0 = 0;
  if (BR == kBwdCmp) {
    const int nkt = (a.ncmp + kBwdChunk - 1) / kBwdChunk;
    const int nseg = (a.nv + kBwdSegCmp - 1) / kBwdSegCmp;
    const int seg = static_cast<int>(item % nseg);
    const long long rest = item / nseg;
    g = static_cast<int>(rest % a.hkv);
    const int kt = static_cast<int>(rest / a.hkv);
    if (kt >= nkt) return;
    key0 = kt * kBwdChunk;
    nkeys = min(kBwdChunk, a.ncmp - key0);
    tok_lo = max(seg * kBwdSegCmp, key0 * a.cmp_stride + a.cmp_len - 1);
    ntok = min((seg + 1) * kBwdSegCmp, a.nv) - tok_lo;
  } else if (BR == kBwdWin) {
    g = static_cast<int>(item % a.hkv);
    key0 = static_cast<int>(item / a.hkv) * kBwdChunk;
    nkeys = min(kBwdChunk, a.nv - key0);
    tok_lo = key0;
    ntok = min(key0 + kBwdChunk - 1 + a.window, a.nv) - tok_lo;
  } else if (BR == kBwdDense) {
    const int nseg = (a.N - a.nv + kBwdSegDense - 1) / kBwdSegDense;
    const int seg = static_cast<int>(item % nseg);
    const long long rest = item / nseg;
    g = static_cast<int>(rest % a.hkv);
    key0 = static_cast<int>(rest / a.hkv) * kBwdChunk;
    nkeys = min(kBwdChunk, a.N - key0);
    tok_lo = max(a.nv + seg * kBwdSegDense, key0);
    ntok = min(a.nv + (seg + 1) * kBwdSegDense, a.N) - tok_lo;
  } else {
    // item = segment * 4 + quarter of the 64-key block; find the segment's bucket
    const int m = a.hkv * a.nsel;
    const long long seg = item / (a.sel_len / kBwdChunk);
    const int quarter = static_cast<int>(item % (a.sel_len / kBwdChunk));
    if (seg >= a.seg_off[m]) return;
    int lo = 0, hi = m;  // largest bucket with seg_off[bucket] <= seg
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (a.seg_off[mid] <= seg) lo = mid;
      else hi = mid;
    }
    const int bucket = lo;
    g = bucket / a.nsel;
    const int j = bucket % a.nsel;
    key0 = j * a.sel_len + quarter * kBwdChunk;
    nkeys = min(kBwdChunk, a.nv - key0);
    ent0 = a.ent_off[bucket] + static_cast<int>(seg - a.seg_off[bucket]) * kBwdSegSel;
    ntok = min(a.ent_off[bucket + 1] - ent0, kBwdSegSel);
  }
  if (ntok <= 0 || nkeys <= 0) return;
  const int h0 = g * G;
  const int slot = BR == kBwdDense ? 0 : BR;
  const __nv_bfloat16* ksrc = BR == kBwdCmp ? a.kc : a.k;
  const __nv_bfloat16* vsrc = BR == kBwdCmp ? a.vc : a.v;
  auto token_at = [&](int p) -> int { return BR == kBwdSel ? (a.list[ent0 + p] >> 6) : tok_lo + p; };
  // ---- the 16 keys (rows past the end are zero)
  constexpr int kUnits = D / 8;
  for (int i = lane; i < kBwdChunk * kUnits; i += 32) {
    const int row = i / kUnits, unit = i % kUnits;
    const bool ok = row < nkeys;
    const size_t src = (static_cast<size_t>(ok ? key0 + row : 0) * a.hkv + g) * D + unit * 8;
    const int dst = row * D + static_cast<int>(swz_unit(row, unit)) * 8;
    cp_async16(&sm.kt[dst], ksrc + src, ok);
    cp_async16(&sm.vt[dst], vsrc + src, ok);
  }
  const int nrows = ntok * G;
  const int nch = (nrows + kBwdChunk - 1) / kBwdChunk;
  auto load_rows = [&](int stg, int c) {
    if (lane < kBwdChunk) {
      const int r = c * kBwdChunk + lane;
      const bool ok = r < nrows;
      const int t = ok ? token_at(r / G) : 0;
      const int h = r % G;
      const size_t o = (static_cast<size_t>(t) * a.hq + h0 + h) * 3;
      const float2 s = ok ? a.stats[o + slot] : make_float2(-INFINITY, 0.f);
      sm.tok[stg][lane] = ok ? t : -1;
      sm.lse[stg][lane] = s.x;
      sm.dg[stg][lane] = s.y;
      sm.gs[stg][lane] = ok ? (BR == kBwdDense ? 1.f : a.gates[o + BR]) : 0.f;
    }
    for (int i = lane; i < kBwdChunk * kUnits; i += 32) {
      const int row = i / kUnits, unit = i % kUnits;
      const int r = c * kBwdChunk + row;
      const bool ok = r < nrows;
      const int t = ok ? token_at(r / G) : 0;
      const size_t src = (static_cast<size_t>(t) * a.hq + h0 + (ok ? r % G : 0)) * D + unit * 8;
      const int dst = row * D + static_cast<int>(swz_unit(row, unit)) * 8;
      cp_async16(&sm.qr[stg][dst], a.q + src, ok);
      cp_async16(&sm.dr[stg][dst], a.dout + src, ok);
    }
  };
  float dk[D / 8][4], dv[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) dk[n][e] = dv[n][e] = 0.f;
  load_rows(0, 0);
  cp_async_commit();  // group 0: keys and the first rows
  const uint32_t kt_addr = smem_u32(sm.kt), vt_addr = smem_u32(sm.vt);
  const int kr0 = lane >> 2;  // this thread's keys: kr0 and kr0 + 8
  for (int c = 0; c < nch; ++c) {
    if (c + 1 < nch) load_rows((c + 1) & 1, c + 1);
    cp_async_commit();
    cp_async_wait_1();
    __syncwarp();
    const int stg = c & 1;
    const uint32_t q_addr = smem_u32(sm.qr[stg]), d_addr = smem_u32(sm.dr[stg]);
    // S^T = K Q^T and dP^T = V dO^T: 16 keys x 16 rows
    float s[2][4], dp[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) s[nt][e] = dp[nt][e] = 0.f;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      const int arow = (lane & 7) + ((lane >> 3) & 1) * 8;
      const int aunit = ks * 2 + (lane >> 4);
      const uint32_t aoff = (arow * D + swz_unit(arow, aunit) * 8) * 2;
      uint32_t ka[4], va[4];
      ldsm_x4(kt_addr + aoff, ka[0], ka[1], ka[2], ka[3]);
      ldsm_x4(vt_addr + aoff, va[0], va[1], va[2], va[3]);
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const int brow = nt * 8 + (lane & 7);
        const int bunit = ks * 2 + ((lane >> 3) & 1);
        const uint32_t boff = (brow * D + swz_unit(brow, bunit) * 8) * 2;
        uint32_t b0, b1, d0, d1;
        asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];" : "=r"(b0), "=r"(b1) : "r"(q_addr + boff));
        asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];" : "=r"(d0), "=r"(d1) : "r"(d_addr + boff));
        mma_bf16_16816(s[nt], ka, b0, b1);
        mma_bf16_16816(dp[nt], va, d0, d1);
      }
    }
    // P^T (times the gate) and dS^T (times scale and gate) as A operands over the 16 rows
    uint32_t pa[4], sa[4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      float pv[4], ds[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = key0 + kr0 + 8 * (e >> 1);
        const int row = nt * 8 + 2 * (lane & 3) + (e & 1);
        const int t = sm.tok[stg][row];
        const float lse = sm.lse[stg][row];
        bool ok = t >= 0 && (kr0 + 8 * (e >> 1)) < nkeys && lse != -INFINITY;
        if (BR == kBwdCmp) ok = ok && key * a.cmp_stride + a.cmp_len - 1 <= t;
        else if (BR == kBwdWin) ok = ok && key <= t && key > t - a.window;
        else ok = ok && key <= t;
        const float p = ok ? ex2_approx(s[nt][e] * a.sl2 - lse) : 0.f;
        const float gsc = sm.gs[stg][row];
        pv[e] = p * gsc;
        ds[e] = p * gsc * a.scale * (dp[nt][e] - sm.dg[stg][row]);
      }
      pa[nt * 2 + 0] = pack_bf16x2(pv[0], pv[1]);
      pa[nt * 2 + 1] = pack_bf16x2(pv[2], pv[3]);
      sa[nt * 2 + 0] = pack_bf16x2(ds[0], ds[1]);
      sa[nt * 2 + 1] = pack_bf16x2(ds[2], ds[3]);
    }
    // dv += P^T dO, dk += dS^T Q (B: the 16 rows (k) x D (n), row-major in smem)
#pragma unroll
    for (int n = 0; n < D / 8; n += 2) {
      const int row = (lane & 7) + ((lane >> 3) & 1) * 8;
      const int unit = n + (lane >> 4);
      const uint32_t off = (row * D + swz_unit(row, unit) * 8) * 2;
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(d_addr + off, b0, b1, b2, b3);
      mma_bf16_16816(dv[n], pa, b0, b1);
      mma_bf16_16816(dv[n + 1], pa, b2, b3);
      ldsm_x4_t(q_addr + off, b0, b1, b2, b3);
      mma_bf16_16816(dk[n], sa, b0, b1);
      mma_bf16_16816(dk[n + 1], sa, b2, b3);
    }
    __syncwarp();  // every lane is done with this stage before it is refilled
  }
  cp_async_wait_0();
  // ---- add this item's sums
  float* dk_dst = BR == kBwdCmp ? a.dkc : a.dk;
  float* dv_dst = BR == kBwdCmp ? a.dvc : a.dv;
  const int c = 2 * (lane & 3);
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int kr = kr0 + 8 * r;
    if (kr >= nkeys) continue;
    const size_t base = (static_cast<size_t>(key0 + kr) * a.hkv + g) * D;
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
      atomicAdd(dk_dst + base + n * 8 + c, dk[n][2 * r]);
      atomicAdd(dk_dst + base + n * 8 + c + 1, dk[n][2 * r + 1]);
      atomicAdd(dv_dst + base + n * 8 + c, dv[n][2 * r]);
      atomicAdd(dv_dst + base + n * 8 + c + 1, dv[n][2 * r + 1]);
    }
  }
}

// ---------------------------------------------------------------- compression backward
// dk[tau][g] += sum over the blocks i holding tau of w[g][tau - i*s] * dkc[i][g], with
// w = 1/l for the mean or the learnable weights; same for v. One thread per element.
__global__ void __launch_bounds__(256) pool_bwd_kernel(const float* __restrict__ dkc, const float* __restrict__ dvc,
                                                       const float* __restrict__ wk, const float* __restrict__ wv,
                                                       float* __restrict__ dk, float* __restrict__ dv, int nv,
                                                       int hkv, int D, int ncmp, int l, int s) {
  const long long total = static_cast<long long>(nv) * hkv * D;
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= total) return;
  const int col = static_cast<int>(idx % D);
  const int g = static_cast<int>((idx / D) % hkv);
  const int tau = static_cast<int>(idx / (static_cast<long long>(D) * hkv));
  const int i_hi = min(tau / s, ncmp - 1);
  const int i_lo = tau >= l ? (tau - l) / s + 1 : 0;  // smallest i with i*s + l > tau
  float ak = 0.f, av = 0.f;
  for (int i = i_lo; i <= i_hi; ++i) {
    const int u = tau - i * s;
    const float w_k = wk ? wk[g * l + u] : 1.0f / static_cast<float>(l);
    const float w_v = wv ? wv[g * l + u] : 1.0f / static_cast<float>(l);
    const size_t o = (static_cast<size_t>(i) * hkv + g) * D + col;
    ak += w_k * dkc[o];
    av += w_v * dvc[o];
  }
  dk[idx] += ak;
  dv[idx] += av;
}

}  // namespace nsa
