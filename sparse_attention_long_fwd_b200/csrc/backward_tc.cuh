// backward_tc.cuh -- the backward on tcgen05: key passes (dK, dV) of the compressed branch,
// the sliding window and the dense text rows; the row pass (dq) over compressed and window
// tiles; the selected blocks' key pass, which also emits the selected branch's dq partials;
// the kept-statistics kernel and the dq merge.
//
// For a branch's keys K, V the key pass accumulates, over every (token, head) row r that
// sees key i,
//   dV[i] += g_r P[r, i] dO_r,   dK[i] += dS[r, i] q_r,
//   P[r, i] = 2^(scale log2e <q_r, K_i> - lse2_r),  dS = g_r P scale (<dO_r, V_i> - D_r),
// with lse2_r and D_r = <dO_r, o_b,r> from the row statistics (the gradient of the forward
// defined in this library; the pages train the model end to end, shd-paper.top page
// "VideoNSA: Native Sparse Attention Scales Video Understanding", abstract). The keys are
// the compressed summaries Kc, Vc (row r of token t sees block i iff i*s + l - 1 <= t), the
// tokens of the window (t - w < i <= t) or, for text rows, every token i <= t (gate 1).
//
// Key pass: one CTA per (tile of 128 keys, KV group, segment of tokens). Its keys sit in
// the 128 TMEM lanes (M = 128) for the whole item; the rows stream in chunks of 64 (T
// tokens x G heads, a 3-D TMA box like the forward's query tiles) through a four-stage ring:
//   S^T = Kc Q^T and dP^T = Vc dO^T   (M = 128 keys, N = 64 rows, K = d; TMEM columns 0, 64)
//   softmax warps: P g and dS as bf16 into TMEM (columns 128 and 160)
//   dV += (P g)^T-rows x dO, dK += dS x Q   (A from TMEM, B = the stage's dO / Q read
//                                            MN-major; accumulators in columns 256, 384)
// The score MMAs of chunk c are issued before the value MMAs of chunk c-1, so they overlap
// its softmax. P and dS of chunk c are stored only once the MMAs of chunk c-1 that read
// those columns have finished (write-after-read on the same TMEM columns). At the end each
// key's dVc, dKc rows are added to the global sums (segments of one key tile share rows).
// Warp roles: warp 0 loads (the TMA boxes, an L2 prefetch a ring's depth ahead, and the rows'
// lse2 / D / gate by cp.async), warp 1 owns TMEM and issues the MMAs, warps 2..17 (four
// warpgroups) take 16 of a chunk's 64 rows each. Every wait is bounded (sm100.cuh).
#pragma once
#include <cuda_bf16.h>
#include <cstdint>
#include "sm100.cuh"
#include "attn_tc.cuh"
#include "backward.cuh"
#include "sel_inv.cuh"

namespace nsa {

constexpr int kBtKeys = 128;   // compressed keys per item (MMA M)
constexpr int kBtRows = 64;    // rows per chunk (MMA N of the score products)
constexpr int kBtWG = 4;  // softmax warpgroups: each takes 64 / kBtWG rows of every chunk
constexpr int kBtThreads = 64 + 128 * kBtWG;
constexpr int kBtSegTokens = 4096;  // tokens per item segment
constexpr int kBtStages = 4;        // row chunks in flight (a chunk's loads take longer than its MMAs)

__device__ __forceinline__ void cp_async_ca8(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_ca4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}

template <int D>
struct BtSmem {
  static constexpr int kChunks = D / 64;
  alignas(1024) uint8_t kc[kChunks][kBtKeys * 128];
  alignas(1024) uint8_t vc[kChunks][kBtKeys * 128];
  alignas(1024) uint8_t q[kBtStages][kChunks][kBtRows * 128];
  alignas(1024) uint8_t dout[kBtStages][kChunks][kBtRows * 128];
  // per row: lse2, D and the gate, each field its own array so that two adjacent rows' values
  // load as one register pair; only rows that exist are written
  float rlse[kBtStages][kBtRows], rd[kBtStages][kBtRows], rg[kBtStages][kBtRows];
  uint64_t kv_full, q_full[kBtStages], q_empty[kBtStages], sd_full, sd_free, p_full, pv_done, drain;
  uint32_t tmem_base;
  int abort_flag;
};

// BR: kBwdCmp (keys: compressed rows, rows: video tokens), kBwdWin (keys: video tokens,
// rows: the video tokens within the window after them), kBwdDense (keys: all tokens, rows: the
// text tokens after them).
template <int D, int BR>
__global__ void __launch_bounds__(kBtThreads, 1)
    bwd_key_tc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap dmap,
                      const __grid_constant__ CUtensorMap kcmap, const __grid_constant__ CUtensorMap vcmap,
                      const BwdArgs a, int nseg) {
  using Smem = BtSmem<D>;
  constexpr int kChunks = Smem::kChunks;
  constexpr uint32_t kColS = 0, kColDP = 64, kColP = 128, kColDS = 160, kColDV = 256, kColDK = 384;
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = a.G;
  const int T = kBtRows / G;  // tokens per chunk
  // ---- the item: key tile (heaviest first: early keys are seen by the most tokens), group, segment
  const int nkeys_all = BR == kBwdCmp ? a.ncmp : (BR == kBwdWin ? a.nv : a.N);
  const int nkt = (nkeys_all + kBtKeys - 1) / kBtKeys;
  const int seg = blockIdx.x % nseg;
  const int g = (blockIdx.x / nseg) % a.hkv;
  const int kt = blockIdx.x / (nseg * a.hkv);
  if (kt >= nkt) return;
  const int key0 = kt * kBtKeys;
  const int nkeys = min(kBtKeys, nkeys_all - key0);
  // rows: the tokens that see at least one of the tile's keys, cut into segments
  int tok_lo, tok_hi;
  if (BR == kBwdCmp) {
    tok_lo = max(seg * kBtSegTokens, key0 * a.cmp_stride + a.cmp_len - 1);
    tok_hi = min((seg + 1) * kBtSegTokens, a.nv);
  } else if (BR == kBwdWin) {
    tok_lo = max(key0 + seg * kBtSegTokens, key0);
    tok_hi = min(min(key0 + (seg + 1) * kBtSegTokens, key0 + nkeys - 1 + a.window), a.nv);
  } else {
    tok_lo = max(a.nv + seg * kBtSegTokens, key0);
    tok_hi = min(a.nv + (seg + 1) * kBtSegTokens, a.N);
  }
  if (tok_lo >= tok_hi) return;  // uniform across the CTA, before any barrier or TMEM
  const int nch = (tok_hi - tok_lo + T - 1) / T;

  if (tid == 0) {
    mbar_init(&sm.kv_full, 1);
    for (int s = 0; s < kBtStages; ++s) {
      mbar_init(&sm.q_full[s], 1 + 32);  // the TMA's expect_tx arrival + the 32 row-constant lanes
      mbar_init(&sm.q_empty[s], 1);
    }
    mbar_init(&sm.sd_full, 1);
    mbar_init(&sm.sd_free, 4 * kBtWG);
    mbar_init(&sm.p_full, 4 * kBtWG);
    mbar_init(&sm.pv_done, 1);
    mbar_init(&sm.drain, 1);
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  if (warp >= 2) {
    // rows T*G .. 63 of the row stages are never written by TMA: keep them finite (zero), as
    // the value products multiply them by P = dS = 0
    const int r0 = T * G;
    const int per = (kBtRows - r0) * 8;  // 16-byte units per (stage, tensor, chunk)
    for (int i = tid - 64; i < kBtStages * 2 * kChunks * per; i += 128 * kBtWG) {
      const int u = i % per, rest = i / per;
      const int c = rest % kChunks, tq = (rest / kChunks) % 2, s = rest / (2 * kChunks);
      uint8_t* base = tq == 0 ? sm.q[s][c] : sm.dout[s][c];
      *reinterpret_cast<uint4*>(base + (r0 + u / 8) * 128 + (u % 8) * 16) = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort_flag = &sm.abort_flag;
  int q_issued = 0;     // producer: row chunks whose TMA was issued
  bool leader = false;  // MMA warp: the lane that issues every tcgen05 op

  if (warp == 0) {
    // ------------------------------------------------------------------ loads
    if (lane == 0) {
      tma_prefetch_desc(&qmap);
      tma_prefetch_desc(&dmap);
      mbar_arrive_expect_tx(&sm.kv_full, 2 * kChunks * kBtKeys * 128);
      for (int c = 0; c < kChunks; ++c) {
        tma_load_3d(&kcmap, &sm.kv_full, sm.kc[c], c * 64, g, key0);
        tma_load_3d(&vcmap, &sm.kv_full, sm.vc[c], c * 64, g, key0);
      }
    }
    for (int c = 0; c < nch; ++c) {
      const int s = c % kBtStages;
      if (c >= kBtStages &&
          !__all_sync(0xffffffffu, mbar_wait(&sm.q_empty[s], ((c / kBtStages) - 1) & 1, abort_flag)))
        break;
      const int t0 = tok_lo + c * T;
      if (lane == 0) {
        mbar_arrive_expect_tx(&sm.q_full[s], 2 * kChunks * T * G * 128);
        for (int ch = 0; ch < kChunks; ++ch) {
          tma_load_3d(&qmap, &sm.q_full[s], sm.q[s][ch], ch * 64, g * G, t0);
          tma_load_3d(&dmap, &sm.q_full[s], sm.dout[s][ch], ch * 64, g * G, t0);
        }
        // the rows a ring's depth further on go to L2 now (they come from HBM)
        if (c + kBtStages < nch) {
          for (int ch = 0; ch < kChunks; ++ch) {
            tma_prefetch_3d(&qmap, ch * 64, g * G, t0 + kBtStages * T);
            tma_prefetch_3d(&dmap, ch * 64, g * G, t0 + kBtStages * T);
          }
        }
      }
      q_issued = c + 1;
      // the rows' constants, (lse2, D) from the row pass and the branch's gate, copied without
      // waiting: each lane's barrier arrival lands with its copies (text rows keep their
      // statistics in slot 0 and have no gate)
#pragma unroll
      for (int k = 0; k < kBtRows / 32; ++k) {
        const int r = lane + 32 * k;
        const int t = t0 + r / G, h = g * G + r % G;
        if (r < T * G && t < tok_hi) {
          const size_t o = (static_cast<size_t>(t) * a.hq + h) * 3;
          const float* st2 = reinterpret_cast<const float*>(a.stats + o + (BR == kBwdDense ? 0 : BR));
          cp_async_ca4(smem_u32(&sm.rlse[s][r]), st2);
          cp_async_ca4(smem_u32(&sm.rd[s][r]), st2 + 1);
          if (BR != kBwdDense) cp_async_ca4(smem_u32(&sm.rg[s][r]), a.gates + o + BR);
        }
      }
      cp_async_arrive_noinc(&sm.q_full[s]);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    leader = elect_one_sync();
    constexpr uint32_t idS = idesc_bf16_f32(kBtKeys, kBtRows, false, false);
    constexpr uint32_t idV = idesc_bf16_f32(kBtKeys, D, false, true);
    auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
    };
    bool ok = wait_all(&sm.kv_full, 0);
    for (int c = 0; ok && c <= nch; ++c) {
      if (c < nch) {
        // S^T and dP^T of chunk c (their columns were read by the softmax of chunk c - 1)
        const int s = c % kBtStages;
        if (!wait_all(&sm.q_full[s], (c / kBtStages) & 1) || (c >= 1 && !wait_all(&sm.sd_free, (c - 1) & 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (leader) {
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const int ch = k >> 2, kk = k & 3;
            umma_bf16_ss(tmem + kColS, sdesc_sw128(smem_u32(sm.kc[ch]) + kk * 32, 16, 1024),
                         sdesc_sw128(smem_u32(sm.q[s][ch]) + kk * 32, 16, 1024), idS, k > 0 ? 1u : 0u);
          }
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const int ch = k >> 2, kk = k & 3;
            umma_bf16_ss(tmem + kColDP, sdesc_sw128(smem_u32(sm.vc[ch]) + kk * 32, 16, 1024),
                         sdesc_sw128(smem_u32(sm.dout[s][ch]) + kk * 32, 16, 1024), idS, k > 0 ? 1u : 0u);
          }
          umma_commit(&sm.sd_full);
        }
        __syncwarp();
      }
      if (c >= 1) {
        // dV += (P g) x dO and dK += dS x Q over chunk c - 1's 64 rows (16 per MMA)
        const int cp = c - 1, sp = cp % kBtStages;
        if (!wait_all(&sm.p_full, cp & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (leader) {
          const uint64_t ddesc = sdesc_sw128(smem_u32(sm.dout[sp][0]), kBtRows * 128, 1024);
          const uint64_t qdesc = sdesc_sw128(smem_u32(sm.q[sp][0]), kBtRows * 128, 1024);
#pragma unroll
          for (int k = 0; k < kBtRows / 16; ++k) {
            const uint32_t acc = (cp > 0 || k > 0) ? 1u : 0u;
            umma_bf16_ts(tmem + kColDV, tmem + kColP + k * 8, ddesc + static_cast<uint64_t>(k * (2048 >> 4)), idV,
                         acc);
            umma_bf16_ts(tmem + kColDK, tmem + kColDS + k * 8, qdesc + static_cast<uint64_t>(k * (2048 >> 4)), idV,
                         acc);
          }
          umma_commit(&sm.pv_done);
          umma_commit(&sm.q_empty[sp]);
        }
        __syncwarp();
      }
    }
  } else {
    // ------------------------------------------------------------------ softmax warps
    constexpr int kRows = kBtRows / kBtWG;  // rows per thread and chunk
    constexpr int kPart = D / kBtWG;        // dV, dK columns per thread
    static_assert(kRows == 16 && (kPart == 32 || kPart == 16), "16-column TMEM loads per chunk");
    const int sw = warp - 2;
    const int wg = sw >> 2;          // rows [kRows wg, kRows wg + kRows) of each chunk
    const int q4 = warp & 3;         // TMEM lane quadrant
    const int kl = q4 * 32 + lane;   // this thread's key (TMEM lane)
    const uint32_t trow = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const int key = key0 + kl;
    const bool key_ok = kl < nkeys;
    // the tokens that see this key: [tk, tk_end]
    const int tk = BR == kBwdCmp ? key * a.cmp_stride + a.cmp_len - 1 : key;
    const int tk_end = BR == kBwdWin ? key + a.window - 1 : 0x7fffffff;
    const float sl2 = a.sl2, scale = a.scale;
    bool ok = true;
    for (int c = 0; c < nch && ok; ++c) {
      const int s = c % kBtStages;
      ok = __all_sync(0xffffffffu, mbar_wait(&sm.sd_full, c & 1, abort_flag) &&
                                       mbar_wait(&sm.q_full[s], (c / kBtStages) & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      float sv[kRows], dp[kRows];
      __syncwarp();
      tmem_ld16(trow + kColS + kRows * wg, sv);
      tmem_ld16(trow + kColDP + kRows * wg, dp);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.sd_free);
      // the chunk's rows r = token slot * G + head that exist and see this key: [r_lo, r_hi)
      // (row token t0 + r / G sees it iff tk <= t <= tk_end; those rows' lse is finite)
      const int t0 = tok_lo + c * T;
      const int r_lo = min(max(tk - t0, 0), T) * G;
      const int n_end = tk_end - t0 >= T ? T : max(tk_end - t0 + 1, 0);  // (tk_end may be INT_MAX)
      const int r_hi = key_ok ? min(n_end, tok_hi - t0) * G : 0;
      uint32_t pp[kRows / 2], pd[kRows / 2];
#pragma unroll
      for (int j = 0; j < kRows; j += 2) {
        // rows r and r + 1 in paired fp32 arithmetic (their constants load as register pairs):
        // P = 2^(S sl2 - lse2), P g, dS = P g scale (dP - D)
        const int r = kRows * wg + j;
        const float2 l2 = *reinterpret_cast<const float2*>(&sm.rlse[s][r]);
        const float2 dd = *reinterpret_cast<const float2*>(&sm.rd[s][r]);
        float x0, x1, pg0, pg1, d0, d1;
        fma2v(x0, x1, sv[j], sv[j + 1], sl2, -l2.x, -l2.y);
        const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
        if (BR == kBwdDense) {
          pg0 = p0;
          pg1 = p1;
        } else {
          const float2 gg = *reinterpret_cast<const float2*>(&sm.rg[s][r]);
          mul2v(pg0, pg1, p0, p1, gg.x, gg.y);
        }
        sub2v(d0, d1, dp[j], dp[j + 1], dd.x, dd.y);
        mul2v(d0, d1, d0, d1, scale, scale);
        mul2v(d0, d1, d0, d1, pg0, pg1);
        const bool vis0 = r >= r_lo && r < r_hi, vis1 = r + 1 >= r_lo && r + 1 < r_hi;
        pp[j / 2] = pack_bf16x2(vis0 ? pg0 : 0.f, vis1 ? pg1 : 0.f);
        pd[j / 2] = pack_bf16x2(vis0 ? d0 : 0.f, vis1 ? d1 : 0.f);
      }
      // P and dS of chunk c go over the columns the value MMAs of chunk c - 1 read
      if (c >= 1) ok = mbar_wait(&sm.pv_done, (c - 1) & 1, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      tmem_st8(trow + kColP + (kRows / 2) * wg, pp);
      tmem_st8(trow + kColDS + (kRows / 2) * wg, pd);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.p_full);
    }
    // ---- the item's sums: this warpgroup's part of the key's dV and dK rows
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&sm.pv_done, (nch - 1) & 1, abort_flag));
    if (ok) {
      tc_fence_after();
      float* dvr = (BR == kBwdCmp ? a.dvc : a.dv) + (static_cast<size_t>(key) * a.hkv + g) * D + wg * kPart;
      float* dkr = (BR == kBwdCmp ? a.dkc : a.dk) + (static_cast<size_t>(key) * a.hkv + g) * D + wg * kPart;
      float v[kPart], kk[kPart];
      __syncwarp();
      if constexpr (kPart == 32) {
        tmem_ld32(trow + kColDV + wg * kPart, v);
        tmem_ld32(trow + kColDK + wg * kPart, kk);
      } else {
        tmem_ld16(trow + kColDV + wg * kPart, v);
        tmem_ld16(trow + kColDK + wg * kPart, kk);
      }
      tmem_wait_ld();
      if (key_ok) {
#pragma unroll
        for (int u = 0; u < kPart; u += 4) {
          atomicAdd(reinterpret_cast<float4*>(dvr + u), make_float4(v[u], v[u + 1], v[u + 2], v[u + 3]));
          atomicAdd(reinterpret_cast<float4*>(dkr + u), make_float4(kk[u], kk[u + 1], kk[u + 2], kk[u + 3]));
        }
      }
    }
    tc_fence_before();
  }

  // ------------------------------------------------------------------ teardown
  __syncthreads();
  if (*abort_flag) {
    // drain: wait (bounded) for the loads issued and for MMAs in flight, so no async write
    // lands after the CTA exits
    if (warp == 0 && lane == 0) {
      long long t_start = clock64();
      while (!mbar_test(&sm.kv_full, 0) && clock64() - t_start < kWaitCycles) {
      }
      for (int c = q_issued - kBtStages > 0 ? q_issued - kBtStages : 0; c < q_issued; ++c) {
        t_start = clock64();
        while (!mbar_test(&sm.q_full[c % kBtStages], (c / kBtStages) & 1) && clock64() - t_start < kWaitCycles) {
        }
      }
    }
    if (warp == 1 && leader) {
      umma_commit(&sm.drain);
      const long long t_start = clock64();
      while (!mbar_test(&sm.drain, 0) && clock64() - t_start < kWaitCycles) {
      }
    }
    __syncwarp();
    __syncthreads();
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace nsa

namespace nsa {

// ---------------------------------------------------------------- row pass, contiguous keys
// dq of the video rows on tcgen05 from branches whose keys are contiguous, given the forward's
// saved log-sum-exp and output of each: per row r (token t, head h) and visible key i of
// branch b,
//   P = 2^(scale log2e <q_r, K_i> - lse2_r,b),  dS = g_r,b scale P (<dO_r, V_i> - D_r,b),
//   dq_r = sum_b sum_i dS K_i,   D_r,b = <dO_r, o_b,r>.
// kFull = false: the compressed branch only (its statistics and gate gradient are written here,
// the warp row pass adds the other branches to dq); kFull = true: the compressed blocks, then
// the window's tokens [t - w + 1, t], with every branch's statistics already in `stats`.
// One CTA per (query tile of T = 128 / G tokens x G heads, KV group): its Q and dO tiles load
// once, the keys stream in 128-key tiles through a two-slot ring:
//   S = Q K^T, dP = dO V^T     (M = 128 rows, N = 128 keys; TMEM columns 0 and 128)
//   softmax warps: dS as bf16 into TMEM (column 384)
//   dQ += dS K                 (A = dS from TMEM, B = the slot's K read MN-major; column 256)
// It writes dq for these rows. Warp 0 loads, warp 1 issues the MMAs, kBrWG softmax warpgroups
// (thread = row) split each tile's key columns; every wait is bounded.
constexpr int kBrWG = 4;  // softmax warpgroups: each takes 128 / kBrWG key columns of every tile
constexpr int kBrThreads = 64 + 128 * kBrWG;
constexpr int kBrSlots = 2;

template <int D>
struct BrSmem {
  static constexpr int kChunks = D / 64;
  alignas(1024) uint8_t q[kChunks][128 * 128];
  alignas(1024) uint8_t dout[kChunks][128 * 128];
  alignas(1024) uint8_t kc[kBrSlots][kChunks][128 * 128];
  alignas(1024) uint8_t vc[kBrSlots][kChunks][128 * 128];
  float rowc[kBrWG][128];  // per row: the warpgroups' parts of <dO, o_cmp>
  uint64_t q_full, kv_full[kBrSlots], kv_empty[kBrSlots], sd_full, sd_free, p_full, pv_done, drain;
  uint32_t tmem_base;
  int abort_flag;
};

template <int D, bool kFull>
__global__ void __launch_bounds__(kBrThreads, 1)
    bwd_row_tc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap dmap,
                      const __grid_constant__ CUtensorMap kcmap, const __grid_constant__ CUtensorMap vcmap,
                      const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                      const BwdArgs a) {
  using Smem = BrSmem<D>;
  constexpr int kChunks = Smem::kChunks;
  constexpr uint32_t kColS = 0, kColDP = 128, kColDQ = 256, kColDS = 384;
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = a.G;
  const int T = 128 / G;
  // the item: query tile (latest first: they see the most keys), group
  const int ntiles = (a.nv + T - 1) / T;
  const int g = blockIdx.x % a.hkv;
  const int tile = ntiles - 1 - static_cast<int>(blockIdx.x / a.hkv);
  if (tile < 0) return;
  const int t0 = tile * T;
  const int t_last = min(t0 + T, a.nv) - 1;
  const int ke = t_last + 1 >= a.cmp_len ? min((t_last + 1 - a.cmp_len) / a.cmp_stride + 1, a.ncmp) : 0;
  const int nkt_c = (ke + 127) / 128;
  const int kb_w = kFull ? max(0, t0 - a.window + 1) : 0;  // window keys [kb_w, t_last]
  const int nkt = nkt_c + (kFull ? (t_last + 1 - kb_w + 127) / 128 : 0);

  if (tid == 0) {
    mbar_init(&sm.q_full, 1);
    for (int s = 0; s < kBrSlots; ++s) {
      mbar_init(&sm.kv_full[s], 1);
      mbar_init(&sm.kv_empty[s], 1);
    }
    mbar_init(&sm.sd_full, 1);
    mbar_init(&sm.sd_free, 4 * kBrWG);
    mbar_init(&sm.p_full, 4 * kBrWG);
    mbar_init(&sm.pv_done, 1);
    mbar_init(&sm.drain, 1);
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  if (warp >= 2) {
    // rows T*G .. 127 of the Q and dO tiles are never written by TMA: keep them finite (zero)
    const int r0 = T * G;
    const int per = (128 - r0) * 8;
    for (int i = tid - 64; i < 2 * kChunks * per; i += 128 * kBrWG) {
      const int u = i % per, rest = i / per;
      const int c = rest % kChunks, tq = rest / kChunks;
      uint8_t* base = tq == 0 ? sm.q[c] : sm.dout[c];
      *reinterpret_cast<uint4*>(base + (r0 + u / 8) * 128 + (u % 8) * 16) = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort_flag = &sm.abort_flag;
  int kv_issued = 0;
  bool leader = false;

  if (warp == 0) {
    // ------------------------------------------------------------------ loads
    if (lane == 0) {
      mbar_arrive_expect_tx(&sm.q_full, 2 * kChunks * T * G * 128);
      for (int c = 0; c < kChunks; ++c) {
        tma_load_3d(&qmap, &sm.q_full, sm.q[c], c * 64, g * G, t0);
        tma_load_3d(&dmap, &sm.q_full, sm.dout[c], c * 64, g * G, t0);
      }
      for (int kt = 0; kt < nkt; ++kt) {
        const int s = kt % kBrSlots;
        if (kt >= kBrSlots && !mbar_wait(&sm.kv_empty[s], ((kt / kBrSlots) - 1) & 1, abort_flag)) break;
        mbar_arrive_expect_tx(&sm.kv_full[s], 2 * kChunks * 128 * 128);
        const bool win = kFull && kt >= nkt_c;
        const int k0 = win ? kb_w + (kt - nkt_c) * 128 : kt * 128;
        for (int c = 0; c < kChunks; ++c) {
          tma_load_3d(win ? &kmap : &kcmap, &sm.kv_full[s], sm.kc[s][c], c * 64, g, k0);
          tma_load_3d(win ? &vmap : &vcmap, &sm.kv_full[s], sm.vc[s][c], c * 64, g, k0);
        }
        // the window's key tiles come from HBM: the one two tiles on goes to L2 now
        if (kFull && kt + 2 >= nkt_c && kt + 2 < nkt) {
          const int kp = kb_w + (kt + 2 - nkt_c) * 128;
          for (int c = 0; c < kChunks; ++c) {
            tma_prefetch_3d(&kmap, c * 64, g, kp);
            tma_prefetch_3d(&vmap, c * 64, g, kp);
          }
        }
        kv_issued = kt + 1;
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    leader = elect_one_sync();
    constexpr uint32_t idS = idesc_bf16_f32(128, 128, false, false);
    constexpr uint32_t idQ = idesc_bf16_f32(128, D, false, true);
    auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
    };
    bool ok = wait_all(&sm.q_full, 0);
    for (int kt = 0; ok && kt <= nkt; ++kt) {
      if (kt < nkt) {
        const int s = kt % kBrSlots;
        if (!wait_all(&sm.kv_full[s], (kt / kBrSlots) & 1) || (kt >= 1 && !wait_all(&sm.sd_free, (kt - 1) & 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (leader) {
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const int ch = k >> 2, kk = k & 3;
            umma_bf16_ss(tmem + kColS, sdesc_sw128(smem_u32(sm.q[ch]) + kk * 32, 16, 1024),
                         sdesc_sw128(smem_u32(sm.kc[s][ch]) + kk * 32, 16, 1024), idS, k > 0 ? 1u : 0u);
          }
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const int ch = k >> 2, kk = k & 3;
            umma_bf16_ss(tmem + kColDP, sdesc_sw128(smem_u32(sm.dout[ch]) + kk * 32, 16, 1024),
                         sdesc_sw128(smem_u32(sm.vc[s][ch]) + kk * 32, 16, 1024), idS, k > 0 ? 1u : 0u);
          }
          umma_commit(&sm.sd_full);
        }
        __syncwarp();
      }
      if (kt >= 1) {
        // dQ += dS Kc over the previous key tile (16 keys per MMA)
        const int kp = kt - 1, sp = kp % kBrSlots;
        if (!wait_all(&sm.p_full, kp & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (leader) {
          const uint64_t kdesc = sdesc_sw128(smem_u32(sm.kc[sp][0]), 128 * 128, 1024);
#pragma unroll
          for (int k = 0; k < 128 / 16; ++k)
            umma_bf16_ts(tmem + kColDQ, tmem + kColDS + k * 8, kdesc + static_cast<uint64_t>(k * (2048 >> 4)), idQ,
                         (kp > 0 || k > 0) ? 1u : 0u);
          umma_commit(&sm.pv_done);
          umma_commit(&sm.kv_empty[sp]);
        }
        __syncwarp();
      }
    }
  } else {
    // ------------------------------------------------------------------ softmax warps
    constexpr int kCols = 128 / kBrWG;  // key columns per thread and tile
    constexpr int kPart = D / kBrWG;    // dq columns per thread
    static_assert(kCols == 32 && (kPart == 32 || kPart == 16), "one 32-column TMEM load per tile");
    const int sw = warp - 2;
    const int wg = sw >> 2;          // key columns [kCols wg, kCols wg + kCols) of each tile
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;    // this thread's row (TMEM lane)
    const uint32_t trow = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const int tok = r / G, hh = r % G;
    const int t = t0 + tok;
    const int h = g * G + hh;
    const bool row_valid = r < T * G && t < a.nv;
    bool ok = true;
    // ---- the row's constants: D = <dO, o_cmp> from the forward's fp16 output, each warpgroup
    // over a part of the head dimension, summed through shared memory (kFull: every branch's
    // statistics are in `stats` already)
    float lse2 = -INFINITY, gs = 0.f, dgr = 0.f;
    float lse2_w = -INFINITY, gs_w = 0.f, dgr_w = 0.f;
    int re = 0;
    if constexpr (kFull) {
      if (row_valid) {
        const size_t o = (static_cast<size_t>(t) * a.hq + h) * 3;
        const float2 sc = a.stats[o + kBwdCmp], sw_ = a.stats[o + kBwdWin];
        lse2 = sc.x;
        dgr = sc.y;
        gs = a.gates[o + kBwdCmp] * a.scale;
        lse2_w = sw_.x;
        dgr_w = sw_.y;
        gs_w = a.gates[o + kBwdWin] * a.scale;
        re = t >= a.cmp_len - 1 ? min((t - a.cmp_len + 1) / a.cmp_stride + 1, a.ncmp) : 0;
      }
    } else {
      float part = 0.f;
      if (row_valid) {
        const size_t row = static_cast<size_t>(t) * a.hq + h;
        const __half* o = a.fwd_ocmp + row * D + wg * kPart;
        const __nv_bfloat16* dop = a.dout + row * D + wg * kPart;
#pragma unroll
        for (int c = 0; c < kPart; c += 8) {
          const uint4 ov = *reinterpret_cast<const uint4*>(o + c);
          const uint4 dv = *reinterpret_cast<const uint4*>(dop + c);
          const __half2* oh = reinterpret_cast<const __half2*>(&ov);
          const __nv_bfloat162* dh = reinterpret_cast<const __nv_bfloat162*>(&dv);
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            const float2 of = __half22float2(oh[x]);
            const float2 df = __bfloat1622float2(dh[x]);
            part += of.x * df.x + of.y * df.y;
          }
        }
        lse2 = a.fwd_lse[row] * 1.4426950408889634f;
        gs = a.gates[row * 3 + kBwdCmp] * a.scale;
        re = t >= a.cmp_len - 1 ? min((t - a.cmp_len + 1) / a.cmp_stride + 1, a.ncmp) : 0;
      }
      sm.rowc[wg][r] = part;
      named_bar_sync(1, 128 * kBrWG);
#pragma unroll
      for (int w = 0; w < kBrWG; ++w) dgr += sm.rowc[w][r];
      if (wg == 0 && row_valid) {
        const size_t o = (static_cast<size_t>(t) * a.hq + h) * 3;
        a.stats[o + kBwdCmp] = make_float2(lse2, dgr);
        a.dgates[o + kBwdCmp] = dgr;
      }
    }
    for (int kt = 0; ok && kt < nkt; ++kt) {
      ok = __all_sync(0xffffffffu, mbar_wait(&sm.sd_full, kt & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      const bool win = kFull && kt >= nkt_c;
      // this thread's keys: [kbase, kbase + kCols), visible in [lo, hi)
      const int kbase = (win ? kb_w + (kt - nkt_c) * 128 : kt * 128) + wg * kCols;
      const int lo = win ? t - a.window + 1 : 0, hi = win ? t + 1 : re;
      const float l2 = win ? lse2_w : lse2, dg = win ? dgr_w : dgr, gsb = win ? gs_w : gs;
      const bool full = __all_sync(0xffffffffu, !row_valid || (kbase >= lo && kbase + kCols <= hi));
      uint32_t pd[kCols / 2];
      {
        float sv[kCols], dp[kCols];
        __syncwarp();
        tmem_ld32(trow + kColS + wg * kCols, sv);
        tmem_ld32(trow + kColDP + wg * kCols, dp);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.sd_free);
#pragma unroll
        for (int j = 0; j < kCols; j += 2) {
          // keys j and j + 1 in paired fp32 arithmetic: P = 2^(S sl2 - lse2), dS = P g scale (dP - D)
          const int kidx = kbase + j;
          const bool ok_row = row_valid && l2 != -INFINITY;
          const bool vis0 = ok_row && (full || (kidx >= lo && kidx < hi));
          const bool vis1 = ok_row && (full || (kidx + 1 >= lo && kidx + 1 < hi));
          float x0, x1, d0, d1;
          fma2(x0, x1, sv[j], sv[j + 1], a.sl2, -l2);
          const float p0 = vis0 ? ex2_approx(x0) : 0.f, p1 = vis1 ? ex2_approx(x1) : 0.f;
          sub2v(d0, d1, dp[j], dp[j + 1], dg, dg);
          mul2v(d0, d1, d0, d1, gsb, gsb);
          mul2v(d0, d1, d0, d1, p0, p1);
          pd[j / 2] = pack_bf16x2(d0, d1);
        }
      }
      // dS of this tile goes over the columns the previous tile's dQ MMAs read
      if (kt >= 1) ok = mbar_wait(&sm.pv_done, (kt - 1) & 1, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      tmem_st16(trow + kColDS + wg * (kCols / 2), pd);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.p_full);
    }
    // ---- dq of this row: this warpgroup's part of D (zero when no key was visible)
    if (ok && nkt > 0) ok = __all_sync(0xffffffffu, mbar_wait(&sm.pv_done, (nkt - 1) & 1, abort_flag));
    if (ok) {
      tc_fence_after();
      float* dst = a.dq + (static_cast<size_t>(t) * a.hq + h) * D + wg * kPart;
      float v[kPart];
      __syncwarp();
      if (nkt > 0) {
        if constexpr (kPart == 32) tmem_ld32(trow + kColDQ + wg * kPart, v);
        else tmem_ld16(trow + kColDQ + wg * kPart, v);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int u = 0; u < kPart; ++u) v[u] = 0.f;
      }
      if (row_valid) {
#pragma unroll
        for (int u = 0; u < kPart; u += 4)
          *reinterpret_cast<float4*>(dst + u) = make_float4(v[u], v[u + 1], v[u + 2], v[u + 3]);
      }
    }
    tc_fence_before();
  }

  // ------------------------------------------------------------------ teardown
  __syncthreads();
  if (*abort_flag) {
    if (warp == 0 && lane == 0) {
      long long t_start = clock64();
      while (!mbar_test(&sm.q_full, 0) && clock64() - t_start < kWaitCycles) {
      }
      for (int kt = kv_issued - kBrSlots > 0 ? kv_issued - kBrSlots : 0; kt < kv_issued; ++kt) {
        t_start = clock64();
        while (!mbar_test(&sm.kv_full[kt % kBrSlots], (kt / kBrSlots) & 1) && clock64() - t_start < kWaitCycles) {
        }
      }
    }
    if (warp == 1 && leader) {
      umma_commit(&sm.drain);
      const long long t_start = clock64();
      while (!mbar_test(&sm.drain, 0) && clock64() - t_start < kWaitCycles) {
      }
    }
    __syncwarp();
    __syncthreads();
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace nsa

namespace nsa {

// ---------------------------------------------------------------- key pass, selected branch
// dK and dV of the selected blocks on tcgen05, over the buckets of (group, block j) that list
// the tokens which chose block j. A tile is 128 gathered rows (T = 128 / G tokens x G heads)
// against the block's 64 keys:
//   S = Q K_j^T, dP = dO V_j^T           (M = 128 rows, N = 64 keys; TMEM, double-buffered)
//   softmax warps: g P and dS = g scale P (dP - D) as bf16 tiles in shared memory
//   dV_j^T += dO^T (g P), dK_j^T += Q^T dS  (M = D = 128 dims, N = 64 keys, K = 128 rows: A and
//                                            B both read MN-major from the tiles already there)
// so all four products run at M = 128 with no padding. dV^T and dK^T accumulate in TMEM over
// the consecutive tiles of one bucket and are added to dv, dk (fp32, lane = dimension, so a
// warp's reductions cover 128 contiguous bytes) after the bucket's last tile in this CTA.
// kDq: also dQ = dS K_j (M = 128 rows, N = D, K = 64 keys; TMEM, double-buffered), stored
// per tile row as an fp16 partial (each 64-column half with a power-of-two factor that keeps
// it finite), which a merge adds to the row's dq: the selected branch's share of dq.
// TMEM columns: S 0, dP 64, dV^T 128, dK^T 192, dQ 256 and 384.
// Persistent: CTA c takes tiles [total c / grid, total (c + 1) / grid).
//   warps 0..2   producers: warp 0 writes the tile records and loads K_j, V_j by TMA once per
//                bucket run; all three gather the tile's Q and dO rows with 16-byte cp.async
//                into the 128-byte-swizzled layout
//   warp 3       MMA issuer
//   warps 4..11  two warpgroups, thread = row; warpgroup w takes keys 32w .. 32w + 31 of each
//                tile and, at a bucket's end, the dV^T (w = 0) or dK^T (w = 1) columns
constexpr int kBsProducers = 3;
constexpr int kBsMmaWarp = 3;
constexpr int kBsFirstSmx = 4;
constexpr int kBsThreads = 32 * kBsFirstSmx + 256;
constexpr int kBsQStages = 2;
constexpr int kBsInfo = 8;

template <int D>
struct BsSmem {
  static constexpr int kChunks = D / 64;
  alignas(1024) uint8_t q[kBsQStages][kChunks][128 * 128];
  alignas(1024) uint8_t dout[kBsQStages][kChunks][128 * 128];
  alignas(1024) uint8_t k[kChunks][64 * 128];
  alignas(1024) uint8_t v[kChunks][64 * 128];
  alignas(1024) uint8_t p[128 * 128];   // g P: 128 rows x 64 keys bf16, 128-byte swizzled rows
  alignas(1024) uint8_t ds[128 * 128];  // dS, the same layout
  SelTileInfo info[kBsInfo];
  uint64_t q_full[kBsQStages], q_empty[kBsQStages], kv_full, kv_empty;
  uint64_t info_full[kBsInfo], info_empty[kBsInfo];
  uint64_t s_full, s_free, pd_full, pd_free, acc_full, dq_full[2], dq_free[2], drain;
  uint32_t tmem_base;
  int abort_flag;
};

template <int D, bool kDq>
__global__ void __launch_bounds__(kBsThreads, 1)
    bwd_sel_key_tc_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                          const BwdArgs a) {
  static_assert(D == 128, "the dV^T and dK^T products take M = D = 128");
  using Smem = BsSmem<D>;
  constexpr int kChunks = Smem::kChunks;
  constexpr int kCpr = D / 8;  // 16-byte pieces per row
  constexpr uint32_t kColAcc = 128, kColDQ = 256;
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = a.G, TT = 128 / G;
  const int m = a.hkv * a.nsel;
  const long long total = a.seg_off[m];
  const int tile_begin = static_cast<int>(total * blockIdx.x / gridDim.x);
  const int tile_end = static_cast<int>(total * (blockIdx.x + 1) / gridDim.x);
  const int n = tile_end - tile_begin;
  if (n <= 0) return;  // uniform across the CTA
  if (tid == 0) {
    for (int s = 0; s < kBsQStages; ++s) {
      mbar_init(&sm.q_full[s], kBsProducers * 32);  // one cp.async arrival per producer lane
      mbar_init(&sm.q_empty[s], 1);
    }
    mbar_init(&sm.kv_full, 1);
    mbar_init(&sm.kv_empty, 1);
    for (int s = 0; s < kBsInfo; ++s) {
      mbar_init(&sm.info_full[s], 1);
      mbar_init(&sm.info_empty[s], 8);
    }
    mbar_init(&sm.s_full, 1);
    mbar_init(&sm.s_free, 8);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.dq_full[b], 1);
      mbar_init(&sm.dq_free[b], 8);
    }
    mbar_init(&sm.pd_full, 8);
    mbar_init(&sm.pd_free, 1);
    mbar_init(&sm.acc_full, 1);
    mbar_init(&sm.drain, 1);
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kBsMmaWarp) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  {
    // rows a tile does not load keep what the stage held before: zero them once so that they
    // are finite (their P and dS are zero, and 0 x NaN would not be)
    uint4* z = reinterpret_cast<uint4*>(&sm.q[0][0][0]);
    const int nq = static_cast<int>(sizeof(sm.q) / 16);
    for (int i = tid; i < nq; i += kBsThreads) z[i] = make_uint4(0, 0, 0, 0);
    z = reinterpret_cast<uint4*>(&sm.dout[0][0][0]);
    for (int i = tid; i < nq; i += kBsThreads) z[i] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort_flag = &sm.abort_flag;
  int kv_issued = 0;  // warp 0: K-V loads issued

  if (warp < kBsProducers) {
    // ------------------------------------------------------------------ producers
    int key = 0, t_base = 0, t_next = 0, e_base = 0, e_next = 0;
    auto fetch = [&](int tile) {
      SelTileMeta r;
      while (t_next <= tile) {  // next bucket with tiles
        ++key;
        t_base = t_next;
        e_base = e_next;
        t_next = a.seg_off[key + 1];
        e_next = a.ent_off[key + 1];
      }
      r.key = key;
      r.e0 = e_base + (tile - t_base) * TT;
      r.cnt = min(TT, e_next - r.e0);
      r.last = (tile == tile_end - 1) || (t_next == tile + 1);
#pragma unroll
      for (int k = 0; k < 4; ++k) r.e[k] = (lane + 32 * k < r.cnt) ? a.list[r.e0 + lane + 32 * k] : 0;
      return r;
    };
    SelTileMeta cur{};
    if (warp == 0) {
      if (lane == 0) {
        tma_prefetch_desc(&kmap);
        tma_prefetch_desc(&vmap);
        int lo = 0, hi = m - 1;  // bucket of the first tile: the last key with seg_off[key] <= tile_begin
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if (a.seg_off[mid] <= tile_begin) lo = mid; else hi = mid - 1;
        }
        key = lo;
      }
      key = __shfl_sync(0xffffffffu, key, 0);
      t_base = a.seg_off[key];
      t_next = a.seg_off[key + 1];
      e_base = a.ent_off[key];
      e_next = a.ent_off[key + 1];
      cur = fetch(tile_begin);
    }
    int kv_key = -1;
    for (int i = 0; i < n; ++i) {
      const int si = i % kBsInfo, sq = i % kBsQStages;
      SelTileInfo& inf = sm.info[si];
      if (warp == 0) {
        if (i >= kBsInfo && !warp_wait(&sm.info_empty[si], ((i / kBsInfo) - 1) & 1, abort_flag)) break;
        const bool first = cur.key != kv_key;
#pragma unroll
        for (int k = 0; k < 4; ++k)
          if (lane + 32 * k < cur.cnt) inf.ent[lane + 32 * k] = cur.e[k];
        if (lane == 0) {
          inf.key = cur.key;
          inf.cnt = cur.cnt;
          inf.kvs = 0;
          inf.flags = (first ? 1 : 0) | (cur.last ? 2 : 0);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.info_full[si]);
      } else if (!warp_wait(&sm.info_full[si], (i / kBsInfo) & 1, abort_flag)) {
        break;
      }
      // Q and dO rows: row R = token slot R / G, head slot R % G; this warp takes the 32-row
      // blocks b with b % 3 == (warp + 1) % 3 (warp 0, which also writes the records, the fewest)
      if (i >= kBsQStages && !warp_wait(&sm.q_empty[sq], ((i / kBsQStages) - 1) & 1, abort_flag)) break;
      {
        const int cnt = inf.cnt;
        const int g = inf.key / a.nsel;
        for (int b = (warp + 1) % kBsProducers; b < 4; b += kBsProducers) {
          const int rbase = b * 32;
          int my_row = -1;
          {
            const int R = rbase + lane;
            const int tok = R / G, hh = R - tok * G;
            if (tok < cnt) my_row = (inf.ent[tok] >> 6) * a.hq + g * G + hh;
          }
          constexpr int kRpi = 32 / kCpr;  // rows per iteration
          const int sub = lane / kCpr, c16 = lane % kCpr;
          const char* q_lane = reinterpret_cast<const char*>(a.q) + c16 * 16;
          const char* d_lane = reinterpret_cast<const char*>(a.dout) + c16 * 16;
          // 128-byte swizzle: piece (c16 & 7) of row R sits at unit (c16 & 7) ^ (R & 7)
          const uint32_t off_lane = (c16 >> 3) * (128 * 128) + (rbase + sub) * 128;
          const uint32_t qdst = smem_u32(sm.q[sq][0]) + off_lane, ddst = smem_u32(sm.dout[sq][0]) + off_lane;
          const uint32_t x_lane = (c16 & 7) ^ sub;
#pragma unroll
          for (int it = 0; it < kCpr; ++it) {
            const int row = __shfl_sync(0xffffffffu, my_row, it * kRpi + sub);
            const uint32_t o = it * kRpi * 128 + ((x_lane ^ ((it * kRpi) & 7)) << 4);
            if (row >= 0) {
              cp_async16_cg(qdst + o, q_lane + static_cast<size_t>(row) * (D * 2));
              cp_async16_cg(ddst + o, d_lane + static_cast<size_t>(row) * (D * 2));
            }
          }
        }
        cp_async_arrive_noinc(&sm.q_full[sq]);
      }
      if (warp == 0) {
        if (cur.key != kv_key) {
          const int u = kv_issued;  // K-V load number
          if (u >= 1 && !warp_wait(&sm.kv_empty, (u - 1) & 1, abort_flag)) break;
          if (lane == 0) {
            const int g = cur.key / a.nsel, j = cur.key % a.nsel;
            mbar_arrive_expect_tx(&sm.kv_full, kChunks * 2 * 64 * 128);
            for (int c = 0; c < kChunks; ++c) {
              tma_load_3d(&kmap, &sm.kv_full, sm.k[c], c * 64, g, j * a.sel_len);
              tma_load_3d(&vmap, &sm.kv_full, sm.v[c], c * 64, g, j * a.sel_len);
            }
          }
          __syncwarp();
          kv_issued = u + 1;
          kv_key = cur.key;
        }
        if (i + 1 < n) cur = fetch(tile_begin + i + 1);
      }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
  } else if (warp == kBsMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(128, 64, false, false);
      constexpr uint32_t idT = idesc_bf16_f32(128, 64, true, true);
      constexpr uint32_t idQ = idesc_bf16_f32(128, D, false, true);
      int ns = 0, np = 0, kv_seen = 0;    // next S tile, next dV/dK tile, K-V loads consumed
      int flags_even = 0, flags_odd = 0;  // flags of the last tiles whose S was issued
      long long last = clock64();
      while (np < n) {
        if (*abort_flag) break;
        bool did = false;
        if (np < ns && mbar_ready(&sm.pd_full, np & 1) &&
            (!kDq || np < 2 || mbar_ready(&sm.dq_free[np & 1], ((np >> 1) - 1) & 1))) {
          const int sq = np % kBsQStages, flags = (np & 1) ? flags_odd : flags_even;
          tc_fence_after();
          const uint64_t pdesc = sdesc_sw128(smem_u32(sm.p), 128 * 128, 1024);
          const uint64_t sdesc = sdesc_sw128(smem_u32(sm.ds), 128 * 128, 1024);
          const uint64_t odesc = sdesc_sw128(smem_u32(sm.dout[sq][0]), 128 * 128, 1024);
          const uint64_t qdesc = sdesc_sw128(smem_u32(sm.q[sq][0]), 128 * 128, 1024);
#pragma unroll
          for (int k = 0; k < 8; ++k) {  // 128 rows, 16 per MMA
            const uint64_t adv = static_cast<uint64_t>(k * (2048 >> 4));
            const uint32_t acc = ((flags & 1) && k == 0) ? 0u : 1u;
            umma_bf16_ss(tmem + kColAcc, odesc + adv, pdesc + adv, idT, acc);
            umma_bf16_ss(tmem + kColAcc + 64, qdesc + adv, sdesc + adv, idT, acc);
          }
          if constexpr (kDq) {
            const uint64_t kdesc = sdesc_sw128(smem_u32(sm.k[0]), 64 * 128, 1024);
#pragma unroll
            for (int k = 0; k < 4; ++k)  // 64 keys, 16 per MMA
              umma_bf16_ss(tmem + kColDQ + (np & 1) * 128, sdesc_sw128(smem_u32(sm.ds) + k * 32, 16, 1024),
                           kdesc + static_cast<uint64_t>(k * (2048 >> 4)), idQ, k > 0 ? 1u : 0u);
            umma_commit(&sm.dq_full[np & 1]);
          }
          umma_commit(&sm.pd_free);
          umma_commit(&sm.q_empty[sq]);
          if (flags & 2) {
            umma_commit(&sm.acc_full);
            umma_commit(&sm.kv_empty);  // K_j and V_j are no longer needed
          }
          ++np;
          did = true;
        } else if (ns < n && ns < np + 2) {
          const int si = ns % kBsInfo, sq = ns % kBsQStages;
          bool ready = mbar_ready(&sm.info_full[si], (ns / kBsInfo) & 1);
          int flags = 0;
          if (ready) {
            flags = sm.info[si].flags;
            if (flags & 1) ready = mbar_ready(&sm.kv_full, kv_seen & 1);
          }
          if (ready) ready = mbar_ready(&sm.q_full[sq], (ns / kBsQStages) & 1);
          if (ready && ns >= 1) ready = mbar_ready(&sm.s_free, (ns - 1) & 1);
          if (ready) {
            if (flags & 1) ++kv_seen;
            if (ns & 1) flags_odd = flags; else flags_even = flags;
            fence_proxy_async_smem();  // Q and dO were written by cp.async (generic proxy)
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < D / 16; ++k) {
              const int c = k >> 2, kk = k & 3;
              umma_bf16_ss(tmem, sdesc_sw128(smem_u32(sm.q[sq][c]) + kk * 32, 16, 1024),
                           sdesc_sw128(smem_u32(sm.k[c]) + kk * 32, 16, 1024), idS, k > 0 ? 1u : 0u);
            }
#pragma unroll
            for (int k = 0; k < D / 16; ++k) {
              const int c = k >> 2, kk = k & 3;
              umma_bf16_ss(tmem + 64, sdesc_sw128(smem_u32(sm.dout[sq][c]) + kk * 32, 16, 1024),
                           sdesc_sw128(smem_u32(sm.v[c]) + kk * 32, 16, 1024), idS, k > 0 ? 1u : 0u);
            }
            umma_commit(&sm.s_full);
            ++ns;
            did = true;
          }
        }
        if (did) {
          last = clock64();
        } else if (clock64() - last > kWaitCycles) {
          *abort_flag = 1;
          record_error(kErrWaitTimeout);
          break;
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ softmax / epilogue
    const int wg = (warp - kBsFirstSmx) >> 2;  // keys 32 wg .. 32 wg + 31
    const int q4 = warp & 3;                   // TMEM lane quadrant
    const int r = q4 * 32 + lane;              // tile row
    const uint32_t trow = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    uint8_t* prow = sm.p + r * 128;
    uint8_t* drow = sm.ds + r * 128;
    int nepi = 0;
    // the fp16 partial of tile x, this warpgroup's half of row r
    auto dq_out = [&](int x) -> bool {
      if (!warp_wait(&sm.dq_full[x & 1], (x >> 1) & 1, abort_flag)) return false;
      tc_fence_after();
      float v[64];
      tmem_ld32(trow + kColDQ + (x & 1) * 128 + 64 * wg, *reinterpret_cast<float(*)[32]>(&v[0]));
      tmem_ld32(trow + kColDQ + (x & 1) * 128 + 64 * wg + 32, *reinterpret_cast<float(*)[32]>(&v[32]));
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.dq_free[x & 1]);
      float am = 0.f;
#pragma unroll
      for (int c = 0; c < 64; ++c) am = fmaxf(am, fabsf(v[c]));
      // 65504 is the largest finite fp16 value; rare rows are scaled down by a power of two
      float c = 1.f;
      if (am > 32768.f && am <= 3.0e38f) c = exp2f(ceilf(log2f(am / 32768.f)));
      const float inv = 1.f / c;
      const size_t prow_g = static_cast<size_t>(tile_begin + x) * 128 + r;
      uint4* dst = reinterpret_cast<uint4*>(a.dq_part + prow_g * D + 64 * wg);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        uint4 w4;
        uint32_t* wp = reinterpret_cast<uint32_t*>(&w4);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const __half2 hv = __floats2half2_rn(v[8 * u + 2 * e] * inv, v[8 * u + 2 * e + 1] * inv);
          wp[e] = *reinterpret_cast<const uint32_t*>(&hv);
        }
        dst[u] = w4;
      }
      reinterpret_cast<float*>(a.part_scale)[2 * prow_g + wg] = c;
      return true;
    };
    for (int i = 0; i < n; ++i) {
      const int si = i % kBsInfo;
      if (!warp_wait(&sm.info_full[si], (i / kBsInfo) & 1, abort_flag)) break;
      const SelTileInfo& inf = sm.info[si];
      const int cnt = inf.cnt, key = inf.key, flags = inf.flags;
      const int g = key / a.nsel, j = key % a.nsel;
      const int tok = r / G, hh = r - (r / G) * G;
      const bool valid = tok < cnt;
      const int t = valid ? inf.ent[tok] >> 6 : 0;
      const int k0 = j * a.sel_len;
      const int key_hi = valid ? min(64, t + 1 - k0) - 32 * wg : 0;  // this thread's keys c < key_hi
      float lse2 = 0.f, dgr = 0.f, gate = 0.f;
      if (valid) {
        const size_t o = (static_cast<size_t>(t) * a.hq + g * G + hh) * 3 + kBwdSel;
        const float2 st = a.stats[o];
        lse2 = st.x;
        dgr = st.y;
        gate = a.gates[o];
      }
      const float gs = gate * a.scale;
      if (!warp_wait(&sm.s_full, i & 1, abort_flag)) break;
      tc_fence_after();
      float sv[32], dp[32];
      tmem_ld32(trow + 32 * wg, sv);
      tmem_ld32(trow + 64 + 32 * wg, dp);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.s_free);
      uint32_t pw[16], dw[16];
#pragma unroll
      for (int c = 0; c < 32; c += 2) {
        float pv[2], dv[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const bool vis = c + e < key_hi && lse2 != -INFINITY;
          const float p = vis ? ex2_approx(fmaf(sv[c + e], a.sl2, -lse2)) : 0.f;
          pv[e] = p * gate;
          dv[e] = p * gs * (dp[c + e] - dgr);
        }
        pw[c / 2] = pack_bf16x2(pv[0], pv[1]);
        dw[c / 2] = pack_bf16x2(dv[0], dv[1]);
      }
      // the previous tile's dV/dK products read the P and dS tiles
      if (i >= 1 && !warp_wait(&sm.pd_free, (i - 1) & 1, abort_flag)) break;
#pragma unroll
      for (int x = 0; x < 4; ++x) {  // 8 keys = one 16-byte unit of the swizzled row
        const int unit = wg * 4 + x;
        const uint32_t off = static_cast<uint32_t>((unit ^ (r & 7)) << 4);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(smem_u32(prow) + off), "r"(pw[4 * x]),
                     "r"(pw[4 * x + 1]), "r"(pw[4 * x + 2]), "r"(pw[4 * x + 3])
                     : "memory");
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(smem_u32(drow) + off), "r"(dw[4 * x]),
                     "r"(dw[4 * x + 1]), "r"(dw[4 * x + 2]), "r"(dw[4 * x + 3])
                     : "memory");
      }
      fence_proxy_async_smem();  // read by the tensor core (async proxy)
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.pd_full);
      // the previous tile's dq partial: read while this tile's products run
      if (kDq && i >= 1 && !dq_out(i - 1)) break;
      if (flags & 2) {
        // the bucket's sums: lane = dimension, column = key; warpgroup 0 dV, warpgroup 1 dK
        if (!warp_wait(&sm.acc_full, nepi & 1, abort_flag)) break;
        ++nepi;
        tc_fence_after();
        float accv[64];
        tmem_ld32(trow + kColAcc + 64 * wg, *reinterpret_cast<float(*)[32]>(&accv[0]));
        tmem_ld32(trow + kColAcc + 64 * wg + 32, *reinterpret_cast<float(*)[32]>(&accv[32]));
        tmem_wait_ld();
        tc_fence_before();
        float* dst = (wg == 0 ? a.dv : a.dk) + (static_cast<size_t>(k0) * a.hkv + g) * D + r;
        const size_t kstride = static_cast<size_t>(a.hkv) * D;
        const int nk = min(64, a.nv - k0);
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (c < nk) atomicAdd(dst + c * kstride, accv[c]);  // result unused: a reduction
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.info_empty[si]);
      if (kDq && i == n - 1) dq_out(i);
    }
  }

  // ------------------------------------------------------------------ teardown
  __syncthreads();
  if (*abort_flag) {
    // drain: wait (bounded) for the last K-V load and for MMAs in flight, so that no async
    // write lands after the CTA exits
    if (warp == 0 && lane == 0 && kv_issued > 0) {
      const long long t_start = clock64();
      while (!mbar_test(&sm.kv_full, (kv_issued - 1) & 1) && clock64() - t_start < kWaitCycles) {
      }
    }
    if (warp == kBsMmaWarp && lane == 0) {
      umma_commit(&sm.drain);
      const long long t_start = clock64();
      while (!mbar_test(&sm.drain, 0) && clock64() - t_start < kWaitCycles) {
      }
    }
    __syncwarp();
    __syncthreads();
  }
  if (warp == kBsMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace nsa

namespace nsa {

// ---------------------------------------------------------------- kept statistics
// Per video row (t, h), from what the forward kept: stats[row][b] = (lse_b log2 e, <dO, o_b>)
// and dgates[row][b] = <dO, o_b> for b = compressed, selected, window. One warp per row;
// lane l takes elements [l D/32, (l + 1) D/32).
template <int D>
__global__ void __launch_bounds__(256) bwd_stats_kernel(const BwdArgs a) {
  constexpr int kPer = D / 32;
  const long long row = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= static_cast<long long>(a.nv) * a.hq) return;
  const size_t off = static_cast<size_t>(row) * D + lane * kPer;
  float dov[kPer];
#pragma unroll
  for (int u = 0; u < kPer; u += 2) {
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(a.dout + off + u));
    dov[u] = f.x;
    dov[u + 1] = f.y;
  }
  const __half* ob[3] = {a.fwd_ocmp, a.fwd_osel, a.fwd_owin};
  const float* lb[3] = {a.fwd_lse, a.fwd_lse_sel, a.fwd_lse_win};
#pragma unroll
  for (int b = 0; b < 3; ++b) {
    float dot = 0.f;
#pragma unroll
    for (int u = 0; u < kPer; u += 2) {
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(ob[b] + off + u));
      dot = fmaf(dov[u], f.x, fmaf(dov[u + 1], f.y, dot));
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
    if (lane == 0) {
      const size_t o3 = static_cast<size_t>(row) * 3 + b;
      a.stats[o3] = make_float2(lb[b][row] * 1.4426950408889634f, dot);
      a.dgates[o3] = dot;
    }
  }
}

// ---------------------------------------------------------------- selected dq merge
// dq[t][h] += sum over the row's selected slots of its fp16 partial (times each half's factor).
// One warp per row; lane l takes elements [l D/32, (l + 1) D/32), in half (l D/32) / 64.
template <int D>
__global__ void __launch_bounds__(256) bwd_sel_dq_merge_kernel(const BwdArgs a) {
  constexpr int kPer = D / 32;
  const long long row = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= static_cast<long long>(a.nv) * a.hq) return;
  const int t = static_cast<int>(row / a.hq), h = static_cast<int>(row % a.hq);
  const int g = h / a.G, hh = h - g * a.G;
  const size_t base = (static_cast<size_t>(t) * a.hkv + g) * a.top_n;
  // lane s holds slot s (and s + 32): its partial row, or -1; top_n <= 64
  int r0 = -1, r1 = -1;
  if (lane < a.top_n && a.sel_idx[base + lane] >= 0) r0 = a.row_of[base + lane] + hh;
  if (lane + 32 < a.top_n && a.sel_idx[base + lane + 32] >= 0) r1 = a.row_of[base + lane + 32] + hh;
  const int half = (lane * kPer) >> 6;
  float acc[kPer];
#pragma unroll
  for (int u = 0; u < kPer; ++u) acc[u] = 0.f;
  for (int s0 = 0; s0 < a.top_n; s0 += 8) {
    uint2 raw[8];
    float c[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int s = s0 + k;
      int pr = __shfl_sync(0xffffffffu, s < 32 ? r0 : r1, s & 31);
      if (s >= a.top_n) pr = -1;
      raw[k] = make_uint2(0u, 0u);
      c[k] = 0.f;
      if (pr >= 0) {
        const __half* p = a.dq_part + static_cast<size_t>(pr) * D + lane * kPer;
        if constexpr (kPer == 4) raw[k] = *reinterpret_cast<const uint2*>(p);
        else raw[k].x = *reinterpret_cast<const uint32_t*>(p);
        c[k] = reinterpret_cast<const float*>(a.part_scale)[2 * static_cast<size_t>(pr) + half];
      }
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&raw[k].x));
      acc[0] = fmaf(c[k], f0.x, acc[0]);
      acc[1] = fmaf(c[k], f0.y, acc[1]);
      if constexpr (kPer == 4) {
        const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&raw[k].y));
        acc[2] = fmaf(c[k], f1.x, acc[2]);
        acc[3] = fmaf(c[k], f1.y, acc[3]);
      }
    }
  }
  float* dst = a.dq + static_cast<size_t>(row) * D + lane * kPer;
  if constexpr (kPer == 4) {
    float4 v = *reinterpret_cast<float4*>(dst);
    v.x += acc[0];
    v.y += acc[1];
    v.z += acc[2];
    v.w += acc[3];
    *reinterpret_cast<float4*>(dst) = v;
  } else {
    float2 v = *reinterpret_cast<float2*>(dst);
    v.x += acc[0];
    v.y += acc[1];
    *reinterpret_cast<float2*>(dst) = v;
  }
}

}  // namespace nsa
