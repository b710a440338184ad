// attn_tc.cuh -- tcgen05 / TMEM attention tile used by three steps of the NSA forward:
//
//   kModeCmp   compressed branch: queries attend to the block summaries Kc/Vc that are
//              complete at their position (block i visible to t iff i*s + l - 1 <= t).
//              Also bins the normalised probabilities into selection-block scores,
//              summed over the GQA group (the selection branch's importance scores;
//              top168.com article on VideoNSA, section "一、革命性的三重注意机制").
//   kModeWin   sliding-window branch over tokens (t - w, t]: o_win (fp16), which the
//              selected branch's merge then folds into the gated combine.
//   kModeDense dense causal rows for the trailing text tokens of the hybrid scheme
//              (shd-paper.top page "VideoNSA: ...", abstract: dense attention for text).
//
// One CTA owns one query tile: T = floor(128 / G) consecutive tokens times the G query
// heads of one KV group, packed as MMA rows r = token * G + head (the heads of a GQA
// group share every key, so they share the B operand). The tile's key range is streamed
// in 128-key tiles through a TMA ring, twice:
//   phase 1  S = Q K^T on the tensor core (TMEM accumulator), then each row's exact
//            log-sum-exp with an online max (no P*V, no output rescaling);
//   phase 2  S again, P = exp2(S*scale*log2e - lse2) already normalised, written to TMEM
//            as bf16 and accumulated O += P V in TMEM by a tcgen05 MMA that reads P
//            from TMEM. Because P is final, the compressed mode
//            can bin it into block scores in the same pass.
// The window and dense modes need no block scores: their phase 1 finds only the row max,
// phase 2 leaves P = exp2(S*scale*log2e - max) unnormalised, and the epilogue divides O
// by the row sum of P (half the exponentials of the two exact passes).
// K and V tiles stream through a ring of shared-memory slots (one tile each); the MMA
// releases a slot as soon as the MMA that read it is done.
// The pages' kernel notes (CSDN blog, section 5.1: fixed 64x64 blocks, prefetching the
// next block while computing the current one, tiling against register pressure) are
// met here by TMA tiles, an mbarrier ring and TMEM accumulators.
//
// Warp roles: warp 0 issues TMA loads, warp 1 owns TMEM and issues the MMAs (one elected
// lane), the softmax warpgroups (four in the compressed mode, two pairs taking turns on the
// key tiles; two otherwise; each thread owns one TMEM lane / MMA row and 64 key columns of a
// tile) do the softmax, the score binning and the epilogue. Every wait is bounded (sm100.cuh).
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>
#include "sm100.cuh"

namespace nsa {

enum AttnMode { kModeCmp = 0, kModeWin = 1, kModeDense = 2 };

struct AttnArgs {
  int q_begin, q_end;      // query tokens handled: [q_begin, q_end)
  int hq, hkv, G, T;       // heads, group size, tokens per tile
  int Gp;                  // MMA rows per token: G, or (kModeCmp) G rounded up to a power of two
  int n_tiles;             // ceil((q_end - q_begin) / T)
  float scale_log2;        // softmax_scale * log2(e)
  int cmp_len, cmp_stride;  // compressed-key visibility (kModeCmp)
  int window;              // kModeWin
  int sel_len;             // selection block (kModeCmp scores)
  __half* o_cmp;           // kModeCmp: write [N_v][Hq][d]
  float* lse;              // kModeCmp: write [N_v][Hq] (natural log)
  float* scores;           // kModeCmp: write [N_v][Hkv][nsel]
  int nsel;
  __half* o_win;           // kModeWin: write [N_v][Hq][d]
  float* lse_win;          // kModeWin: write [N_v][Hq] (natural log) when not null
  void* out;               // kModeDense: write [N][Hq][d]
  int out_f32;
  // Packed batches (null for one sequence). vinfo [video stream tokens]: per token the stream
  // index of its sequence's first video token (x), its sequence's first compressed-key row (y,
  // a multiple of 128), its sequence's first selection block (z) and its row in the packed
  // batch (w). tinfo [text stream rows] (kModeDense): per row its row in the packed batch (x)
  // and its sequence's first row there (y); keys are then rows of the packed batch.
  const int4* vinfo;
  const int2* tinfo;
};

// Softmax warpgroups, by mode. Two warpgroups share each S tile, one per 64-column half.
// The compressed mode (two exponentials and the block scores per element) runs two such
// pairs that take turns on the key tiles (pair p owns S buffer p): while one pair is in its
// exponentials the other loads, reduces and stores, so the exponential unit and the issue
// slots are not left idle by warps that all reach the same step at once. The window and
// dense modes (one exponential per element, a few tiles per item) run one pair, which
// measured faster for them than two.
template <int MODE>
struct AttnCfg {
  static constexpr int kPairs = MODE == 0 ? 2 : 1;  // warpgroup pairs taking turns on key tiles
  static constexpr int kWG = 2 * kPairs;
  static constexpr int kThreads = 64 + 128 * kWG;  // producer warp, MMA warp, softmax warps
  static constexpr int kCols = 64;                  // key columns per warpgroup per tile
  static constexpr int kBins = kCols / 4;           // selection blocks per warpgroup per tile
  static constexpr bool kPersistent = MODE != 0;    // one CTA per SM looping over the items
};
constexpr int kMaxSoftmaxWG = 4;
constexpr int kBN = 128;      // keys per tile

template <int D, int MODE>
struct AttnSmem {
  static constexpr int kChunks = D / 64;             // 64-element (128 B) column chunks
  static constexpr int kTileBytes = 128 * 128;       // one chunk of a 128-row tile
  static constexpr int kSlotBytes = kChunks * kTileBytes;
  // ring of K/V tile slots: as many as fit beside the Q tile in 227 KB
  static constexpr int kSlots = D == 128 ? 5 : 8;
  alignas(1024) uint8_t q[kChunks][kTileBytes];
  alignas(1024) uint8_t slot[kSlots][kChunks][kTileBytes];
  float lse_x[kMaxSoftmaxWG][128][2];  // per warpgroup: (scaled max, sum) of the row's columns
  float carry[2][128];                 // (compressed, two pairs) half of a tile's last block, per row
  uint64_t carry_full[2], carry_free[2];
  uint64_t q_full, q_tmem, q_empty, qcols_free;
  uint64_t full[kSlots], empty[kSlots];
  uint64_t s_full[2], s_free[2];
  uint64_t p_full, p_free[2], o_full, o_free, drain;
  uint32_t tmem_base;
  int abort_flag;
};

// P (bf16, packed in pairs) goes to its own double-buffered TMEM columns and is read back
// by the tensor core as the A operand of the P.V MMA ("TS" form: A from TMEM; a column
// holds two consecutive keys, the lower key in the low half).
__device__ __forceinline__ void umma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[0]),
               "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// Sum over 32 columns of 2^(s*sl2 - ms), in 8 independent chains.
__device__ __forceinline__ float chunk_sum_ex2(const float (&s)[32], float sl2, float ms) {
  float acc[8];
#pragma unroll
  for (int c = 0; c < 8; c += 2) {
    float x0, x1;
    fma2(x0, x1, s[c], s[c + 1], sl2, -ms);
    acc[c] = ex2_approx(x0);
    acc[c + 1] = ex2_approx(x1);
  }
#pragma unroll
  for (int i = 8; i < 32; i += 8)
#pragma unroll
    for (int c = 0; c < 8; c += 2) {
      float x0, x1;
      fma2(x0, x1, s[i + c], s[i + c + 1], sl2, -ms);
      add2(acc[c], acc[c + 1], ex2_approx(x0), ex2_approx(x1));
    }
  add2(acc[0], acc[1], acc[2], acc[3]);
  add2(acc[4], acc[5], acc[6], acc[7]);
  add2(acc[0], acc[1], acc[4], acc[5]);
  return acc[0] + acc[1];
}

// s[i] = 2^(s[i]*sl2 - off) for the columns kbase+i in [rb, re), 0 elsewhere.
__device__ __forceinline__ void chunk_ex2(float (&s)[32], float sl2, float off, bool full, int kbase, int rb, int re) {
  if (full) {
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
      float x0, x1;
      fma2(x0, x1, s[i], s[i + 1], sl2, -off);
      s[i] = ex2_approx(x0);
      s[i + 1] = ex2_approx(x1);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int kidx = kbase + i;
      s[i] = (kidx >= rb && kidx < re) ? ex2_approx(fmaf(s[i], sl2, -off)) : 0.f;
    }
  }
}

// TMA load sequence of a tile: phase 1 reads K(0 .. nkt-1); phase 2 reads K(0), K(1), V(0),
// K(2), V(1), ..., K(nkt-1), V(nkt-2), V(nkt-1): each K tile comes one step ahead of the V
// tile issued beside it, because the score MMA runs two jobs ahead of the P.V MMA.
__device__ __forceinline__ int p2_k_pos(int x) { return x == 0 ? 0 : 2 * x - 1; }
__device__ __forceinline__ int p2_v_pos(int x, int nkt) { return min(2 * x + 2, 2 * nkt - 1); }
__device__ __forceinline__ void p2_item(int p, int nkt, bool& is_v, int& x) {
  if (p == 0) {
    is_v = false;
    x = 0;
  } else if (p == 2 * nkt - 1) {
    is_v = true;
    x = nkt - 1;
  } else if (p & 1) {
    is_v = false;
    x = (p + 1) >> 1;
  } else {
    is_v = true;
    x = (p >> 1) - 1;
  }
}

__device__ __forceinline__ int ncmp_visible(int t, int l, int s) { return (t + 1 >= l) ? (t + 1 - l) / s + 1 : 0; }

// Reduce over groups of GP adjacent lanes of NB per-lane values. With GP <= NB each lane
// ends with NB/GP group sums, bin[0 .. NB/GP) = entries [(l%GP)*NB/GP, ...). With GP > NB
// the halving stops at one entry and the remaining stages add; lane l then holds entry
// (l%GP) / (GP/NB), shared with the GP/NB - 1 lanes next to it.
template <int GP, int NB, int O = GP / 2, int N = NB>
__device__ __forceinline__ void group_reduce_scatter(float (&bin)[NB], int lane) {
  // one halving stage per lane bit O (compile-time recursion: every bin index is static)
  if constexpr (O >= 1) {
    if constexpr (N > 1) {
      const bool upper = (lane & O) != 0;
#pragma unroll
      for (int i = 0; i < N / 2; ++i) {
        const float send = upper ? bin[i] : bin[i + N / 2];
        const float keep = upper ? bin[i + N / 2] : bin[i];
        bin[i] = keep + __shfl_xor_sync(0xffffffffu, send, O);
      }
      group_reduce_scatter<GP, NB, O / 2, N / 2>(bin, lane);
    } else {
      bin[0] += __shfl_xor_sync(0xffffffffu, bin[0], O);
      group_reduce_scatter<GP, NB, O / 2, N>(bin, lane);
    }
  }
}

// PACKED: the rows belong to a packed batch (AttnArgs::vinfo / tinfo); a single sequence
// compiles without those lookups.
template <int D, int MODE, bool PACKED = false>
__global__ void __launch_bounds__(AttnCfg<MODE>::kThreads, 1)
    attn_tile_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                     const __grid_constant__ CUtensorMap vmap, const AttnArgs args) {
  using Smem = AttnSmem<D, MODE>;
  constexpr int kChunks = Smem::kChunks;
  constexpr int kSoftmaxWG = AttnCfg<MODE>::kWG;
  constexpr int kPairs = AttnCfg<MODE>::kPairs;
  constexpr int kTileWG = kSoftmaxWG / kPairs;  // warpgroups that share one S tile
  constexpr int kSoftmaxThreads = 128 * kSoftmaxWG;
  constexpr int kColsPerWG = AttnCfg<MODE>::kCols;
  constexpr int kBinsPerWG = AttnCfg<MODE>::kBins;
  constexpr uint32_t kTmemCols = 512;
  constexpr uint32_t kColO = 256;  // S buffers at columns 0 and 128, O at 256
  constexpr uint32_t kColP = 384;  // P (bf16 pairs, 64 columns)
  constexpr uint32_t kColQ = 448;  // Q (bf16 pairs, D/2 columns): the A operand of every S MMA
  constexpr int kSlots = Smem::kSlots;
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int G = args.G, T = args.T;
  // Work items (query tile, KV group), heavy tiles (most keys) first for the causal modes.
  // Window and dense: one CTA per SM, persistent, CTA c taking items c, c + gridDim.x, ...,
  // so each item's start overlaps the previous item's epilogue (these items are short).
  // Compressed: one item per CTA (its items are long, and the hardware's launch order then
  // balances them); the loops below run once and compile as such.
  constexpr bool kPersist = AttnCfg<MODE>::kPersistent;
  const int n_items = args.n_tiles * args.hkv;
  auto item_geo = [&](int item, int& g, int& t0, int& kb, int& nkt) {
    const int rank = item / args.hkv;
    g = item % args.hkv;
    const int tile = (MODE == kModeWin) ? rank : (args.n_tiles - 1 - rank);
    t0 = args.q_begin + tile * T;
    const int t_last = min(t0 + T, args.q_end) - 1;
    // the tile's key range runs from its first row's first key to its last row's last key
    // (rows are in order, and so are their sequences)
    int ke;
    if (MODE == kModeCmp) {
      if ((PACKED && args.vinfo != nullptr)) {
        const int4 a = args.vinfo[t0], z = args.vinfo[t_last];
        kb = a.y;
        ke = z.y + ncmp_visible(t_last - z.x, args.cmp_len, args.cmp_stride);
      } else {
        kb = 0;
        ke = ncmp_visible(t_last, args.cmp_len, args.cmp_stride);
      }
    } else if (MODE == kModeWin) {
      kb = max((PACKED && args.vinfo != nullptr) ? args.vinfo[t0].x : 0, t0 - args.window + 1);
      ke = t_last + 1;
    } else if ((PACKED && args.tinfo != nullptr)) {
      kb = args.tinfo[t0].y;
      ke = args.tinfo[t_last].x + 1;
    } else {
      kb = 0;
      ke = t_last + 1;
    }
    nkt = (ke - kb + kBN - 1) / kBN;
  };

  if (tid == 0) {
    mbar_init(&sm.q_full, 1);
    mbar_init(&sm.q_tmem, 4 * kSoftmaxWG);
    mbar_init(&sm.q_empty, 4 * kSoftmaxWG);
    mbar_init(&sm.qcols_free, 1);
    for (int x = 0; x < Smem::kSlots; ++x) {
      mbar_init(&sm.full[x], 1);
      mbar_init(&sm.empty[x], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.s_full[b], 1);
      mbar_init(&sm.s_free[b], 4 * kTileWG);
      mbar_init(&sm.carry_full[b], 4);
      mbar_init(&sm.carry_free[b], 4);
    }
    mbar_init(&sm.p_full, 4 * kTileWG);
    mbar_init(&sm.p_free[0], 1);
    mbar_init(&sm.p_free[1], 1);
    mbar_init(&sm.o_full, 1);
    mbar_init(&sm.o_free, 4 * kSoftmaxWG);
    mbar_init(&sm.drain, 1);
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (warp >= 2) {
    // rows T*Gp .. 127 of the Q tile are never written by TMA: keep them finite (zero)
    const int r0 = T * args.Gp;
    for (int i = tid - 64; i < (128 - r0) * 8 * kChunks; i += kSoftmaxThreads) {
      const int c = i / ((128 - r0) * 8);
      const int rem = i % ((128 - r0) * 8);
      *reinterpret_cast<uint4*>(&sm.q[c][(r0 + rem / 8) * 128 + (rem % 8) * 16]) = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort_flag = &sm.abort_flag;
  int issued = 0;    // producer: K/V loads whose TMA was issued
  int q_issued = 0;  // producer: Q tiles whose TMA was issued
  bool leader = false;  // MMA warp: the lane that issues every tcgen05 op

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    // Per item: its Q tile (into the single Q buffer, once the softmax warps have moved the
    // previous one into TMEM), then its K/V loads. Load l of an item: l < nkt -> K tile l
    // (phase 1); else position l - nkt of the phase-2 sequence (p2_item). The CTA-wide load
    // counter L picks slot L % kSlots, which is reused once the MMA has released load
    // L - kSlots. The next item's Q is issued as soon as the buffer frees up.
    if (lane == 0 && blockIdx.x < n_items) {
      tma_prefetch_desc(&qmap);
      tma_prefetch_desc(&kmap);
      tma_prefetch_desc(&vmap);
      auto load_q = [&](int item) {
        int g, t0, kb, nkt;
        item_geo(item, g, t0, kb, nkt);
        mbar_arrive_expect_tx(&sm.q_full, kChunks * T * args.Gp * 128);
        for (int c = 0; c < kChunks; ++c) tma_load_3d(&qmap, &sm.q_full, sm.q[c], c * 64, g * G, t0);
        ++q_issued;
      };
      load_q(blockIdx.x);
      bool ok = true;
      int L = 0;
      for (int it = 0; ok && (kPersist || it == 0); ++it) {
        const int item = blockIdx.x + it * gridDim.x;
        if (item >= n_items) break;
        int g, t0, kb, nkt;
        item_geo(item, g, t0, kb, nkt);
        const bool has_next = kPersist && item + static_cast<int>(gridDim.x) < n_items;
        bool next_q = !has_next;
        for (int l = 0; l < 3 * nkt; ++l, ++L) {
          if (!next_q && mbar_ready(&sm.q_empty, it & 1)) {
            load_q(item + gridDim.x);
            next_q = true;
          }
          const int x = L % kSlots;
          if (L >= kSlots && !mbar_wait(&sm.empty[x], ((L / kSlots) - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          bool is_v = false;
          int kt = l;
          if (l >= nkt) p2_item(l - nkt, nkt, is_v, kt);
          const int kpos = kb + kt * kBN;
          mbar_arrive_expect_tx(&sm.full[x], Smem::kSlotBytes);
          for (int c = 0; c < kChunks; ++c)
            tma_load_3d(is_v ? &vmap : &kmap, &sm.full[x], sm.slot[x][c], c * 64, g, kpos);
          issued = L + 1;
        }
        if (ok && !next_q) {
          if (!mbar_wait(&sm.q_empty, it & 1, abort_flag)) break;
          load_q(item + gridDim.x);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    // The whole warp runs the issue loop (waits, descriptor arithmetic) in lockstep and one
    // elected lane issues each tcgen05 instruction: the operands stay warp-uniform, so the
    // issuing warp needs few of the scheduler's slots, which it shares with four softmax warps.
    // Barrier phases run on across items: an item has 2*nkt MMA jobs (nkt per S buffer),
    // nkt P.V products and 3*nkt loads, so `base` (the CTA's tiles so far) fixes every parity.
    leader = elect_one_sync();
    constexpr uint32_t idS = idesc_bf16_f32(128, kBN, false, false);
    constexpr uint32_t idO = idesc_bf16_f32(128, D, false, true);
    auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
    };
    bool ok = true;
    int base = 0;
    for (int it = 0; ok && (kPersist || it == 0); ++it) {
      const int item = blockIdx.x + it * gridDim.x;
      if (item >= n_items) break;
      int g, t0, kb, nkt;
      item_geo(item, g, t0, kb, nkt);
      const int njobs = 2 * nkt;
      ok = wait_all(&sm.q_tmem, it & 1);  // Q staged in TMEM by the softmax warps
      auto wait_load = [&](int l) -> bool {
        const int L = 3 * base + l;
        return wait_all(&sm.full[L % kSlots], (L / kSlots) & 1);
      };
      auto issue_s = [&](int job) -> bool {
        const int l = job < nkt ? job : nkt + p2_k_pos(job - nkt);
        const int x = (3 * base + l) % kSlots;
        const int b = job & 1;
        if (!wait_load(l)) return false;
        // S(job) reuses the buffer of the job two before it (possibly of the previous item)
        const int use = base + (job >> 1);
        if (use >= 1 && !wait_all(&sm.s_free[b], (use - 1) & 1)) return false;
        tc_fence_after();
        // A = Q from TMEM (dims 16k .. 16k+15 in columns kColQ + 8k ..), B = K from smem;
        // the B descriptor advances by constant offsets (start address field in 16-byte units)
        const uint64_t kdesc = sdesc_sw128(smem_u32(sm.slot[x][0]), 16, 1024);
        const uint32_t sbuf = tmem + b * kBN, qcol = tmem + kColQ;
        if (leader) {
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const int c = k >> 2, kk = k & 3;
            const uint64_t bd = kdesc + static_cast<uint64_t>((c * Smem::kTileBytes + kk * 32) >> 4);
            umma_bf16_ts(sbuf, qcol + k * 8, bd, idS, k > 0 ? 1u : 0u);
          }
          umma_commit(&sm.s_full[b]);
          umma_commit(&sm.empty[x]);  // the K tile is no longer needed
          // after the item's last score tile, Q's TMEM columns may take the next item's Q
          if (job == njobs - 1) umma_commit(&sm.qcols_free);
        }
        __syncwarp();
        return true;
      };
      // Score tiles run two jobs ahead: S(job + 2) waits only for its buffer, which the pair
      // that read S(job) frees as soon as the scores are in registers, so it computes while
      // that pair is still in its softmax; P.V(job) follows once P(job) is in TMEM.
      if (ok && njobs > 0) ok = issue_s(0);
      if (ok && njobs > 1) ok = issue_s(1);
      for (int job = 0; ok && job < njobs; ++job) {
        if (job + 2 < njobs && !issue_s(job + 2)) {
          ok = false;
          break;
        }
        if (job >= nkt) {
          const int kt2 = job - nkt;
          const int l = nkt + p2_v_pos(kt2, nkt);  // V tile
          const int x = (3 * base + l) % kSlots;
          if (!wait_load(l) || !wait_all(&sm.p_full, (base + kt2) & 1)) {
            ok = false;
            break;
          }
          // the first P.V of an item overwrites O: the previous item's epilogue has read it
          if (kt2 == 0 && it > 0 && !wait_all(&sm.o_free, (it - 1) & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t vdesc = sdesc_sw128(smem_u32(sm.slot[x][0]), Smem::kTileBytes, 1024);
          const uint32_t ocol = tmem + kColO, pcol = tmem + kColP;
          if (leader) {
#pragma unroll
            for (int k = 0; k < kBN / 16; ++k)  // keys 16k .. 16k+15 (P columns kColP + 8k ..)
              umma_bf16_ts(ocol, pcol + k * 8, vdesc + static_cast<uint64_t>(k * (2048 >> 4)), idO,
                           (kt2 > 0 || k > 0) ? 1u : 0u);
            // this P.V (and its reads of P from TMEM) is done; counted per pair of the tile
            umma_commit(&sm.p_free[kPairs == 1 ? 0 : (job & 1)]);
            umma_commit(&sm.empty[x]);  // the V tile is no longer needed
          }
          __syncwarp();
        }
      }
      // An item without keys commits at once; it still waits for the previous item's epilogue,
      // so o_full never completes twice before the softmax warps have waited for the first
      // of the two (the waits tell phases apart by parity only).
      if (ok && njobs == 0 && it > 0) ok = wait_all(&sm.o_free, (it - 1) & 1);
      if (ok && leader) {
        if (njobs == 0) umma_commit(&sm.qcols_free);  // (no MMA of this item: arrives at once)
        umma_commit(&sm.o_full);
      }
      __syncwarp();
      base += nkt;
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ softmax / epilogue
    // Warpgroup `wg` belongs to pair wg / kTileWG, which handles the MMA jobs (S tiles) of
    // parity `pair` (S buffer `pair`); within the pair it owns key columns
    // [half*64, half*64+64) of each 128-key tile. In the epilogue it owns D/kSoftmaxWG output
    // columns. Its thread of TMEM lane r handles MMA row r.
    const int sw = warp - 2;                 // softmax warp
    const int wg = sw >> 2;                  // warpgroup
    const int pair = wg / kTileWG;
    const int half = wg % kTileWG;           // column slice within a tile
    const int q4 = warp & 3;                 // TMEM lane quadrant of this warp
    const int r = q4 * 32 + lane;            // MMA row
    const int Gp = args.Gp;
    const int tok = r / Gp, hh = r % Gp;
    const uint32_t trow = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const int col0 = half * kColsPerWG;
    const float sl2 = args.scale_log2;
    // (kModeCmp) the scores are reduced over the heads per 32-column chunk (8 selection
    // blocks): lane hh then holds blocks [hh*bpl, (hh+1)*bpl) of the chunk (Gp <= 8), or block
    // hh/share shared with its neighbours (Gp > 8)
    constexpr int kChunkBins = 8;  // selection blocks per 32-column chunk
    const int sc_bpl = Gp <= kChunkBins ? kChunkBins / Gp : 1;
    const int sc_share = Gp <= kChunkBins ? 1 : Gp / kChunkBins;
    const int sc_j0 = half * kBinsPerWG + (hh / sc_share) * sc_bpl;
    // (kModeCmp) carry slot `p` takes half of column 127 of the tiles of pair p (written by
    // its upper half, read by the lower half of the other pair); uses counted across items
    int carry_writes = 0, carry_reads = 0;
    int other_pv = 0;  // (two pairs) P.V products of the other pair's tiles in earlier items
    bool ok = true;

    // ---- Q rows into TMEM, packed in bf16 pairs like P: this warpgroup copies dims
    // [wg*D/kSoftmaxWG, ...) of row r from the 128-byte-swizzled smem image (16-byte unit u
    // of a row sits at unit u ^ (row & 7)); rows past the tile are the zeros written at the
    // start. Q of item `it` waits for its TMA and, after the first item, for the last score
    // MMA of the previous item (which read the same TMEM columns).
    auto stage_q = [&](int it) -> bool {
      bool w = mbar_wait(&sm.q_full, it & 1, abort_flag);
      if (w && it > 0) w = mbar_wait(&sm.qcols_free, (it - 1) & 1, abort_flag);
      if (!__all_sync(0xffffffffu, w)) return false;
      tc_fence_after();
      constexpr int kDimsPerWG = D / kSoftmaxWG;  // 32 or 64 (D=128), 16 or 32 (D=64)
      uint32_t qv[kDimsPerWG / 2];
#pragma unroll
      for (int i = 0; i < kDimsPerWG / 8; ++i) {
        const int dim0 = wg * kDimsPerWG + 8 * i;
        const int c = dim0 / 64, u = (dim0 % 64) / 8;
        const uint4 w4 = *reinterpret_cast<const uint4*>(&sm.q[c][r * 128 + ((u ^ (r & 7)) << 4)]);
        qv[4 * i] = w4.x;
        qv[4 * i + 1] = w4.y;
        qv[4 * i + 2] = w4.z;
        qv[4 * i + 3] = w4.w;
      }
      __syncwarp();
      if constexpr (kDimsPerWG / 2 >= 16) {
#pragma unroll
        for (int hx = 0; hx < kDimsPerWG / 32; ++hx)
          tmem_st16(trow + kColQ + wg * (kDimsPerWG / 2) + 16 * hx,
                    *reinterpret_cast<const uint32_t(*)[16]>(&qv[16 * hx]));
      } else {
        tmem_st8(trow + kColQ + wg * 8, *reinterpret_cast<const uint32_t(*)[8]>(&qv[0]));
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&sm.q_tmem);
        mbar_arrive(&sm.q_empty);  // the smem Q buffer may take the next item's tile
      }
      return true;
    };
    if (blockIdx.x < n_items) ok = stage_q(0);

    // Every softmax thread runs every item, also after a failed wait (its waits are then
    // skipped): the named barriers below are passed the same number of times by all of them.
    int base = 0;
    for (int it = 0; kPersist || it == 0; ++it) {
      const int item = blockIdx.x + it * gridDim.x;
      if (item >= n_items) break;
      int g, t0, kb, nkt;
      item_geo(item, g, t0, kb, nkt);
      const int t = t0 + tok;
      const int h = g * G + hh;
      const bool row_valid = (r < T * Gp) && (hh < G) && (t < args.q_end);
      int rb = 0, re = 0;  // visible key range of this row
      int s_first = 0;     // (packed) stream index of the first video token of the row's sequence
      if (row_valid) {
        if (MODE == kModeCmp) {
          if ((PACKED && args.vinfo != nullptr)) {
            const int4 a = args.vinfo[t];
            s_first = a.x;
            rb = a.y;
            re = a.y + ncmp_visible(t - a.x, args.cmp_len, args.cmp_stride);
          } else {
            re = ncmp_visible(t, args.cmp_len, args.cmp_stride);
          }
        } else if (MODE == kModeWin) {
          if ((PACKED && args.vinfo != nullptr)) s_first = args.vinfo[t].x;
          rb = max(s_first, t - args.window + 1);
          re = t + 1;
        } else if ((PACKED && args.tinfo != nullptr)) {
          const int2 a = args.tinfo[t];
          rb = a.y;
          re = a.x + 1;
        } else {
          re = t + 1;
        }
      }
      // ---- phase 1: log-sum-exp (base 2) of this row's column slice, combined below
      float m = -INFINITY, lsum = 0.f;  // m: running max of the raw (unscaled) scores
      for (int kt = kPairs == 1 ? 0 : pair; kt < nkt && ok; kt += kPairs) {
        const int b = kt & 1;
        // tcgen05.ld is warp-collective: every wait result is made warp-uniform
        ok = __all_sync(0xffffffffu, mbar_wait(&sm.s_full[b], (base + (kt >> 1)) & 1, abort_flag));
        if (!ok) break;
        tc_fence_after();
        const int kbase = kb + kt * kBN + col0;
        // warp-uniform: the unmasked path only when every row of the warp sees the whole
        // slice; rows without keys (head padding, past the end) follow the others, their
        // probabilities being forced to 0 through lse2 = +inf
        const bool full = __all_sync(0xffffffffu, !row_valid || (kbase >= rb && kbase + kColsPerWG <= re));
        // the slice's columns are loaded with one wait, and S is released at once; then 32
        // columns at a time (an online max across the chunks)
        static_assert(kColsPerWG % 32 == 0, "phase 1 reads 32-column chunks");
        float s_all[kColsPerWG];
        __syncwarp();
#pragma unroll
        for (int hc = 0; hc < kColsPerWG / 32; ++hc)
          tmem_ld32(trow + b * kBN + col0 + 32 * hc, *reinterpret_cast<float(*)[32]>(&s_all[32 * hc]));
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.s_free[b]);  // S is in registers: the buffer may be reused
        if (!full) {
#pragma unroll
          for (int i = 0; i < kColsPerWG; ++i) {
            const int kidx = kbase + i;
            s_all[i] = (kidx >= rb && kidx < re) ? s_all[i] : -INFINITY;
          }
        }
        // one max over the whole slice (eight independent chains), then one rescale of the sum
        float mx[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) mx[c] = fmaxf(s_all[c], s_all[c + 8]);
#pragma unroll
        for (int c = 16; c < kColsPerWG; c += 16)
#pragma unroll
          for (int u = 0; u < 8; ++u) mx[u] = fmax3f(mx[u], s_all[c + u], s_all[c + 8 + u]);
        const float cmax = fmax3f(fmax3f(mx[0], mx[1], mx[2]), fmax3f(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
        const float mnew = fmaxf(m, cmax);
        if (MODE != kModeCmp) {
          m = mnew;  // the window and dense branches need only the row max here
        } else if (mnew != -INFINITY) {
          const float ms = mnew * sl2;
          float part = 0.f;
#pragma unroll
          for (int hc = 0; hc < kColsPerWG / 32; ++hc)
            part += chunk_sum_ex2(*reinterpret_cast<float(*)[32]>(&s_all[32 * hc]), sl2, ms);
          lsum = lsum * ex2_approx((m - mnew) * sl2) + part;
          m = mnew;
        }
      }
      sm.lse_x[wg][r][0] = (m == -INFINITY) ? -INFINITY : m * sl2;
      sm.lse_x[wg][r][1] = lsum;
      named_bar_sync(3, kSoftmaxThreads);
      float lse2;
      bool has_keys;
      {
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kSoftmaxWG; ++w) M = fmaxf(M, sm.lse_x[w][r][0]);
        float Lsum = 0.f;
        if (M != -INFINITY) {
#pragma unroll
          for (int w = 0; w < kSoftmaxWG; ++w) Lsum += sm.lse_x[w][r][1] * ex2_approx(sm.lse_x[w][r][0] - M);
        }
        if (MODE == kModeCmp) {
          has_keys = row_valid && Lsum > 0.f;
          lse2 = has_keys ? M + __log2f(Lsum) : INFINITY;
        } else {
          // P = exp2(S*scale*log2e - max) unnormalised; the row sum divides O at the end
          has_keys = row_valid && M != -INFINITY;
          lse2 = has_keys ? M : INFINITY;
        }
      }
      float psum = 0.f;  // (window, dense) this thread's part of the row sum of P
      // ---- phase 2: normalised probabilities -> P (TMEM, bf16) and block scores
      // Block scores (kModeCmp): compressed block i covers tokens [16i, 16i+32) and selection
      // block j covers [64j, 64j+64), so block j takes all of compressed blocks 4j..4j+2 and
      // half of 4j-1 and 4j+3. A 128-key tile holds selection blocks kt2*32 .. kt2*32+31;
      // this warpgroup's columns hold kBinsPerWG of them. The compressed block that straddles
      // the two column halves (column 63) is re-read from TMEM by the upper half. The one that
      // straddles two tiles (column 127 of the previous tile, which the other pair handled)
      // arrives through a shared-memory slot: the upper half of each tile leaves half of its
      // column-127 probability there and the lower half of the next tile picks it up (guarded
      // by carry_full / carry_free). The G heads of a token sit in Gp adjacent lanes; a shuffle
      // reduce-scatter sums them.
      float carry_last = 0.f;  // upper half, last tile: half of its last compressed block
      const bool sc_store = MODE == kModeCmp && t < args.q_end && (hh % sc_share) == 0;
      // (packed) a row whose sequence starts after the tile's first key row sees its own
      // blocks from column (rb - kb) on, a multiple of 128: its block indices are offset by
      // sc_joff; rows padding the tile hold no position
      int sc_jt = t / args.sel_len, sc_joff = 0;
      if (MODE == kModeCmp && (PACKED && args.vinfo != nullptr)) {
        const int4 a = args.vinfo[min(t, args.q_end - 1)];
        sc_jt = (t - a.x) / args.sel_len;
        sc_joff = (a.y - kb) / 4;
      }
      float* const sc_dst = args.scores + (static_cast<size_t>(t) * args.hkv + g) * args.nsel;
      // this pair's phase-2 jobs are those of parity `pair`: job nkt + kt2
      for (int kt2 = kPairs == 1 ? 0 : ((pair + nkt) & 1); ok && kt2 < nkt; kt2 += kPairs) {
        const int job = nkt + kt2;
        const int b = job & 1;
        ok = __all_sync(0xffffffffu, mbar_wait(&sm.s_full[b], (base + (job >> 1)) & 1, abort_flag));
        if (!ok) break;
        tc_fence_after();
        const int kbase = kb + kt2 * kBN + col0;
        const bool full = __all_sync(0xffffffffu, !row_valid || (kbase >= rb && kbase + kColsPerWG <= re));
        float half_in = 0.f;
        // 32 columns at a time: read from TMEM, exponentials, then (kModeCmp) the chunk's 8
        // block scores, then the chunk's P packed to bf16 pairs, so only one chunk is ever held
        // in fp32
        static_assert(kColsPerWG % 32 == 0, "P is stored 16 columns (32 keys) at a time");
        uint32_t pk[kColsPerWG / 2];
        float prev_last = 0.f;  // (kModeCmp) p of the previous chunk's last column
        // window / dense: the slice's columns with one wait, S released at once. Compressed:
        // chunk by chunk (its P and block scores leave no registers for a second chunk)
        float s2_all[kColsPerWG];
        uint32_t xv = 0;
        auto release_s = [&]() {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.s_free[b]);  // S is in registers: the buffer may be reused
        };
        if constexpr (MODE != kModeCmp) {
          __syncwarp();
#pragma unroll
          for (int hc = 0; hc < kColsPerWG / 32; ++hc)
            tmem_ld32(trow + b * kBN + col0 + 32 * hc, *reinterpret_cast<float(*)[32]>(&s2_all[32 * hc]));
          tmem_wait_ld();
          release_s();
        }
#pragma unroll
        for (int hc = 0; hc < kColsPerWG / 32; ++hc) {
          float(&sc)[32] = *reinterpret_cast<float(*)[32]>(&s2_all[32 * hc]);
          if constexpr (MODE == kModeCmp) {
            __syncwarp();
            tmem_ld32(trow + b * kBN + col0 + 32 * hc, sc);
            if (hc == 0 && half > 0)
              asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(xv) : "r"(trow + b * kBN + col0 - 1));
            tmem_wait_ld();
            if (hc == kColsPerWG / 32 - 1) release_s();
          }
          if (MODE == kModeCmp && hc == 0 && half > 0) {
            const int xk = kb + kt2 * kBN + col0 - 1;
            half_in = (xk >= rb && xk < re) ? 0.5f * ex2_approx(fmaf(__uint_as_float(xv), sl2, -lse2)) : 0.f;
          }
          chunk_ex2(sc, sl2, lse2, full, kbase + 32 * hc, rb, re);
          if (MODE != kModeCmp) {
            float ps[4] = {sc[0], sc[1], sc[2], sc[3]};
#pragma unroll
            for (int i = 4; i < 32; i += 4) {
              add2(ps[0], ps[1], sc[i], sc[i + 1]);
              add2(ps[2], ps[3], sc[i + 2], sc[i + 3]);
            }
            add2(ps[0], ps[1], ps[2], ps[3]);
            psum += ps[0] + ps[1];
          }
          if (MODE == kModeCmp) {
            if (hc == 0 && half == 0 && kt2 > 0) {
              // half of the previous tile's column 127, left by the other pair in its slot
              const int slot = pair ^ 1;
              if (ok) ok = mbar_wait(&sm.carry_full[slot], carry_reads & 1, abort_flag);
              half_in = sm.carry[slot][r];
              ++carry_reads;
              __syncwarp();
              if (lane == 0) mbar_arrive(&sm.carry_free[slot]);
            }
            if (hc == kColsPerWG / 32 - 1 && half == kTileWG - 1) {
              // hand half of column 127 to the next tile's lower half (the other pair)
              const float c127 = 0.5f * sc[31];
              if (kt2 + 1 < nkt) {
                const int slot = pair;
                if (carry_writes > 0 && ok)
                  ok = mbar_wait(&sm.carry_free[slot], (carry_writes - 1) & 1, abort_flag);
                sm.carry[slot][r] = c127;
                ++carry_writes;
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.carry_full[slot]);
              } else {
                carry_last = c127;
              }
            }
            // bins u and u + 1 in one paired pass; the compressed block between them (4u + 3)
            // gives half to each
            float bin[kChunkBins];
            static_assert(kChunkBins % 2 == 0, "bins are computed in pairs");
#pragma unroll
            for (int u = 0; u < kChunkBins; u += 2) {
              // the outer halves: block 4u - 1 (left of bin u; 2 x half_in is exact) and 4u + 7
              const float outer = u > 0 ? sc[4 * u - 1] : (hc == 0 ? 2.f * half_in : prev_last);
              float b0 = sc[4 * u], b1 = sc[4 * u + 4];
              add2(b0, b1, sc[4 * u + 1], sc[4 * u + 5]);
              add2(b0, b1, sc[4 * u + 2], sc[4 * u + 6]);
              fma2v(b0, b1, sc[4 * u + 3], sc[4 * u + 3], 0.5f, b0, b1);
              fma2v(bin[u], bin[u + 1], outer, sc[4 * u + 7], 0.5f, b0, b1);
            }
            prev_last = sc[31];
            switch (Gp) {
              case 2: group_reduce_scatter<2, kChunkBins>(bin, lane); break;
              case 4: group_reduce_scatter<4, kChunkBins>(bin, lane); break;
              case 8: group_reduce_scatter<8, kChunkBins>(bin, lane); break;
              case 16: group_reduce_scatter<16, kChunkBins>(bin, lane); break;
              default: break;
            }
            if (sc_store) {
              const int j0 = kt2 * 32 + hc * kChunkBins + sc_j0 - sc_joff;
              if (sc_bpl == 1) {
                if (j0 >= 0 && j0 <= sc_jt) sc_dst[j0] = bin[0];
              } else {
#pragma unroll
                for (int i = 0; i < kChunkBins; ++i)
                  if (i < sc_bpl && j0 + i >= 0 && j0 + i <= sc_jt) sc_dst[j0 + i] = bin[i];
              }
            }
          }
#pragma unroll
          for (int i = 0; i < 16; ++i) pk[16 * hc + i] = pack_bf16x2(sc[2 * i], sc[2 * i + 1]);
        }
        // P row r, keys col0 .. col0+kColsPerWG-1 -> packed bf16 pairs in TMEM columns
        // kColP + col0/2 .. . P(kt2) is stored only once the P.V MMA of the previous tile has
        // finished: tcgen05.st into TMEM while a P.V that reads its A operand from TMEM was
        // still running corrupted rows 0-31 of the output on B200 even while P was
        // double-buffered in disjoint columns; with that wait in place one P buffer suffices.
        // The wait comes after the exponentials, which overlap the previous P.V. The P.V of
        // tile kt2 - 1 is the last one before it: its completion (counted on the barrier of the
        // pair that owned that tile) means every earlier P.V has finished too. For the first
        // tile of an item the previous item's epilogue already saw all of its P.V products
        // finish.
        if (ok && kt2 > 0) {
          if (kPairs == 1) {
            ok = mbar_wait(&sm.p_free[0], (base + kt2 - 1) & 1, abort_flag);
          } else {
            // P.V products of the other pair up to tile kt2 - 1 (its tiles are those whose job
            // nkt + k has its parity): the last of them is the one to wait for
            const int other = pair ^ 1;
            const int n = other_pv + ((kt2 + (other == (nkt & 1) ? 1 : 0)) >> 1) - 1;
            ok = mbar_wait(&sm.p_free[other], n & 1, abort_flag);
          }
        }
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
#pragma unroll
        for (int hc = 0; hc < kColsPerWG / 32; ++hc)
          tmem_st16(trow + kColP + col0 / 2 + 16 * hc, *reinterpret_cast<const uint32_t(*)[16]>(&pk[16 * hc]));
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.p_full);
      }
      if (MODE == kModeCmp && ok && wg == kSoftmaxWG - 1) {
        // the half-block after the last tile lands in selection block nkt*32; the last
        // phase-2 job (2*nkt - 1) is odd, so this warpgroup (upper half of pair 1) holds it.
        // When no key tile exists at all, that is block 0 with score 0.
        float c = carry_last;
#pragma unroll
        for (int o = 1; o < 16; o <<= 1)
          if (o < Gp) c += __shfl_xor_sync(0xffffffffu, c, o);
        const int j = nkt * 32 - sc_joff;
        if (hh == 0 && t < args.q_end && j >= 0 && j <= sc_jt)
          args.scores[(static_cast<size_t>(t) * args.hkv + g) * args.nsel + j] = c;
      }
      float inv_l = 1.f;  // (window, dense) 1 / row sum of P over all column slices
      if (MODE != kModeCmp) {
        sm.lse_x[wg][r][1] = psum;
        named_bar_sync(3, kSoftmaxThreads);
        float Lsum = 0.f;
#pragma unroll
        for (int w = 0; w < kSoftmaxWG; ++w) Lsum += sm.lse_x[w][r][1];
        inv_l = Lsum > 0.f ? 1.f / Lsum : 0.f;
      }
      // the next item's Q goes into TMEM now, so its score MMAs overlap this epilogue
      if (kPersist && ok && item + static_cast<int>(gridDim.x) < n_items) ok = stage_q(it + 1);
      // ---- epilogue (every lane loads its TMEM row; only valid rows are stored)
      if (ok) {
        ok = __all_sync(0xffffffffu, mbar_wait(&sm.o_full, it & 1, abort_flag));
        tc_fence_after();
      }
      // (after a failed wait the work below is skipped, but the named barrier is still passed)
      const size_t orow = (static_cast<size_t>(t) * args.hq + h) * D;
      // (packed text rows) the dense output goes to the row's place in the packed batch
      const size_t drow = (MODE == kModeDense && (PACKED && args.tinfo != nullptr) && row_valid)
                              ? (static_cast<size_t>(args.tinfo[t].x) * args.hq + h) * D
                              : orow;
      constexpr int kOC = D / kSoftmaxWG < 32 ? D / kSoftmaxWG : 32;  // output columns per load
      constexpr int kOLoads = (D / kSoftmaxWG + 31) / 32;
      float o[kOLoads][32];
      // O row r, this warpgroup's columns: into registers, then O's TMEM may take the next
      // item's P.V while the stores run
      __syncwarp();
      if (ok) {
#pragma unroll
        for (int cc = 0; cc < kOLoads; ++cc) {
          const int c0 = wg * (D / kSoftmaxWG) + cc * 32;
          if (kOC == 32) {
            tmem_ld32(trow + kColO + c0, o[cc]);
          } else {
            tmem_ld16(trow + kColO + c0, *reinterpret_cast<float(*)[16]>(&o[cc][0]));
          }
        }
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.o_free);
      }
      if (!ok || nkt == 0) {
#pragma unroll
        for (int cc = 0; cc < kOLoads; ++cc)
#pragma unroll
          for (int i = 0; i < 32; ++i) o[cc][i] = 0.f;
      }
      if constexpr (MODE == kModeWin) {
        // o_win = O / row sum in fp16, this warpgroup's columns of row r (the gated combine
        // reads it in the selected branch's merge, whole rows per warp)
        static_assert(kOC % 8 == 0, "o_win is written in 8-column units");
        if (ok && row_valid) {
#pragma unroll
          for (int cc = 0; cc < kOLoads; ++cc) {
            const int c0 = wg * (D / kSoftmaxWG) + cc * 32;
            uint4* dst = reinterpret_cast<uint4*>(args.o_win + orow + c0);
#pragma unroll
            for (int u8 = 0; u8 < kOC / 8; ++u8) {
              uint4 w4;
              uint32_t* wp = reinterpret_cast<uint32_t*>(&w4);
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const __half2 hv =
                    __floats2half2_rn(o[cc][u8 * 8 + 2 * i] * inv_l, o[cc][u8 * 8 + 2 * i + 1] * inv_l);
                wp[i] = *reinterpret_cast<const uint32_t*>(&hv);
              }
              dst[u8] = w4;
            }
          }
        }
      } else {
#pragma unroll
        for (int cc = 0; cc < kOLoads; ++cc) {
          const int c0 = wg * (D / kSoftmaxWG) + cc * 32;  // output columns c0 .. c0+kOC-1
          float* oc_ = o[cc];
          if (!row_valid || !ok) {
            // nothing to store for padding rows
          } else if (MODE == kModeCmp) {
            uint4* dst = reinterpret_cast<uint4*>(args.o_cmp + orow + c0);
#pragma unroll
            for (int u = 0; u < kOC / 8; ++u) {
              uint4 w4;
              uint32_t* wp = reinterpret_cast<uint32_t*>(&w4);
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const __half2 hv = __floats2half2_rn(oc_[8 * u + 2 * i], oc_[8 * u + 2 * i + 1]);
                wp[i] = *reinterpret_cast<const uint32_t*>(&hv);
              }
              dst[u] = w4;
            }
          } else {
#pragma unroll
            for (int u = 0; u < kOC; ++u) oc_[u] *= inv_l;
            if (args.out_f32) {
              float4* dst = reinterpret_cast<float4*>(static_cast<float*>(args.out) + drow + c0);
#pragma unroll
              for (int u = 0; u < kOC / 4; ++u)
                dst[u] = make_float4(oc_[4 * u], oc_[4 * u + 1], oc_[4 * u + 2], oc_[4 * u + 3]);
            } else {
              uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(args.out) + drow + c0);
#pragma unroll
              for (int u = 0; u < kOC / 8; ++u)
                dst[u] = make_uint4(pack_bf16x2(oc_[8 * u], oc_[8 * u + 1]), pack_bf16x2(oc_[8 * u + 2], oc_[8 * u + 3]),
                                    pack_bf16x2(oc_[8 * u + 4], oc_[8 * u + 5]), pack_bf16x2(oc_[8 * u + 6], oc_[8 * u + 7]));
            }
          }
        }
      }
      if (MODE == kModeCmp && ok && row_valid && wg == 0)
        args.lse[static_cast<size_t>(t) * args.hq + h] = has_keys ? lse2 * 0.69314718055994530942f : -INFINITY;
      // (window) lse2 holds the row max and 1 / inv_l the row sum of exp2(S*sl2 - max)
      if (MODE == kModeWin && args.lse_win != nullptr && ok && row_valid && wg == 0)
        args.lse_win[static_cast<size_t>(t) * args.hq + h] =
            has_keys && inv_l > 0.f ? (lse2 - __log2f(inv_l)) * 0.69314718055994530942f : -INFINITY;
      base += nkt;
      other_pv += (nkt + ((pair ^ 1) == (nkt & 1) ? 1 : 0)) >> 1;
    }
    tc_fence_before();
  }

  // ------------------------------------------------------------------ teardown
  __syncthreads();
  if (*abort_flag) {
    // drain: wait (bounded) for TMA loads that were issued but never consumed and for
    // MMAs still in flight, so no async write lands after the CTA exits.
    if (warp == 0 && lane == 0) {
      if (q_issued > 0) {
        const long long t_start = clock64();
        while (!mbar_test(&sm.q_full, (q_issued - 1) & 1) && clock64() - t_start < kWaitCycles) {
        }
      }
      // the last load issued into each slot (earlier ones completed before it was issued)
      for (int L = issued - kSlots > 0 ? issued - kSlots : 0; L < issued; ++L) {
        const long long t_start = clock64();
        while (!mbar_test(&sm.full[L % kSlots], (L / kSlots) & 1) && clock64() - t_start < kWaitCycles) {
        }
      }
    }
    if (warp == 1) {
      // the commit tracks the MMAs of the lane that issued them
      if (leader) {
        umma_commit(&sm.drain);
        const long long t_start = clock64();
        while (!mbar_test(&sm.drain, 0) && clock64() - t_start < kWaitCycles) {
        }
      }
    }
    __syncwarp();
    __syncthreads();
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace nsa
