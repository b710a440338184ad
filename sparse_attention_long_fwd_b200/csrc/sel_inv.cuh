// sel_inv.cuh -- selection branch, step 3 (prefill), block-major form.
//
// Every (token, KV group) attends to its own top-n blocks of 64 tokens (selection branch,
// top168.com article on VideoNSA, section "一、革命性的三重注意机制"). Gathering each
// token's blocks separately moves every block once per token that chose it. Here the loop
// is inverted: the (token, slot) pairs are bucketed by (group, block), and one CTA takes
// up to 128/Gp tokens that chose the same block, so the block's 64 keys and values are
// loaded once and the tensor core runs full 128-row tiles (token x head rows, heads
// padded to Gp, a power of two). Each row's softmax over that block gives a partial
// (max, sum, output / sum); sel_merge_kernel combines a row's partials as an online softmax
// would. The sum is taken over the bf16-rounded P that the tensor core multiplies, so each
// partial is an exact convex combination of values. Partials live in tile order: tile k
// owns rows 128k .. 128k+127 (MMA row r = token slot r / Gp, head slot r % Gp), so a warp
// writes its 32 rows with one TMA store per 64 output columns (Gp = G: 7 heads pack 18 tokens
// into 126 rows; the last two rows are unused); sel_scatter_kernel records
// where each (token, group, slot) landed. The partial output is stored in fp16 (2^-12
// relative rounding); a 64-column half whose largest magnitude would overflow fp16 is
// stored divided by a power of two c, kept with the row's (max, sum).
//
//   sel_count_kernel    entries per (group, block)
//   sel_scan_kernel     exclusive scans of entries and of tiles per (group, block)
//   sel_scatter_kernel  bucket (token, slot) pairs
//   sel_tile_kernel     persistent 128-row tcgen05 tiles: S = Q K^T, softmax, O = P V
//   sel_merge_kernel    o_sel[t][h] from the row's partials, then the gated combine
//                       out = g_cmp*o_cmp + g_sel*o_sel + g_win*o_win (o_sel is not stored)
#pragma once
#include <cuda_fp16.h>
#include "attn_tc.cuh"

namespace nsa {

struct SelInvArgs {
  int nv, hq, hkv, G, Gp, TT;   // rows: TT tokens x Gp head slots per tile
  int nsel, top_n, sel_len;
  float sl2;
  const int32_t* sel_idx;       // [nv][hkv][top_n]
  int* cnt;                     // [hkv*nsel] entries per (group, block); zeroed by the host
  int* cursor;                  // [hkv*nsel] scatter cursors; zeroed by the host
  int* ent_off;                 // [hkv*nsel + 1] exclusive scan of cnt
  int* tile_off;                // [hkv*nsel + 1] exclusive scan of ceil(cnt/TT)
  int* list;                    // [nv*hkv*top_n] bucketed entries: t * 64 + slot
  int* row_of;                  // [nv][hkv][top_n] first partial row of each (token, group, slot)
  const __nv_bfloat16* q;       // [nv][hq][D]
  long long part_rows;          // partial rows (128 x the tile bound)
  const __half* part_o;         // [part_rows][D] output / (sum * c_half) of each partial, half h in
                                // columns [64h, 64h+64): a row is one contiguous 2D-byte segment
  float4* part_ml;              // [part_rows] (max in log2 units, sum, c of half 0, c of half 1)
  const __half* o_cmp;          // [nv][hq][D] compressed branch
  const __half* o_win;          // [nv][hq][D] sliding-window branch
  const float* gates;           // [N][hq][3] (g_cmp, g_sel, g_win)
  void* out;                    // [N][hq][D] rows < nv: the gated combine, bf16 or fp32
  int out_f32;
  __half* o_sel;                // [nv][hq][D] the selected branch's output, kept when not null
  float* lse_sel;               // [nv][hq] its log-sum-exp (natural log), kept with o_sel
  // Packed batches (null for one sequence): vinfo as in AttnArgs (token -> its sequence's
  // first stream token, first selection block and its row in the batch); blk_tok [nsel]: the
  // stream token where each selection block starts. Block j of a row's sequence is bucket
  // column vinfo.z + j (nsel counts the blocks of all sequences), and out / gates use the
  // row in the batch.
  const int4* vinfo;
  const int* blk_tok;
};

// Bucket column of block j of token t: its sequence's blocks come after the earlier sequences'.
__device__ __forceinline__ int sel_block_col(const SelInvArgs& a, int t, int j) {
  return a.vinfo != nullptr ? a.vinfo[t].z + j : j;
}

// Block 0 is kept by every token, so its buckets take one entry per token of their group:
// those entries are counted (and, in the scatter, placed) per CTA in shared memory and
// added to the global counters once per CTA, instead of by one global atomic each.
__global__ void __launch_bounds__(256) sel_count_kernel(const SelInvArgs a) {
  __shared__ int zero_cnt[16];
  if (threadIdx.x < 16) zero_cnt[threadIdx.x] = 0;
  __syncthreads();
  const long long n = static_cast<long long>(a.nv) * a.hkv * a.top_n;
  for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < n;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int j = a.sel_idx[e];
    const int g = static_cast<int>((e / a.top_n) % a.hkv);
    if (j == 0 && g < 16 && a.vinfo == nullptr) {
      atomicAdd(&zero_cnt[g], 1);
    } else if (j >= 0 && j < a.nsel) {
      const int t = static_cast<int>(e / (static_cast<long long>(a.top_n) * a.hkv));
      atomicAdd(&a.cnt[g * a.nsel + sel_block_col(a, t, j)], 1);
    }
  }
  __syncthreads();
  if (threadIdx.x < min(a.hkv, 16) && zero_cnt[threadIdx.x] > 0)
    atomicAdd(&a.cnt[threadIdx.x * a.nsel], zero_cnt[threadIdx.x]);
}

// One CTA of 1024 threads scans hkv*nsel counters (<= 16 * 8192).
__global__ void __launch_bounds__(1024) sel_scan_kernel(const SelInvArgs a) {
  __shared__ int wsum_e[32], wsum_t[32];
  __shared__ int carry_e, carry_t;
  const int m = a.hkv * a.nsel;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) {
    carry_e = 0;
    carry_t = 0;
  }
  __syncthreads();
  for (int base = 0; base < m; base += 1024) {
    const int i = base + tid;
    const int ce = i < m ? a.cnt[i] : 0;
    const int ct = (ce + a.TT - 1) / a.TT;
    int se = ce, st = ct;  // inclusive warp scans
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int ye = __shfl_up_sync(0xffffffffu, se, o);
      const int yt = __shfl_up_sync(0xffffffffu, st, o);
      if (lane >= o) {
        se += ye;
        st += yt;
      }
    }
    if (lane == 31) {
      wsum_e[warp] = se;
      wsum_t[warp] = st;
    }
    __syncthreads();
    if (warp == 0) {
      int xe = wsum_e[lane], xt = wsum_t[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int ye = __shfl_up_sync(0xffffffffu, xe, o);
        const int yt = __shfl_up_sync(0xffffffffu, xt, o);
        if (lane >= o) {
          xe += ye;
          xt += yt;
        }
      }
      wsum_e[lane] = xe;  // inclusive over warps
      wsum_t[lane] = xt;
    }
    __syncthreads();
    const int pe = (warp > 0 ? wsum_e[warp - 1] : 0) + se - ce + carry_e;
    const int pt = (warp > 0 ? wsum_t[warp - 1] : 0) + st - ct + carry_t;
    if (i < m) {
      a.ent_off[i] = pe;
      a.tile_off[i] = pt;
    }
    __syncthreads();
    if (tid == 0) {
      carry_e += wsum_e[31];
      carry_t += wsum_t[31];
    }
    __syncthreads();
  }
  if (tid == 0) {
    a.ent_off[m] = carry_e;
    a.tile_off[m] = carry_t;
  }
}

__global__ void __launch_bounds__(256) sel_scatter_kernel(const SelInvArgs a) {
  __shared__ int zero_cnt[16], zero_base[16];
  const long long n = static_cast<long long>(a.nv) * a.hkv * a.top_n;
  // rounds of blockDim.x consecutive entries; every thread takes part in every round
  for (long long base = static_cast<long long>(blockIdx.x) * blockDim.x; base < n;
       base += static_cast<long long>(gridDim.x) * blockDim.x) {
    if (threadIdx.x < 16) zero_cnt[threadIdx.x] = 0;
    __syncthreads();
    const long long e = base + threadIdx.x;
    const int j = e < n ? a.sel_idx[e] : -1;
    const bool valid = j >= 0 && j < a.nsel;
    const int slot = static_cast<int>(e % a.top_n);
    const long long tg = e / a.top_n;
    const int g = static_cast<int>(tg % a.hkv);
    const int t = static_cast<int>(tg / a.hkv);
    const int key = g * a.nsel + (valid ? sel_block_col(a, t, j) : 0);
    // groups past 16, and the per-sequence block 0 of packed batches, use the global counter
    const bool agg = valid && j == 0 && g < 16 && a.vinfo == nullptr;
    int local = 0;
    if (agg) local = atomicAdd(&zero_cnt[g], 1);
    else if (valid) local = atomicAdd(&a.cursor[key], 1);
    __syncthreads();
    if (threadIdx.x < min(a.hkv, 16) && zero_cnt[threadIdx.x] > 0)
      zero_base[threadIdx.x] = atomicAdd(&a.cursor[threadIdx.x * a.nsel], zero_cnt[threadIdx.x]);
    __syncthreads();
    if (valid) {
      if (agg) local += zero_base[g];
      a.list[a.ent_off[key] + local] = t * 64 + slot;
      a.row_of[e] = (a.tile_off[key] + local / a.TT) * 128 + (local % a.TT) * a.Gp;
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------- partial attention tiles
// Persistent: one CTA per SM takes a contiguous range of bucket tiles, so consecutive
// tiles of the same (group, block) reuse the K and V already in shared memory.
//   warps 0..2   producers: warp 0 writes the tile records (list entries prefetched two
//                tiles ahead) and loads K and V by TMA once per bucket; all three gather
//                the tile's Q rows (32-row blocks) with 16-byte cp.async straight into the
//                128-byte-swizzled layout (one small TMA box per token was issue-bound)
//   warp 3       MMA issuer: S = Q K^T into the TMEM of the tile's warpgroup, then O = P V,
//                issuing whichever of the next S or the next P.V has its inputs ready
//   warps 4..15  three softmax / epilogue warpgroups taking tiles in turn; thread = MMA row
// A warpgroup's 128 TMEM columns hold S (64 columns) and, once S has been read, O over it.
// P goes from registers to shared memory (128-byte swizzled, K-major) and the P.V product
// reads it there, so no thread writes TMEM while an MMA runs.
constexpr int kSelWG = 3;
constexpr int kSelProducers = 3;
constexpr int kSelMmaWarp = kSelProducers;
constexpr int kSelFirstSmxWarp = kSelProducers + 1;
constexpr int kSelTileThreads = 32 * kSelFirstSmxWarp + kSelWG * 128;  // 16 warps: 128 registers each
constexpr int kSelQStages = 3;
constexpr int kSelKVStages = 2;
constexpr int kSelInfo = 8;

struct SelTileInfo {
  int key, cnt, kvs, flags;  // flags: 1 = first tile of its K/V stage, 2 = last
  int ent[128];
};

template <int D>
struct SelTileSmem {
  static constexpr int kChunks = D / 64;
  alignas(1024) uint8_t q[kSelQStages][kChunks][128 * 128];
  alignas(1024) uint8_t k[kSelKVStages][kChunks][64 * 128];
  alignas(1024) uint8_t v[kSelKVStages][kChunks][64 * 128];
  alignas(1024) uint8_t p[kSelWG][128 * 128];  // 128 rows x 64 keys bf16
  SelTileInfo info[kSelInfo];
  uint64_t q_full[kSelQStages], q_empty[kSelQStages];
  uint64_t kv_full[kSelKVStages], kv_empty[kSelKVStages];
  uint64_t info_full[kSelInfo], info_empty[kSelInfo];
  uint64_t s_full[kSelWG], p_full[kSelWG], o_full[kSelWG], o_free[kSelWG];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

// Bounded wait by every lane of a warp, with a warp-uniform result.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
}

__device__ __forceinline__ void cp_async16_cg(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
// The barrier receives one arrival once all of this thread's earlier cp.async copies land.
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Tile record of the producer: bucket, first list entry, entry count, last-of-bucket, and
// (prefetched) list entries x = lane + 32k.
struct SelTileMeta {
  int key, e0, cnt, last;
  int e[4];
};

template <int D>
__global__ void __launch_bounds__(kSelTileThreads, 1)
    sel_tile_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                    const __grid_constant__ CUtensorMap omap, const SelInvArgs a) {
  using Smem = SelTileSmem<D>;
  constexpr int kChunks = Smem::kChunks;
  constexpr int kCpr = D / 8;          // 16-byte pieces per Q row
  constexpr uint32_t kTmemCols = 512;  // warpgroup w: columns 128w .. 128w+127 (S, then O)
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int m = a.hkv * a.nsel;
  const long long total = a.tile_off[m];
  const int tile_begin = static_cast<int>(total * blockIdx.x / gridDim.x);
  const int tile_end = static_cast<int>(total * (blockIdx.x + 1) / gridDim.x);
  const int n = tile_end - tile_begin;
  if (n <= 0) return;  // uniform across the CTA
  if (tid == 0) {
    for (int s = 0; s < kSelQStages; ++s) {
      mbar_init(&sm.q_full[s], kSelProducers * 32);  // one cp.async arrival per producer lane
      mbar_init(&sm.q_empty[s], 1);
    }
    for (int s = 0; s < kSelKVStages; ++s) {
      mbar_init(&sm.kv_full[s], 1);
      mbar_init(&sm.kv_empty[s], 1);
    }
    for (int s = 0; s < kSelInfo; ++s) {
      mbar_init(&sm.info_full[s], 1);
      mbar_init(&sm.info_empty[s], 4);
    }
    for (int w = 0; w < kSelWG; ++w) {
      mbar_init(&sm.s_full[w], 1);
      mbar_init(&sm.p_full[w], 4);
      mbar_init(&sm.o_full[w], 1);
      mbar_init(&sm.o_free[w], 4);
    }
    mbar_init(&sm.drain, 1);
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kSelMmaWarp) {
    tmem_alloc(&sm.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort_flag = &sm.abort_flag;
  const int Gp = a.Gp, G = a.G;
  int kv_issued = 0;  // warp 0: K-V loads issued

  if (warp < kSelProducers) {
    // ------------------------------------------------------------------ producers
    int key = 0, t_base = 0, t_next = 0, e_base = 0, e_next = 0;
    SelTileMeta m0{}, m1{}, m2{};
    auto fetch = [&](int tile) {
      SelTileMeta r;
      while (t_next <= tile) {  // next bucket with tiles
        ++key;
        t_base = t_next;
        e_base = e_next;
        t_next = a.tile_off[key + 1];
        e_next = a.ent_off[key + 1];
      }
      r.key = key;
      r.e0 = e_base + (tile - t_base) * a.TT;
      r.cnt = min(a.TT, e_next - r.e0);
      r.last = (tile == tile_end - 1) || (t_next == tile + 1);
#pragma unroll
      for (int k = 0; k < 4; ++k) r.e[k] = (lane + 32 * k < r.cnt) ? a.list[r.e0 + lane + 32 * k] : 0;
      return r;
    };
    if (warp == 0) {
      if (lane == 0) {
        tma_prefetch_desc(&kmap);
        tma_prefetch_desc(&vmap);
        int lo = 0, hi = m - 1;  // bucket of the first tile: the last key with tile_off[key] <= tile_begin
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if (a.tile_off[mid] <= tile_begin) lo = mid; else hi = mid - 1;
        }
        key = lo;
      }
      key = __shfl_sync(0xffffffffu, key, 0);
      t_base = a.tile_off[key];
      t_next = a.tile_off[key + 1];
      e_base = a.ent_off[key];
      e_next = a.ent_off[key + 1];
      m0 = fetch(tile_begin);
      if (n > 1) m1 = fetch(tile_begin + 1);
      if (n > 2) m2 = fetch(tile_begin + 2);
    }
    int kv_key = -1;
    // one tile; `cur` is warp 0's record of tile i, refilled with tile i + 3 at the end (in
    // place: moving records whose list loads are in flight would wait for those loads)
    auto tile_step = [&](int i, SelTileMeta& cur) -> bool {
      const int si = i % kSelInfo, sq = i % kSelQStages;
      SelTileInfo& inf = sm.info[si];
      if (warp == 0) {
        if (i >= kSelInfo && !warp_wait(&sm.info_empty[si], ((i / kSelInfo) - 1) & 1, abort_flag)) return false;
        const bool first = cur.key != kv_key;
        const int kvs = first ? kv_issued % kSelKVStages : (kv_issued - 1) % kSelKVStages;
#pragma unroll
        for (int k = 0; k < 4; ++k)
          if (lane + 32 * k < cur.cnt) inf.ent[lane + 32 * k] = cur.e[k];
        if (lane == 0) {
          inf.key = cur.key;
          inf.cnt = cur.cnt;
          inf.kvs = kvs;
          inf.flags = (first ? 1 : 0) | (cur.last ? 2 : 0);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.info_full[si]);
      } else if (!warp_wait(&sm.info_full[si], (i / kSelInfo) & 1, abort_flag)) {
        return false;
      }
      // Q rows of this tile: row R = token slot R / Gp, head slot R % Gp; this warp takes the
      // 32-row blocks b with b % kSelProducers == (warp + 1) % kSelProducers (warp 0, which
      // also writes the records, takes the fewest)
      if (i >= kSelQStages && !warp_wait(&sm.q_empty[sq], ((i / kSelQStages) - 1) & 1, abort_flag)) return false;
      {
        const int cnt = inf.cnt;
        const int g = inf.key / a.nsel;
        for (int b = (warp + 1) % kSelProducers; b < 4; b += kSelProducers) {
          const int rbase = b * 32;
          // lane L finds the source row of tile row rbase + L (-1: not loaded); the copy loop
          // then takes row it * kRpi + lane / kCpr in iteration it, piece lane % kCpr of it
          int my_row = -1;
          {
            const int R = rbase + lane;
            const int tok = R / Gp, hh = R - tok * Gp;
            if (tok < cnt && hh < G && g * G + hh < a.hq) my_row = (inf.ent[tok] >> 6) * a.hq + g * G + hh;
          }
          constexpr int kRpi = 32 / kCpr;  // rows per iteration
          const int sub = lane / kCpr, c16 = lane % kCpr;
          const char* src_lane = reinterpret_cast<const char*>(a.q) + c16 * 16;
          // 128-byte swizzle: piece (c16 & 7) of row R sits at unit (c16 & 7) ^ (R & 7); R & 7 =
          // ((it * kRpi) & 7) ^ sub because rbase is a multiple of 32 and sub < kRpi
          const uint32_t dst_lane = smem_u32(sm.q[sq][0]) + (c16 >> 3) * (128 * 128) + (rbase + sub) * 128;
          const uint32_t x_lane = (c16 & 7) ^ sub;
#pragma unroll
          for (int it = 0; it < kCpr; ++it) {
            const int row = __shfl_sync(0xffffffffu, my_row, it * kRpi + sub);
            const uint32_t dst = dst_lane + it * kRpi * 128 + ((x_lane ^ ((it * kRpi) & 7)) << 4);
            if (row >= 0) cp_async16_cg(dst, src_lane + static_cast<size_t>(row) * (D * 2));
          }
        }
        cp_async_arrive_noinc(&sm.q_full[sq]);
      }
      if (warp == 0) {
        if (cur.key != kv_key) {
          const int u = kv_issued;  // K-V load number
          const int kvs = u % kSelKVStages;
          if (u >= kSelKVStages && !warp_wait(&sm.kv_empty[kvs], ((u / kSelKVStages) - 1) & 1, abort_flag)) return false;
          if (lane == 0) {
            const int g = cur.key / a.nsel, j = cur.key % a.nsel;
            const int k0 = a.blk_tok != nullptr ? a.blk_tok[j] : j * a.sel_len;  // first key token
            mbar_arrive_expect_tx(&sm.kv_full[kvs], kChunks * 2 * 64 * 128);
            for (int c = 0; c < kChunks; ++c) {
              tma_load_3d(&kmap, &sm.kv_full[kvs], sm.k[kvs][c], c * 64, g, k0);
              tma_load_3d(&vmap, &sm.kv_full[kvs], sm.v[kvs][c], c * 64, g, k0);
            }
          }
          __syncwarp();
          kv_issued = u + 1;
          kv_key = cur.key;
        }
        if (i + 3 < n) cur = fetch(tile_begin + i + 3);
      }
      return true;
    };
    for (int i = 0; i < n; i += 3) {
      if (!tile_step(i, m0)) break;
      if (i + 1 < n && !tile_step(i + 1, m1)) break;
      if (i + 2 < n && !tile_step(i + 2, m2)) break;
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
  } else if (warp == kSelMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(128, 64, false, false);
      constexpr uint32_t idO = idesc_bf16_f32(128, D, false, true);
      int ns = 0, np = 0, kv_seen = 0;  // next S tile, next P.V tile, K-V loads consumed
      long long last = clock64();
      while (np < n) {
        if (*abort_flag) break;
        bool did = false;
        if (np < ns && mbar_ready(&sm.p_full[np % kSelWG], (np / kSelWG) & 1)) {
          // O = P V over the warpgroup's columns (S there has been read)
          const int w = np % kSelWG;
          const SelTileInfo& inf = sm.info[np % kSelInfo];
          const int kvs = inf.kvs, flags = inf.flags;
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < 4; ++k)  // 64 keys, 16 per MMA
            umma_bf16_ss(tmem + w * 128, sdesc_sw128(smem_u32(sm.p[w]) + k * 32, 16, 1024),
                         sdesc_sw128(smem_u32(sm.v[kvs][0]) + k * 2048, 64 * 128, 1024), idO, k > 0 ? 1u : 0u);
          umma_commit(&sm.o_full[w]);
          if (flags & 2) umma_commit(&sm.kv_empty[kvs]);
          ++np;
          did = true;
        } else if (ns < n) {
          const int w = ns % kSelWG, jj = ns / kSelWG;
          const int si = ns % kSelInfo, sq = ns % kSelQStages;
          bool ready = mbar_ready(&sm.info_full[si], (ns / kSelInfo) & 1);
          int kvs = 0, flags = 0;
          if (ready) {
            kvs = sm.info[si].kvs;
            flags = sm.info[si].flags;
            if (flags & 1) ready = mbar_ready(&sm.kv_full[kvs], (kv_seen / kSelKVStages) & 1);
          }
          if (ready) ready = mbar_ready(&sm.q_full[sq], (ns / kSelQStages) & 1);
          if (ready && jj >= 1) ready = mbar_ready(&sm.o_free[w], (jj - 1) & 1);  // O of the last tile read
          if (ready) {
            if (flags & 1) ++kv_seen;
            fence_proxy_async_smem();  // Q was written by cp.async (generic proxy); the MMA reads it
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < D / 16; ++k) {
              const int c = k >> 2, kk = k & 3;
              umma_bf16_ss(tmem + w * 128, sdesc_sw128(smem_u32(sm.q[sq][c]) + kk * 32, 16, 1024),
                           sdesc_sw128(smem_u32(sm.k[kvs][c]) + kk * 32, 16, 1024), idS, k > 0 ? 1u : 0u);
            }
            umma_commit(&sm.s_full[w]);
            umma_commit(&sm.q_empty[sq]);
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
  } else if (warp >= kSelFirstSmxWarp) {
    // ------------------------------------------------------------------ softmax / epilogue
    const int w = (warp - kSelFirstSmxWarp) >> 2;  // warpgroup
    const int q4 = warp & 3;         // TMEM lane quadrant
    const int r = q4 * 32 + lane;    // MMA row: token slot r / Gp, head slot r % Gp
    const int hh = r % Gp;
    const uint32_t trow = tmem + (static_cast<uint32_t>(q4 * 32) << 16) + w * 128;
    uint8_t* prow_smem = sm.p[w] + r * 128;
    for (int i = w; i < n; i += kSelWG) {
      const int jj = i / kSelWG;
      const int si = i % kSelInfo;
      if (!warp_wait(&sm.info_full[si], (i / kSelInfo) & 1, abort_flag)) break;
      const SelTileInfo& inf = sm.info[si];
      const int cnt = inf.cnt, key = inf.key;
      const int j = key % a.nsel;
      const int tok = r / Gp;
      const bool valid = tok < cnt && hh < G;
      const int ent = tok < cnt ? inf.ent[tok] : 0;
      const int t = ent >> 6;
      const int k0 = a.blk_tok != nullptr ? a.blk_tok[j] : j * a.sel_len;
      const int key_hi = valid ? min(64, t + 1 - k0) : 0;  // keys k0 + c, c < key_hi
      if (!warp_wait(&sm.s_full[w], jj & 1, abort_flag)) break;
      tc_fence_after();
      float s[64];
      tmem_ld32(trow, *reinterpret_cast<float(*)[32]>(&s[0]));
      tmem_ld32(trow + 32, *reinterpret_cast<float(*)[32]>(&s[32]));
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < 64; ++c) s[c] = c < key_hi ? s[c] : -INFINITY;
      float mx[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) mx[c] = fmax3f(s[c], s[c + 8], s[c + 16]);
#pragma unroll
      for (int c = 24; c < 64; c += 16)
#pragma unroll
        for (int u = 0; u < 8; ++u) mx[u] = fmax3f(mx[u], s[c + u], s[c + 8 + u]);
      const float mraw = fmax3f(fmax3f(mx[0], mx[1], mx[2]), fmax3f(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
      const float mrow = mraw * a.sl2;  // row max in log2 units (the scale is positive)
      const float bias = mraw == -INFINITY ? 0.f : -mrow;
      // this warp's rows of P were the staging buffer of its previous tile's partial store
      if (lane == 0) bulk_wait_read_all();
      __syncwarp();
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {  // 8 keys = one 16-byte chunk of the swizzled P row
        uint32_t wv[4];
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const int c = ch * 8 + 2 * x;
          const uint32_t pw =
              pack_bf16x2(ex2_approx(fmaf(s[c], a.sl2, bias)), ex2_approx(fmaf(s[c + 1], a.sl2, bias)));
          wv[x] = pw;
          acc[x + (ch & 1) * 4] += __uint_as_float(pw << 16) + __uint_as_float(pw & 0xffff0000u);
        }
        const uint32_t dst = smem_u32(prow_smem + ((ch ^ (r & 7)) << 4));
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(wv[0]), "r"(wv[1]), "r"(wv[2]),
                     "r"(wv[3])
                     : "memory");
      }
      const float lrow = ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
      fence_proxy_async_smem();  // P is read by the tensor core (async proxy)
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.p_full[w]);
      if (!warp_wait(&sm.o_full[w], jj & 1, abort_flag)) break;
      tc_fence_after();
      const float inv = lrow > 0.f ? 1.f / lrow : 0.f;
      // partial rows: fp16, staged in this warp's 32 rows of P (the P.V product is done with
      // them) in the 128-byte-swizzled layout, then one TMA store per 64-column half
      const int prow = (tile_begin + i) * 128 + r;
      uint8_t* stg = sm.p[w] + q4 * 32 * 128;
      float c_lo = 1.f, c_hi = 1.f;
#pragma unroll 1
      for (int h = 0; h < kChunks; ++h) {
        float o[64];
        tmem_ld32(trow + h * 64, *reinterpret_cast<float(*)[32]>(&o[0]));
        tmem_ld32(trow + h * 64 + 32, *reinterpret_cast<float(*)[32]>(&o[32]));
        tmem_wait_ld();
        float am[8];
#pragma unroll
        for (int x = 0; x < 8; ++x) am[x] = fmax3f(fabsf(o[x]), fabsf(o[x + 8]), fabsf(o[x + 16]));
#pragma unroll
        for (int u = 24; u < 64; u += 16)
#pragma unroll
          for (int x = 0; x < 8; ++x) am[x] = fmax3f(am[x], fabsf(o[u + x]), fabsf(o[u + 8 + x]));
        const float amax = fmax3f(fmax3f(am[0], am[1], am[2]), fmax3f(am[3], am[4], am[5]), fmaxf(am[6], am[7])) * inv;
        // 65504 is the largest finite fp16 value; rare rows are scaled down by a power of two
        float c = 1.f, sc = inv;
        if (amax > 65504.f) {
          if (amax <= 3.0e38f) c = exp2f(ceilf(log2f(amax / 32768.f)));
          sc = inv / c;
        }
        if (h == 0) c_lo = c; else c_hi = c;
        if (h > 0) {
          if (lane == 0) bulk_wait_read_all();
          __syncwarp();
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          uint32_t wv[4];
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            __half2 hv = __floats2half2_rn(o[8 * u + 2 * x] * sc, o[8 * u + 2 * x + 1] * sc);
            wv[x] = *reinterpret_cast<uint32_t*>(&hv);
          }
          const uint32_t dst = smem_u32(stg + lane * 128 + ((u ^ (lane & 7)) << 4));
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(wv[0]), "r"(wv[1]), "r"(wv[2]),
                       "r"(wv[3])
                       : "memory");
        }
        fence_proxy_async_smem();  // the TMA store reads the staged rows (async proxy)
        __syncwarp();
        if (lane == 0) {
          tma_store_3d(&omap, stg, 0, h, (tile_begin + i) * 128 + q4 * 32);
          bulk_commit_group();
        }
      }
      if (valid) a.part_ml[prow] = make_float4(mrow, lrow, c_lo, c_hi);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&sm.o_free[w]);
        mbar_arrive(&sm.info_empty[si]);
      }
    }
    if (lane == 0) bulk_wait_all();  // partial rows written before the CTA exits
    __syncwarp();
  }

  // ------------------------------------------------------------------ teardown
  __syncthreads();
  if (*abort_flag) {
    // drain: wait (bounded) for the last TMA load issued into each stage and for MMAs in
    // flight, so no async write lands after the CTA exits
    if (warp == 0 && lane == 0) {
      for (int u = kv_issued - kSelKVStages > 0 ? kv_issued - kSelKVStages : 0; u < kv_issued; ++u) {
        const long long t_start = clock64();
        while (!mbar_test(&sm.kv_full[u % kSelKVStages], (u / kSelKVStages) & 1) &&
               clock64() - t_start < kWaitCycles) {
        }
      }
    }
    if (warp == kSelMmaWarp && lane == 0) {
      umma_commit(&sm.drain);
      const long long t_start = clock64();
      while (!mbar_test(&sm.drain, 0) && clock64() - t_start < kWaitCycles) {
      }
    }
    __syncwarp();
    __syncthreads();
  }
  if (warp == kSelMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// One warp per (token, head): merges the row's partials (the slots holding a block index).
// Lane l owns output elements [l * D/32, (l+1) * D/32), all in 64-column half
// (l * D/32) / 64 of the partial rows. The partial rows are loaded as soon as their row
// numbers are known, alongside the (max, sum) records that weight them.
template <int D>
__global__ void __launch_bounds__(256, 4) sel_merge_kernel(const SelInvArgs a) {
  constexpr int kPer = D / 32;
  const long long row = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= static_cast<long long>(a.nv) * a.hq) return;
  const int t = static_cast<int>(row / a.hq), h = static_cast<int>(row % a.hq);
  const int g = h / a.G, hh = h - g * a.G;
  const size_t base = (static_cast<size_t>(t) * a.hkv + g) * a.top_n;
  // the combine's other inputs go out first: their latency overlaps the partials' loads
  const size_t orow = static_cast<size_t>(row) * D + lane * kPer;
  // (packed) gates and out use the row's place in the batch
  const size_t brow = a.vinfo != nullptr ? static_cast<size_t>(a.vinfo[t].w) * a.hq + h : static_cast<size_t>(row);
  const size_t out_off = brow * D + lane * kPer;
  const float gc = __ldg(a.gates + brow * 3 + 0);
  const float gs = __ldg(a.gates + brow * 3 + 1);
  const float gw = __ldg(a.gates + brow * 3 + 2);
  float oc[kPer], ow[kPer];
  if constexpr (kPer == 4) {
    const uint2 c2 = __ldg(reinterpret_cast<const uint2*>(a.o_cmp + orow));
    const uint2 w2 = __ldg(reinterpret_cast<const uint2*>(a.o_win + orow));
    const float2 ca = __half22float2(*reinterpret_cast<const __half2*>(&c2.x));
    const float2 cb = __half22float2(*reinterpret_cast<const __half2*>(&c2.y));
    oc[0] = ca.x; oc[1] = ca.y; oc[2] = cb.x; oc[3] = cb.y;
    const float2 wa = __half22float2(*reinterpret_cast<const __half2*>(&w2.x));
    const float2 wb = __half22float2(*reinterpret_cast<const __half2*>(&w2.y));
    ow[0] = wa.x; ow[1] = wa.y; ow[2] = wb.x; ow[3] = wb.y;
  } else {
    const uint32_t c1 = __ldg(reinterpret_cast<const unsigned int*>(a.o_cmp + orow));
    const uint32_t w1 = __ldg(reinterpret_cast<const unsigned int*>(a.o_win + orow));
    const float2 ca = __half22float2(*reinterpret_cast<const __half2*>(&c1));
    oc[0] = ca.x; oc[1] = ca.y;
    const float2 wa = __half22float2(*reinterpret_cast<const __half2*>(&w1));
    ow[0] = wa.x; ow[1] = wa.y;
  }
  // lane s holds slot s (and s + 32): its partial row, or -1; top_n <= 64
  int r0 = -1, r1 = -1;
  if (lane < a.top_n) {
    const int j = a.sel_idx[base + lane];
    const int rb = a.row_of[base + lane];
    if (j >= 0 && j < a.nsel) r0 = rb + hh;
  }
  if (lane + 32 < a.top_n) {
    const int j = a.sel_idx[base + lane + 32];
    const int rb = a.row_of[base + lane + 32];
    if (j >= 0 && j < a.nsel) r1 = rb + hh;
  }
  const float4 none = make_float4(-INFINITY, 0.f, 1.f, 1.f);
  const float4 x0 = r0 >= 0 ? a.part_ml[r0] : none;
  const float4 x1 = r1 >= 0 ? a.part_ml[r1] : none;
  const int half = (lane * kPer) >> 6;
  const int col = (lane * kPer) & 63;
  const __half* po = a.part_o + static_cast<size_t>(half) * 64 + col;
  float acc[kPer];
#pragma unroll
  for (int u = 0; u < kPer; ++u) acc[u] = 0.f;
  float M = -INFINITY, w0 = 0.f, w1 = 0.f, L = 0.f;
  // partial rows in batches of kMB slots: their loads go out together
  constexpr int kMB = 8;
  for (int s0 = 0; s0 < a.top_n; s0 += kMB) {
    const bool lo = s0 < 32;
    uint32_t raw[kMB][kPer / 2];
    int prow[kMB];
#pragma unroll
    for (int k = 0; k < kMB; ++k) {
      prow[k] = __shfl_sync(0xffffffffu, lo ? r0 : r1, (s0 + k) & 31);
      if (s0 + k >= a.top_n) prow[k] = -1;
      const __half* p = po + static_cast<size_t>(prow[k] < 0 ? 0 : prow[k]) * D;
      if (prow[k] >= 0) {
        if constexpr (kPer == 4) {
          const uint2 v = *reinterpret_cast<const uint2*>(p);
          raw[k][0] = v.x;
          raw[k][1] = v.y;
        } else {
          raw[k][0] = *reinterpret_cast<const uint32_t*>(p);
        }
      } else {
#pragma unroll
        for (int u = 0; u < kPer / 2; ++u) raw[k][u] = 0u;
      }
    }
    if (s0 == 0) {  // weights: exp2(max - M) * sum over the slots with keys
      M = fmaxf(x0.y > 0.f ? x0.x : -INFINITY, x1.y > 0.f ? x1.x : -INFINITY);
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
      w0 = (x0.y > 0.f) ? x0.y * ex2_approx(x0.x - M) : 0.f;
      w1 = (x1.y > 0.f) ? x1.y * ex2_approx(x1.x - M) : 0.f;
      L = warp_sum(w0 + w1);
    }
#pragma unroll
    for (int k = 0; k < kMB; ++k) {
      const int src = (s0 + k) & 31;
      const float w = __shfl_sync(0xffffffffu, lo ? w0 : w1, src);
      const float c = __shfl_sync(0xffffffffu, lo ? (half == 0 ? x0.z : x0.w) : (half == 0 ? x1.z : x1.w), src);
      const float wc = prow[k] >= 0 ? w * c : 0.f;
#pragma unroll
      for (int u = 0; u < kPer / 2; ++u) {
        const float2 y = __half22float2(*reinterpret_cast<const __half2*>(&raw[k][u]));
        acc[2 * u] += wc * y.x;
        acc[2 * u + 1] += wc * y.y;
      }
    }
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  if (a.o_sel != nullptr) {
    __half* dst = a.o_sel + orow;
    if constexpr (kPer == 4) {
      const __half2 h0 = __floats2half2_rn(acc[0] * inv, acc[1] * inv), h1 = __floats2half2_rn(acc[2] * inv, acc[3] * inv);
      *reinterpret_cast<uint2*>(dst) =
          make_uint2(*reinterpret_cast<const uint32_t*>(&h0), *reinterpret_cast<const uint32_t*>(&h1));
    } else {
      const __half2 h0 = __floats2half2_rn(acc[0] * inv, acc[1] * inv);
      *reinterpret_cast<uint32_t*>(dst) = *reinterpret_cast<const uint32_t*>(&h0);
    }
    // M is the largest partial max in log2 units, L the sum in those units
    if (lane == 0) a.lse_sel[row] = L > 0.f ? (M + __log2f(L)) * 0.69314718055994530942f : -INFINITY;
  }
  float res[kPer];
#pragma unroll
  for (int u = 0; u < kPer; ++u) res[u] = gc * oc[u] + gs * (acc[u] * inv) + gw * ow[u];
  if (a.out_f32) {
    float* dst = static_cast<float*>(a.out) + out_off;
    if constexpr (kPer == 4)
      *reinterpret_cast<float4*>(dst) = make_float4(res[0], res[1], res[2], res[3]);
    else
      *reinterpret_cast<float2*>(dst) = make_float2(res[0], res[1]);
  } else {
    __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(a.out) + out_off;
    if constexpr (kPer == 4)
      *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16x2(res[0], res[1]), pack_bf16x2(res[2], res[3]));
    else
      *reinterpret_cast<uint32_t*>(dst) = pack_bf16x2(res[0], res[1]);
  }
}

}  // namespace nsa
