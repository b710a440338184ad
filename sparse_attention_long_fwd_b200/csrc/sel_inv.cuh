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
// partial is an exact convex combination of values. The partial output is stored in fp16
// (2^-12 relative rounding); a row whose largest magnitude would overflow fp16 is stored
// divided by a power of two c, kept with the row's (max, sum).
//
//   sel_count_kernel    entries per (group, block)
//   sel_scan_kernel     exclusive scans of entries and of tiles per (group, block)
//   sel_scatter_kernel  bucket (token, slot) pairs
//   sel_partial_kernel  one 128-row tcgen05 tile per CTA: S = Q K^T, softmax, O = P V
//   sel_merge_kernel    o_sel[t][h] from the row's partials
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
  __half* part_o;               // [nv][hq][top_n][D] output / (sum * c) of each partial
  float4* part_ml;              // [nv][hq][top_n] (max in log2 units, sum, c, 0)
  float* o_sel;                 // [nv][hq][D]
};

__global__ void __launch_bounds__(256) sel_count_kernel(const SelInvArgs a) {
  const long long n = static_cast<long long>(a.nv) * a.hkv * a.top_n;
  for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < n;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int j = a.sel_idx[e];
    const int g = static_cast<int>((e / a.top_n) % a.hkv);
    if (j >= 0 && j < a.nsel) atomicAdd(&a.cnt[g * a.nsel + j], 1);
  }
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
  const long long n = static_cast<long long>(a.nv) * a.hkv * a.top_n;
  for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < n;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int j = a.sel_idx[e];
    if (j < 0 || j >= a.nsel) continue;
    const int slot = static_cast<int>(e % a.top_n);
    const long long tg = e / a.top_n;
    const int g = static_cast<int>(tg % a.hkv);
    const int t = static_cast<int>(tg / a.hkv);
    const int key = g * a.nsel + j;
    const int pos = a.ent_off[key] + atomicAdd(&a.cursor[key], 1);
    a.list[pos] = t * 64 + slot;
  }
}

// 32 fp32 values times `scale` to fp16 (round to nearest even), 64 contiguous bytes
__device__ __forceinline__ void store_half32(__half* dst, const float (&o)[32], float scale) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    uint32_t w[4];
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      __half2 h = __floats2half2_rn(o[8 * u + 2 * x] * scale, o[8 * u + 2 * x + 1] * scale);
      w[x] = *reinterpret_cast<uint32_t*>(&h);
    }
    d4[u] = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

constexpr int kSelInvThreads = 192;  // TMA warp, MMA warp, 4 softmax / epilogue warps

template <int D>
struct SelInvSmem {
  static constexpr int kChunks = D / 64;
  alignas(1024) uint8_t q[kChunks][128 * 128];  // 128 rows x 128 B per chunk
  alignas(1024) uint8_t k[kChunks][64 * 128];   // the block's 64 keys
  alignas(1024) uint8_t v[kChunks][64 * 128];   // and values
  uint64_t full, s_full, p_full, o_full, drain;
  uint32_t tmem_base;
  int abort_flag;
  int g, j, e0, cnt;
  int ent[128];  // t * 64 + slot of this tile's tokens
};

// grid: an upper bound on the tile count; CTAs past tile_off[hkv*nsel] return at once.
template <int D>
__global__ void __launch_bounds__(kSelInvThreads, 1)
    sel_partial_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                       const __grid_constant__ CUtensorMap vmap, const SelInvArgs a) {
  using Smem = SelInvSmem<D>;
  constexpr int kChunks = Smem::kChunks;
  constexpr uint32_t kTmemCols = 256;  // S at 0 (64), O at 64 (D <= 128), P at 192 (32)
  constexpr uint32_t kColO = 64, kColP = 192;
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int m = a.hkv * a.nsel;
  const int tile = blockIdx.x;
  if (tile >= a.tile_off[m]) return;  // uniform across the CTA
  if (tid == 0) {
    // (group, block) of this tile: last key with tile_off[key] <= tile
    int lo = 0, hi = m - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (a.tile_off[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    const int first = a.ent_off[lo] + (tile - a.tile_off[lo]) * a.TT;
    sm.g = lo / a.nsel;
    sm.j = lo % a.nsel;
    sm.e0 = first;
    sm.cnt = min(a.TT, a.ent_off[lo + 1] - first);
    mbar_init(&sm.full, 1);
    mbar_init(&sm.s_full, 1);
    mbar_init(&sm.p_full, 4);
    mbar_init(&sm.o_full, 1);
    mbar_init(&sm.drain, 1);
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  __syncthreads();
  const int g = sm.g, j = sm.j, cnt = sm.cnt;
  for (int i = tid; i < cnt; i += kSelInvThreads) sm.ent[i] = a.list[sm.e0 + i];
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort_flag = &sm.abort_flag;
  const int Gp = a.Gp, G = a.G;

  if (warp == 0) {
    if (lane == 0) {
      mbar_arrive_expect_tx(&sm.full, kChunks * (cnt * Gp * 128 + 2 * 64 * 128));
      for (int c = 0; c < kChunks; ++c) {
        for (int i = 0; i < cnt; ++i)
          tma_load_3d(&qmap, &sm.full, &sm.q[c][i * Gp * 128], c * 64, g * G, sm.ent[i] >> 6);
        tma_load_3d(&kmap, &sm.full, sm.k[c], c * 64, g, j * a.sel_len);
        tma_load_3d(&vmap, &sm.full, sm.v[c], c * 64, g, j * a.sel_len);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(128, 64, false, false);
      constexpr uint32_t idO = idesc_bf16_f32(128, D, false, true);
      bool ok = mbar_wait(&sm.full, 0, abort_flag);
      if (ok) {
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const int c = k >> 2, kk = k & 3;
          umma_bf16_ss(tmem, sdesc_sw128(smem_u32(sm.q[c]) + kk * 32, 16, 1024),
                       sdesc_sw128(smem_u32(sm.k[c]) + kk * 32, 16, 1024), idS, k > 0 ? 1u : 0u);
        }
        umma_commit(&sm.s_full);
        ok = mbar_wait(&sm.p_full, 0, abort_flag);
      }
      if (ok) {
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < 4; ++k)  // 64 keys, 16 per MMA
          umma_bf16_ts(tmem + kColO, tmem + kColP + k * 8,
                       sdesc_sw128(smem_u32(sm.v[0]) + k * 2048, 64 * 128, 1024), idO, k > 0 ? 1u : 0u);
        umma_commit(&sm.o_full);
      }
    }
    __syncwarp();
  } else {
    // one thread per MMA row: token slot i = r / Gp, head slot hh = r % Gp
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const int i = r / Gp, hh = r % Gp;
    const bool valid = i < cnt && hh < G;
    const int ent = i < cnt ? sm.ent[i] : 0;
    const int t = ent >> 6, slot = ent & 63;
    const int key_hi = valid ? min(64, t + 1 - j * a.sel_len) : 0;  // keys j*64 + c, c < key_hi
    const uint32_t trow = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    bool ok = __all_sync(0xffffffffu, mbar_wait(&sm.s_full, 0, abort_flag));
    float mrow = -INFINITY, lrow = 0.f;
    if (ok) {
      tc_fence_after();
      float s[64];
      __syncwarp();
      tmem_ld32(trow, *reinterpret_cast<float(*)[32]>(&s[0]));
      tmem_ld32(trow + 32, *reinterpret_cast<float(*)[32]>(&s[32]));
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < 64; ++c) s[c] = c < key_hi ? s[c] * a.sl2 : -INFINITY;
      float mx[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) mx[c] = s[c];
#pragma unroll
      for (int c = 8; c < 64; c += 8)
#pragma unroll
        for (int u = 0; u < 8; ++u) mx[u] = fmaxf(mx[u], s[c + u]);
      mrow = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])), fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      uint32_t pk[32];
#pragma unroll
      for (int c = 0; c < 64; c += 2) {
        const float p0 = mrow == -INFINITY ? 0.f : ex2_approx(s[c] - mrow);
        const float p1 = mrow == -INFINITY ? 0.f : ex2_approx(s[c + 1] - mrow);
        const uint32_t w = pack_bf16x2(p0, p1);
        pk[c >> 1] = w;
        acc[(c >> 1) & 7] += __uint_as_float(w << 16) + __uint_as_float(w & 0xffff0000u);
      }
      lrow = ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
      tmem_st16(trow + kColP, *reinterpret_cast<uint32_t(*)[16]>(&pk[0]));
      tmem_st16(trow + kColP + 16, *reinterpret_cast<uint32_t(*)[16]>(&pk[16]));
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.p_full);
      ok = __all_sync(0xffffffffu, mbar_wait(&sm.o_full, 0, abort_flag));
    }
    if (ok) {
      tc_fence_after();
      const float inv = lrow > 0.f ? 1.f / lrow : 0.f;
      const size_t prow = (static_cast<size_t>(t) * a.hq + g * G + hh) * a.top_n + slot;
      // fp16 stores; 65504 is the largest finite fp16 value
      float amax = 0.f;
#pragma unroll 1
      for (int cb = 0; cb < D / 32; ++cb) {
        float o[32];
        __syncwarp();
        tmem_ld32(trow + kColO + cb * 32, o);
        tmem_wait_ld();
#pragma unroll
        for (int u = 0; u < 32; ++u) amax = fmaxf(amax, fabsf(o[u] * inv));
        if (valid) store_half32(a.part_o + prow * D + cb * 32, o, inv);
      }
      float c = 1.f;
      if (__any_sync(0xffffffffu, valid && !(amax < 65504.f))) {
        // rare: rescale the row by a power of two (exact) and store it again
        if (amax > 65504.f && amax <= 3.0e38f) c = exp2f(ceilf(log2f(amax / 32768.f)));
        const float inv_c = inv / c;
#pragma unroll 1
        for (int cb = 0; cb < D / 32; ++cb) {
          float o[32];
          __syncwarp();
          tmem_ld32(trow + kColO + cb * 32, o);
          tmem_wait_ld();
          if (valid) store_half32(a.part_o + prow * D + cb * 32, o, inv_c);
        }
      }
      if (valid) a.part_ml[prow] = make_float4(mrow, lrow, c, 0.f);
    }
    tc_fence_before();
  }
  __syncthreads();
  if (*abort_flag) {
    if (warp == 0 && lane == 0) {
      const long long t_start = clock64();
      while (!mbar_test(&sm.full, 0) && clock64() - t_start < kWaitCycles) {
      }
    }
    if (warp == 1 && lane == 0) {
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
    tmem_dealloc(tmem, kTmemCols);
  }
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// One warp per (token, head): merges the row's partials (the slots holding a block index).
// Lane l owns output elements [l * D/32, (l+1) * D/32).
template <int D>
__global__ void __launch_bounds__(256) sel_merge_kernel(const SelInvArgs a) {
  constexpr int kPer = D / 32;
  const long long row = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= static_cast<long long>(a.nv) * a.hq) return;
  const int t = static_cast<int>(row / a.hq), h = static_cast<int>(row % a.hq);
  const int g = h / a.G;
  const int32_t* sel = a.sel_idx + (static_cast<size_t>(t) * a.hkv + g) * a.top_n;
  const float4* ml = a.part_ml + static_cast<size_t>(row) * a.top_n;
  // lane s holds slot s's (max, sum, c); top_n <= 64
  float4 x0 = make_float4(-INFINITY, 0.f, 1.f, 0.f), x1 = x0;
  if (lane < a.top_n) {
    const int j = sel[lane];
    if (j >= 0 && j < a.nsel) x0 = ml[lane];
  }
  if (lane + 32 < a.top_n) {
    const int j = sel[lane + 32];
    if (j >= 0 && j < a.nsel) x1 = ml[lane + 32];
  }
  float M = fmaxf(x0.y > 0.f ? x0.x : -INFINITY, x1.y > 0.f ? x1.x : -INFINITY);
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  const float w0 = (x0.y > 0.f) ? x0.y * ex2_approx(x0.x - M) : 0.f;
  const float w1 = (x1.y > 0.f) ? x1.y * ex2_approx(x1.x - M) : 0.f;
  const float L = warp_sum(w0 + w1);
  const float wc0 = w0 * x0.z, wc1 = w1 * x1.z;
  float acc[kPer];
#pragma unroll
  for (int u = 0; u < kPer; ++u) acc[u] = 0.f;
  const __half* po = a.part_o + static_cast<size_t>(row) * a.top_n * D + lane * kPer;
  for (int s = 0; s < a.top_n; ++s) {
    const float w = __shfl_sync(0xffffffffu, s < 32 ? wc0 : wc1, s & 31);
    if (w == 0.f) continue;  // uniform across the warp
    const __half* src = po + static_cast<size_t>(s) * D;
    if constexpr (kPer == 4) {
      const uint2 raw = *reinterpret_cast<const uint2*>(src);
      const float2 y0 = __half22float2(*reinterpret_cast<const __half2*>(&raw.x));
      const float2 y1 = __half22float2(*reinterpret_cast<const __half2*>(&raw.y));
      acc[0] += w * y0.x;
      acc[1] += w * y0.y;
      acc[2] += w * y1.x;
      acc[3] += w * y1.y;
    } else {
      const uint32_t raw = *reinterpret_cast<const uint32_t*>(src);
      const float2 y0 = __half22float2(*reinterpret_cast<const __half2*>(&raw));
      acc[0] += w * y0.x;
      acc[1] += w * y0.y;
    }
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  float* dst = a.o_sel + static_cast<size_t>(row) * D + lane * kPer;
  if constexpr (kPer == 4)
    *reinterpret_cast<float4*>(dst) = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
  else
    *reinterpret_cast<float2*>(dst) = make_float2(acc[0] * inv, acc[1] * inv);
}

}  // namespace nsa
