// gate.cuh -- the gate network that mixes the three branches.
//
// Every head gets three gates (compressed, selected, window) that a softmax normalises to
// sum to one, produced by a small MLP: dim -> dim/2 linear, exact GELU, dim/2 -> 3 linear
// (CSDN blog "VideoNSA：重新定义视频理解的稀疏注意力机制", vcloud.csdn.net, section 3.1
// "动态门控机制详解"). The blog's module averages its input over the tokens first; this
// file has both forms:
//   gate_mlp_kernel     per row (one token of one head): the first layer is a dense
//                       [128 rows x dim] x [dim x dim/2] contraction on the tensor cores
//                       (tcgen05, bf16 in, fp32 accumulator in TMEM); GELU (erf to 1.5e-7,
//                       Abramowitz & Stegun 7.1.26), the second layer and the softmax run
//                       on the CUDA cores, one thread per row.
//   gate_mean_partial_kernel + gate_pooled_kernel
//                       the averaged form: fp64 column sums over token chunks, then one
//                       CTA per (sequence, head) finishes the mean and evaluates the MLP in
//                       fp64, optionally writing the triple once per token.
// Weights use the linear-layer layout [out][in]: W1 [dim/2][dim] bf16, b1 [dim/2],
// W2 [3][dim/2] and b2 [3] fp32.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "sm100.cuh"

namespace nsa {

// erf(x) by Abramowitz & Stegun, Handbook of Mathematical Functions, formula 7.1.26:
// erf(x) = 1 - (a1 t + a2 t^2 + a3 t^3 + a4 t^4 + a5 t^5) exp(-x^2), t = 1 / (1 + p x), x >= 0,
// with |error| <= 1.5e-7; odd in x. One reciprocal, one exp2 and a degree-5 polynomial.
__device__ __forceinline__ float erf_as7126(float x) {
  const float ax = fabsf(x);
  const float t = __fdividef(1.0f, fmaf(0.3275911f, ax, 1.0f));
  float poly = fmaf(1.061405429f, t, -1.453152027f);
  poly = fmaf(poly, t, 1.421413741f);
  poly = fmaf(poly, t, -0.284496736f);
  poly = fmaf(poly, t, 0.254829592f);
  poly *= t;
  const float e = ex2_approx(-ax * ax * 1.4426950408889634f);  // exp(-x^2)
  return copysignf(fmaf(-poly, e, 1.0f), x);
}

template <int DIM>
struct GateSmem {
  static constexpr int kHid = DIM / 2;
  static constexpr int kChunks = DIM / 64;  // 64-element (128-byte) column chunks, one per TMA box
  static constexpr int kTmemCols = kHid < 32 ? 32 : kHid;
  static constexpr uint32_t kTxBytes = static_cast<uint32_t>(kChunks) * (128 + kHid) * 128;
  alignas(1024) uint8_t x[kChunks][128 * 128];   // 128 rows x 128 B per chunk, 128B-swizzled
  alignas(1024) uint8_t w1[kChunks][kHid * 128];  // kHid rows x 128 B per chunk
  float4 wb[kHid];  // per hidden unit j: (b1[j], W2[0][j], W2[1][j], W2[2][j])
  float b2[4];
  uint64_t full;
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort_flag;
};

template <class S>
__device__ __forceinline__ S& align_smem_1024(uint8_t* raw) {
  const uint32_t a = smem_u32(raw);
  return *reinterpret_cast<S*>(raw + (((a + 1023u) & ~1023u) - a));
}

// Per-row gates. x [rows][DIM] bf16 through xmap (box 64 x 128), W1 [DIM/2][DIM] bf16
// through wmap (box 64 x DIM/2); gates [rows][3] fp32. One CTA of 4 warps per 128 rows.
template <int DIM>
__global__ void __launch_bounds__(128) gate_mlp_kernel(const __grid_constant__ CUtensorMap xmap,
                                                       const __grid_constant__ CUtensorMap wmap,
                                                       const float* __restrict__ b1, const float* __restrict__ w2,
                                                       const float* __restrict__ b2, float* __restrict__ gates,
                                                       long long rows) {
  using S = GateSmem<DIM>;
  constexpr int kHid = S::kHid;
  extern __shared__ uint8_t gate_smem_raw[];
  S& sm = align_smem_1024<S>(gate_smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long row0 = static_cast<long long>(blockIdx.x) * 128;
  if (tid == 0) {
    mbar_init(&sm.full, 1);
    mbar_init(&sm.mma_done, 1);
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&sm.tmem_base, S::kTmemCols);
    tmem_relinquish();
  }
  for (int j = tid; j < kHid; j += 128) sm.wb[j] = make_float4(b1[j], w2[j], w2[kHid + j], w2[2 * kHid + j]);
  if (tid < 3) sm.b2[tid] = b2[tid];
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  // load, then the first layer: D[128 x kHid] = X[128 x DIM] . W1^T, K = DIM in steps of 16
  bool issued = false;
  if (warp == 0) {
    if (elect_one_sync()) {
      mbar_arrive_expect_tx(&sm.full, S::kTxBytes);
#pragma unroll
      for (int c = 0; c < S::kChunks; ++c) {
        tma_load_3d(&xmap, &sm.full, sm.x[c], c * 64, static_cast<int>(row0), 0);
        tma_load_3d(&wmap, &sm.full, sm.w1[c], c * 64, 0, 0);
      }
      if (mbar_wait(&sm.full, 0, &sm.abort_flag)) {
        tc_fence_after();
        constexpr uint32_t idesc = idesc_bf16_f32(128, kHid, false, false);
#pragma unroll
        for (int k = 0; k < DIM / 16; ++k) {
          const int c = k >> 2, kk = k & 3;
          const uint64_t ad = sdesc_sw128(smem_u32(sm.x[c]), 16, 1024) + static_cast<uint64_t>((kk * 32) >> 4);
          const uint64_t bd = sdesc_sw128(smem_u32(sm.w1[c]), 16, 1024) + static_cast<uint64_t>((kk * 32) >> 4);
          umma_bf16_ss(tmem, ad, bd, idesc, k > 0 ? 1u : 0u);
        }
        umma_commit(&sm.mma_done);
        issued = true;
      }
    }
    __syncwarp();
  }

  // epilogue: warp w owns TMEM lanes (rows) 32w .. 32w+31
  const bool ready = mbar_wait(&sm.mma_done, 0, &sm.abort_flag);
  if (ready) {
    tc_fence_after();
    float acc[kHid];
    const uint32_t taddr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
#pragma unroll
    for (int c = 0; c < kHid; c += 32) {
      float part[32];
      tmem_ld32(taddr + c, part);
#pragma unroll
      for (int j = 0; j < 32; ++j) acc[c + j] = part[j];
    }
    tmem_wait_ld();
    float l0 = sm.b2[0], l1 = sm.b2[1], l2 = sm.b2[2];
#pragma unroll
    for (int j = 0; j < kHid; ++j) {
      const float4 w = sm.wb[j];
      const float h = acc[j] + w.x;
      const float g = 0.5f * h * (1.0f + erf_as7126(h * 0.70710678118654752f));
      l0 = fmaf(w.y, g, l0);
      l1 = fmaf(w.z, g, l1);
      l2 = fmaf(w.w, g, l2);
    }
    const float m = fmaxf(l0, fmaxf(l1, l2));
    const float e0 = expf(l0 - m), e1 = expf(l1 - m), e2 = expf(l2 - m);
    const float inv = 1.0f / (e0 + e1 + e2);
    const long long row = row0 + warp * 32 + lane;
    if (row < rows) {
      float* g = gates + row * 3;
      g[0] = e0 * inv;
      g[1] = e1 * inv;
      g[2] = e2 * inv;
    }
  } else if (warp == 0 && issued && lane == 0) {
    // the wait gave up: let the issued MMAs finish before the TMEM is released
    const long long t0 = clock64();
    while (!mbar_test(&sm.mma_done, 0) && clock64() - t0 < kWaitCycles) {
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, S::kTmemCols);
  }
}

// Averaged form, step 1: fp64 column sums of x [B][T][cols] bf16 (cols = H*DIM) over the
// token chunk [c*chunk, min(T, (c+1)*chunk)) of sequence b = blockIdx.y, c = blockIdx.x;
// partial [nchunk][B][cols] fp64. A thread owns up to kGatePairs bf16x2 column pairs,
// blockDim.x apart, and walks the chunk's tokens once, so its loads for one token are
// independent of one another.
constexpr int kGatePairs = 8;
__global__ void __launch_bounds__(256) gate_mean_partial_kernel(const __nv_bfloat16* __restrict__ x,
                                                                double* __restrict__ partial, int B, int T,
                                                                int cols, int chunk) {
  const int c = blockIdx.x, b = blockIdx.y;
  const int t0 = c * chunk, t1 = min(T, t0 + chunk);
  const int pairs = cols / 2;
  const __nv_bfloat162* base = reinterpret_cast<const __nv_bfloat162*>(x + static_cast<size_t>(b) * T * cols);
  double* out = partial + (static_cast<size_t>(c) * B + b) * cols;
  for (int p0 = threadIdx.x; p0 < pairs; p0 += blockDim.x * kGatePairs) {
    double s0[kGatePairs], s1[kGatePairs];
#pragma unroll
    for (int u = 0; u < kGatePairs; ++u) s0[u] = s1[u] = 0.0;
    for (int t = t0; t < t1; ++t) {
      const __nv_bfloat162* row = base + static_cast<size_t>(t) * pairs;
      float2 v[kGatePairs];
#pragma unroll
      for (int u = 0; u < kGatePairs; ++u) {
        const int p = p0 + u * blockDim.x;
        v[u] = p < pairs ? __bfloat1622float2(row[p]) : make_float2(0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < kGatePairs; ++u) {
        s0[u] += static_cast<double>(v[u].x);
        s1[u] += static_cast<double>(v[u].y);
      }
    }
#pragma unroll
    for (int u = 0; u < kGatePairs; ++u) {
      const int p = p0 + u * blockDim.x;
      if (p < pairs) {
        out[2 * p] = s0[u];
        out[2 * p + 1] = s1[u];
      }
    }
  }
}

// Averaged form, step 2: CTA (b, h) = (blockIdx.x / H, blockIdx.x % H) adds the nchunk
// partials (kPooledSplit interleaved runs per column, then the runs in order), divides by
// T and evaluates the MLP and softmax in fp64, then writes the triple to
// gates[b][r][h][0..2] for every r < repeat. kPooledSplit * DIM threads.
constexpr int kPooledSplit = 4;
template <int DIM>
__global__ void __launch_bounds__(kPooledSplit * DIM) gate_pooled_kernel(const double* __restrict__ partial,
                                                          const __nv_bfloat16* __restrict__ w1,
                                                          const float* __restrict__ b1,
                                                          const float* __restrict__ w2,
                                                          const float* __restrict__ b2, float* __restrict__ gates,
                                                          int B, int T, int H, int nchunk, int repeat) {
  constexpr int kHid = DIM / 2;
  __shared__ double run[kPooledSplit][DIM];
  __shared__ double mean[DIM];
  __shared__ double hid[kHid];
  __shared__ float res[3];
  const int b = blockIdx.x / H, h = blockIdx.x % H;
  const int j = threadIdx.x % DIM, part = threadIdx.x / DIM;
  const size_t cols = static_cast<size_t>(H) * DIM;
  double s = 0.0;
  for (int c = part; c < nchunk; c += kPooledSplit)
    s += partial[(static_cast<size_t>(c) * B + b) * cols + static_cast<size_t>(h) * DIM + j];
  run[part][j] = s;
  __syncthreads();
  if (threadIdx.x < DIM) {
    double m = 0.0;
#pragma unroll
    for (int q = 0; q < kPooledSplit; ++q) m += run[q][j];
    mean[j] = m / static_cast<double>(T);
  }
  __syncthreads();
  if (threadIdx.x < kHid) {
    double a = static_cast<double>(b1[j]);
    for (int i = 0; i < DIM; ++i)
      a += static_cast<double>(__bfloat162float(w1[static_cast<size_t>(j) * DIM + i])) * mean[i];
    hid[j] = 0.5 * a * (1.0 + erf(a * 0.70710678118654752440));
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double lg[3];
    for (int c = 0; c < 3; ++c) {
      double a = static_cast<double>(b2[c]);
      for (int i = 0; i < kHid; ++i) a += static_cast<double>(w2[c * kHid + i]) * hid[i];
      lg[c] = a;
    }
    const double m = fmax(lg[0], fmax(lg[1], lg[2]));
    const double e0 = exp(lg[0] - m), e1 = exp(lg[1] - m), e2 = exp(lg[2] - m);
    const double z = e0 + e1 + e2;
    res[0] = static_cast<float>(e0 / z);
    res[1] = static_cast<float>(e1 / z);
    res[2] = static_cast<float>(e2 / z);
  }
  __syncthreads();
  for (int r = threadIdx.x; r < repeat; r += blockDim.x) {
    float* g = gates + ((static_cast<size_t>(b) * repeat + r) * H + h) * 3;
    g[0] = res[0];
    g[1] = res[1];
    g[2] = res[2];
  }
}

}  // namespace nsa
