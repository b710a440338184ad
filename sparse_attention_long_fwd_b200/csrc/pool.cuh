// pool.cuh -- compression branch, step 1: mean-pool K and V into block summaries.
//
// The compression branch merges consecutive tokens into representative summaries
// (top168.com article on VideoNSA, section "一、革命性的三重注意机制", compression
// branch). This library's summary is the plain mean of each complete block of
// l = cmp_block tokens taken at stride s = cmp_stride, rounded once to bf16:
//   Kc[i] = bf16_rne( (1/l) * sum_{u<l} K[i*s + u] ).
// The sum runs in fp64 in token order, so it is exact for any bf16 inputs whose
// exponents span less than ~40 binades, and the mean is rounded to bf16 in a single
// step (fp64 -> fp32 with round-to-odd, then fp32 -> bf16 to nearest even; rounding to
// odd at a precision with >= 2 extra bits makes the second rounding correct, Boldo &
// Melquiond, "When double rounding is odd", 2005).
//
// Learnable form: the pages steer the sparse pattern with learned parameters
// (shd-paper.top page "VideoNSA: Native Sparse Attention Scales Video Understanding",
// section "方法详解", key design (1)) without giving their form. Given per-head weights
// w [hkv][l] (fp32), a summary is the weighted sum instead of the mean:
//   Kc[i][g] = bf16_rne( sum_{u<l} w[g][u] * K[i*s + u][g] ).
// An fp32 weight times a bf16 key is exact in fp64, so this sum is rounded exactly like
// the mean's; w = 1/l with l a power of two reproduces the mean bit for bit.
//
// HBM-bound: each token row is read by l/s = 2 overlapping blocks (the second read hits
// L2); one thread owns two adjacent dims (a bf16x2 word) of one (sequence, block, head).
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

namespace nsa {

__device__ __forceinline__ __nv_bfloat16 f64_to_bf16_rne(double x) {
  float f = __double2float_rz(x);
  if (static_cast<double>(f) != x && !isnan(x)) f = __uint_as_float(__float_as_uint(f) | 1u);
  return __float2bfloat16_rn(f);
}

// src: [nseq][T][hkv][d] bf16; dst: [nseq][ncmp][hkv][d] bf16. blockIdx.z: 0 -> K, 1 -> V.
// wk, wv: [hkv][l] fp32 weights of the learnable form, or both null for the mean.
// Each thread handles one bf16x2 column pair of one (seq, block i, head g).
// row_tok (packed batches; nseq = 1): [ncmp] the token row of every summary's first token,
// or -1 for a row that pads a sequence's summaries to a multiple of 128 (written as zeros).
__global__ void __launch_bounds__(256) pool_kernel(const __nv_bfloat16* __restrict__ k,
                                                   const __nv_bfloat16* __restrict__ v,
                                                   __nv_bfloat16* __restrict__ kc, __nv_bfloat16* __restrict__ vc,
                                                   const float* __restrict__ wk, const float* __restrict__ wv,
                                                   int nseq, int T, int hkv, int d, int ncmp, int l, int s,
                                                   const int* __restrict__ row_tok) {
  const __nv_bfloat16* src = blockIdx.z == 0 ? k : v;
  __nv_bfloat16* dst = blockIdx.z == 0 ? kc : vc;
  const float* w = blockIdx.z == 0 ? wk : wv;
  const int pairs = d / 2;
  const long long total = static_cast<long long>(nseq) * ncmp * hkv * pairs;
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= total) return;
  const int p = static_cast<int>(idx % pairs);
  long long rest = idx / pairs;
  const int g = static_cast<int>(rest % hkv);
  rest /= hkv;
  const int i = static_cast<int>(rest % ncmp);
  const int b = static_cast<int>(rest / ncmp);
  const size_t row_elems = static_cast<size_t>(hkv) * d;
  const long long tok0 = row_tok != nullptr ? row_tok[i] : static_cast<long long>(b) * T + static_cast<long long>(i) * s;
  __nv_bfloat16* const out_row = dst + ((static_cast<size_t>(b) * ncmp + i) * hkv + g) * d;
  if (tok0 < 0) {
    reinterpret_cast<__nv_bfloat162*>(out_row)[p] = __floats2bfloat162_rn(0.f, 0.f);
    return;
  }
  const __nv_bfloat162* in = reinterpret_cast<const __nv_bfloat162*>(
      src + static_cast<size_t>(tok0) * row_elems + static_cast<size_t>(g) * d) + p;
  double a0 = 0.0, a1 = 0.0;
  __nv_bfloat162 o;
  if (w == nullptr) {
    for (int u = 0; u < l; ++u) {
      const float2 x = __bfloat1622float2(in[static_cast<size_t>(u) * (row_elems / 2)]);
      a0 += static_cast<double>(x.x);
      a1 += static_cast<double>(x.y);
    }
    const double dl = static_cast<double>(l);
    o.x = f64_to_bf16_rne(a0 / dl);
    o.y = f64_to_bf16_rne(a1 / dl);
  } else {
    const float* wg = w + static_cast<size_t>(g) * l;
    for (int u = 0; u < l; ++u) {
      const float2 x = __bfloat1622float2(in[static_cast<size_t>(u) * (row_elems / 2)]);
      const double wu = static_cast<double>(__ldg(wg + u));
      a0 += wu * static_cast<double>(x.x);  // exact product: fusing it into an fma changes nothing
      a1 += wu * static_cast<double>(x.y);
    }
    o.x = f64_to_bf16_rne(a0);
    o.y = f64_to_bf16_rne(a1);
  }
  reinterpret_cast<__nv_bfloat162*>(out_row)[p] = o;
}

}  // namespace nsa
