// sel.cuh -- selection branch, step 3 (prefill): exact attention over the selected blocks.
//
// For every video token t and KV group g, the G query heads attend to the tokens
// tau <= t of the blocks chosen by topn_kernel (selection branch, top168.com article on
// VideoNSA, section "一、革命性的三重注意机制"). Each (token, group) has its own key set,
// so one warp handles one (token, group): the gathered 64-token blocks are streamed in
// 32-key chunks through the warp's two-stage cp.async ring (warp_attn.cuh) and reused by
// all G heads. Output: o_sel [N_v][Hq][d] fp32 (normalised). Every gathered byte passes
// through shared memory twice (cp.async write, ldmatrix read), which bounds this kernel
// by shared-memory bandwidth rather than by the L2 gathers; eight warps with a deeper
// ring of 16-key chunks measured no faster than four warps with 32-key chunks.
#pragma once
#include "warp_attn.cuh"

namespace nsa {

constexpr int kSelWarps = 4;
constexpr int kSelChunk = 32;   // keys per gathered chunk
constexpr int kSelStages = 2;   // per-warp cp.async ring depth

template <int D>
struct SelSmem {
  WarpChunkBuf<D, kSelChunk, kSelStages> buf[kSelWarps];
  int chunk_start[kSelWarps][256];
};

// Compact the valid `ck`-key chunks of a selection list (ascending block indices, -1
// padded) into `out` (shared, >= top_n * sel_len / ck entries); returns the count. A chunk
// is valid if it starts at or before t.
__device__ __forceinline__ int build_chunk_list(const int32_t* __restrict__ blocks, int top_n, int sel_len, int t,
                                                int* out, int lane, int ck = kChunkKeys) {
  const int per = sel_len / ck;
  int count = 0;
  for (int base = 0; base < per * top_n; base += 32) {
    const int ci = base + lane;
    int start = -1;
    if (ci < per * top_n) {
      const int j = blocks[ci / per];
      const int s = j * sel_len + (ci % per) * ck;
      if (j >= 0 && s <= t) start = s;
    }
    const uint32_t m = __ballot_sync(0xffffffffu, start >= 0);
    if (start >= 0) out[count + __popc(m & ((1u << lane) - 1u))] = start;
    count += __popc(m);
  }
  __syncwarp();
  return count;
}

template <int D>
__global__ void __launch_bounds__(kSelWarps * 32) sel_branch_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
    const int32_t* __restrict__ sel_idx, int n_video, int hq, int hkv, int top_n, int sel_len, float sl2,
    float* __restrict__ o_sel) {
  extern __shared__ uint8_t sel_smem_raw[];
  SelSmem<D>& sm = *reinterpret_cast<SelSmem<D>*>((reinterpret_cast<uintptr_t>(sel_smem_raw) + 127) & ~uintptr_t(127));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int item = blockIdx.x * kSelWarps + warp;
  if (item >= n_video * hkv) return;
  const int t = item / hkv, g = item % hkv;
  const int G = hq / hkv;
  uint32_t qa[D / 16][4];
  load_q_frags<D>(qa, q + (static_cast<size_t>(t) * hq + g * G) * D, G, lane);
  int* list = sm.chunk_start[warp];
  const int nch =
      build_chunk_list(sel_idx + static_cast<size_t>(item) * top_n, top_n, sel_len, t, list, lane, kSelChunk);
  const __nv_bfloat16* kb = k + static_cast<size_t>(g) * D;
  const __nv_bfloat16* vb = v + static_cast<size_t>(g) * D;
  const size_t rs = static_cast<size_t>(hkv) * D;
  auto& buf = sm.buf[warp];
  WarpAttnState<D> st;
  state_init(st);
  // kSelStages-deep ring: chunks ci+1 .. ci+kSelStages-1 are in flight while ci is used
#pragma unroll
  for (int p = 0; p < kSelStages - 1; ++p) {
    if (p < nch) load_chunk<D>(buf, p, kb, vb, rs, list[p], t + 1, lane);
    cp_async_commit();
  }
  for (int ci = 0; ci < nch; ++ci) {
    const int nx = ci + kSelStages - 1;
    if (nx < nch) load_chunk<D>(buf, nx % kSelStages, kb, vb, rs, list[nx], t + 1, lane);
    cp_async_commit();
    asm volatile("cp.async.wait_group %0;" ::"n"(kSelStages - 1) : "memory");
    __syncwarp();
    attend_chunk<D>(st, qa, buf, ci % kSelStages, list[ci], 0, t + 1, sl2, lane);
    __syncwarp();
  }
  cp_async_wait_0();
  state_reduce_l(st);
  const int r0 = lane >> 2, c = 2 * (lane & 3);
  const float inv0 = st.l[0] > 0.f ? 1.f / st.l[0] : 0.f;
  const float inv1 = st.l[1] > 0.f ? 1.f / st.l[1] : 0.f;
  float* dst = o_sel + (static_cast<size_t>(t) * hq + g * G) * D;
#pragma unroll
  for (int n = 0; n < D / 8; ++n) {
    if (r0 < G)
      *reinterpret_cast<float2*>(dst + r0 * D + n * 8 + c) = make_float2(st.o[n][0] * inv0, st.o[n][1] * inv0);
    if (r0 + 8 < G)
      *reinterpret_cast<float2*>(dst + (r0 + 8) * D + n * 8 + c) = make_float2(st.o[n][2] * inv1, st.o[n][3] * inv1);
  }
}

}  // namespace nsa
