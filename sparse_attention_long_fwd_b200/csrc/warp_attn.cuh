// warp_attn.cuh -- warp-level attention over gathered key chunks (mma.sync m16n8k16).
//
// Used where the keys differ per query token, so no two tokens share a B operand and
// an M=128 tensor-core tile cannot be filled: the selection branch (each (token, group)
// attends to its own top-n blocks of 64 tokens; top168.com article on VideoNSA, section
// "一、革命性的三重注意机制") and the single-query decode. One warp owns the G query heads
// of one KV group for one token (rows 0..G-1 of a 16-row MMA tile, G <= 16): the whole
// GQA group reuses each gathered key/value chunk. Key chunks of 32 tokens are copied
// global -> shared with cp.async into a two-stage per-warp ring while the previous chunk
// is being used (the pages' prefetch-the-next-block advice, CSDN blog section 5.1).
// Softmax is online in fp32 (base 2); the output accumulates in registers.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>
#include "sm100.cuh"

namespace nsa {

constexpr int kChunkKeys = 32;

// Per-warp ring of NST stages, each CK key rows and CK value rows of D bf16; 16-byte
// units are XOR-swizzled by (key & 7) so ldmatrix reads are conflict-free.
template <int D, int CK = kChunkKeys, int NST = 2>
struct WarpChunkBuf {
  alignas(128) __nv_bfloat16 kv[NST][2][CK * D];
};

template <int D>
struct WarpAttnState {
  float m[2];            // running max (base-2 logits) of rows lane/4 and lane/4 + 8
  float l[2];            // this thread's partial row sums (reduced over the quad at the end)
  float o[D / 8][4];     // output accumulator fragments
};

__device__ __forceinline__ uint32_t swz_unit(int row, int unit) { return static_cast<uint32_t>(unit ^ (row & 7)); }

__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
  const uint32_t d = smem_u32(dst);
  const int n = valid ? 16 : 0;  // zero-fill when the source row is out of range
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(n) : "memory");
}
// L2 policy for data read once (a stream): its lines are the first evicted, so what the
// stream's kernel writes for the next kernel stays in L2.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
// L2 policy for data the next kernel reads back: its lines are the last evicted.
__device__ __forceinline__ uint64_t l2_evict_last_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ void st_f32_hint(float* dst, float v, uint64_t policy) {
  asm volatile("st.global.L2::cache_hint.f32 [%0], %1, %2;" ::"l"(dst), "f"(v), "l"(policy) : "memory");
}
__device__ __forceinline__ void cp_async16_hint(void* dst, const void* src, bool valid, uint64_t policy) {
  const uint32_t d = smem_u32(dst);
  const int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2, %3;" ::"r"(d), "l"(src), "r"(n),
               "l"(policy)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_0() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// A fragments of the 16-row query tile: rows 0..G-1 are the group's heads (row stride D
// elements from `q`), rows >= G are zero.
template <int D>
__device__ __forceinline__ void load_q_frags(uint32_t (&a)[D / 16][4], const __nv_bfloat16* q, int G, int lane) {
  const int r0 = lane >> 2, r1 = r0 + 8, c = 2 * (lane & 3);
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks) {
    const int col = ks * 16 + c;
    a[ks][0] = r0 < G ? *reinterpret_cast<const uint32_t*>(q + r0 * D + col) : 0u;
    a[ks][1] = r1 < G ? *reinterpret_cast<const uint32_t*>(q + r1 * D + col) : 0u;
    a[ks][2] = r0 < G ? *reinterpret_cast<const uint32_t*>(q + r0 * D + col + 8) : 0u;
    a[ks][3] = r1 < G ? *reinterpret_cast<const uint32_t*>(q + r1 * D + col + 8) : 0u;
  }
}

// Copy CK key rows (and value rows) starting at token `start` into ring stage `st`.
// Rows at or beyond `row_end` are zero-filled and never read from global memory.
// K/V row `tok` of the head lives at base + tok * row_stride.
// policy: 0, or an L2 policy the copies carry (l2_evict_first_policy for data read once).
template <int D, int CK, int NST>
__device__ __forceinline__ void load_chunk(WarpChunkBuf<D, CK, NST>& buf, int st, const __nv_bfloat16* kbase,
                                           const __nv_bfloat16* vbase, size_t row_stride, int start, int row_end,
                                           int lane, uint64_t policy = 0) {
  constexpr int kUnits = D / 8;  // 16-byte units per row
#pragma unroll
  for (int i = lane; i < CK * kUnits; i += 32) {
    const int row = i / kUnits, unit = i % kUnits;
    const int tok = start + row;
    const bool valid = tok < row_end;
    const size_t src = static_cast<size_t>(valid ? tok : 0) * row_stride + unit * 8;
    const int dst = row * D + static_cast<int>(swz_unit(row, unit)) * 8;
    if (policy != 0) {
      cp_async16_hint(&buf.kv[st][0][dst], kbase + src, valid, policy);
      cp_async16_hint(&buf.kv[st][1][dst], vbase + src, valid, policy);
    } else {
      cp_async16(&buf.kv[st][0][dst], kbase + src, valid);
      cp_async16(&buf.kv[st][1][dst], vbase + src, valid);
    }
  }
}

template <int D>
__device__ __forceinline__ void state_init(WarpAttnState<D>& s) {
  s.m[0] = s.m[1] = -INFINITY;
  s.l[0] = s.l[1] = 0.f;
#pragma unroll
  for (int n = 0; n < D / 8; ++n) s.o[n][0] = s.o[n][1] = s.o[n][2] = s.o[n][3] = 0.f;
}

// One CK-key chunk from ring stage `st`: keys start .. start+CK-1; key `start + c` is
// used iff key_lo <= start + c < key_hi. `sl2` = softmax scale * log2(e).
// If `logits` is non-null, the scaled base-2 logits of rows < G are stored there:
// logits[row * logit_stride + (start + c - logit_base)] for valid keys.
template <int D, int CK, int NST>
__device__ __forceinline__ void attend_chunk(WarpAttnState<D>& s, const uint32_t (&qa)[D / 16][4],
                                             const WarpChunkBuf<D, CK, NST>& buf, int st, int start, int key_lo,
                                             int key_hi, float sl2, int lane, float* logits = nullptr,
                                             int logit_stride = 0, int logit_base = 0, int G = 0) {
  constexpr int NT = CK / 8;   // n-tiles of 8 keys
  constexpr int KS = CK / 16;  // 16-key k-steps of P V
  const uint32_t kaddr = smem_u32(&buf.kv[st][0][0]);
  const uint32_t vaddr = smem_u32(&buf.kv[st][1][0]);
  // ---- S = Q K^T : 16 rows x CK keys (NT n-tiles of 8 keys)
  float sc[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
    for (int ks = 0; ks < D / 16; ks += 2) {
      const int row = nt * 8 + (lane & 7);
      const int unit = ks * 2 + (lane >> 3);  // (ks, lo), (ks, hi), (ks+1, lo), (ks+1, hi)
      uint32_t b0, b1, b2, b3;
      ldsm_x4(kaddr + (row * D + swz_unit(row, unit) * 8) * 2, b0, b1, b2, b3);
      mma_bf16_16816(sc[nt], qa[ks], b0, b1);
      mma_bf16_16816(sc[nt], qa[ks + 1], b2, b3);
    }
  }
  // ---- online softmax (rows r0 = lane/4 -> elements 0,1; r1 = r0+8 -> elements 2,3)
  float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int key = start + nt * 8 + 2 * (lane & 3) + (e & 1);
      const float z = (key >= key_lo && key < key_hi) ? sc[nt][e] * sl2 : -INFINITY;
      sc[nt][e] = z;
      mx[e >> 1] = fmaxf(mx[e >> 1], z);
    }
  }
  if (logits != nullptr) {
    // the next kernel reads these back: they are stored with an L2 evict-last policy
    const uint64_t keep = l2_evict_last_policy();
    const int r0 = lane >> 2;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int row = r0 + (e >> 1) * 8;
        const int key = start + nt * 8 + 2 * (lane & 3) + (e & 1);
        if (row < G && key >= key_lo && key < key_hi)
          st_f32_hint(logits + static_cast<size_t>(row) * logit_stride + (key - logit_base), sc[nt][e], keep);
      }
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
  uint32_t pa[KS][4];  // P as A fragments for the 16-key k-steps
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
    const int kk = nt >> 1, half = nt & 1;
    pa[kk][half * 2 + 0] = pack_bf16x2(p[0], p[1]);
    pa[kk][half * 2 + 1] = pack_bf16x2(p[2], p[3]);
  }
#pragma unroll
  for (int n = 0; n < D / 8; ++n) {
    s.o[n][0] *= alpha[0];
    s.o[n][1] *= alpha[0];
    s.o[n][2] *= alpha[1];
    s.o[n][3] *= alpha[1];
  }
  // ---- O += P V : V chunk rows are keys (k), columns are output dims (n)
#pragma unroll
  for (int kk = 0; kk < KS; ++kk) {
#pragma unroll
    for (int n = 0; n < D / 8; n += 2) {
      const int row = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
      const int unit = n + (lane >> 4);
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(vaddr + (row * D + swz_unit(row, unit) * 8) * 2, b0, b1, b2, b3);
      mma_bf16_16816(s.o[n], pa[kk], b0, b1);
      mma_bf16_16816(s.o[n + 1], pa[kk], b2, b3);
    }
  }
}

// Reduce the per-thread partial row sums over the quad that shares a row.
template <int D>
__device__ __forceinline__ void state_reduce_l(WarpAttnState<D>& s) {
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    s.l[r] += __shfl_xor_sync(0xffffffffu, s.l[r], 1);
    s.l[r] += __shfl_xor_sync(0xffffffffu, s.l[r], 2);
  }
}

// Partial softmax state of one warp in shared memory: rows 0..15, for cross-warp merges.
template <int D>
struct WarpPartial {
  float m[16], l[16];
  float o[16][D];
};

template <int D>
__device__ __forceinline__ void state_store(const WarpAttnState<D>& s, WarpPartial<D>& p, int lane) {
  const int r0 = lane >> 2, c = 2 * (lane & 3);
  if ((lane & 3) == 0) {
    p.m[r0] = s.m[0];
    p.m[r0 + 8] = s.m[1];
    p.l[r0] = s.l[0];
    p.l[r0 + 8] = s.l[1];
  }
#pragma unroll
  for (int n = 0; n < D / 8; ++n) {
    p.o[r0][n * 8 + c] = s.o[n][0];
    p.o[r0][n * 8 + c + 1] = s.o[n][1];
    p.o[r0 + 8][n * 8 + c] = s.o[n][2];
    p.o[r0 + 8][n * 8 + c + 1] = s.o[n][3];
  }
}

}  // namespace nsa
