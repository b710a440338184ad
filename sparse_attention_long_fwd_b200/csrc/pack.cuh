// pack.cuh -- tables and gathers for packed batches whose sequences interleave video and
// text segments.
//
// Video tokens get NSA and text tokens dense attention (shd-paper.top page "VideoNSA:
// Native Sparse Attention Scales Video Understanding", abstract); request lengths vary
// (CSDN blog on VideoNSA, vcloud.csdn.net, section 5.2, item 3). Every stage then runs once
// over the whole batch: the video tokens of all sequences, in order, form one video stream
// (each sequence's video tokens counted as that sequence's positions), and the text rows
// form a text stream whose keys are the rows of the packed batch. These kernels write the
// per-token tables the stages read and, where the streams are not the batch itself, copy
// the rows into them.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

namespace nsa {

// Host-built plan, copied into the workspace.
//   segment s: kPackSeg ints = physical first row, length, video (1) or text (0), first index
//              in its stream, its sequence's first physical row, its sequence's first video
//              stream index, first compressed row and first selection block
//   sequence b: kPackSeq ints = first video stream index, video tokens, first compressed row
//              (a multiple of 128), compressed rows, first selection block, selection blocks
constexpr int kPackSeg = 8;
constexpr int kPackSeq = 6;

struct PackArgs {
  const int* seg;            // [nseg][kPackSeg]
  const int* seq;            // [nseq][kPackSeq]
  int nseg, nseq;
  long long ntok;            // rows of the packed batch
  int hq, hkv, d;
  int cmp_stride, sel_len;
  const __nv_bfloat16 *q, *k, *v;  // packed batch
  __nv_bfloat16 *qv, *kv, *vv;     // video stream copies, or null (the stream is the batch)
  __nv_bfloat16* qt;               // text stream queries, or null (no text rows)
  int4* vinfo;                     // [video stream]
  int2* tinfo;                     // [text stream]
  int* row_tok;                    // [compressed rows]
  int* blk_tok;                    // [selection blocks]
};

__device__ __forceinline__ void copy_row(const __nv_bfloat16* src, __nv_bfloat16* dst, int elems, int lane) {
  const uint4* s = reinterpret_cast<const uint4*>(src);
  uint4* o = reinterpret_cast<uint4*>(dst);
  for (int i = lane; i < elems / 8; i += 32) o[i] = s[i];
}

// One warp per row of the packed batch: its segment (binary search), then its table entry
// and, where needed, the copy of its rows into the stream.
__global__ void __launch_bounds__(256) pack_rows_kernel(const PackArgs a) {
  const long long row = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= a.ntok) return;
  int lo = 0, hi = a.nseg - 1;  // the last segment starting at or before the row
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (a.seg[mid * kPackSeg] <= row) lo = mid; else hi = mid - 1;
  }
  const int* sg = a.seg + lo * kPackSeg;
  const int idx = sg[3] + static_cast<int>(row - sg[0]);  // index in the segment's stream
  const size_t qe = static_cast<size_t>(a.hq) * a.d, ke = static_cast<size_t>(a.hkv) * a.d;
  if (sg[2]) {
    if (lane == 0) a.vinfo[idx] = make_int4(sg[5], sg[6], sg[7], static_cast<int>(row));
    if (a.qv != nullptr) {
      copy_row(a.q + row * qe, a.qv + idx * qe, static_cast<int>(qe), lane);
      copy_row(a.k + row * ke, a.kv + idx * ke, static_cast<int>(ke), lane);
      copy_row(a.v + row * ke, a.vv + idx * ke, static_cast<int>(ke), lane);
    }
  } else {
    if (lane == 0) a.tinfo[idx] = make_int2(static_cast<int>(row), sg[4]);
    copy_row(a.q + row * qe, a.qt + idx * qe, static_cast<int>(qe), lane);
  }
}

// One CTA per sequence: the first stream token of every compressed row (-1 for the rows that
// pad the sequence's rows to a multiple of 128) and of every selection block.
__global__ void __launch_bounds__(256) pack_blocks_kernel(const PackArgs a) {
  const int* sq = a.seq + blockIdx.x * kPackSeq;
  const int v0 = sq[0], cb = sq[2], ncmp = sq[3], gb = sq[4], nsel = sq[5];
  const int padded = (ncmp + 127) / 128 * 128;
  for (int i = threadIdx.x; i < padded; i += blockDim.x) a.row_tok[cb + i] = i < ncmp ? v0 + i * a.cmp_stride : -1;
  for (int j = threadIdx.x; j < nsel; j += blockDim.x) a.blk_tok[gb + j] = v0 + j * a.sel_len;
}

}  // namespace nsa
