// nsa_api.cu -- the C ABI declared in include/nsa.h: argument validation, workspace
// layout, TMA tensor maps and kernel launches for the NSA forward pass on sm_100a.
// The whole library is this one translation unit (the kernels are header-only).
#include <cuda_runtime.h>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include "nsa.h"
#include "sm100.cuh"
#include "tma_host.h"
#include "pool.cuh"
#include "attn_tc.cuh"
#include "topn.cuh"
#include "sel.cuh"
#include "sel_inv.cuh"
#include "decode.cuh"
#include "gate.cuh"
#include "backward.cuh"
#include "backward_tc.cuh"
#include "pack.cuh"

namespace nsa {

// Self-test of the failure-detection path: one warp waits, through the same bounded wait
// every kernel of the library uses, on an mbarrier that nothing ever arrives at. The wait
// gives up after `limit` clock cycles, sets the timeout bit of the device error word and
// the kernel returns normally, leaving the context usable.
__global__ void __launch_bounds__(32) bounded_wait_selftest_kernel(long long limit) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  // phase 0 never completes: no thread arrives and no copy is counted on the barrier
  (void)mbar_wait(&bar, 0, &abort_flag, limit);
}

}  // namespace nsa

namespace {

using nsa::AttnArgs;

constexpr size_t kAlign = 256;
constexpr int kMaxWindowDecode = 4096;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

int ncmp_of(int T, int l, int s) { return T >= l ? (T - l) / s + 1 : 0; }
int nsel_of(int T, int ls) { return (T + ls - 1) / ls; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

// Checks shared by every entry point. Returns NSA_OK or an error code.
int check_common(const nsa_params_t* p) {
  if (p == nullptr) return NSA_ERR_INVALID_ARG;
  if (p->n_tokens < 1 || p->num_q_heads < 1 || p->num_kv_heads < 1 || p->head_dim < 1) return NSA_ERR_INVALID_ARG;
  if (p->num_q_heads % p->num_kv_heads != 0) return NSA_ERR_INVALID_ARG;
  if (p->cmp_block < 1 || p->cmp_stride < 1 || p->sel_block < 1 || p->window < 1 || p->top_n < 1)
    return NSA_ERR_INVALID_ARG;
  if (p->out_dtype != NSA_OUT_BF16 && p->out_dtype != NSA_OUT_F32) return NSA_ERR_INVALID_ARG;
  if (p->keep_branch_stats != 0 && p->keep_branch_stats != 1) return NSA_ERR_INVALID_ARG;
  if (p->head_dim != 64 && p->head_dim != 128) return NSA_ERR_UNSUPPORTED;
  if (p->num_q_heads / p->num_kv_heads > 16) return NSA_ERR_UNSUPPORTED;
  if (p->cmp_block != 32 || p->cmp_stride != 16 || p->sel_block != 64) return NSA_ERR_UNSUPPORTED;
  if (p->top_n < 3 || p->top_n > 64) return NSA_ERR_UNSUPPORTED;
  // element counts of the largest tensors must stay within 2^31 rows for the TMA maps
  if (static_cast<long long>(p->n_tokens) * p->num_q_heads > (1LL << 31)) return NSA_ERR_UNSUPPORTED;
  return NSA_OK;
}

int check_device() {
  static std::mutex mu;
  static int cached[64];
  static bool init = false;
  std::lock_guard<std::mutex> lock(mu);
  if (!init) {
    for (int& c : cached) c = -1;
    init = true;
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return NSA_ERR_CUDA;
  if (dev < 0 || dev >= 64) return NSA_ERR_UNSUPPORTED;
  if (cached[dev] < 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return NSA_ERR_CUDA;
    cached[dev] = (major == 10 && minor == 0) ? 1 : 0;
  }
  return cached[dev] == 1 ? NSA_OK : NSA_ERR_UNSUPPORTED;
}

struct PrefillLayout {
  size_t kc, vc, o_cmp, lse, scores, sel_idx, o_win, total;
  size_t o_sel, lse_sel, lse_win;  // kept branch statistics, or 0
  // block-major selected branch: bucket counters, offsets, bucketed entries, partials
  size_t sel_cnt, sel_eoff, sel_toff, sel_list, sel_row, part_o, part_ml;
  long long part_rows;  // 128 x the bound on selected-branch tiles
  int ncmp, nsel;
  int score_stride;     // floats per score row: nsel rounded up to 4, so rows are 16-byte aligned
};

// Workspace layout of the NSA rows of one call: nv stream rows, ncmp_rows compressed rows,
// nsel_cols selection-block columns per group (the bucket space) and score rows of up to
// nsel_max blocks (one sequence: ncmp_rows = Ncmp(nv), nsel_cols = nsel_max = Nsel(nv)).
PrefillLayout video_layout(int nv, int ncmp_rows, int nsel_cols, int nsel_max, int hq, int hkv, int d, int top_n,
                           bool keep = false) {
  PrefillLayout L{};
  L.ncmp = ncmp_rows;
  L.nsel = nsel_cols;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + (bytes > 0 ? bytes : 1));
    return at;
  };
  const size_t cmp_rows = static_cast<size_t>(L.ncmp > 0 ? L.ncmp : 1);
  L.kc = take(cmp_rows * hkv * d * 2);
  L.vc = take(cmp_rows * hkv * d * 2);
  L.o_cmp = take(static_cast<size_t>(nv) * hq * d * 2);
  L.lse = take(static_cast<size_t>(nv) * hq * 4);
  L.score_stride = (nsel_max + 3) / 4 * 4;
  L.scores = take(static_cast<size_t>(nv) * hkv * (L.score_stride > 0 ? L.score_stride : 4) * 4);
  L.sel_idx = take(static_cast<size_t>(nv) * hkv * top_n * 4);
  L.o_win = take(static_cast<size_t>(nv) * hq * d * 2);
  const size_t buckets = static_cast<size_t>(hkv) * (L.nsel > 0 ? L.nsel : 1);
  const size_t entries = static_cast<size_t>(nv) * hkv * top_n;
  L.sel_cnt = take(2 * buckets * 4);
  L.sel_eoff = take((buckets + 1) * 4);
  L.sel_toff = take((buckets + 1) * 4);
  L.sel_list = take(entries * 4);
  L.sel_row = take(entries * 4);
  {
    const int G = hq / (hkv > 0 ? hkv : 1);  // a token's heads take G consecutive tile rows
    const size_t tiles = (entries + (128 / G) - 1) / (128 / G) + buckets;
    L.part_rows = static_cast<long long>(tiles) * 128;
  }
  L.part_o = take(static_cast<size_t>(L.part_rows) * d * 2);
  L.part_ml = take(static_cast<size_t>(L.part_rows) * 16);
  if (keep) {
    L.o_sel = take(static_cast<size_t>(nv) * hq * d * 2);
    L.lse_sel = take(static_cast<size_t>(nv) * hq * 4);
    L.lse_win = take(static_cast<size_t>(nv) * hq * 4);
  }
  L.total = off;
  return L;
}

PrefillLayout prefill_layout(const nsa_params_t* p) {
  const int nv = p->n_video;
  const int ns = nsel_of(nv, p->sel_block);
  return video_layout(nv, ncmp_of(nv, p->cmp_block, p->cmp_stride), ns, ns, p->num_q_heads, p->num_kv_heads,
                      p->head_dim, p->top_n, p->keep_branch_stats != 0);
}

struct DecodeLayout {
  size_t logits, part, o_cmp, lse, scores, sel_idx, o_win, total;
  int ncmax, nsel_max, nsplit;
};

DecodeLayout decode_layout(const nsa_params_t* p) {
  DecodeLayout L{};
  const int B = p->batch, hq = p->num_q_heads, hkv = p->num_kv_heads, d = p->head_dim;
  const int G = hq / hkv;
  L.ncmax = ncmp_of(p->n_tokens, p->cmp_block, p->cmp_stride);
  L.nsel_max = nsel_of(p->n_tokens, p->sel_block);
  L.nsplit = (L.ncmax + 511) / 512;
  if (L.nsplit < 1) L.nsplit = 1;
  if (L.nsplit > 64) L.nsplit = 64;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + (bytes > 0 ? bytes : 1));
    return at;
  };
  // logit rows of ncmax rounded up to 4 floats (16-byte rows: dec_select reads them as float4)
  L.logits = take(static_cast<size_t>(B) * hkv * G * ((L.ncmax + 3) / 4 * 4 > 0 ? (L.ncmax + 3) / 4 * 4 : 4) * 4);
  L.part = take(static_cast<size_t>(B) * hkv * L.nsplit * G * (2 + d) * 4);
  L.o_cmp = take(static_cast<size_t>(B) * hq * d * 4);
  L.lse = take(static_cast<size_t>(B) * hq * 4);
  L.scores = take(static_cast<size_t>(B) * hkv * L.nsel_max * 4);
  L.sel_idx = take(static_cast<size_t>(B) * hkv * p->top_n * 4);
  L.o_win = take(static_cast<size_t>(B) * hq * d * 4);
  L.total = off;
  return L;
}

// NSA_DEBUG_SYNC=1 in the environment: synchronise after every launch and report each
// kernel's completion (and any error) on stderr. Off by default; costs a sync per kernel.
bool debug_sync() {
  static const bool on = [] {
    const char* e = std::getenv("NSA_DEBUG_SYNC");
    return e != nullptr && e[0] == '1';
  }();
  return on;
}

// Caller-registered stage events (nsa_profile_stages); g_stage_next counts the events
// recorded by the current call. Per host thread: a registration made on one thread never
// records events for calls made on another.
thread_local void* const* g_stage_events = nullptr;
thread_local int g_stage_count = 0;
thread_local int g_stage_next = 0;

void stage_begin(cudaStream_t st) {
  g_stage_next = 0;
  if (g_stage_count > 0) cudaEventRecord(static_cast<cudaEvent_t>(g_stage_events[g_stage_next++]), st);
}

int launch_status(const char* name = "kernel", cudaStream_t st = nullptr, bool stage_end = true) {
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess && stage_end && g_stage_next < g_stage_count)
    e = cudaEventRecord(static_cast<cudaEvent_t>(g_stage_events[g_stage_next++]), st);
  if (e == cudaSuccess && debug_sync()) {
    std::fprintf(stderr, "[nsa] %s launched\n", name);
    std::fflush(stderr);
    e = cudaStreamSynchronize(st);
    unsigned int word = 0;
    cudaMemcpyFromSymbol(&word, nsa::g_device_error, sizeof(word));
    std::fprintf(stderr, "[nsa] %s finished: %s, device error word %u\n", name, cudaGetErrorString(e), word);
    std::fflush(stderr);
  }
  return e == cudaSuccess ? NSA_OK : NSA_ERR_CUDA;
}

// Streaming multiprocessors of the current device (cached per device); 0 on error.
int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cached[dev] = n;
  }
  return cached[dev];
}

template <typename K>
int set_smem(K kernel, size_t bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes)) ==
                 cudaSuccess
             ? NSA_OK
             : NSA_ERR_CUDA;
}

// ------------------------------------------------------------------ launchers
// wk, wv: per-head block weights [hkv][l] of the learnable compression, or null for the mean
int launch_pool(const void* k, const void* v, void* kc, void* vc, int nseq, int T, int hkv, int d, int ncmp, int l,
                int s, cudaStream_t st, const float* wk = nullptr, const float* wv = nullptr,
                const int* row_tok = nullptr) {
  if (ncmp <= 0) return NSA_OK;
  const long long threads = static_cast<long long>(nseq) * ncmp * hkv * (d / 2);
  const unsigned blocks = static_cast<unsigned>((threads + 255) / 256);
  nsa::pool_kernel<<<dim3(blocks, 1, 2), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v), static_cast<__nv_bfloat16*>(kc),
      static_cast<__nv_bfloat16*>(vc), wk, wv, nseq, T, hkv, d, ncmp, l, s, row_tok);
  return launch_status("pool", st);
}

template <int D, int MODE>
int launch_attn(const CUtensorMap& qm, const CUtensorMap& km, const CUtensorMap& vm, const AttnArgs& a,
                cudaStream_t st) {
  if (a.n_tiles <= 0) return NSA_OK;
  const size_t smem = sizeof(nsa::AttnSmem<D, MODE>) + 1024;
  const bool packed = a.vinfo != nullptr || a.tinfo != nullptr;
  auto kern = packed ? nsa::attn_tile_kernel<D, MODE, true> : nsa::attn_tile_kernel<D, MODE, false>;
  if (set_smem(kern, smem) != NSA_OK) return NSA_ERR_CUDA;
  // persistent modes: one CTA per SM walks the (tile, group) items; otherwise one CTA per item
  const long long items = static_cast<long long>(a.n_tiles) * a.hkv;
  const int sms = sm_count();
  if (sms <= 0) return NSA_ERR_CUDA;
  const unsigned grid =
      static_cast<unsigned>(nsa::AttnCfg<MODE>::kPersistent && items > sms ? sms : items);
  kern<<<grid, nsa::AttnCfg<MODE>::kThreads, smem, st>>>(qm, km, vm, a);
  return launch_status(MODE == nsa::kModeCmp ? "attn_cmp" : MODE == nsa::kModeWin ? "attn_win" : "attn_dense", st);
}

// What one prefill call computes, stage by stage: NSA over the rows of a video stream and
// dense causal attention over a set of text rows. One sequence: the stream is the video
// prefix itself and the text rows follow it. A packed batch: the stream is every sequence's
// video tokens back to back (tables give each token its sequence), and the text rows are
// gathered into a stream of their own whose keys are the rows of the packed batch.
struct StageGeo {
  const void *q, *k, *v;   // video stream: q [rows][hq][D], k, v [rows][hkv][D]
  int rows;                // rows of those tensors (the extent of their TMA maps)
  int nv;                  // NSA rows: stream rows [0, nv)
  const int4* vinfo;       // packed: per stream row (sequence's first row, first compressed row,
                           // first selection block, row in the batch); null: one sequence
  const int* row_tok;      // packed: first stream token of every compressed row (-1: padding)
  const int* blk_tok;      // packed: first stream token of every selection block
  int nsel_max;            // selection blocks of the longest sequence
  const void* qt;          // text rows: queries [qt_rows][hq][D]
  int qt_rows, t_begin, t_end;  // dense rows [t_begin, t_end) of qt
  const int2* tinfo;       // packed: per text row (row in the batch, first row of its sequence)
  const void *kd, *vd;     // keys and values of the dense rows [kd_rows][hkv][D]
  int kd_rows;
  const float* gates;      // [rows of the batch][hq][3]
  void* out;               // [rows of the batch][hq][D]
};

template <int D>
int video_stages(const nsa_params_t* p, const StageGeo& geo, const PrefillLayout& L, int32_t* out_sel_idx,
                 uint8_t* ws, cudaStream_t st, const float* phi_k, const float* phi_v) {
  const int nv = geo.nv, hq = p->num_q_heads, hkv = p->num_kv_heads;
  const int G = hq / hkv;
  const int T = 128 / G;
  int Gc = 1;  // compressed mode: G rounded up to a power of two, so a token's heads share a warp
  while (Gc < G) Gc <<= 1;
  const int Tc = 128 / Gc;
  const float scale = p->softmax_scale > 0.f ? p->softmax_scale : 1.0f / std::sqrt(static_cast<float>(D));
  const float sl2 = scale * 1.4426950408889634f;
  int rc;
  CUtensorMap qmap, qcmap, kmap, vmap, kcmap, vcmap;
  const uint64_t qs1 = static_cast<uint64_t>(D) * 2, qs2 = static_cast<uint64_t>(hq) * D * 2;
  const uint64_t ks1 = static_cast<uint64_t>(D) * 2, ks2 = static_cast<uint64_t>(hkv) * D * 2;
  auto* kc = ws + L.kc;
  auto* vc = ws + L.vc;
  const int ncmp_rows = L.ncmp > 0 ? L.ncmp : 1;
  if (!nsa::make_tmap_bf16_3d(&qmap, geo.q, D, hq, geo.rows, qs1, qs2, 64, G, T) ||
      !nsa::make_tmap_bf16_3d(&kmap, geo.k, D, hkv, geo.rows, ks1, ks2, 64, 1, nsa::kBN) ||
      !nsa::make_tmap_bf16_3d(&vmap, geo.v, D, hkv, geo.rows, ks1, ks2, 64, 1, nsa::kBN) ||
      !nsa::make_tmap_bf16_3d(&kcmap, kc, D, hkv, ncmp_rows, ks1, ks2, 64, 1, nsa::kBN) ||
      !nsa::make_tmap_bf16_3d(&vcmap, vc, D, hkv, ncmp_rows, ks1, ks2, 64, 1, nsa::kBN) ||
      !nsa::make_tmap_bf16_3d(&qcmap, geo.q, D, hq, geo.rows, qs1, qs2, 64, Gc, Tc))
    return NSA_ERR_CUDA;
  AttnArgs a{};
  a.hq = hq;
  a.hkv = hkv;
  a.G = G;
  a.T = T;
  a.Gp = G;
  a.scale_log2 = sl2;
  a.cmp_len = p->cmp_block;
  a.cmp_stride = p->cmp_stride;
  a.window = p->window;
  a.sel_len = p->sel_block;
  a.nsel = L.score_stride;  // the score rows' stride
  a.out = geo.out;
  a.out_f32 = p->out_dtype == NSA_OUT_F32;
  a.vinfo = geo.vinfo;
  // 1. compression: Kc, Vc of the video stream
  if ((rc = launch_pool(geo.k, geo.v, kc, vc, 1, nv, hkv, D, L.ncmp, p->cmp_block, p->cmp_stride, st, phi_k, phi_v,
                        geo.row_tok)) != NSA_OK)
    return rc;
  // 2. compressed branch + block scores
  a.q_begin = 0;
  a.q_end = nv;
  a.o_cmp = reinterpret_cast<__half*>(ws + L.o_cmp);
  a.lse = reinterpret_cast<float*>(ws + L.lse);
  a.scores = reinterpret_cast<float*>(ws + L.scores);
  {
    AttnArgs ac = a;
    ac.Gp = Gc;
    ac.T = Tc;
    ac.n_tiles = (nv + Tc - 1) / Tc;
    if ((rc = launch_attn<D, nsa::kModeCmp>(qcmap, kcmap, vcmap, ac, st)) != NSA_OK) return rc;
  }
  a.n_tiles = (nv + T - 1) / T;
  // 3. top-n selection
  {
    const int nitems = nv * hkv;
    const int nwords = (geo.nsel_max + 31) / 32;
    // every row on the register path (fewer than 2,048 blocks, top_n <= 32): 64 list
    // entries per warp, so shared memory does not limit the warps per SM
    const bool regs_only = geo.nsel_max <= 32 * 64 && p->top_n <= 32;
    const size_t smem =
        static_cast<size_t>(nsa::kTopnWarps) * (regs_only ? 64 : 2 * geo.nsel_max + nwords) * 4;
    const bool packed = geo.vinfo != nullptr;
    auto kern = regs_only ? (packed ? nsa::topn_kernel<true, true> : nsa::topn_kernel<true, false>)
                          : (packed ? nsa::topn_kernel<false, true> : nsa::topn_kernel<false, false>);
    if (set_smem(kern, smem) != NSA_OK) return NSA_ERR_CUDA;
    int blocks = (nitems + nsa::kTopnWarps - 1) / nsa::kTopnWarps;
    if (blocks > 148 * 32) blocks = 148 * 32;
    kern<<<blocks, nsa::kTopnWarps * 32, smem, st>>>(a.scores, nitems, hkv, geo.nsel_max, L.score_stride,
                                                      p->sel_block, p->top_n,
                                                      reinterpret_cast<int32_t*>(ws + L.sel_idx), out_sel_idx,
                                                      geo.vinfo);
    if ((rc = launch_status("topn", st)) != NSA_OK) return rc;
  }
  // 4. selected branch, block-major: bucket (token, slot) pairs by (group, block),
  //    one tensor-core tile per bucket tile, then merge each row's partials
  const int m = hkv * L.nsel;
  const int Gp = G;  // tile rows token * G + head: no padding heads
  const int TT = 128 / Gp;
  const long long entries = static_cast<long long>(nv) * hkv * p->top_n;
  nsa::SelInvArgs sa{};
  sa.nv = nv;
  sa.hq = hq;
  sa.hkv = hkv;
  sa.G = G;
  sa.Gp = Gp;
  sa.TT = TT;
  sa.nsel = L.nsel;
  sa.top_n = p->top_n;
  sa.sel_len = p->sel_block;
  sa.sl2 = sl2;
  sa.sel_idx = reinterpret_cast<const int32_t*>(ws + L.sel_idx);
  sa.cnt = reinterpret_cast<int*>(ws + L.sel_cnt);
  sa.cursor = sa.cnt + m;
  sa.ent_off = reinterpret_cast<int*>(ws + L.sel_eoff);
  sa.tile_off = reinterpret_cast<int*>(ws + L.sel_toff);
  sa.list = reinterpret_cast<int*>(ws + L.sel_list);
  sa.row_of = reinterpret_cast<int*>(ws + L.sel_row);
  sa.part_rows = L.part_rows;
  sa.part_o = reinterpret_cast<const __half*>(ws + L.part_o);
  sa.part_ml = reinterpret_cast<float4*>(ws + L.part_ml);
  sa.o_cmp = reinterpret_cast<const __half*>(ws + L.o_cmp);
  sa.o_win = reinterpret_cast<const __half*>(ws + L.o_win);
  sa.o_sel = L.o_sel != 0 ? reinterpret_cast<__half*>(ws + L.o_sel) : nullptr;
  sa.lse_sel = L.lse_sel != 0 ? reinterpret_cast<float*>(ws + L.lse_sel) : nullptr;
  sa.gates = geo.gates;
  sa.out = geo.out;
  sa.out_f32 = p->out_dtype == NSA_OUT_F32;
  sa.q = static_cast<const __nv_bfloat16*>(geo.q);
  sa.vinfo = geo.vinfo;
  sa.blk_tok = geo.blk_tok;
  CUtensorMap k64map, v64map, omap;
  // partial rows [part_rows][D] fp16: a store box is 32 rows x one 64-column half
  if (!nsa::make_tmap_f16_3d(&omap, ws + L.part_o, 64, D / 64, static_cast<uint64_t>(L.part_rows), 128,
                             static_cast<uint64_t>(D) * 2, 64, 1, 32) ||
      !nsa::make_tmap_bf16_3d(&k64map, geo.k, D, hkv, geo.rows, ks1, ks2, 64, 1, 64) ||
      !nsa::make_tmap_bf16_3d(&v64map, geo.v, D, hkv, geo.rows, ks1, ks2, 64, 1, 64))
    return NSA_ERR_CUDA;
  if (cudaMemsetAsync(sa.cnt, 0, 2 * static_cast<size_t>(m) * 4, st) != cudaSuccess) return NSA_ERR_CUDA;
  long long eb = (entries + 255) / 256;
  const unsigned ebl = static_cast<unsigned>(eb < 148 * 16 ? (eb > 0 ? eb : 1) : 148 * 16);
  nsa::sel_count_kernel<<<ebl, 256, 0, st>>>(sa);
  if ((rc = launch_status("sel_count", st, false)) != NSA_OK) return rc;
  nsa::sel_scan_kernel<<<1, 1024, 0, st>>>(sa);
  if ((rc = launch_status("sel_scan", st, false)) != NSA_OK) return rc;
  nsa::sel_scatter_kernel<<<ebl, 256, 0, st>>>(sa);
  if ((rc = launch_status("sel_scatter", st)) != NSA_OK) return rc;
  {
    // persistent: one CTA per SM (512 TMEM columns each; the shared-memory request keeps
    // a second CTA off the SM)
    size_t smem = sizeof(nsa::SelTileSmem<D>) + 1024;
    if (smem < 116 * 1024) smem = 116 * 1024;
    auto kern = nsa::sel_tile_kernel<D>;
    if (set_smem(kern, smem) != NSA_OK) return NSA_ERR_CUDA;
    const long long max_tiles = L.part_rows / 128;
    const int nsm = sm_count();
    if (nsm <= 0) return NSA_ERR_CUDA;
    const unsigned grid = static_cast<unsigned>(max_tiles < nsm ? max_tiles : nsm);
    kern<<<grid, nsa::kSelTileThreads, smem, st>>>(k64map, v64map, omap, sa);
    if ((rc = launch_status("sel_tile", st)) != NSA_OK) return rc;
  }
  // 5. sliding window -> o_win
  a.o_win = reinterpret_cast<__half*>(ws + L.o_win);
  a.lse_win = L.lse_win != 0 ? reinterpret_cast<float*>(ws + L.lse_win) : nullptr;
  if ((rc = launch_attn<D, nsa::kModeWin>(qmap, kmap, vmap, a, st)) != NSA_OK) return rc;
  // 6. merge of the selected partials + gated combine -> out (the NSA rows)
  const long long rows = static_cast<long long>(nv) * hq;
  nsa::sel_merge_kernel<D><<<static_cast<unsigned>((rows + 7) / 8), 256, 0, st>>>(sa);
  return launch_status("sel_merge", st);
}

// Dense causal attention of the text rows [t_begin, t_end) of geo.qt.
template <int D>
int text_stage(const nsa_params_t* p, const StageGeo& geo, cudaStream_t st) {
  if (geo.t_end <= geo.t_begin) return NSA_OK;
  const int hq = p->num_q_heads, hkv = p->num_kv_heads;
  const int G = hq / hkv;
  const int T = 128 / G;
  const float scale = p->softmax_scale > 0.f ? p->softmax_scale : 1.0f / std::sqrt(static_cast<float>(D));
  CUtensorMap qmap, kmap, vmap;
  const uint64_t qs1 = static_cast<uint64_t>(D) * 2, qs2 = static_cast<uint64_t>(hq) * D * 2;
  const uint64_t ks1 = static_cast<uint64_t>(D) * 2, ks2 = static_cast<uint64_t>(hkv) * D * 2;
  if (!nsa::make_tmap_bf16_3d(&qmap, geo.qt, D, hq, geo.qt_rows, qs1, qs2, 64, G, T) ||
      !nsa::make_tmap_bf16_3d(&kmap, geo.kd, D, hkv, geo.kd_rows, ks1, ks2, 64, 1, nsa::kBN) ||
      !nsa::make_tmap_bf16_3d(&vmap, geo.vd, D, hkv, geo.kd_rows, ks1, ks2, 64, 1, nsa::kBN))
    return NSA_ERR_CUDA;
  AttnArgs a{};
  a.hq = hq;
  a.hkv = hkv;
  a.G = G;
  a.T = T;
  a.Gp = G;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.cmp_len = p->cmp_block;
  a.cmp_stride = p->cmp_stride;
  a.window = p->window;
  a.sel_len = p->sel_block;
  a.out = geo.out;
  a.out_f32 = p->out_dtype == NSA_OUT_F32;
  a.tinfo = geo.tinfo;
  a.q_begin = geo.t_begin;
  a.q_end = geo.t_end;
  a.n_tiles = (geo.t_end - geo.t_begin + T - 1) / T;
  return launch_attn<D, nsa::kModeDense>(qmap, kmap, vmap, a, st);
}

template <int D>
int prefill_impl(const nsa_params_t* p, const void* q, const void* k, const void* v, const float* gates, void* out,
                 int32_t* out_sel_idx, uint8_t* ws, cudaStream_t st, const float* phi_k = nullptr,
                 const float* phi_v = nullptr) {
  const PrefillLayout L = prefill_layout(p);
  const int N = p->n_tokens, nv = p->n_video;
  StageGeo geo{};
  geo.q = q;
  geo.k = k;
  geo.v = v;
  geo.rows = N;
  geo.nv = nv;
  geo.nsel_max = L.nsel;
  geo.qt = q;
  geo.qt_rows = N;
  geo.t_begin = nv;  // the trailing text rows
  geo.t_end = N;
  geo.kd = k;
  geo.vd = v;
  geo.kd_rows = N;
  geo.gates = gates;
  geo.out = out;
  int rc;
  if (nv > 0 && (rc = video_stages<D>(p, geo, L, out_sel_idx, ws, st, phi_k, phi_v)) != NSA_OK) return rc;
  return text_stage<D>(p, geo, st);
}

// Launch with programmatic stream serialisation: the kernel may start while the previous
// one in the stream finishes, and waits for it (griddepcontrol.wait) before reading its
// results.
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                             Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

template <int D>
int decode_impl(const nsa_params_t* p, const void* q, const void* kcache, const void* vcache, const void* kcmp,
                const void* vcmp, const int32_t* seq_lens, const float* gates, void* out, int32_t* out_sel_idx,
                uint8_t* ws, cudaStream_t st) {
  const DecodeLayout L = decode_layout(p);
  nsa::DecArgs a{};
  a.batch = p->batch;
  a.lmax = p->n_tokens;
  a.hq = p->num_q_heads;
  a.hkv = p->num_kv_heads;
  a.G = a.hq / a.hkv;
  a.d = D;
  a.ncmax = L.ncmax;
  a.lstride = (L.ncmax + 3) / 4 * 4;
  a.nsplit = L.nsplit;
  a.cmp_len = p->cmp_block;
  a.cmp_stride = p->cmp_stride;
  a.sel_len = p->sel_block;
  a.top_n = p->top_n;
  a.window = p->window;
  a.nsel_max = L.nsel_max;
  const float scale = p->softmax_scale > 0.f ? p->softmax_scale : 1.0f / std::sqrt(static_cast<float>(D));
  a.sl2 = scale * 1.4426950408889634f;
  a.logits = reinterpret_cast<float*>(ws + L.logits);
  a.part = reinterpret_cast<float*>(ws + L.part);
  a.o_cmp = reinterpret_cast<float*>(ws + L.o_cmp);
  a.lse = reinterpret_cast<float*>(ws + L.lse);
  a.scores = reinterpret_cast<float*>(ws + L.scores);
  a.sel_idx = reinterpret_cast<int32_t*>(ws + L.sel_idx);
  a.o_win = reinterpret_cast<float*>(ws + L.o_win);
  a.gates = gates;
  a.out = out;
  a.out_f32 = p->out_dtype == NSA_OUT_F32;
  const auto* qq = static_cast<const __nv_bfloat16*>(q);
  int rc;
  const size_t smem = sizeof(nsa::DecSmem<D>) + 128;
  {
    auto kern = nsa::dec_cmp_kernel<D>;
    if (set_smem(kern, smem) != NSA_OK) return NSA_ERR_CUDA;
    // x < nsplit: slices of the compressed cache; x = nsplit: the window branch
    kern<<<dim3(L.nsplit + 1, a.batch * a.hkv), nsa::kDecWarps * 32, smem, st>>>(
        qq, static_cast<const __nv_bfloat16*>(kcmp), static_cast<const __nv_bfloat16*>(vcmp),
        static_cast<const __nv_bfloat16*>(kcache), static_cast<const __nv_bfloat16*>(vcache), seq_lens, a);
    if ((rc = launch_status("dec_cmp", st)) != NSA_OK) return rc;
  }
  {
    const size_t ssm = (2 * static_cast<size_t>(L.nsel_max) + L.nsel_max / 32 + 1 + 16) * 4;
    auto kern = nsa::dec_select_kernel<D>;
    if (set_smem(kern, ssm) != NSA_OK) return NSA_ERR_CUDA;
    if (launch_dependent(kern, dim3(a.batch * a.hkv), dim3(256), ssm, st, seq_lens, a, out_sel_idx) != cudaSuccess) {
      cudaGetLastError();  // (clear it: the status is returned here)
      return NSA_ERR_CUDA;
    }
    if ((rc = launch_status("dec_select", st)) != NSA_OK) return rc;
  }
  {
    auto kern = nsa::dec_branch_kernel<D>;
    if (set_smem(kern, smem) != NSA_OK) return NSA_ERR_CUDA;
    if (launch_dependent(kern, dim3(a.batch * a.hkv), dim3(nsa::kDecWarps * 32), smem, st, qq,
                         static_cast<const __nv_bfloat16*>(kcache), static_cast<const __nv_bfloat16*>(vcache), seq_lens,
                         a) != cudaSuccess) {
      cudaGetLastError();  // (clear it: the status is returned here)
      return NSA_ERR_CUDA;
    }
    if ((rc = launch_status("dec_branch", st)) != NSA_OK) return rc;
  }
  return NSA_OK;
}

// ------------------------------------------------------------------ packed batches
// A plan of a packed batch, built on the host from cu_seqlens and the segment list.
struct PackPlan {
  int B = 0, S = 0;
  long long N = 0;
  int nv = 0, nt = 0;         // video stream rows, text stream rows
  int kc_rows = 0;            // compressed rows of all sequences, each padded to 128
  int nsel_cols = 0;          // selection blocks of all sequences
  int nsel_max = 0;           // selection blocks of the longest video stream
  bool gather = false;        // the video stream is not the batch itself (text precedes video)
  std::vector<int> seg, seq;  // nsa::kPackSeg ints per segment, nsa::kPackSeq per sequence
};

int build_plan(const nsa_params_t* p, const int32_t* cu, int batch, const int32_t* seg_lens, const uint8_t* seg_video,
               int nseg, PackPlan& P) {
  int rc = check_common(p);
  if (rc != NSA_OK) return rc;
  if (!cu || batch < 1 || cu[0] != 0 || cu[batch] != p->n_tokens || nseg < 0 || (nseg > 0 && (!seg_lens || !seg_video)))
    return NSA_ERR_INVALID_ARG;
  P = PackPlan{};
  P.B = batch;
  P.S = nseg;
  P.N = p->n_tokens;
  P.seg.resize(static_cast<size_t>(nseg) * nsa::kPackSeg);
  P.seq.resize(static_cast<size_t>(batch) * nsa::kPackSeq);
  long long pos = 0;
  int s = 0;
  bool text_seen = false;
  for (int b = 0; b < batch; ++b) {
    if (cu[b + 1] < cu[b]) return NSA_ERR_INVALID_ARG;
    const int v0 = P.nv;
    int nvb = 0;
    // the sequence's segments: first pass for its video count, second for the table
    const int s_first = s;
    while (pos < cu[b + 1]) {
      if (s >= nseg || seg_lens[s] <= 0 || pos + seg_lens[s] > cu[b + 1]) return NSA_ERR_INVALID_ARG;
      if (seg_video[s] > 1) return NSA_ERR_INVALID_ARG;
      if (seg_video[s]) {
        nvb += seg_lens[s];
        if (text_seen) P.gather = true;
      } else {
        text_seen = true;
      }
      pos += seg_lens[s];
      ++s;
    }
    const int ncmp = ncmp_of(nvb, p->cmp_block, p->cmp_stride);
    const int nsel = nsel_of(nvb, p->sel_block);
    int* sq = &P.seq[static_cast<size_t>(b) * nsa::kPackSeq];
    sq[0] = v0;
    sq[1] = nvb;
    sq[2] = P.kc_rows;
    sq[3] = ncmp;
    sq[4] = P.nsel_cols;
    sq[5] = nsel;
    long long sp = cu[b];
    int vidx = v0;
    for (int x = s_first; x < s; ++x) {
      int* sg = &P.seg[static_cast<size_t>(x) * nsa::kPackSeg];
      sg[0] = static_cast<int>(sp);
      sg[1] = seg_lens[x];
      sg[2] = seg_video[x] ? 1 : 0;
      sg[3] = seg_video[x] ? vidx : P.nt;
      sg[4] = cu[b];
      sg[5] = v0;
      sg[6] = sq[2];
      sg[7] = sq[4];
      if (seg_video[x]) vidx += seg_lens[x];
      else P.nt += seg_lens[x];
      sp += seg_lens[x];
    }
    P.nv += nvb;
    P.kc_rows += (ncmp + 127) / 128 * 128;
    P.nsel_cols += nsel;
    if (nsel > P.nsel_max) P.nsel_max = nsel;
  }
  if (s != nseg) return NSA_ERR_INVALID_ARG;
  if (P.nsel_max > 8192) return NSA_ERR_UNSUPPORTED;
  // the packed video stream keeps every stage's indices in 32 bits
  if (static_cast<long long>(P.nsel_cols) * p->num_kv_heads > (1LL << 30)) return NSA_ERR_UNSUPPORTED;
  return NSA_OK;
}

// Workspace of a packed call: the plan, the tables, the stream copies, then the NSA rows.
struct PackLayout {
  size_t seg, seq, vinfo, tinfo, row_tok, blk_tok, qv, kv, vv, qt, video, total;
  PrefillLayout L;
};

PackLayout pack_layout(const nsa_params_t* p, const PackPlan& P) {
  PackLayout W{};
  const size_t hq = p->num_q_heads, hkv = p->num_kv_heads, d = p->head_dim;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + (bytes > 0 ? bytes : 1));
    return at;
  };
  W.seg = take(P.seg.size() * 4);
  W.seq = take(P.seq.size() * 4);
  W.vinfo = take(static_cast<size_t>(P.nv) * 16);
  W.tinfo = take(static_cast<size_t>(P.nt) * 8);
  W.row_tok = take(static_cast<size_t>(P.kc_rows) * 4);
  W.blk_tok = take(static_cast<size_t>(P.nsel_cols) * 4);
  const size_t nvg = P.gather ? static_cast<size_t>(P.nv) : 0;
  W.qv = take(nvg * hq * d * 2);
  W.kv = take(nvg * hkv * d * 2);
  W.vv = take(nvg * hkv * d * 2);
  W.qt = take(static_cast<size_t>(P.nt) * hq * d * 2);
  W.L = video_layout(P.nv, P.kc_rows, P.nsel_cols, P.nsel_max, p->num_q_heads, p->num_kv_heads, p->head_dim,
                     p->top_n);
  W.video = take(W.L.total);
  W.total = off;
  return W;
}

template <int D>
int packed_impl(const nsa_params_t* p, const PackPlan& P, const PackLayout& W, const void* q, const void* k,
                const void* v, const float* gates, void* out, int32_t* out_sel_idx, uint8_t* ws, cudaStream_t st) {
  int rc;
  // the plan's two tables, one copy each from host memory (a copy from pageable memory is
  // staged by the driver before cudaMemcpyAsync returns, so the plan may go out of scope)
  if (P.seg.size() > 0 &&
      cudaMemcpyAsync(ws + W.seg, P.seg.data(), P.seg.size() * 4, cudaMemcpyHostToDevice, st) != cudaSuccess)
    return NSA_ERR_CUDA;
  if (cudaMemcpyAsync(ws + W.seq, P.seq.data(), P.seq.size() * 4, cudaMemcpyHostToDevice, st) != cudaSuccess)
    return NSA_ERR_CUDA;
  nsa::PackArgs pa{};
  pa.seg = reinterpret_cast<const int*>(ws + W.seg);
  pa.seq = reinterpret_cast<const int*>(ws + W.seq);
  pa.nseg = P.S;
  pa.nseq = P.B;
  pa.ntok = P.N;
  pa.hq = p->num_q_heads;
  pa.hkv = p->num_kv_heads;
  pa.d = D;
  pa.cmp_stride = p->cmp_stride;
  pa.sel_len = p->sel_block;
  pa.q = static_cast<const __nv_bfloat16*>(q);
  pa.k = static_cast<const __nv_bfloat16*>(k);
  pa.v = static_cast<const __nv_bfloat16*>(v);
  pa.qv = P.gather ? reinterpret_cast<__nv_bfloat16*>(ws + W.qv) : nullptr;
  pa.kv = P.gather ? reinterpret_cast<__nv_bfloat16*>(ws + W.kv) : nullptr;
  pa.vv = P.gather ? reinterpret_cast<__nv_bfloat16*>(ws + W.vv) : nullptr;
  pa.qt = P.nt > 0 ? reinterpret_cast<__nv_bfloat16*>(ws + W.qt) : nullptr;
  pa.vinfo = reinterpret_cast<int4*>(ws + W.vinfo);
  pa.tinfo = reinterpret_cast<int2*>(ws + W.tinfo);
  pa.row_tok = reinterpret_cast<int*>(ws + W.row_tok);
  pa.blk_tok = reinterpret_cast<int*>(ws + W.blk_tok);
  if (P.N > 0) {
    nsa::pack_rows_kernel<<<static_cast<unsigned>((P.N + 7) / 8), 256, 0, st>>>(pa);
    if ((rc = launch_status("pack_rows", st, false)) != NSA_OK) return rc;
  }
  if (P.nv > 0) {
    nsa::pack_blocks_kernel<<<P.B, 256, 0, st>>>(pa);
    if ((rc = launch_status("pack_blocks", st, false)) != NSA_OK) return rc;
  }
  StageGeo geo{};
  geo.q = P.gather ? static_cast<const void*>(pa.qv) : q;
  geo.k = P.gather ? static_cast<const void*>(pa.kv) : k;
  geo.v = P.gather ? static_cast<const void*>(pa.vv) : v;
  geo.rows = P.gather ? P.nv : static_cast<int>(P.N);
  geo.nv = P.nv;
  geo.vinfo = pa.vinfo;
  geo.row_tok = pa.row_tok;
  geo.blk_tok = pa.blk_tok;
  geo.nsel_max = P.nsel_max;
  geo.qt = pa.qt;
  geo.qt_rows = P.nt;
  geo.t_begin = 0;
  geo.t_end = P.nt;
  geo.tinfo = pa.tinfo;
  geo.kd = k;
  geo.vd = v;
  geo.kd_rows = static_cast<int>(P.N);
  geo.gates = gates;
  geo.out = out;
  if (P.nv > 0 && (rc = video_stages<D>(p, geo, W.L, out_sel_idx, ws + W.video, st, nullptr, nullptr)) != NSA_OK)
    return rc;
  return text_stage<D>(p, geo, st);
}

int packed_entry(const void* q, const void* k, const void* v, const float* gates, const int32_t* cu, int batch,
                 const int32_t* seg_lens, const uint8_t* seg_video, int nseg, const nsa_params_t* params, void* out,
                 int32_t* out_sel_idx, void* workspace, size_t workspace_bytes, void* stream) {
  PackPlan P;
  int rc = build_plan(params, cu, batch, seg_lens, seg_video, nseg, P);
  if (rc != NSA_OK) return rc;
  if (!q || !k || !v || !out || !workspace || (!gates && P.nv > 0)) return NSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || (gates && !aligned16(gates)) ||
      (out_sel_idx && !aligned16(out_sel_idx)) || (reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0)
    return NSA_ERR_INVALID_ARG;
  const PackLayout W = pack_layout(params, P);
  if (workspace_bytes < W.total) return NSA_ERR_WORKSPACE_TOO_SMALL;
  if ((rc = check_device()) != NSA_OK) return rc;
  auto* ws = static_cast<uint8_t*>(workspace);
  auto st = static_cast<cudaStream_t>(stream);
  stage_begin(st);
  if (params->head_dim == 64) return packed_impl<64>(params, P, W, q, k, v, gates, out, out_sel_idx, ws, st);
  return packed_impl<128>(params, P, W, q, k, v, gates, out, out_sel_idx, ws, st);
}

// The varlen layout (video prefix, then text, per sequence) as a segment list.
void varlen_segments(const int32_t* cu, const int32_t* nv, int batch, std::vector<int32_t>& lens,
                     std::vector<uint8_t>& vid) {
  for (int b = 0; b < batch; ++b) {
    const int len = cu[b + 1] - cu[b];
    if (nv[b] > 0) {
      lens.push_back(nv[b]);
      vid.push_back(1);
    }
    if (len > nv[b]) {
      lens.push_back(len - nv[b]);
      vid.push_back(0);
    }
  }
}

}  // namespace

extern "C" {

const char* nsa_version(void) { return "nsa-b200 0.1.0 sm_100a"; }

const char* nsa_error_string(int status) {
  switch (status) {
    case NSA_OK:
      return "ok";
    case NSA_ERR_INVALID_ARG:
      return "invalid argument (null pointer, bad shape, misalignment or bad constant)";
    case NSA_ERR_UNSUPPORTED:
      return "unsupported configuration or device (needs sm_100, head_dim 64/128, l=32, s=16, l'=64, 3<=top_n<=64)";
    case NSA_ERR_WORKSPACE_TOO_SMALL:
      return "workspace smaller than nsa_workspace_size()";
    case NSA_ERR_CUDA:
      return "a CUDA runtime call or kernel launch failed";
    case NSA_ERR_NOALLOC_TOO_LARGE:
      return "the decode needs more scratch than nsa_decode_noalloc's fixed array (NSA_NOALLOC_SCRATCH_BYTES)";
    default:
      return "unknown status";
  }
}

size_t nsa_workspace_size(const nsa_params_t* params, int is_decode) {
  if (check_common(params) != NSA_OK) return 0;
  if (is_decode) {
    if (params->batch < 1) return 0;
    return decode_layout(params).total;
  }
  if (params->n_video < 0 || params->n_video > params->n_tokens) return 0;
  return prefill_layout(params).total;
}

int nsa_prefill_workspace_layout(const nsa_params_t* params, nsa_prefill_layout_t* layout) {
  if (layout == nullptr || check_common(params) != NSA_OK || params->n_video < 0 ||
      params->n_video > params->n_tokens)
    return NSA_ERR_INVALID_ARG;
  const PrefillLayout L = prefill_layout(params);
  layout->kc = L.kc;
  layout->vc = L.vc;
  layout->o_cmp = L.o_cmp;
  layout->lse = L.lse;
  layout->scores = L.scores;
  layout->sel_idx = L.sel_idx;
  layout->o_win = L.o_win;
  layout->total = L.total;
  layout->n_cmp = L.ncmp;
  layout->n_sel = L.nsel;
  layout->score_stride = L.score_stride;
  layout->o_sel = L.o_sel;
  layout->lse_sel = L.lse_sel;
  layout->lse_win = L.lse_win;
  return NSA_OK;
}

}  // extern "C"

namespace {
int prefill_entry(const void* q, const void* k, const void* v, const float* gates, const float* phi_k,
                  const float* phi_v, const nsa_params_t* params, void* out, int32_t* out_sel_idx, void* workspace,
                  size_t workspace_bytes, void* stream) {
  int rc = check_common(params);
  if (rc != NSA_OK) return rc;
  if (params->n_video < 0 || params->n_video > params->n_tokens) return NSA_ERR_INVALID_ARG;
  if (!q || !k || !v || !out || !workspace || (!gates && params->n_video > 0)) return NSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || (gates && !aligned16(gates)) ||
      (out_sel_idx && !aligned16(out_sel_idx)) || (reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0)
    return NSA_ERR_INVALID_ARG;
  if (nsel_of(params->n_video, params->sel_block) > 8192) return NSA_ERR_UNSUPPORTED;
  if (workspace_bytes < prefill_layout(params).total) return NSA_ERR_WORKSPACE_TOO_SMALL;
  if ((rc = check_device()) != NSA_OK) return rc;
  auto* ws = static_cast<uint8_t*>(workspace);
  auto st = static_cast<cudaStream_t>(stream);
  stage_begin(st);
  if (params->head_dim == 64) return prefill_impl<64>(params, q, k, v, gates, out, out_sel_idx, ws, st, phi_k, phi_v);
  return prefill_impl<128>(params, q, k, v, gates, out, out_sel_idx, ws, st, phi_k, phi_v);
}
}  // namespace

extern "C" {

int nsa_prefill(const void* q, const void* k, const void* v, const float* gates, const nsa_params_t* params,
                void* out, int32_t* out_sel_idx, void* workspace, size_t workspace_bytes, void* stream) {
  return prefill_entry(q, k, v, gates, nullptr, nullptr, params, out, out_sel_idx, workspace, workspace_bytes,
                       stream);
}

int nsa_prefill_phi(const void* q, const void* k, const void* v, const float* gates, const float* phi_k,
                    const float* phi_v, const nsa_params_t* params, void* out, int32_t* out_sel_idx, void* workspace,
                    size_t workspace_bytes, void* stream) {
  if (!phi_k || !phi_v || !aligned4(phi_k) || !aligned4(phi_v)) return NSA_ERR_INVALID_ARG;
  return prefill_entry(q, k, v, gates, phi_k, phi_v, params, out, out_sel_idx, workspace, workspace_bytes, stream);
}

size_t nsa_prefill_packed_workspace_size(const nsa_params_t* params, const int32_t* cu_seqlens, int batch,
                                         const int32_t* seg_lens, const uint8_t* seg_video, int nseg) {
  PackPlan P;
  if (build_plan(params, cu_seqlens, batch, seg_lens, seg_video, nseg, P) != NSA_OK) return 0;
  return pack_layout(params, P).total;
}

int nsa_prefill_packed(const void* q, const void* k, const void* v, const float* gates, const int32_t* cu_seqlens,
                       int batch, const int32_t* seg_lens, const uint8_t* seg_video, int nseg,
                       const nsa_params_t* params, void* out, int32_t* out_sel_idx, void* workspace,
                       size_t workspace_bytes, void* stream) {
  return packed_entry(q, k, v, gates, cu_seqlens, batch, seg_lens, seg_video, nseg, params, out, out_sel_idx,
                      workspace, workspace_bytes, stream);
}

}  // extern "C"

namespace {
// The varlen call's host arrays as a segment list, after checking them.
int varlen_to_segments(const nsa_params_t* params, const int32_t* cu, const int32_t* nv, int batch,
                       std::vector<int32_t>& lens, std::vector<uint8_t>& vid) {
  if (params == nullptr || !cu || !nv || batch < 1 || cu[0] != 0 || cu[batch] != params->n_tokens)
    return NSA_ERR_INVALID_ARG;
  for (int b = 0; b < batch; ++b) {
    const int len = cu[b + 1] - cu[b];
    if (len < 0 || nv[b] < 0 || nv[b] > len) return NSA_ERR_INVALID_ARG;
  }
  varlen_segments(cu, nv, batch, lens, vid);
  return NSA_OK;
}
}  // namespace

extern "C" {

size_t nsa_prefill_varlen_workspace_size(const nsa_params_t* params, const int32_t* cu_seqlens,
                                         const int32_t* n_video, int batch) {
  std::vector<int32_t> lens;
  std::vector<uint8_t> vid;
  if (varlen_to_segments(params, cu_seqlens, n_video, batch, lens, vid) != NSA_OK) return 0;
  return nsa_prefill_packed_workspace_size(params, cu_seqlens, batch, lens.data(), vid.data(),
                                           static_cast<int>(lens.size()));
}

int nsa_prefill_varlen(const void* q, const void* k, const void* v, const float* gates, const int32_t* cu_seqlens,
                       const int32_t* n_video, int batch, const nsa_params_t* params, void* out,
                       int32_t* out_sel_idx, void* workspace, size_t workspace_bytes, void* stream) {
  std::vector<int32_t> lens;
  std::vector<uint8_t> vid;
  const int rc = varlen_to_segments(params, cu_seqlens, n_video, batch, lens, vid);
  if (rc != NSA_OK) return rc;
  return packed_entry(q, k, v, gates, cu_seqlens, batch, lens.data(), vid.data(), static_cast<int>(lens.size()),
                      params, out, out_sel_idx, workspace, workspace_bytes, stream);
}

int nsa_decode(const void* q, const void* kcache, const void* vcache, const void* kcmp, const void* vcmp,
               const int32_t* seq_lens, const float* gates, const nsa_params_t* params, void* out,
               int32_t* out_sel_idx, void* workspace, size_t workspace_bytes, void* stream) {
  int rc = check_common(params);
  if (rc != NSA_OK) return rc;
  if (params->batch < 1) return NSA_ERR_INVALID_ARG;
  if (params->window > kMaxWindowDecode) return NSA_ERR_UNSUPPORTED;
  if (!q || !kcache || !vcache || !kcmp || !vcmp || !seq_lens || !gates || !out || !workspace)
    return NSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(kcache) || !aligned16(vcache) || !aligned16(kcmp) || !aligned16(vcmp) ||
      !aligned16(out) || (out_sel_idx && !aligned16(out_sel_idx)) ||
      (reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0)
    return NSA_ERR_INVALID_ARG;
  if (nsel_of(params->n_tokens, params->sel_block) > 8192) return NSA_ERR_UNSUPPORTED;
  if (workspace_bytes < decode_layout(params).total) return NSA_ERR_WORKSPACE_TOO_SMALL;
  if ((rc = check_device()) != NSA_OK) return rc;
  auto* ws = static_cast<uint8_t*>(workspace);
  auto st = static_cast<cudaStream_t>(stream);
  stage_begin(st);
  if (params->head_dim == 64)
    return decode_impl<64>(params, q, kcache, vcache, kcmp, vcmp, seq_lens, gates, out, out_sel_idx, ws, st);
  return decode_impl<128>(params, q, kcache, vcache, kcmp, vcmp, seq_lens, gates, out, out_sel_idx, ws, st);
}

// ------------------------------------------------------------------ decode with no caller scratch
// nsa_decode_noalloc keeps its scratch in this fixed device array instead of a caller
// workspace. Every GPU that loads the library holds the array until the process exits.
// Host code must not pass the symbol itself to a kernel: on the host it is only a
// stand-in, so the device address is looked up with cudaGetSymbolAddress, once per
// device, with that device current. The cached address is valid for as long as the
// device's primary context lives; a reset of that context (cudaDeviceReset) moves the array,
// and the header forbids calls after one.
static __device__ __align__(256) unsigned char g_noalloc_scratch[NSA_NOALLOC_SCRATCH_BYTES];

static int noalloc_scratch_address(void** out) {
  static std::mutex mu;
  static void* addr[64] = {};
  std::lock_guard<std::mutex> lock(mu);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return NSA_ERR_CUDA;
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return NSA_ERR_CUDA;
    addr[dev] = p;
  }
  *out = addr[dev];
  return NSA_OK;
}

int nsa_decode_noalloc(const void* q, const void* kcache, const void* vcache, const void* kcmp, const void* vcmp,
                       const int32_t* seq_lens, const float* gates, const nsa_params_t* params, void* out,
                       int32_t* out_sel_idx, void* stream) {
  int rc = check_common(params);
  if (rc != NSA_OK) return rc;
  if (params->batch < 1) return NSA_ERR_INVALID_ARG;
  if (params->window > kMaxWindowDecode) return NSA_ERR_UNSUPPORTED;
  if (!q || !kcache || !vcache || !kcmp || !vcmp || !seq_lens || !gates || !out) return NSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(kcache) || !aligned16(vcache) || !aligned16(kcmp) || !aligned16(vcmp) ||
      !aligned16(out) || (out_sel_idx && !aligned16(out_sel_idx)))
    return NSA_ERR_INVALID_ARG;
  if (nsel_of(params->n_tokens, params->sel_block) > 8192) return NSA_ERR_UNSUPPORTED;
  if (decode_layout(params).total > NSA_NOALLOC_SCRATCH_BYTES) return NSA_ERR_NOALLOC_TOO_LARGE;
  if ((rc = check_device()) != NSA_OK) return rc;
  void* scratch = nullptr;
  if ((rc = noalloc_scratch_address(&scratch)) != NSA_OK) return rc;
  auto* ws = static_cast<uint8_t*>(scratch);
  auto st = static_cast<cudaStream_t>(stream);
  stage_begin(st);
  if (params->head_dim == 64)
    return decode_impl<64>(params, q, kcache, vcache, kcmp, vcmp, seq_lens, gates, out, out_sel_idx, ws, st);
  return decode_impl<128>(params, q, kcache, vcache, kcmp, vcmp, seq_lens, gates, out, out_sel_idx, ws, st);
}

int nsa_compress(const void* k, const void* v, const nsa_params_t* params, void* kcmp, void* vcmp, void* stream) {
  int rc = check_common(params);
  if (rc != NSA_OK) return rc;
  if (params->batch < 1 || !k || !v || !kcmp || !vcmp) return NSA_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(v) || !aligned16(kcmp) || !aligned16(vcmp)) return NSA_ERR_INVALID_ARG;
  if ((rc = check_device()) != NSA_OK) return rc;
  const int ncmp = ncmp_of(params->n_tokens, params->cmp_block, params->cmp_stride);
  return launch_pool(k, v, kcmp, vcmp, params->batch, params->n_tokens, params->num_kv_heads, params->head_dim, ncmp,
                     params->cmp_block, params->cmp_stride, static_cast<cudaStream_t>(stream));
}

int nsa_compress_weighted(const void* k, const void* v, const float* phi_k, const float* phi_v,
                          const nsa_params_t* params, void* kcmp, void* vcmp, void* stream) {
  int rc = check_common(params);
  if (rc != NSA_OK) return rc;
  if (params->batch < 1 || !k || !v || !kcmp || !vcmp || !phi_k || !phi_v) return NSA_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(v) || !aligned16(kcmp) || !aligned16(vcmp) || !aligned4(phi_k) ||
      !aligned4(phi_v))
    return NSA_ERR_INVALID_ARG;
  if ((rc = check_device()) != NSA_OK) return rc;
  const int ncmp = ncmp_of(params->n_tokens, params->cmp_block, params->cmp_stride);
  return launch_pool(k, v, kcmp, vcmp, params->batch, params->n_tokens, params->num_kv_heads, params->head_dim, ncmp,
                     params->cmp_block, params->cmp_stride, static_cast<cudaStream_t>(stream), phi_k, phi_v);
}

// ------------------------------------------------------------------ gate network
}  // extern "C"

namespace {

bool gate_weights_ok(const void* w1, const float* b1, const float* w2, const float* b2) {
  return w1 && b1 && w2 && b2 && aligned16(w1) && aligned4(b1) && aligned4(w2) && aligned4(b2);
}

template <int DIM>
int launch_gate_mlp(const void* x, const void* w1, const float* b1, const float* w2, const float* b2, int64_t rows,
                    float* gates, cudaStream_t st) {
  CUtensorMap xmap, wmap;
  const uint64_t pitch = static_cast<uint64_t>(DIM) * 2;
  if (!nsa::make_tmap_bf16_3d(&xmap, x, DIM, static_cast<uint64_t>(rows), 1, pitch, pitch * rows, 64, 128, 1) ||
      !nsa::make_tmap_bf16_3d(&wmap, w1, DIM, DIM / 2, 1, pitch, pitch * (DIM / 2), 64, DIM / 2, 1))
    return NSA_ERR_CUDA;
  const size_t smem = sizeof(nsa::GateSmem<DIM>) + 1024;
  auto kern = nsa::gate_mlp_kernel<DIM>;
  if (set_smem(kern, smem) != NSA_OK) return NSA_ERR_CUDA;
  const unsigned grid = static_cast<unsigned>((rows + 127) / 128);
  kern<<<grid, 128, smem, st>>>(xmap, wmap, b1, w2, b2, gates, static_cast<long long>(rows));
  return launch_status("gate_mlp", st, false);
}

// Token chunk of the averaged gate's first pass: about 1,184 CTAs (8 per SM of a 148-SM
// part) over the whole batch, at least 64 tokens each. Fixed by the shapes alone, so the
// workspace size does not depend on the device.
int gate_chunk(int batch, int seq_len) {
  const int per_seq = batch >= 1184 ? 1 : 1184 / batch;
  const int c = (seq_len + per_seq - 1) / per_seq;
  return c < 64 ? 64 : c;
}

bool pooled_args_ok(int batch, int seq_len, int heads, int dim, int repeat) {
  return batch >= 1 && seq_len >= 1 && heads >= 1 && repeat >= 1 && (dim == 64 || dim == 128) &&
         static_cast<long long>(heads) * dim <= (1LL << 20);
}

}  // namespace

extern "C" {

int nsa_gate_mlp(const void* x, const void* w1, const float* b1, const float* w2, const float* b2, int64_t rows,
                 int dim, float* gates, void* stream) {
  if (!x || !gates || rows < 0 || !gate_weights_ok(w1, b1, w2, b2)) return NSA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned4(gates)) return NSA_ERR_INVALID_ARG;
  if (dim != 64 && dim != 128) return NSA_ERR_UNSUPPORTED;
  if (rows > (1LL << 31) - 128) return NSA_ERR_UNSUPPORTED;  // TMA row coordinates are 32-bit
  if (rows == 0) return NSA_OK;
  int rc = check_device();
  if (rc != NSA_OK) return rc;
  auto st = static_cast<cudaStream_t>(stream);
  return dim == 64 ? launch_gate_mlp<64>(x, w1, b1, w2, b2, rows, gates, st)
                   : launch_gate_mlp<128>(x, w1, b1, w2, b2, rows, gates, st);
}

size_t nsa_gate_mlp_pooled_workspace_size(int batch, int seq_len, int heads, int dim) {
  if (!pooled_args_ok(batch, seq_len, heads, dim, 1)) return 0;
  const int chunk = gate_chunk(batch, seq_len);
  const size_t nchunk = static_cast<size_t>((seq_len + chunk - 1) / chunk);
  return align_up(nchunk * batch * heads * dim * sizeof(double));
}

int nsa_gate_mlp_pooled(const void* x, const void* w1, const float* b1, const float* w2, const float* b2, int batch,
                        int seq_len, int heads, int dim, int repeat, float* gates, void* workspace,
                        size_t workspace_bytes, void* stream) {
  if (!x || !gates || !workspace || !gate_weights_ok(w1, b1, w2, b2)) return NSA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned4(gates) || (reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0)
    return NSA_ERR_INVALID_ARG;
  if (!pooled_args_ok(batch, seq_len, heads, dim, repeat)) return dim == 64 || dim == 128 ? NSA_ERR_INVALID_ARG
                                                                                           : NSA_ERR_UNSUPPORTED;
  if (workspace_bytes < nsa_gate_mlp_pooled_workspace_size(batch, seq_len, heads, dim))
    return NSA_ERR_WORKSPACE_TOO_SMALL;
  int rc = check_device();
  if (rc != NSA_OK) return rc;
  auto st = static_cast<cudaStream_t>(stream);
  const int chunk = gate_chunk(batch, seq_len);
  const int nchunk = (seq_len + chunk - 1) / chunk;
  auto* part = static_cast<double*>(workspace);
  nsa::gate_mean_partial_kernel<<<dim3(nchunk, batch), 256, 0, st>>>(static_cast<const __nv_bfloat16*>(x), part,
                                                                      batch, seq_len, heads * dim, chunk);
  if ((rc = launch_status("gate_mean_partial", st, false)) != NSA_OK) return rc;
  const unsigned grid = static_cast<unsigned>(batch) * heads;
  const auto* w1b = static_cast<const __nv_bfloat16*>(w1);
  if (dim == 64)
    nsa::gate_pooled_kernel<64><<<grid, nsa::kPooledSplit * 64, 0, st>>>(part, w1b, b1, w2, b2, gates, batch,
                                                                          seq_len, heads, nchunk, repeat);
  else
    nsa::gate_pooled_kernel<128><<<grid, nsa::kPooledSplit * 128, 0, st>>>(part, w1b, b1, w2, b2, gates, batch,
                                                                            seq_len, heads, nchunk, repeat);
  return launch_status("gate_pooled", st, false);
}

// ------------------------------------------------------------------ backward
}  // extern "C"

namespace {

struct BwdLayout {
  size_t kc, vc, dkc, dvc, stats, cnt, ent_off, seg_off, list, row_of, total;
  size_t dq_part, part_scale;  // (kept statistics, d = 128) the selected branch's dq partials
  long long part_rows;
  int ncmp, nsel;
};

BwdLayout bwd_layout(const nsa_params_t* p) {
  BwdLayout L{};
  const size_t N = p->n_tokens, nv = p->n_video, hq = p->num_q_heads, hkv = p->num_kv_heads, d = p->head_dim;
  L.ncmp = ncmp_of(p->n_video, p->cmp_block, p->cmp_stride);
  L.nsel = nsel_of(p->n_video, p->sel_block);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + (bytes > 0 ? bytes : 1));
    return at;
  };
  const size_t nc = L.ncmp > 0 ? L.ncmp : 1;
  const size_t buckets = hkv * (L.nsel > 0 ? L.nsel : 1);
  const size_t entries = nv * hkv * p->top_n;
  L.kc = take(nc * hkv * d * 2);
  L.vc = take(nc * hkv * d * 2);
  L.dkc = take(nc * hkv * d * 4);
  L.dvc = take(nc * hkv * d * 4);
  L.stats = take(N * hq * 3 * 8);
  L.cnt = take(2 * buckets * 4);  // counters and scatter cursors, zeroed together
  L.ent_off = take((buckets + 1) * 4);
  L.seg_off = take((buckets + 1) * 4);
  L.list = take(entries * 4);
  L.row_of = take(entries * 4);
  if (p->keep_branch_stats && d == 128 && nv > 0) {
    const size_t G = hq / hkv;  // 128-row tiles of 128 / G tokens, at most one partial tile per bucket
    L.part_rows = static_cast<long long>((entries + (128 / G) - 1) / (128 / G) + buckets) * 128;
    L.dq_part = take(static_cast<size_t>(L.part_rows) * d * 2);
    L.part_scale = take(static_cast<size_t>(L.part_rows) * 8);
  }
  L.total = off;
  return L;
}

template <int D, int BR>
int launch_bwd_key(const nsa::BwdArgs& a, long long n_items, cudaStream_t st) {
  if (n_items <= 0) return NSA_OK;
  const size_t smem = nsa::kBwdWarps * sizeof(nsa::BwdKeySmem<D>);
  auto kern = nsa::bwd_key_kernel<D, BR>;
  if (set_smem(kern, smem) != NSA_OK) return NSA_ERR_CUDA;
  const long long grid = (n_items + nsa::kBwdWarps - 1) / nsa::kBwdWarps;
  if (grid > 0x7fffffffLL) return NSA_ERR_UNSUPPORTED;
  kern<<<static_cast<unsigned>(grid), 32 * nsa::kBwdWarps, smem, st>>>(a, n_items);
  return launch_status(BR == nsa::kBwdCmp ? "bwd_key_cmp" : BR == nsa::kBwdSel ? "bwd_key_sel"
                                                          : BR == nsa::kBwdWin ? "bwd_key_win" : "bwd_key_dense",
                       st);
}

// The tcgen05 key pass of one branch: keys from (kk, vk) with `key_rows` rows in their tensor
// maps; `span` tokens of rows bound the segments per key tile.
template <int D, int BR>
int launch_bwd_key_tc(const nsa::BwdArgs& a, const void* q, const void* d_out, const void* kk, const void* vk,
                      int key_rows, int span, cudaStream_t st) {
  const int G = a.G, hq = a.hq, hkv = a.hkv, N = a.N;
  const int nkeys = BR == nsa::kBwdCmp ? a.ncmp : (BR == nsa::kBwdWin ? a.nv : a.N);
  if (nkeys <= 0) return NSA_OK;
  CUtensorMap qmap, dmap, kmap, vmap;
  const int Tb = nsa::kBtRows / G;
  const uint64_t qs1 = static_cast<uint64_t>(D) * 2, qs2 = static_cast<uint64_t>(hq) * D * 2;
  const uint64_t ks1 = static_cast<uint64_t>(D) * 2, ks2 = static_cast<uint64_t>(hkv) * D * 2;
  if (!nsa::make_tmap_bf16_3d(&qmap, q, D, hq, N, qs1, qs2, 64, G, Tb) ||
      !nsa::make_tmap_bf16_3d(&dmap, d_out, D, hq, N, qs1, qs2, 64, G, Tb) ||
      !nsa::make_tmap_bf16_3d(&kmap, kk, D, hkv, key_rows, ks1, ks2, 64, 1, nsa::kBtKeys) ||
      !nsa::make_tmap_bf16_3d(&vmap, vk, D, hkv, key_rows, ks1, ks2, 64, 1, nsa::kBtKeys))
    return NSA_ERR_CUDA;
  const int nseg = (span + nsa::kBtSegTokens - 1) / nsa::kBtSegTokens;
  const long long items = static_cast<long long>((nkeys + nsa::kBtKeys - 1) / nsa::kBtKeys) * hkv * nseg;
  if (items > 0x7fffffffLL) return NSA_ERR_UNSUPPORTED;
  const size_t smem = sizeof(nsa::BtSmem<D>) + 1024;
  auto kern = nsa::bwd_key_tc_kernel<D, BR>;
  if (set_smem(kern, smem) != NSA_OK) return NSA_ERR_CUDA;
  kern<<<static_cast<unsigned>(items), nsa::kBtThreads, smem, st>>>(qmap, dmap, kmap, vmap, a, nseg);
  return launch_status(BR == nsa::kBwdCmp ? "bwd_key_cmp" : BR == nsa::kBwdWin ? "bwd_key_win" : "bwd_key_dense", st);
}

// The selected blocks' key pass on tcgen05 (d = 128): persistent, one CTA per SM over the bucket
// tiles, whose count the bucket scan left on the device; kDq also writes the selected branch's
// dq partials.
template <bool kDq>
int launch_bwd_sel_key_tc(const nsa::BwdArgs& a, const void* k, const void* v, cudaStream_t st) {
  constexpr int D = 128;
  CUtensorMap kmap, vmap;
  const uint64_t ks1 = static_cast<uint64_t>(D) * 2, ks2 = static_cast<uint64_t>(a.hkv) * D * 2;
  if (!nsa::make_tmap_bf16_3d(&kmap, k, D, a.hkv, a.N, ks1, ks2, 64, 1, 64) ||
      !nsa::make_tmap_bf16_3d(&vmap, v, D, a.hkv, a.N, ks1, ks2, 64, 1, 64))
    return NSA_ERR_CUDA;
  const size_t smem = sizeof(nsa::BsSmem<D>) + 1024;
  auto kern = nsa::bwd_sel_key_tc_kernel<D, kDq>;
  if (set_smem(kern, smem) != NSA_OK) return NSA_ERR_CUDA;
  const int nsm = sm_count();
  if (nsm <= 0) return NSA_ERR_CUDA;
  kern<<<static_cast<unsigned>(nsm), nsa::kBsThreads, smem, st>>>(kmap, vmap, a);
  return launch_status("bwd_key_sel", st);
}

// The video rows' dq on tcgen05 from branches with contiguous keys and kept statistics: the
// compressed branch (kFull = false: also its statistics and gate gradient), or the compressed
// branch and the window (kFull = true: every branch's statistics are in a.stats already).
template <int D, bool kFull>
int launch_bwd_row_tc(const nsa::BwdArgs& a, const void* q, const void* d_out, cudaStream_t st) {
  const int G = a.G, hq = a.hq, hkv = a.hkv;
  if (G > 128) return NSA_ERR_UNSUPPORTED;
  const int T = 128 / G;
  CUtensorMap qmap, dmap, kcmap, vcmap, kmap, vmap;
  const uint64_t qs1 = static_cast<uint64_t>(D) * 2, qs2 = static_cast<uint64_t>(hq) * D * 2;
  const uint64_t ks1 = static_cast<uint64_t>(D) * 2, ks2 = static_cast<uint64_t>(hkv) * D * 2;
  const int crows = a.ncmp > 0 ? a.ncmp : 1;  // the workspace holds at least one compressed row
  if (!nsa::make_tmap_bf16_3d(&qmap, q, D, hq, a.N, qs1, qs2, 64, G, T) ||
      !nsa::make_tmap_bf16_3d(&dmap, d_out, D, hq, a.N, qs1, qs2, 64, G, T) ||
      !nsa::make_tmap_bf16_3d(&kcmap, a.kc, D, hkv, crows, ks1, ks2, 64, 1, 128) ||
      !nsa::make_tmap_bf16_3d(&vcmap, a.vc, D, hkv, crows, ks1, ks2, 64, 1, 128) ||
      !nsa::make_tmap_bf16_3d(&kmap, a.k, D, hkv, a.N, ks1, ks2, 64, 1, 128) ||
      !nsa::make_tmap_bf16_3d(&vmap, a.v, D, hkv, a.N, ks1, ks2, 64, 1, 128))
    return NSA_ERR_CUDA;
  const long long items = static_cast<long long>((a.nv + T - 1) / T) * hkv;
  if (items > 0x7fffffffLL) return NSA_ERR_UNSUPPORTED;
  const size_t smem = sizeof(nsa::BrSmem<D>) + 1024;
  auto kern = nsa::bwd_row_tc_kernel<D, kFull>;
  if (set_smem(kern, smem) != NSA_OK) return NSA_ERR_CUDA;
  kern<<<static_cast<unsigned>(items), nsa::kBrThreads, smem, st>>>(qmap, dmap, kcmap, vcmap, kmap, vmap, a);
  return launch_status(kFull ? "bwd_row_tc" : "bwd_row_cmp", st);
}

template <int D>
int backward_impl(const nsa_params_t* p, const void* q, const void* k, const void* v, const float* gates,
                  const void* d_out, const int32_t* sel_idx, const uint8_t* fwd_ws, const float* phi_k,
                  const float* phi_v, float* dq, float* dk, float* dv, float* dgates, uint8_t* ws, cudaStream_t st) {
  const BwdLayout L = bwd_layout(p);
  const int N = p->n_tokens, nv = p->n_video, hq = p->num_q_heads, hkv = p->num_kv_heads;
  const int G = hq / hkv;
  const float scale = p->softmax_scale > 0.f ? p->softmax_scale : 1.0f / std::sqrt(static_cast<float>(D));
  int rc;
  nsa::BwdArgs a{};
  a.N = N;
  a.nv = nv;
  a.hq = hq;
  a.hkv = hkv;
  a.G = G;
  a.ncmp = L.ncmp;
  a.nsel = L.nsel;
  a.top_n = p->top_n;
  a.cmp_len = p->cmp_block;
  a.cmp_stride = p->cmp_stride;
  a.sel_len = p->sel_block;
  a.window = p->window;
  a.scale = scale;
  a.sl2 = scale * 1.4426950408889634f;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.k = static_cast<const __nv_bfloat16*>(k);
  a.v = static_cast<const __nv_bfloat16*>(v);
  a.kc = reinterpret_cast<const __nv_bfloat16*>(ws + L.kc);
  a.vc = reinterpret_cast<const __nv_bfloat16*>(ws + L.vc);
  a.dout = static_cast<const __nv_bfloat16*>(d_out);
  a.gates = gates;
  a.sel_idx = sel_idx;
  a.stats = reinterpret_cast<float2*>(ws + L.stats);
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.dkc = reinterpret_cast<float*>(ws + L.dkc);
  a.dvc = reinterpret_cast<float*>(ws + L.dvc);
  a.dgates = dgates;
  a.ent_off = reinterpret_cast<const int*>(ws + L.ent_off);
  a.seg_off = reinterpret_cast<const int*>(ws + L.seg_off);
  a.list = reinterpret_cast<const int*>(ws + L.list);
  // full: the forward kept every branch's statistics, and every video row runs on the tensor
  // cores (d = 128)
  bool full = false;
  if (fwd_ws != nullptr && nv > 0) {
    const PrefillLayout F = prefill_layout(p);
    a.fwd_lse = reinterpret_cast<const float*>(fwd_ws + F.lse);
    a.fwd_ocmp = reinterpret_cast<const __half*>(fwd_ws + F.o_cmp);
    if (D == 128 && p->keep_branch_stats && F.o_sel != 0) {
      full = true;
      a.fwd_osel = reinterpret_cast<const __half*>(fwd_ws + F.o_sel);
      a.fwd_lse_sel = reinterpret_cast<const float*>(fwd_ws + F.lse_sel);
      a.fwd_owin = reinterpret_cast<const __half*>(fwd_ws + F.o_win);
      a.fwd_lse_win = reinterpret_cast<const float*>(fwd_ws + F.lse_win);
      a.video_rows_done = 1;
      a.row_of = reinterpret_cast<const int*>(ws + L.row_of);
      a.dq_part = reinterpret_cast<__half*>(ws + L.dq_part);
      a.part_scale = reinterpret_cast<float2*>(ws + L.part_scale);
    }
  }
  const size_t kv_bytes = static_cast<size_t>(N) * hkv * D * 4;
  if (cudaMemsetAsync(dk, 0, kv_bytes, st) != cudaSuccess || cudaMemsetAsync(dv, 0, kv_bytes, st) != cudaSuccess)
    return NSA_ERR_CUDA;
  if (L.ncmp > 0) {
    const size_t cb = static_cast<size_t>(L.ncmp) * hkv * D * 4;
    if (cudaMemsetAsync(ws + L.dkc, 0, cb, st) != cudaSuccess || cudaMemsetAsync(ws + L.dvc, 0, cb, st) != cudaSuccess)
      return NSA_ERR_CUDA;
    // the compressed keys and values the forward attended
    if ((rc = launch_pool(k, v, ws + L.kc, ws + L.vc, 1, nv, hkv, D, L.ncmp, p->cmp_block, p->cmp_stride, st, phi_k,
                          phi_v)) != NSA_OK)
      return rc;
  }
  // row pass: dq, the gates' gradient and the per-branch statistics. full: the statistics of
  // the video rows come from the forward's, the warp row pass takes the text rows only, and
  // the video rows' dq is written by the tensor-core kernels below. Else, with the forward's
  // compressed-branch statistics, that branch's share runs first on tcgen05.
  if (full) {
    const long long rows = static_cast<long long>(nv) * hq;
    nsa::bwd_stats_kernel<D><<<static_cast<unsigned>((rows + 7) / 8), 256, 0, st>>>(a);
    if ((rc = launch_status("bwd_stats", st)) != NSA_OK) return rc;
  } else if (a.fwd_lse != nullptr && L.ncmp > 0) {
    if ((rc = launch_bwd_row_tc<D, false>(a, q, d_out, st)) != NSA_OK) return rc;
    a.cmp_rows_done = 1;
  }
  if (!full || N > nv) {
    const size_t smem = nsa::kBwdWarps * sizeof(nsa::BwdRowSmem<D>);
    auto kern = nsa::bwd_row_kernel<D>;
    if (set_smem(kern, smem) != NSA_OK) return NSA_ERR_CUDA;
    const int tpw = G <= 8 ? 2 : 1;  // tokens per warp, as the kernel pairs them
    const long long items = static_cast<long long>((nv + tpw - 1) / tpw + (N - nv + tpw - 1) / tpw) * hkv;
    kern<<<static_cast<unsigned>((items + nsa::kBwdWarps - 1) / nsa::kBwdWarps), 32 * nsa::kBwdWarps, smem, st>>>(a);
    if ((rc = launch_status("bwd_row", st)) != NSA_OK) return rc;
  }
  if (nv > 0) {
    // buckets of the selected branch: which tokens chose each (group, block)
    const int m = hkv * L.nsel;
    nsa::SelInvArgs sa{};
    sa.nv = nv;
    sa.hq = hq;
    sa.hkv = hkv;
    sa.G = G;
    sa.Gp = G;
    // d = 128: buckets cut into tcgen05 tiles of 128 rows (128 / G tokens); else warp segments
    sa.TT = D == 128 ? 128 / G : nsa::kBwdSegSel;
    sa.nsel = L.nsel;
    sa.top_n = p->top_n;
    sa.sel_len = p->sel_block;
    sa.sel_idx = sel_idx;
    sa.cnt = reinterpret_cast<int*>(ws + L.cnt);
    sa.cursor = sa.cnt + m;
    sa.ent_off = reinterpret_cast<int*>(ws + L.ent_off);
    sa.tile_off = reinterpret_cast<int*>(ws + L.seg_off);
    sa.list = reinterpret_cast<int*>(ws + L.list);
    sa.row_of = reinterpret_cast<int*>(ws + L.row_of);
    if (cudaMemsetAsync(sa.cnt, 0, 2 * static_cast<size_t>(m) * 4, st) != cudaSuccess) return NSA_ERR_CUDA;
    const long long entries = static_cast<long long>(nv) * hkv * p->top_n;
    const long long eb = (entries + 255) / 256;
    const unsigned ebl = static_cast<unsigned>(eb < 148 * 16 ? (eb > 0 ? eb : 1) : 148 * 16);
    nsa::sel_count_kernel<<<ebl, 256, 0, st>>>(sa);
    if ((rc = launch_status("bwd_sel_count", st, false)) != NSA_OK) return rc;
    nsa::sel_scan_kernel<<<1, 1024, 0, st>>>(sa);
    if ((rc = launch_status("bwd_sel_scan", st, false)) != NSA_OK) return rc;
    nsa::sel_scatter_kernel<<<ebl, 256, 0, st>>>(sa);
    if ((rc = launch_status("bwd_sel_scatter", st)) != NSA_OK) return rc;
    // key pass, one launch per branch: the compressed keys and the window on tcgen05 (128 keys
    // x 64-row chunks), the selected blocks' on warp tiles over their buckets
    if (L.ncmp > 0 &&
        (rc = launch_bwd_key_tc<D, nsa::kBwdCmp>(a, q, d_out, ws + L.kc, ws + L.vc, L.ncmp, nv, st)) != NSA_OK)
      return rc;
    if constexpr (D == 128) {
      if ((rc = full ? launch_bwd_sel_key_tc<true>(a, k, v, st) : launch_bwd_sel_key_tc<false>(a, k, v, st)) !=
          NSA_OK)
        return rc;
      if (full) {
        // the video rows' dq: compressed and window tiles, then the selected partials
        if ((rc = launch_bwd_row_tc<D, true>(a, q, d_out, st)) != NSA_OK) return rc;
        const long long rows = static_cast<long long>(nv) * hq;
        nsa::bwd_sel_dq_merge_kernel<D><<<static_cast<unsigned>((rows + 7) / 8), 256, 0, st>>>(a);
        if ((rc = launch_status("bwd_sel_dq_merge", st)) != NSA_OK) return rc;
      }
    } else {
      const long long segs = entries / nsa::kBwdSegSel + m + 1;  // >= sum over buckets of ceil(count / segment)
      if ((rc = launch_bwd_key<D, nsa::kBwdSel>(a, segs * (p->sel_block / nsa::kBwdChunk), st)) != NSA_OK) return rc;
    }
    // a window key tile's rows span 128 + w - 1 tokens
    if ((rc = launch_bwd_key_tc<D, nsa::kBwdWin>(a, q, d_out, k, v, N, nsa::kBtKeys + p->window, st)) != NSA_OK)
      return rc;
  }
  if (N > nv && (rc = launch_bwd_key_tc<D, nsa::kBwdDense>(a, q, d_out, k, v, N, N - nv, st)) != NSA_OK) return rc;
  if (L.ncmp > 0) {
    const long long total = static_cast<long long>(nv) * hkv * D;
    nsa::pool_bwd_kernel<<<static_cast<unsigned>((total + 255) / 256), 256, 0, st>>>(
        a.dkc, a.dvc, phi_k, phi_v, dk, dv, nv, hkv, D, L.ncmp, p->cmp_block, p->cmp_stride);
    if ((rc = launch_status("pool_bwd", st)) != NSA_OK) return rc;
  }
  return NSA_OK;
}

}  // namespace

extern "C" {

size_t nsa_backward_workspace_size(const nsa_params_t* params) {
  if (check_common(params) != NSA_OK || params->n_video < 0 || params->n_video > params->n_tokens) return 0;
  return bwd_layout(params).total;
}

int nsa_backward(const void* q, const void* k, const void* v, const float* gates, const void* d_out,
                 const int32_t* sel_idx, const void* fwd_workspace, size_t fwd_workspace_bytes, const float* phi_k,
                 const float* phi_v, const nsa_params_t* params, float* dq, float* dk, float* dv, float* dgates,
                 void* workspace, size_t workspace_bytes, void* stream) {
  int rc = check_common(params);
  if (rc != NSA_OK) return rc;
  if (params->n_video < 0 || params->n_video > params->n_tokens) return NSA_ERR_INVALID_ARG;
  const bool video = params->n_video > 0;
  if (!q || !k || !v || !d_out || !dq || !dk || !dv || !dgates || !workspace || (video && (!gates || !sel_idx)))
    return NSA_ERR_INVALID_ARG;
  if ((phi_k == nullptr) != (phi_v == nullptr)) return NSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(d_out) || !aligned16(dq) || !aligned16(dk) ||
      !aligned16(dv) || !aligned4(dgates) || (gates && !aligned4(gates)) || (sel_idx && !aligned4(sel_idx)) ||
      (phi_k && (!aligned4(phi_k) || !aligned4(phi_v))) || (reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0 ||
      (reinterpret_cast<uintptr_t>(fwd_workspace) % kAlign) != 0)
    return NSA_ERR_INVALID_ARG;
  if (nsel_of(params->n_video, params->sel_block) > 8192) return NSA_ERR_UNSUPPORTED;
  if (workspace_bytes < bwd_layout(params).total) return NSA_ERR_WORKSPACE_TOO_SMALL;
  // the forward's workspace must hold the layout these params give it (with keep_branch_stats,
  // the kept statistics too): a workspace from a call with other params is refused, not read past
  if (fwd_workspace != nullptr && fwd_workspace_bytes < prefill_layout(params).total)
    return NSA_ERR_WORKSPACE_TOO_SMALL;
  if ((rc = check_device()) != NSA_OK) return rc;
  auto* ws = static_cast<uint8_t*>(workspace);
  auto st = static_cast<cudaStream_t>(stream);
  // stage events registered by nsa_profile_stages belong to the forward calls
  const int saved_count = g_stage_count;
  g_stage_count = 0;
  rc = params->head_dim == 64
           ? backward_impl<64>(params, q, k, v, gates, d_out, sel_idx, static_cast<const uint8_t*>(fwd_workspace),
                               phi_k, phi_v, dq, dk, dv, dgates, ws, st)
           : backward_impl<128>(params, q, k, v, gates, d_out, sel_idx, static_cast<const uint8_t*>(fwd_workspace),
                                phi_k, phi_v, dq, dk, dv, dgates, ws, st);
  g_stage_count = saved_count;
  return rc;
}

int nsa_profile_stages(void* const* events, int count) {
  if (count < 0 || (count > 0 && events == nullptr)) return NSA_ERR_INVALID_ARG;
  g_stage_events = count > 0 ? events : nullptr;
  g_stage_count = count > 0 ? count : 0;
  g_stage_next = 0;
  return NSA_OK;
}

int nsa_selftest_wait_timeout(int64_t limit_cycles, void* stream) {
  if (limit_cycles < 1 || limit_cycles > nsa::kWaitCycles) return NSA_ERR_INVALID_ARG;
  int rc = check_device();
  if (rc != NSA_OK) return rc;
  nsa::bounded_wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_cycles);
  return launch_status("bounded_wait_selftest", static_cast<cudaStream_t>(stream), false);
}

int nsa_get_device_error(uint32_t* word, int clear) {
  if (word == nullptr) return NSA_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return NSA_ERR_CUDA;
  unsigned int w = 0;
  if (cudaMemcpyFromSymbol(&w, nsa::g_device_error, sizeof(w)) != cudaSuccess) return NSA_ERR_CUDA;
  *word = w;
  if (clear) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(nsa::g_device_error, &zero, sizeof(zero)) != cudaSuccess) return NSA_ERR_CUDA;
  }
  return NSA_OK;
}

}  // extern "C"
