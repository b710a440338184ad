/*
 * nsa.h -- C ABI of the B200 (sm_100a) Native Sparse Attention forward pass.
 *
 * The operation is the attention layer of VideoNSA: video tokens get Native Sparse
 * Attention, made of three branches -- a compressed branch over block summaries, a
 * selected branch over the most important token blocks, and a sliding-window branch --
 * whose outputs are mixed per token and head by gates; trailing text tokens get dense
 * causal attention. Sources: top168.com article on VideoNSA, section
 * "一、革命性的三重注意机制" (the three branches and their gated combination);
 * shd-paper.top page "VideoNSA: Native Sparse Attention Scales Video Understanding",
 * abstract (dense attention for text, NSA for video; scaling to 128K tokens); CSDN blog
 * "VideoNSA：重新定义视频理解的稀疏注意力机制", section 2.2 (CMP / SLC / SWA branches)
 * and section 3.1 (one gate per branch and head).
 *
 * The pages fix no constants. This library computes, for query token t and head h of
 * GQA group g = h / (Hq/Hkv), with scale = softmax_scale (<= 0: 1/sqrt(head_dim)):
 *   Kc[i] = bf16_rne(mean_{u<l} K[i*s+u])                   (compression, l = cmp_block, s = cmp_stride)
 *   o_cmp = softmax over compressed blocks i with i*s + l - 1 <= t  (0 if there are none)
 *   score[t,g,j] = sum_{h in g} sum_i P_cmp[t,h,i] * |tokens(i) & tokens(j)| / l
 *   selection: blocks 0, t/l' and t/l' - 1 always, then the best top_n - |forced| other
 *              blocks j <= t/l' by (score desc, index asc)   (l' = sel_block)
 *   o_sel = softmax over tokens tau <= t of the selected blocks
 *   o_win = softmax over tokens max(0, t-window+1) .. t
 *   out   = gates[t,h,0]*o_cmp + gates[t,h,1]*o_sel + gates[t,h,2]*o_win
 *   rows t >= n_video (text): out = dense causal softmax over tokens 0..t.
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers, 16-byte aligned, contiguous, token-major.
 *     bf16 tensors are IEEE bfloat16; gates are fp32.
 *   - The caller owns every buffer. The library allocates nothing per call; it keeps no
 *     state besides a device error word. Scratch memory is the caller's `workspace`,
 *     sized by nsa_workspace_size().
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL = legacy
 *     default stream). Host-side validation errors return before anything is enqueued.
 *   - Return value: NSA_OK (0) or one of the nsa_status codes below. No exception
 *     crosses the ABI. Faults inside kernels surface at the caller's next sync; a kernel
 *     whose internal wait timed out records it in the device error word
 *     (nsa_get_device_error) and returns early instead of hanging.
 *   - Supported on sm_100 (B200) only: head_dim in {64, 128}; Hq % Hkv == 0 with
 *     Hq/Hkv <= 16; cmp_block = 32, cmp_stride = 16, sel_block = 64;
 *     3 <= top_n <= 64; window >= 1.
 */
#ifndef NSA_H_
#define NSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum nsa_status {
  NSA_OK = 0,
  NSA_ERR_INVALID_ARG = 1,         /* null pointer, bad shape, misalignment, bad constant */
  NSA_ERR_UNSUPPORTED = 2,         /* valid but not implemented here (head_dim, block sizes, device) */
  NSA_ERR_WORKSPACE_TOO_SMALL = 3, /* workspace_bytes < nsa_workspace_size() */
  NSA_ERR_CUDA = 4,                /* a CUDA runtime call or launch failed */
  NSA_ERR_NOALLOC_TOO_LARGE = 5    /* nsa_decode_noalloc: the problem needs more than its fixed scratch */
};

enum nsa_out_dtype { NSA_OUT_BF16 = 0, NSA_OUT_F32 = 1 };

typedef struct {
  int32_t n_tokens;      /* prefill: N tokens; decode / compress: cache capacity Lmax */
  int32_t n_video;       /* prefill: N_v, the NSA-attended prefix (0 <= N_v <= N); rows >= N_v are text */
  int32_t num_q_heads;   /* Hq */
  int32_t num_kv_heads;  /* Hkv */
  int32_t head_dim;      /* d */
  int32_t cmp_block;     /* l  (compression block length) */
  int32_t cmp_stride;    /* s  (compression stride) */
  int32_t sel_block;     /* l' (selection block length) */
  int32_t top_n;         /* n  (selected blocks per token and group, forced blocks included) */
  int32_t window;        /* w  (sliding-window length, the query token included) */
  float softmax_scale;   /* <= 0 selects 1/sqrt(head_dim) */
  int32_t out_dtype;     /* enum nsa_out_dtype */
  int32_t batch;         /* decode / compress: number of sequences B (prefill: ignored) */
  int32_t keep_branch_stats; /* prefill (one sequence) and backward: 1 = the prefill also keeps the
                                selected branch's output and the selected and window branches'
                                log-sum-exp in its workspace (larger workspace, one more fp16
                                write of the selected rows), and nsa_backward, given that
                                workspace and the same params, reuses them; 0 = neither */
} nsa_params_t;

/*
 * Prefill: one sequence of N tokens.
 *   q     [N][Hq][d] bf16        k, v [N][Hkv][d] bf16       gates [N][Hq][3] fp32 (cmp, sel, win)
 *   out   [N][Hq][d] bf16 or fp32 (params->out_dtype)
 *   out_sel_idx  NULL, or [N_v][Hkv][top_n] int32: the selected block indices of every video
 *                row, ascending, padded with -1.
 *   workspace    device scratch of at least nsa_workspace_size(params, 0) bytes (256-byte aligned).
 * Rows t < N_v follow NSA; rows t >= N_v get dense causal attention (gates unused).
 * The call only enqueues kernels and device memsets on `stream` (no host copies, no
 * synchronisation), so it can be captured in a CUDA graph and replayed; nsa_decode,
 * nsa_compress and nsa_backward can be captured the same way.
 */
int nsa_prefill(const void* q, const void* k, const void* v, const float* gates, const nsa_params_t* params,
                void* out, int32_t* out_sel_idx, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Varlen prefill: B independent sequences packed back to back, the batch form a server
 * uses. Sequence lengths vary from clip to clip (CSDN blog on VideoNSA, vcloud.csdn.net,
 * section 5.2, item 3), and a hybrid sequence carries text rows after its video tokens
 * (shd-paper.top page "VideoNSA: Native Sparse Attention Scales Video Understanding",
 * abstract).
 *   cu_seqlens  HOST array [B+1]: sequence b owns packed tokens [cu_seqlens[b], cu_seqlens[b+1]);
 *               cu_seqlens[0] = 0, non-decreasing, cu_seqlens[B] = params->n_tokens.
 *   n_video     HOST array [B]: sequence b's NSA-attended prefix, 0 <= n_video[b] <= its
 *               length (params->n_video is ignored).
 *   q, k, v, gates, out: as nsa_prefill, over the params->n_tokens packed tokens.
 *   out_sel_idx NULL, or [sum of n_video][Hkv][top_n] int32: the video rows of every sequence,
 *               sequence after sequence.
 *   workspace   at least nsa_prefill_varlen_workspace_size(params, cu_seqlens, n_video, B) bytes.
 * Each sequence gets what nsa_prefill computes for it alone (the same selection, outputs equal
 * up to fp32 summation order); positions restart at 0 in every sequence. This is
 * nsa_prefill_packed with each sequence's video prefix and trailing text as its two
 * segments: every stage is launched once for the whole batch. Errors as nsa_prefill, plus
 * NSA_ERR_INVALID_ARG for malformed cu_seqlens / n_video; nothing is enqueued then.
 */
int nsa_prefill_varlen(const void* q, const void* k, const void* v, const float* gates, const int32_t* cu_seqlens,
                       const int32_t* n_video, int batch, const nsa_params_t* params, void* out,
                       int32_t* out_sel_idx, void* workspace, size_t workspace_bytes, void* stream);

/* Workspace bytes nsa_prefill_varlen needs; 0 if the arguments are invalid. */
size_t nsa_prefill_varlen_workspace_size(const nsa_params_t* params, const int32_t* cu_seqlens,
                                         const int32_t* n_video, int batch);

/*
 * Packed prefill with video and text segments in any order: B sequences back to back, each a
 * run of segments. Video tokens get NSA and text tokens dense attention (shd-paper.top page
 * "VideoNSA: Native Sparse Attention Scales Video Understanding", abstract); clip lengths vary
 * from request to request (CSDN blog on VideoNSA, vcloud.csdn.net, section 5.2, item 3). The
 * pages never put text between video segments; this library's reading, which reduces to the
 * trailing-text layout of nsa_prefill:
 *   - a video row gets NSA over its sequence's video tokens only, taken in order as one
 *     stream: compression and selection blocks, the window and causality count positions in
 *     that stream, exactly as for a sequence made of those video tokens alone;
 *   - a text row gets dense causal attention over every earlier token of its sequence, video
 *     and text, and itself (gates unused).
 * Arguments:
 *   cu_seqlens  HOST [B+1]: sequence b owns packed rows [cu_seqlens[b], cu_seqlens[b+1]);
 *               cu_seqlens[0] = 0, non-decreasing, cu_seqlens[B] = params->n_tokens.
 *   seg_lens    HOST [nseg]: segment lengths (> 0) in packed order; the segments tile every
 *               sequence exactly (an empty sequence has none).
 *   seg_video   HOST [nseg]: 1 for a video segment, 0 for a text segment.
 *   q, k, v, gates, out: as nsa_prefill over the params->n_tokens packed rows (params->n_video
 *               is ignored; gates may be NULL when there is no video row).
 *   out_sel_idx NULL, or [total video rows][Hkv][top_n] int32: every video row's selection,
 *               in packed order (sequence after sequence, segment after segment).
 *   workspace   at least nsa_prefill_packed_workspace_size(...) bytes, 256-byte aligned.
 * Every stage is launched once for the whole batch (tiles span sequences); the plan (two small
 * tables) is copied to the workspace with cudaMemcpyAsync from host memory first, from a host
 * buffer that lives only during the call: do not capture this call (or nsa_prefill_varlen) in a
 * CUDA graph. Errors as
 * nsa_prefill, plus NSA_ERR_INVALID_ARG for malformed sequence or segment arrays, and
 * NSA_ERR_UNSUPPORTED when a video stream has more than 8,192 selection blocks; nothing is
 * enqueued then.
 */
int nsa_prefill_packed(const void* q, const void* k, const void* v, const float* gates, const int32_t* cu_seqlens,
                       int batch, const int32_t* seg_lens, const uint8_t* seg_video, int nseg,
                       const nsa_params_t* params, void* out, int32_t* out_sel_idx, void* workspace,
                       size_t workspace_bytes, void* stream);

/* Workspace bytes nsa_prefill_packed needs; 0 if the arguments are invalid. */
size_t nsa_prefill_packed_workspace_size(const nsa_params_t* params, const int32_t* cu_seqlens, int batch,
                                         const int32_t* seg_lens, const uint8_t* seg_video, int nseg);

/*
 * Decode: one query token per sequence against a KV cache and its compressed cache.
 *   q       [B][Hq][d] bf16, the query at position seq_lens[b]-1 (its own K/V are in the cache)
 *   kcache, vcache [B][Lmax][Hkv][d] bf16 (Lmax = params->n_tokens)
 *   kcmp, vcmp     [B][Ncmp(Lmax)][Hkv][d] bf16, Ncmp(L) = L >= l ? (L-l)/s + 1 : 0, as written by
 *                  nsa_compress (used as given: block i of sequence b is read only if complete,
 *                  i*s + l <= seq_lens[b])
 *   seq_lens [B] int32, 1 <= seq_lens[b] <= Lmax       gates [B][Hq][3] fp32
 *   out     [B][Hq][d] bf16 or fp32                    out_sel_idx NULL or [B][Hkv][top_n] int32
 *   workspace at least nsa_workspace_size(params, 1) bytes.
 */
int nsa_decode(const void* q, const void* kcache, const void* vcache, const void* kcmp, const void* vcmp,
               const int32_t* seq_lens, const float* gates, const nsa_params_t* params, void* out,
               int32_t* out_sel_idx, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Decode that allocates nothing and takes no workspace. The pages describe no such
 * variant; it exists for callers that cannot call cudaMalloc or hand over scratch memory:
 * for example a plugin or C program whose device memory is owned and pre-partitioned by
 * a host framework that forbids allocation on its serving path, or a caller with a device
 * memory budget fixed at start-up. Same arguments, results and kernels as nsa_decode,
 * except that the scratch lives in one fixed device array of NSA_NOALLOC_SCRATCH_BYTES
 * (32 MiB) compiled into the library; every GPU that loads the library holds that array
 * until the process exits.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call before any
 *     stream capture on the device. The address is kept for the life of the process: do
 *     not call nsa_decode_noalloc on a device after cudaDeviceReset (or any other reset of
 *     its primary context) in the same process, since the array then moves.
 *   - A problem whose scratch (nsa_workspace_size(params, 1)) exceeds the array returns
 *     NSA_ERR_NOALLOC_TOO_LARGE before anything is enqueued; use nsa_decode for it.
 *   - All calls share the one array and it keeps the last call's contents; no kernel reads
 *     scratch it has not written in the same call, so nothing needs clearing. Calls whose
 *     execution overlaps on the GPU (other streams, other threads) race on the array:
 *     serialise them.
 * Calls no cudaMalloc, cudaFree or allocating library routine.
 */
#define NSA_NOALLOC_SCRATCH_BYTES (32u << 20)
int nsa_decode_noalloc(const void* q, const void* kcache, const void* vcache, const void* kcmp, const void* vcmp,
                       const int32_t* seq_lens, const float* gates, const nsa_params_t* params, void* out,
                       int32_t* out_sel_idx, void* stream);

/*
 * Compression only: kcmp[b][i] = bf16_rne(mean_{u<l} k[b][i*s+u]) for every complete block
 * i < Ncmp(Lmax), same for v. k, v [B][Lmax][Hkv][d]; kcmp, vcmp [B][Ncmp(Lmax)][Hkv][d].
 * B = params->batch (>= 1), Lmax = params->n_tokens. Builds the decode's compressed cache.
 */
int nsa_compress(const void* k, const void* v, const nsa_params_t* params, void* kcmp, void* vcmp, void* stream);

/*
 * Learnable compression. The pages steer the sparse pattern with learned parameters
 * (shd-paper.top page "VideoNSA: Native Sparse Attention Scales Video Understanding",
 * section "方法详解", key design (1)) without giving their form; this library's form is a
 * per-head weighting of the l positions of a block in place of the mean:
 *   kcmp[b][i][g] = bf16_rne( sum_{u<l} phi_k[g][u] * k[b][i*s+u][g] ), same for v with phi_v.
 * phi_k, phi_v: device [Hkv][l] fp32, 4-byte aligned; everything else as nsa_compress.
 * The fp64 sum of exact products is rounded once; phi = 1/l (l a power of two) gives
 * exactly nsa_compress's mean.
 */
int nsa_compress_weighted(const void* k, const void* v, const float* phi_k, const float* phi_v,
                          const nsa_params_t* params, void* kcmp, void* vcmp, void* stream);

/*
 * nsa_prefill with the learnable compression above building the compressed keys and
 * values of the video prefix (phi_k, phi_v: device [Hkv][l] fp32, both required). Same
 * arguments, workspace, results and errors as nsa_prefill otherwise.
 */
int nsa_prefill_phi(const void* q, const void* k, const void* v, const float* gates, const float* phi_k,
                    const float* phi_v, const nsa_params_t* params, void* out, int32_t* out_sel_idx, void* workspace,
                    size_t workspace_bytes, void* stream);

/*
 * Gate network: three softmax-normalised gates per head from a two-layer MLP, dim -> dim/2
 * with an exact (erf) GELU, then dim/2 -> 3 (CSDN blog "VideoNSA：重新定义视频理解的稀疏注意力
 * 机制", vcloud.csdn.net, section 3.1 "动态门控机制详解"). Per row r:
 *   gates[r] = softmax( W2 . GELU(W1 . x[r] + b1) + b2 )
 *   x      [rows][dim] bf16, 16-byte aligned; e.g. a prefill's q [N][Hq][d] seen as N*Hq rows
 *          of dim = d, which yields the [N][Hq][3] gates nsa_prefill takes.
 *   w1     [dim/2][dim] bf16 (linear-layer layout [out][in]), 16-byte aligned
 *   b1     [dim/2] fp32     w2 [3][dim/2] fp32     b2 [3] fp32      gates [rows][3] fp32
 * dim must be 64 or 128 (else NSA_ERR_UNSUPPORTED). The first layer runs on the tensor
 * cores in fp32 accumulation; rows = 0 enqueues nothing. All pointers are device memory
 * owned by the caller; errors (NSA_ERR_INVALID_ARG for null or misaligned pointers, rows
 * < 0) are returned before anything is enqueued.
 */
int nsa_gate_mlp(const void* x, const void* w1, const float* b1, const float* w2, const float* b2, int64_t rows,
                 int dim, float* gates, void* stream);

/*
 * The blog's averaged gate: the MLP above applied, per sequence and head, to the mean of
 * x over the sequence's tokens, all in fp64.
 *   x       [batch][seq_len][heads][dim] bf16, 16-byte aligned
 *   gates   [batch][repeat][heads][3] fp32: the triple of (b, h) written to every r < repeat
 *           (repeat = 1 gives nsa_decode's [B][Hq][3]; repeat = seq_len gives per-token gates
 *           for nsa_prefill)
 *   workspace  device scratch of nsa_gate_mlp_pooled_workspace_size(...) bytes, 256-byte aligned
 * Weights, dim and errors as nsa_gate_mlp, plus NSA_ERR_WORKSPACE_TOO_SMALL.
 */
int nsa_gate_mlp_pooled(const void* x, const void* w1, const float* b1, const float* w2, const float* b2, int batch,
                        int seq_len, int heads, int dim, int repeat, float* gates, void* workspace,
                        size_t workspace_bytes, void* stream);

/* Workspace bytes nsa_gate_mlp_pooled needs; 0 if the arguments are invalid. */
size_t nsa_gate_mlp_pooled_workspace_size(int batch, int seq_len, int heads, int dim);

/*
 * Backward of nsa_prefill: the gradients of a loss L given dL/dout. The pages train the
 * model end to end (shd-paper.top page "VideoNSA: Native Sparse Attention Scales Video
 * Understanding", abstract); the selection is held constant (block indices carry no
 * gradient), and the compressed keys' gradient returns to their tokens with the
 * compression's weights (the bf16 rounding of the summaries passes gradients unchanged).
 *   q, k, v, gates, params: as given to nsa_prefill (or nsa_prefill_phi)
 *   d_out    [N][Hq][d] bf16, dL/dout
 *   sel_idx  [N_v][Hkv][top_n] int32: the forward's selection (nsa_prefill's out_sel_idx)
 *   fwd_workspace  NULL, or the workspace of the nsa_prefill / nsa_prefill_phi call being
 *            differentiated, unchanged since: its compressed-branch log-sum-exp and output
 *            (nsa_prefill_workspace_layout: lse, o_cmp) then replace a recomputation; if
 *            params.keep_branch_stats = 1 (for both calls) the selected and window branches'
 *            too (o_sel, lse_sel, o_win, lse_win), and every video row's dq, statistics and
 *            gate gradient come from single passes on the tensor cores
 *   fwd_workspace_bytes  its size; smaller than nsa_workspace_size(params, 0) (for example a
 *            workspace of a forward call without keep_branch_stats, given to a backward call
 *            with it) returns NSA_ERR_WORKSPACE_TOO_SMALL; ignored when fwd_workspace is NULL
 *   phi_k, phi_v  both NULL (mean compression) or both the learnable weights [Hkv][l] fp32
 *   dq       [N][Hq][d] fp32     dk, dv [N][Hkv][d] fp32    (written, not accumulated)
 *   dgates   [N][Hq][3] fp32: <dL/dout, o_b> per branch; 0 for text rows
 *   workspace    at least nsa_backward_workspace_size(params) bytes, 256-byte aligned
 * All device pointers; q, k, v, d_out, dq, dk, dv 16-byte aligned. Errors as nsa_prefill,
 * returned before anything is enqueued. dk and dv are sums of fp32 atomic adds, so their
 * last bits vary from run to run.
 */
int nsa_backward(const void* q, const void* k, const void* v, const float* gates, const void* d_out,
                 const int32_t* sel_idx, const void* fwd_workspace, size_t fwd_workspace_bytes, const float* phi_k,
                 const float* phi_v, const nsa_params_t* params, float* dq, float* dk, float* dv, float* dgates,
                 void* workspace, size_t workspace_bytes, void* stream);

/* Workspace bytes nsa_backward needs; 0 if params are invalid. */
size_t nsa_backward_workspace_size(const nsa_params_t* params);

/* Workspace bytes nsa_prefill (is_decode = 0) or nsa_decode (is_decode = 1) needs; 0 if params are invalid. */
size_t nsa_workspace_size(const nsa_params_t* params, int is_decode);

/*
 * Where nsa_prefill keeps its intermediates inside the workspace (byte offsets), for
 * inspection after the stream has been synchronised. Every field is an offset from the
 * workspace base; layouts are row-major:
 *   kc, vc   [Ncmp(N_v)][Hkv][d] bf16     o_cmp [N_v][Hq][d] fp16     lse [N_v][Hq] fp32 (natural log)
 *   scores   [N_v][Hkv][score_stride] fp32: block j of row (t, g) at j, Nsel = ceil(N_v / l')
 *            blocks (score_stride = Nsel rounded up to a multiple of 4); only j <= t/l' is written
 *   sel_idx  [N_v][Hkv][top_n] int32      o_win [N_v][Hq][d] fp16 (window branch)
 * With params.keep_branch_stats = 1 the selected branch's output and the two other
 * log-sum-exps are kept too (else these offsets are 0 and the selected output goes straight
 * into the gated combine):
 *   o_sel [N_v][Hq][d] fp16     lse_sel, lse_win [N_v][Hq] fp32 (natural log; -inf: no key)
 * Returns NSA_OK or NSA_ERR_INVALID_ARG.
 */
typedef struct {
  size_t kc, vc, o_cmp, lse, scores, sel_idx, o_win, total;
  int32_t n_cmp, n_sel;
  int32_t score_stride;  /* floats between consecutive (t, g) score rows */
  size_t o_sel, lse_sel, lse_win;
} nsa_prefill_layout_t;
int nsa_prefill_workspace_layout(const nsa_params_t* params, nsa_prefill_layout_t* layout);

/* Human-readable text of a status code (static storage). */
const char* nsa_error_string(int status);

/*
 * Device error word: bit 0 = a kernel's bounded wait timed out (the kernel stopped
 * early, its output is invalid); bit 1 = a kernel met an out-of-range index and skipped
 * the access. Synchronises the current device, reads the word and, if `clear` is
 * non-zero, resets it. Returns NSA_OK or NSA_ERR_CUDA.
 */
int nsa_get_device_error(uint32_t* word, int clear);

/*
 * Self-test of failure detection. Every wait inside this library's kernels is bounded; a
 * wait that runs out records bit 0 of the device error word and its kernel returns early
 * instead of hanging. This entry point exercises exactly that path without any fault: it
 * launches one warp that waits, through the library's bounded wait, on a barrier nothing
 * ever arrives at, with a budget of `limit_cycles` GPU clock cycles (1 .. 4e9; e.g. 2e6 is
 * about 1 ms). After the stream drains, nsa_get_device_error reports bit 0 set; the
 * context stays usable. Returns NSA_OK, NSA_ERR_INVALID_ARG (limit out of range),
 * NSA_ERR_UNSUPPORTED (not sm_100) or NSA_ERR_CUDA.
 */
int nsa_selftest_wait_timeout(int64_t limit_cycles, void* stream);

/*
 * Stage timing (diagnostics). After nsa_profile_stages(events, count) with count > 0,
 * every nsa_prefill / nsa_decode call records events[i] (cudaEvent_t handles owned by
 * the caller) on its stream at its stage boundaries: events[0] before the first kernel,
 * then one event after each kernel, in launch order (prefill: pool, compressed attention,
 * top-n, selected buckets, selected tiles, window, merge + gated combine, dense text rows;
 * decode: compressed split, select, branches + gated combine). Stages that do not run
 * record nothing; events beyond `count` are not recorded. count = 0 (or events = NULL)
 * switches recording off. The
 * registration belongs to the calling host thread: it applies to the calls that thread
 * makes, and other threads' calls record nothing. Returns NSA_OK or NSA_ERR_INVALID_ARG.
 */
int nsa_profile_stages(void* const* events, int count);

/* Library version string, e.g. "nsa-b200 0.1.0 sm_100a". */
const char* nsa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* NSA_H_ */
