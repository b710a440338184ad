"""Python binding of the C ABI in include/nsa.h (argument marshalling only).

Every function named like the C entry point takes torch tensors (or raw device
addresses) and forwards them unchanged; all computation happens in the sm_100a kernels
of libnsa_b200.so. There is no fallback: if the library is missing or fails to load,
every call raises NsaLibraryError.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

NSA_OK = 0
NSA_ERR_INVALID_ARG = 1
NSA_ERR_UNSUPPORTED = 2
NSA_ERR_WORKSPACE_TOO_SMALL = 3
NSA_ERR_CUDA = 4
NSA_ERR_NOALLOC_TOO_LARGE = 5
NSA_NOALLOC_SCRATCH_BYTES = 32 << 20

NSA_OUT_BF16 = 0
NSA_OUT_F32 = 1

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libnsa_b200.so")

EXPORTED = (
    "nsa_prefill", "nsa_decode", "nsa_compress", "nsa_workspace_size", "nsa_prefill_workspace_layout",
    "nsa_error_string", "nsa_get_device_error", "nsa_version", "nsa_profile_stages", "nsa_decode_noalloc",
    "nsa_prefill_varlen", "nsa_prefill_varlen_workspace_size", "nsa_compress_weighted", "nsa_prefill_phi",
    "nsa_gate_mlp", "nsa_gate_mlp_pooled", "nsa_gate_mlp_pooled_workspace_size", "nsa_backward",
    "nsa_backward_workspace_size", "nsa_selftest_wait_timeout", "nsa_prefill_packed",
    "nsa_prefill_packed_workspace_size",
)


class NsaLibraryError(RuntimeError):
    pass


class NsaError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {nsa_error_string(status)} (status {status})")
        self.status = status


class NsaParams(ctypes.Structure):
    _fields_ = [
        ("n_tokens", ctypes.c_int32), ("n_video", ctypes.c_int32), ("num_q_heads", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("cmp_block", ctypes.c_int32),
        ("cmp_stride", ctypes.c_int32), ("sel_block", ctypes.c_int32), ("top_n", ctypes.c_int32),
        ("window", ctypes.c_int32), ("softmax_scale", ctypes.c_float), ("out_dtype", ctypes.c_int32),
        ("batch", ctypes.c_int32), ("keep_branch_stats", ctypes.c_int32),
    ]


class NsaPrefillLayout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in ("kc", "vc", "o_cmp", "lse", "scores", "sel_idx", "o_win", "total")] + [
        ("n_cmp", ctypes.c_int32), ("n_sel", ctypes.c_int32), ("score_stride", ctypes.c_int32)] + [
        (n, ctypes.c_size_t) for n in ("o_sel", "lse_sel", "lse_win")]


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libnsa_b200.so (built by sparse_attention_long_fwd_b200.build)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise NsaLibraryError(f"{path} is missing: build it with `python -m sparse_attention_long_fwd_b200.build`")
    try:
        lib = ctypes.CDLL(path)
    except OSError as e:  # pragma: no cover
        raise NsaLibraryError(f"cannot load {path}: {e}") from e
    P, I, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    PP = ctypes.POINTER(NsaParams)
    lib.nsa_prefill.argtypes = [P, P, P, P, PP, P, P, P, S, P]
    lib.nsa_prefill.restype = I
    I32P = ctypes.POINTER(ctypes.c_int32)
    lib.nsa_prefill_varlen.argtypes = [P, P, P, P, I32P, I32P, I, PP, P, P, P, S, P]
    lib.nsa_prefill_varlen.restype = I
    lib.nsa_prefill_varlen_workspace_size.argtypes = [PP, I32P, I32P, I]
    lib.nsa_prefill_varlen_workspace_size.restype = S
    U8P = ctypes.POINTER(ctypes.c_uint8)
    lib.nsa_prefill_packed.argtypes = [P, P, P, P, I32P, I, I32P, U8P, I, PP, P, P, P, S, P]
    lib.nsa_prefill_packed.restype = I
    lib.nsa_prefill_packed_workspace_size.argtypes = [PP, I32P, I, I32P, U8P, I]
    lib.nsa_prefill_packed_workspace_size.restype = S
    lib.nsa_decode.argtypes = [P, P, P, P, P, P, P, PP, P, P, P, S, P]
    lib.nsa_decode.restype = I
    lib.nsa_decode_noalloc.argtypes = [P, P, P, P, P, P, P, PP, P, P, P]
    lib.nsa_decode_noalloc.restype = I
    lib.nsa_compress.argtypes = [P, P, PP, P, P, P]
    lib.nsa_compress.restype = I
    lib.nsa_compress_weighted.argtypes = [P, P, P, P, PP, P, P, P]
    lib.nsa_compress_weighted.restype = I
    lib.nsa_prefill_phi.argtypes = [P, P, P, P, P, P, PP, P, P, P, S, P]
    lib.nsa_prefill_phi.restype = I
    lib.nsa_gate_mlp.argtypes = [P, P, P, P, P, ctypes.c_int64, I, P, P]
    lib.nsa_gate_mlp.restype = I
    lib.nsa_gate_mlp_pooled.argtypes = [P, P, P, P, P, I, I, I, I, I, P, P, S, P]
    lib.nsa_gate_mlp_pooled.restype = I
    lib.nsa_gate_mlp_pooled_workspace_size.argtypes = [I, I, I, I]
    lib.nsa_gate_mlp_pooled_workspace_size.restype = S
    lib.nsa_backward.argtypes = [P, P, P, P, P, P, P, S, P, P, PP, P, P, P, P, P, S, P]
    lib.nsa_backward.restype = I
    lib.nsa_backward_workspace_size.argtypes = [PP]
    lib.nsa_backward_workspace_size.restype = S
    lib.nsa_workspace_size.argtypes = [PP, I]
    lib.nsa_workspace_size.restype = S
    lib.nsa_prefill_workspace_layout.argtypes = [PP, ctypes.POINTER(NsaPrefillLayout)]
    lib.nsa_prefill_workspace_layout.restype = I
    lib.nsa_error_string.argtypes = [I]
    lib.nsa_error_string.restype = ctypes.c_char_p
    lib.nsa_get_device_error.argtypes = [ctypes.POINTER(ctypes.c_uint32), I]
    lib.nsa_get_device_error.restype = I
    lib.nsa_version.argtypes = []
    lib.nsa_version.restype = ctypes.c_char_p
    lib.nsa_profile_stages.argtypes = [ctypes.POINTER(ctypes.c_void_p), I]
    lib.nsa_profile_stages.restype = I
    lib.nsa_selftest_wait_timeout.argtypes = [ctypes.c_int64, P]
    lib.nsa_selftest_wait_timeout.restype = I
    _lib = lib
    return lib


def make_params(n_tokens: int, n_video: int | None = None, num_q_heads: int = 28, num_kv_heads: int = 4,
                head_dim: int = 128, cmp_block: int = 32, cmp_stride: int = 16, sel_block: int = 64, top_n: int = 16,
                window: int = 512, softmax_scale: float = 0.0, out_dtype: int = NSA_OUT_F32,
                batch: int = 0, keep_branch_stats: bool = False) -> NsaParams:
    return NsaParams(n_tokens, n_tokens if n_video is None else n_video, num_q_heads, num_kv_heads, head_dim,
                     cmp_block, cmp_stride, sel_block, top_n, window, softmax_scale, out_dtype, batch,
                     1 if keep_branch_stats else 0)


def _addr(x) -> int | None:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


# ------------------------------------------------------------------ C entry points, same names

def nsa_prefill(q, k, v, gates, params: NsaParams, out, out_sel_idx, workspace, workspace_bytes: int,
                stream=None) -> int:
    return load_library().nsa_prefill(_addr(q), _addr(k), _addr(v), _addr(gates), ctypes.byref(params), _addr(out),
                                      _addr(out_sel_idx), _addr(workspace), workspace_bytes, _stream(stream))


def _host_i32(values):
    """A host int32 array (ctypes) from a sequence of ints."""
    vals = [int(x) for x in values]
    return (ctypes.c_int32 * len(vals))(*vals)


def nsa_prefill_varlen(q, k, v, gates, cu_seqlens, n_video, params: NsaParams, out, out_sel_idx, workspace,
                       workspace_bytes: int, stream=None) -> int:
    """Packed batch prefill; cu_seqlens ([B+1]) and n_video ([B]) are host integer sequences."""
    cu, nv = _host_i32(cu_seqlens), _host_i32(n_video)
    return load_library().nsa_prefill_varlen(_addr(q), _addr(k), _addr(v), _addr(gates), cu, nv, len(nv),
                                             ctypes.byref(params), _addr(out), _addr(out_sel_idx),
                                             _addr(workspace), workspace_bytes, _stream(stream))


def nsa_prefill_varlen_workspace_size(params: NsaParams, cu_seqlens, n_video) -> int:
    cu, nv = _host_i32(cu_seqlens), _host_i32(n_video)
    return load_library().nsa_prefill_varlen_workspace_size(ctypes.byref(params), cu, nv, len(nv))


def _host_u8(values):
    vals = [int(x) for x in values]
    return (ctypes.c_uint8 * max(len(vals), 1))(*vals)


def nsa_prefill_packed(q, k, v, gates, cu_seqlens, seg_lens, seg_video, params: NsaParams, out, out_sel_idx,
                       workspace, workspace_bytes: int, stream=None) -> int:
    """Packed batch with video and text segments in any order; cu_seqlens ([B+1]), seg_lens and
    seg_video ([S]) are host integer sequences."""
    cu, sl, sv = _host_i32(cu_seqlens), _host_i32(seg_lens), _host_u8(seg_video)
    return load_library().nsa_prefill_packed(_addr(q), _addr(k), _addr(v), _addr(gates), cu, len(cu) - 1, sl, sv,
                                             len(seg_lens), ctypes.byref(params), _addr(out), _addr(out_sel_idx),
                                             _addr(workspace), workspace_bytes, _stream(stream))


def nsa_prefill_packed_workspace_size(params: NsaParams, cu_seqlens, seg_lens, seg_video) -> int:
    cu, sl, sv = _host_i32(cu_seqlens), _host_i32(seg_lens), _host_u8(seg_video)
    return int(load_library().nsa_prefill_packed_workspace_size(ctypes.byref(params), cu, len(cu) - 1, sl, sv,
                                                                 len(seg_lens)))


def nsa_decode(q, kcache, vcache, kcmp, vcmp, seq_lens, gates, params: NsaParams, out, out_sel_idx, workspace,
               workspace_bytes: int, stream=None) -> int:
    return load_library().nsa_decode(_addr(q), _addr(kcache), _addr(vcache), _addr(kcmp), _addr(vcmp),
                                     _addr(seq_lens), _addr(gates), ctypes.byref(params), _addr(out),
                                     _addr(out_sel_idx), _addr(workspace), workspace_bytes, _stream(stream))


def nsa_decode_noalloc(q, kcache, vcache, kcmp, vcmp, seq_lens, gates, params: NsaParams, out, out_sel_idx,
                       stream=None) -> int:
    """nsa_decode without a workspace: for callers that cannot allocate device memory
    (scratch lives in the library's fixed NSA_NOALLOC_SCRATCH_BYTES device array)."""
    return load_library().nsa_decode_noalloc(_addr(q), _addr(kcache), _addr(vcache), _addr(kcmp), _addr(vcmp),
                                             _addr(seq_lens), _addr(gates), ctypes.byref(params), _addr(out),
                                             _addr(out_sel_idx), _stream(stream))


def nsa_compress(k, v, params: NsaParams, kcmp, vcmp, stream=None) -> int:
    return load_library().nsa_compress(_addr(k), _addr(v), ctypes.byref(params), _addr(kcmp), _addr(vcmp),
                                       _stream(stream))


def nsa_compress_weighted(k, v, phi_k, phi_v, params: NsaParams, kcmp, vcmp, stream=None) -> int:
    return load_library().nsa_compress_weighted(_addr(k), _addr(v), _addr(phi_k), _addr(phi_v), ctypes.byref(params),
                                                _addr(kcmp), _addr(vcmp), _stream(stream))


def nsa_prefill_phi(q, k, v, gates, phi_k, phi_v, params: NsaParams, out, out_sel_idx, workspace,
                    workspace_bytes: int, stream=None) -> int:
    return load_library().nsa_prefill_phi(_addr(q), _addr(k), _addr(v), _addr(gates), _addr(phi_k), _addr(phi_v),
                                          ctypes.byref(params), _addr(out), _addr(out_sel_idx), _addr(workspace),
                                          workspace_bytes, _stream(stream))


def nsa_gate_mlp(x, w1, b1, w2, b2, rows: int, dim: int, gates, stream=None) -> int:
    return load_library().nsa_gate_mlp(_addr(x), _addr(w1), _addr(b1), _addr(w2), _addr(b2), rows, dim,
                                       _addr(gates), _stream(stream))


def nsa_gate_mlp_pooled(x, w1, b1, w2, b2, batch: int, seq_len: int, heads: int, dim: int, repeat: int, gates,
                        workspace, workspace_bytes: int, stream=None) -> int:
    return load_library().nsa_gate_mlp_pooled(_addr(x), _addr(w1), _addr(b1), _addr(w2), _addr(b2), batch, seq_len,
                                              heads, dim, repeat, _addr(gates), _addr(workspace), workspace_bytes,
                                              _stream(stream))


def nsa_gate_mlp_pooled_workspace_size(batch: int, seq_len: int, heads: int, dim: int) -> int:
    return int(load_library().nsa_gate_mlp_pooled_workspace_size(batch, seq_len, heads, dim))


def nsa_backward(q, k, v, gates, d_out, sel_idx, fwd_workspace, fwd_workspace_bytes: int, phi_k, phi_v,
                 params: NsaParams, dq, dk, dv, dgates, workspace, workspace_bytes: int, stream=None) -> int:
    return load_library().nsa_backward(_addr(q), _addr(k), _addr(v), _addr(gates), _addr(d_out), _addr(sel_idx),
                                       _addr(fwd_workspace), fwd_workspace_bytes, _addr(phi_k), _addr(phi_v),
                                       ctypes.byref(params), _addr(dq), _addr(dk), _addr(dv), _addr(dgates),
                                       _addr(workspace), workspace_bytes, _stream(stream))


def nsa_backward_workspace_size(params: NsaParams) -> int:
    return int(load_library().nsa_backward_workspace_size(ctypes.byref(params)))


def nsa_workspace_size(params: NsaParams, is_decode: bool) -> int:
    return int(load_library().nsa_workspace_size(ctypes.byref(params), int(bool(is_decode))))


def nsa_prefill_workspace_layout(params: NsaParams) -> dict:
    lay = NsaPrefillLayout()
    rc = load_library().nsa_prefill_workspace_layout(ctypes.byref(params), ctypes.byref(lay))
    if rc != NSA_OK:
        raise NsaError(rc, "nsa_prefill_workspace_layout")
    return {n: getattr(lay, n) for n, _ in NsaPrefillLayout._fields_}


def nsa_error_string(status: int) -> str:
    return load_library().nsa_error_string(status).decode()


def nsa_get_device_error(clear: bool = True) -> int:
    w = ctypes.c_uint32(0)
    rc = load_library().nsa_get_device_error(ctypes.byref(w), int(bool(clear)))
    if rc != NSA_OK:
        raise NsaError(rc, "nsa_get_device_error")
    return int(w.value)


def nsa_selftest_wait_timeout(limit_cycles: int, stream=None) -> int:
    """Launch the failure-detection self-test: a bounded wait on a barrier nothing arrives
    at, which must give up after limit_cycles and set bit 0 of the device error word."""
    return load_library().nsa_selftest_wait_timeout(int(limit_cycles), _stream(stream))


def nsa_version() -> str:
    return load_library().nsa_version().decode()


_stage_handles = None


def nsa_profile_stages(events) -> int:
    """Register torch.cuda.Event objects (or raw cudaEvent_t handles) recorded at stage
    boundaries of every following call; an empty list switches recording off."""
    global _stage_handles
    handles = [e.cuda_event if hasattr(e, "cuda_event") else int(e) for e in (events or [])]
    _stage_handles = (ctypes.c_void_p * max(len(handles), 1))(*handles)
    return load_library().nsa_profile_stages(_stage_handles if handles else None, len(handles))


# ------------------------------------------------------------------ torch conveniences

def _check(rc: int, where: str):
    if rc != NSA_OK:
        raise NsaError(rc, where)


def alloc_workspace(params: NsaParams, is_decode: bool, device) -> torch.Tensor:
    n = nsa_workspace_size(params, is_decode)
    if n == 0:
        raise NsaError(NSA_ERR_INVALID_ARG, "nsa_workspace_size")
    # torch's caching allocator returns 512-byte aligned blocks
    return torch.empty(n, dtype=torch.uint8, device=device)


def prefill(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, gates: torch.Tensor, *, n_video: int | None = None,
            top_n: int = 16, window: int = 512, softmax_scale: float = 0.0, out_dtype=torch.float32,
            return_sel: bool = False, workspace: torch.Tensor | None = None, phi=None,
            keep_branch_stats: bool = False, stream=None):
    """NSA prefill of one sequence: q [N,Hq,d], k/v [N,Hkv,d] bf16, gates [N,Hq,3] fp32 (device tensors).
    phi = (phi_k, phi_v), each [Hkv, 32] fp32, selects the learnable compression.
    keep_branch_stats keeps in the workspace what backward(..., keep_branch_stats=True) reuses."""
    N, hq, d = q.shape
    hkv = k.shape[1]
    p = make_params(N, n_video, hq, hkv, d, top_n=top_n, window=window, softmax_scale=softmax_scale,
                    out_dtype=NSA_OUT_F32 if out_dtype == torch.float32 else NSA_OUT_BF16,
                    keep_branch_stats=keep_branch_stats)
    out = torch.empty((N, hq, d), dtype=out_dtype, device=q.device)
    sel = torch.empty((p.n_video, hkv, top_n), dtype=torch.int32, device=q.device) if return_sel else None
    if workspace is None:
        workspace = alloc_workspace(p, False, q.device)
    if phi is None:
        _check(nsa_prefill(q, k, v, gates, p, out, sel, workspace, workspace.numel(), stream), "nsa_prefill")
    else:
        _check(nsa_prefill_phi(q, k, v, gates, phi[0], phi[1], p, out, sel, workspace, workspace.numel(), stream),
               "nsa_prefill_phi")
    return (out, sel) if return_sel else out


def compress(k: torch.Tensor, v: torch.Tensor, phi=None, stream=None):
    """Compressed cache of a [B, L, Hkv, d] (or [L, Hkv, d]) bf16 K/V pair; phi = (phi_k, phi_v),
    each [Hkv, 32] fp32, selects the learnable compression."""
    squeeze = k.dim() == 3
    if squeeze:
        k, v = k.unsqueeze(0), v.unsqueeze(0)
    B, L, hkv, d = k.shape
    p = make_params(L, L, hkv, hkv, d, batch=B)
    nc = (L - p.cmp_block) // p.cmp_stride + 1 if L >= p.cmp_block else 0  # Ncmp(L) of the params' l and s
    kc = torch.empty((B, nc, hkv, d), dtype=k.dtype, device=k.device)
    vc = torch.empty_like(kc)
    if phi is None:
        _check(nsa_compress(k, v, p, kc, vc, stream), "nsa_compress")
    else:
        _check(nsa_compress_weighted(k, v, phi[0], phi[1], p, kc, vc, stream), "nsa_compress_weighted")
    return (kc[0], vc[0]) if squeeze else (kc, vc)


def decode(q, kcache, vcache, kcmp, vcmp, seq_lens, gates, *, top_n: int = 16, window: int = 512,
           softmax_scale: float = 0.0, out_dtype=torch.float32, return_sel: bool = False,
           workspace: torch.Tensor | None = None, stream=None):
    """NSA decode: q [B,Hq,d], caches [B,Lmax,Hkv,d], compressed caches [B,Ncmp,Hkv,d], seq_lens [B] int32."""
    B, hq, d = q.shape
    Lmax, hkv = kcache.shape[1], kcache.shape[2]
    p = make_params(Lmax, Lmax, hq, hkv, d, top_n=top_n, window=window, softmax_scale=softmax_scale,
                    out_dtype=NSA_OUT_F32 if out_dtype == torch.float32 else NSA_OUT_BF16, batch=B)
    out = torch.empty((B, hq, d), dtype=out_dtype, device=q.device)
    sel = torch.empty((B, hkv, top_n), dtype=torch.int32, device=q.device) if return_sel else None
    if workspace is None:
        workspace = alloc_workspace(p, True, q.device)
    _check(nsa_decode(q, kcache, vcache, kcmp, vcmp, seq_lens, gates, p, out, sel, workspace, workspace.numel(),
                      stream), "nsa_decode")
    return (out, sel) if return_sel else out


def backward(q, k, v, gates, d_out, sel_idx, *, n_video: int | None = None, top_n: int = 16, window: int = 512,
             softmax_scale: float = 0.0, phi=None, fwd_workspace: torch.Tensor | None = None,
             keep_branch_stats: bool = False, workspace: torch.Tensor | None = None, stream=None):
    """Gradients of the prefill: returns dq [N,Hq,d], dk, dv [N,Hkv,d] and dgates [N,Hq,3] (fp32),
    given dL/dout (bf16) and the forward's selection sel_idx [N_v,Hkv,top_n]; fwd_workspace, the
    forward call's workspace, lets the compressed branch reuse its saved statistics, and every
    branch when both calls pass keep_branch_stats=True."""
    N, hq, d = q.shape
    hkv = k.shape[1]
    p = make_params(N, n_video, hq, hkv, d, top_n=top_n, window=window, softmax_scale=softmax_scale,
                    keep_branch_stats=keep_branch_stats)
    dq = torch.empty((N, hq, d), dtype=torch.float32, device=q.device)
    dk = torch.empty((N, hkv, d), dtype=torch.float32, device=q.device)
    dv = torch.empty_like(dk)
    dgates = torch.empty((N, hq, 3), dtype=torch.float32, device=q.device)
    if workspace is None:
        n = nsa_backward_workspace_size(p)
        if n == 0:
            raise NsaError(NSA_ERR_INVALID_ARG, "nsa_backward_workspace_size")
        workspace = torch.empty(n, dtype=torch.uint8, device=q.device)
    pk, pv = (None, None) if phi is None else phi
    fwd_bytes = fwd_workspace.numel() if fwd_workspace is not None else 0
    _check(nsa_backward(q, k, v, gates, d_out, sel_idx, fwd_workspace, fwd_bytes, pk, pv, p, dq, dk, dv, dgates,
                        workspace, workspace.numel(), stream), "nsa_backward")
    return dq, dk, dv, dgates


def gate_mlp(x: torch.Tensor, w1: torch.Tensor, b1: torch.Tensor, w2: torch.Tensor, b2: torch.Tensor, stream=None):
    """Per-row gates: x [..., dim] bf16 -> [..., 3] fp32 (w1 [dim/2, dim] bf16; b1, w2, b2 fp32)."""
    dim = x.shape[-1]
    gates = torch.empty((*x.shape[:-1], 3), dtype=torch.float32, device=x.device)
    _check(nsa_gate_mlp(x, w1, b1, w2, b2, x.numel() // dim, dim, gates, stream), "nsa_gate_mlp")
    return gates


def gate_mlp_pooled(x: torch.Tensor, w1, b1, w2, b2, repeat: int = 1, stream=None):
    """Averaged gates: x [B, T, H, dim] bf16 -> [B, repeat, H, 3] fp32 (the (b, h) triple repeated)."""
    B, T, H, dim = x.shape
    gates = torch.empty((B, repeat, H, 3), dtype=torch.float32, device=x.device)
    ws = torch.empty(max(nsa_gate_mlp_pooled_workspace_size(B, T, H, dim), 1), dtype=torch.uint8, device=x.device)
    _check(nsa_gate_mlp_pooled(x, w1, b1, w2, b2, B, T, H, dim, repeat, gates, ws, ws.numel(), stream),
           "nsa_gate_mlp_pooled")
    return gates


def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)
