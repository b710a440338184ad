"""ctypes front end of the fp64 CPU oracle (nsa_oracle.c).

TEST INFRASTRUCTURE ONLY: imported by tests/, by ``__graft_entry__.smoke()`` and by the
CPU-baseline leg of ``bench.py``. It never imports the CUDA package and the CUDA package
never imports it. bf16 tensors cross this boundary as their raw 16-bit patterns
(``numpy.uint16``), so the oracle consumes exactly the bytes the GPU consumed.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nsa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_build", "libnsa_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile nsa_oracle.c with gcc (-O2, OpenMP, no fast-math) into oracle/_build/."""
    os.makedirs(os.path.dirname(_LIB_PATH), exist_ok=True)
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class _Cfg(ctypes.Structure):
    _fields_ = [
        ("n_tokens", ctypes.c_int), ("n_video", ctypes.c_int), ("hq", ctypes.c_int), ("hkv", ctypes.c_int),
        ("d", ctypes.c_int), ("cmp_len", ctypes.c_int), ("cmp_stride", ctypes.c_int), ("sel_len", ctypes.c_int),
        ("top_n", ctypes.c_int), ("window", ctypes.c_int), ("scale", ctypes.c_double),
    ]


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        lib.oracle_double_to_bf16.restype = ctypes.c_uint16
        lib.oracle_double_to_bf16.argtypes = [ctypes.c_double]
        lib.oracle_bf16_to_double.restype = ctypes.c_double
        lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
        lib.oracle_round_bf16_array.argtypes = [P, P, ctypes.c_size_t]
        lib.oracle_num_cmp.argtypes = [ctypes.c_int] * 3
        lib.oracle_num_sel.argtypes = [ctypes.c_int] * 2
        lib.oracle_compress.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, P]
        lib.oracle_compress_weighted.argtypes = [P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                 ctypes.c_int, P]
        lib.oracle_prefill_rows.argtypes = [ctypes.POINTER(_Cfg), P, P, P, P, P, P, ctypes.c_int, P, P, P, P, P,
                                            ctypes.c_int, P, P, P, P, P, P, P, ctypes.c_int]
        lib.oracle_decode.argtypes = [ctypes.POINTER(_Cfg), P, P, P, P, P, P, P, ctypes.c_int, P, P, P, P, P,
                                      ctypes.c_int, P, P, P, P, P, ctypes.c_int]
        _lib = lib
    return _lib


@dataclass
class OracleConfig:
    """Shapes and NSA constants: l = cmp_len, s = cmp_stride, l' = sel_len, n = top_n, w = window."""
    n_tokens: int
    n_video: int
    hq: int
    hkv: int
    d: int
    cmp_len: int = 32
    cmp_stride: int = 16
    sel_len: int = 64
    top_n: int = 16
    window: int = 512
    scale: float = 0.0  # <= 0 selects 1/sqrt(d)

    def c(self) -> _Cfg:
        sc = self.scale if self.scale > 0 else 1.0 / math.sqrt(self.d)
        return _Cfg(self.n_tokens, self.n_video, self.hq, self.hkv, self.d, self.cmp_len, self.cmp_stride,
                    self.sel_len, self.top_n, self.window, sc)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError("bf16 data must be passed as uint16 bit patterns")
    return a


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to float64."""
    return (np.ascontiguousarray(bits).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def round_bf16(x: np.ndarray) -> np.ndarray:
    """fp64 -> bf16 bit patterns, round to nearest even, one rounding step."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.uint16)
    _load().oracle_round_bf16_array(_ptr(x), _ptr(out), x.size)
    return out


def num_cmp(T: int, l: int = 32, s: int = 16) -> int:
    return int(_load().oracle_num_cmp(T, l, s))


def num_sel(T: int, lsel: int = 64) -> int:
    return int(_load().oracle_num_sel(T, lsel))


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def compress(k_bits: np.ndarray, l: int = 32, s: int = 16) -> np.ndarray:
    """Mean-pool [T, h, d] bf16 keys (values) into [Ncmp(T), h, d] bf16 summaries."""
    k_bits = _u16(k_bits)
    T, h, d = k_bits.shape
    nc = num_cmp(T, l, s)
    out = np.zeros((max(nc, 0), h, d), dtype=np.uint16)
    _load().oracle_compress(_ptr(k_bits), T, h, d, l, s, _ptr(out))
    return out


def compress_weighted(k_bits: np.ndarray, w: np.ndarray, l: int = 32, s: int = 16) -> np.ndarray:
    """Learnable compression of [T, h, d] bf16 keys (values): every complete block is the
    w-weighted sum of its l tokens, w [h, l] float32 per head, rounded once to bf16."""
    k_bits = _u16(k_bits)
    T, h, d = k_bits.shape
    w = np.ascontiguousarray(w, dtype=np.float32)
    if w.shape != (h, l):
        raise ValueError(f"weights must be [{h}, {l}], got {w.shape}")
    nc = num_cmp(T, l, s)
    out = np.zeros((max(nc, 0), h, d), dtype=np.uint16)
    _load().oracle_compress_weighted(_ptr(k_bits), _ptr(w), T, h, d, l, s, _ptr(out))
    return out


def _alloc_outputs(n: int, cfg: OracleConfig, nsel_w: int, want: tuple):
    o = {"out": np.zeros((n, cfg.hq, cfg.d))}
    if "sel" in want:
        o["sel"] = np.zeros((n, cfg.hkv, cfg.top_n), dtype=np.int32)
    if "scores" in want:
        o["scores"] = np.zeros((n, cfg.hkv, nsel_w))
    for key in ("o_cmp", "o_sel", "o_win"):
        if key in want:
            o[key] = np.zeros((n, cfg.hq, cfg.d))
    for key in ("lse", "lse_sel", "lse_win"):
        if key in want:
            o[key] = np.zeros((n, cfg.hq))
    if "tie_gap" in want:
        o["tie_gap"] = np.zeros((n, cfg.hkv))
    return o


ALL = ("sel", "scores", "o_cmp", "lse", "o_sel", "o_win", "tie_gap")


def prefill_rows(cfg: OracleConfig, q, k, v, gates, rows, kc=None, vc=None, sel_override=None, want=ALL,
                 nthreads: int = 0) -> dict:
    """Evaluate the listed query rows of a prefill. q [N,hq,d], k/v [N,hkv,d] (uint16 bf16 bits),
    gates [N,hq,3] float32. kc/vc default to compress() of the video prefix."""
    q, k, v = _u16(q), _u16(k), _u16(v)
    gates = np.ascontiguousarray(gates, dtype=np.float32)
    rows = np.ascontiguousarray(rows, dtype=np.int32)
    if kc is None:
        kc = compress(k[: cfg.n_video], cfg.cmp_len, cfg.cmp_stride)
    if vc is None:
        vc = compress(v[: cfg.n_video], cfg.cmp_len, cfg.cmp_stride)
    kc, vc = _u16(kc), _u16(vc)
    nsel_w = max(num_sel(cfg.n_video, cfg.sel_len), 1)
    o = _alloc_outputs(len(rows), cfg, nsel_w, want)
    so = None if sel_override is None else np.ascontiguousarray(sel_override, dtype=np.int32)
    c = cfg.c()
    rc = _load().oracle_prefill_rows(ctypes.byref(c), _ptr(q), _ptr(k), _ptr(v), _ptr(gates), _ptr(kc), _ptr(vc),
                                     len(rows), _ptr(rows), _ptr(so), _ptr(o["out"]), _ptr(o.get("sel")),
                                     _ptr(o.get("scores")), nsel_w, _ptr(o.get("o_cmp")), _ptr(o.get("lse")),
                                     _ptr(o.get("o_sel")), _ptr(o.get("o_win")), _ptr(o.get("tie_gap")),
                                     _ptr(o.get("lse_sel")), _ptr(o.get("lse_win")), nthreads)
    if rc != 0:
        raise ValueError("oracle_prefill_rows rejected its arguments")
    return o


def decode(cfg: OracleConfig, q, kcache, vcache, kcmp, vcmp, seq_lens, gates, seqs=None, sel_override=None,
           want=ALL, nthreads: int = 0) -> dict:
    """Single-query decode for the listed sequences (default: all). cfg.n_tokens = cache capacity."""
    q, kcache, vcache, kcmp, vcmp = (_u16(a) for a in (q, kcache, vcache, kcmp, vcmp))
    seq_lens = np.ascontiguousarray(seq_lens, dtype=np.int32)
    gates = np.ascontiguousarray(gates, dtype=np.float32)
    if seqs is None:
        seqs = np.arange(len(seq_lens), dtype=np.int32)
    seqs = np.ascontiguousarray(seqs, dtype=np.int32)
    nsel_w = max(num_sel(cfg.n_tokens, cfg.sel_len), 1)
    o = _alloc_outputs(len(seqs), cfg, nsel_w, want)
    so = None if sel_override is None else np.ascontiguousarray(sel_override, dtype=np.int32)
    c = cfg.c()
    rc = _load().oracle_decode(ctypes.byref(c), _ptr(q), _ptr(kcache), _ptr(vcache), _ptr(kcmp), _ptr(vcmp),
                               _ptr(seq_lens), _ptr(gates), len(seqs), _ptr(seqs), _ptr(so), _ptr(o["out"]),
                               _ptr(o.get("sel")), _ptr(o.get("scores")), nsel_w, _ptr(o.get("o_cmp")),
                               _ptr(o.get("lse")), _ptr(o.get("o_sel")), _ptr(o.get("o_win")),
                               _ptr(o.get("tie_gap")), nthreads)
    if rc != 0:
        raise ValueError("oracle_decode rejected its arguments")
    return o
