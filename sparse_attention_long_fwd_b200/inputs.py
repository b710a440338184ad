"""Seeded synthetic inputs for the NSA forward pass (shared by tests and the benchmark).

This module only draws random tensors with the shapes and distributions of the named
workloads; it holds none of the attention arithmetic. Video tokens are laid out as
frames of 64 tokens (a 50,176-pixel frame at 28x28 pixels per merged vision token),
token-major: q [N, Hq, d], k/v [N, Hkv, d] in bf16, gates [N, Hq, 3] in fp32 ordered
(cmp, sel, win).
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace

import torch

TOKENS_PER_FRAME = 64


@dataclass(frozen=True)
class Workload:
    name: str
    n_tokens: int            # N (prefill) or cache capacity (decode)
    n_video: int             # NSA-attended prefix; the rest are trailing text rows
    hq: int = 28
    hkv: int = 4
    d: int = 128
    cmp_len: int = 32
    cmp_stride: int = 16
    sel_len: int = 64
    top_n: int = 16
    window: int = 512
    frame_mean_var: float = 0.0  # variance of the per-(frame, kv head, dim) mean added to K
    batch: int = 0           # > 0: decode workload with this many sequences
    extra: dict = field(default_factory=dict)

    @property
    def is_decode(self) -> bool:
        return self.batch > 0


WORKLOADS = {
    # 1 sequence, 2048 video tokens, small heads
    "tiny": Workload("tiny", 2048, 2048, hq=4, hkv=1, d=64, top_n=4, window=256),
    # Qwen2.5-VL-7B attention shape: 564 frames x 64 video tokens, then 256 text tokens
    "qwen36k_hybrid": Workload("qwen36k_hybrid", 36352, 36096),
    # 2048 frames x 64 tokens, per-frame correlated keys so selection is non-uniform
    "v128k": Workload("v128k", 131072, 131072, frame_mean_var=0.5),
    "sweep128k_n4_w256": Workload("sweep128k_n4_w256", 131072, 131072, top_n=4, window=256, frame_mean_var=0.5),
    "sweep128k_n16_w512": Workload("sweep128k_n16_w512", 131072, 131072, top_n=16, window=512,
                                   frame_mean_var=0.5),
    "sweep128k_n48_w1024": Workload("sweep128k_n48_w1024", 131072, 131072, top_n=48, window=1024,
                                    frame_mean_var=0.5),
    # a 32,768-token cut of the 128K workload (inputs still larger than L2), for kernel profiles
    "v32k": Workload("v32k", 32768, 32768, frame_mean_var=0.5),
    # a 16,384-token cut (about 3 GB on the device), for multi-pass kernel profiles
    "v16k": Workload("v16k", 16384, 16384, frame_mean_var=0.5),
    # 64 sequences x 131,072-token cache, one query each
    "decode64x128k": Workload("decode64x128k", 131072, 131072, batch=64),
}


def scaled(w: Workload, **kw) -> Workload:
    """A copy of a workload with some fields replaced (smaller test cases)."""
    return replace(w, **kw)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def prefill_inputs(w: Workload, seed: int = 0, device="cpu"):
    """q, k, v (bf16) and gates (fp32) for a prefill workload.

    q, v ~ N(0,1); k ~ N(0,1) plus, when frame_mean_var > 0, a mean drawn once per
    (frame, kv head, dim) from N(0, frame_mean_var) and shared by the frame's 64 tokens;
    gates ~ U(0,1). Values are drawn in fp32 and rounded to bf16.
    """
    g = _gen(seed, device)
    N = w.n_tokens
    q = torch.randn((N, w.hq, w.d), generator=g, device=device).to(torch.bfloat16)
    k = torch.randn((N, w.hkv, w.d), generator=g, device=device)
    v = torch.randn((N, w.hkv, w.d), generator=g, device=device).to(torch.bfloat16)
    gates = torch.rand((N, w.hq, 3), generator=g, device=device)
    if w.frame_mean_var > 0:
        nframes = (N + TOKENS_PER_FRAME - 1) // TOKENS_PER_FRAME
        mu = torch.randn((nframes, w.hkv, w.d), generator=g, device=device) * (w.frame_mean_var ** 0.5)
        k = k + mu.repeat_interleave(TOKENS_PER_FRAME, dim=0)[:N]
    return q, k.to(torch.bfloat16), v, gates


def decode_inputs(w: Workload, seed: int = 0, device="cpu", seq_lens=None):
    """q [B,Hq,d], kcache/vcache [B,L,Hkv,d] (bf16, N(0,1)), gates [B,Hq,3] U(0,1), seq_lens [B] int32.

    By default every sequence is full (L = n_tokens)."""
    g = _gen(seed, device)
    B, L = w.batch, w.n_tokens
    q = torch.randn((B, w.hq, w.d), generator=g, device=device).to(torch.bfloat16)
    kc = torch.randn((B, L, w.hkv, w.d), generator=g, device=device).to(torch.bfloat16)
    vc = torch.randn((B, L, w.hkv, w.d), generator=g, device=device).to(torch.bfloat16)
    gates = torch.rand((B, w.hq, 3), generator=g, device=device)
    if seq_lens is None:
        seq_lens = torch.full((B,), L, dtype=torch.int32, device=device)
    else:
        seq_lens = torch.as_tensor(seq_lens, dtype=torch.int32, device=device)
    return q, kc, vc, gates, seq_lens


def phi_weights(hkv: int, l: int = 32, seed: int = 0, device="cpu"):
    """Weights of the learnable compression, phi_k and phi_v [hkv, l] fp32: (1 + N(0, 0.25)) / l,
    a perturbed mean."""
    g = _gen(seed, device)
    wk = (1.0 + 0.5 * torch.randn((hkv, l), generator=g, device=device)) / l
    wv = (1.0 + 0.5 * torch.randn((hkv, l), generator=g, device=device)) / l
    return wk.contiguous(), wv.contiguous()


def gate_weights(dim: int, seed: int = 0, device="cpu"):
    """Gate-network weights: W1 [dim/2, dim] bf16 ~ N(0, 1/dim); b1 [dim/2] ~ N(0, 0.01);
    W2 [3, dim/2] ~ N(0, 2/dim); b2 [3] ~ N(0, 0.01) (fp32)."""
    g = _gen(seed, device)
    hid = dim // 2
    w1 = (torch.randn((hid, dim), generator=g, device=device) / dim ** 0.5).to(torch.bfloat16)
    b1 = torch.randn((hid,), generator=g, device=device) * 0.1
    w2 = torch.randn((3, hid), generator=g, device=device) / hid ** 0.5
    b2 = torch.randn((3,), generator=g, device=device) * 0.1
    return w1, b1, w2, b2


def bf16_bits(t: torch.Tensor):
    """Raw 16-bit patterns of a bf16 tensor as a numpy uint16 array (host copy)."""
    import numpy as np

    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
