"""fp64 oracle of the gate network that mixes the three NSA branches.

TEST INFRASTRUCTURE ONLY: imported by tests/, by ``__graft_entry__.smoke()`` and by the
CPU-baseline leg of ``bench.py``. It shares no code with the CUDA package.

What it computes follows the CSDN blog "VideoNSA：重新定义视频理解的稀疏注意力机制"
(vcloud.csdn.net), section 3.1 "动态门控机制详解":
  - every attention head gets three gates (compressed, selected, window), normalised by a
    softmax so that they sum to one;
  - the gates come from a small MLP: a linear map from dim to dim/2, an exact (erf) GELU,
    a linear map from dim/2 to 3, then the softmax;
  - the blog's module averages its input over the token axis first, giving one gate triple
    per (sequence, head).
Readings where the blog is silent:
  - the MLP's input for head h is that head's own feature vector (dim = head_dim), and one
    set of weights serves every head (the blog builds a single module);
  - ``gate_mlp`` applies the MLP to every (token, head) row without the average, the
    per-token gating that feeds a prefill's [N][Hq][3] gate tensor;
    ``gate_mlp_pooled`` is the blog's averaged form.
Weights use the linear-layer layout [out][in]; W1 holds bf16 values (the tensor-core
operand), b1, W2 and b2 are fp32, all widened exactly to fp64.
"""
from __future__ import annotations

import math

import numpy as np

from .oracle import bf16_bits_to_f64

_erf = np.vectorize(math.erf, otypes=[np.float64])


def gelu(x: np.ndarray) -> np.ndarray:
    """Exact GELU, x * Phi(x) with Phi the standard normal CDF written through erf."""
    x = np.asarray(x, dtype=np.float64)
    return 0.5 * x * (1.0 + _erf(x / math.sqrt(2.0)))


def softmax(z: np.ndarray) -> np.ndarray:
    """Softmax over the last axis, shifted by the row maximum."""
    z = np.asarray(z, dtype=np.float64)
    e = np.exp(z - z.max(axis=-1, keepdims=True))
    return e / e.sum(axis=-1, keepdims=True)


def _weights(w1_bits, b1, w2, b2):
    w1 = bf16_bits_to_f64(w1_bits)
    hid, dim = w1.shape
    if dim != 2 * hid:
        raise ValueError(f"W1 must be [dim/2, dim], got {w1.shape}")
    b1 = np.asarray(b1, dtype=np.float32).astype(np.float64)
    w2 = np.asarray(w2, dtype=np.float32).astype(np.float64)
    b2 = np.asarray(b2, dtype=np.float32).astype(np.float64)
    if b1.shape != (hid,) or w2.shape != (3, hid) or b2.shape != (3,):
        raise ValueError("b1 [dim/2], W2 [3, dim/2], b2 [3] expected")
    return w1, b1, w2, b2


def mlp_gates(x: np.ndarray, w1_bits, b1, w2, b2) -> np.ndarray:
    """softmax(W2 . GELU(W1 . x + b1) + b2) for every row of x [R, dim] (fp64 values)."""
    w1, b1, w2, b2 = _weights(w1_bits, b1, w2, b2)
    x = np.asarray(x, dtype=np.float64)
    hidden = gelu(x @ w1.T + b1)
    return softmax(hidden @ w2.T + b2)


def gate_mlp(x_bits: np.ndarray, w1_bits, b1, w2, b2) -> np.ndarray:
    """Per-row gates: x [..., dim] bf16 bits -> [..., 3] fp64 (one row per token and head)."""
    x = bf16_bits_to_f64(x_bits)
    lead = x.shape[:-1]
    return mlp_gates(x.reshape(-1, x.shape[-1]), w1_bits, b1, w2, b2).reshape(*lead, 3)


def gate_mlp_pooled(x_bits: np.ndarray, w1_bits, b1, w2, b2) -> np.ndarray:
    """The blog's averaged form: x [B, T, H, dim] bf16 bits -> gates [B, H, 3] fp64, the MLP
    applied to each (sequence, head) mean over the T tokens."""
    x = bf16_bits_to_f64(x_bits)
    if x.ndim != 4:
        raise ValueError("x must be [B, T, H, dim]")
    mean = x.mean(axis=1)
    B, H, dim = mean.shape
    return mlp_gates(mean.reshape(B * H, dim), w1_bits, b1, w2, b2).reshape(B, H, 3)
