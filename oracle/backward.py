"""fp64 oracle of the NSA prefill backward pass (gradients of the forward in nsa_oracle.c).

TEST INFRASTRUCTURE ONLY: imported by tests/ and by the CPU-baseline leg of ``bench.py``.
It shares no code with the CUDA package.

The pages train the model end to end (shd-paper.top page "VideoNSA: Native Sparse
Attention Scales Video Understanding", abstract: end-to-end training on 216K video
instructions), so the forward has a backward. They do not spell it out; this is the
gradient of the forward the oracle computes, with these readings:
  - the selection (which blocks each (token, group) attends) is held constant: block
    indices are not differentiable, so the block scores get no gradient;
  - the compressed keys and values are the bf16-rounded summaries the forward used, and
    the rounding passes gradients unchanged: d Kc[i] flows to the l tokens of block i
    with the compression's weights (1/l for the mean, phi[g][u] for the learnable form);
  - trailing text rows (t >= n_video) are dense causal attention with no gates.
For one row (token t, head h) and one branch with keys K_b, values V_b and gate g_b:
    P = softmax(scale * K_b q),  o_b = P V_b,  out = sum_b g_b o_b
    d g_b = <dO, o_b>;   dP_j = g_b <dO, v_j>;   dS_j = P_j (dP_j - g_b <dO, o_b>)
    dq += scale * sum_j dS_j k_j;   dk_j += scale * dS_j q;   dv_j += g_b P_j dO
Everything is evaluated in fp64 from the exact bf16 inputs.
"""
from __future__ import annotations

import math

import numpy as np

from . import oracle as orc


def _keysets(cfg: orc.OracleConfig, t: int, sel_row, ncmp_total: int):
    """Key index sets of row t: (cmp block indices, selected tokens, window tokens) for a
    video row, or (None, None, dense tokens) for a text row."""
    if t >= cfg.n_video:
        return None, None, np.arange(t + 1)
    nc = (t - cfg.cmp_len + 1) // cfg.cmp_stride + 1 if t >= cfg.cmp_len - 1 else 0  # blocks with i*s + l - 1 <= t
    cmp_idx = np.arange(min(nc, ncmp_total))
    toks = []
    for j in sel_row:
        if j < 0:
            continue
        lo, hi = j * cfg.sel_len, min((j + 1) * cfg.sel_len, t + 1)
        toks.extend(range(lo, hi))
    sel_idx = np.array(sorted(set(toks)), dtype=np.int64)
    win_idx = np.arange(max(0, t - cfg.window + 1), t + 1)
    return cmp_idx, sel_idx, win_idx


def _branch(Q, K, V, g, dO, scale):
    """One branch for the heads of one group. Q, dO [G, d]; K, V [n, d]; g [G].
    Returns o [G, d], dq [G, d], dK [n, d], dV [n, d], dg [G]."""
    G, d = Q.shape
    if K.shape[0] == 0:
        z = np.zeros((G, d))
        return z, z.copy(), np.zeros((0, d)), np.zeros((0, d)), np.zeros(G)
    s = scale * (Q @ K.T)
    p = np.exp(s - s.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    o = p @ V
    dg = np.einsum("gd,gd->g", dO, o)
    dOb = g[:, None] * dO
    dP = dOb @ V.T
    D = g * dg
    dS = p * (dP - D[:, None])
    dq = scale * dS @ K
    dK = scale * dS.T @ Q
    dV = p.T @ dOb
    return o, dq, dK, dV, dg


def compressed_f64(k: np.ndarray, cfg: orc.OracleConfig, phi=None, rounded: bool = True) -> np.ndarray:
    """Compressed keys (values) as fp64: the forward's bf16 summaries when `rounded`, else the
    exact weighted sums (a smooth function of k, for finite-difference checks). k [T, hkv, d]
    fp64 (rounded=False) or bf16 bits (rounded=True)."""
    if rounded:
        bits = orc.compress(k, cfg.cmp_len, cfg.cmp_stride) if phi is None else \
            orc.compress_weighted(k, phi, cfg.cmp_len, cfg.cmp_stride)
        return orc.bf16_bits_to_f64(bits)
    T, h, d = k.shape
    nc = orc.num_cmp(T, cfg.cmp_len, cfg.cmp_stride)
    w = np.full((h, cfg.cmp_len), 1.0 / cfg.cmp_len) if phi is None else np.asarray(phi, np.float64)
    out = np.zeros((max(nc, 0), h, d))
    for i in range(nc):
        blk = k[i * cfg.cmp_stride: i * cfg.cmp_stride + cfg.cmp_len]  # [l, h, d]
        out[i] = np.einsum("lh,lhd->hd", w.T, blk)
    return out


def forward_backward(cfg: orc.OracleConfig, q, k, v, gates, d_out, sel, kc=None, vc=None, phi_k=None, phi_v=None):
    """Forward outputs and gradients of one prefill.

    q [N, hq, d], k, v [N, hkv, d], d_out [N, hq, d]: fp64 arrays (widen bf16 inputs with
    orc.bf16_bits_to_f64); gates [N, hq, 3]; sel [n_video, hkv, top_n] block indices (-1
    padded). kc, vc: the compressed keys and values (fp64) the forward attended; phi_k, phi_v:
    the learnable compression's weights [hkv, l] for keys and values (None for the mean), used
    for the gradient's way back to the tokens.
    Returns dict(out, dq, dk, dv, dgates); dgates of text rows are 0."""
    q, k, v, d_out = (np.asarray(a, dtype=np.float64) for a in (q, k, v, d_out))
    gates = np.asarray(gates, dtype=np.float64)
    N, hq, d = q.shape
    hkv = k.shape[1]
    G = hq // hkv
    scale = cfg.scale if cfg.scale > 0 else 1.0 / math.sqrt(d)
    nv = cfg.n_video
    ncmp = kc.shape[0] if kc is not None else 0
    out = np.zeros_like(q)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    dkc = np.zeros((ncmp, hkv, d))
    dvc = np.zeros((ncmp, hkv, d))
    dgates = np.zeros((N, hq, 3))
    for t in range(N):
        for g in range(hkv):
            hs = slice(g * G, (g + 1) * G)
            Q, dO = q[t, hs], d_out[t, hs]
            cmp_idx, sel_idx, win_idx = _keysets(cfg, t, sel[t, g] if t < nv else (), ncmp)
            if cmp_idx is None:  # text row: dense, no gates
                o, dqq, dKb, dVb, _ = _branch(Q, k[win_idx, g], v[win_idx, g], np.ones(G), dO, scale)
                out[t, hs] = o
                dq[t, hs] += dqq
                dk[win_idx, g] += dKb
                dv[win_idx, g] += dVb
                continue
            for b, (src_k, src_v, idx, dks, dvs) in enumerate(
                    ((kc, vc, cmp_idx, dkc, dvc), (k, v, sel_idx, dk, dv), (k, v, win_idx, dk, dv))):
                gb = gates[t, hs, b]
                Kb = src_k[idx, g] if len(idx) else np.zeros((0, d))
                Vb = src_v[idx, g] if len(idx) else np.zeros((0, d))
                o, dqq, dKb, dVb, dg = _branch(Q, Kb, Vb, gb, dO, scale)
                out[t, hs] += gb[:, None] * o
                dq[t, hs] += dqq
                if len(idx):
                    np.add.at(dks, (idx, g), dKb)
                    np.add.at(dvs, (idx, g), dVb)
                dgates[t, hs, b] = dg
    # the compressed keys' gradient flows back to their tokens with the compression's weights
    mean = np.full((hkv, cfg.cmp_len), 1.0 / cfg.cmp_len)
    wk = mean if phi_k is None else np.asarray(phi_k, np.float64)
    wv = mean if phi_v is None else np.asarray(phi_v, np.float64)
    for i in range(ncmp):
        for u in range(cfg.cmp_len):
            tau = i * cfg.cmp_stride + u
            dk[tau] += wk[:, u, None] * dkc[i]
            dv[tau] += wv[:, u, None] * dvc[i]
    return {"out": out, "dq": dq, "dk": dk, "dv": dv, "dgates": dgates}


def prefill_backward(cfg: orc.OracleConfig, q_bits, k_bits, v_bits, gates, d_out_bits, sel, phi_k=None,
                     phi_v=None) -> dict:
    """Gradients of the prefill the forward oracle computes, on the exact bf16 inputs it
    consumed (uint16 bit patterns) and its bf16 compressed keys and values."""
    kb = np.ascontiguousarray(k_bits)[: cfg.n_video]
    vb = np.ascontiguousarray(v_bits)[: cfg.n_video]
    kc = compressed_f64(kb, cfg, phi_k)
    vc = compressed_f64(vb, cfg, phi_v)
    f = orc.bf16_bits_to_f64
    return forward_backward(cfg, f(q_bits), f(k_bits), f(v_bits), gates, f(d_out_bits), sel, kc, vc, phi_k, phi_v)
