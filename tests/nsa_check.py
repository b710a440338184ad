"""Comparison helpers shared by the GPU parity tests (test infrastructure)."""
from __future__ import annotations

import numpy as np
import torch

from oracle import oracle as orc
from sparse_attention_long_fwd_b200 import nsa
from sparse_attention_long_fwd_b200.inputs import Workload, bf16_bits

# Acceptance: fp32 outputs within max-abs 1e-2 and mean-abs 1e-3 of the fp64 oracle for
# N(0,1) inputs; selected blocks identical except where the oracle's own scores of the
# differing blocks are within a relative 1e-3 of each other (a near-tie), in which case
# the oracle is re-run with the GPU's selection and the output must still match.
MAX_ABS = 1e-2
MEAN_ABS = 1e-3
TIE_REL = 1e-3


def oracle_cfg(w: Workload) -> orc.OracleConfig:
    return orc.OracleConfig(w.n_tokens, w.n_video, w.hq, w.hkv, w.d, w.cmp_len, w.cmp_stride, w.sel_len, w.top_n,
                            w.window)


def run_prefill(w: Workload, q, k, v, gates, out_dtype=torch.float32, phi=None, keep=False):
    """Call nsa_prefill (nsa_prefill_phi when phi = (phi_k, phi_v) is given) through the C ABI;
    returns (out, sel, workspace, layout). keep: the workspace also keeps the selected and window
    branches' statistics."""
    p = nsa.make_params(w.n_tokens, w.n_video, w.hq, w.hkv, w.d, w.cmp_len, w.cmp_stride, w.sel_len, w.top_n,
                        w.window, out_dtype=nsa.NSA_OUT_F32 if out_dtype == torch.float32 else nsa.NSA_OUT_BF16,
                        keep_branch_stats=keep)
    ws = nsa.alloc_workspace(p, False, q.device)
    out = torch.empty((w.n_tokens, w.hq, w.d), dtype=out_dtype, device=q.device)
    sel = torch.full((max(w.n_video, 1), w.hkv, w.top_n), -7, dtype=torch.int32, device=q.device)
    sel_arg = sel if w.n_video > 0 else None
    if phi is None:
        rc = nsa.nsa_prefill(q, k, v, gates, p, out, sel_arg, ws, ws.numel())
    else:
        rc = nsa.nsa_prefill_phi(q, k, v, gates, phi[0], phi[1], p, out, sel_arg, ws, ws.numel())
    assert rc == nsa.NSA_OK, nsa.nsa_error_string(rc)
    torch.cuda.synchronize()
    assert nsa.nsa_get_device_error(clear=True) == 0
    return out, sel[: w.n_video], ws, nsa.nsa_prefill_workspace_layout(p)


def ws_view(ws: torch.Tensor, off: int, shape, dtype) -> torch.Tensor:
    n = int(np.prod(shape)) * torch.tensor([], dtype=dtype).element_size()
    return ws[off: off + n].view(dtype).view(*shape)


def host_bits(*ts):
    return [bf16_bits(t) for t in ts]


def check_selection(gpu_sel: np.ndarray, ora_sel: np.ndarray, ora_scores: np.ndarray):
    """Returns (row indices needing replay, number of near-tie (row, group) pairs). Asserts
    that every mismatch is a near-tie under the oracle's scores."""
    replay, ties = [], 0
    for r in range(gpu_sel.shape[0]):
        row_bad = False
        for g in range(gpu_sel.shape[1]):
            a = gpu_sel[r, g]
            b = ora_sel[r, g]
            if np.array_equal(a, b):
                continue
            A = sorted(set(int(x) for x in a if x >= 0) - set(int(x) for x in b if x >= 0))
            B = sorted(set(int(x) for x in b if x >= 0) - set(int(x) for x in a if x >= 0))
            assert len(A) == len(B) and len(A) > 0, (r, g, a, b)
            sc = ora_scores[r, g]
            for x in A:
                for y in B:
                    assert abs(sc[x] - sc[y]) <= TIE_REL * max(sc[x], sc[y]), (r, g, x, y, sc[x], sc[y])
            ties += 1
            row_bad = True
        if row_bad:
            replay.append(r)
    return replay, ties


def assert_close(got: np.ndarray, ref: np.ndarray, what: str, max_abs=MAX_ABS, mean_abs=MEAN_ABS):
    err = np.abs(got.astype(np.float64) - ref)
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    mx, mn = float(err.max()) if err.size else 0.0, float(err.mean()) if err.size else 0.0
    assert mx <= max_abs and mn <= mean_abs, f"{what}: max-abs {mx:.3e} mean-abs {mn:.3e}"
    return mx, mn


def compare_prefill_rows(w: Workload, q, k, v, gates, rows, out, sel, ws, layout, check_intermediates=True,
                         nthreads=0, phi=None):
    """Element-wise comparison of the listed rows against the oracle (plus replay on near-ties).
    phi = (phi_k, phi_v) selects the oracle's learnable compression."""
    qb, kb, vb = host_bits(q, k, v)
    g = gates.detach().cpu().numpy()
    rows = np.asarray(rows, dtype=np.int32)
    cfg = oracle_cfg(w)
    if phi is None:
        kc_o = orc.compress(kb[: w.n_video])
        vc_o = orc.compress(vb[: w.n_video])
    else:
        kc_o = orc.compress_weighted(kb[: w.n_video], phi[0].cpu().numpy())
        vc_o = orc.compress_weighted(vb[: w.n_video], phi[1].cpu().numpy())
    o = orc.prefill_rows(cfg, qb, kb, vb, g, rows, kc=kc_o, vc=vc_o, nthreads=nthreads)
    vid = rows < w.n_video
    vrows = rows[vid]
    stats = {"rows": len(rows), "ties": 0}
    if check_intermediates and w.n_video > 0:
        nc = layout["n_cmp"]
        if nc > 0:
            kc_g = bf16_bits(ws_view(ws, layout["kc"], (nc, w.hkv, w.d), torch.bfloat16))
            vc_g = bf16_bits(ws_view(ws, layout["vc"], (nc, w.hkv, w.d), torch.bfloat16))
            assert np.array_equal(kc_g, kc_o) and np.array_equal(vc_g, vc_o), "compressed K/V not bit-exact"
        if len(vrows):
            ocmp = ws_view(ws, layout["o_cmp"], (w.n_video, w.hq, w.d), torch.float16)[vrows].float().cpu().numpy()
            stats["o_cmp"] = assert_close(ocmp, o["o_cmp"][vid], "o_cmp")
            owin = ws_view(ws, layout["o_win"], (w.n_video, w.hq, w.d), torch.float16)[vrows].float().cpu().numpy()
            stats["o_win"] = assert_close(owin, o["o_win"][vid], "o_win")
            lse = ws_view(ws, layout["lse"], (w.n_video, w.hq), torch.float32)[vrows].cpu().numpy()
            fin = np.isfinite(o["lse"][vid])
            assert np.array_equal(np.isfinite(lse), fin)
            if fin.any():
                assert np.abs(lse[fin] - o["lse"][vid][fin]).max() < 1e-3
            nsel = layout["n_sel"]
            sc = ws_view(ws, layout["scores"], (w.n_video, w.hkv, layout["score_stride"]),
                         torch.float32)[vrows, :, :nsel].cpu().numpy()
            for i, t in enumerate(vrows):
                jt = t // w.sel_len
                ref = o["scores"][vid][i][:, : jt + 1]
                assert np.abs(sc[i][:, : jt + 1] - ref).max() <= 1e-5 + 1e-4 * np.abs(ref).max(), f"scores row {t}"
    out_h = out.float()[rows].cpu().numpy()
    ref = o["out"].copy()
    if len(vrows):
        gsel = sel[vrows].cpu().numpy()
        replay, ties = check_selection(gsel, o["sel"][vid], o["scores"][vid])
        stats["ties"] = ties
        vidx = np.nonzero(vid)[0]
        if replay:
            rr = vrows[replay]
            o2 = orc.prefill_rows(cfg, qb, kb, vb, g, rr, kc=kc_o, vc=vc_o, sel_override=gsel[replay],
                                  want=("o_sel",), nthreads=nthreads)
            ref[vidx[replay]] = o2["out"]
    if out.dtype == torch.float32:
        stats["out"] = assert_close(out_h, ref, "out")
    else:
        # bf16 output: within one bf16 ulp of the oracle or inside the fp32 tolerance
        err = np.abs(out_h - ref)
        ulp = np.abs(ref) * 2.0 ** -7 + 1e-30
        assert np.all((err <= ulp) | (err <= MAX_ABS)), "bf16 out"
        stats["out"] = (float(err.max()), float(err.mean()))
    return stats


def sample_rows(n_video: int, n_tokens: int, n_random: int, seed: int = 0):
    """First 64 tokens, tokens around early block boundaries, the last 512 video tokens
    (strided), some text rows, and random rows."""
    rng = np.random.default_rng(seed)
    rows = set(range(min(64, n_video)))
    for b in (31, 32, 47, 48, 63, 64, 127, 128, 129, 191, 255, 256, 511, 512, 1023, 2047, 2048, 2079):
        if b < n_video:
            rows.add(b)
    rows.update(range(max(0, n_video - 512), n_video, 37))
    if n_video > 0:
        rows.add(n_video - 1)
        rows.update(int(x) for x in rng.integers(0, n_video, n_random))
    if n_tokens > n_video:
        rows.update(range(n_video, n_tokens, max(1, (n_tokens - n_video) // 16)))
        rows.add(n_tokens - 1)
    return np.array(sorted(rows), dtype=np.int32)
