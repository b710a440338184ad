"""GPU parity of the prefill backward (nsa_backward through the C ABI) against the fp64 oracle.

The selection is an input of the backward: both sides use the one the GPU forward chose.
Tolerance, per gradient tensor, relative to its largest reference magnitude M:
max-abs error <= 1e-2 M and mean-abs error <= 1e-3 M. The kernels round P (times the gate)
and dS to bf16 as tensor-core operands (2^-9 relative each) and accumulate in fp32, so an
element's error stays below about 2^-8 of the sum of its terms' magnitudes; with the
cancellation in dS = P (dP - <dO, o>) that sum can exceed the element itself several-fold.
"""
import numpy as np
import pytest
import torch

from oracle import backward as bwd_orc
from oracle import oracle as orc
from sparse_attention_long_fwd_b200 import nsa
from sparse_attention_long_fwd_b200.inputs import WORKLOADS, bf16_bits, phi_weights, prefill_inputs, scaled

from nsa_check import run_prefill

pytestmark = pytest.mark.gpu
DEV = "cuda"
REL_MAX = 1e-2
REL_MEAN = 1e-3


def _grad_close(got, ref, what):
    got = got.detach().cpu().numpy().astype(np.float64) if torch.is_tensor(got) else got
    m = max(float(np.abs(ref).max()), 1e-30)
    err = np.abs(got - ref)
    assert np.isfinite(got).all(), f"{what}: non-finite"
    mx, mn = float(err.max()) / m, float(err.mean()) / m
    assert mx <= REL_MAX and mn <= REL_MEAN, f"{what}: max {mx:.3e} mean {mn:.3e} (relative to {m:.3e})"
    return round(mx, 6), round(mn, 7)


def _run(w, seed, phi=None, saved=False):
    """saved: False (the backward recomputes every statistic), True (the forward's compressed-branch
    statistics) or "keep" (the forward keeps every branch's statistics for the backward)."""
    keep = saved == "keep"
    q, k, v, g = prefill_inputs(w, seed=seed, device=DEV)
    out, sel, ws, lay = run_prefill(w, q, k, v, g, phi=phi, keep=keep)
    gen = torch.Generator(device=DEV).manual_seed(seed + 100)
    d_out = torch.randn((w.n_tokens, w.hq, w.d), generator=gen, device=DEV).to(torch.bfloat16)
    sel_arg = sel if w.n_video > 0 else torch.zeros(1, dtype=torch.int32, device=DEV)
    dq, dk, dv, dgates = nsa.backward(q, k, v, g, d_out, sel_arg, n_video=w.n_video, top_n=w.top_n,
                                      window=w.window, phi=phi, fwd_workspace=ws if saved else None,
                                      keep_branch_stats=keep)
    torch.cuda.synchronize()
    assert nsa.nsa_get_device_error(clear=True) == 0
    return q, k, v, g, d_out, sel, (dq, dk, dv, dgates)


def _compare(w, q, k, v, g, d_out, sel, grads, phi=None):
    cfg = orc.OracleConfig(w.n_tokens, w.n_video, w.hq, w.hkv, w.d, w.cmp_len, w.cmp_stride, w.sel_len, w.top_n,
                           w.window)
    pk, pv = (None, None) if phi is None else (phi[0].cpu().numpy(), phi[1].cpu().numpy())
    ref = bwd_orc.prefill_backward(cfg, bf16_bits(q), bf16_bits(k), bf16_bits(v), g.cpu().numpy(), bf16_bits(d_out),
                                   sel.cpu().numpy()[: w.n_video], pk, pv)
    stats = {}
    for name, got in zip(("dq", "dk", "dv", "dgates"), grads):
        stats[name] = _grad_close(got, ref[name], name)
    return stats


@pytest.mark.parametrize("name,n,nv,hq,hkv,d,top_n,window", [
    ("tiny", None, None, None, None, None, None, None),
    ("v128k", 1000, 1000, 28, 4, 128, 16, 512),      # G = 7, several tiles, ragged tail
    ("v128k", 777, 777, 8, 1, 64, 5, 100),            # G = 8, d = 64, short window
    ("qwen36k_hybrid", 1200, 1000, 28, 4, 128, 16, 512),  # trailing text rows (dense branch)
    ("v128k", 300, 0, 4, 2, 64, 4, 64),               # all text
    ("v128k", 40, 40, 4, 2, 128, 3, 16),              # shorter than two compression blocks
    ("v128k", 600, 600, 48, 4, 128, 16, 256),         # G = 12: one token per warp in the row pass
    ("qwen36k_hybrid", 520, 450, 32, 2, 64, 12, 128),  # G = 16, d = 64, with text rows
    ("v128k", 4300, 4300, 8, 2, 64, 8, 64),           # 267 compressed blocks: three 128-key tiles
])
@pytest.mark.parametrize("saved", [False, True, "keep"])
def test_backward_every_element(name, n, nv, hq, hkv, d, top_n, window, saved):
    """saved: see _run; "keep" with d = 128 runs every video row on the tensor-core kernels."""
    w = WORKLOADS[name] if n is None else scaled(WORKLOADS[name], n_tokens=n, n_video=nv, hq=hq, hkv=hkv, d=d,
                                                    top_n=top_n, window=window)
    q, k, v, g, d_out, sel, grads = _run(w, seed=21, saved=saved)
    sel = sel if w.n_video > 0 else torch.zeros((0, w.hkv, w.top_n), dtype=torch.int32)
    print(_compare(w, q, k, v, g, d_out, sel, grads))


@pytest.mark.parametrize("saved", [True, "keep"])
def test_backward_learnable_compression(saved):
    w = scaled(WORKLOADS["v128k"], n_tokens=900, n_video=900)
    phi = phi_weights(w.hkv, 32, seed=22, device=DEV)
    q, k, v, g, d_out, sel, grads = _run(w, seed=23, phi=phi, saved=saved)
    print(_compare(w, q, k, v, g, d_out, sel, grads, phi=phi))


def test_backward_kept_statistics_agree_with_recomputed():
    """The two saved modes differ only in where the statistics come from; at a size past the
    oracle's reach (several 128-key tiles in every branch) their gradients agree to the
    tolerance of the bf16 operands."""
    w = scaled(WORKLOADS["v16k"], n_tokens=6000, n_video=6000)
    a = _run(w, seed=25, saved=True)[-1]
    b = _run(w, seed=25, saved="keep")[-1]
    for name, x, y in zip(("dq", "dk", "dv", "dgates"), a, b):
        _grad_close(y, x.detach().cpu().numpy().astype(np.float64), name)


def test_backward_sum_identities_at_16k():
    """At any size: the key gradients of each group sum to zero (the dS of a row sum to
    zero and the mean's weights sum to one), and the value gradients sum to the dO of each
    row weighted by the gates of its non-empty branches."""
    w = WORKLOADS["v16k"]
    q, k, v, g, d_out, sel, (dq, dk, dv, dgates) = _run(w, seed=24, saved="keep")
    G = w.hq // w.hkv
    do = d_out.double()
    rows = torch.arange(w.n_tokens, device=DEV)
    wgt = g.double()[..., 0] * (rows >= w.cmp_len - 1)[:, None] + g.double()[..., 1] + g.double()[..., 2]
    for grp in range(w.hkv):
        hs = slice(grp * G, (grp + 1) * G)
        want = (wgt[:, hs, None] * do[:, hs]).sum(dim=(0, 1))
        got = dv[:, grp].double().sum(0)
        assert (got - want).abs().max().item() <= 5e-3 * want.abs().max().item() + 5e-2
        ksum = dk[:, grp].double().sum(0)
        assert ksum.abs().max().item() <= 1e-3 * dk[:, grp].double().abs().sum(0).max().item()
    assert torch.isfinite(dq).all() and torch.isfinite(dgates).all()
