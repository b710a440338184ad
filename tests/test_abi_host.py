"""Host-side checks of the C ABI that need no GPU: the library loads, exports every entry
point declared in include/nsa.h, validates arguments and reports error codes, and
computes consistent workspace layouts. No kernel is launched here."""
import ctypes
import os
import re

import pytest

from sparse_attention_long_fwd_b200 import nsa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    text = open(os.path.join(ROOT, "include", "nsa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(nsa_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    lib = nsa.load_library()
    declared = _declared_functions()
    assert "nsa_prefill" in declared and "nsa_decode" in declared and "nsa_compress" in declared
    for name in declared:
        assert hasattr(lib, name), name
    assert set(nsa.EXPORTED) <= set(declared)


def test_version_and_error_strings():
    assert "sm_100a" in nsa.nsa_version()
    for s in range(5):
        assert nsa.nsa_error_string(s)
    assert nsa.nsa_error_string(99) == "unknown status"


def _p(**kw):
    base = dict(n_tokens=4096, n_video=4096, num_q_heads=28, num_kv_heads=4, head_dim=128, top_n=16, window=512)
    base.update(kw)
    return nsa.make_params(**base)


@pytest.mark.parametrize("kw,code", [
    (dict(head_dim=96), nsa.NSA_ERR_UNSUPPORTED),
    (dict(num_q_heads=30), nsa.NSA_ERR_INVALID_ARG),          # Hq % Hkv != 0
    (dict(num_q_heads=68, num_kv_heads=4), nsa.NSA_ERR_UNSUPPORTED),  # G = 17 > 16
    (dict(top_n=0), nsa.NSA_ERR_INVALID_ARG),
    (dict(top_n=2), nsa.NSA_ERR_UNSUPPORTED),
    (dict(top_n=65), nsa.NSA_ERR_UNSUPPORTED),
    (dict(cmp_block=64), nsa.NSA_ERR_UNSUPPORTED),
    (dict(window=0), nsa.NSA_ERR_INVALID_ARG),
    (dict(n_video=5000), nsa.NSA_ERR_INVALID_ARG),
    (dict(n_tokens=0, n_video=0), nsa.NSA_ERR_INVALID_ARG),
])
def test_prefill_validation_codes(kw, code):
    p = _p(**kw)
    fake = 1 << 20  # never dereferenced: validation fails first
    assert nsa.nsa_prefill(fake, fake, fake, fake, p, fake, None, fake, 1 << 40, None) == code


def test_null_and_misaligned_pointers_rejected():
    p = _p()
    f = 1 << 20
    assert nsa.nsa_prefill(None, f, f, f, p, f, None, f, 1 << 40, None) == nsa.NSA_ERR_INVALID_ARG
    assert nsa.nsa_prefill(f + 2, f, f, f, p, f, None, f, 1 << 40, None) == nsa.NSA_ERR_INVALID_ARG
    assert nsa.nsa_prefill(f, f, f, f, p, f, None, f + 16, 1 << 40, None) == nsa.NSA_ERR_INVALID_ARG
    assert nsa.nsa_prefill(f, f, f, f, p, f, None, f, 1000, None) == nsa.NSA_ERR_WORKSPACE_TOO_SMALL
    pd = nsa.make_params(1024, batch=0)
    assert nsa.nsa_decode(f, f, f, f, f, f, f, pd, f, None, f, 1 << 40, None) == nsa.NSA_ERR_INVALID_ARG
    pd = nsa.make_params(1024, batch=2, window=5000)
    assert nsa.nsa_decode(f, f, f, f, f, f, f, pd, f, None, f, 1 << 40, None) == nsa.NSA_ERR_UNSUPPORTED
    assert nsa.nsa_compress(None, f, nsa.make_params(64, batch=1), f, f, None) == nsa.NSA_ERR_INVALID_ARG


def test_prefill_layout_is_aligned_and_disjoint():
    for n, nv in ((131072, 131072), (36352, 36096), (2048, 2048), (300, 0), (20, 20)):
        p = _p(n_tokens=n, n_video=nv)
        lay = nsa.nsa_prefill_workspace_layout(p)
        assert lay["total"] == nsa.nsa_workspace_size(p, False)
        ncmp = (nv - 32) // 16 + 1 if nv >= 32 else 0
        assert lay["n_cmp"] == ncmp and lay["n_sel"] == (nv + 63) // 64
        # score rows are 16-byte aligned: the stride is n_sel rounded up to a multiple of 4
        assert lay["score_stride"] % 4 == 0 and 0 <= lay["score_stride"] - lay["n_sel"] < 4
        keys = ["kc", "vc", "o_cmp", "lse", "scores", "sel_idx", "o_win"]
        offs = [lay[k] for k in keys] + [lay["total"]]
        assert all(o % 256 == 0 for o in offs)
        sizes = [max(ncmp, 1) * 4 * 128 * 2] * 2 + [nv * 28 * 128 * 2, nv * 28 * 4,
                                                    nv * 4 * max(lay["score_stride"], 4) * 4,
                                                    nv * 4 * 16 * 4, nv * 28 * 128 * 2]
        for i, sz in enumerate(sizes):
            assert offs[i] + sz <= offs[i + 1], keys[i]


def test_kept_branch_statistics_layout():
    nv = 5000
    p0 = nsa.make_params(nv)
    p1 = nsa.make_params(nv, keep_branch_stats=True)
    l0, l1 = nsa.nsa_prefill_workspace_layout(p0), nsa.nsa_prefill_workspace_layout(p1)
    assert l0["o_sel"] == l0["lse_sel"] == l0["lse_win"] == 0
    # the kept arrays follow everything else, 256-byte aligned, and do not overlap
    offs = [l1["o_sel"], l1["lse_sel"], l1["lse_win"], l1["total"]]
    sizes = [nv * 28 * 128 * 2, nv * 28 * 4, nv * 28 * 4]
    assert offs[0] >= l0["total"] and all(o % 256 == 0 for o in offs)
    for i, sz in enumerate(sizes):
        assert offs[i] + sz <= offs[i + 1]
    assert {k: l1[k] for k in ("kc", "o_cmp", "o_win", "scores")} == {k: l0[k] for k in ("kc", "o_cmp", "o_win", "scores")}
    # the backward keeps the selected branch's dq partials (d = 128 only)
    assert nsa.nsa_backward_workspace_size(p1) > nsa.nsa_backward_workspace_size(p0)
    p64 = nsa.make_params(nv, head_dim=64)
    p64k = nsa.make_params(nv, head_dim=64, keep_branch_stats=True)
    assert nsa.nsa_backward_workspace_size(p64k) == nsa.nsa_backward_workspace_size(p64)
    bad = nsa.make_params(nv)
    bad.keep_branch_stats = 2
    assert nsa.nsa_workspace_size(bad, False) == 0


def test_decode_workspace_scales_with_batch():
    a = nsa.nsa_workspace_size(nsa.make_params(131072, batch=1), True)
    b = nsa.nsa_workspace_size(nsa.make_params(131072, batch=64), True)
    assert 0 < a < b
    assert nsa.nsa_workspace_size(nsa.make_params(131072, head_dim=80, batch=64), True) == 0


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(nsa.NsaLibraryError):
        nsa._lib_saved = nsa._lib
        try:
            nsa._lib = None
            nsa.load_library(str(tmp_path / "absent.so"))
        finally:
            nsa._lib = nsa._lib_saved


@pytest.mark.parametrize("cu,nv,code", [
    ([0, 100, 4096], [100, 3000], nsa.NSA_OK),              # well formed (stops at the device check)
    ([1, 100, 4096], [99, 100], nsa.NSA_ERR_INVALID_ARG),   # does not start at 0
    ([0, 200, 100, 4096], [10, 0, 10], nsa.NSA_ERR_INVALID_ARG),  # decreasing
    ([0, 100, 4000], [100, 100], nsa.NSA_ERR_INVALID_ARG),  # does not end at n_tokens
    ([0, 100, 4096], [101, 100], nsa.NSA_ERR_INVALID_ARG),  # video prefix longer than its sequence
    ([0, 100, 4096], [-1, 100], nsa.NSA_ERR_INVALID_ARG),
])
def test_prefill_varlen_validation(cu, nv, code):
    p = _p()
    f = 1 << 20
    rc = nsa.nsa_prefill_varlen(f, f, f, f, cu, nv, p, f, None, f, 1 << 40, None)
    if code == nsa.NSA_OK:
        assert rc not in (nsa.NSA_ERR_INVALID_ARG, nsa.NSA_ERR_WORKSPACE_TOO_SMALL)  # only the device check fails here
        assert nsa.nsa_prefill_varlen_workspace_size(p, cu, nv) > 0
    else:
        assert rc == code
        assert nsa.nsa_prefill_varlen_workspace_size(p, cu, nv) == 0


def test_prefill_varlen_workspace_is_that_of_its_packed_segments():
    """A varlen batch is the packed batch whose sequences are a video prefix and trailing text;
    its one-grid workspace holds the whole batch's video stream."""
    p = _p(n_tokens=5000)
    cu, nv = [0, 700, 700, 2200, 5000], [600, 0, 1500, 2800]
    need = nsa.nsa_prefill_varlen_workspace_size(p, cu, nv)
    assert need == nsa.nsa_prefill_packed_workspace_size(p, cu, [600, 100, 1500, 2800], [1, 0, 1, 1])
    single = max(nsa.nsa_workspace_size(_p(n_tokens=cu[b + 1] - cu[b], n_video=nv[b]), 0)
                 for b in range(4) if cu[b + 1] > cu[b])
    assert need >= single
    f = 1 << 20
    assert nsa.nsa_prefill_varlen(f, f, f, f, cu, nv, p, f, None, f, need - 1, None) == nsa.NSA_ERR_WORKSPACE_TOO_SMALL


def test_learnable_compression_and_gate_validation():
    f = 1 << 20
    p = _p()
    pc = nsa.make_params(64, batch=1)
    # learnable compression: both weight arrays are required and 4-byte aligned
    assert nsa.nsa_compress_weighted(f, f, None, f, pc, f, f, None) == nsa.NSA_ERR_INVALID_ARG
    assert nsa.nsa_compress_weighted(f, f, f, f + 2, pc, f, f, None) == nsa.NSA_ERR_INVALID_ARG
    assert nsa.nsa_prefill_phi(f, f, f, f, None, f, p, f, None, f, 1 << 40, None) == nsa.NSA_ERR_INVALID_ARG
    assert nsa.nsa_prefill_phi(f, f, f, f, f, f, p, f, None, f, 1000, None) == nsa.NSA_ERR_WORKSPACE_TOO_SMALL
    # gate MLP
    assert nsa.nsa_gate_mlp(f, f, f, f, f, 100, 128, None, None) == nsa.NSA_ERR_INVALID_ARG
    assert nsa.nsa_gate_mlp(f + 8, f, f, f, f, 100, 128, f, None) == nsa.NSA_ERR_INVALID_ARG
    assert nsa.nsa_gate_mlp(f, f, f, f, f, -1, 128, f, None) == nsa.NSA_ERR_INVALID_ARG
    assert nsa.nsa_gate_mlp(f, f, f, f, f, 100, 96, f, None) == nsa.NSA_ERR_UNSUPPORTED
    assert nsa.nsa_gate_mlp(f, f, f, f, f, 0, 128, f, None) == nsa.NSA_OK  # nothing to do, nothing enqueued
    # averaged gate: workspace sizing and checks
    need = nsa.nsa_gate_mlp_pooled_workspace_size(2, 131072, 28, 128)
    assert need > 0 and need % 256 == 0 and need <= 8 * 1184 * 28 * 128 + 256
    assert nsa.nsa_gate_mlp_pooled_workspace_size(0, 10, 28, 128) == 0
    assert nsa.nsa_gate_mlp_pooled_workspace_size(1, 10, 28, 96) == 0
    assert nsa.nsa_gate_mlp_pooled(f, f, f, f, f, 2, 131072, 28, 128, 1, f, f, need - 1, None) == \
        nsa.NSA_ERR_WORKSPACE_TOO_SMALL
    assert nsa.nsa_gate_mlp_pooled(f, f, f, f, f, 2, 131072, 28, 128, 0, f, f, need, None) == nsa.NSA_ERR_INVALID_ARG
    assert nsa.nsa_gate_mlp_pooled(f, f, f, f, f, 1, 100, 28, 96, 1, f, f, 1 << 30, None) == nsa.NSA_ERR_UNSUPPORTED


def test_backward_validation():
    f = 1 << 20
    p = _p()
    need = nsa.nsa_backward_workspace_size(p)
    assert need > 0 and need % 256 == 0
    ok_args = [f] * 6 + [None, 0, None, None, p] + [f] * 5
    assert nsa.nsa_backward(*ok_args, need - 1, None) == nsa.NSA_ERR_WORKSPACE_TOO_SMALL
    bad = list(ok_args)
    bad[5] = None  # the forward's selection is required when there are video rows
    assert nsa.nsa_backward(*bad, need, None) == nsa.NSA_ERR_INVALID_ARG
    bad = list(ok_args)
    bad[8] = f  # phi_k without phi_v
    assert nsa.nsa_backward(*bad, need, None) == nsa.NSA_ERR_INVALID_ARG
    bad = list(ok_args)
    bad[11] = f + 4  # dq misaligned
    assert nsa.nsa_backward(*bad, need, None) == nsa.NSA_ERR_INVALID_ARG
    bad = list(ok_args)
    bad[6] = f + 128  # the forward's workspace must be 256-byte aligned
    bad[7] = 1 << 40
    assert nsa.nsa_backward(*bad, need, None) == nsa.NSA_ERR_INVALID_ARG
    # the forward's workspace must hold the layout of these params: one from a call without
    # keep_branch_stats is too small for a backward with it
    fwd_plain = nsa.nsa_workspace_size(p, False)
    pk = _p()
    pk.keep_branch_stats = 1
    fwd_keep = nsa.nsa_workspace_size(pk, False)
    assert fwd_keep > fwd_plain
    need_k = nsa.nsa_backward_workspace_size(pk)
    args = [f] * 6 + [f, fwd_plain, None, None, pk] + [f] * 5
    assert nsa.nsa_backward(*args, need_k, None) == nsa.NSA_ERR_WORKSPACE_TOO_SMALL
    assert nsa.nsa_backward_workspace_size(_p(head_dim=96)) == 0


def test_gate_kernel_erf_constants_meet_their_published_bound():
    """The gate kernel's erf follows Abramowitz & Stegun 7.1.26, |error| <= 1.5e-7. Read the
    constants from the kernel source and evaluate the formula in float64 against math.erf,
    so a mistyped digit fails here even where the gate tolerance would hide it."""
    import math

    src = open(os.path.join(ROOT, "sparse_attention_long_fwd_b200", "csrc", "gate.cuh")).read()
    body = src[src.index("float erf_as7126(float x)"):]
    body = body[: body.index("\n}\n")]
    consts = [float(c) for c in re.findall(r"(-?\d+\.\d+)f", body) if float(c) != 1.0]
    # in source order (the 1.0 literals aside): p, then the Horner coefficients a5 .. a1, then log2(e)
    p, a5, a4, a3, a2, a1, log2e = consts
    assert abs(log2e - 1 / math.log(2)) < 1e-12
    worst = 0.0
    for i in range(6001):
        x = i * 1e-3
        t = 1.0 / (1.0 + p * x)
        poly = ((((a5 * t + a4) * t + a3) * t + a2) * t + a1) * t
        worst = max(worst, abs(1.0 - poly * math.exp(-x * x) - math.erf(x)))
    assert worst <= 1.5e-7, worst


def test_selftest_budget_validated_before_any_launch():
    # limits outside 1 .. 4e9 cycles are rejected on the host, before the device is touched
    assert nsa.nsa_selftest_wait_timeout(0) == nsa.NSA_ERR_INVALID_ARG
    assert nsa.nsa_selftest_wait_timeout(-5) == nsa.NSA_ERR_INVALID_ARG
    assert nsa.nsa_selftest_wait_timeout(4_000_000_001) == nsa.NSA_ERR_INVALID_ARG
