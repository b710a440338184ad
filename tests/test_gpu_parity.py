"""GPU parity: the CUDA path (called through the C ABI) against the fp64 oracle.

Sizes the oracle finishes in seconds compare every row and every intermediate; the
full-size workloads (36K hybrid, 128K, 64 x 128K decode) compare sampled rows, in the
same launch configuration the benchmark times.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as orc
from sparse_attention_long_fwd_b200 import nsa
from sparse_attention_long_fwd_b200.inputs import WORKLOADS, bf16_bits, decode_inputs, prefill_inputs, scaled

from nsa_check import (MAX_ABS, MEAN_ABS, assert_close, check_selection, compare_prefill_rows, oracle_cfg,
                       run_prefill, sample_rows)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _prefill_case(w, seed, rows=None, out_dtype=torch.float32, nthreads=0):
    q, k, v, g = prefill_inputs(w, seed=seed, device=DEV)
    out, sel, ws, lay = run_prefill(w, q, k, v, g, out_dtype=out_dtype)
    if rows is None:
        rows = np.arange(w.n_tokens)
    return compare_prefill_rows(w, q, k, v, g, rows, out, sel, ws, lay, nthreads=nthreads)


def test_compress_bit_exact():
    w = scaled(WORKLOADS["v128k"], n_tokens=4099, n_video=4099)
    q, k, v, g = prefill_inputs(w, seed=3, device=DEV)
    kc, vc = nsa.compress(k, v)
    torch.cuda.synchronize()
    kb, vb = bf16_bits(k), bf16_bits(v)
    assert np.array_equal(bf16_bits(kc), orc.compress(kb))
    assert np.array_equal(bf16_bits(vc), orc.compress(vb))


def test_compress_batched_bit_exact():
    w = scaled(WORKLOADS["decode64x128k"], batch=3, n_tokens=1000)
    q, kc, vc, g, sl = decode_inputs(w, seed=4, device=DEV)
    kcmp, vcmp = nsa.compress(kc, vc)
    torch.cuda.synchronize()
    for b in range(3):
        assert np.array_equal(bf16_bits(kcmp[b]), orc.compress(bf16_bits(kc[b])))
        assert np.array_equal(bf16_bits(vcmp[b]), orc.compress(bf16_bits(vc[b])))


def test_prefill_tiny_all_rows():
    """The 2048-token, 4-head, d=64 workload: every row and every intermediate."""
    st = _prefill_case(WORKLOADS["tiny"], seed=0)
    print(st)


@pytest.mark.parametrize("n,hq,hkv,d,top_n,window", [
    (1000, 28, 4, 128, 16, 512),     # several tiles, ragged tail (1000 = 55 * 18 + 10)
    (777, 8, 1, 64, 5, 100),         # G = 8, d = 64, tiny window
    (1500, 16, 16, 128, 4, 300),     # G = 1 (no GQA)
    (640, 12, 3, 128, 64, 2048),     # top_n and window cover everything: dense special case
    (1100, 48, 4, 128, 16, 512),     # G = 12: 16-lane head groups (4 padding heads), 10-token tiles
    (900, 32, 2, 128, 12, 256),      # G = 16: 8-token tiles, every lane a real head
    (700, 24, 2, 64, 8, 200),        # G = 12 with d = 64
])
def test_prefill_shapes_all_rows(n, hq, hkv, d, top_n, window):
    w = scaled(WORKLOADS["v128k"], n_tokens=n, n_video=n, hq=hq, hkv=hkv, d=d, top_n=top_n, window=window)
    st = _prefill_case(w, seed=n)
    print(st)


def test_prefill_hybrid_small_all_rows():
    w = scaled(WORKLOADS["qwen36k_hybrid"], n_tokens=1300, n_video=1100)
    st = _prefill_case(w, seed=5)
    print(st)


def test_prefill_edge_lengths():
    for n in (1, 17, 31, 32, 33, 64, 65, 129):
        w = scaled(WORKLOADS["qwen36k_hybrid"], n_tokens=n, n_video=n)
        _prefill_case(w, seed=100 + n)
    # all text (no video prefix): dense causal only
    w = scaled(WORKLOADS["qwen36k_hybrid"], n_tokens=300, n_video=0)
    _prefill_case(w, seed=7)


def test_prefill_g16_9k_sampled():
    """G = 16 (every lane of a 16-lane head group a real head) at 9,000 tokens: many
    compressed key tiles and selected buckets of mixed sizes; the first rows, rows around
    4K and 8K, the last row and random rows, every intermediate."""
    w = scaled(WORKLOADS["v128k"], n_tokens=9000, n_video=9000, hq=32, hkv=2, d=128, top_n=16, window=512)
    q, k, v, g = prefill_inputs(w, seed=31, device=DEV)
    out, sel, ws, lay = run_prefill(w, q, k, v, g)
    rows = set(range(0, 70)) | {4094, 4095, 4096, 4097, 8190, 8191, 8192, 8193, 8999}
    rows |= set(int(x) for x in np.random.default_rng(31).integers(0, 9000, 60))
    st = compare_prefill_rows(w, q, k, v, g, np.array(sorted(rows), dtype=np.int32), out, sel, ws, lay)
    print(st)


def test_prefill_bf16_output():
    w = scaled(WORKLOADS["qwen36k_hybrid"], n_tokens=900, n_video=800)
    _prefill_case(w, seed=9, out_dtype=torch.bfloat16)


def test_prefill_one_hot_gates_isolate_branches():
    w = scaled(WORKLOADS["qwen36k_hybrid"], n_tokens=700, n_video=700)
    q, k, v, g = prefill_inputs(w, seed=11, device=DEV)
    outs = []
    for which in range(3):
        gg = torch.zeros_like(g)
        gg[..., which] = 1.0
        out, sel, ws, lay = run_prefill(w, q, k, v, gg)
        outs.append((out.clone(), ws, lay, sel.clone()))
    from nsa_check import ws_view, host_bits
    ocmp = ws_view(outs[0][1], outs[0][2]["o_cmp"], (700, w.hq, w.d), torch.float16)
    owin = ws_view(outs[2][1], outs[2][2]["o_win"], (700, w.hq, w.d), torch.float16)
    assert torch.equal(outs[0][0], ocmp.float())
    assert torch.equal(outs[2][0], owin.float())
    # the selected branch is never stored on its own: with g_sel = 1 the output is o_sel,
    # checked against the oracle on the blocks this run selected (near-ties may differ)
    qb, kb, vb = host_bits(q, k, v)
    rows = np.arange(0, 700, 7, dtype=np.int32)
    gg = torch.zeros_like(g)
    gg[..., 1] = 1.0
    o = orc.prefill_rows(oracle_cfg(w), qb, kb, vb, gg.cpu().numpy(), rows,
                         sel_override=outs[1][3][rows].cpu().numpy(), want=("o_sel",))
    assert_close(outs[1][0][rows].cpu().numpy(), o["o_sel"], "o_sel through g_sel = 1")


@pytest.mark.parametrize("n,nv,hq,hkv,d", [(1000, 1000, 28, 4, 128), (777, 700, 8, 1, 64)])
def test_prefill_kept_branch_statistics(n, nv, hq, hkv, d):
    """keep_branch_stats: the output is bit-identical to a run without it, and the kept o_sel,
    lse_sel and lse_win match the oracle's selected and window branches (on the blocks this run
    selected, so near-ties cannot differ)."""
    from nsa_check import ws_view, host_bits
    w = scaled(WORKLOADS["qwen36k_hybrid"], n_tokens=n, n_video=nv, hq=hq, hkv=hkv, d=d)
    q, k, v, g = prefill_inputs(w, seed=13, device=DEV)
    out0, sel0, _, _ = run_prefill(w, q, k, v, g)
    out, sel, ws, lay = run_prefill(w, q, k, v, g, keep=True)
    assert torch.equal(out, out0) and torch.equal(sel, sel0)
    assert lay["o_sel"] > 0 and lay["lse_sel"] > 0 and lay["lse_win"] > 0
    o_sel = ws_view(ws, lay["o_sel"], (nv, hq, d), torch.float16).float().cpu().numpy()
    lse_sel = ws_view(ws, lay["lse_sel"], (nv, hq), torch.float32).cpu().numpy()
    lse_win = ws_view(ws, lay["lse_win"], (nv, hq), torch.float32).cpu().numpy()
    qb, kb, vb = host_bits(q, k, v)
    rows = np.concatenate([np.arange(0, 70), np.arange(70, nv, 5), [nv - 1]]).astype(np.int32)
    o = orc.prefill_rows(oracle_cfg(w), qb, kb, vb, g.cpu().numpy(), rows, sel_override=sel[rows].cpu().numpy(),
                         want=("o_sel", "lse_sel", "lse_win"))
    assert_close(o_sel[rows], o["o_sel"], "kept o_sel")
    # log-sum-exp: the kernels sum P as the bf16 value the tensor core multiplies (relative
    # rounding <= 2^-9 per term), so with one dominant key ln(sum) is off by up to ln(1 + 2^-8)
    assert_close(lse_sel[rows], o["lse_sel"], "kept lse_sel", max_abs=4e-3, mean_abs=2e-4)
    assert_close(lse_win[rows], o["lse_win"], "kept lse_win", max_abs=4e-3, mean_abs=2e-4)


@pytest.mark.parametrize("n", [9000, 40000])
def test_prefill_constant_keys_exact_ties(n):
    """Every key equal: the compressed probabilities are uniform, so all interior selection
    blocks tie exactly (in fp32 here and in fp64 in the oracle) and thousands of candidates
    sit at the top-n bound; the lower block index must win every tie."""
    w = scaled(WORKLOADS["v128k"], n_tokens=n, n_video=n)
    q, k, v, g = prefill_inputs(w, seed=13, device=DEV)
    k = k[:1].expand_as(k).contiguous()
    out, sel, ws, lay = run_prefill(w, q, k, v, g)
    rows = np.unique(np.concatenate([np.arange(0, n, 97), np.arange(n - 64, n)])).astype(np.int32)
    st = compare_prefill_rows(w, q, k, v, g, rows, out, sel, ws, lay)
    assert st["ties"] == 0, st  # exact ties resolve the same way on both sides


def test_prefill_qwen36k_hybrid_sampled():
    w = WORKLOADS["qwen36k_hybrid"]
    q, k, v, g = prefill_inputs(w, seed=1, device=DEV)
    out, sel, ws, lay = run_prefill(w, q, k, v, g)
    rows = sample_rows(w.n_video, w.n_tokens, 64, seed=1)
    st = compare_prefill_rows(w, q, k, v, g, rows, out, sel, ws, lay)
    print(st)


def test_prefill_v128k_sampled():
    w = WORKLOADS["v128k"]
    q, k, v, g = prefill_inputs(w, seed=2, device=DEV)
    out, sel, ws, lay = run_prefill(w, q, k, v, g)
    rows = sample_rows(w.n_video, w.n_tokens, 48, seed=2)
    st = compare_prefill_rows(w, q, k, v, g, rows, out, sel, ws, lay)
    print(st)


def test_prefill_and_decode_graph_replay_match_direct_calls():
    """The C ABI only enqueues work on the given stream, so a call can be captured in a CUDA
    graph: its replay gives the direct call's output and selection bit for bit."""
    w = scaled(WORKLOADS["qwen36k_hybrid"], n_tokens=1500, n_video=1300)
    q, k, v, g = prefill_inputs(w, seed=17, device=DEV)
    p = nsa.make_params(w.n_tokens, w.n_video, w.hq, w.hkv, w.d, w.cmp_len, w.cmp_stride, w.sel_len, w.top_n,
                        w.window, out_dtype=nsa.NSA_OUT_F32)
    ws = nsa.alloc_workspace(p, False, q.device)
    out0 = torch.empty((w.n_tokens, w.hq, w.d), device=DEV)
    sel0 = torch.empty((w.n_video, w.hkv, w.top_n), dtype=torch.int32, device=DEV)
    assert nsa.nsa_prefill(q, k, v, g, p, out0, sel0, ws, ws.numel()) == nsa.NSA_OK
    torch.cuda.synchronize()
    out1, sel1 = torch.full_like(out0, float("nan")), torch.full_like(sel0, -7)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        assert nsa.nsa_prefill(q, k, v, g, p, out1, sel1, ws, ws.numel()) == nsa.NSA_OK
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(out1, out0) and torch.equal(sel1, sel0)
    del graph
    # decode (three kernels with dependent launches) the same way
    wd = scaled(WORKLOADS["decode64x128k"], batch=4, n_tokens=3000)
    qd, kc, vc, gd, sl = decode_inputs(wd, seed=18, device=DEV)
    kcmp, vcmp = nsa.compress(kc, vc)
    pd = nsa.make_params(wd.n_tokens, wd.n_tokens, wd.hq, wd.hkv, wd.d, top_n=wd.top_n, window=wd.window,
                         out_dtype=nsa.NSA_OUT_F32, batch=wd.batch)
    wsd = nsa.alloc_workspace(pd, True, qd.device)
    d0 = torch.empty((wd.batch, wd.hq, wd.d), device=DEV)
    assert nsa.nsa_decode(qd, kc, vc, kcmp, vcmp, sl, gd, pd, d0, None, wsd, wsd.numel()) == nsa.NSA_OK
    torch.cuda.synchronize()
    d1 = torch.full_like(d0, float("nan"))
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        assert nsa.nsa_decode(qd, kc, vc, kcmp, vcmp, sl, gd, pd, d1, None, wsd, wsd.numel()) == nsa.NSA_OK
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(d1, d0)
    assert nsa.nsa_get_device_error(clear=True) == 0


@pytest.mark.parametrize("n", [8192, 32768, 131072])
def test_prefill_error_by_length(n):
    """The fp16 intermediates (o_cmp, o_win, the selected partials) against sequence length:
    the same row sampling at 8K, 32K and 128K stays inside the prefill tolerance; the printed
    errors per length are the length study (each row's error comes from its own softmax, and
    more keys only lengthen its fp32 sums)."""
    w = scaled(WORKLOADS["v128k"], n_tokens=n, n_video=n)
    q, k, v, g = prefill_inputs(w, seed=2, device=DEV)
    out, sel, ws, lay = run_prefill(w, q, k, v, g)
    rows = sample_rows(w.n_video, w.n_tokens, 48, seed=2)
    st = compare_prefill_rows(w, q, k, v, g, rows, out, sel, ws, lay)
    print(f"n={n} out max/mean {st['out']} o_cmp {st.get('o_cmp')} o_win {st.get('o_win')}")
    assert st["out"][0] <= MAX_ABS and st["out"][1] <= MEAN_ABS


@pytest.mark.parametrize("name", ["sweep128k_n4_w256", "sweep128k_n48_w1024"])
def test_prefill_sweep_points_sampled(name):
    w = WORKLOADS[name]
    q, k, v, g = prefill_inputs(w, seed=2, device=DEV)
    out, sel, ws, lay = run_prefill(w, q, k, v, g)
    rows = sample_rows(w.n_video, w.n_tokens, 16, seed=3)
    compare_prefill_rows(w, q, k, v, g, rows, out, sel, ws, lay, check_intermediates=False)


# ---------------------------------------------------------------- decode

def _decode_case(w, seed, seq_lens=None, seqs=None):
    q, kc, vc, g, sl = decode_inputs(w, seed=seed, device=DEV, seq_lens=seq_lens)
    kcmp, vcmp = nsa.compress(kc, vc)
    out, sel = nsa.decode(q, kc, vc, kcmp, vcmp, sl, g, top_n=w.top_n, window=w.window, return_sel=True)
    torch.cuda.synchronize()
    assert nsa.nsa_get_device_error(clear=True) == 0
    cfg = orc.OracleConfig(w.n_tokens, w.n_tokens, w.hq, w.hkv, w.d, top_n=w.top_n, window=w.window)
    qb, kb, vb, kcb, vcb = (bf16_bits(t) for t in (q, kc, vc, kcmp, vcmp))
    gh, slh = g.cpu().numpy(), sl.cpu().numpy()
    if seqs is None:
        seqs = np.arange(w.batch)
    o = orc.decode(cfg, qb, kb, vb, kcb, vcb, slh, gh, seqs=seqs)
    gsel = sel.cpu().numpy()[seqs]
    replay, ties = check_selection(gsel, o["sel"], o["scores"])
    ref = o["out"]
    if replay:
        o2 = orc.decode(cfg, qb, kb, vb, kcb, vcb, slh, gh, seqs=np.asarray(seqs)[replay], sel_override=gsel[replay])
        ref[replay] = o2["out"]
    return assert_close(out.cpu().numpy()[seqs], ref, "decode out"), ties


def test_decode_small_varied_lengths():
    w = scaled(WORKLOADS["decode64x128k"], batch=8, n_tokens=3000)
    lens = [3000, 1, 31, 32, 33, 64, 1000, 2049]
    print(_decode_case(w, seed=21, seq_lens=lens))


def test_decode_d64_window_covers_all():
    w = scaled(WORKLOADS["decode64x128k"], batch=4, n_tokens=700, hq=8, hkv=2, d=64, top_n=12, window=1024)
    print(_decode_case(w, seed=22, seq_lens=[700, 350, 64, 129]))


def test_decode_top_n_48_shared_memory_selection():
    """top_n > 32 takes the shared-memory warp selection in decode."""
    w = scaled(WORKLOADS["decode64x128k"], batch=6, n_tokens=9000, top_n=48, window=512)
    print(_decode_case(w, seed=23, seq_lens=[9000, 8999, 4000, 3100, 2047, 1]))


@pytest.mark.parametrize("hq,hkv,d", [(48, 4, 128), (32, 2, 64)])
def test_decode_large_groups(hq, hkv, d):
    """G = 12 and G = 16 query heads per group in the decode tiles."""
    w = scaled(WORKLOADS["decode64x128k"], batch=5, n_tokens=5000, hq=hq, hkv=hkv, d=d, top_n=16, window=512)
    print(_decode_case(w, seed=24, seq_lens=[5000, 4097, 1000, 65, 30]))


def test_decode_64x128k_sampled():
    w = WORKLOADS["decode64x128k"]
    print(_decode_case(w, seed=4, seqs=np.arange(0, 64, 4)))


# ---------------------------------------------------------------- error paths on a device

def test_device_errors_are_reported_not_raised():
    w = scaled(WORKLOADS["tiny"], n_tokens=256, n_video=256)
    q, k, v, g = prefill_inputs(w, seed=0, device=DEV)
    p = nsa.make_params(256, 256, 4, 1, 64, top_n=4, window=64)
    ws = nsa.alloc_workspace(p, False, DEV)
    out = torch.empty((256, 4, 64), device=DEV)
    assert nsa.nsa_prefill(q, k, v, g, p, out, None, ws, ws.numel() - 256) == nsa.NSA_ERR_WORKSPACE_TOO_SMALL
    assert nsa.nsa_prefill(q, k, v, g, p, out, None, ws[1:], ws.numel() - 1) == nsa.NSA_ERR_INVALID_ARG
    bad = nsa.make_params(256, 256, 4, 1, 96, top_n=4, window=64)
    assert nsa.nsa_prefill(q, k, v, g, bad, out, None, ws, ws.numel()) == nsa.NSA_ERR_UNSUPPORTED
    assert nsa.nsa_get_device_error(clear=True) == 0


def test_prefill_varlen_packed_batch():
    """A packed batch (hybrid, empty, all-video, shorter-than-a-block and ragged sequences)
    matches nsa_prefill on each sequence alone: the same selection (up to reported near-ties)
    and outputs within the oracle tolerance (packing moves tile boundaries, so the fp32
    summation order differs); three sequences are checked against the oracle on every row."""
    base = scaled(WORKLOADS["qwen36k_hybrid"], n_tokens=700, n_video=600)
    lens, nvs = [700, 0, 1500, 33, 257], [600, 0, 1500, 33, 200]
    parts = []
    for b, (n, nv) in enumerate(zip(lens, nvs)):
        w = scaled(base, n_tokens=max(n, 1), n_video=min(nv, max(n, 1)))
        parts.append(prefill_inputs(w, seed=20 + b, device=DEV) if n > 0 else None)
    cat = lambda i: torch.cat([pp[i] for pp in parts if pp is not None], dim=0)
    q, k, v, g = cat(0), cat(1), cat(2), cat(3)
    cu = np.concatenate([[0], np.cumsum(lens)]).tolist()
    p = nsa.make_params(cu[-1], 0, base.hq, base.hkv, base.d, base.cmp_len, base.cmp_stride, base.sel_len,
                        base.top_n, base.window, out_dtype=nsa.NSA_OUT_F32)
    need = nsa.nsa_prefill_varlen_workspace_size(p, cu, nvs)
    ws = torch.empty(need, dtype=torch.uint8, device=DEV)
    out = torch.empty((cu[-1], base.hq, base.d), dtype=torch.float32, device=DEV)
    sel = torch.full((sum(nvs), base.hkv, base.top_n), -7, dtype=torch.int32, device=DEV)
    rc = nsa.nsa_prefill_varlen(q, k, v, g, cu, nvs, p, out, sel, ws, need)
    assert rc == nsa.NSA_OK, nsa.nsa_error_string(rc)
    torch.cuda.synchronize()
    assert nsa.nsa_get_device_error(clear=True) == 0
    srow = 0
    for b, (n, nv) in enumerate(zip(lens, nvs)):
        if n == 0:
            continue
        w = scaled(base, n_tokens=n, n_video=nv)
        qb, kb, vb, gb = (t[cu[b]: cu[b + 1]].contiguous() for t in (q, k, v, g))
        o1, s1, ws1, lay1 = run_prefill(w, qb, kb, vb, gb)
        err = (out[cu[b]: cu[b + 1]].double() - o1.double()).abs()
        assert err.max().item() <= MAX_ABS and err.mean().item() <= MEAN_ABS, f"sequence {b}: out differs"
        assert (sel[srow: srow + nv] != s1).sum().item() <= 4 * nv // 100, f"sequence {b}: selection differs"
        if b in (0, 3, 4):
            compare_prefill_rows(w, qb, kb, vb, gb, np.arange(n), out[cu[b]: cu[b + 1]], sel[srow: srow + nv], ws1,
                                 lay1, check_intermediates=False)
        srow += nv
