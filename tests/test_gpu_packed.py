"""GPU parity of packed batches (nsa_prefill_packed, nsa_prefill_varlen) against the fp64
oracle of oracle/packed.py: sequences of video and text segments in any order, every row
compared; every stage of the call is launched once for the whole batch."""
import numpy as np
import pytest
import torch

from oracle import oracle as orc
from oracle import packed as pk_orc
from sparse_attention_long_fwd_b200 import nsa
from sparse_attention_long_fwd_b200.inputs import WORKLOADS, bf16_bits, prefill_inputs, scaled

from nsa_check import assert_close, check_selection

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _layout(seqs):
    lens = [sum(n for n, _ in s) for s in seqs]
    cu = [0] + np.cumsum(lens).tolist()
    seg_lens = [n for s in seqs for n, _ in s]
    seg_vid = [1 if vid else 0 for s in seqs for _, vid in s]
    return cu, seg_lens, seg_vid


def _run_packed(seqs, hq=28, hkv=4, d=128, top_n=16, window=512, seed=0, out_dtype=torch.float32):
    cu, seg_lens, seg_vid = _layout(seqs)
    N = cu[-1]
    nv = sum(n for n, vid in zip(seg_lens, seg_vid) if vid)
    w = scaled(WORKLOADS["qwen36k_hybrid"], n_tokens=N, n_video=N, hq=hq, hkv=hkv, d=d, top_n=top_n, window=window)
    q, k, v, g = prefill_inputs(w, seed=seed, device=DEV)
    p = nsa.make_params(N, 0, hq, hkv, d, top_n=top_n, window=window,
                        out_dtype=nsa.NSA_OUT_F32 if out_dtype == torch.float32 else nsa.NSA_OUT_BF16)
    need = nsa.nsa_prefill_packed_workspace_size(p, cu, seg_lens, seg_vid)
    assert need > 0
    ws = torch.empty(need, dtype=torch.uint8, device=DEV)
    out = torch.full((N, hq, d), float("nan"), dtype=out_dtype, device=DEV)
    sel = torch.full((max(nv, 1), hkv, top_n), -7, dtype=torch.int32, device=DEV)
    rc = nsa.nsa_prefill_packed(q, k, v, g, cu, seg_lens, seg_vid, p, out, sel if nv else None, ws, need)
    assert rc == nsa.NSA_OK, nsa.nsa_error_string(rc)
    torch.cuda.synchronize()
    assert nsa.nsa_get_device_error(clear=True) == 0
    return (cu, seg_lens, seg_vid), (q, k, v, g), out, sel[:nv]


def _check_packed(lay, tensors, out, sel, hq, hkv, d, top_n, window, nthreads=0):
    cu, seg_lens, seg_vid = lay
    q, k, v, g = tensors
    N = cu[-1]
    cfg = orc.OracleConfig(N, N, hq, hkv, d, top_n=top_n, window=window)
    qb, kb, vb = (bf16_bits(x) for x in (q, k, v))
    gh = g.cpu().numpy()
    o = pk_orc.packed_prefill(cfg, qb, kb, vb, gh, cu, seg_lens, seg_vid, nthreads=nthreads)
    gsel = sel.cpu().numpy()
    ties, at = 0, 0
    for sc in o["scores"]:  # per sequence with video rows, in order
        n = sc.shape[0]
        _, t = check_selection(gsel[at: at + n], o["sel"][at: at + n], sc)
        ties += t
        at += n
    assert at == gsel.shape[0]
    ref = o["out"]
    if ties:
        ref = pk_orc.packed_prefill(cfg, qb, kb, vb, gh, cu, seg_lens, seg_vid, nthreads=nthreads,
                                    sel_override=gsel)["out"]
    got = out.float().cpu().numpy()
    if out.dtype == torch.float32:
        return assert_close(got, ref, "packed out"), ties
    err = np.abs(got - ref)
    assert np.all((err <= np.abs(ref) * 2.0 ** -7 + 1e-30) | (err <= 1e-2)), "bf16 packed out"
    return (float(err.max()), float(err.mean())), ties


def test_packed_interleaved_segments_every_row():
    """One sequence of three video segments with text between and after them."""
    seqs = [[(600, True), (40, False), (500, True), (30, False), (300, True), (25, False)]]
    lay, t, out, sel = _run_packed(seqs, seed=41)
    print(_check_packed(lay, t, out, sel, 28, 4, 128, 16, 512))


def test_packed_batch_mixed_layouts_every_row():
    """Text first, video only, text only, video-text-video, empty and shorter-than-a-block
    sequences in one batch (G = 4, d = 64: different tile shapes)."""
    seqs = [[(50, True), (20, False)], [], [(100, False), (700, True), (20, False)], [(33, True)],
            [(90, False)], [(900, True), (60, False), (257, True)], [(20, True), (5, False), (17, True)]]
    lay, t, out, sel = _run_packed(seqs, hq=16, hkv=4, d=64, top_n=6, window=200, seed=42)
    print(_check_packed(lay, t, out, sel, 16, 4, 64, 6, 200))


def test_packed_bf16_output_and_gqa7():
    seqs = [[(1200, True), (80, False)], [(64, False), (1000, True)]]
    lay, t, out, sel = _run_packed(seqs, top_n=12, window=256, seed=43, out_dtype=torch.bfloat16)
    print(_check_packed(lay, t, out, sel, 28, 4, 128, 12, 256))


def test_packed_all_text_and_no_video_rows():
    seqs = [[(300, False)], [(129, False)]]
    lay, t, out, sel = _run_packed(seqs, hq=8, hkv=2, d=128, top_n=4, window=64, seed=44)
    print(_check_packed(lay, t, out, sel, 8, 2, 128, 4, 64))


def test_varlen_64_clips_of_2k_in_one_launch_chain():
    """64 all-video clips of 2,048 tokens: the serving batch the one-grid form is for. Four
    clips (first, two middle, last) are checked on every row against the oracle; the whole
    batch's output must be finite and its selections well formed."""
    B, L = 64, 2048
    w = scaled(WORKLOADS["v128k"], n_tokens=B * L, n_video=B * L)
    q, k, v, g = prefill_inputs(w, seed=45, device=DEV)
    cu = [b * L for b in range(B + 1)]
    nvs = [L] * B
    p = nsa.make_params(B * L, 0, w.hq, w.hkv, w.d, top_n=16, window=512, out_dtype=nsa.NSA_OUT_F32)
    need = nsa.nsa_prefill_varlen_workspace_size(p, cu, nvs)
    ws = torch.empty(need, dtype=torch.uint8, device=DEV)
    out = torch.empty((B * L, w.hq, w.d), dtype=torch.float32, device=DEV)
    sel = torch.full((B * L, w.hkv, 16), -7, dtype=torch.int32, device=DEV)
    assert nsa.nsa_prefill_varlen(q, k, v, g, cu, nvs, p, out, sel, ws, need) == nsa.NSA_OK
    torch.cuda.synchronize()
    assert nsa.nsa_get_device_error(clear=True) == 0
    assert torch.isfinite(out).all()
    s = sel.view(B, L, w.hkv, 16)
    assert (s[:, :, :, 0] == 0).all()  # block 0 always kept, and listed first (ascending)
    for b in (0, 21, 42, 63):
        sl = slice(b * L, (b + 1) * L)
        lay = ([0, L], [L], [1])
        print(b, _check_packed(lay, (q[sl], k[sl], v[sl], g[sl]), out[sl], sel[sl], w.hq, w.hkv, w.d, 16, 512))


def test_packed_rejects_malformed_segments():
    p = nsa.make_params(100, 0, 4, 1, 64, top_n=4, window=64)
    f = 1 << 20  # never dereferenced: validation fails first
    assert nsa.nsa_prefill_packed(f, f, f, f, [0, 100], [60, 50], [1, 0], p, f, None, f, 1 << 40) == \
        nsa.NSA_ERR_INVALID_ARG  # segments overrun the sequence
    assert nsa.nsa_prefill_packed(f, f, f, f, [0, 100], [60, 40, 1], [1, 0, 1], p, f, None, f, 1 << 40) == \
        nsa.NSA_ERR_INVALID_ARG  # more segments than rows
    assert nsa.nsa_prefill_packed(f, f, f, f, [0, 100], [100], [2], p, f, None, f, 1 << 40) == \
        nsa.NSA_ERR_INVALID_ARG  # segment kind must be 0 or 1
    assert nsa.nsa_prefill_packed_workspace_size(p, [0, 100], [100], [1]) > 0
    assert nsa.nsa_prefill_packed_workspace_size(p, [0, 99], [99], [1]) == 0  # cu_seqlens[B] != n_tokens
