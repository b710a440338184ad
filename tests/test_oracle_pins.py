"""Pins for the fp64 oracle, against things other than the oracle itself.

Each test checks the oracle against a closed form, a hand-worked case, an invariant the
method guarantees, an independent formulation, or a library routine (torch SDPA in
float64 on the CPU). No expected value here comes from the CUDA path.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _rand_bf16(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * scale).to(torch.bfloat16)


def _f64(bits):
    return torch.from_numpy(orc.bf16_bits_to_f64(bits))


def _sdpa_causal(q, k, v, scale):
    """Dense causal attention in float64 via torch SDPA. q [N,hq,d], k/v [N,hkv,d] (float64)."""
    hq, hkv = q.shape[1], k.shape[1]
    rep = hq // hkv
    kk = k.repeat_interleave(rep, dim=1)
    vv = v.repeat_interleave(rep, dim=1)
    o = torch.nn.functional.scaled_dot_product_attention(
        q.transpose(0, 1), kk.transpose(0, 1), vv.transpose(0, 1), is_causal=True, scale=scale)
    return o.transpose(0, 1)


def _exact_bf16(x: Fraction) -> int:
    """Nearest bf16 to an exact rational, ties to even, by direct search (independent of the oracle)."""
    if x == 0:
        return 0
    sign = 0x8000 if x < 0 else 0
    a = abs(x)
    e = math.floor(math.log2(a))
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, -126)
    ulp = Fraction(2) ** (e - 7)
    lo = (a // ulp) * ulp
    hi = lo + ulp
    if a - lo < hi - a:
        r = lo
    elif a - lo > hi - a:
        r = hi
    else:
        r = lo if (lo / ulp) % 2 == 0 else hi
    f = np.array([float(r)], dtype=np.float32)
    return sign | int(f.view(np.uint32)[0] >> 16)


# ---------------------------------------------------------------- bf16 rounding

def test_round_bf16_matches_torch_on_float32_values():
    g = torch.Generator().manual_seed(1)
    x = torch.randn(20000, generator=g) * torch.exp(torch.randn(20000, generator=g) * 20)
    x = torch.cat([x, torch.tensor([0.0, -0.0, 1e-40, -3e-39, 3.0e38, 65504.0, 1.0 + 2 ** -8])])
    ref = _bits(x.to(torch.bfloat16))
    got = orc.round_bf16(x.double().numpy())
    assert np.array_equal(got, ref)


def test_round_bf16_single_rounding_step():
    # 1 + 2^-8 + 2^-30 lies just above the midpoint of bf16 neighbours 1.0 (0x3F80) and
    # 1 + 2^-7 (0x3F81): the correctly rounded result is 0x3F81. Rounding through fp32
    # first would drop the 2^-30 and then tie to even (0x3F80).
    x = 1.0 + 2.0 ** -8 + 2.0 ** -30
    assert orc.round_bf16(np.array([x]))[0] == 0x3F81
    assert orc.round_bf16(np.array([1.0 + 2.0 ** -8]))[0] == 0x3F80       # exact tie -> even
    assert orc.round_bf16(np.array([1.0 + 3 * 2.0 ** -8]))[0] == 0x3F82   # exact tie -> even
    big = (2 - 2 ** -8) * 2.0 ** 127                                       # max + half ulp -> inf
    assert orc.round_bf16(np.array([big, -big]))[0] == 0x7F80
    assert orc.round_bf16(np.array([big * (1 - 2 ** -20)]))[0] == 0x7F7F  # just below -> max


def test_round_bf16_exact_rationals():
    rng = np.random.default_rng(7)
    xs = rng.standard_normal(400) * np.exp2(rng.integers(-140, 120, 400))
    got = orc.round_bf16(xs)
    for x, b in zip(xs, got):
        assert b == _exact_bf16(Fraction(float(x))), x


# ---------------------------------------------------------------- compression

@pytest.mark.parametrize("l,s", [(32, 16), (8, 4), (6, 3), (5, 5)])
def test_compress_is_rounded_exact_mean(l, s):
    T, h, d = 150, 2, 8
    k = _bits(_rand_bf16((T, h, d), seed=l * 100 + s))
    kc = orc.compress(k, l, s)
    nc = (T - l) // s + 1
    assert kc.shape == (nc, h, d)
    kf = orc.bf16_bits_to_f64(k)
    for i in range(nc):
        for g in range(h):
            for c in range(0, d, 3):
                mean = sum(Fraction(float(kf[i * s + u, g, c])) for u in range(l)) / l
                assert kc[i, g, c] == _exact_bf16(mean)


def test_compress_block_one_is_identity():
    k = _bits(_rand_bf16((40, 3, 16), seed=3))
    assert np.array_equal(orc.compress(k, 1, 1), k)


def test_compress_short_sequence_has_no_blocks():
    k = _bits(_rand_bf16((31, 1, 8), seed=4))
    assert orc.compress(k, 32, 16).shape[0] == 0
    assert orc.num_cmp(31) == 0 and orc.num_cmp(32) == 1 and orc.num_cmp(47) == 1 and orc.num_cmp(48) == 2


def test_compress_integer_inputs_exact():
    rng = np.random.default_rng(5)
    ints = rng.integers(0, 8, (96, 1, 4)).astype(np.float32)
    k = _bits(torch.from_numpy(ints).to(torch.bfloat16))
    kc = orc.bf16_bits_to_f64(orc.compress(k, 32, 16))
    for i in range(kc.shape[0]):
        assert np.array_equal(kc[i], ints[i * 16:i * 16 + 32].mean(axis=0))


# ---------------------------------------------------------------- closed forms from the pages

def test_block_counts_closed_forms():
    assert (orc.num_cmp(131072), orc.num_sel(131072)) == (8191, 2048)
    assert (orc.num_cmp(36096), orc.num_sel(36096)) == (2255, 564)
    assert (orc.num_cmp(2048), orc.num_sel(2048)) == (127, 32)


def test_page_numbers_shapes_and_dense_count():
    pages = json.load(open(os.path.join(GOLDEN, "pages_numbers.json")))
    from sparse_attention_long_fwd_b200.inputs import TOKENS_PER_FRAME

    # a 50,176-pixel frame at 28x28 pixels per merged vision token is 64 tokens
    assert pages["max_pixels_per_frame"]["value"] // (28 * 28) == TOKENS_PER_FRAME
    # the dense causal (query, key) pair count at 128K tokens is the ~8.2e9 the pages quote
    n = pages["scales_to_tokens"]["value"]
    pairs = n * (n + 1) // 2
    assert abs(pairs - pages["dense_attention_ops_at_128k"]["value"]) / pairs < 0.01
    # 36K context = 564 frames of 64 tokens (36,096), the hybrid workload's video prefix
    assert 564 * TOKENS_PER_FRAME <= pages["max_training_context_tokens"]["value"] * 1.003


# ---------------------------------------------------------------- branches vs library / invariants

def _case(N, hq, hkv, d, seed, nv=None, **kw):
    q = _rand_bf16((N, hq, d), seed)
    k = _rand_bf16((N, hkv, d), seed + 1)
    v = _rand_bf16((N, hkv, d), seed + 2)
    g = torch.rand((N, hq, 3), generator=torch.Generator().manual_seed(seed + 3))
    cfg = orc.OracleConfig(N, N if nv is None else nv, hq, hkv, d, **kw)
    return cfg, q, k, v, g


def test_cmp_branch_with_unit_blocks_is_dense_causal_attention():
    cfg, q, k, v, g = _case(96, 4, 2, 16, 11, cmp_len=1, cmp_stride=1, sel_len=8, top_n=4, window=16)
    rows = np.arange(96)
    o = orc.prefill_rows(cfg, _bits(q), _bits(k), _bits(v), g.numpy(), rows)
    scale = 1 / math.sqrt(16)
    qd, kd, vd = _f64(_bits(q)), _f64(_bits(k)), _f64(_bits(v))
    ref = _sdpa_causal(qd, kd, vd, scale)
    assert np.allclose(o["o_cmp"], ref.numpy(), atol=1e-12, rtol=0)
    # log-sum-exp against torch.logsumexp of the causal score rows
    for t in (0, 5, 95):
        for h in range(4):
            z = (kd[: t + 1, h // 2] @ qd[t, h]) * scale
            assert abs(o["lse"][t, h] - torch.logsumexp(z, 0).item()) < 1e-12


def test_full_budget_selection_and_window_are_dense_attention():
    N = 200
    cfg, q, k, v, g = _case(N, 6, 2, 16, 21, top_n=orc.num_sel(N, 64) + 2, window=N + 5)
    o = orc.prefill_rows(cfg, _bits(q), _bits(k), _bits(v), g.numpy(), np.arange(N),
                         want=orc.ALL + ("lse_sel", "lse_win"))
    qd, kd, vd = _f64(_bits(q)), _f64(_bits(k)), _f64(_bits(v))
    ref = _sdpa_causal(qd, kd, vd, 1 / 4.0).numpy()
    assert np.allclose(o["o_sel"], ref, atol=1e-12, rtol=0)
    assert np.allclose(o["o_win"], ref, atol=1e-12, rtol=0)
    # both branches' log-sum-exp: torch.logsumexp of the causal score rows
    for t in (0, 63, 64, 199):
        for h in range(6):
            want = torch.logsumexp((kd[: t + 1, h // 3] @ qd[t, h]) / 4.0, 0).item()
            assert abs(o["lse_sel"][t, h] - want) < 1e-12
            assert abs(o["lse_win"][t, h] - want) < 1e-12


def test_unit_window_log_sum_exp_is_the_own_score():
    # w = 1: the window holds the query token alone, so its log-sum-exp is that one scaled score
    cfg, q, k, v, g = _case(130, 4, 2, 16, 23, top_n=3, window=1)
    rows = np.array([0, 1, 64, 129])
    o = orc.prefill_rows(cfg, _bits(q), _bits(k), _bits(v), g.numpy(), rows, want=("lse_win", "o_win"))
    qd, kd, vd = _f64(_bits(q)), _f64(_bits(k)), _f64(_bits(v))
    for r, t in enumerate(rows):
        for h in range(4):
            assert abs(o["lse_win"][r, h] - float(qd[t, h] @ kd[t, h // 2]) / 4.0) < 1e-12
            assert np.array_equal(o["o_win"][r, h], vd[t, h // 2].numpy())


def test_constant_keys_log_sum_exp_counts_the_keys():
    # every key equal: each branch's log-sum-exp is the common score plus the log of its key count
    N, w = 300, 40
    cfg, q, k, v, g = _case(N, 2, 1, 16, 25, top_n=3, window=w)
    k = k[:1].expand(N, -1, -1).contiguous()
    rows = np.array([0, 10, 39, 40, 63, 64, 150, 299])
    o = orc.prefill_rows(cfg, _bits(q), _bits(k), _bits(v), g.numpy(), rows,
                         want=("sel", "lse_sel", "lse_win"))
    qd, kd = _f64(_bits(q)), _f64(_bits(k))
    for r, t in enumerate(rows):
        nsel_keys = sum(min(64, t + 1 - 64 * j) for j in o["sel"][r, 0] if j >= 0)
        for h in range(2):
            z = float(qd[t, h] @ kd[0, 0]) / 4.0
            assert abs(o["lse_win"][r, h] - (z + math.log(min(w, t + 1)))) < 1e-12
            assert abs(o["lse_sel"][r, h] - (z + math.log(nsel_keys))) < 1e-12


def test_first_token_attends_to_itself_only():
    cfg, q, k, v, g = _case(64, 4, 1, 8, 31, top_n=4, window=16)
    o = orc.prefill_rows(cfg, _bits(q), _bits(k), _bits(v), g.numpy(), np.array([0]))
    v0 = orc.bf16_bits_to_f64(_bits(v))[0, 0]
    for h in range(4):
        assert np.allclose(o["o_sel"][0, h], v0, atol=1e-15)
        assert np.allclose(o["o_win"][0, h], v0, atol=1e-15)
        assert np.all(o["o_cmp"][0, h] == 0) and o["lse"][0, h] == -np.inf
    assert list(o["sel"][0, 0]) == [0, -1, -1, -1]


@pytest.mark.parametrize("which", [0, 1, 2])
def test_one_hot_gates_isolate_a_branch(which):
    cfg, q, k, v, _ = _case(300, 4, 2, 16, 41, top_n=4, window=40)
    g = np.zeros((300, 4, 3), dtype=np.float32)
    g[..., which] = 1.0
    rows = np.array([0, 31, 32, 100, 200, 299])
    o = orc.prefill_rows(cfg, _bits(q), _bits(k), _bits(v), g, rows)
    key = ("o_cmp", "o_sel", "o_win")[which]
    assert np.array_equal(o["out"], o[key])


def test_text_rows_are_dense_causal_attention():
    N, nv = 260, 192
    cfg, q, k, v, g = _case(N, 4, 2, 16, 51, nv=nv, top_n=4, window=32)
    rows = np.arange(nv, N)
    o = orc.prefill_rows(cfg, _bits(q), _bits(k), _bits(v), g.numpy(), rows)
    ref = _sdpa_causal(_f64(_bits(q)), _f64(_bits(k)), _f64(_bits(v)), 0.25).numpy()
    assert np.allclose(o["out"], ref[nv:], atol=1e-12, rtol=0)


def test_outputs_are_convex_combinations_of_values():
    cfg, q, k, v, g = _case(400, 4, 2, 16, 61, top_n=5, window=50)
    rows = np.arange(0, 400, 7)
    o = orc.prefill_rows(cfg, _bits(q), _bits(k), _bits(v), g.numpy(), rows)
    vd = orc.bf16_bits_to_f64(_bits(v))
    vcd = orc.bf16_bits_to_f64(orc.compress(_bits(v)))
    for key, src in (("o_sel", vd), ("o_win", vd)):
        for gi in range(2):
            lo, hi = src[:, gi].min(0), src[:, gi].max(0)
            blk = o[key][:, gi * 2:(gi + 1) * 2]
            assert np.all(blk >= lo - 1e-12) and np.all(blk <= hi + 1e-12)
    for gi in range(2):
        blk = o["o_cmp"][:, gi * 2:(gi + 1) * 2]
        assert np.all(blk >= vcd[:, gi].min(0) - 1e-12) and np.all(blk <= vcd[:, gi].max(0) + 1e-12)


# ---------------------------------------------------------------- block scores and selection

def test_scores_equal_token_density_formulation():
    """Independent formulation: spread each compression block's probability evenly over its
    l tokens, then sum the token densities inside each selection block and over the group."""
    N, hq, hkv, d = 700, 6, 2, 16
    cfg, q, k, v, g = _case(N, hq, hkv, d, 71, top_n=6, window=64)
    rows = np.array([31, 47, 63, 64, 130, 333, 640, 699])
    o = orc.prefill_rows(cfg, _bits(q), _bits(k), _bits(v), g.numpy(), rows)
    kc = _f64(orc.compress(_bits(k)))
    qd = _f64(_bits(q))
    G = hq // hkv
    for r, t in enumerate(rows):
        nc = orc.num_cmp(t + 1)
        for gi in range(hkv):
            dens = torch.zeros(N, dtype=torch.float64)
            for hh in range(G):
                h = gi * G + hh
                p = torch.softmax((kc[:nc, gi] @ qd[t, h]) / 4.0, 0)
                for i in range(nc):
                    dens[16 * i:16 * i + 32] += p[i] / 32
            jt = t // 64
            ref = [dens[64 * j:64 * j + 64].sum().item() for j in range(jt + 1)]
            assert np.allclose(o["scores"][r, gi, :jt + 1], ref, atol=1e-13, rtol=0)
            assert np.all(o["scores"][r, gi, jt + 1:] == 0)


def test_scores_conserve_mass():
    cfg, q, k, v, g = _case(1500, 8, 2, 16, 81, top_n=6, window=64)
    rows = np.arange(0, 1500, 13)
    o = orc.prefill_rows(cfg, _bits(q), _bits(k), _bits(v), g.numpy(), rows)
    for r, t in enumerate(rows):
        tot = o["scores"][r].sum(axis=1)
        expect = 4.0 if t >= 31 else 0.0
        assert np.allclose(tot, expect, atol=1e-12)


def test_selection_invariants_on_random_scores():
    N, n = 2000, 7
    cfg, q, k, v, g = _case(N, 4, 2, 16, 91, top_n=n, window=64)
    rows = np.arange(0, N, 9)
    o = orc.prefill_rows(cfg, _bits(q), _bits(k), _bits(v), g.numpy(), rows)
    for r, t in enumerate(rows):
        jt = t // 64
        for gi in range(2):
            sel = o["sel"][r, gi]
            chosen = [int(x) for x in sel if x >= 0]
            assert chosen == sorted(set(chosen))
            assert len(chosen) == min(n, jt + 1)
            assert all(x < 0 for x in sel[len(chosen):])
            forced = {0, jt, jt - 1} & set(range(jt + 1))
            assert forced <= set(chosen)
            sc = o["scores"][r, gi]
            free = [j for j in chosen if j not in forced]
            rest = [j for j in range(jt + 1) if j not in chosen]
            for a in free:
                for b in rest:
                    assert sc[a] > sc[b] or (sc[a] == sc[b] and a < b)


def test_constant_keys_hand_worked_case():
    case = json.load(open(os.path.join(GOLDEN, "constant_keys_case.json")))
    c = case["config"]
    N, hq, hkv, d = c["n_tokens"], c["hq"], c["hkv"], c["d"]
    q = _rand_bf16((N, hq, d), 101)
    krow = _rand_bf16((1, hkv, d), 102)
    k = krow.expand(N, hkv, d).contiguous()
    v = _rand_bf16((N, hkv, d), 103)
    g = torch.rand((N, hq, 3), generator=torch.Generator().manual_seed(104))
    cfg = orc.OracleConfig(N, c["n_video"], hq, hkv, d, c["cmp_len"], c["cmp_stride"], c["sel_len"], c["top_n"],
                           c["window"])
    rows = np.array([int(x) for x in case["rows"]])
    o = orc.prefill_rows(cfg, _bits(q), _bits(k), _bits(v), g.numpy(), rows)
    vd = orc.bf16_bits_to_f64(_bits(v))
    vcd = orc.bf16_bits_to_f64(orc.compress(_bits(v)))
    for r, t in enumerate(rows):
        exp = case["rows"][str(t)]
        assert list(o["sel"][r, 0]) == exp["sel"]
        for key, den in (("scores_numerators_over_61", 61), ("scores_numerators_over_7", 7)):
            if key in exp:
                num = exp[key]
                assert np.allclose(o["scores"][r, 0, :len(num)], np.array(num) / den, atol=1e-14)
        # uniform scores: each branch output is the plain mean of its values
        keys = [tau for j in exp["sel"] if j >= 0 for tau in range(64 * j, 64 * j + 64) if tau <= t]
        win = list(range(max(0, t - c["window"] + 1), t + 1))
        nc = orc.num_cmp(t + 1)
        for h in range(hq):
            assert np.allclose(o["o_sel"][r, h], vd[keys, 0].mean(0), atol=1e-14)
            assert np.allclose(o["o_win"][r, h], vd[win, 0].mean(0), atol=1e-14)
            ref_cmp = vcd[:nc, 0].mean(0) if nc else np.zeros(d)
            assert np.allclose(o["o_cmp"][r, h], ref_cmp, atol=1e-14)


def test_replay_with_own_selection_is_identity():
    cfg, q, k, v, g = _case(900, 4, 2, 16, 111, top_n=5, window=100)
    rows = np.array([100, 400, 899])
    a = orc.prefill_rows(cfg, _bits(q), _bits(k), _bits(v), g.numpy(), rows)
    b = orc.prefill_rows(cfg, _bits(q), _bits(k), _bits(v), g.numpy(), rows, sel_override=a["sel"])
    assert np.array_equal(a["out"], b["out"])
    # replay with a different selection changes only the selection branch
    alt = a["sel"].copy()
    alt[2, 0, 1] = 3 if alt[2, 0, 1] != 3 else 4
    c = orc.prefill_rows(cfg, _bits(q), _bits(k), _bits(v), g.numpy(), rows, sel_override=alt)
    assert np.array_equal(c["o_cmp"], a["o_cmp"]) and np.array_equal(c["o_win"], a["o_win"])
    assert not np.allclose(c["o_sel"][2, :2], a["o_sel"][2, :2])


# ---------------------------------------------------------------- decode

def test_decode_equals_prefill_last_row():
    B, Lmax, hq, hkv, d = 3, 400, 4, 2, 16
    kcache = _rand_bf16((B, Lmax, hkv, d), 121)
    vcache = _rand_bf16((B, Lmax, hkv, d), 122)
    q = _rand_bf16((B, hq, d), 123)
    gates = torch.rand((B, hq, 3), generator=torch.Generator().manual_seed(124))
    seq_lens = np.array([400, 257, 31], dtype=np.int32)
    kcmp = np.stack([orc.compress(_bits(kcache[b])) for b in range(B)])
    vcmp = np.stack([orc.compress(_bits(vcache[b])) for b in range(B)])
    cfg = orc.OracleConfig(Lmax, Lmax, hq, hkv, d, top_n=5, window=64)
    dec = orc.decode(cfg, _bits(q), _bits(kcache), _bits(vcache), kcmp, vcmp, seq_lens, gates.numpy())
    for b in range(B):
        L = int(seq_lens[b])
        qq = torch.zeros((L, hq, d), dtype=torch.bfloat16)
        qq[L - 1] = q[b]
        gg = torch.zeros((L, hq, 3))
        gg[L - 1] = gates[b]
        pc = orc.OracleConfig(L, L, hq, hkv, d, top_n=5, window=64)
        pre = orc.prefill_rows(pc, _bits(qq), _bits(kcache[b, :L].contiguous()), _bits(vcache[b, :L].contiguous()),
                               gg.numpy(), np.array([L - 1]))
        assert np.array_equal(dec["out"][b], pre["out"][0])
        assert np.array_equal(dec["sel"][b], pre["sel"][0])


# ---------------------------------------------------------------- learnable compression

def _rand_weights(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return (torch.rand(shape, generator=g) * 0.1 - 0.02).numpy().astype(np.float32)


def test_weighted_compress_is_rounded_exact_weighted_sum():
    # the definition evaluated in exact rationals, rounded by direct search
    T, h, d, l, s = 40, 2, 4, 8, 4
    k = _bits(_rand_bf16((T, h, d), 31))
    w = _rand_weights((h, l), 32)
    got = orc.compress_weighted(k, w, l, s)
    kf = orc.bf16_bits_to_f64(k)
    nc = (T - l) // s + 1
    assert got.shape == (nc, h, d)
    for i in range(nc):
        for g in range(h):
            for c in range(d):
                exact = sum(Fraction(float(w[g, u])) * Fraction(float(kf[i * s + u, g, c])) for u in range(l))
                assert int(got[i, g, c]) == _exact_bf16(exact), (i, g, c)


def test_weighted_compress_uniform_weights_equal_mean():
    k = _bits(_rand_bf16((300, 3, 16), 33))
    w = np.full((3, 32), 1.0 / 32, dtype=np.float32)  # 1/32 is exact, so the sums agree bit for bit
    assert np.array_equal(orc.compress_weighted(k, w, 32, 16), orc.compress(k, 32, 16))


def test_weighted_compress_one_hot_copies_a_token_per_head():
    T, h, d, l, s = 200, 3, 8, 32, 16
    k = _bits(_rand_bf16((T, h, d), 34))
    w = np.zeros((h, l), dtype=np.float32)
    pos = [0, 17, 31]
    for g in range(h):
        w[g, pos[g]] = 1.0
    got = orc.compress_weighted(k, w, l, s)
    for g in range(h):
        want = k[pos[g]::s, g][: got.shape[0]]
        assert np.array_equal(got[:, g], want), g


# ---------------------------------------------------------------- gate network

from oracle import gate as gate_orc  # noqa: E402

# standard normal CDF at 1, -1 and 2 (textbook values)
_PHI_1 = 0.8413447460685429
_PHI_M1 = 0.15865525393145707
_PHI_2 = 0.9772498680518208


def test_gelu_textbook_values():
    got = gate_orc.gelu(np.array([0.0, 1.0, -1.0, 2.0]))
    assert got[0] == 0.0
    assert got[1] == pytest.approx(_PHI_1, abs=1e-15)
    assert got[2] == pytest.approx(-_PHI_M1, abs=1e-15)
    assert got[3] == pytest.approx(2 * _PHI_2, abs=1e-15)
    # x*Phi(x) - (-x)*Phi(-x) = x, for any x
    xs = np.linspace(-6, 6, 101)
    assert np.allclose(gate_orc.gelu(xs) - gate_orc.gelu(-xs), xs, atol=1e-14)


def test_gates_zero_weights_are_softmax_of_bias():
    dim = 8
    x = _bits(_rand_bf16((5, dim), 40))
    w1 = np.zeros((dim // 2, dim), dtype=np.uint16)
    got = gate_orc.gate_mlp(x, w1, np.zeros(dim // 2), np.zeros((3, dim // 2)),
                            np.array([0.0, math.log(2), math.log(3)], dtype=np.float32))
    b2 = np.array([0.0, math.log(2), math.log(3)], dtype=np.float32).astype(np.float64)
    want = np.exp(b2) / np.exp(b2).sum()  # (1, 2, 3)/6 up to the fp32 rounding of the logs
    assert np.allclose(got, want[None, :], atol=1e-15)
    assert np.allclose(want, [1 / 6, 2 / 6, 3 / 6], atol=1e-7)


def test_gates_hand_worked_case_pins_layouts_and_gelu():
    # hidden unit j reads input j with sign (+, -, +); gate c reads hidden unit (c + 2) % 3
    dim, hid = 6, 3
    x = _bits(torch.tensor([[1.0, 1.0, 2.0, 0.0, 0.0, 0.0]], dtype=torch.bfloat16))
    w1 = torch.zeros(hid, dim)
    w1[0, 0], w1[1, 1], w1[2, 2] = 1.0, -1.0, 1.0
    w2 = np.zeros((3, hid), dtype=np.float32)
    w2[0, 2], w2[1, 0], w2[2, 1] = 1.0, 1.0, 1.0
    got = gate_orc.gate_mlp(x, _bits(w1.to(torch.bfloat16)), np.zeros(hid), w2, np.zeros(3))
    logits = [2 * _PHI_2, _PHI_1, -_PHI_M1]
    z = sum(math.exp(v) for v in logits)
    assert np.allclose(got[0], [math.exp(v) / z for v in logits], atol=1e-14)


def _torch_gate_module(dim, w1_bits, b1, w2, b2):
    """The two-layer gate network evaluated with torch.nn.functional in float64."""
    W1 = _f64(w1_bits)
    B1, W2, B2 = (torch.from_numpy(np.asarray(a, np.float32).astype(np.float64)) for a in (b1, w2, b2))

    def mlp(x):
        return torch.nn.functional.linear(torch.nn.functional.gelu(torch.nn.functional.linear(x, W1, B1)), W2, B2)

    return mlp


def _rand_gate_weights(dim, seed):
    g = torch.Generator().manual_seed(seed)
    w1 = _bits((torch.randn(dim // 2, dim, generator=g) / math.sqrt(dim)).to(torch.bfloat16))
    b1 = (torch.randn(dim // 2, generator=g) * 0.1).numpy().astype(np.float32)
    w2 = (torch.randn(3, dim // 2, generator=g) / math.sqrt(dim // 2)).numpy().astype(np.float32)
    b2 = (torch.randn(3, generator=g) * 0.1).numpy().astype(np.float32)
    return w1, b1, w2, b2


@pytest.mark.parametrize("dim", [64, 128])
def test_gates_match_torch_module(dim):
    w1, b1, w2, b2 = _rand_gate_weights(dim, 41)
    x = _bits(_rand_bf16((7, 4, dim), 42))
    got = gate_orc.gate_mlp(x, w1, b1, w2, b2)
    m = _torch_gate_module(dim, w1, b1, w2, b2)
    want = torch.softmax(m(_f64(x)), dim=-1).numpy()
    assert np.allclose(got, want, atol=1e-13)
    assert np.allclose(got.sum(-1), 1.0, atol=1e-14) and (got > 0).all()
    # adding a constant to every logit leaves the gates unchanged
    shifted = gate_orc.gate_mlp(x, w1, b1, w2, b2 + np.float32(3.0))
    assert np.allclose(shifted, got, atol=1e-13)


def test_pooled_gates_match_torch_per_head():
    B, T, H, dim = 2, 9, 3, 64
    w1, b1, w2, b2 = _rand_gate_weights(dim, 43)
    x = _bits(_rand_bf16((B, T, H, dim), 44))
    got = gate_orc.gate_mlp_pooled(x, w1, b1, w2, b2)
    m = _torch_gate_module(dim, w1, b1, w2, b2)
    xf = _f64(x)
    for h in range(H):
        want = torch.softmax(m(xf[:, :, h, :].mean(dim=1)), dim=-1).numpy()  # averaged over tokens, one head
        assert np.allclose(got[:, h], want, atol=1e-13), h
    # tokens that are all equal pool to the per-token gate
    same = np.repeat(x[:, :1], T, axis=1)
    assert np.allclose(gate_orc.gate_mlp_pooled(same, w1, b1, w2, b2),
                       gate_orc.gate_mlp(same[:, 0], w1, b1, w2, b2), atol=1e-14)


# ---------------------------------------------------------------- backward

from oracle import backward as bwd_orc  # noqa: E402


def _bwd_case(N, nv, hq, hkv, d, seed, top_n=4, window=40):
    cfg = orc.OracleConfig(N, nv, hq, hkv, d, top_n=top_n, window=window)
    q = _bits(_rand_bf16((N, hq, d), seed))
    k = _bits(_rand_bf16((N, hkv, d), seed + 1))
    v = _bits(_rand_bf16((N, hkv, d), seed + 2))
    g = torch.rand((N, hq, 3), generator=torch.Generator().manual_seed(seed + 3)).numpy().astype(np.float32)
    dout = _bits(_rand_bf16((N, hq, d), seed + 4))
    o = orc.prefill_rows(cfg, q, k, v, g, np.arange(N, dtype=np.int32), want=("sel",))
    return cfg, q, k, v, g, dout, o


def test_backward_forward_equals_the_forward_oracle():
    # the backward's own forward (key sets, compression, combine, text rows) against the C oracle
    cfg, q, k, v, g, dout, o = _bwd_case(300, 260, 4, 2, 16, 50)
    r = bwd_orc.prefill_backward(cfg, q, k, v, g, dout, o["sel"][: cfg.n_video])
    assert np.abs(r["out"] - o["out"]).max() < 1e-12


def _loss_and_grads(cfg, q, k, v, g, dout, sel, phi=None):
    pk, pv = (None, None) if phi is None else phi
    kc = bwd_orc.compressed_f64(k[: cfg.n_video], cfg, pk, rounded=False)
    vc = bwd_orc.compressed_f64(v[: cfg.n_video], cfg, pv, rounded=False)
    r = bwd_orc.forward_backward(cfg, q, k, v, g, dout, sel, kc, vc, pk, pv)
    return float((r["out"] * dout).sum()), r


@pytest.mark.parametrize("use_phi", [False, True])
def test_backward_finite_differences(use_phi):
    # central differences of L = <dO, out> along random directions, on the smooth forward
    # (exact fp64 summaries): agreement to ~1e-8 relative pins every gradient term
    cfg, qb, kb, vb, g, doutb, o = _bwd_case(150, 130, 4, 2, 8, 60, top_n=3, window=24)
    f = orc.bf16_bits_to_f64
    q, k, v, dout = f(qb), f(kb), f(vb), f(doutb)
    g = g.astype(np.float64)
    sel = o["sel"][: cfg.n_video]
    prng = np.random.default_rng(61)
    phi = tuple((1.0 + 0.5 * prng.standard_normal((2, 32))) / 32 for _ in range(2)) if use_phi else None
    _, r = _loss_and_grads(cfg, q, k, v, g, dout, sel, phi)
    rng = np.random.default_rng(62)
    eps = 1e-5
    for name, x, grad in (("q", q, r["dq"]), ("k", k, r["dk"]), ("v", v, r["dv"]), ("gates", g, r["dgates"])):
        delta = rng.standard_normal(x.shape)
        if name == "gates":
            delta[cfg.n_video:] = 0.0  # text rows ignore their gates
        args = {"q": q, "k": k, "v": v, "gates": g}
        hi = dict(args, **{name: x + eps * delta})
        lo = dict(args, **{name: x - eps * delta})
        lp, _ = _loss_and_grads(cfg, hi["q"], hi["k"], hi["v"], hi["gates"], dout, sel, phi)
        lm, _ = _loss_and_grads(cfg, lo["q"], lo["k"], lo["v"], lo["gates"], dout, sel, phi)
        fd = (lp - lm) / (2 * eps)
        an = float((grad * delta).sum())
        assert abs(fd - an) <= 1e-7 * max(1.0, abs(an)), (name, fd, an)


def test_backward_matches_torch_autograd_dense_masks():
    # an independent formulation: each branch as a dense masked softmax over all keys,
    # differentiated by torch autograd in float64
    cfg, qb, kb, vb, gb, doutb, o = _bwd_case(200, 170, 6, 2, 16, 70, top_n=3, window=30)
    f = orc.bf16_bits_to_f64
    q, k, v, dout = (torch.from_numpy(f(a)).requires_grad_(True) for a in (qb, kb, vb, doutb))
    gates = torch.from_numpy(gb.astype(np.float64)).requires_grad_(True)
    N, nv, hq, hkv, d = cfg.n_tokens, cfg.n_video, cfg.hq, cfg.hkv, cfg.d
    G, l, s, ls = hq // hkv, cfg.cmp_len, cfg.cmp_stride, cfg.sel_len
    sel = o["sel"][:nv]
    scale = 1.0 / math.sqrt(d)
    nc = (nv - l) // s + 1
    kc = torch.stack([k[i * s: i * s + l].mean(0) for i in range(nc)])
    vc = torch.stack([v[i * s: i * s + l].mean(0) for i in range(nc)])
    t_idx = torch.arange(N)[:, None]
    tok = torch.arange(N)[None, :]
    m_cmp = ((torch.arange(nc)[None, :] * s + l - 1) <= t_idx) & (t_idx < nv)
    m_win = (tok <= t_idx) & (tok > t_idx - cfg.window) & (t_idx < nv)
    m_txt = (tok <= t_idx) & (t_idx >= nv)
    m_sel = torch.zeros((hkv, N, N), dtype=torch.bool)
    for t in range(nv):
        for g in range(hkv):
            for j in sel[t, g]:
                if j >= 0:
                    m_sel[g, t, j * ls: min((j + 1) * ls, t + 1)] = True

    def attend(K, V, mask):  # mask [hkv or 1, N, n]
        S = torch.einsum("thd,nhd->htn", q, K.repeat_interleave(G, dim=1)) * scale
        M = mask.repeat_interleave(G, dim=0) if mask.shape[0] == hkv else mask.expand(hq, -1, -1)
        P = torch.softmax(S.masked_fill(~M, float("-inf")), dim=-1)
        P = torch.where(M.any(-1, keepdim=True), P, torch.zeros_like(P))
        return torch.einsum("htn,nhd->thd", P, V.repeat_interleave(G, dim=1))

    out = (gates[..., 0:1] * attend(kc, vc, m_cmp[None]) + gates[..., 1:2] * attend(k, v, m_sel)
           + gates[..., 2:3] * attend(k, v, m_win[None]) + attend(k, v, m_txt[None]))
    (out * dout).sum().backward()
    _, r = _loss_and_grads(cfg, f(qb), f(kb), f(vb), gb.astype(np.float64), f(doutb), sel)
    assert np.abs(out.detach().numpy() - r["out"]).max() < 1e-12
    for name, tg in (("dq", q.grad), ("dk", k.grad), ("dv", v.grad)):
        assert np.abs(tg.numpy() - r[name]).max() < 1e-11, name
    gg = gates.grad.numpy().copy()
    gg[nv:] = 0.0
    assert np.abs(gg - r["dgates"]).max() < 1e-11


def test_backward_value_gradient_sums_to_gated_output_gradient():
    # sum over tokens of dV equals, per group, the sum of dO weighted by the gates of the
    # non-empty branches (probabilities sum to one; the compression's weights sum to one)
    cfg, q, k, v, g, dout, o = _bwd_case(260, 220, 4, 2, 16, 80)
    r = bwd_orc.prefill_backward(cfg, q, k, v, g, dout, o["sel"][: cfg.n_video])
    do = orc.bf16_bits_to_f64(dout)
    G = cfg.hq // cfg.hkv
    w = np.ones((cfg.n_tokens, cfg.hq))
    rows = np.arange(cfg.n_video)
    has_cmp = rows >= cfg.cmp_len - 1
    w[: cfg.n_video] = g[: cfg.n_video, :, 0] * has_cmp[:, None] + g[: cfg.n_video, :, 1] + g[: cfg.n_video, :, 2]
    for grp in range(cfg.hkv):
        hs = slice(grp * G, (grp + 1) * G)
        want = (w[:, hs, None] * do[:, hs]).sum(axis=(0, 1))
        assert np.allclose(r["dv"][:, grp].sum(0), want, atol=1e-10)


# ---------------------------------------------------------------- packed batches, interleaved segments

from oracle import packed as pk_orc  # noqa: E402


def _packed_case(seqs, hq=4, hkv=2, d=16, seed=71, **kw):
    """seqs: per sequence a list of (length, is_video) segments."""
    lens = [sum(n for n, _ in s) for s in seqs]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    seg_lens = [n for s in seqs for n, _ in s]
    seg_vid = [vid for s in seqs for _, vid in s]
    N = int(cu[-1])
    cfg, q, k, v, g = _case(N, hq, hkv, d, seed, **kw)
    return cfg, _bits(q), _bits(k), _bits(v), g.numpy(), cu, seg_lens, seg_vid


def test_packed_trailing_text_equals_the_single_sequence_hybrid():
    """[video][text] in one sequence is the hybrid layout prefill_rows already computes."""
    cfg, q, k, v, g, cu, sl, sv = _packed_case([[(190, True), (70, False)]], top_n=4, window=40)
    o = pk_orc.packed_prefill(cfg, q, k, v, g, cu, sl, sv)
    from dataclasses import replace
    ref = orc.prefill_rows(replace(cfg, n_tokens=260, n_video=190), q, k, v, g, np.arange(260))
    assert np.allclose(o["out"], ref["out"], atol=1e-12, rtol=0)
    assert np.array_equal(o["sel"], ref["sel"][:190])


def test_packed_text_rows_are_dense_over_every_earlier_token():
    """Text rows between and after video segments attend densely to all earlier tokens of
    their own sequence (numpy fp64 softmax, independent of the oracle's C code)."""
    seqs = [[(70, True), (20, False), (90, True), (15, False)], [(40, False), (64, True), (9, False)]]
    cfg, q, k, v, g, cu, sl, sv = _packed_case(seqs, top_n=3, window=32, seed=72)
    o = pk_orc.packed_prefill(cfg, q, k, v, g, cu, sl, sv)
    qd, kd, vd = (orc.bf16_bits_to_f64(x) for x in (q, k, v))
    G = cfg.hq // cfg.hkv
    per = pk_orc.segments_of(cu, sl, sv)
    for b, segs in enumerate(per):
        s0 = int(cu[b])
        for t in pk_orc.text_positions(segs):
            for h in range(cfg.hq):
                z = kd[s0: t + 1, h // G] @ qd[t, h] / math.sqrt(cfg.d)
                p = np.exp(z - z.max())
                ref = (p / p.sum()) @ vd[s0: t + 1, h // G]
                assert np.allclose(o["out"][t, h], ref, atol=1e-12, rtol=0), (b, t, h)


def test_packed_video_rows_ignore_text_segments():
    """Taking the text segments out of a sequence leaves every video row unchanged: video
    positions count in the video stream."""
    seqs = [[(100, True), (30, False), (80, True), (11, False), (50, True)]]
    cfg, q, k, v, g, cu, sl, sv = _packed_case(seqs, top_n=4, window=48, seed=73)
    o = pk_orc.packed_prefill(cfg, q, k, v, g, cu, sl, sv)
    vp = o["video_rows"]
    o2 = pk_orc.packed_prefill(cfg, q[vp], k[vp], v[vp], g[vp], [0, len(vp)], [len(vp)], [True])
    assert np.array_equal(o["out"][vp], o2["out"])
    assert np.array_equal(o["sel"], o2["sel"])


def test_packed_full_budget_video_rows_are_dense_over_the_video_stream():
    """With every block selected and a window covering the stream, the selected and window
    branches of a video row are dense causal attention over the earlier video tokens only
    (torch SDPA on the video tokens alone); text tokens between them are invisible."""
    seqs = [[(80, True), (25, False), (60, True), (7, False), (33, True)]]
    nv = 173
    lens = [n for n, _ in seqs[0]]
    N = sum(lens)
    cfg, q, k, v, _, cu, sl, sv = _packed_case(seqs, top_n=orc.num_sel(nv, 64) + 1, window=nv + 3, seed=74)
    for which in (1, 2):
        g = np.zeros((N, cfg.hq, 3), dtype=np.float32)
        g[..., which] = 1.0
        o = pk_orc.packed_prefill(cfg, q, k, v, g, cu, sl, sv)
        vp = o["video_rows"]
        ref = _sdpa_causal(_f64(q[vp]), _f64(k[vp]), _f64(v[vp]), 1 / math.sqrt(cfg.d)).numpy()
        assert np.allclose(o["out"][vp], ref, atol=1e-12, rtol=0)


def test_packed_sequences_are_independent():
    """A packed batch equals its sequences evaluated one at a time (positions restart)."""
    seqs = [[(120, True), (10, False)], [(33, True)], [(12, False), (70, True), (5, False), (40, True)]]
    cfg, q, k, v, g, cu, sl, sv = _packed_case(seqs, top_n=5, window=60, seed=75)
    o = pk_orc.packed_prefill(cfg, q, k, v, g, cu, sl, sv)
    si = 0
    sels = []
    for b, segs in enumerate(seqs):
        s0, s1 = int(cu[b]), int(cu[b + 1])
        n = len(segs)
        ob = pk_orc.packed_prefill(cfg, q[s0:s1], k[s0:s1], v[s0:s1], g[s0:s1], [0, s1 - s0], sl[si: si + n],
                                   sv[si: si + n])
        assert np.array_equal(o["out"][s0:s1], ob["out"])
        sels.append(ob["sel"])
        si += n
    assert np.array_equal(o["sel"], np.concatenate(sels))


def test_packed_rejects_segments_that_cross_sequences():
    cfg, q, k, v, g, cu, sl, sv = _packed_case([[(50, True)], [(30, False)]])
    with pytest.raises(ValueError):
        pk_orc.packed_prefill(cfg, q, k, v, g, cu, [60, 20], [True, False])
