"""GPU parity of the learnable compression and the gate network (C ABI against the fp64 oracle).

Tolerances:
  - learnable compression: bit-exact (both sides round the same exact fp64 sum once);
  - prefill with learnable compression: the prefill's own acceptance (max-abs 1e-2,
    mean-abs 1e-3, selection identical up to near-ties);
  - per-row gates: max-abs 1e-4, mean-abs 1e-6. The first layer accumulates dim exact
    bf16 x bf16 products in fp32 (relative error at most dim * 2^-24 of sum |x w|, ~5e-5
    absolute for N(0,1) inputs and N(0, 1/dim) weights in the worst case, ~1e-6 typical);
    erff, expf and the second layer add a few fp32 ulps; a softmax moves by at most half
    the largest logit error;
  - averaged gates: max-abs 1e-6 (fp64 throughout; only the order of the token sum and
    the final fp32 rounding differ).
"""
import numpy as np
import pytest
import torch

from oracle import gate as gate_orc
from oracle import oracle as orc
from sparse_attention_long_fwd_b200 import nsa
from sparse_attention_long_fwd_b200.inputs import (WORKLOADS, bf16_bits, decode_inputs, gate_weights, phi_weights,
                                                   prefill_inputs, scaled)

from nsa_check import compare_prefill_rows, run_prefill

pytestmark = pytest.mark.gpu
DEV = "cuda"

GATE_MAX_ABS = 1e-4
GATE_MEAN_ABS = 1e-6
POOLED_MAX_ABS = 1e-6


def _np(t):
    return t.detach().cpu().numpy()


# ---------------------------------------------------------------- learnable compression

def test_compress_weighted_bit_exact():
    w = scaled(WORKLOADS["v128k"], n_tokens=4099, n_video=4099)
    q, k, v, g = prefill_inputs(w, seed=5, device=DEV)
    pk, pv = phi_weights(w.hkv, 32, seed=6, device=DEV)
    kc, vc = nsa.compress(k, v, phi=(pk, pv))
    torch.cuda.synchronize()
    assert np.array_equal(bf16_bits(kc), orc.compress_weighted(bf16_bits(k), _np(pk)))
    assert np.array_equal(bf16_bits(vc), orc.compress_weighted(bf16_bits(v), _np(pv)))


def test_compress_weighted_batched_bit_exact_and_uniform_is_mean():
    w = scaled(WORKLOADS["decode64x128k"], batch=3, n_tokens=1000)
    q, kc, vc, g, sl = decode_inputs(w, seed=7, device=DEV)
    pk, pv = phi_weights(w.hkv, 32, seed=8, device=DEV)
    kcmp, vcmp = nsa.compress(kc, vc, phi=(pk, pv))
    torch.cuda.synchronize()
    for b in range(3):
        assert np.array_equal(bf16_bits(kcmp[b]), orc.compress_weighted(bf16_bits(kc[b]), _np(pk)))
        assert np.array_equal(bf16_bits(vcmp[b]), orc.compress_weighted(bf16_bits(vc[b]), _np(pv)))
    uni = torch.full((w.hkv, 32), 1.0 / 32, device=DEV)
    ku, vu = nsa.compress(kc, vc, phi=(uni, uni))
    km, vm = nsa.compress(kc, vc)
    torch.cuda.synchronize()
    assert torch.equal(ku, km) and torch.equal(vu, vm)


@pytest.mark.parametrize("name,n,nv", [("tiny", None, None), ("v128k", 1000, 1000), ("qwen36k_hybrid", 1200, 1000)])
def test_prefill_phi_all_rows(name, n, nv):
    w = WORKLOADS[name] if n is None else scaled(WORKLOADS[name], n_tokens=n, n_video=nv)
    q, k, v, g = prefill_inputs(w, seed=9, device=DEV)
    phi = phi_weights(w.hkv, 32, seed=10, device=DEV)
    out, sel, ws, lay = run_prefill(w, q, k, v, g, phi=phi)
    st = compare_prefill_rows(w, q, k, v, g, np.arange(w.n_tokens), out, sel, ws, lay, phi=phi)
    print(st)


# ---------------------------------------------------------------- gate network

def _gate_close(got, ref, what, max_abs=GATE_MAX_ABS, mean_abs=GATE_MEAN_ABS):
    err = np.abs(got.astype(np.float64) - ref)
    assert np.isfinite(got).all(), what
    assert err.max() <= max_abs and err.mean() <= mean_abs, f"{what}: max {err.max():.3e} mean {err.mean():.3e}"
    return float(err.max()), float(err.mean())


@pytest.mark.parametrize("n,hq,d", [(1000, 28, 128), (777, 8, 64), (1, 3, 128), (5, 1, 64)])
def test_gate_mlp_every_row(n, hq, d):
    """Rows = n * hq: several 128-row tiles and a ragged tail (28,000 = 218 * 128 + 96), plus
    a single partial tile."""
    g = torch.Generator(device=DEV).manual_seed(11)
    x = torch.randn((n, hq, d), generator=g, device=DEV).to(torch.bfloat16)
    w1, b1, w2, b2 = gate_weights(d, seed=12, device=DEV)
    gates = nsa.gate_mlp(x, w1, b1, w2, b2)
    torch.cuda.synchronize()
    assert nsa.nsa_get_device_error(clear=True) == 0
    ref = gate_orc.gate_mlp(bf16_bits(x), bf16_bits(w1), _np(b1), _np(w2), _np(b2))
    print(_gate_close(_np(gates), ref, f"gates n={n} hq={hq} d={d}"))


def test_gate_mlp_full_size_sampled():
    """The 128K workload's queries (3,670,016 rows of d = 128), in the configuration the
    benchmark times: every row sums to one; sampled rows against the oracle."""
    w = WORKLOADS["v128k"]
    q, k, v, g = prefill_inputs(w, seed=13, device=DEV)
    del k, v, g
    w1, b1, w2, b2 = gate_weights(w.d, seed=14, device=DEV)
    gates = nsa.gate_mlp(q, w1, b1, w2, b2)
    torch.cuda.synchronize()
    assert nsa.nsa_get_device_error(clear=True) == 0
    assert torch.isfinite(gates).all()
    assert (gates.sum(-1) - 1).abs().max().item() < 1e-6
    rng = np.random.default_rng(15)
    rows = np.unique(np.concatenate([rng.integers(0, w.n_tokens, 2048), [0, 1, w.n_tokens - 1]]))
    xs = bf16_bits(q[torch.as_tensor(rows, device=DEV)])
    ref = gate_orc.gate_mlp(xs, bf16_bits(w1), _np(b1), _np(w2), _np(b2))
    print(_gate_close(_np(gates[torch.as_tensor(rows, device=DEV)]), ref, "gates v128k"))


def test_gate_mlp_zero_weights_give_softmax_of_bias():
    x = torch.randn((300, 4, 128), device=DEV).to(torch.bfloat16)
    w1 = torch.zeros((64, 128), device=DEV, dtype=torch.bfloat16)
    b1 = torch.zeros(64, device=DEV)
    w2 = torch.zeros((3, 64), device=DEV)
    b2 = torch.tensor([0.0, float(np.log(2.0)), float(np.log(3.0))], device=DEV)
    gates = nsa.gate_mlp(x, w1, b1, w2, b2)
    torch.cuda.synchronize()
    want = np.array([1 / 6, 2 / 6, 3 / 6])
    assert np.abs(_np(gates) - want).max() < 1e-6


@pytest.mark.parametrize("B,T,H,d,repeat", [(2, 1000, 28, 128, 1), (1, 8191, 4, 64, 8191), (3, 7, 2, 128, 7)])
def test_gate_mlp_pooled(B, T, H, d, repeat):
    g = torch.Generator(device=DEV).manual_seed(16)
    x = torch.randn((B, T, H, d), generator=g, device=DEV).to(torch.bfloat16)
    w1, b1, w2, b2 = gate_weights(d, seed=17, device=DEV)
    gates = nsa.gate_mlp_pooled(x, w1, b1, w2, b2, repeat=repeat)
    torch.cuda.synchronize()
    assert nsa.nsa_get_device_error(clear=True) == 0
    ref = gate_orc.gate_mlp_pooled(bf16_bits(x), bf16_bits(w1), _np(b1), _np(w2), _np(b2))
    got = _np(gates)
    assert np.array_equal(got, np.broadcast_to(got[:, :1], got.shape))  # every copy identical
    print(_gate_close(got[:, 0], ref, "pooled gates", max_abs=POOLED_MAX_ABS, mean_abs=POOLED_MAX_ABS))
