"""nsa_decode_noalloc: the decode for callers that cannot allocate device memory.

Some callers of this library cannot call cudaMalloc or hand over a scratch buffer (a
plugin whose host framework owns and pre-partitions all device memory and forbids
allocation on its serving path, or a program with a device-memory budget fixed at
start-up). For them nsa_decode_noalloc keeps its scratch in a fixed device array inside
the library. This file is collected last so that a run that stops at the first failure
has already run every other test; it also passes on its own in a fresh process.
"""
import numpy as np
import pytest
import torch

from sparse_attention_long_fwd_b200 import nsa
from sparse_attention_long_fwd_b200.inputs import WORKLOADS, decode_inputs, scaled

from nsa_check import MAX_ABS, MEAN_ABS

pytestmark = pytest.mark.gpu


def _params(w, batch):
    return nsa.make_params(w.n_tokens, w.n_tokens, w.hq, w.hkv, w.d, top_n=w.top_n, window=w.window,
                           out_dtype=nsa.NSA_OUT_F32, batch=batch)


def test_noalloc_decode_matches_workspace_decode_twice():
    w = scaled(WORKLOADS["decode64x128k"], batch=6, n_tokens=6000)
    p = _params(w, w.batch)
    assert nsa.nsa_workspace_size(p, True) <= nsa.NSA_NOALLOC_SCRATCH_BYTES
    # two calls in a row with different inputs and lengths: the second call runs over the
    # scratch the first one left behind
    for call, lens in enumerate(([6000, 5999, 3000, 129, 64, 31], [1, 2048, 6000, 777, 4097, 33])):
        q, kc, vc, g, sl = decode_inputs(w, seed=50 + call, device="cuda", seq_lens=lens)
        kcmp, vcmp = nsa.compress(kc, vc)
        ref, ref_sel = nsa.decode(q, kc, vc, kcmp, vcmp, sl, g, top_n=w.top_n, window=w.window, return_sel=True)
        out = torch.full_like(ref, float("nan"))
        sel = torch.full_like(ref_sel, -9)
        rc = nsa.nsa_decode_noalloc(q, kc, vc, kcmp, vcmp, sl, g, p, out, sel)
        assert rc == nsa.NSA_OK, nsa.nsa_error_string(rc)
        torch.cuda.synchronize()
        assert nsa.nsa_get_device_error(clear=True) == 0
        err = (out.double() - ref.double()).abs()
        assert torch.isfinite(out).all()
        assert err.max().item() <= MAX_ABS and err.mean().item() <= MEAN_ABS, (call, err.max().item())
        assert torch.equal(sel, ref_sel), call


def test_noalloc_decode_rejects_problems_beyond_its_scratch():
    w = WORKLOADS["decode64x128k"]
    p = _params(w, w.batch)  # 64 x 131,072 tokens needs ~78 MB of scratch
    assert nsa.nsa_workspace_size(p, True) > nsa.NSA_NOALLOC_SCRATCH_BYTES
    f = 1 << 20  # never dereferenced: the size check comes first
    assert nsa.nsa_decode_noalloc(f, f, f, f, f, f, f, p, f, None) == nsa.NSA_ERR_NOALLOC_TOO_LARGE
    assert "fixed" in nsa.nsa_error_string(nsa.NSA_ERR_NOALLOC_TOO_LARGE)
