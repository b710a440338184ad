"""Failure detection on the GPU without a fault.

Every wait inside the library's kernels is bounded: when a wait runs out it sets bit 0 of
the device error word, and the kernel drains its own work and returns instead of hanging.
nsa_selftest_wait_timeout runs that exact wait on a barrier that nothing ever arrives at,
with a budget of about a millisecond, so the timeout path is exercised for real: no trap,
no bad address and no endless loop are involved, and the context must stay usable."""
import numpy as np
import pytest
import torch

from sparse_attention_long_fwd_b200 import nsa
from sparse_attention_long_fwd_b200.inputs import WORKLOADS, prefill_inputs, scaled

from nsa_check import compare_prefill_rows, run_prefill

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_reports():
    assert nsa.nsa_get_device_error(clear=True) == 0
    # ~1 ms at 1.9 GHz: the wait must give up, record the timeout and let the kernel return
    assert nsa.nsa_selftest_wait_timeout(2_000_000) == nsa.NSA_OK
    torch.cuda.synchronize()
    word = nsa.nsa_get_device_error(clear=True)
    assert word & 1, f"timeout bit not set (word {word})"
    assert word == 1, f"unexpected bits (word {word})"
    # cleared, and it stays clear when nothing times out
    assert nsa.nsa_get_device_error(clear=True) == 0


def test_context_usable_after_a_timeout():
    assert nsa.nsa_selftest_wait_timeout(500_000) == nsa.NSA_OK
    assert nsa.nsa_get_device_error(clear=True) == 1
    w = scaled(WORKLOADS["tiny"], n_tokens=300, n_video=300)
    q, k, v, g = prefill_inputs(w, seed=77, device="cuda")
    out, sel, ws, lay = run_prefill(w, q, k, v, g)  # also asserts the error word stays 0
    compare_prefill_rows(w, q, k, v, g, np.arange(300), out, sel, ws, lay)


def test_selftest_rejects_out_of_range_budgets():
    assert nsa.nsa_selftest_wait_timeout(0) == nsa.NSA_ERR_INVALID_ARG
    assert nsa.nsa_selftest_wait_timeout(5_000_000_000) == nsa.NSA_ERR_INVALID_ARG
