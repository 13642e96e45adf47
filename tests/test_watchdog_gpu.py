"""The device-side watchdog on a GPU, without faulting it.

Every wait in the kernels is bounded: a wait that does not finish within the
library's limit (1 s) raises the CTA's abort flag and the device status word
and returns, so the other roles of the CTA give up too and the kernel ends.
fa_selftest_wait_timeout runs those same wait routines on an mbarrier phase
that nothing completes (the failure is the missing arrival, made on purpose;
nothing faults, traps or hangs).  The test checks the results, that the
status is reported once and cleared, and that the context still runs a
correct forward afterwards."""
import numpy as np
import pytest
import torch

import exact_attention_113_b200 as fa
import oracle
from exact_attention_113_b200 import inputs as W
from exact_attention_113_b200.inputs import make_qkv, to_bits

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_reports():
    r = fa.selftest_wait_timeout(0)
    assert r["done_ok"] == 1           # a completed phase is seen at once
    assert r["never_ok"] == 0          # the abandoned wait reports failure ...
    assert r["abort_flag"] == 1        # ... raises the CTA's abort flag
    assert 950 <= r["wait_ms"] <= 3000  # ... after the 1 s limit, not sooner
    assert r["follower_ok"] == 0       # a second waiter gives up on the flag,
    assert r["follower_ms"] < 950      # before its own limit (about 0.5 s)
    assert r["status"] == -8           # FA_ERR_TIMEOUT, reported once ...
    assert fa.fa_get_device_status(torch.cuda.current_stream().cuda_stream) == 0  # ... and cleared


def test_context_usable_after_timeout():
    fa.selftest_wait_timeout(0)
    w = W.TINY[0]
    q, k, v = make_qkv(w)
    out, lse = fa.flash_fwd(q.cuda(), k.cuda(), v.cuda(), scale=w.softmax_scale, causal=w.causal)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == 0
    ref, ref_lse = oracle.attention(to_bits(q), to_bits(k), to_bits(v), w.dtype, w.softmax_scale,
                                    w.causal)
    assert np.abs(out.double().cpu().numpy() - ref).max() <= 3e-3 + 2 ** -11
    assert np.abs(lse.double().cpu().numpy() - ref_lse).max() <= 1e-3
