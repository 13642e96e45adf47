"""fa_fwd_splitkv_static (the split-KV forward on the library's static
scratch, for callers that cannot allocate device memory) against the
existing split-KV entry point with a caller workspace, and against the fp64
oracle.

Collected last on purpose: the static entry does its one-time set-up (the
scratch's device address) on its first call, and these tests must pass both
alone and after every other test in the same process.  The pages have no
counterpart to this entry point; the gate is the parity gate of the plain
forward (3e-3 + half an output ulp on O, 1e-3 on lse, and the aggregate
check of tests/parity.py against the oracle)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import exact_attention_113_b200 as fa
from exact_attention_113_b200.inputs import BF16, F16, Workload, make_qkv
from tests.parity import LSE_TOL, O_TOL, compare, half_ulp, reference

pytestmark = pytest.mark.gpu


def _run(w, n_splits, static):
    q, k, v = (t.cuda() for t in make_qkv(w))
    out = torch.full_like(q, float("nan"))
    lse = torch.full((w.B, w.H, w.L_q), float("nan"), dtype=torch.float32, device="cuda")
    fa.flash_fwd(q, k, v, scale=w.softmax_scale, causal=w.causal,
                 window_left=w.window_left, window_right=w.window_right, out=out, lse=lse,
                 n_splits=n_splits, workspace="static" if static else None)
    return out, lse


def _close(a, b, dtype):
    a64 = a.double().cpu().numpy()
    b64 = b.double().cpu().numpy()
    assert np.all(np.isfinite(a64))
    assert np.all(np.abs(a64 - b64) <= O_TOL + half_ulp(b64, dtype))


CASES = [
    Workload(name="static_decode_gqa", B=4, H=16, H_kv=4, L_q=1, L_k=9000, D=128,
             dtype=BF16, seed=4001),
    Workload(name="static_spec_causal", B=2, H=8, H_kv=8, L_q=40, L_k=3000, D=64,
             dtype=F16, window_right=3000 - 40, seed=4002),
]


def test_two_calls_in_a_row_match_the_workspace_entry():
    # two different problems back to back on the one scratch
    for w, n_splits in ((CASES[0], 8), (CASES[1], 5)):
        out_s, lse_s = _run(w, n_splits, static=True)
        out_w, lse_w = _run(w, n_splits, static=False)
        torch.cuda.synchronize()
        assert fa.fa_get_device_status() == 0
        _close(out_s, out_w, w.dtype)
        assert (lse_s - lse_w).abs().max().item() <= LSE_TOL


def test_repeated_calls_are_stable():
    w = CASES[0]
    first, _ = _run(w, 8, static=True)
    second, _ = _run(w, 8, static=True)
    ref, _ = fa.flash_fwd(*(t.cuda() for t in make_qkv(w)), scale=w.softmax_scale)
    torch.cuda.synchronize()
    _close(first, ref, w.dtype)
    _close(second, ref, w.dtype)


def test_oversized_problem_is_refused():
    # 32768 query rows x 2 slices need 33.5 MB of partials, more than the
    # 16 MiB scratch: refused with FA_ERR_SCRATCH, nothing launched
    q = torch.zeros(1, 64, 512, 128, dtype=torch.float16, device="cuda")
    k = torch.zeros(1, 64, 256, 128, dtype=torch.float16, device="cuda")
    assert fa.fa_splitkv_workspace_bytes(1, 64, 512, 128, 2) > fa.binding.STATIC_SCRATCH_BYTES
    with pytest.raises(fa.FaError) as e:
        fa.flash_fwd(q, k, k, n_splits=2, workspace="static")
    assert e.value.status == -10


def _against_oracle(w, out, lse):
    ref, ref_lse, pr, heads = reference(w, *make_qkv(w))
    compare(out.float().cpu().numpy().reshape(-1, w.D), lse.cpu().numpy().reshape(-1), ref,
            ref_lse, w.dtype, w.name, pr, False, heads)


def test_matches_the_oracle():
    for w, n_splits in ((CASES[0], 8), (CASES[1], 5)):
        out, lse = _run(w, n_splits, static=True)
        torch.cuda.synchronize()
        assert fa.fa_get_device_status() == 0
        _against_oracle(w, out, lse)


def test_large_call_then_small_call_on_one_stream():
    # a call that fills much of the scratch (many rows, many slices), then a
    # smaller one with another head dim on the same stream: the second reads
    # only partials it wrote itself
    big = Workload(name="static_big", B=8, H=32, H_kv=8, L_q=4, L_k=4096, D=128,
                   dtype=F16, seed=4003)
    small = Workload(name="static_small_d16", B=3, H=4, H_kv=2, L_q=7, L_k=1500, D=16,
                     dtype=BF16, causal=True, seed=4004)
    assert fa.fa_splitkv_workspace_bytes(big.B, big.H, big.L_q, big.D, 16) > \
        fa.fa_splitkv_workspace_bytes(small.B, small.H, small.L_q, small.D, 3)
    out_b, lse_b = _run(big, 16, static=True)
    out_s, lse_s = _run(small, 3, static=True)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == 0
    _against_oracle(small, out_s, lse_s)
    _against_oracle(big, out_b, lse_b)


def test_one_slice_and_empty_keys():
    w = Workload(name="static_one_slice", B=2, H=4, H_kv=4, L_q=3, L_k=700, D=64,
                 dtype=F16, seed=4005)
    out, lse = _run(w, 1, static=True)
    torch.cuda.synchronize()
    _against_oracle(w, out, lse)
    # no keys: O = 0 and lse = -inf, nothing read from the scratch
    q = torch.randn(1, 2, 5, 64, device="cuda", dtype=torch.float16)
    k = torch.zeros(1, 2, 0, 64, device="cuda", dtype=torch.float16)
    out0, lse0 = fa.flash_fwd(q, k, k, n_splits=4, workspace="static")
    torch.cuda.synchronize()
    assert torch.all(out0 == 0) and torch.all(torch.isneginf(lse0))
