"""fa_fwd_host (host buffers, chunked copies overlapped with the kernels)
against the device-buffer forward and the oracle.

Each chunk runs the same kernel on a contiguous range of K/V heads (whole
GQA groups), so the result equals fa_fwd on the whole problem within the
forward's gate; the tiny case is also checked against the oracle."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from exact_attention_113_b200.inputs import BF16, F16, Workload, make_qkv, to_bits
from tests.parity import compare

pytestmark = pytest.mark.gpu


def _w(**kw):
    base = dict(name="host", B=2, H=8, H_kv=4, L_q=300, L_k=300, D=64, dtype=F16, seed=8500)
    base.update(kw)
    return Workload(**base)


@pytest.mark.parametrize("n_chunks", [1, 3, 8, 100])
@pytest.mark.parametrize("pinned", [True, False])
def test_matches_device_forward(n_chunks, pinned):
    import exact_attention_113_b200 as fa
    w = _w(causal=True, seed=8500 + n_chunks)
    q, k, v = make_qkv(w)
    hq, hk, hv = (t.pin_memory() if pinned else t for t in (q, k, v))
    out, lse = fa.flash_fwd_host(hq, hk, hv, scale=w.softmax_scale, causal=True,
                                 n_chunks=n_chunks)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == 0
    ref, ref_lse = fa.flash_fwd(q.cuda(), k.cuda(), v.cuda(), scale=w.softmax_scale, causal=True)
    torch.cuda.synchronize()
    assert (out.float() - ref.float().cpu()).abs().max().item() <= 2e-3
    assert (lse - ref_lse.cpu()).abs().max().item() <= 1e-4


def test_against_oracle():
    import exact_attention_113_b200 as fa
    w = _w(B=1, H=4, H_kv=2, L_q=200, L_k=333, D=128, dtype=BF16, seed=8600)
    q, k, v = make_qkv(w)
    out, lse = fa.flash_fwd_host(q.pin_memory(), k.pin_memory(), v.pin_memory(),
                                 scale=w.softmax_scale, n_chunks=2)
    torch.cuda.synchronize()
    ref, ref_lse, _ = oracle.attention_rows(to_bits(q), to_bits(k), to_bits(v), w.dtype,
                                            w.softmax_scale, False, -1, -1)
    compare(out.float().numpy().reshape(-1, w.D), lse.numpy().reshape(-1), ref, ref_lse,
            w.dtype, w.name)


def test_back_to_back_calls_share_the_pipeline():
    import exact_attention_113_b200 as fa
    for seed in (8700, 8701, 8702):
        w = _w(H=4, H_kv=4, L_q=129, L_k=700, D=96, dtype=BF16, seed=seed)
        q, k, v = make_qkv(w)
        out, lse = fa.flash_fwd_host(q.pin_memory(), k.pin_memory(), v.pin_memory(),
                                     scale=w.softmax_scale, n_chunks=3)
        torch.cuda.synchronize()
        ref, _ = fa.flash_fwd(q.cuda(), k.cuda(), v.cuda(), scale=w.softmax_scale)
        torch.cuda.synchronize()
        assert (out.float() - ref.float().cpu()).abs().max().item() <= 4e-3


def test_empty_keys():
    import exact_attention_113_b200 as fa
    q = torch.randn(1, 2, 5, 64, dtype=torch.float16).pin_memory()
    k = torch.empty(1, 2, 0, 64, dtype=torch.float16).pin_memory()
    out, lse = fa.flash_fwd_host(q, k, k, n_chunks=2)
    torch.cuda.synchronize()
    assert torch.all(out == 0) and torch.all(torch.isneginf(lse))
