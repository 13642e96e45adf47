"""fa_fwd_splitkv on the GPU against the fp64 oracle.

The key range of each query tile is cut into n_splits slices, each slice
written as an unnormalised partial with its (max, normaliser), then merged
with the online-softmax rescaling ("FlashAttention算法原理与性能优化实战"
§1.2.2; the hierarchical blocking of its §6.1).  The merge changes only the
order of fp32 additions, so the gate is the one of the plain forward.
Workspaces start NaN-filled: a partial the kernel fails to write poisons the
merged row."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from exact_attention_113_b200 import inputs as W
from exact_attention_113_b200.inputs import BF16, F16, Workload, make_qkv
from tests.parity import check_full, check_rows, run_gpu

pytestmark = pytest.mark.gpu


def _w(name, **kw):
    base = dict(B=1, H=4, H_kv=4, L_q=1, L_k=1000, D=64, dtype=BF16, seed=3000)
    base.update(kw)
    return Workload(name=name, **base)


@pytest.mark.parametrize("D", [16, 32, 64, 128])
@pytest.mark.parametrize("dtype", [F16, BF16])
@pytest.mark.parametrize("n_splits", [1, 3, 8])
def test_decode_one_query(D, dtype, n_splits):
    w = _w(f"dec_d{D}", D=D, dtype=dtype, H=8, H_kv=2, L_k=4097, seed=3001 + D)
    check_full(w, n_splits=n_splits)


@pytest.mark.parametrize("L_q", [16, 129, 300])
@pytest.mark.parametrize("n_splits", [2, 5])
@pytest.mark.parametrize("causal", [False, True])
def test_several_query_tiles(L_q, n_splits, causal):
    w = _w("dec_tiles", L_q=L_q, L_k=1500, D=128, causal=causal, seed=3010)
    check_full(w, n_splits=n_splits, derived=causal)


@pytest.mark.parametrize("n_splits", [7, 64])
def test_more_slices_than_key_blocks(n_splits):
    # 300 keys = 3 blocks: most slices are empty and must merge as nothing
    w = _w("dec_empty_slices", L_q=5, L_k=300, D=64, dtype=F16, seed=3020)
    check_full(w, n_splits=n_splits)


@pytest.mark.parametrize("wl,wr", [(200, 0), (1000, 32), (-1, 0), (64, -1)])
def test_windows(wl, wr):
    w = _w("dec_window", L_q=260, L_k=2000, D=128, window_left=wl, window_right=wr,
           seed=3030)
    check_full(w, n_splits=4, derived=True)


def test_speculative_queries_at_the_end_of_the_cache():
    L_q, L_k = 16, 5000
    w = _w("dec_spec", H=8, H_kv=2, L_q=L_q, L_k=L_k, D=128, window_right=L_k - L_q,
           seed=3040)
    check_full(w, n_splits=6)


def test_fully_masked_rows():
    # window_left 0 with causal: row i sees key i only; rows past L_k see nothing
    w = _w("dec_masked", L_q=300, L_k=200, D=64, causal=True, window_left=0, seed=3050)
    q, k, v = make_qkv(w)
    out, lse = run_gpu(q, k, v, w, True, n_splits=3)
    assert torch.all(out[:, :, 200:] == 0)
    assert torch.all(torch.isneginf(lse[:, :, 200:]))
    check_full(w, n_splits=3, derived=True)


def test_empty_keys_and_queries():
    import exact_attention_113_b200 as fa
    q = torch.randn(1, 2, 7, 64, device="cuda", dtype=torch.float16)
    k = torch.empty(1, 2, 0, 64, device="cuda", dtype=torch.float16)
    out, lse = fa.flash_fwd(q, k, k, n_splits=4)
    torch.cuda.synchronize()
    assert torch.all(out == 0) and torch.all(torch.isneginf(lse))
    q0 = torch.empty(1, 2, 0, 64, device="cuda", dtype=torch.float16)
    k1 = torch.randn(1, 2, 9, 64, device="cuda", dtype=torch.float16)
    out, lse = fa.flash_fwd(q0, k1, k1, n_splits=4)
    torch.cuda.synchronize()
    assert out.numel() == 0 and fa.fa_get_device_status() == 0


def test_without_lse():
    check_full(_w("dec_nolse", L_q=3, L_k=3000, seed=3060), with_lse=False, n_splits=5)


@pytest.mark.parametrize("n_splits", [2, 9])
def test_matches_plain_forward(n_splits):
    # same inputs through fa_fwd and fa_fwd_splitkv: both within the gate of
    # the oracle, and within a few fp32 roundings of each other
    w = _w("dec_vs_plain", B=2, H=8, H_kv=8, L_q=200, L_k=3000, D=128, dtype=F16,
           seed=3070)
    q, k, v = make_qkv(w)
    o1, l1 = run_gpu(q, k, v, w, True)
    o2, l2 = run_gpu(q, k, v, w, True, n_splits=n_splits)
    assert (o1.float() - o2.float()).abs().max().item() <= 2e-3
    assert (l1 - l2).abs().max().item() <= 1e-4


def test_workspace_reuse_across_shapes():
    # one workspace serves two calls of different shapes in a row
    import exact_attention_113_b200 as fa
    wa = _w("dec_reuse_a", H=8, L_q=40, L_k=2500, D=128, seed=3080)
    wb = _w("dec_reuse_b", H=2, H_kv=2, L_q=7, L_k=900, D=32, dtype=F16, seed=3081)
    nbytes = max(fa.fa_splitkv_workspace_bytes(w.B, w.H, w.L_q, w.D, 6) for w in (wa, wb))
    ws = torch.full((nbytes // 4,), float("nan"), device="cuda").view(torch.uint8)
    for w in (wa, wb, wa):
        q, k, v = (t.cuda() for t in make_qkv(w))
        out, lse = fa.flash_fwd(q, k, v, scale=w.softmax_scale, n_splits=6, workspace=ws)
        ref = fa.flash_fwd(q, k, v, scale=w.softmax_scale)[0]
        torch.cuda.synchronize()
        assert (out.float() - ref.float()).abs().max().item() <= 4e-3


def test_auto_splits_runs():
    w = _w("dec_auto", H=8, H_kv=2, L_q=1, L_k=20000, D=128, seed=3090)
    q, k, v = (t.cuda() for t in make_qkv(w))
    import exact_attention_113_b200 as fa
    out, _ = fa.flash_fwd(q, k, v, n_splits="auto")
    ref, _ = fa.flash_fwd(q, k, v)
    torch.cuda.synchronize()
    assert (out.float() - ref.float()).abs().max().item() <= 4e-3


@pytest.mark.parametrize("w", W.DECODE, ids=lambda w: w.name)
def test_decode_workloads_sampled(w):
    import exact_attention_113_b200 as fa
    rows = np.arange(w.B * w.H * w.L_q, dtype=np.int64)     # every row: a few hundred
    check_rows(w, rows, n_splits=fa.choose_splits(w.B, w.H, w.L_q, w.L_k, H_kv=w.H_kv))
