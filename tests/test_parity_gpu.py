"""GPU parity: the CUDA path (through the C ABI) against the fp64 CPU oracle,
element by element on the same seeded inputs.  Small and medium workloads are
compared in full; the full-size workloads on a deterministic row sample.
Named workloads use the target gate; the extra edge-case shapes use the
derived gate of tests/parity.py (P rounded to the input type)."""
import dataclasses
import math

import numpy as np
import pytest
import torch

import oracle
from exact_attention_113_b200 import inputs as W
from exact_attention_113_b200.inputs import BF16, F16, Workload, make_qkv, to_bits
from tests.parity import check_full, check_rows, compare, run_gpu

pytestmark = pytest.mark.gpu


def _w(**kw):
    base = dict(name="case", B=1, H=2, H_kv=2, L_q=128, L_k=128, D=64, seed=77)
    base.update(kw)
    return Workload(**base)


# ------------------------------------------------------------ named workloads
@pytest.mark.parametrize("w", W.TINY, ids=lambda w: w.name)
def test_tiny(w):
    check_full(w)


def test_gpt2_shape():
    check_full(W.GPT2)


@pytest.mark.parametrize("w", W.MEMTABLE, ids=lambda w: w.name)
def test_memory_table_shape(w):
    check_full(w)


# ------------------------------------------------------------ ragged / edges
EDGE_L = [1, 17, 127, 128, 129, 255, 256, 300, 513]


@pytest.mark.parametrize("D", [16, 32, 64, 128])
@pytest.mark.parametrize("L", EDGE_L)
@pytest.mark.parametrize("causal", [False, True])
def test_ragged_lengths(D, L, causal):
    dtype = BF16 if (L + D) % 2 else F16
    check_full(_w(L_q=L, L_k=L, D=D, dtype=dtype, causal=causal, seed=L * 7 + D), derived=True)


@pytest.mark.parametrize("L_q,L_k", [(1, 300), (300, 1), (129, 700), (700, 129),
                                     (64, 4096), (1000, 250)])
@pytest.mark.parametrize("causal", [False, True])
def test_unequal_lengths(L_q, L_k, causal):
    # rows past the last key under causal/top-left alignment are fully masked
    check_full(_w(L_q=L_q, L_k=L_k, D=64, causal=causal, seed=L_q + 3 * L_k), derived=True)


@pytest.mark.parametrize("wl,wr,causal", [(0, -1, True), (1, -1, True), (127, -1, True),
                                          (128, -1, True), (200, -1, True), (5, 7, False),
                                          (-1, 0, False), (-1, 130, False), (300, 300, False),
                                          (0, 0, False), (1000, -1, True)])
@pytest.mark.parametrize("D", [32, 128])
def test_windows(wl, wr, causal, D):
    check_full(_w(B=2, H=2, H_kv=1, L_q=777, L_k=777, D=D, causal=causal, window_left=wl,
                  window_right=wr, dtype=BF16 if D == 128 else F16, seed=wl + 11 * wr + D),
               derived=True)


@pytest.mark.parametrize("H,H_kv", [(8, 1), (8, 2), (6, 3), (4, 4)])
def test_gqa_mqa(H, H_kv):
    check_full(_w(B=2, H=H, H_kv=H_kv, L_q=333, L_k=333, D=128, causal=True, seed=H * 10 + H_kv), derived=True)


def test_fully_masked_rows_give_zero_and_neg_inf():
    w = _w(L_q=600, L_k=200, D=64, causal=True, window_left=0)
    stats = check_full(w, derived=True)
    q, k, v = make_qkv(w)
    out, lse = run_gpu(q, k, v, w)
    assert torch.all(out[:, :, 200:] == 0)
    assert torch.all(torch.isneginf(lse[:, :, 200:]))


def test_scale_zero_is_mean_of_visible_values():
    w = _w(L_q=300, L_k=300, D=64, causal=True, scale=0.0)
    check_full(w)


def test_empty_keys_and_queries():
    import exact_attention_113_b200 as fa
    q = torch.randn(1, 2, 5, 64, device="cuda", dtype=torch.float16)
    k = torch.randn(1, 2, 0, 64, device="cuda", dtype=torch.float16)
    out, lse = fa.flash_fwd(q, k, k)
    torch.cuda.synchronize()
    assert torch.all(out == 0) and torch.all(torch.isneginf(lse))
    q0 = torch.randn(1, 2, 0, 64, device="cuda", dtype=torch.float16)
    out0, lse0 = fa.flash_fwd(q0, q, q)
    assert out0.numel() == 0 and lse0.numel() == 0


def test_without_lse():
    w = _w(L_q=500, L_k=500, D=128, causal=True)
    check_full(w, with_lse=False)


# ------------------------------------------------------------ properties
def test_gqa_equals_mha_with_repeated_heads_bitwise():
    w = _w(B=2, H=8, H_kv=2, L_q=1000, L_k=1000, D=128, dtype=BF16, causal=True)
    q, k, v = make_qkv(w)
    o1, l1 = run_gpu(q, k, v, w)
    wm = dataclasses.replace(w, H_kv=8)
    o2, l2 = run_gpu(q, k.repeat_interleave(4, dim=1), v.repeat_interleave(4, dim=1), wm)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_deterministic():
    w = _w(B=1, H=4, H_kv=4, L_q=2000, L_k=2000, D=64, causal=False)
    q, k, v = make_qkv(w)
    o1, l1 = run_gpu(q, k, v, w)
    o2, l2 = run_gpu(q, k, v, w)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


# ------------------------------------------------------------ full-size, sampled
@pytest.mark.parametrize("w", W.SWEEP, ids=lambda w: w.name)
def test_sweep_sampled(w):
    check_rows(w, W.sample_rows(w, per_head_random=4))


def test_gqa_window_full_size_sampled():
    w = W.GQA_WINDOW
    check_rows(w, W.sample_rows(w, per_head_random=4))


def test_roofline_config_sampled():
    w = W.ROOFLINE
    check_rows(w, W.sample_rows(w, per_head_random=4))


def test_device_status_clean_at_end():
    import exact_attention_113_b200 as fa
    assert fa.fa_get_device_status() == 0


# ------------------------------------------------------------ GQA packing
# With H / H_kv a power of two and L_q < 128, one 128-row tile holds
# 128 / group query positions of each head of a group (the Q / O boxes are
# [group, 128 / group, cols]); (12, 2) is a group of 6 and stays unpacked.
@pytest.mark.parametrize("H,H_kv", [(4, 2), (8, 2), (16, 2), (32, 4), (128, 1), (12, 2)])
@pytest.mark.parametrize("L_q", [1, 5, 31, 32, 33, 127])
def test_gqa_packed_short_queries(H, H_kv, L_q):
    check_full(_w(B=2, H=H, H_kv=H_kv, L_q=L_q, L_k=700, D=128, seed=5000 + H + L_q))


@pytest.mark.parametrize("wl,wr,causal", [(-1, -1, True), (16, -1, True), (-1, 650, False),
                                          (200, 40, False)])
@pytest.mark.parametrize("D", [32, 64])
def test_gqa_packed_masks(wl, wr, causal, D):
    check_full(_w(B=1, H=16, H_kv=4, L_q=100, L_k=700, D=D, causal=causal, window_left=wl,
                  window_right=wr, seed=5100 + D), derived=True)


def test_gqa_packed_matches_repeated_heads():
    # the packed tile and the per-head tile compute the same rows; they may
    # differ in the last bits (rows of one warp share rescale decisions)
    w = _w(B=2, H=8, H_kv=2, L_q=20, L_k=3000, D=128, dtype=BF16, seed=5200)
    q, k, v = make_qkv(w)
    o1, l1 = run_gpu(q, k, v, w)
    wm = dataclasses.replace(w, H_kv=8)
    o2, l2 = run_gpu(q, k.repeat_interleave(4, dim=1), v.repeat_interleave(4, dim=1), wm)
    assert (o1.float() - o2.float()).abs().max().item() <= 2 * 3e-3 + 4e-3   # two gates
    assert (l1 - l2).abs().max().item() <= 1e-4


# ------------------------------------------------------------ non-power-of-two head dims
# Rows of 96, 160, 192 and 224 bytes: 32-, 32-, 64- and 32-byte swizzle
# atoms (3, 5, 3, 7 per row); O chunks with a 16-column tail.
@pytest.mark.parametrize("D", [48, 80, 96, 112])
@pytest.mark.parametrize("L", [1, 129, 300])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("dtype", [F16, BF16])
def test_non_pow2_head_dims(D, L, causal, dtype):
    check_full(_w(H=3, H_kv=3, L_q=L, L_k=L, D=D, causal=causal, dtype=dtype,
                  seed=5300 + D + L), derived=True)


@pytest.mark.parametrize("D", [48, 96])
def test_non_pow2_gqa_packed_and_long(D):
    check_full(_w(B=2, H=8, H_kv=2, L_q=20, L_k=1500, D=D, seed=5400 + D))
    check_full(_w(B=1, H=2, H_kv=2, L_q=2000, L_k=2000, D=D, causal=True, seed=5410 + D),
               derived=True)


@pytest.mark.parametrize("D", [80, 112])
def test_non_pow2_split_kv(D):
    check_full(_w(B=1, H=4, H_kv=4, L_q=3, L_k=3000, D=D, seed=5500 + D), n_splits=5)
