"""Decoding shapes (a few query rows per K/V head, a long cache) on the GPU
against the fp64 oracle.

Problems with at most two query rows per K/V head (one new token per head,
two tokens, or a GQA group of two) run on the CUDA-core decode kernel
(fa_decode_kernel.cuh): fa_fwd as whole heads, fa_fwd_splitkv /
fa_fwd_fp8_splitkv as equal key ranges merged by the split-KV merge kernel.
That kernel keeps the weights in fp32 (it has no tensor-core P.V product),
so the target gate of tests/parity.py applies, with its aggregate check.
GQA groups of three and four (and longer query ranges, 7 and 16 rows) run on
the tensor-core kernel and are checked beside them.  Workspaces start
NaN-filled, so a partial that no slice wrote poisons its row."""
from __future__ import annotations

import pytest
import torch

from exact_attention_113_b200.inputs import BF16, F16, Workload, make_qkv
from tests.parity import check_full, run_gpu

pytestmark = pytest.mark.gpu

SHAPES = {"mha_1": dict(L_q=1, H=8, H_kv=8), "mha_2": dict(L_q=2, H=4, H_kv=4),
          "gqa2_1": dict(L_q=1, H=8, H_kv=4), "gqa3_1": dict(L_q=1, H=6, H_kv=2),
          "gqa4_1": dict(L_q=1, H=8, H_kv=2), "gqa2_2": dict(L_q=2, H=8, H_kv=4)}


def _w(name, **kw):
    base = dict(B=2, H=4, H_kv=4, L_q=1, L_k=1000, D=64, dtype=F16, seed=5000)
    base.update(kw)
    return Workload(name=name, **base)


def _check(w, **kw):
    """check_full with the target gate on the decode kernel's shapes and the
    derived gate (P rounded to the input type) on the tensor-core ones."""
    kw.setdefault("derived", w.L_q * (w.H // w.H_kv) > 2)
    return check_full(w, **kw)


@pytest.mark.parametrize("D", [16, 32, 64, 128])
@pytest.mark.parametrize("dtype", [F16, BF16])
@pytest.mark.parametrize("shape", sorted(SHAPES))
@pytest.mark.parametrize("n_splits", [0, 1, 5])
def test_decode_shapes(D, dtype, shape, n_splits):
    w = _w(f"dec_{shape}_d{D}", D=D, dtype=dtype, L_k=2500, seed=5000 + D + dtype,
           **SHAPES[shape])
    _check(w, n_splits=n_splits)


@pytest.mark.parametrize("L_k", [1, 2, 63, 64, 65, 127, 129, 4097])
@pytest.mark.parametrize("n_splits", [0, 3])
def test_ragged_cache_lengths(L_k, n_splits):
    _check(_w("dec_ragged", L_k=L_k, D=64, seed=5100 + L_k), n_splits=n_splits)


@pytest.mark.parametrize("n_splits", [17, 64])
def test_more_slices_than_chunks(n_splits):
    # 300 keys = 5 chunks of 64: most slices are empty and merge as nothing
    _check(_w("dec_empty_slices", L_k=300, D=128, dtype=BF16, seed=5200),
               n_splits=n_splits)


@pytest.mark.parametrize("shape", sorted(SHAPES))
@pytest.mark.parametrize("mask", ["causal", "speculative", "window", "window_causal"])
def test_masks(shape, mask):
    L_k = 3000
    kw = dict(SHAPES[shape])
    if mask == "causal":            # top-left aligned: row i sees keys 0..i
        kw.update(causal=True)
    elif mask == "speculative":     # the new rows sit at the end of the cache
        kw.update(window_right=L_k - kw["L_q"])
    elif mask == "window":
        kw.update(window_left=0, window_right=200)
    else:
        kw.update(causal=True, window_left=1)
    w = _w(f"dec_{mask}", L_k=L_k, D=128, dtype=BF16, seed=5300, **kw)
    for n_splits in (0, 4):
        _check(w, n_splits=n_splits)


def test_large_values_move_the_reference_maximum():
    # std 4: scores spread over a wide range, so the reference maximum moves
    # past the rescale threshold from chunk to chunk
    for n_splits in (0, 6):
        _check(_w("dec_std4", L_k=5000, D=128, std=4.0, seed=5400, **SHAPES["gqa2_1"]),
                   n_splits=n_splits)


def test_many_heads_round_robin():
    # more work items than SMs: the persistent grid walks several per CTA
    w = _w("dec_many", B=8, H=48, H_kv=48, L_q=1, L_k=1111, D=64, seed=5500)
    for n_splits in (0, 2, 9):
        _check(w, n_splits=n_splits)


def test_without_lse_and_fully_masked_rows():
    w = _w("dec_nolse", L_k=700, D=32, seed=5600, **SHAPES["mha_2"])
    _check(w, with_lse=False, n_splits=3)
    # window_left 0 and causal on two rows of a one-key cache: row 1 sees nothing
    w2 = _w("dec_masked", L_k=1, D=64, causal=True, window_left=0, seed=5601, **SHAPES["mha_2"])
    q, k, v = make_qkv(w2)
    out, lse = run_gpu(q, k, v, w2, True, n_splits=0)
    assert torch.all(out[:, :, 1] == 0) and torch.all(torch.isneginf(lse[:, :, 1]))
    _check(w2)


@pytest.mark.parametrize("L_q", [7, 16])
def test_longer_query_ranges_on_the_tensor_core_path(L_q):
    for n_splits in (0, 4):
        _check(_w("dec_lq", L_q=L_q, H=8, H_kv=8, L_k=3000, D=64, seed=5700 + L_q),
                   n_splits=n_splits, derived=True)


@pytest.mark.parametrize("D", [32, 64, 128])
@pytest.mark.parametrize("shape", ["mha_1", "gqa2_1", "gqa4_1"])
@pytest.mark.parametrize("n_splits", [0, 4])
def test_fp8_cache(D, shape, n_splits):
    from tests.test_fp8_gpu import _w as w8, check_fp8
    check_fp8(w8(L_k=3000, D=D, seed=5800 + D, **SHAPES[shape]), descale=(0.5, 2.0, 0.25),
              n_splits=n_splits)

