"""Pins of the oracle's masked forward and its softmax statistics (CPU).

The mask's meaning is a reading (attention_ref.c states it); these checks
tie the oracle to it and to facts that hold whatever the code:
  - an all-false bool mask, or an all-zero float mask, changes nothing;
  - a bool mask of the causal pattern equals causal attention, and so does
    a float mask of -inf / 0;
  - adding a constant c_i to a whole row changes O not at all and lse by c_i;
  - an additive mask log(w_j) reweights the keys: O = sum w_j e^{s_j} v_j /
    sum w_j e^{s_j} (brute force in numpy);
  - softmax_max is the row maximum of the masked scores (brute force) and
    lse = softmax_max + ln(softmax_sum);
  - broadcast strides equal the materialised mask."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from exact_attention_113_b200.inputs import BF16, F16, Workload, make_qkv, to_bits

W = Workload(name="m", B=2, H=4, H_kv=2, L_q=9, L_k=11, D=8, dtype=F16, seed=9000)


def _bits(w=W):
    q, k, v = make_qkv(w)
    return to_bits(q), to_bits(k), to_bits(v), q, k, v


def _ex(orc, mask=None, causal=False, scale=0.3, w=W, wl=-1, wr=-1):
    qb, kb, vb, *_ = _bits(w)
    return orc.attention_rows_ex(qb, kb, vb, w.dtype, scale, causal, wl, wr, mask=mask)


def _plain(orc, causal=False, scale=0.3, w=W, wl=-1, wr=-1):
    qb, kb, vb, *_ = _bits(w)
    return orc.attention_rows(qb, kb, vb, w.dtype, scale, causal, wl, wr)


def _causal_bool(L_q=W.L_q, L_k=W.L_k):
    i = np.arange(L_q)[:, None]
    j = np.arange(L_k)[None, :]
    return (j > i)[None, None]                      # true = hidden


def test_empty_masks_change_nothing(orc):
    out0, lse0, _ = _plain(orc)
    for m in (np.zeros((1, 1, W.L_q, W.L_k), dtype=bool),
              np.zeros((W.B, W.H, W.L_q, W.L_k), dtype=np.float32),
              np.zeros((1, W.H, 1, W.L_k), dtype=np.float16)):
        out, lse, _, _ = _ex(orc, m)
        assert np.array_equal(out, out0) and np.array_equal(lse, lse0)


def test_causal_pattern_masks(orc):
    out_c, lse_c, _ = _plain(orc, causal=True)
    hb = _causal_bool()
    hf = np.where(hb, -np.inf, 0.0).astype(np.float32)
    for m in (hb, hf, hf.astype(np.float16)):
        out, lse, _, _ = _ex(orc, m)
        assert np.array_equal(out, out_c) and np.array_equal(lse, lse_c)


def test_row_constant_shift(orc):
    c = np.linspace(-3.0, 5.0, W.L_q).astype(np.float32)
    m = np.broadcast_to(c[None, None, :, None], (1, 1, W.L_q, W.L_k)).copy()
    out0, lse0, _ = _plain(orc, causal=True)
    out, lse, _, _ = _ex(orc, m, causal=True)
    np.testing.assert_allclose(out, out0, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(lse, lse0 + np.tile(c.astype(np.float64), W.B * W.H),
                               rtol=1e-12, atol=1e-12)


def test_log_weight_mask_reweights_keys(orc):
    rng = np.random.default_rng(1)
    wts = rng.uniform(0.1, 3.0, size=W.L_k)
    m = np.log(wts).astype(np.float32)[None, None, None, :]
    out, _, _, _ = _ex(orc, m)
    wts32 = np.exp(m[0, 0, 0].astype(np.float64))   # the weights the fp32 mask encodes
    _, _, _, q, k, v = _bits()
    q, k, v = (t.double().numpy() for t in (q, k, v))
    k = np.repeat(k, W.H // W.H_kv, axis=1)
    v = np.repeat(v, W.H // W.H_kv, axis=1)
    s = 0.3 * q @ k.transpose(0, 1, 3, 2)
    e = wts32 * np.exp(s - s.max(-1, keepdims=True))
    want = (e / e.sum(-1, keepdims=True)) @ v
    np.testing.assert_allclose(out.reshape(want.shape), want, rtol=1e-11, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_statistics(orc, causal):
    m = np.random.default_rng(2).uniform(-2, 2, size=(W.B, 1, W.L_q, W.L_k)).astype(np.float32)
    out, lse, smax, ssum = _ex(orc, m, causal=causal)
    _, _, _, q, k, v = _bits()
    q, k = q.double().numpy(), np.repeat(k.double().numpy(), W.H // W.H_kv, axis=1)
    s = 0.3 * q @ k.transpose(0, 1, 3, 2) + m.astype(np.float64)
    if causal:
        s = np.where(_causal_bool(), -np.inf, s)
    np.testing.assert_allclose(smax, s.max(-1).reshape(-1), rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(lse, smax + np.log(ssum), rtol=1e-13, atol=1e-13)
    assert np.all(ssum >= 1.0)


def test_fully_hidden_rows(orc):
    hb = np.zeros((1, 1, W.L_q, W.L_k), dtype=bool)
    hb[0, 0, 3, :] = True
    out, lse, smax, ssum = _ex(orc, hb)
    rows = np.arange(W.B * W.H * W.L_q) % W.L_q == 3
    assert np.all(out[rows] == 0) and np.all(np.isneginf(lse[rows]))
    assert np.all(np.isneginf(smax[rows])) and np.all(ssum[rows] == 0)


def test_broadcast_strides_equal_materialised(orc):
    rng = np.random.default_rng(3)
    small = rng.uniform(-1, 1, size=(1, W.H, 1, W.L_k)).astype(np.float16)
    full = np.ascontiguousarray(np.broadcast_to(small, (W.B, W.H, W.L_q, W.L_k)))
    a = _ex(orc, small, causal=True)
    b = _ex(orc, full, causal=True)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)
