"""Pins of the oracle's backward (CPU only).

The pages print no gradient formulas (they only say the backward recomputes
the attention matrix from Q, K, V and the saved softmax statistics), so the
oracle's backward is the plain definition: the gradient of sum(dO * O).
These checks tie it to things other than its own formulas:
  - central finite differences of the oracle's fp64 forward;
  - torch fp64 autograd of softmax(scale Q K^T + mask) V (library autograd,
    independent of the C code);
  - closed forms: one key (dQ = dK = 0, dV = sum of dO), scale 0 (uniform
    weights), constant values (dQ = dK = 0);
  - GQA: a shared head's gradient is the sum over the heads that read it;
  - linearity in dO, and the bit-pattern entry equals the fp64 entry;
  - the error scales bound the gradients and carry the delta term."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from exact_attention_113_b200.inputs import BF16, F16

CASES = [
    dict(B=1, H=2, H_kv=1, L_q=5, L_k=7, D=4, causal=False, wl=-1, wr=-1),
    dict(B=1, H=2, H_kv=2, L_q=6, L_k=6, D=3, causal=True, wl=-1, wr=-1),
    dict(B=2, H=4, H_kv=2, L_q=7, L_k=9, D=5, causal=False, wl=2, wr=1),
    # rows 6 and 7 see no key (i - 1 > L_k - 1): fully masked
    dict(B=1, H=1, H_kv=1, L_q=8, L_k=5, D=4, causal=True, wl=1, wr=-1),
]
IDS = ["gqa_plain", "causal", "window", "masked_rows"]


def _inputs(c, seed=0):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((c["B"], c["H"], c["L_q"], c["D"]))
    k = rng.standard_normal((c["B"], c["H_kv"], c["L_k"], c["D"]))
    v = rng.standard_normal((c["B"], c["H_kv"], c["L_k"], c["D"]))
    do = rng.standard_normal((c["B"], c["H"], c["L_q"], c["D"]))
    return q, k, v, do


def _bwd(orc, c, q, k, v, do, scale=0.7, **kw):
    return orc.attention_bwd_f64(q, k, v, do, scale, c["causal"], c["wl"], c["wr"], **kw)


@pytest.mark.parametrize("c", CASES, ids=IDS)
def test_finite_differences_of_the_forward(orc, c):
    q, k, v, do = _inputs(c, 1)
    scale = 0.7
    dq, dk, dv = _bwd(orc, c, q, k, v, do, scale)

    def f(qq, kk, vv):
        out, _ = orc.attention_f64(qq, kk, vv, scale, c["causal"], c["wl"], c["wr"])
        return float((out * do).sum())

    eps = 1e-5
    rng = np.random.default_rng(2)
    for idx, (x, g) in enumerate(((q, dq), (k, dk), (v, dv))):
        for flat in rng.choice(x.size, size=min(x.size, 24), replace=False):
            pos = np.unravel_index(flat, x.shape)
            xp, xm = x.copy(), x.copy()
            xp[pos] += eps
            xm[pos] -= eps
            args_p = [q, k, v]
            args_m = [q, k, v]
            args_p[idx], args_m[idx] = xp, xm
            fd = (f(*args_p) - f(*args_m)) / (2 * eps)
            assert abs(fd - g[pos]) <= 1e-7 * (1 + abs(g[pos])), (idx, pos, fd, g[pos])


def _torch_attention(q, k, v, scale, causal, wl, wr):
    B, H, L_q, D = q.shape
    H_kv, L_k = k.shape[1], k.shape[2]
    kk = k.repeat_interleave(H // H_kv, dim=1)
    vv = v.repeat_interleave(H // H_kv, dim=1)
    i = torch.arange(L_q).view(-1, 1)
    j = torch.arange(L_k).view(1, -1)
    vis = torch.ones(L_q, L_k, dtype=torch.bool)
    if causal:
        vis &= j <= i
    if wl >= 0:
        vis &= j >= i - wl
    if wr >= 0:
        vis &= j <= i + wr
    s = scale * q @ kk.transpose(-1, -2)
    s = s.masked_fill(~vis, float("-inf"))
    p = torch.softmax(s, dim=-1)
    p = torch.where(vis.any(dim=-1, keepdim=True), p, torch.zeros_like(p))
    return p @ vv


@pytest.mark.parametrize("c", CASES, ids=IDS)
def test_matches_torch_fp64_autograd(orc, c):
    q, k, v, do = _inputs(c, 3)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    out = _torch_attention(tq, tk, tv, 0.7, c["causal"], c["wl"], c["wr"])
    out.backward(torch.tensor(do))
    dq, dk, dv = _bwd(orc, c, q, k, v, do)
    np.testing.assert_allclose(dq, tq.grad.numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(dk, tk.grad.numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(dv, tv.grad.numpy(), rtol=1e-11, atol=1e-12)


def test_single_key(orc):
    # one key: P = 1 for every row, so dS = 0 and dV sums dO over the
    # query rows of every head that reads the key
    c = dict(B=2, H=4, H_kv=2, L_q=3, L_k=1, D=6, causal=False, wl=-1, wr=-1)
    q, k, v, do = _inputs(c, 4)
    dq, dk, dv = _bwd(orc, c, q, k, v, do)
    assert np.all(dq == 0) and np.all(dk == 0)
    want = do.reshape(2, 2, 2, 3, 6).sum(axis=(2, 3)).reshape(2, 2, 1, 6)
    np.testing.assert_allclose(dv, want, rtol=1e-14, atol=1e-14)


def test_scale_zero(orc):
    # uniform weights 1/n_i over each row's visible keys; no score gradient
    c = dict(B=1, H=1, H_kv=1, L_q=6, L_k=6, D=3, causal=True, wl=-1, wr=-1)
    q, k, v, do = _inputs(c, 5)
    dq, dk, dv = _bwd(orc, c, q, k, v, do, scale=0.0)
    assert np.all(dq == 0) and np.all(dk == 0)
    want = np.zeros_like(dv)
    for i in range(6):
        for j in range(i + 1):
            want[0, 0, j] += do[0, 0, i] / (i + 1)
    np.testing.assert_allclose(dv, want, rtol=1e-13, atol=1e-14)


def test_constant_values(orc):
    # every value row equal: O does not depend on the weights, so dQ = dK = 0
    c = CASES[2]
    q, k, v, do = _inputs(c, 6)
    v[:] = v[:, :, :1, :]
    dq, dk, _ = _bwd(orc, c, q, k, v, do)
    assert np.abs(dq).max() < 1e-13 and np.abs(dk).max() < 1e-13


def test_gqa_gradient_sums_the_group(orc):
    c = dict(B=1, H=6, H_kv=2, L_q=5, L_k=8, D=4, causal=True, wl=-1, wr=-1)
    q, k, v, do = _inputs(c, 7)
    dq, dk, dv = _bwd(orc, c, q, k, v, do)
    cm = dict(c, H_kv=6)
    dq_m, dk_m, dv_m = _bwd(orc, cm, q, np.repeat(k, 3, axis=1), np.repeat(v, 3, axis=1), do)
    np.testing.assert_allclose(dq, dq_m, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(dk, dk_m.reshape(1, 2, 3, 8, 4).sum(axis=2), rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(dv, dv_m.reshape(1, 2, 3, 8, 4).sum(axis=2), rtol=1e-13, atol=1e-14)


def test_linear_in_dout(orc):
    c = CASES[0]
    q, k, v, do = _inputs(c, 8)
    g1 = _bwd(orc, c, q, k, v, do)
    g2 = _bwd(orc, c, q, k, v, 2.0 * do)
    for a, b in zip(g1, g2):
        assert np.array_equal(2.0 * a, b)


@pytest.mark.parametrize("dtype", [F16, BF16])
def test_bit_pattern_entry_decodes_exactly(orc, dtype):
    c = CASES[1]
    q, k, v, do = _inputs(c, 9)
    tdt = torch.float16 if dtype == F16 else torch.bfloat16
    bits = [torch.tensor(x).to(tdt).view(torch.int16).numpy().view(np.uint16)
            for x in (q, k, v, do)]
    dec = [torch.tensor(x).to(tdt).double().numpy() for x in (q, k, v, do)]
    g1 = orc.attention_bwd(*bits, dtype, 0.5, True)
    g2 = orc.attention_bwd_f64(*dec, 0.5, True)
    for a, b in zip(g1, g2):
        assert np.array_equal(a, b)


def test_error_scales(orc):
    c = CASES[2]
    q, k, v, do = _inputs(c, 10)
    dq, dk, dv, dqa, dka, dva = _bwd(orc, c, q, k, v, do, with_abs=True)
    assert np.all(dqa >= np.abs(dq) - 1e-12) and np.all(dka >= np.abs(dk) - 1e-12)
    assert np.all(dva >= np.abs(dv) - 1e-12)
    # with dO >= 0 the weighted magnitude is dV itself
    _, _, dv_pos, _, _, dva_pos = _bwd(orc, c, q, k, v, np.abs(do), with_abs=True)
    np.testing.assert_allclose(dva_pos, dv_pos, rtol=1e-14, atol=0)
    # one key: dS = 0, so the scales are the delta term alone
    c1 = dict(B=1, H=1, H_kv=1, L_q=2, L_k=1, D=3, causal=False, wl=-1, wr=-1)
    q, k, v, do = _inputs(c1, 11)
    e = np.array([0.25, 0.5]).reshape(1, 1, 2)
    dq, dk, dv, dqa, dka, dva = _bwd(orc, c1, q, k, v, do, scale=0.7, delta_err=e,
                                     with_abs=True)
    np.testing.assert_allclose(dqa[0, 0], 0.7 * e[0, 0, :, None] * np.abs(k[0, 0, 0]),
                               rtol=1e-14)
    np.testing.assert_allclose(dka[0, 0, 0], 0.7 * (e[0, 0, :, None] * np.abs(q[0, 0])).sum(0),
                               rtol=1e-14)


def test_module_level_entries():
    # the GPU tests call these through the module
    import oracle
    c = CASES[0]
    q, k, v, do = _inputs(c, 12)
    assert np.array_equal(oracle.attention_bwd_f64(q, k, v, do, 0.7)[0],
                          oracle.get().attention_bwd_f64(q, k, v, do, 0.7)[0])
    assert callable(oracle.attention_bwd) and callable(oracle.attention_f64)


# ------------------------------------------------------------ with a mask
def test_masked_backward_finite_differences(orc):
    # an additive mask is a constant: the gradient of the masked forward
    c = CASES[0]
    q, k, v, do = _inputs(c, 13)
    rng = np.random.default_rng(14)
    m = rng.uniform(-2, 2, size=(1, c["H"], c["L_q"], c["L_k"])).astype(np.float32)
    m[0, 0, 1, :3] = -np.inf                                         # hidden keys
    dq, dk, dv = orc.attention_bwd_f64(q, k, v, do, 0.7, mask=m)

    def f(qq, kk, vv):
        return float((_masked_forward(qq, kk, vv, m) * do).sum())

    eps = 1e-5
    for idx, (x, g) in enumerate(((q, dq), (k, dk), (v, dv))):
        for flat in np.random.default_rng(15).choice(x.size, size=12, replace=False):
            pos = np.unravel_index(flat, x.shape)
            xp, xm = x.copy(), x.copy()
            xp[pos] += eps
            xm[pos] -= eps
            a, b = [q, k, v], [q, k, v]
            a[idx], b[idx] = xp, xm
            fd = (f(*a) - f(*b)) / (2 * eps)
            assert abs(fd - g[pos]) <= 1e-7 * (1 + abs(g[pos])), (idx, pos, fd, g[pos])


def _masked_forward(q, k, v, m):
    # fp64 forward with an additive mask (numpy; the same rule written out)
    H, H_kv = q.shape[1], k.shape[1]
    kk = np.repeat(k, H // H_kv, axis=1)
    vv = np.repeat(v, H // H_kv, axis=1)
    s = 0.7 * q @ kk.transpose(0, 1, 3, 2) + m.astype(np.float64)
    mx = s.max(-1, keepdims=True)
    e = np.exp(s - mx)
    return (e / e.sum(-1, keepdims=True)) @ vv


def test_masked_backward_matches_torch_autograd(orc):
    c = CASES[2]
    q, k, v, do = _inputs(c, 16)
    rng = np.random.default_rng(17)
    hide = rng.uniform(size=(c["B"], 1, c["L_q"], c["L_k"])) < 0.3
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    kk = tk.repeat_interleave(c["H"] // c["H_kv"], dim=1)
    vv = tv.repeat_interleave(c["H"] // c["H_kv"], dim=1)
    i = torch.arange(c["L_q"]).view(-1, 1)
    j = torch.arange(c["L_k"]).view(1, -1)
    vis = (j >= i - c["wl"]) & (j <= i + c["wr"]) & ~torch.tensor(hide)
    s = (0.7 * tq @ kk.transpose(-1, -2)).masked_fill(~vis, float("-inf"))
    p = torch.softmax(s, dim=-1)
    p = torch.where(vis.any(dim=-1, keepdim=True), p, torch.zeros_like(p))
    (p @ vv).backward(torch.tensor(do))
    dq, dk, dv = orc.attention_bwd_f64(q, k, v, do, 0.7, False, c["wl"], c["wr"], mask=hide)
    np.testing.assert_allclose(dq, tq.grad.numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(dk, tk.grad.numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(dv, tv.grad.numpy(), rtol=1e-11, atol=1e-12)


def test_causal_pattern_mask_equals_causal_backward(orc):
    c = CASES[1]
    q, k, v, do = _inputs(c, 18)
    i = np.arange(c["L_q"])[:, None]
    j = np.arange(c["L_k"])[None, :]
    g1 = orc.attention_bwd_f64(q, k, v, do, 0.7, True)
    g2 = orc.attention_bwd_f64(q, k, v, do, 0.7, False, mask=(j > i)[None, None])
    for a, b in zip(g1, g2):
        assert np.array_equal(a, b)
