"""fa_bwd on the GPU against the fp64 oracle's gradients.

Inputs: seeded Q, K, V, dO; O and lse from the oracle's forward (O rounded
to the input type as a forward would write it, lse rounded to fp32), or from
the GPU forward in the end-to-end test.

Gate, derived from the arithmetic of the kernel (per element of dQ, dK, dV):
  |g - g_ref| <= ulp(g_ref)/2 + 2u * g_abs + t_sub + 1e-6
  - ulp/2: the gradient is rounded to the input type;
  - u = 2^-8 (bf16) / 2^-11 (fp16): P (for dV) and dS (for dK, dQ) enter
    the tensor cores rounded to the input type, a relative error u each;
    the factor 2 covers second-order terms and fp32 accumulation;
  - delta_i = dO_i . O_i is computed from the given O instead of the exact
    O*, an absolute error of at most
    e_i = sum_d |dO_id| (|O_id - O*_id| + 2^-23 |O_id|), which moves dS_ij
    by P_ij e_i (not relative to anything);
  - g_abs (from the oracle) is the product with |P| (dV) or |dS| + P e'
    (dK, dQ) and |operands|; the oracle is given e' = e / (2u), so that
    2u * g_abs = 2u * (rounding part) + 1 * (delta part);
  - t_sub (fp16 only): weights below 2^-14 are subnormal in fp16, absolute
    error 2^-25 each, over n summed terms of the largest operand."""
from __future__ import annotations

import dataclasses

import numpy as np
import pytest
import torch

import oracle
from exact_attention_113_b200.inputs import (BF16, F16, TORCH_DTYPE, Workload, make_dout,
                                             make_qkv, to_bits)
from tests.parity import half_ulp

pytestmark = pytest.mark.gpu
U = {F16: 2.0 ** -11, BF16: 2.0 ** -8}


def _w(**kw):
    base = dict(name="bwd", B=1, H=2, H_kv=2, L_q=128, L_k=128, D=64, seed=6000)
    base.update(kw)
    return Workload(**base)


def _oracle_forward(w, q, k, v, mask=None):
    out, lse, _, _ = oracle.attention_rows_ex(to_bits(q), to_bits(k), to_bits(v), w.dtype,
                                              w.softmax_scale, w.causal, w.window_left,
                                              w.window_right, mask=mask)
    return out.reshape(w.B, w.H, w.L_q, w.D), lse.reshape(w.B, w.H, w.L_q)


def check_bwd(w: Workload, o_lse_from_gpu: bool = False, mask=None):
    """``mask``: a CPU torch mask (bool / float16 / float32, broadcastable
    to [B, H, L_q, L_k]) used by the forward and the backward."""
    import exact_attention_113_b200 as fa
    q, k, v = make_qkv(w)
    do = make_dout(w)
    mnp = None if mask is None else mask.numpy()
    md = None if mask is None else mask.cuda()
    o_exact, lse_exact = _oracle_forward(w, q, k, v, mnp)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    if o_lse_from_gpu:
        out, lse = fa.flash_fwd(qd, kd, vd, scale=w.softmax_scale, causal=w.causal,
                                window_left=w.window_left, window_right=w.window_right)[:2] \
            if mask is None else \
            fa.flash_fwd(qd, kd, vd, scale=w.softmax_scale, causal=w.causal,
                         window_left=w.window_left, window_right=w.window_right, mask=md)[:2]
    else:
        out = torch.from_numpy(o_exact).to(TORCH_DTYPE[w.dtype]).cuda()
        lse = torch.from_numpy(lse_exact).float().cuda()
    dq = torch.full_like(qd, float("nan"))
    dk = torch.full_like(kd, float("nan"))
    dv = torch.full_like(vd, float("nan"))
    fa.flash_bwd(qd, kd, vd, out, dod, lse, scale=w.softmax_scale, causal=w.causal,
                 window_left=w.window_left, window_right=w.window_right, dq=dq, dk=dk, dv=dv,
                 mask=md)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == 0, "device watchdog fired"

    o_in = out.double().cpu().numpy()
    do64 = do.double().numpy()
    u = U[w.dtype]
    e = (np.abs(do64) * (np.abs(o_in - o_exact) + 2.0 ** -23 * np.abs(o_in))).sum(-1)
    dq_r, dk_r, dv_r, dq_a, dk_a, dv_a = oracle.attention_bwd(
        to_bits(q), to_bits(k), to_bits(v), to_bits(do), w.dtype, w.softmax_scale, w.causal,
        w.window_left, w.window_right, delta_err=e / (2 * u), with_abs=True, mask=mnp)
    group = w.H // w.H_kv
    sub = 2.0 ** -25 if w.dtype == F16 else 0.0
    stats = {}
    for name, g, ref, gabs, n_terms, opnd in (
            ("dq", dq, dq_r, dq_a, w.L_k, w.softmax_scale * np.abs(k.double().numpy()).max(initial=0)),
            ("dk", dk, dk_r, dk_a, w.L_q * group, w.softmax_scale * np.abs(q.double().numpy()).max(initial=0)),
            ("dv", dv, dv_r, dv_a, w.L_q * group, np.abs(do64).max(initial=0))):
        got = g.double().cpu().numpy()
        assert np.all(np.isfinite(got)), f"{w.name} {name}: non-finite (unwritten?) values"
        err = np.abs(got - ref)
        bound = half_ulp(ref, w.dtype) + 2 * u * gabs + sub * n_terms * opnd + 1e-6
        bad = err > bound
        stats[name] = float(err.max(initial=0.0))
        assert not bad.any(), (f"{w.name} {name}: {int(bad.sum())} beyond the gate; max err "
                               f"{err.max():.3g}, at {np.unravel_index((err - bound).argmax(), err.shape)}")
    return stats


@pytest.mark.parametrize("dtype", [F16, BF16])
@pytest.mark.parametrize("causal", [False, True])
def test_tiny(dtype, causal):
    check_bwd(_w(dtype=dtype, causal=causal, seed=6001))


@pytest.mark.parametrize("D", [16, 32, 64, 128])
@pytest.mark.parametrize("L", [1, 17, 129, 300])
@pytest.mark.parametrize("causal", [False, True])
def test_ragged_lengths(D, L, causal):
    check_bwd(_w(L_q=L, L_k=L, D=D, causal=causal, dtype=BF16, seed=6100 + L + D))


@pytest.mark.parametrize("L_q,L_k", [(1, 300), (300, 1), (129, 700), (700, 129)])
@pytest.mark.parametrize("causal", [False, True])
def test_unequal_lengths(L_q, L_k, causal):
    check_bwd(_w(L_q=L_q, L_k=L_k, D=128, causal=causal, dtype=F16, seed=6200 + L_q))


@pytest.mark.parametrize("wl,wr,causal", [(0, -1, True), (127, -1, True), (200, 50, False),
                                          (-1, 0, False), (64, 64, False)])
def test_windows(wl, wr, causal):
    check_bwd(_w(L_q=400, L_k=400, D=64, causal=causal, window_left=wl, window_right=wr,
                 seed=6300))


@pytest.mark.parametrize("H,H_kv", [(8, 2), (8, 1), (6, 3)])
def test_gqa(H, H_kv):
    check_bwd(_w(B=2, H=H, H_kv=H_kv, L_q=300, L_k=300, D=128, causal=True, dtype=BF16,
                 seed=6400 + H + H_kv))


@pytest.mark.parametrize("D", [16, 32, 48])
@pytest.mark.parametrize("dtype", [F16, BF16])
def test_small_head_dims_over_many_steps(D, dtype):
    # the four-warpgroup layout (D <= 64) and, at D = 16, P^T in its own
    # TMEM columns with S^T of the next step started early: GQA groups of
    # three heads, a causal window, several query blocks per key block
    check_bwd(_w(B=2, H=6, H_kv=2, L_q=520, L_k=520, D=D, causal=True, window_left=300,
                 dtype=dtype, seed=6450 + D + dtype))


def test_fully_masked_rows():
    # rows 200.. see no key: lse = -inf, their dq is 0, they add nothing
    w = _w(L_q=500, L_k=200, D=64, causal=True, window_left=0, seed=6500)
    check_bwd(w)


def test_scale_zero():
    check_bwd(_w(L_q=300, L_k=300, D=64, scale=0.0, causal=True, seed=6600))


def test_larger_causal_bf16():
    check_bwd(_w(B=2, H=4, H_kv=4, L_q=1024, L_k=1024, D=128, causal=True, dtype=BF16,
                 seed=6700))


def test_end_to_end_with_gpu_forward():
    # O and lse from the GPU forward; the gate's delta term uses its real
    # deviation from the exact output
    check_bwd(_w(B=1, H=4, H_kv=2, L_q=700, L_k=700, D=128, causal=True, dtype=BF16,
                 seed=6800), o_lse_from_gpu=True)


def test_empty():
    import exact_attention_113_b200 as fa
    q = torch.randn(1, 2, 0, 64, device="cuda", dtype=torch.float16)
    k = torch.randn(1, 2, 9, 64, device="cuda", dtype=torch.float16)
    lse = torch.empty(1, 2, 0, device="cuda")
    dq, dk, dv = fa.flash_bwd(q, k, k, q, q, lse)
    torch.cuda.synchronize()
    assert torch.all(dk == 0) and torch.all(dv == 0) and dq.numel() == 0
    q = torch.randn(1, 2, 7, 64, device="cuda", dtype=torch.float16)
    k = torch.randn(1, 2, 0, 64, device="cuda", dtype=torch.float16)
    lse = torch.full((1, 2, 7), float("-inf"), device="cuda")
    dq, dk, dv = fa.flash_bwd(q, k, k, q, q, lse)
    torch.cuda.synchronize()
    assert torch.all(dq == 0) and dk.numel() == 0


# ------------------------------------------------------------ with a mask
def _mask(shape, kind, seed, p_hide=0.3):
    g = torch.Generator().manual_seed(seed)
    if kind == "bool":
        return torch.rand(shape, generator=g) < p_hide
    x = torch.randn(shape, generator=g)
    x = torch.where(torch.rand(shape, generator=g) < p_hide, torch.tensor(float("-inf")), x)
    return x.to(torch.float16 if kind == "f16" else torch.float32)


@pytest.mark.parametrize("kind", ["bool", "f16", "f32"])
@pytest.mark.parametrize("D", [64, 128])
def test_masked(kind, D):
    w = _w(B=2, H=4, H_kv=2, L_q=300, L_k=333, D=D, dtype=BF16, seed=6900 + D)
    check_bwd(w, mask=_mask((w.B, w.H, w.L_q, w.L_k), kind, 6910 + D))


@pytest.mark.parametrize("shape", ["qk", "key_padding"])
def test_masked_broadcast_and_causal(shape):
    w = _w(B=2, H=4, H_kv=4, L_q=257, L_k=257, D=32, causal=True, dtype=F16, seed=6950)
    dims = (1, 1, w.L_q, w.L_k) if shape == "qk" else (w.B, 1, 1, w.L_k)
    check_bwd(w, mask=_mask(dims, "f32", 6951))


def test_masked_end_to_end_with_gpu_forward():
    w = _w(B=1, H=4, H_kv=2, L_q=500, L_k=500, D=128, dtype=BF16, seed=6960)
    check_bwd(w, o_lse_from_gpu=True, mask=_mask((w.B, w.H, w.L_q, w.L_k), "bool", 6961))


# ------------------------------------------------------------ non-power-of-two head dims
# 16-column fp32 dQ boxes (64-byte swizzle) when D is an odd multiple of 16,
# a partial last drain round (D = 80, 96, 112), one dO stage at D = 112
@pytest.mark.parametrize("D", [48, 80, 96, 112])
@pytest.mark.parametrize("causal", [False, True])
def test_non_pow2_head_dims(D, causal):
    check_bwd(_w(B=1, H=4, H_kv=2, L_q=300, L_k=300, D=D, causal=causal, dtype=BF16,
                 seed=7100 + D))


def test_non_pow2_with_mask():
    w = _w(B=1, H=2, H_kv=2, L_q=257, L_k=333, D=80, dtype=F16, seed=7200)
    check_bwd(w, mask=_mask((1, 1, w.L_q, w.L_k), "f32", 7201))
