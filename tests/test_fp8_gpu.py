"""fa_fwd_fp8 on the GPU against the fp64 oracle on the same E4M3 codes.

Gate, derived from the arithmetic (per output element):
  |O - O_ref| <= 3e-3 + ulp_bf16(O_ref)/2 + 2 u8 * wabs + 2^-10 * vabs / ssum
  - the output is bf16;
  - P enters the fp8 P.V product rounded to E4M3: a relative error of at
    most u8 = 2^-4 for normal weights (first order: u8 * wabs, doubled),
    and an absolute error of at most 2^-10 (half the subnormal spacing
    2^-9) for weights below 2^-6; those sum to at most
    2^-10 * sum_j |v_j| / l, with l >= softmax_sum of the row;
  - all scaled by descale_v.
lse (fp32 normaliser of the unrounded weights) within 1e-3 as the 16-bit
forward."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from exact_attention_113_b200.inputs import F16, Workload, make_qkv_fp8, to_bits
from tests.parity import half_ulp

pytestmark = pytest.mark.gpu
E4M3, BF16 = 2, 1


def _w(**kw):
    base = dict(name="fp8", B=2, H=4, H_kv=4, L_q=300, L_k=300, D=128, dtype=F16, seed=8000)
    base.update(kw)
    return Workload(**base)


def check_fp8(w, descale=(1.0, 1.0, 1.0)):
    import exact_attention_113_b200 as fa
    dq, dk, dv = descale
    q, k, v = make_qkv_fp8(w)
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    out, lse = fa.flash_fwd_fp8(qd, kd, vd, scale=w.softmax_scale, descale_q=dq, descale_k=dk,
                                descale_v=dv, causal=w.causal, window_left=w.window_left,
                                window_right=w.window_right)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == 0
    s_eff = w.softmax_scale * dq * dk
    ref, ref_lse, _, ssum, wabs = oracle.attention_rows_ex(
        to_bits(q), to_bits(k), to_bits(v), E4M3, s_eff, w.causal, w.window_left,
        w.window_right, with_wabs=True)
    ref = ref * dv
    wabs = wabs * dv
    vabs = np.abs(v.float().double().numpy()).sum(axis=2) * dv       # [B, H_kv, D]
    vabs = np.repeat(vabs, w.H // w.H_kv, axis=1)[:, :, None, :]       # per query head
    vabs = np.broadcast_to(vabs, (w.B, w.H, w.L_q, w.D)).reshape(-1, w.D)
    got = out.double().cpu().numpy().reshape(-1, w.D)
    assert np.all(np.isfinite(got))
    with np.errstate(divide="ignore", invalid="ignore"):
        sub = np.where(ssum[:, None] > 0, 2.0 ** -10 * vabs / ssum[:, None], 0.0)
    bound = 3e-3 + half_ulp(ref, BF16) + 2 * 2.0 ** -4 * wabs + sub
    err = np.abs(got - ref)
    assert np.all(err <= bound), (w.name, float(err.max()), float((err - bound).max()))
    gl = lse.cpu().numpy().reshape(-1).astype(np.float64)
    inf = np.isneginf(ref_lse)
    assert np.array_equal(np.isneginf(gl), inf)
    assert np.abs(gl[~inf] - ref_lse[~inf]).max(initial=0) <= 1e-3
    return float(err.max())


@pytest.mark.parametrize("D", [32, 64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_fp8_shapes(D, causal):
    check_fp8(_w(D=D, causal=causal, seed=8000 + D))


@pytest.mark.parametrize("L_q,L_k", [(1, 700), (129, 513), (700, 129), (1000, 1000)])
def test_fp8_lengths(L_q, L_k):
    check_fp8(_w(L_q=L_q, L_k=L_k, D=128, causal=False, seed=8100 + L_q))


def test_fp8_descale():
    check_fp8(_w(D=64, causal=True, seed=8200), descale=(0.5, 2.0, 0.25))


@pytest.mark.parametrize("H,H_kv,L_q", [(8, 2, 300), (8, 2, 5), (16, 1, 17)])
def test_fp8_gqa_and_packing(H, H_kv, L_q):
    check_fp8(_w(H=H, H_kv=H_kv, L_q=L_q, L_k=600, D=128, seed=8300 + H + L_q))


def test_fp8_window():
    check_fp8(_w(L_q=500, L_k=500, D=64, causal=True, window_left=100, seed=8400))
