"""fa_fwd_fp8 on the GPU against the fp64 oracle on the same E4M3 codes.

Gate (tests/parity.py, derived from the arithmetic, per output element):
  |O - O_ref| <= 3e-3 + ulp_bf16(O_ref)/2 + min(worst, 8 sigma_P)
  - the output is bf16;
  - P enters the fp8 P.V product rounded to E4M3: a relative error of at
    most u8 = 2^-4 for normal weights, and an absolute error of at most
    2^-10 (half the subnormal spacing 2^-9) for weights below 2^-6,
    divided by the kernel's normaliser, which is at least softmax_sum;
  - worst = u8 * wabs + 2^-10 * sum_j |v_j| / ssum (every error at its
    bound with one sign); sigma_P = sqrt((u8 wrss)^2 + (2^-10 vrss /
    ssum)^2) / sqrt(3), the standard deviation of independent roundings;
  - all scaled by descale_v;
plus the aggregate check of tests/parity.py: per head, the mean of
error^2 over the model's variance stays below 1.5, which a head scaled by
1 + 2^-4 or a dropped key block exceeds (tests/test_gate_sensitivity.py).
lse (fp32 normaliser of the unrounded weights) within 1e-3 as the 16-bit
forward."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from exact_attention_113_b200.inputs import F16, Workload, make_qkv_fp8, to_bits
from tests.parity import compare, reference

pytestmark = pytest.mark.gpu
E4M3, BF16 = 2, 1


def _w(**kw):
    base = dict(name="fp8", B=2, H=4, H_kv=4, L_q=300, L_k=300, D=128, dtype=F16, seed=8000)
    base.update(kw)
    return Workload(**base)


def check_fp8(w, descale=(1.0, 1.0, 1.0), n_splits=0, mask=None, stats=False):
    import exact_attention_113_b200 as fa
    dq, dk, dv = descale
    q, k, v = make_qkv_fp8(w)
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    ws = None
    if n_splits:
        # NaN-filled: a partial the merge reads but no slice wrote poisons its row
        nb = fa.fa_splitkv_workspace_bytes(w.B, w.H, w.L_q, w.D, n_splits)
        ws = torch.full((nb // 4,), float("nan"), dtype=torch.float32,
                        device="cuda").view(torch.uint8)
    kw = {}
    if mask is not None or stats:
        kw = dict(mask=None if mask is None else mask.cuda(), return_softmax_stats=stats)
    res = fa.flash_fwd_fp8(qd, kd, vd, scale=w.softmax_scale, descale_q=dq, descale_k=dk,
                           descale_v=dv, causal=w.causal, window_left=w.window_left,
                           window_right=w.window_right, n_splits=n_splits, workspace=ws, **kw)
    out, lse = res[0], res[1]
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == 0
    s_eff = w.softmax_scale * dq * dk
    m = None if mask is None else mask.numpy()
    ref, ref_lse, pr, heads, ref_max, ssum = reference(w, q, k, v, mask=m, in_dtype=E4M3,
                                                       scale=s_eff, out_scale=dv, stats=True)
    got = out.double().cpu().numpy().reshape(-1, w.D)
    st = compare(got, None, ref, None, E4M3, w.name, pr, True, heads, out_dtype=BF16)
    gl = lse.cpu().numpy().reshape(-1).astype(np.float64)
    inf = np.isneginf(ref_lse)
    assert np.array_equal(np.isneginf(gl), inf)
    assert np.abs(gl[~inf] - ref_lse[~inf]).max(initial=0) <= 1e-3
    if stats:
        gm = res[2].cpu().numpy().reshape(-1).astype(np.float64)
        gs = res[3].cpu().numpy().reshape(-1).astype(np.float64)
        minf = np.isneginf(ref_max)
        assert np.array_equal(np.isneginf(gm), minf)
        assert np.all(gs[minf] == 0)
        assert np.abs(gm[~minf] - ref_max[~minf]).max(initial=0) <= 1e-3
        assert np.all(np.abs(gs[~minf] - ssum[~minf]) <= 1e-3 * ssum[~minf])
    return st["o_max_abs"]


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


# ------------------------------------------------------------ split-KV (fp8 cache)
# fa_fwd_fp8_splitkv: the key range in slices, merged with descale_v into
# bf16; the same gate as the single pass (the slices only reorder the fp32
# sums).
@pytest.mark.parametrize("D", [32, 64, 128])
@pytest.mark.parametrize("n_splits", [1, 3, 8])
def test_fp8_splitkv_decode(D, n_splits):
    check_fp8(_w(B=2, H=8, H_kv=2, L_q=1, L_k=3000, D=D, seed=8500 + D), n_splits=n_splits)


@pytest.mark.parametrize("L_q,causal", [(16, False), (300, True)])
def test_fp8_splitkv_tiles(L_q, causal):
    check_fp8(_w(B=1, H=4, H_kv=4, L_q=L_q, L_k=2500, D=128, causal=causal, seed=8600 + L_q),
              descale=(0.5, 2.0, 0.25), n_splits=5)


def test_fp8_splitkv_more_slices_than_blocks_and_window():
    check_fp8(_w(B=1, H=2, H_kv=1, L_q=3, L_k=200, D=64, seed=8700), n_splits=9)
    check_fp8(_w(B=1, H=4, H_kv=2, L_q=200, L_k=1200, D=128, causal=True, window_left=300,
                 seed=8710), n_splits=4)


def test_fp8_splitkv_matches_single_pass():
    import exact_attention_113_b200 as fa
    w = _w(B=2, H=16, H_kv=4, L_q=1, L_k=8192, D=128, seed=8800)
    q, k, v = (t.cuda() for t in make_qkv_fp8(w))
    o1, l1 = fa.flash_fwd_fp8(q, k, v, descale_v=0.5)
    o2, l2 = fa.flash_fwd_fp8(q, k, v, descale_v=0.5, n_splits="auto")
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == 0
    # both bf16 roundings of nearly the same fp32 value
    assert (o1.float() - o2.float()).abs().max().item() <= 2 * 2.0 ** -8
    assert (l1 - l2).abs().max().item() <= 1e-4


# ------------------------------------------------------------ both D = 128 schedules
# One query tile per CTA (fewer 128-row tiles than SMs) takes the dual
# softmax, more tiles the two-tile ping-pong: B 2 x H 40 at L_q 300 is 240
# tiles (ping-pong), B 1 x H 3 is 9 (dual).  std 3 moves the running max
# past the rescale threshold inside blocks.
@pytest.mark.parametrize("shape", ["two", "one"])
@pytest.mark.parametrize("causal,std", [(False, 1.0), (True, 1.0), (False, 3.0)])
def test_fp8_both_schedules(shape, causal, std):
    hw = dict(B=2, H=40, H_kv=40) if shape == "two" else dict(B=1, H=3, H_kv=3)
    check_fp8(_w(L_q=300, L_k=400, D=128, causal=causal, std=std,
                 seed=8900 + int(causal) + int(std), **hw))


# ------------------------------------------------------------ mask and statistics
# fa_fwd_fp8_ex: the 16-bit mask semantics on the full-scale fp8 scores.
@pytest.mark.parametrize("shape", ["two", "one"])
@pytest.mark.parametrize("D,kind", [(128, "bool"), (64, "f32"), (32, "f16")])
def test_fp8_mask_and_stats(shape, D, kind):
    from tests.test_mask_gpu import _mask
    hw = dict(B=2, H=40, H_kv=40) if shape == "two" else dict(B=2, H=4, H_kv=2)
    w = _w(L_q=300, L_k=333, D=D, seed=9600 + D, **hw)
    check_fp8(w, descale=(0.5, 2.0, 0.25), mask=_mask((w.B, w.H, w.L_q, w.L_k), kind, 9700 + D),
              stats=True)


def test_fp8_broadcast_mask_with_causal():
    from tests.test_mask_gpu import _mask
    w = _w(B=2, H=4, H_kv=4, L_q=260, L_k=260, D=128, causal=True, seed=9800)
    check_fp8(w, mask=_mask((1, 1, 1, w.L_k), "bool", 9801), stats=True)


def test_fp8_stats_without_mask():
    check_fp8(_w(L_q=200, L_k=500, D=64, seed=9900), stats=True)
