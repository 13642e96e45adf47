"""fa_fwd_ex on the GPU: attention mask and softmax statistics against the
fp64 oracle (attention_rows_ex).

Masks: bool (true hides the key), fp16 and fp32 (added to the scaled
scores), full [B, H, L_q, L_k] or broadcast ([L_q, L_k], key padding
[B, 1, 1, L_k], per-head [1, H, 1, L_k]), with and without the causal /
window rule, aligned (16-byte vector loads) and unaligned strides.

Gate: O as the plain forward's derived gate (3e-3 + ulp/2 + P's rounding
term, min(u wabs, 8 sigma_P): a random mask leaves some rows a handful of
keys) and the aggregate check of tests/parity.py; lse, softmax_max within
1e-3 (both log-domain quantities); softmax_sum within a relative 1e-3 (its
log is lse - softmax_max)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from exact_attention_113_b200.inputs import BF16, F16, Workload, make_qkv, to_bits
from tests.parity import compare, reference

pytestmark = pytest.mark.gpu


def _w(**kw):
    base = dict(name="mask", B=2, H=4, H_kv=2, L_q=300, L_k=333, D=64, dtype=F16, seed=7000)
    base.update(kw)
    return Workload(**base)


def _mask(shape, kind, seed, p_hide=0.3):
    g = torch.Generator().manual_seed(seed)
    if kind == "bool":
        return torch.rand(shape, generator=g) < p_hide
    x = torch.randn(shape, generator=g) * 2.0
    x = torch.where(torch.rand(shape, generator=g) < p_hide, torch.tensor(float("-inf")), x)
    return x.to(torch.float16 if kind == "f16" else torch.float32)


def check_masked(w, mask, stats=True):
    import exact_attention_113_b200 as fa
    q, k, v = make_qkv(w)
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    md = mask.cuda() if mask is not None else None
    out = torch.full_like(qd, float("nan"))
    lse = torch.full((w.B, w.H, w.L_q), float("nan"), device="cuda")
    out, lse, smax, ssum = fa.flash_fwd(qd, kd, vd, scale=w.softmax_scale, causal=w.causal,
                                        window_left=w.window_left, window_right=w.window_right,
                                        out=out, lse=lse, mask=md, return_softmax_stats=stats)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == 0
    mnp = None if mask is None else mask.numpy()
    ref, ref_lse, pr, heads, ref_max, ref_sum = reference(w, q, k, v, mask=mnp, stats=True)
    compare(out.float().cpu().numpy().reshape(-1, w.D), lse.cpu().numpy().reshape(-1), ref,
            ref_lse, w.dtype, w.name, pr, True, heads)
    if stats:
        gm = smax.cpu().numpy().reshape(-1).astype(np.float64)
        gs = ssum.cpu().numpy().reshape(-1).astype(np.float64)
        inf = np.isneginf(ref_max)
        assert np.array_equal(np.isneginf(gm), inf)
        assert np.all(gs[inf] == 0)
        assert np.abs(gm[~inf] - ref_max[~inf]).max(initial=0) <= 1e-3
        assert np.all(np.abs(gs[~inf] - ref_sum[~inf]) <= 1e-3 * ref_sum[~inf])


@pytest.mark.parametrize("kind", ["bool", "f16", "f32"])
@pytest.mark.parametrize("D", [32, 64, 128])
def test_full_masks(kind, D):
    w = _w(D=D, seed=7000 + D)
    check_masked(w, _mask((w.B, w.H, w.L_q, w.L_k), kind, 7100 + D))


@pytest.mark.parametrize("kind", ["bool", "f32"])
@pytest.mark.parametrize("shape", ["qk", "key_padding", "per_head_keys"])
def test_broadcast_masks(kind, shape):
    w = _w(L_q=257, L_k=640, D=128, dtype=BF16, seed=7200)
    dims = {"qk": (1, 1, w.L_q, w.L_k), "key_padding": (w.B, 1, 1, w.L_k),
            "per_head_keys": (1, w.H, 1, w.L_k)}[shape]
    check_masked(w, _mask(dims, kind, 7300))


@pytest.mark.parametrize("causal,wl,wr", [(True, -1, -1), (False, 64, 32), (True, 100, -1)])
def test_mask_with_causal_and_window(causal, wl, wr):
    w = _w(causal=causal, window_left=wl, window_right=wr, D=64, seed=7400)
    check_masked(w, _mask((w.B, w.H, w.L_q, w.L_k), "f16", 7401))


def test_unaligned_mask_strides():
    # L_k = 333 bool / fp16 rows are not 16-byte multiples: scalar loads
    w = _w(L_k=333, D=64, seed=7500)
    for kind in ("bool", "f16"):
        check_masked(w, _mask((1, 1, w.L_q, w.L_k), kind, 7501))


def test_fully_hidden_rows_and_keys():
    w = _w(L_q=200, L_k=256, D=64, seed=7600)
    m = torch.zeros((w.B, w.H, w.L_q, w.L_k), dtype=torch.bool)
    m[:, :, 5, :] = True          # row 5 sees nothing
    m[:, :, :, 100:] = True       # keys past 100 hidden for everybody
    check_masked(w, m)


def test_statistics_without_mask():
    check_masked(_w(D=128, dtype=BF16, causal=True, seed=7700), None)


def test_gqa_packed_with_mask():
    # short query range with a power-of-two group: the packed-tile path
    w = _w(B=2, H=8, H_kv=2, L_q=20, L_k=900, D=128, seed=7800)
    check_masked(w, _mask((w.B, w.H, w.L_q, w.L_k), "bool", 7801))


def test_mask_matches_equivalent_causal():
    # a bool mask of the causal pattern gives the causal forward bit for bit
    import exact_attention_113_b200 as fa
    w = _w(L_q=400, L_k=400, D=128, seed=7900)
    q, k, v = (t.cuda() for t in make_qkv(w))
    i = torch.arange(w.L_q).view(-1, 1)
    j = torch.arange(w.L_k).view(1, -1)
    m = (j > i).view(1, 1, w.L_q, w.L_k).cuda()
    o1, l1 = fa.flash_fwd(q, k, v, scale=w.softmax_scale, causal=True)
    o2, l2, _, _ = fa.flash_fwd(q, k, v, scale=w.softmax_scale, mask=m)
    torch.cuda.synchronize()
    assert (o1.float() - o2.float()).abs().max().item() <= 2e-3
    assert (l1 - l2).abs().max().item() <= 1e-4


@pytest.mark.parametrize("D", [48, 112])
def test_non_pow2_head_dim_with_mask(D):
    w = _w(D=D, seed=7950 + D)
    check_masked(w, _mask((1, w.H, w.L_q, w.L_k), "f32", 7960 + D))
