"""Pins for the fp64 CPU oracle: facts fixed by the pages and the mathematics,
checked against something other than the oracle itself (closed forms,
invariants, library routines, an independent brute force, the pages' worked
example).  CPU only."""
import math
import os

import numpy as np
import pytest
import torch

from exact_attention_113_b200.inputs import F16, BF16, TORCH_DTYPE

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, rhs = line.split("=", 1)
            vals[key.strip()] = [float(t) for t in rhs.split(",")]
    return vals


def _rand_bits(shape, dtype, seed, std=1.0):
    g = torch.Generator().manual_seed(seed)
    x = (torch.randn(shape, generator=g) * std).to(TORCH_DTYPE[dtype])
    return x.view(torch.int16).numpy().view(np.uint16)


def _lib_decode(bits, dtype):
    """Decode with library routines (numpy for fp16, torch for bf16)."""
    bits = np.asarray(bits, dtype=np.uint16)
    if dtype == F16:
        return bits.view(np.float16).astype(np.float64)
    t = torch.from_numpy(bits.astype(np.int16)).view(torch.bfloat16)
    return t.to(torch.float64).numpy()


def _lib_encode(x, dtype):
    x = np.asarray(x, dtype=np.float64)
    if dtype == F16:
        with np.errstate(over="ignore"):
            return x.astype(np.float16).view(np.uint16)
    t = torch.from_numpy(x).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


# ------------------------------------------------------------------ formats
@pytest.mark.parametrize("dtype", [F16, BF16])
def test_decode_matches_library_on_every_pattern(orc, dtype):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = orc.decode(bits, dtype)
    ref = _lib_decode(bits, dtype)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])


def test_round_f16_matches_numpy(orc):
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.normal(size=4000) * 10.0 ** rng.integers(-9, 6, size=4000),
        # exact ties between adjacent fp16 values (round half to even)
        (np.arange(1024, 1100) + 0.5) * 2.0 ** -10,
        (np.arange(1, 60) + 0.5) * 2.0 ** -24,          # subnormal ties
        [65504.0, 65519.99, 65520.0, 1e6, -1e6, 0.0, -0.0, 2.0 ** -25,
         2.0 ** -25 * 1.0000001, 6.1e-5],
    ])
    ours = orc.round_to(x, F16)
    assert np.array_equal(ours, _lib_encode(x, F16))


def test_round_bf16_matches_torch(orc):
    # fp32-representable inputs, so torch's float->bf16 rounding is the
    # single correctly rounded step from the exact value
    rng = np.random.default_rng(2)
    x = (rng.normal(size=4000) * 10.0 ** rng.integers(-30, 30, size=4000))
    x = np.concatenate([x, (np.arange(128, 200) + 0.5) * 2.0 ** -7,
                        [3.3895313892515355e38, 0.0, -0.0, 1e-39]])
    x = x.astype(np.float32).astype(np.float64)
    ours = orc.round_to(x, BF16)
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16)
    assert np.array_equal(ours, ref.view(torch.int16).numpy().view(np.uint16))


def test_fp16_overflow_fact(orc):
    # e^11 < 65504 (the fp16 maximum) < e^11.1: the naive softmax's numerator
    # e^x leaves fp16 range at x of about 11; the safe form keeps e^{x-m} <= 1.
    assert orc.f16_to_f64(0x7BFF) == 65504.0
    assert math.exp(11.0) < 65504.0 < math.exp(11.1)
    a, d, m = orc.safe_softmax([11.1, 0.0, -3.0])
    assert m == 11.1 and all(0.0 <= t <= 1.0 for t in a)
    assert abs(sum(a) - 1.0) < 1e-15


# ------------------------------------------------------------------ softmax
def test_online_softmax_worked_example(orc):
    g = _golden("online_softmax_example.txt")
    x = g["x"]
    total = sum(math.exp(t - max(x)) for t in x)
    expect = [math.exp(t - max(x)) / total for t in x]
    for fn in (orc.online_softmax, orc.safe_softmax):
        a, d, m = fn(x)
        assert m == max(x)
        assert abs(d - total) < 1e-14
        assert np.allclose(a, expect, rtol=0, atol=1e-15)
        assert abs(a.sum() - g["sum"][0]) < 1e-15
    # the values spelled out: e^{i-5}/(1+e^-1+e^-2+e^-3+e^-4)
    assert np.allclose(orc.online_softmax(x)[0],
                       [0.011656230956039607, 0.031684920796124276,
                        0.08612854443626873, 0.23412165725273662,
                        0.6364086465588308], atol=1e-15)


def test_page_listing_reading_is_rejected():
    """The page's listing keeps e^{x_i - m_i} (the running max at step i) and
    divides by d_N; on its own example that sums to about 3.18, not 1.  The
    oracle follows the derivation instead (a_i = e^{x_i - m_N}/d_N)."""
    x = [1.0, 2.0, 3.0, 4.0, 5.0]
    m, d, kept = -math.inf, 0.0, []
    for xi in x:
        m_new = max(m, xi)
        d = d * math.exp(m - m_new) + math.exp(xi - m_new)
        kept.append(math.exp(xi - m_new))
        m = m_new
    assert abs(sum(v / d for v in kept) - 3.182043) < 1e-5


def test_online_equals_three_pass_random(orc):
    rng = np.random.default_rng(3)
    for n in (1, 2, 7, 128, 1000):
        x = rng.normal(size=n) * 20
        x[rng.random(n) < 0.2] = -np.inf
        if np.all(np.isinf(x)):
            x[0] = 0.0
        a1, d1, m1 = orc.online_softmax(x)
        a2, d2, m2 = orc.safe_softmax(x)
        assert m1 == m2
        assert abs(d1 - d2) <= 1e-12 * d2
        assert np.allclose(a1, a2, rtol=1e-12, atol=1e-300)
        assert abs(a1.sum() - 1) < 1e-12


def test_all_masked_softmax_is_zero(orc):
    a, d, m = orc.safe_softmax([-np.inf, -np.inf])
    assert m == -np.inf and d == 0.0 and np.all(a == 0)


# --------------------------------------------------------- brute force
def _visible(i, j, L_k, causal, wl, wr):
    if not 0 <= j < L_k:
        return False
    if causal and j > i:
        return False
    if wl >= 0 and j < i - wl:
        return False
    if wr >= 0 and j > i + wr:
        return False
    return True


def _brute(qf, kf, vf, scale, causal, wl, wr):
    """Independent fp64 double loop in plain Python (math only)."""
    B, H, L_q, D = qf.shape
    H_kv, L_k = kf.shape[1], kf.shape[2]
    grp = H // H_kv
    out = np.zeros((B, H, L_q, D))
    lse = np.zeros((B, H, L_q))
    wabs = np.zeros((B, H, L_q, D))
    wrss = np.zeros((B, H, L_q, D))
    for b in range(B):
        for h in range(H):
            g = h // grp
            for i in range(L_q):
                s = []
                for j in range(L_k):
                    if _visible(i, j, L_k, causal, wl, wr):
                        s.append((j, scale * math.fsum(
                            float(qf[b, h, i, d]) * float(kf[b, g, j, d])
                            for d in range(D))))
                if not s:
                    lse[b, h, i] = -math.inf
                    continue
                m = max(t for _, t in s)
                den = math.fsum(math.exp(t - m) for _, t in s)
                for d in range(D):
                    out[b, h, i, d] = math.fsum(
                        math.exp(t - m) / den * float(vf[b, g, j, d])
                        for j, t in s)
                    wabs[b, h, i, d] = math.fsum(
                        math.exp(t - m) / den * abs(float(vf[b, g, j, d]))
                        for j, t in s)
                    wrss[b, h, i, d] = math.sqrt(math.fsum(
                        (math.exp(t - m) / den * float(vf[b, g, j, d])) ** 2
                        for j, t in s))
                lse[b, h, i] = m + math.log(den)
    return out, lse, wabs, wrss


BRUTE_CASES = [
    # B, H, H_kv, L_q, L_k, D, dtype, causal, wl, wr
    (1, 2, 2, 5, 5, 4, F16, False, -1, -1),
    (1, 2, 2, 7, 7, 8, F16, True, -1, -1),
    (2, 4, 2, 6, 9, 4, BF16, False, -1, -1),
    (1, 4, 1, 9, 9, 4, F16, True, 2, -1),
    (1, 2, 2, 8, 8, 4, BF16, False, 1, 2),
    (1, 2, 1, 3, 5, 4, F16, True, -1, -1),     # L_q < L_k
    (1, 2, 2, 6, 3, 4, F16, True, 0, -1),      # rows 3.. fully masked
    (1, 1, 1, 4, 6, 4, F16, False, -1, 0),     # window_right only
]


@pytest.mark.parametrize("case", BRUTE_CASES)
def test_matches_brute_force(orc, case):
    B, H, H_kv, L_q, L_k, D, dtype, causal, wl, wr = case
    q = _rand_bits((B, H, L_q, D), dtype, 11)
    k = _rand_bits((B, H_kv, L_k, D), dtype, 12)
    v = _rand_bits((B, H_kv, L_k, D), dtype, 13)
    scale = 1.0 / math.sqrt(D)
    out, lse = orc.attention(q, k, v, dtype, scale, causal, wl, wr)
    ro, rl, rw, rr = _brute(_lib_decode(q, dtype), _lib_decode(k, dtype),
                            _lib_decode(v, dtype), scale, causal, wl, wr)
    assert np.allclose(out, ro, rtol=0, atol=1e-12)
    _, _, _, wabs = orc.attention_rows(q, k, v, dtype, scale, causal, wl, wr,
                                       with_wabs=True)
    assert np.allclose(wabs, rw.reshape(wabs.shape), rtol=0, atol=1e-12)
    _, _, _, wabs2, wrss = orc.attention_rows(q, k, v, dtype, scale, causal, wl, wr,
                                              with_wrss=True)
    assert np.array_equal(wabs2, wabs)
    assert np.allclose(wrss, rr.reshape(wrss.shape), rtol=0, atol=1e-12)
    inf = np.isinf(rl)
    assert np.array_equal(np.isinf(lse), inf)
    assert np.allclose(lse[~inf], rl[~inf], rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_matches_torch_fp64_softmax(orc, causal):
    """The pages' GPT-2 check compares against PyTorch's softmax (a safe
    softmax); here the same comparison in fp64 on the CPU."""
    B, H, L, D = 1, 3, 40, 16
    q, k, v = (_rand_bits((B, H, L, D), F16, s) for s in (21, 22, 23))
    qf, kf, vf = (torch.from_numpy(_lib_decode(t, F16)) for t in (q, k, v))
    s = (qf @ kf.transpose(-1, -2)) * 0.125
    if causal:
        s = s.masked_fill(torch.ones(L, L, dtype=torch.bool).triu(1), -math.inf)
    ref = torch.softmax(s, dim=-1) @ vf
    ref_lse = torch.logsumexp(s, dim=-1)
    out, lse = orc.attention(q, k, v, F16, 0.125, causal)
    assert np.allclose(out, ref.numpy(), rtol=0, atol=1e-12)
    assert np.allclose(lse, ref_lse.numpy(), rtol=0, atol=1e-12)


# --------------------------------------------------------- closed forms
def _const_bits(shape, value, dtype):
    return np.full(shape, _lib_encode([value], dtype)[0], dtype=np.uint16)


@pytest.mark.parametrize("mask", [(False, -1, -1), (True, -1, -1), (True, 3, -1),
                                  (False, 2, 1)])
def test_constant_v_gives_that_constant(orc, mask):
    causal, wl, wr = mask
    B, H, H_kv, L, D = 1, 4, 2, 17, 8
    q = _rand_bits((B, H, L, D), F16, 31)
    k = _rand_bits((B, H_kv, L, D), F16, 32)
    row = _rand_bits((D,), F16, 33)
    v = np.broadcast_to(row, (B, H_kv, L, D)).copy()
    out, lse = orc.attention(q, k, v, F16, 0.3, causal, wl, wr)
    assert np.allclose(out, np.broadcast_to(_lib_decode(row, F16), out.shape),
                       rtol=1e-14, atol=1e-14)


@pytest.mark.parametrize("causal,wl", [(False, -1), (True, -1), (True, 4)])
def test_zero_keys_give_mean_of_visible_values(orc, causal, wl):
    B, H, L, D = 1, 2, 12, 8
    q = _rand_bits((B, H, L, D), BF16, 41)
    k = _const_bits((B, H, L, D), 0.0, BF16)
    v = _rand_bits((B, H, L, D), BF16, 42)
    vf = _lib_decode(v, BF16)
    for kk, scale in ((k, 0.7), (_rand_bits((B, H, L, D), BF16, 43), 0.0)):
        out, lse = orc.attention(q, kk, v, BF16, scale, causal, wl, -1)
        for i in range(L):
            lo = 0 if wl < 0 else max(0, i - wl)
            hi = i if causal else L - 1
            n = hi - lo + 1
            assert np.allclose(out[:, :, i], vf[:, :, lo:hi + 1].mean(axis=2),
                               rtol=0, atol=1e-13)
            assert np.allclose(lse[:, :, i], math.log(n), rtol=0, atol=1e-13)


def test_causal_row_zero_is_v0(orc):
    B, H, L, D = 2, 3, 10, 16
    q, k, v = (_rand_bits((B, H, L, D), F16, s) for s in (51, 52, 53))
    scale = 0.25
    out, lse = orc.attention(q, k, v, F16, scale, True)
    qf, kf, vf = (_lib_decode(t, F16) for t in (q, k, v))
    assert np.array_equal(out[:, :, 0], vf[:, :, 0])
    for b in range(B):
        for h in range(H):
            dot = math.fsum(qf[b, h, 0, d] * kf[b, h, 0, d] for d in range(D))
            assert abs(lse[b, h, 0] - scale * dot) < 1e-13


def test_weighted_abs_value_closed_forms(orc):
    # constant V rows = c  =>  sum_j p_j |c| = |c|;  one key  =>  |v_0|
    B, H, L, D = 1, 2, 9, 4
    q = _rand_bits((B, H, L, D), F16, 141)
    k = _rand_bits((B, H, L, D), F16, 142)
    row = _rand_bits((D,), F16, 143)
    v = np.broadcast_to(row, (B, H, L, D)).copy()
    _, _, _, w = orc.attention_rows(q, k, v, F16, 0.3, True, with_wabs=True)
    assert np.allclose(w, np.abs(_lib_decode(row, F16)), rtol=1e-14, atol=0)
    k1, v1 = k[:, :, :1], _rand_bits((B, H, 1, D), F16, 144)
    _, _, _, w1 = orc.attention_rows(q, k1, v1, F16, 0.3, False, with_wabs=True)
    assert np.array_equal(w1.reshape(B, H, L, D),
                          np.broadcast_to(np.abs(_lib_decode(v1, F16)), (B, H, L, D)))


def test_weighted_rss_closed_forms(orc):
    # K = 0: every visible key weighs 1/n, so wrss = sqrt(sum_vis v^2) / n;
    # one key: wrss = |v_0|; wrss <= wabs <= sqrt(n) * wrss (Cauchy-Schwarz)
    B, H, L, D = 1, 2, 11, 4
    q = _rand_bits((B, H, L, D), BF16, 151)
    k = _const_bits((B, H, L, D), 0.0, BF16)
    v = _rand_bits((B, H, L, D), BF16, 152)
    vf = _lib_decode(v, BF16)
    _, _, _, wabs, wrss = orc.attention_rows(q, k, v, BF16, 0.7, True, 3, -1, with_wrss=True)
    wrss = wrss.reshape(B, H, L, D)
    wabs = wabs.reshape(B, H, L, D)
    for i in range(L):
        lo = max(0, i - 3)
        n = i - lo + 1
        want = np.sqrt((vf[:, :, lo:i + 1] ** 2).sum(axis=2)) / n
        assert np.allclose(wrss[:, :, i], want, rtol=1e-14, atol=0)
        assert np.all(wrss[:, :, i] <= wabs[:, :, i] * (1 + 1e-14))
        assert np.all(wabs[:, :, i] <= np.sqrt(n) * wrss[:, :, i] * (1 + 1e-14))
    k1, v1 = _rand_bits((B, H, 1, D), BF16, 153), _rand_bits((B, H, 1, D), BF16, 154)
    _, _, _, _, w1 = orc.attention_rows(q, k1, v1, BF16, 0.3, False, with_wrss=True)
    assert np.array_equal(w1.reshape(B, H, L, D),
                          np.broadcast_to(np.abs(_lib_decode(v1, BF16)), (B, H, L, D)))


def test_single_key_is_v0(orc):
    B, H, L_q, D = 1, 2, 9, 8
    q = _rand_bits((B, H, L_q, D), F16, 61)
    k = _rand_bits((B, H, 1, D), F16, 62)
    v = _rand_bits((B, H, 1, D), F16, 63)
    out, _ = orc.attention(q, k, v, F16, 0.5, False)
    vf = _lib_decode(v, F16)
    assert np.array_equal(out, np.broadcast_to(vf, out.shape))


def test_fully_masked_rows(orc):
    # L_q > L_k with causal and a zero left window: row i sees only key i
    q = _rand_bits((1, 1, 5, 4), F16, 71)
    k = _rand_bits((1, 1, 3, 4), F16, 72)
    v = _rand_bits((1, 1, 3, 4), F16, 73)
    out, lse = orc.attention(q, k, v, F16, 0.5, True, 0, -1)
    vf = _lib_decode(v, F16)
    assert np.array_equal(out[0, 0, :3], vf[0, 0, :3])
    assert np.all(out[0, 0, 3:] == 0) and np.all(np.isneginf(lse[0, 0, 3:]))


def test_top_left_alignment_when_lq_lt_lk(orc):
    # with L_q = 3 < L_k = 5, causal row 0 sees key 0 only (raw indices)
    q = _rand_bits((1, 1, 3, 4), F16, 81)
    k = _rand_bits((1, 1, 5, 4), F16, 82)
    v = _rand_bits((1, 1, 5, 4), F16, 83)
    out, _ = orc.attention(q, k, v, F16, 0.5, True)
    assert np.array_equal(out[0, 0, 0], _lib_decode(v, F16)[0, 0, 0])


# --------------------------------------------------------- invariants
def test_permuting_keys_with_values(orc):
    B, H, L, D = 1, 2, 33, 8
    q, k, v = (_rand_bits((B, H, L, D), F16, s) for s in (91, 92, 93))
    out, lse = orc.attention(q, k, v, F16, 0.35, False)
    perm = np.random.default_rng(0).permutation(L)
    out2, lse2 = orc.attention(q, k[:, :, perm], v[:, :, perm], F16, 0.35, False)
    assert np.allclose(out, out2, rtol=0, atol=1e-13)
    assert np.allclose(lse, lse2, rtol=0, atol=1e-13)


def test_shifting_every_key(orc):
    """k_j -> k_j + u shifts row i's scores by scale*q_i.u: O is unchanged and
    lse moves by that amount.  Values are small multiples of 1/8 so that the
    shifted keys are exact in fp16."""
    rng = np.random.default_rng(5)
    B, H, L, D = 1, 2, 20, 8
    qf = rng.integers(-8, 9, size=(B, H, L, D)) / 8.0
    kf = rng.integers(-8, 9, size=(B, H, L, D)) / 8.0
    vf = rng.normal(size=(B, H, L, D))
    u = rng.integers(-4, 5, size=D) / 8.0
    q, k, k2, v = (_lib_encode(t, F16) for t in (qf, kf, kf + u, vf))
    for causal in (False, True):
        out, lse = orc.attention(q, k, v, F16, 0.4, causal)
        out2, lse2 = orc.attention(q, k2, v, F16, 0.4, causal)
        assert np.allclose(out, out2, rtol=0, atol=1e-12)
        assert np.allclose(lse2 - lse, 0.4 * (qf @ u), rtol=0, atol=1e-12)


def test_gqa_equals_mha_with_repeated_heads(orc):
    B, H, H_kv, L, D = 2, 6, 2, 11, 8
    q = _rand_bits((B, H, L, D), BF16, 101)
    k = _rand_bits((B, H_kv, L, D), BF16, 102)
    v = _rand_bits((B, H_kv, L, D), BF16, 103)
    grp = H // H_kv
    out, lse = orc.attention(q, k, v, BF16, 0.3, True)
    out2, lse2 = orc.attention(q, np.repeat(k, grp, axis=1),
                               np.repeat(v, grp, axis=1), BF16, 0.3, True)
    assert np.array_equal(out, out2) and np.array_equal(lse, lse2)


def test_window_equivalences(orc):
    B, H, L, D = 1, 2, 24, 8
    q, k, v = (_rand_bits((B, H, L, D), F16, s) for s in (111, 112, 113))
    causal = orc.attention(q, k, v, F16, 0.3, True)
    wide = orc.attention(q, k, v, F16, 0.3, True, L, -1)
    right0 = orc.attention(q, k, v, F16, 0.3, False, -1, 0)
    for a, b in zip(causal, wide):
        assert np.array_equal(a, b)
    for a, b in zip(causal, right0):
        assert np.array_equal(a, b)


# --------------------------------------------------------- tiled method
@pytest.mark.parametrize("block", [1, 3, 16, 128])
@pytest.mark.parametrize("mask", [(False, -1, -1), (True, -1, -1), (True, 5, -1)])
def test_fa2_recurrence_reaches_the_definition(orc, block, mask):
    causal, wl, wr = mask
    B, H, H_kv, L, D = 1, 4, 2, 45, 16
    q = _rand_bits((B, H, L, D), F16, 121)
    k = _rand_bits((B, H_kv, L, D), F16, 122)
    v = _rand_bits((B, H_kv, L, D), F16, 123)
    ref, ref_lse, _ = orc.attention_rows(q, k, v, F16, 0.25, causal, wl, wr)
    out, lse = orc.attention_rows_online(q, k, v, F16, 0.25, causal, wl, wr,
                                         block=block)
    assert np.allclose(out, ref, rtol=0, atol=1e-12)
    assert np.allclose(lse, ref_lse, rtol=0, atol=1e-12)


def test_row_subset_equals_full(orc):
    B, H, L, D = 2, 3, 30, 8
    q, k, v = (_rand_bits((B, H, L, D), BF16, s) for s in (131, 132, 133))
    full, full_lse, _ = orc.attention_rows(q, k, v, BF16, 0.3, True)
    rows = np.array([0, 5, 29, 31, 95, 179], dtype=np.int64)
    out, lse, _ = orc.attention_rows(q, k, v, BF16, 0.3, True, rows=rows)
    assert np.array_equal(out, full[rows]) and np.array_equal(lse, full_lse[rows])
