"""The parity gate of tests/parity.py can tell a right result from a wrong
one (CPU only).

An emulation of the kernel's arithmetic, written here from the method and
independent of the oracle's code, produces what a correct kernel returns:
the weights p_j = e^(s_j - m_ref) against a reference maximum that lags the
true one by up to 2^8 (the conditional rescale), each p_j rounded to P's
format (fp16 / bf16 / E4M3) for the P.V product, the normaliser summed from
the unrounded weights, the output rounded to its format.  The gate must
accept that, and must reject the same emulation with one planted mistake:
one head's output scaled by 1 + 2^-8 (2^-4 for E4M3, the size of P's own
rounding there), one key block of one head dropped, one head reading its
neighbour's values, a causal mask that hides the diagonal."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from exact_attention_113_b200.inputs import BF16, F16, Workload, make_qkv, make_qkv_fp8
from tests.parity import E4M3, compare, reference

FMT = {F16: torch.float16, BF16: torch.bfloat16, E4M3: torch.float8_e4m3fn}


def _round(x: np.ndarray, fmt: int) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(FMT[fmt]).to(torch.float64).numpy()


def emulate(w: Workload, q, k, v, in_fmt: int, out_fmt: int, scale: float, plant=None,
            seed: int = 5):
    """[B*H*L_q, D] output of a kernel that follows the method with the
    stated roundings; ``plant`` names one mistake to make."""
    qf, kf, vf = (t.to(torch.float64).numpy() for t in (q, k, v))
    g = w.H // w.H_kv
    rng = np.random.default_rng(seed)
    i = np.arange(w.L_q)[:, None]
    j = np.arange(w.L_k)[None, :]
    vis = np.ones((w.L_q, w.L_k), dtype=bool)
    wr = 0 if w.causal else w.window_right
    if w.window_left >= 0:
        vis &= j >= i - w.window_left
    if wr >= 0:
        vis &= j <= i + wr
    if plant == "causal_hides_diagonal":
        vis &= j < i
    out = np.zeros((w.B, w.H, w.L_q, w.D))
    for b in range(w.B):
        for h in range(w.H):
            hk = h // g
            if plant == "neighbour_values" and (b, h) == (0, 0):
                hk = (hk + 1) % w.H_kv
            s = scale * qf[b, h] @ kf[b, h // g].T
            vmask = vis.copy()
            if plant == "drop_block" and (b, h) == (0, 1):
                vmask[:, 128:256] = False
            s = np.where(vmask, s, -np.inf)
            m = s.max(axis=1, keepdims=True)
            m = np.where(np.isfinite(m), m, 0.0)
            lag = rng.uniform(0.0, 8.0 * np.log(2.0), size=m.shape)   # m_ref = m - lag
            p = np.exp(s - (m - lag))
            l = p.sum(axis=1, keepdims=True)
            o = _round(p, in_fmt) @ vf[b, hk]
            o = np.where(l > 0, o / np.where(l > 0, l, 1.0), 0.0)
            if plant == "scaled_head" and (b, h) == (1, 2):
                o = o * (1.0 + (2.0 ** -4 if in_fmt == E4M3 else 2.0 ** -8))
            out[b, h] = _round(o, out_fmt)
    return out.reshape(-1, w.D)


CASES = [
    # in_fmt, D, causal
    (F16, 64, False),
    (BF16, 128, True),
    (E4M3, 128, False),
]
PLANTS = ["scaled_head", "drop_block", "neighbour_values", "causal_hides_diagonal"]


def _setup(in_fmt, D, causal):
    w = Workload(name="gate", B=2, H=4, H_kv=2, L_q=300, L_k=300, D=D,
                 dtype=F16 if in_fmt == E4M3 else in_fmt, causal=causal, seed=6100 + D)
    if in_fmt == E4M3:
        q, k, v = make_qkv_fp8(w)
        out_fmt = BF16
    else:
        q, k, v = make_qkv(w)
        out_fmt = in_fmt
    ref, ref_lse, pr, heads = reference(w, q, k, v, in_dtype=in_fmt)
    return w, (q, k, v), out_fmt, ref, pr, heads


@pytest.mark.parametrize("case", CASES)
def test_gate_accepts_the_method_with_its_roundings(case):
    in_fmt, D, causal = case
    w, (q, k, v), out_fmt, ref, pr, heads = _setup(*case)
    for seed in (5, 6):
        got = emulate(w, q, k, v, in_fmt, out_fmt, w.softmax_scale, seed=seed)
        st = compare(got, None, ref, None, in_fmt, "emulation", pr, True, heads,
                     out_dtype=out_fmt)
        assert st["ms_ratio_max"] < 1.0


@pytest.mark.parametrize("plant", PLANTS)
@pytest.mark.parametrize("case", CASES)
def test_gate_rejects_a_planted_mistake(case, plant):
    in_fmt, D, causal = case
    if plant == "causal_hides_diagonal" and not causal:
        pytest.skip("needs a causal case")
    w, (q, k, v), out_fmt, ref, pr, heads = _setup(*case)
    got = emulate(w, q, k, v, in_fmt, out_fmt, w.softmax_scale, plant=plant)
    with pytest.raises(AssertionError):
        compare(got, None, ref, None, in_fmt, "emulation", pr, True, heads, out_dtype=out_fmt)


def test_scaled_head_passes_the_per_element_bound_alone():
    # the planted E4M3 scale error hides inside the per-element bound (P's
    # own rounding noise is of the same size); only the aggregate check
    # catches it, which is why the gate has one
    in_fmt, D, causal = CASES[2]
    w, (q, k, v), out_fmt, ref, pr, heads = _setup(in_fmt, D, causal)
    got = emulate(w, q, k, v, in_fmt, out_fmt, w.softmax_scale, plant="scaled_head")
    compare(got, None, ref, None, in_fmt, "emulation", pr, True, heads, out_dtype=out_fmt,
            aggregate=False)
    with pytest.raises(AssertionError, match="mean square"):
        compare(got, None, ref, None, in_fmt, "emulation", pr, True, heads, out_dtype=out_fmt)
