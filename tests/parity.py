"""Shared helpers for the GPU-vs-oracle parity tests.

Gate on the named workloads (the target tolerances, widened by the output
rounding the target cannot avoid): |O_gpu - O_oracle| <= 3e-3 +
ulp_dtype(O_oracle)/2 element by element, |lse_gpu - lse_oracle| <= 1e-3,
and -inf lse exactly where the oracle has it.  The half-ulp term is the RNE
rounding of the fp32 result to fp16/bf16: bf16's half ulp is 3.9e-3 for |O|
in [1, 2).

Derived gate for the extra edge-case shapes (rows that see a handful of
keys): the PV product takes P rounded to the input type, so each weight p_j
carries a relative error up to u = 2^-8 (bf16) or 2^-11 (fp16), while the
normaliser l sums the unrounded fp32 weights.  That moves O[d] by at most
u * sum_j w_j |v_j[d]| = u * wabs[d] (wabs from the oracle).  With a row of
two keys this term alone exceeds 3e-3 for bf16, whatever the implementation,
so the derived gate adds it, doubled for the second-order terms and the fp32
rounding of the accumulation: 3e-3 + ulp/2 + 2u * wabs."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from exact_attention_113_b200.inputs import BF16, F16, Workload, make_qkv, to_bits

O_TOL = 3e-3
LSE_TOL = 1e-3
P_UNIT_ROUNDOFF = {F16: 2.0 ** -11, BF16: 2.0 ** -8}


def half_ulp(x: np.ndarray, dtype: int) -> np.ndarray:
    mbits, emin = (10, -14) if dtype == F16 else (7, -126)
    a = np.abs(x)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, emin)
    return 0.5 * np.exp2(e - mbits)


def compare(out_gpu: np.ndarray, lse_gpu: np.ndarray | None, out_ref: np.ndarray,
            lse_ref: np.ndarray | None, dtype: int, where: str = "",
            wabs: np.ndarray | None = None) -> dict:
    """Assert the gate (the derived one when ``wabs`` is given); return max
    errors for reporting."""
    out_gpu = np.asarray(out_gpu, dtype=np.float64)
    assert out_gpu.shape == out_ref.shape, (out_gpu.shape, out_ref.shape)
    assert np.all(np.isfinite(out_gpu)), f"{where}: non-finite output"
    err = np.abs(out_gpu - out_ref)
    bound = O_TOL + half_ulp(out_ref, dtype)
    if wabs is not None:
        bound = bound + 2.0 * P_UNIT_ROUNDOFF[dtype] * wabs.reshape(out_ref.shape)
    bad = err > bound
    stats = {"o_max_abs": float(err.max(initial=0.0)),
             "o_worst_excess": float((err - bound).max(initial=-1.0))}
    assert not bad.any(), (f"{where}: {int(bad.sum())} outputs beyond tolerance; "
                           f"max err {err.max():.3g} at {np.unravel_index(err.argmax(), err.shape)}")
    if lse_ref is not None:
        lse_gpu = np.asarray(lse_gpu, dtype=np.float64)
        inf_ref = np.isneginf(lse_ref)
        assert np.array_equal(np.isneginf(lse_gpu), inf_ref), f"{where}: -inf lse mismatch"
        fin = ~inf_ref
        lerr = np.abs(lse_gpu[fin] - lse_ref[fin])
        stats["lse_max_abs"] = float(lerr.max(initial=0.0))
        assert np.all(np.isfinite(lse_gpu[fin])), f"{where}: non-finite lse"
        assert (lerr <= LSE_TOL).all(), f"{where}: lse err {lerr.max():.3g}"
    return stats


def run_gpu(q, k, v, w: Workload, with_lse: bool = True, n_splits=0):
    """Run the CUDA path; outputs pre-filled with NaN so unwritten rows show.
    ``n_splits`` > 0 goes through fa_fwd_splitkv with a NaN-filled
    workspace, so a partial the kernel forgot to write shows too."""
    import exact_attention_113_b200 as fa
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    out = torch.full_like(qd, float("nan"))
    lse = torch.full((w.B, w.H, w.L_q), float("nan"), dtype=torch.float32,
                     device="cuda") if with_lse else None
    ws = None
    if n_splits:
        nbytes = fa.fa_splitkv_workspace_bytes(w.B, w.H, w.L_q, w.D, n_splits)
        ws = torch.full((max(nbytes, 4) // 4,), float("nan"), dtype=torch.float32,
                        device="cuda").view(torch.uint8)
    fa.flash_fwd(qd, kd, vd, scale=w.softmax_scale, causal=w.causal,
                 window_left=w.window_left, window_right=w.window_right,
                 return_lse=with_lse, out=out, lse=lse, n_splits=n_splits, workspace=ws)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == 0, "device watchdog fired"
    return out, lse


def check_full(w: Workload, with_lse: bool = True, derived: bool = False,
               n_splits=0) -> dict:
    """Every row against the oracle (``derived``: the edge-case gate)."""
    q, k, v = make_qkv(w)
    out, lse = run_gpu(q, k, v, w, with_lse, n_splits)
    ref, ref_lse, _, wabs = oracle.attention_rows(
        to_bits(q), to_bits(k), to_bits(v), w.dtype, w.softmax_scale, w.causal,
        w.window_left, w.window_right, with_wabs=True)
    ref = ref.reshape(w.B, w.H, w.L_q, w.D)
    ref_lse = ref_lse.reshape(w.B, w.H, w.L_q)
    return compare(out.float().cpu().numpy(), lse.cpu().numpy() if with_lse else None,
                   ref, ref_lse if with_lse else None, w.dtype, w.name,
                   wabs if derived else None)


_cache = {}


def cached_qkv(w: Workload):
    """make_qkv with a one-entry cache: variants of one shape share inputs."""
    key = (w.B, w.H, w.H_kv, w.L_q, w.L_k, w.D, w.dtype, w.std, w.seed)
    if key not in _cache:
        _cache.clear()
        _cache[key] = make_qkv(w)
    return _cache[key]


def check_rows(w: Workload, rows: np.ndarray, inputs=None, n_splits=0) -> dict:
    """Sampled rows (flattened ids (b*H+h)*L_q+i) against the oracle."""
    q, k, v = inputs if inputs is not None else cached_qkv(w)
    out, lse = run_gpu(q, k, v, w, True, n_splits)
    ref, ref_lse, _ = oracle.attention_rows(to_bits(q), to_bits(k), to_bits(v), w.dtype,
                                            w.softmax_scale, w.causal, w.window_left,
                                            w.window_right, rows=rows)
    o = out.reshape(-1, w.D)[torch.from_numpy(rows).cuda()].float().cpu().numpy()
    lz = lse.reshape(-1)[torch.from_numpy(rows).cuda()].cpu().numpy()
    return compare(o, lz, ref, ref_lse, w.dtype, w.name)
