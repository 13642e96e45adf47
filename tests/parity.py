"""Shared helpers for the GPU-vs-oracle parity tests.

Gate on the named workloads (the target tolerances, widened by the output
rounding the target cannot avoid): |O_gpu - O_oracle| <= 3e-3 +
ulp_out(O_oracle)/2 element by element, |lse_gpu - lse_oracle| <= 1e-3,
and -inf lse exactly where the oracle has it.  The half-ulp term is the RNE
rounding of the fp32 result to fp16/bf16: bf16's half ulp is 3.9e-3 for |O|
in [1, 2).

Rounding model of P (the kernel's only rounding beyond fp32 and the output):
the P.V product takes every weight p_j rounded to the input format, so
p_j becomes p_j (1 + d_j) with |d_j| <= u (u = 2^-11 fp16, 2^-8 bf16, 2^-4
E4M3 in its normal range; below that an absolute error of half the
subnormal spacing), while the normaliser l sums the unrounded fp32 weights.
With w_j = p_j / l the error this adds to O[d] is exactly
    e[d] = sum_j w_j d_j v_j[d],
so (oracle error scales, see attention_ref.c)
  - worst case: |e| <= u * wabs,        wabs = sum_j w_j |v_j[d]|;
  - statistics: the d_j are independent and uniform within half an ulp,
    so e has mean 0 and a standard deviation of at most
    sigma_P = u / sqrt(3) * wrss,       wrss = sqrt(sum_j w_j^2 v_j[d]^2).
    e is a sum of independent bounded terms: for n terms of equal size it
    cannot exceed sqrt(3 n) sigma_P at all, and for many terms its tail is
    lighter than a normal one, so |e| > 8 sigma_P has a probability below
    1e-15 per element.

Derived gate (edge-case shapes where rows see a handful of keys, bf16 rows
of two keys exceed 3e-3 under any implementation of the method):
    3e-3 + ulp/2 + min(u * wabs, 8 sigma_P).

Aggregate check (every comparison that has the error scales, named
workloads included): per head, the mean over its elements of
e_total^2 / var must stay below 1.5 (1 + 8 sqrt(2/N) for N < 512
elements), where
    var = sigma_P^2 + ulp_out^2 / 12 + (2^-18 wabs)^2
is the variance the model allows: P's rounding, the output's RNE rounding
(uniform within half an ulp) and a floor for the fp32 arithmetic (scores,
exponentials, accumulation; each well below 2^-18 relative).  A correct
kernel has an expected ratio of at most 1 (about 0.5 for uniformly spread
mantissas); a head scaled by 1 + 2^-8 (fp16) or 1 + 2^-4 (E4M3), a dropped
key block or a neighbour head's values push it far above
(tests/test_gate_sensitivity.py shows this on an emulation of the kernel's
arithmetic)."""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

import oracle
from exact_attention_113_b200.inputs import BF16, F16, Workload, make_qkv, to_bits

O_TOL = 3e-3
LSE_TOL = 1e-3
E4M3 = 2
P_UNIT_ROUNDOFF = {F16: 2.0 ** -11, BF16: 2.0 ** -8, E4M3: 2.0 ** -4}
# half the subnormal spacing of P's format (absolute error of a tiny weight)
P_SUB_HALF_SPACING = {F16: 2.0 ** -25, BF16: 2.0 ** -134, E4M3: 2.0 ** -10}
Z_SIGMA = 8.0            # standard deviations of the statistical per-element bound
FLOOR_REL = 2.0 ** -18   # fp32 arithmetic besides P's rounding, relative to wabs
MS_MAX = 1.5             # aggregate: largest mean of e^2 / var per head


def half_ulp(x: np.ndarray, dtype: int) -> np.ndarray:
    mbits, emin = (10, -14) if dtype == F16 else (7, -126)
    a = np.abs(x)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, emin)
    return 0.5 * np.exp2(e - mbits)


@dataclass
class PRounding:
    """Error scales of P's rounding for one output tensor ([n, D] each).

    ``sub_abs`` / ``sub_rss``: the absolute (subnormal) part of the weights'
    rounding, worst case and root sum of squares over the keys."""
    u: float
    wabs: np.ndarray
    wrss: np.ndarray
    sub_abs: object = 0.0
    sub_rss: object = 0.0

    def worst(self) -> np.ndarray:
        return self.u * self.wabs + self.sub_abs

    def sigma(self) -> np.ndarray:
        return np.sqrt((self.u * self.wrss) ** 2 + np.square(self.sub_rss)) / np.sqrt(3.0)

    def scaled(self, c: float) -> "PRounding":
        return PRounding(self.u, self.wabs * c, self.wrss * c,
                         np.multiply(self.sub_abs, c), np.multiply(self.sub_rss, c))


def p_rounding(dtype: int, wabs, wrss, v_bits=None, ssum=None, rows_head=None,
               group: int = 1) -> PRounding:
    """PRounding for P in ``dtype``'s format.  With ``v_bits`` ([B, H_kv, L_k,
    D] codes), ``ssum`` (the rows' softmax sums) and ``rows_head`` (each
    row's query head index b*H + h), the subnormal part is bounded over all
    keys of the row's K/V head: half the subnormal spacing per key, divided
    by the kernel's normaliser, which is at least ssum."""
    pr = PRounding(P_UNIT_ROUNDOFF[dtype], np.asarray(wabs), np.asarray(wrss))
    if v_bits is not None:
        vf = oracle.decode(v_bits, dtype).astype(np.float64)
        B, H_kv, L_k, D = vf.shape
        vabs = np.abs(vf).sum(axis=2).reshape(B * H_kv, D)
        vrss = np.sqrt((vf ** 2).sum(axis=2)).reshape(B * H_kv, D)
        kv = np.asarray(rows_head) // group
        with np.errstate(divide="ignore", invalid="ignore"):
            inv = np.where(ssum > 0, P_SUB_HALF_SPACING[dtype] / np.where(ssum > 0, ssum, 1), 0.0)
        pr.sub_abs = vabs[kv] * inv[:, None]
        pr.sub_rss = vrss[kv] * inv[:, None]
    return pr


def _groups_of(n_rows: int, groups) -> np.ndarray:
    return np.zeros(n_rows, dtype=np.int64) if groups is None else np.asarray(groups).reshape(-1)


def mean_square_ratios(err: np.ndarray, out_ref: np.ndarray, out_dtype: int, pr: PRounding,
                       groups=None) -> list:
    """[(group, N, mean of err^2 / var, threshold)] per group of rows (groups
    with fewer than 512 elements are pooled)."""
    D = err.shape[-1]
    e = err.reshape(-1, D)
    var = (pr.sigma().reshape(-1, D) ** 2 + half_ulp(out_ref, out_dtype).reshape(-1, D) ** 2 / 3.0
           + (FLOOR_REL * pr.wabs.reshape(-1, D)) ** 2 + 1e-30)
    z2 = (e ** 2 / var).sum(axis=1)
    g = _groups_of(e.shape[0], groups)
    ids, inv, counts = np.unique(g, return_inverse=True, return_counts=True)
    small = counts * D < 512
    key = np.where(small[inv], -1, g)
    res = []
    for gid in np.unique(key):
        sel = key == gid
        n = int(sel.sum()) * D
        ratio = float(z2[sel].sum() / n)
        thr = max(MS_MAX, 1.0 + 8.0 * np.sqrt(2.0 / n))
        res.append((int(gid), n, ratio, thr))
    return res


def compare(out_gpu: np.ndarray, lse_gpu: np.ndarray | None, out_ref: np.ndarray,
            lse_ref: np.ndarray | None, dtype: int, where: str = "",
            pr: PRounding | None = None, derived: bool = False, groups=None,
            out_dtype: int | None = None, aggregate: bool = True) -> dict:
    """Assert the gate: the target gate, plus P's rounding term when
    ``derived``; the aggregate check whenever ``pr`` is given and
    ``aggregate`` (``groups``: the head of every row).  ``out_dtype``: the
    output format (default ``dtype``).  Returns the errors and ratios for
    reporting."""
    out_dtype = dtype if out_dtype is None else out_dtype
    out_gpu = np.asarray(out_gpu, dtype=np.float64)
    assert out_gpu.shape == out_ref.shape, (out_gpu.shape, out_ref.shape)
    assert np.all(np.isfinite(out_gpu)), f"{where}: non-finite output"
    err = np.abs(out_gpu - out_ref)
    bound = O_TOL + half_ulp(out_ref, out_dtype)
    if derived:
        assert pr is not None
        bound = bound + np.minimum(pr.worst(), Z_SIGMA * pr.sigma()).reshape(out_ref.shape)
    bad = err > bound
    stats = {"o_max_abs": float(err.max(initial=0.0)),
             "o_worst_excess": float((err - bound).max(initial=-1.0))}
    assert not bad.any(), (f"{where}: {int(bad.sum())} outputs beyond tolerance; "
                           f"max err {err.max():.3g} at {np.unravel_index(err.argmax(), err.shape)}")
    if pr is not None and aggregate:
        ratios = mean_square_ratios(out_gpu - out_ref, out_ref, out_dtype, pr, groups)
        stats["ms_ratio_max"] = max(r[2] for r in ratios)
        worst = [r for r in ratios if r[2] > r[3]]
        assert not worst, (f"{where}: mean square error beyond the rounding model "
                           f"(group, elements, ratio, limit): {worst[:4]}")
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


def reference(w: Workload, q, k, v, rows=None, mask=None, in_dtype=None, scale=None,
              out_scale: float = 1.0, stats: bool = False):
    """Oracle rows of workload ``w`` with their error scales: (out [n, D],
    lse [n], PRounding, head of every row), plus (softmax_max, softmax_sum)
    with ``stats``.  ``in_dtype``: the inputs' code format (E4M3 for the
    fp8 entry; default w.dtype), which is also P's format; ``scale``: the
    effective score scale (default w.softmax_scale); ``out_scale``
    multiplies O and its error scales (descale_v)."""
    in_dtype = w.dtype if in_dtype is None else in_dtype
    scale = w.softmax_scale if scale is None else scale
    ref, ref_lse, smax, ssum, wabs, wrss = oracle.attention_rows_ex(
        to_bits(q), to_bits(k), to_bits(v), in_dtype, scale, w.causal,
        w.window_left, w.window_right, mask=mask, rows=rows, with_wabs=True, with_wrss=True)
    n_all = w.B * w.H * w.L_q
    rid = np.arange(n_all) if rows is None else np.asarray(rows)
    heads = rid // max(w.L_q, 1)
    pr = p_rounding(in_dtype, wabs, wrss, to_bits(v), ssum, heads, w.H // w.H_kv)
    if out_scale != 1.0:
        ref = ref * out_scale
        pr = pr.scaled(out_scale)
    if stats:
        return ref, ref_lse, pr, heads, smax, ssum
    return ref, ref_lse, pr, heads


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
    ref, ref_lse, pr, heads = reference(w, q, k, v)
    return compare(out.float().cpu().numpy().reshape(-1, w.D),
                   lse.cpu().numpy().reshape(-1) if with_lse else None,
                   ref, ref_lse if with_lse else None, w.dtype, w.name, pr, derived, heads)


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
    ref, ref_lse, pr, heads = reference(w, q, k, v, rows)
    o = out.reshape(-1, w.D)[torch.from_numpy(rows).cuda()].float().cpu().numpy()
    lz = lse.reshape(-1)[torch.from_numpy(rows).cuda()].cpu().numpy()
    return compare(o, lz, ref, ref_lse, w.dtype, w.name, pr, False, heads)
