"""fp64 CPU oracle for exact attention forward -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU baseline
leg may import this package.  The product path (``exact_attention_113_b200``)
never imports it, and it imports nothing from the product path: the two share
no code.  The only module both sides use is the seeded input generator
``exact_attention_113_b200.inputs``, which holds none of the method's
arithmetic.

The C source ``attention_ref.c`` states, function by function, which passage
of the pages it follows.  This module is a ctypes shim around it plus the
build step that compiles it with gcc.

Functions whose parity is pinned (see tests/test_oracle_pins.py and
tests/test_oracle_bwd_pins.py):
  attention, attention_rows, attention_rows_online, safe_softmax,
  online_softmax, f16/bf16 decode and round-to-nearest-even,
  attention_f64, attention_bwd_f64 / attention_bwd (gradients),
  attention_rows_ex (mask, softmax max / sum; tests/test_oracle_mask_pins.py).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attention_ref.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "liboracle.so")
_lock = threading.Lock()

F16, BF16, E4M3 = 0, 1, 2


def build(force: bool = False, src: str = _SRC, out: str = _LIB_PATH) -> str:
    """Compile the oracle C source into a shared library (gcc, OpenMP)."""
    os.makedirs(os.path.dirname(out), exist_ok=True)
    stale = (not os.path.exists(out)
             or os.path.getmtime(out) < os.path.getmtime(src))
    if force or stale:
        tmp = out + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
               "-fno-fast-math", "-o", tmp, src, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, out)
    return out


def _ptr(a: np.ndarray, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _bits(x) -> np.ndarray:
    """Accept a numpy uint16/int16 array of fp16/bf16 bit patterns, or a
    uint8/int8 array of fp8 e4m3 codes (widened to uint16)."""
    a = np.ascontiguousarray(x)
    if a.dtype == np.int16:
        a = a.view(np.uint16)
    if a.dtype == np.int8:
        a = a.view(np.uint8)
    if a.dtype == np.uint8:
        a = a.astype(np.uint16)
    if a.dtype != np.uint16:
        raise TypeError("oracle inputs are fp16/bf16 (uint16) or e4m3 (uint8) bit patterns")
    return a


def _shape_args(q, k, v):
    q, k, v = _bits(q), _bits(k), _bits(v)
    if q.ndim != 4 or k.ndim != 4 or v.ndim != 4:
        raise ValueError("q, k, v must be 4-D [B, H, L, D]")
    B, H, L_q, D = q.shape
    Bk, H_kv, L_k, Dk = k.shape
    if k.shape != v.shape or Bk != B or Dk != D:
        raise ValueError("k and v must be [B, H_kv, L_k, D] with q's B and D")
    return q, k, v, B, H, H_kv, L_q, L_k, D


class Oracle:
    """ctypes view of one build of attention_ref.c."""

    def __init__(self, lib_path: str):
        lib = ctypes.CDLL(lib_path)
        u16p = ctypes.POINTER(ctypes.c_uint16)
        dp = ctypes.POINTER(ctypes.c_double)
        i64p = ctypes.POINTER(ctypes.c_int64)
        i64 = ctypes.c_int64
        lib.oracle_f16_to_f64.argtypes = [ctypes.c_uint16]
        lib.oracle_f16_to_f64.restype = ctypes.c_double
        lib.oracle_bf16_to_f64.argtypes = [ctypes.c_uint16]
        lib.oracle_bf16_to_f64.restype = ctypes.c_double
        lib.oracle_e4m3_to_f64.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_to_f64.restype = ctypes.c_double
        lib.oracle_f64_to_f16.argtypes = [ctypes.c_double]
        lib.oracle_f64_to_f16.restype = ctypes.c_uint16
        lib.oracle_f64_to_bf16.argtypes = [ctypes.c_double]
        lib.oracle_f64_to_bf16.restype = ctypes.c_uint16
        for name in ("oracle_safe_softmax", "oracle_online_softmax"):
            fn = getattr(lib, name)
            fn.argtypes = [dp, i64, dp, dp, dp]
            fn.restype = None
        lib.oracle_attention_rows.argtypes = [
            u16p, u16p, u16p, ctypes.c_int, i64, i64, i64, i64, i64, i64,
            ctypes.c_double, ctypes.c_int, i64, i64, i64p, i64, dp, dp, dp,
            ctypes.c_int]
        lib.oracle_attention_rows.restype = ctypes.c_int
        lib.oracle_attention_rows_online.argtypes = [
            u16p, u16p, u16p, ctypes.c_int, i64, i64, i64, i64, i64, i64,
            ctypes.c_double, ctypes.c_int, i64, i64, i64p, i64, i64, dp, dp]
        lib.oracle_attention_rows_online.restype = ctypes.c_int
        lib.oracle_attention_rows_ex.argtypes = [
            u16p, u16p, u16p, ctypes.c_int, i64, i64, i64, i64, i64, i64,
            ctypes.c_double, ctypes.c_int, i64, i64, ctypes.c_void_p, ctypes.c_int, i64, i64,
            i64, i64p, i64, dp, dp, dp, dp, dp, dp, ctypes.c_int]
        lib.oracle_attention_rows_ex.restype = ctypes.c_int
        lib.oracle_attention_f64.argtypes = [dp, dp, dp, i64, i64, i64, i64, i64, i64,
                                             ctypes.c_double, ctypes.c_int, i64, i64, dp, dp]
        lib.oracle_attention_f64.restype = ctypes.c_int
        lib.oracle_attention_bwd_f64.argtypes = [
            dp, dp, dp, dp, i64, i64, i64, i64, i64, i64, ctypes.c_double, ctypes.c_int,
            i64, i64, dp, dp, dp, dp, dp, dp, dp, ctypes.c_int]
        lib.oracle_attention_bwd_f64.restype = ctypes.c_int
        lib.oracle_attention_bwd_f64_ex.argtypes = [
            dp, dp, dp, dp, i64, i64, i64, i64, i64, i64, ctypes.c_double, ctypes.c_int,
            i64, i64, ctypes.c_void_p, ctypes.c_int, i64, i64, i64,
            dp, dp, dp, dp, dp, dp, dp, ctypes.c_int]
        lib.oracle_attention_bwd_f64_ex.restype = ctypes.c_int
        self.lib = lib
        self._tables = {}

    # ------------------------------------------------------------- formats
    def f16_to_f64(self, bits: int) -> float:
        return self.lib.oracle_f16_to_f64(int(bits) & 0xFFFF)

    def bf16_to_f64(self, bits: int) -> float:
        return self.lib.oracle_bf16_to_f64(int(bits) & 0xFFFF)

    def e4m3_to_f64(self, bits: int) -> float:
        return self.lib.oracle_e4m3_to_f64(int(bits) & 0xFF)

    def f64_to_f16(self, x: float) -> int:
        return int(self.lib.oracle_f64_to_f16(float(x)))

    def f64_to_bf16(self, x: float) -> int:
        return int(self.lib.oracle_f64_to_bf16(float(x)))

    def decode(self, bits, dtype: int) -> np.ndarray:
        """Elementwise decode of fp16/bf16 (or e4m3) bit patterns to float64."""
        dtype = int(dtype)
        if dtype not in self._tables:
            fn = {F16: self.f16_to_f64, BF16: self.bf16_to_f64, E4M3: self.e4m3_to_f64}[dtype]
            self._tables[dtype] = np.array([fn(b) for b in range(65536)],
                                           dtype=np.float64)
        return self._tables[dtype][_bits(bits)]

    def round_to(self, x, dtype: int) -> np.ndarray:
        """Round float64 values to fp16/bf16 (ties to even); returns bits."""
        fn = self.f64_to_f16 if dtype == F16 else self.f64_to_bf16
        flat = np.asarray(x, dtype=np.float64).ravel()
        return np.array([fn(v) for v in flat],
                        dtype=np.uint16).reshape(np.shape(x))

    # ------------------------------------------------------------- softmax
    def _softmax(self, fn, x):
        x = np.ascontiguousarray(x, dtype=np.float64)
        out = np.empty_like(x)
        d = ctypes.c_double()
        m = ctypes.c_double()
        fn(_ptr(x, ctypes.c_double), x.size, _ptr(out, ctypes.c_double),
           ctypes.byref(d), ctypes.byref(m))
        return out, d.value, m.value

    def safe_softmax(self, x):
        """Three-pass safe softmax; returns (a, d, m)."""
        return self._softmax(self.lib.oracle_safe_softmax, x)

    def online_softmax(self, x):
        """Online-normaliser softmax; returns (a, d, m)."""
        return self._softmax(self.lib.oracle_online_softmax, x)

    # ------------------------------------------------------------- attention
    def attention_rows(self, q, k, v, dtype, scale, causal=False,
                       window_left=-1, window_right=-1, rows=None,
                       n_threads=0, with_wabs=False, with_wrss=False):
        """Exact attention for flattened row ids r = (b*H + h)*L_q + i
        (None = every row).  Returns (out [n, D], lse [n], threads_used), or
        (out, lse, threads_used, wabs [n, D]) with ``with_wabs``; with
        ``with_wrss`` the error scales wabs and wrss [n, D] are appended
        (out, lse, threads_used, wabs, wrss)."""
        if with_wrss:
            out, lse, _, _, wabs, wrss = self.attention_rows_ex(
                q, k, v, dtype, scale, causal, window_left, window_right, rows=rows,
                n_threads=n_threads, with_wabs=True, with_wrss=True)
            return out, lse, 0, wabs, wrss
        q, k, v, B, H, H_kv, L_q, L_k, D = _shape_args(q, k, v)
        if rows is None:
            n, rows_p = B * H * L_q, None
        else:
            rows = np.ascontiguousarray(rows, dtype=np.int64)
            n, rows_p = rows.size, _ptr(rows, ctypes.c_int64)
        out = np.zeros((n, D), dtype=np.float64)
        lse = np.zeros((n,), dtype=np.float64)
        wabs = np.zeros((n, D), dtype=np.float64) if with_wabs else None
        used = self.lib.oracle_attention_rows(
            _ptr(q, ctypes.c_uint16), _ptr(k, ctypes.c_uint16),
            _ptr(v, ctypes.c_uint16), int(dtype), B, H, H_kv, L_q, L_k, D,
            float(scale), int(bool(causal)), int(window_left),
            int(window_right), rows_p, n, _ptr(out, ctypes.c_double),
            _ptr(lse, ctypes.c_double),
            _ptr(wabs, ctypes.c_double) if with_wabs else None, int(n_threads))
        if used < 0:
            raise ValueError("oracle rejected the arguments")
        if with_wabs:
            return out, lse, used, wabs
        return out, lse, used

    def attention(self, q, k, v, dtype, scale, causal=False, window_left=-1,
                  window_right=-1, n_threads=0):
        """Every row; returns (out [B,H,L_q,D], lse [B,H,L_q])."""
        _, _, _, B, H, _, L_q, _, D = _shape_args(q, k, v)
        out, lse, _ = self.attention_rows(q, k, v, dtype, scale, causal,
                                          window_left, window_right, None,
                                          n_threads)
        return out.reshape(B, H, L_q, D), lse.reshape(B, H, L_q)

    def attention_rows_online(self, q, k, v, dtype, scale, causal=False,
                              window_left=-1, window_right=-1, rows=None,
                              block=128):
        """The FA2 block recurrence in fp64; returns (out [n, D], lse [n])."""
        q, k, v, B, H, H_kv, L_q, L_k, D = _shape_args(q, k, v)
        if rows is None:
            n, rows_p = B * H * L_q, None
        else:
            rows = np.ascontiguousarray(rows, dtype=np.int64)
            n, rows_p = rows.size, _ptr(rows, ctypes.c_int64)
        out = np.zeros((n, D), dtype=np.float64)
        lse = np.zeros((n,), dtype=np.float64)
        rc = self.lib.oracle_attention_rows_online(
            _ptr(q, ctypes.c_uint16), _ptr(k, ctypes.c_uint16),
            _ptr(v, ctypes.c_uint16), int(dtype), B, H, H_kv, L_q, L_k, D,
            float(scale), int(bool(causal)), int(window_left),
            int(window_right), rows_p, n, int(block),
            _ptr(out, ctypes.c_double), _ptr(lse, ctypes.c_double))
        if rc < 0:
            raise ValueError("oracle rejected the arguments")
        return out, lse


    # ------------------------------------------------------------- mask, statistics
    @staticmethod
    def mask_args(mask, B, H, L_q, L_k):
        """(pointer-owner array, type, stride_b, stride_h, stride_q) for a
        mask array of shape (B|1, H|1, L_q|1, L_k), dtype bool / float16 /
        float32, contiguous along the last axis; a size-1 axis broadcasts."""
        if mask is None:
            return None, 0, 0, 0, 0
        m = np.asarray(mask)
        types = {np.dtype(np.bool_): 1, np.dtype(np.uint8): 1, np.dtype(np.float16): 2,
                 np.dtype(np.float32): 3}
        if m.ndim != 4 or m.dtype not in types:
            raise ValueError("mask must be 4-D bool / float16 / float32")
        if m.shape[3] != L_k or m.strides[3] != m.itemsize:
            raise ValueError("mask must be contiguous along keys")
        want = (B, H, L_q)
        st = []
        for d in range(3):
            if m.shape[d] == 1:
                st.append(0)
            elif m.shape[d] == want[d]:
                st.append(m.strides[d] // m.itemsize)
            else:
                raise ValueError("mask shape does not broadcast")
        return m, types[m.dtype], st[0], st[1], st[2]

    def attention_rows_ex(self, q, k, v, dtype, scale, causal=False, window_left=-1,
                          window_right=-1, mask=None, rows=None, n_threads=0,
                          with_wabs=False, with_wrss=False):
        """Exact attention with an optional mask (see attention_ref.c for
        its reading); returns (out [n, D], lse, softmax_max, softmax_sum),
        plus wabs [n, D] with ``with_wabs`` and then wrss [n, D] with
        ``with_wrss`` (the two error scales stated in attention_ref.c)."""
        q, k, v, B, H, H_kv, L_q, L_k, D = _shape_args(q, k, v)
        m, mtype, sb, sh, sq = self.mask_args(mask, B, H, L_q, L_k)
        if rows is None:
            n, rows_p = B * H * L_q, None
        else:
            rows = np.ascontiguousarray(rows, dtype=np.int64)
            n, rows_p = rows.size, _ptr(rows, ctypes.c_int64)
        out = np.zeros((n, D), dtype=np.float64)
        wabs = np.zeros((n, D), dtype=np.float64) if with_wabs else None
        wrss = np.zeros((n, D), dtype=np.float64) if with_wrss else None
        lse, smax, ssum = (np.zeros((n,), dtype=np.float64) for _ in range(3))
        rc = self.lib.oracle_attention_rows_ex(
            _ptr(q, ctypes.c_uint16), _ptr(k, ctypes.c_uint16), _ptr(v, ctypes.c_uint16),
            int(dtype), B, H, H_kv, L_q, L_k, D, float(scale), int(bool(causal)),
            int(window_left), int(window_right),
            m.ctypes.data_as(ctypes.c_void_p) if m is not None else None, mtype, sb, sh, sq,
            rows_p, n, _ptr(out, ctypes.c_double), _ptr(lse, ctypes.c_double),
            _ptr(wabs, ctypes.c_double) if with_wabs else None,
            _ptr(wrss, ctypes.c_double) if with_wrss else None,
            _ptr(smax, ctypes.c_double), _ptr(ssum, ctypes.c_double), int(n_threads))
        if rc < 0:
            raise ValueError("oracle rejected the arguments")
        res = (out, lse, smax, ssum)
        if with_wabs:
            res = res + (wabs,)
        if with_wrss:
            res = res + (wrss,)
        return res

    # ------------------------------------------------------------- fp64 inputs
    @staticmethod
    def _f64(x):
        return np.ascontiguousarray(x, dtype=np.float64)

    def attention_f64(self, q, k, v, scale, causal=False, window_left=-1, window_right=-1):
        """Forward on float64 arrays q [B,H,L_q,D], k, v [B,H_kv,L_k,D] (no
        rounding anywhere); returns (out [B,H,L_q,D], lse [B,H,L_q])."""
        q, k, v = self._f64(q), self._f64(k), self._f64(v)
        B, H, L_q, D = q.shape
        _, H_kv, L_k, _ = k.shape
        out = np.zeros_like(q)
        lse = np.zeros((B, H, L_q), dtype=np.float64)
        rc = self.lib.oracle_attention_f64(
            _ptr(q, ctypes.c_double), _ptr(k, ctypes.c_double), _ptr(v, ctypes.c_double),
            B, H, H_kv, L_q, L_k, D, float(scale), int(bool(causal)), int(window_left),
            int(window_right), _ptr(out, ctypes.c_double), _ptr(lse, ctypes.c_double))
        if rc < 0:
            raise ValueError("oracle rejected the arguments")
        return out, lse

    def attention_bwd_f64(self, q, k, v, dout, scale, causal=False, window_left=-1,
                          window_right=-1, delta_err=None, with_abs=False, n_threads=0,
                          mask=None):
        """Gradients of sum(dout * O) on float64 arrays: returns (dq, dk, dv),
        or (dq, dk, dv, dq_abs, dk_abs, dv_abs) with ``with_abs`` (the error
        scales documented in attention_ref.c; ``delta_err`` [B,H,L_q]).
        ``mask``: as attention_rows_ex."""
        q, k, v, dout = self._f64(q), self._f64(k), self._f64(v), self._f64(dout)
        B, H, L_q, D = q.shape
        _, H_kv, L_k, _ = k.shape
        m, mtype, sb, sh, sq = self.mask_args(mask, B, H, L_q, L_k)
        dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
        absb = [np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)] if with_abs else None
        de = None if delta_err is None else self._f64(delta_err).reshape(B, H, L_q)
        c = ctypes.c_double
        rc = self.lib.oracle_attention_bwd_f64_ex(
            _ptr(q, c), _ptr(k, c), _ptr(v, c), _ptr(dout, c), B, H, H_kv, L_q, L_k, D,
            float(scale), int(bool(causal)), int(window_left), int(window_right),
            m.ctypes.data_as(ctypes.c_void_p) if m is not None else None, mtype, sb, sh, sq,
            _ptr(dq, c), _ptr(dk, c), _ptr(dv, c), _ptr(de, c) if de is not None else None,
            _ptr(absb[0], c) if with_abs else None, _ptr(absb[1], c) if with_abs else None,
            _ptr(absb[2], c) if with_abs else None, int(n_threads))
        if rc < 0:
            raise ValueError("oracle rejected the arguments")
        if with_abs:
            return dq, dk, dv, absb[0], absb[1], absb[2]
        return dq, dk, dv

    def attention_bwd(self, q, k, v, dout, dtype, scale, causal=False, window_left=-1,
                      window_right=-1, delta_err=None, with_abs=False, mask=None):
        """attention_bwd_f64 on fp16/bf16 bit patterns (decoded exactly)."""
        dec = [self.decode(x, dtype) for x in (q, k, v, dout)]
        return self.attention_bwd_f64(*dec, scale, causal, window_left, window_right,
                                      delta_err, with_abs, mask=mask)


_default = None


def get() -> Oracle:
    """The oracle built from attention_ref.c (compiled on first use)."""
    global _default
    with _lock:
        if _default is None:
            _default = Oracle(build())
    return _default


def __getattr__(name):
    # module-level convenience: oracle.attention(...), oracle.decode(...), ...
    if name in {"f16_to_f64", "bf16_to_f64", "e4m3_to_f64", "f64_to_f16", "f64_to_bf16",
                "decode", "round_to", "safe_softmax", "online_softmax",
                "attention_rows", "attention", "attention_rows_online",
                "attention_f64", "attention_bwd_f64", "attention_bwd",
                "attention_rows_ex", "mask_args"}:
        return getattr(get(), name)
    raise AttributeError(name)
