"""Python binding of the C ABI in include/fa.h (argument marshalling only).

``fa_fwd`` mirrors the C entry point one to one (raw pointers and sizes).
``flash_fwd`` is the convenience call for torch tensors: it checks shapes,
allocates ``out`` / ``lse`` with torch and passes the current stream; every
step of the attention itself runs in libfa.so's kernels.  There is no CPU or
eager fallback: if libfa.so cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import math
import os
import threading

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "lib", "libfa.so")

FA_F16, FA_BF16 = 0, 1
FA_OK = 0
STATUS = {
    0: "FA_OK", -1: "FA_ERR_NULL", -2: "FA_ERR_SHAPE", -3: "FA_ERR_HEADDIM",
    -4: "FA_ERR_DTYPE", -5: "FA_ERR_ALIGN", -6: "FA_ERR_ARG", -7: "FA_ERR_CUDA",
    -8: "FA_ERR_TIMEOUT", -9: "FA_ERR_WORKSPACE", -10: "FA_ERR_SCRATCH",
}
FA_MASK_NONE, FA_MASK_BOOL, FA_MASK_F16, FA_MASK_F32 = 0, 1, 2, 3
EXPORTS = ("fa_bwd", "fa_bwd_ex", "fa_bwd_workspace_bytes", "fa_fwd", "fa_fwd_ex", "fa_fwd_fp8",
           "fa_fwd_fp8_ex", "fa_fwd_fp8_splitkv",
           "fa_fwd_host", "fa_fwd_host_workspace_bytes", "fa_fwd_splitkv",
           "fa_fwd_splitkv_static", "fa_get_device_status", "fa_selftest_wait_timeout",
           "fa_splitkv_auto_splits", "fa_splitkv_workspace_bytes", "fa_status_string",
           "fa_version")
# size of the library's static split-KV scratch (FA_STATIC_SCRATCH_BYTES)
STATIC_SCRATCH_BYTES = 16 << 20

_lock = threading.Lock()
_lib = None


class FaError(RuntimeError):
    """A non-zero status from libfa.so."""

    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)} "
                         f"({status_string(status) if _lib is not None else ''})")


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libfa.so (in-tree build) and declare the C signatures."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(path):
            raise RuntimeError(
                f"libfa.so not found at {path}; build it with "
                "`python -m exact_attention_113_b200.build` (nvcc, sm_100a)")
        lib = ctypes.CDLL(path)
        vp, i = ctypes.c_void_p, ctypes.c_int
        lib.fa_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, ctypes.c_float,
                               i, i, i, i, vp]
        lib.fa_fwd.restype = i
        ll = ctypes.c_longlong
        lib.fa_fwd_ex.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i, ll, ll, ll, i, i, i, i, i,
                                  i, ctypes.c_float, i, i, i, i, vp]
        lib.fa_fwd_ex.restype = i
        f = ctypes.c_float
        lib.fa_fwd_fp8.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, f, f, f, i, i, i, vp]
        lib.fa_fwd_fp8.restype = i
        lib.fa_fwd_fp8_ex.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i, ll, ll, ll, i, i, i, i,
                                      i, i, f, f, f, f, i, i, i, vp]
        lib.fa_fwd_fp8_ex.restype = i
        lib.fa_fwd_fp8_splitkv.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, f, f, f, i, i,
                                           i, i, vp, ctypes.c_size_t, vp]
        lib.fa_fwd_fp8_splitkv.restype = i
        lib.fa_fwd_host.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, i, i, i, vp,
                                    ctypes.c_size_t, i, vp]
        lib.fa_fwd_host.restype = i
        lib.fa_fwd_host_workspace_bytes.argtypes = [i, i, i, i, i, i, i]
        lib.fa_fwd_host_workspace_bytes.restype = ctypes.c_size_t
        lib.fa_fwd_splitkv.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, ctypes.c_float,
                                       i, i, i, i, i, vp, ctypes.c_size_t, vp]
        lib.fa_fwd_splitkv.restype = i
        lib.fa_fwd_splitkv_static.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i,
                                              ctypes.c_float, i, i, i, i, i, vp]
        lib.fa_fwd_splitkv_static.restype = i
        lib.fa_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i,
                               ctypes.c_float, i, i, i, i, vp, ctypes.c_size_t, vp]
        lib.fa_bwd.restype = i
        lib.fa_bwd_ex.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, ctypes.c_longlong,
                                  ctypes.c_longlong, ctypes.c_longlong, i, i, i, i, i, i,
                                  ctypes.c_float, i, i, i, i, vp, ctypes.c_size_t, vp]
        lib.fa_bwd_ex.restype = i
        lib.fa_bwd_workspace_bytes.argtypes = [i, i, i, i]
        lib.fa_bwd_workspace_bytes.restype = ctypes.c_size_t
        lib.fa_splitkv_workspace_bytes.argtypes = [i, i, i, i, i]
        lib.fa_splitkv_workspace_bytes.restype = ctypes.c_size_t
        lib.fa_splitkv_auto_splits.argtypes = [i, i, i, i, i, i, i]
        lib.fa_splitkv_auto_splits.restype = i
        lib.fa_get_device_status.argtypes = [vp]
        lib.fa_get_device_status.restype = i
        lib.fa_selftest_wait_timeout.argtypes = [vp, vp]
        lib.fa_selftest_wait_timeout.restype = i
        lib.fa_status_string.argtypes = [i]
        lib.fa_status_string.restype = ctypes.c_char_p
        lib.fa_version.argtypes = []
        lib.fa_version.restype = i
        _lib = lib
        return lib


# ------------------------------------------------------------ raw C calls
def fa_fwd(q, k, v, out, lse, B, H, H_kv, L_q, L_k, D, scale, causal,
           window_left, window_right, dtype, stream) -> int:
    """The C entry point, unchanged: pointers as ints, returns the status."""
    return load().fa_fwd(q, k, v, out, lse, B, H, H_kv, L_q, L_k, D,
                         float(scale), int(causal), int(window_left),
                         int(window_right), int(dtype), stream)


def fa_fwd_ex(q, k, v, out, lse, softmax_max, softmax_sum, mask, mask_type, mask_stride_b,
              mask_stride_h, mask_stride_q, B, H, H_kv, L_q, L_k, D, scale, causal,
              window_left, window_right, dtype, stream) -> int:
    """The masked / statistics C entry point, unchanged."""
    return load().fa_fwd_ex(q, k, v, out, lse, softmax_max, softmax_sum, mask, int(mask_type),
                            int(mask_stride_b), int(mask_stride_h), int(mask_stride_q), B, H,
                            H_kv, L_q, L_k, D, float(scale), int(causal), int(window_left),
                            int(window_right), int(dtype), stream)


def fa_fwd_fp8(q, k, v, out, lse, B, H, H_kv, L_q, L_k, D, scale, descale_q, descale_k,
               descale_v, causal, window_left, window_right, stream) -> int:
    """The fp8 (E4M3) C entry point, unchanged."""
    return load().fa_fwd_fp8(q, k, v, out, lse, B, H, H_kv, L_q, L_k, D, float(scale),
                             float(descale_q), float(descale_k), float(descale_v), int(causal),
                             int(window_left), int(window_right), stream)


def fa_fwd_fp8_ex(q, k, v, out, lse, smax, ssum, mask, mask_type, mask_stride_b, mask_stride_h,
                  mask_stride_q, B, H, H_kv, L_q, L_k, D, scale, descale_q, descale_k,
                  descale_v, causal, window_left, window_right, stream) -> int:
    """The fp8 (E4M3) C entry point with mask and statistics, unchanged."""
    return load().fa_fwd_fp8_ex(q, k, v, out, lse, smax, ssum, mask, int(mask_type),
                                int(mask_stride_b), int(mask_stride_h), int(mask_stride_q), B, H,
                                H_kv, L_q, L_k, D, float(scale), float(descale_q),
                                float(descale_k), float(descale_v), int(causal),
                                int(window_left), int(window_right), stream)


def fa_fwd_fp8_splitkv(q, k, v, out, lse, B, H, H_kv, L_q, L_k, D, scale, descale_q,
                       descale_k, descale_v, causal, window_left, window_right, n_splits,
                       workspace, workspace_bytes, stream) -> int:
    """The fp8 (E4M3) split-KV C entry point, unchanged."""
    return load().fa_fwd_fp8_splitkv(q, k, v, out, lse, B, H, H_kv, L_q, L_k, D, float(scale),
                                     float(descale_q), float(descale_k), float(descale_v),
                                     int(causal), int(window_left), int(window_right),
                                     int(n_splits), workspace, int(workspace_bytes), stream)


def fa_fwd_host(q, k, v, out, lse, B, H, H_kv, L_q, L_k, D, scale, causal, window_left,
                window_right, dtype, workspace, workspace_bytes, n_chunks, stream) -> int:
    """The host-buffer (pipelined) C entry point, unchanged."""
    return load().fa_fwd_host(q, k, v, out, lse, B, H, H_kv, L_q, L_k, D, float(scale),
                              int(causal), int(window_left), int(window_right), int(dtype),
                              workspace, int(workspace_bytes), int(n_chunks), stream)


def fa_fwd_host_workspace_bytes(B, H, H_kv, L_q, L_k, D, n_chunks) -> int:
    return int(load().fa_fwd_host_workspace_bytes(B, H, H_kv, L_q, L_k, D, n_chunks))


def mask_layout(mask, B, H, L_q, L_k):
    """(type, stride_b, stride_h, stride_q) of a torch mask of shape
    (B|1, H|1, L_q|1, L_k), dtype bool / float16 / float32, contiguous along
    the keys; a size-1 axis broadcasts (stride 0)."""
    import torch
    types = {torch.bool: FA_MASK_BOOL, torch.uint8: FA_MASK_BOOL, torch.float16: FA_MASK_F16,
             torch.float32: FA_MASK_F32}
    if mask.dim() != 4 or mask.dtype not in types:
        raise ValueError("mask must be 4-D bool / uint8 / float16 / float32")
    if mask.shape[3] != L_k or (L_k > 1 and mask.stride(3) != 1):
        raise ValueError("mask must be [.., .., .., L_k], contiguous along the keys")
    st = []
    for d, want in enumerate((B, H, L_q)):
        if mask.shape[d] == 1:
            st.append(0)
        elif mask.shape[d] == want:
            st.append(mask.stride(d))
        else:
            raise ValueError("mask shape does not broadcast to [B, H, L_q, L_k]")
    return types[mask.dtype], st[0], st[1], st[2]


def fa_fwd_splitkv(q, k, v, out, lse, B, H, H_kv, L_q, L_k, D, scale, causal,
                   window_left, window_right, dtype, n_splits, workspace,
                   workspace_bytes, stream) -> int:
    """The split-KV C entry point, unchanged."""
    return load().fa_fwd_splitkv(q, k, v, out, lse, B, H, H_kv, L_q, L_k, D,
                                 float(scale), int(causal), int(window_left),
                                 int(window_right), int(dtype), int(n_splits),
                                 workspace, int(workspace_bytes), stream)


def fa_fwd_splitkv_static(q, k, v, out, lse, B, H, H_kv, L_q, L_k, D, scale, causal,
                          window_left, window_right, dtype, n_splits, stream) -> int:
    """The no-allocation split-KV C entry point, unchanged (its partials
    live in the library's static scratch; see include/fa.h)."""
    return load().fa_fwd_splitkv_static(q, k, v, out, lse, B, H, H_kv, L_q, L_k, D,
                                        float(scale), int(causal), int(window_left),
                                        int(window_right), int(dtype), int(n_splits), stream)


def fa_bwd(q, k, v, out, dout, lse, dq, dk, dv, B, H, H_kv, L_q, L_k, D, scale, causal,
           window_left, window_right, dtype, workspace, workspace_bytes, stream) -> int:
    """The backward C entry point, unchanged."""
    return load().fa_bwd(q, k, v, out, dout, lse, dq, dk, dv, B, H, H_kv, L_q, L_k, D,
                         float(scale), int(causal), int(window_left), int(window_right),
                         int(dtype), workspace, int(workspace_bytes), stream)


def fa_bwd_ex(q, k, v, out, dout, lse, dq, dk, dv, mask, mask_type, mask_stride_b,
              mask_stride_h, mask_stride_q, B, H, H_kv, L_q, L_k, D, scale, causal, window_left,
              window_right, dtype, workspace, workspace_bytes, stream) -> int:
    """The masked backward C entry point, unchanged."""
    return load().fa_bwd_ex(q, k, v, out, dout, lse, dq, dk, dv, mask, int(mask_type),
                            int(mask_stride_b), int(mask_stride_h), int(mask_stride_q), B, H,
                            H_kv, L_q, L_k, D, float(scale), int(causal), int(window_left),
                            int(window_right), int(dtype), workspace, int(workspace_bytes),
                            stream)


def fa_bwd_workspace_bytes(B, H, L_q, D) -> int:
    return int(load().fa_bwd_workspace_bytes(B, H, L_q, D))


def fa_splitkv_workspace_bytes(B, H, L_q, D, n_splits) -> int:
    return int(load().fa_splitkv_workspace_bytes(B, H, L_q, D, n_splits))


def query_tiles(B, H, H_kv, L_q) -> int:
    """128-row query tiles of a launch.  With GQA (H / H_kv a power of two)
    and L_q < 128 the library packs a group's heads into one tile:
    128 / group query positions of each head."""
    g = H // H_kv
    if 2 <= g <= 128 and (g & (g - 1)) == 0 and L_q < 128:
        return B * H_kv * max(1, -(-L_q // (128 // g)))
    return B * H * max(1, -(-L_q // 128))


def choose_splits(B, H, L_q, L_k, sm_count=None, H_kv=None, D=128, dtype=FA_F16) -> int:
    """Key slices for fa_fwd_splitkv: the library's own choice
    (fa_splitkv_auto_splits, on the current device; ``sm_count`` is not
    used, the device's count is).  dtype 2 = E4M3 inputs."""
    return int(load().fa_splitkv_auto_splits(B, H, H if H_kv is None else H_kv, L_q, L_k, D,
                                             dtype))


def fa_get_device_status(stream=None) -> int:
    return load().fa_get_device_status(stream)


def fa_selftest_wait_timeout(result, stream=None) -> int:
    """The C entry point: `result` is a device pointer to 6 ints."""
    return load().fa_selftest_wait_timeout(result, stream)


def selftest_wait_timeout(device=None) -> dict:
    """Run the watchdog self-test on `device` (about 1 s of one SM) and
    return its six result fields plus the device status read afterwards."""
    import torch
    dev = torch.device("cuda", torch.cuda.current_device() if device is None else device)
    with torch.cuda.device(dev):
        res = torch.full((6,), -1, dtype=torch.int32, device=dev)
        stream = torch.cuda.current_stream(dev)
        st = fa_selftest_wait_timeout(res.data_ptr(), stream.cuda_stream)
        if st != 0:
            raise FaError(st, "fa_selftest_wait_timeout")
        status = fa_get_device_status(stream.cuda_stream)
        r = [int(x) for x in res.cpu()]
    keys = ("done_ok", "never_ok", "abort_flag", "wait_ms", "follower_ok", "follower_ms")
    out = dict(zip(keys, r))
    out["status"] = status
    return out


def status_string(status: int) -> str:
    return load().fa_status_string(int(status)).decode()


def fa_version() -> int:
    return load().fa_version()


# ------------------------------------------------------------ torch call
def flash_fwd(q, k, v, scale=None, causal=False, window_left=-1, window_right=-1,
              return_lse=True, out=None, lse=None, stream=None, n_splits=0,
              workspace=None, mask=None, return_softmax_stats=False):
    """Exact attention forward on CUDA tensors.

    q: [B, H, L_q, D]; k, v: [B, H_kv, L_k, D]; fp16 or bf16, contiguous, on
    one CUDA device.  ``scale`` defaults to 1/sqrt(D).  Returns ``(out, lse)``
    (``lse`` is None unless ``return_lse``).  Launches asynchronously on
    ``stream`` (default: torch's current stream).

    ``n_splits`` > 0 computes the same result through fa_fwd_splitkv with
    that many key slices ("auto" picks them with ``choose_splits``); the
    workspace is allocated here with torch unless ``workspace`` (a uint8
    CUDA tensor, 256-byte aligned) is given.  ``workspace="static"`` calls
    fa_fwd_splitkv_static instead, which uses the library's fixed scratch
    and allocates nothing (calls must not overlap on the GPU).

    ``mask`` (bool: True hides the key; float16 / float32: added to the
    scaled scores), shape (B|1, H|1, L_q|1, L_k), and
    ``return_softmax_stats`` (the row max and sum_j exp(s_j - max)) go
    through fa_fwd_ex; the result is then (out, lse, softmax_max,
    softmax_sum).
    """
    import torch

    if q.dim() != 4 or k.dim() != 4 or v.dim() != 4:
        raise ValueError("q, k, v must be 4-D [B, H, L, D]")
    B, H, L_q, D = q.shape
    Bk, H_kv, L_k, Dk = k.shape
    if tuple(v.shape) != tuple(k.shape) or Bk != B or Dk != D:
        raise ValueError("k, v must be [B, H_kv, L_k, D] with q's B and D")
    if q.dtype not in (torch.float16, torch.bfloat16) or k.dtype != q.dtype \
            or v.dtype != q.dtype:
        raise TypeError("q, k, v must share dtype float16 or bfloat16")
    if not (q.is_cuda and k.is_cuda and v.is_cuda):
        raise ValueError("q, k, v must be CUDA tensors")
    if not (q.is_contiguous() and k.is_contiguous() and v.is_contiguous()):
        raise ValueError("q, k, v must be contiguous")
    dtype = FA_F16 if q.dtype == torch.float16 else FA_BF16
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q)
    if return_lse and lse is None:
        lse = torch.empty((B, H, L_q), dtype=torch.float32, device=q.device)
    if not return_lse:
        lse = None
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    if mask is not None or return_softmax_stats:
        if n_splits:
            raise ValueError("mask / softmax statistics are not available with n_splits")
        mtype, sb, sh, sq = (FA_MASK_NONE, 0, 0, 0) if mask is None else \
            mask_layout(mask, B, H, L_q, L_k)
        if mask is not None and (not mask.is_cuda or mask.device != q.device):
            raise ValueError("mask must be on q's device")
        smax = ssum = None
        if return_softmax_stats:
            smax = torch.empty((B, H, L_q), dtype=torch.float32, device=q.device)
            ssum = torch.empty_like(smax)
        with torch.cuda.device(q.device):
            st = fa_fwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                           lse.data_ptr() if lse is not None else None,
                           smax.data_ptr() if smax is not None else None,
                           ssum.data_ptr() if ssum is not None else None,
                           mask.data_ptr() if mask is not None else None, mtype, sb, sh, sq,
                           B, H, H_kv, L_q, L_k, D, scale, causal, window_left, window_right,
                           dtype, stream.cuda_stream)
        if st != FA_OK:
            raise FaError(st, "fa_fwd_ex")
        return out, lse, smax, ssum
    if n_splits == "auto":
        with torch.cuda.device(q.device):
            n_splits = choose_splits(B, H, L_q, L_k, H_kv=H_kv, D=D, dtype=dtype)
    with torch.cuda.device(q.device):
        if not n_splits:
            st = fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                        lse.data_ptr() if lse is not None else None,
                        B, H, H_kv, L_q, L_k, D, scale, causal, window_left,
                        window_right, dtype, stream.cuda_stream)
            where = "fa_fwd"
        elif isinstance(workspace, str) and workspace == "static":
            st = fa_fwd_splitkv_static(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                       lse.data_ptr() if lse is not None else None,
                                       B, H, H_kv, L_q, L_k, D, scale, causal, window_left,
                                       window_right, dtype, n_splits, stream.cuda_stream)
            where = "fa_fwd_splitkv_static"
        else:
            need = fa_splitkv_workspace_bytes(B, H, L_q, D, n_splits)
            if workspace is None:
                workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
            st = fa_fwd_splitkv(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                lse.data_ptr() if lse is not None else None,
                                B, H, H_kv, L_q, L_k, D, scale, causal, window_left,
                                window_right, dtype, n_splits, workspace.data_ptr(),
                                workspace.numel(), stream.cuda_stream)
            where = "fa_fwd_splitkv"
    if st != FA_OK:
        raise FaError(st, where)
    return out, lse


def flash_bwd(q, k, v, out, dout, lse, scale=None, causal=False, window_left=-1,
              window_right=-1, dq=None, dk=None, dv=None, workspace=None, stream=None,
              mask=None):
    """Exact attention backward on CUDA tensors: returns (dq, dk, dv).

    q, out, dout: [B, H, L_q, D]; k, v: [B, H_kv, L_k, D]; lse: [B, H, L_q]
    fp32 from the forward (same scale and mask).  The workspace is allocated
    here with torch unless given (a uint8 CUDA tensor, 256-byte aligned).
    ``mask``: the forward's attention mask (as flash_fwd), through fa_bwd_ex."""
    import torch

    B, H, L_q, D = q.shape
    _, H_kv, L_k, _ = k.shape
    for name, t, shape in (("out", out, q.shape), ("dout", dout, q.shape), ("v", v, k.shape)):
        if tuple(t.shape) != tuple(shape):
            raise ValueError(f"{name} must have shape {tuple(shape)}")
    if tuple(lse.shape) != (B, H, L_q) or lse.dtype != torch.float32:
        raise ValueError("lse must be fp32 [B, H, L_q]")
    if q.dtype not in (torch.float16, torch.bfloat16) or any(
            t.dtype != q.dtype for t in (k, v, out, dout)):
        raise TypeError("q, k, v, out, dout must share dtype float16 or bfloat16")
    ts = (q, k, v, out, dout, lse)
    if not all(t.is_cuda for t in ts) or not all(t.is_contiguous() for t in ts):
        raise ValueError("inputs must be contiguous CUDA tensors")
    dtype = FA_F16 if q.dtype == torch.float16 else FA_BF16
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if workspace is None:
        workspace = torch.empty(max(fa_bwd_workspace_bytes(B, H, L_q, D), 1), dtype=torch.uint8,
                                device=q.device)
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    with torch.cuda.device(q.device):
        if mask is None:
            st = fa_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                        dout.data_ptr(), lse.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                        dv.data_ptr(), B, H, H_kv, L_q, L_k, D, scale, causal, window_left,
                        window_right, dtype, workspace.data_ptr(), workspace.numel(),
                        stream.cuda_stream)
            where = "fa_bwd"
        else:
            if not mask.is_cuda or mask.device != q.device:
                raise ValueError("mask must be on q's device")
            mtype, sb, sh, sq = mask_layout(mask, B, H, L_q, L_k)
            st = fa_bwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                           dout.data_ptr(), lse.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                           dv.data_ptr(), mask.data_ptr(), mtype, sb, sh, sq, B, H, H_kv, L_q,
                           L_k, D, scale, causal, window_left, window_right, dtype,
                           workspace.data_ptr(), workspace.numel(), stream.cuda_stream)
            where = "fa_bwd_ex"
    if st != FA_OK:
        raise FaError(st, where)
    return dq, dk, dv


def flash_fwd_fp8(q, k, v, scale=None, descale_q=1.0, descale_k=1.0, descale_v=1.0,
                  causal=False, window_left=-1, window_right=-1, return_lse=True, out=None,
                  lse=None, stream=None, n_splits=0, workspace=None, mask=None,
                  return_softmax_stats=False):
    """Exact attention forward on fp8 E4M3 CUDA tensors (torch.float8_e4m3fn
    or uint8 codes), q [B, H, L_q, D], k, v [B, H_kv, L_k, D]; real values are
    code * descale.  Returns (out bf16 [B, H, L_q, D], lse or None).
    ``n_splits`` > 0 (or "auto") goes through fa_fwd_fp8_splitkv with that
    many key slices; the workspace is allocated here with torch unless
    given (a uint8 CUDA tensor, 256-byte aligned).  ``mask`` and
    ``return_softmax_stats`` as in flash_fwd (through fa_fwd_fp8_ex; the
    result is then (out, lse, softmax_max, softmax_sum))."""
    import torch

    B, H, L_q, D = q.shape
    _, H_kv, L_k, _ = k.shape
    ok_types = (torch.float8_e4m3fn, torch.uint8)
    if any(t.dtype not in ok_types for t in (q, k, v)) or tuple(v.shape) != tuple(k.shape):
        raise TypeError("q, k, v must be float8_e4m3fn (or uint8 codes), k and v of one shape")
    if not all(t.is_cuda and t.is_contiguous() for t in (q, k, v)):
        raise ValueError("q, k, v must be contiguous CUDA tensors")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty((B, H, L_q, D), dtype=torch.bfloat16, device=q.device)
    if return_lse and lse is None:
        lse = torch.empty((B, H, L_q), dtype=torch.float32, device=q.device)
    if not return_lse:
        lse = None
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    if mask is not None or return_softmax_stats:
        if n_splits:
            raise ValueError("mask / softmax statistics are not available with n_splits")
        mtype, sb, sh, sq = (FA_MASK_NONE, 0, 0, 0) if mask is None else \
            mask_layout(mask, B, H, L_q, L_k)
        if mask is not None and (not mask.is_cuda or mask.device != q.device):
            raise ValueError("mask must be on q's device")
        smax = ssum = None
        if return_softmax_stats:
            smax = torch.empty((B, H, L_q), dtype=torch.float32, device=q.device)
            ssum = torch.empty_like(smax)
        with torch.cuda.device(q.device):
            st = fa_fwd_fp8_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                               lse.data_ptr() if lse is not None else None,
                               smax.data_ptr() if smax is not None else None,
                               ssum.data_ptr() if ssum is not None else None,
                               mask.data_ptr() if mask is not None else None, mtype, sb, sh, sq,
                               B, H, H_kv, L_q, L_k, D, scale, descale_q, descale_k, descale_v,
                               causal, window_left, window_right, stream.cuda_stream)
        if st != FA_OK:
            raise FaError(st, "fa_fwd_fp8_ex")
        return out, lse, smax, ssum
    if n_splits == "auto":
        with torch.cuda.device(q.device):
            n_splits = choose_splits(B, H, L_q, L_k, H_kv=H_kv, D=D, dtype=2)
    with torch.cuda.device(q.device):
        if not n_splits:
            st = fa_fwd_fp8(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                            lse.data_ptr() if lse is not None else None, B, H, H_kv, L_q, L_k,
                            D, scale, descale_q, descale_k, descale_v, causal, window_left,
                            window_right, stream.cuda_stream)
            where = "fa_fwd_fp8"
        else:
            need = fa_splitkv_workspace_bytes(B, H, L_q, D, n_splits)
            if workspace is None:
                workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
            st = fa_fwd_fp8_splitkv(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                    lse.data_ptr() if lse is not None else None, B, H, H_kv,
                                    L_q, L_k, D, scale, descale_q, descale_k, descale_v, causal,
                                    window_left, window_right, n_splits, workspace.data_ptr(),
                                    workspace.numel(), stream.cuda_stream)
            where = "fa_fwd_fp8_splitkv"
    if st != FA_OK:
        raise FaError(st, where)
    return out, lse


def flash_fwd_host(q, k, v, scale=None, causal=False, window_left=-1, window_right=-1,
                   out=None, lse=None, n_chunks=8, workspace=None, device=None, stream=None):
    """Exact attention forward on host (CPU, preferably pinned) tensors
    through fa_fwd_host: chunked copies in, kernels, copies out, overlapped.
    Returns (out, lse) as host tensors, valid once ``stream`` (default: the
    device's current stream) is synchronised.  The device workspace is
    allocated here with torch unless given."""
    import torch

    B, H, L_q, D = q.shape
    _, H_kv, L_k, _ = k.shape
    if q.is_cuda or k.is_cuda or v.is_cuda:
        raise ValueError("flash_fwd_host takes host tensors")
    if q.dtype not in (torch.float16, torch.bfloat16) or k.dtype != q.dtype or v.dtype != q.dtype:
        raise TypeError("q, k, v must share dtype float16 or bfloat16")
    if not (q.is_contiguous() and k.is_contiguous() and v.is_contiguous()):
        raise ValueError("q, k, v must be contiguous")
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    dtype = FA_F16 if q.dtype == torch.float16 else FA_BF16
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    pin = q.is_pinned()
    if out is None:
        out = torch.empty(q.shape, dtype=q.dtype, pin_memory=pin)
    if lse is None:
        lse = torch.empty((B, H, L_q), dtype=torch.float32, pin_memory=pin)
    if workspace is None:
        nbytes = fa_fwd_host_workspace_bytes(B, H, H_kv, L_q, L_k, D, n_chunks)
        workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=dev)
    if stream is None:
        stream = torch.cuda.current_stream(dev)
    with torch.cuda.device(dev):
        st = fa_fwd_host(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                         lse.data_ptr(), B, H, H_kv, L_q, L_k, D, scale, causal, window_left,
                         window_right, dtype, workspace.data_ptr(), workspace.numel(), n_chunks,
                         stream.cuda_stream)
    if st != FA_OK:
        raise FaError(st, "fa_fwd_host")
    return out, lse
