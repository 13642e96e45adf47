"""Host-side checks of the C ABI (CPU only: no kernel is launched).

The library must load without a GPU, export every function include/fa.h
declares, and reject bad arguments with the documented status codes before
any CUDA call is made."""
import os
import re
import subprocess

import pytest

import exact_attention_113_b200 as fa
from exact_attention_113_b200 import binding
from exact_attention_113_b200.build import build, LIB_PATH

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "fa.h")


@pytest.fixture(scope="module")
def lib():
    build()
    return fa.load()


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(fa_\w+)\s*\(", text, re.M)))


def test_header_declares_the_boundary():
    assert _declared() == sorted(binding.EXPORTS)


def test_every_declared_symbol_is_exported(lib):
    for name in _declared():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (\w+)$", out, re.M))
    assert set(_declared()) <= exported


def test_status_strings_and_version(lib):
    assert fa.fa_version() >= 10000
    for code, name in binding.STATUS.items():
        assert fa.status_string(code).startswith(name)
    assert fa.status_string(12345) == "unknown fa status"


GOOD = dict(q=16, k=16, v=16, out=16, lse=0, B=1, H=4, H_kv=2, L_q=8, L_k=8, D=64,
            scale=0.125, causal=0, wl=-1, wr=-1, dtype=0)


def _call(**kw):
    a = dict(GOOD)
    a.update(kw)
    return fa.fa_fwd(a["q"], a["k"], a["v"], a["out"], a["lse"], a["B"], a["H"], a["H_kv"],
                     a["L_q"], a["L_k"], a["D"], a["scale"], a["causal"], a["wl"], a["wr"],
                     a["dtype"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=0), -1), (dict(k=0), -1), (dict(v=0), -1), (dict(out=0), -1),
    (dict(B=0), -2), (dict(H=0), -2), (dict(H_kv=0), -2), (dict(H=4, H_kv=3), -2),
    (dict(L_q=-1), -2), (dict(L_k=-5), -2), (dict(L_q=(1 << 30) + 1), -2),
    (dict(B=1 << 16, H=1 << 15, L_q=1 << 10), -2),
    (dict(D=0), -3), (dict(D=40), -3), (dict(D=8), -3), (dict(D=144), -3), (dict(D=256), -3),
    (dict(dtype=2), -4), (dict(dtype=-1), -4),
    (dict(q=24), -5), (dict(out=8), -5), (dict(v=4), -5), (dict(lse=2), -5),
    (dict(scale=-0.5), -6), (dict(scale=float("nan")), -6), (dict(scale=float("inf")), -6),
])
def test_argument_errors(lib, kw, code):
    assert _call(**kw) == code


def test_empty_query_is_a_no_op(lib):
    # L_q == 0 returns before touching the device (pointers are never read)
    assert _call(L_q=0) == 0
    # tensors with no elements may have NULL pointers
    assert _call(L_q=0, q=0, out=0) == 0
    assert _call(L_q=0, q=0, out=0, L_k=0, k=0, v=0) == 0


def test_flash_fwd_rejects_bad_tensors(lib):
    import torch
    q = torch.zeros(1, 2, 8, 64, dtype=torch.float16)
    with pytest.raises(ValueError):
        fa.flash_fwd(q, q, q)                       # CPU tensors
    with pytest.raises(ValueError):
        fa.flash_fwd(q[0], q, q)                    # not 4-D
    with pytest.raises(TypeError):
        fa.flash_fwd(q.float(), q.float(), q.float())
    with pytest.raises(ValueError):
        fa.flash_fwd(q, q[:, :, :, :32], q)         # D mismatch


def test_other_wrappers_reject_bad_tensors(lib):
    import torch
    q = torch.zeros(1, 2, 8, 64, dtype=torch.float16)
    c = torch.zeros(1, 2, 8, 64, dtype=torch.uint8)
    with pytest.raises(TypeError):
        fa.flash_fwd_fp8(q, q, q)                   # not E4M3 codes
    with pytest.raises(ValueError):
        fa.flash_fwd_fp8(c, c, c)                   # CPU tensors
    with pytest.raises(TypeError):
        fa.flash_fwd_host(q.float(), q.float(), q.float())


# ------------------------------------------------------------ split-KV entry
def _call_split(n_splits=2, ws=256, ws_bytes=None, **kw):
    a = dict(GOOD)
    a.update(kw)
    if ws_bytes is None:
        ws_bytes = fa.fa_splitkv_workspace_bytes(a["B"], a["H"], a["L_q"], a["D"],
                                                 max(1, min(64, n_splits)))
    return fa.fa_fwd_splitkv(a["q"], a["k"], a["v"], a["out"], a["lse"], a["B"], a["H"],
                             a["H_kv"], a["L_q"], a["L_k"], a["D"], a["scale"], a["causal"],
                             a["wl"], a["wr"], a["dtype"], n_splits, ws, ws_bytes, None)


def test_splitkv_workspace_bytes(lib):
    # B*H*L_q rows of D fp32 per slice, then (m, l) float2 per row and slice
    rows, D, S = 2 * 4 * 8, 64, 3
    o = S * rows * D * 4
    assert fa.fa_splitkv_workspace_bytes(2, 4, 8, D, S) == ((o + 255) // 256) * 256 + S * rows * 8
    assert fa.fa_splitkv_workspace_bytes(2, 4, 8, 40, S) == 0
    assert fa.fa_splitkv_workspace_bytes(2, 4, 8, 48, S) > 0          # any multiple of 16
    assert fa.fa_splitkv_workspace_bytes(2, 4, 8, 64, 0) == 0
    assert fa.fa_splitkv_workspace_bytes(2, 4, 8, 64, 65) == 0


@pytest.mark.parametrize("kw,code", [
    (dict(n_splits=0), -6), (dict(n_splits=65), -6), (dict(n_splits=-1), -6),
    (dict(ws=0), -1), (dict(ws=128), -5), (dict(ws_bytes=100), -9),
    (dict(q=0), -1), (dict(D=40), -3), (dict(scale=-1.0), -6),
])
def test_splitkv_argument_errors(lib, kw, code):
    assert _call_split(**kw) == code


def test_choose_splits():
    # decoding shapes (one or two rows per K/V head) go to the CUDA-core kernel,
    # whose slots let every one of the 148 SMs take an equal share of the keys:
    # ceil(148 / heads) + 2 slots, or whole heads from 3 heads per 4 SMs on
    assert fa.choose_splits(1, 32, 1, 32768) == 7       # 32 heads -> 5 + 2
    assert fa.choose_splits(4, 32, 1, 16384) == 1       # 128 heads: whole heads, no merge
    assert fa.choose_splits(1, 1, 1, 128) == 1          # too few keys to split
    assert fa.choose_splits(1, 1, 1, 1 << 20) == 64     # capped
    # the tensor-core kernel: query tiles x slices in waves of one CTA per SM
    assert fa.choose_splits(4, 48, 8192, 8192) == 1     # already many waves
    # GQA packing: 32 query heads over 8 K/V heads, one query row -> 8 tiles
    assert fa.binding.query_tiles(1, 32, 8, 1) == 8
    assert fa.binding.query_tiles(1, 32, 8, 40) == 16      # 32 rows per head per tile
    assert fa.binding.query_tiles(1, 12, 2, 1) == 12       # group 6: not packed
    assert fa.binding.query_tiles(1, 32, 8, 128) == 32     # long enough: not packed
    assert fa.choose_splits(1, 32, 1, 32768, H_kv=8) == 18  # 144 CTAs, one wave
    assert fa.choose_splits(8, 32, 1, 32768, H_kv=8) == 2   # 128 CTAs, one wave


# ------------------------------------------------------------ static-scratch entry
def _call_static(n_splits=2, **kw):
    a = dict(GOOD)
    a.update(kw)
    return fa.fa_fwd_splitkv_static(a["q"], a["k"], a["v"], a["out"], a["lse"], a["B"], a["H"],
                                    a["H_kv"], a["L_q"], a["L_k"], a["D"], a["scale"],
                                    a["causal"], a["wl"], a["wr"], a["dtype"], n_splits, None)


def test_static_scratch_size_matches_header():
    text = open(HEADER).read()
    assert "#define FA_STATIC_SCRATCH_BYTES ((size_t)16 << 20)" in text
    assert binding.STATIC_SCRATCH_BYTES == 16 << 20


@pytest.mark.parametrize("kw,code", [
    (dict(n_splits=0), -6), (dict(n_splits=65), -6),
    # 32768 rows x 2 slices x (128 fp32 + one float2) = 33.5 MB > 16 MiB:
    # refused before any CUDA call
    (dict(n_splits=2, B=1, H=64, H_kv=64, L_q=512, D=128), -10),
    (dict(n_splits=64, B=1, H=8, H_kv=8, L_q=128, D=128), -10),
])
def test_static_entry_refuses_before_the_gpu(lib, kw, code):
    assert _call_static(**kw) == code


# ------------------------------------------------------------ backward entry
BWD_GOOD = dict(q=16, k=16, v=16, out=16, dout=16, lse=16, dq=16, dk=16, dv=16, B=1, H=4,
                H_kv=2, L_q=8, L_k=8, D=64, scale=0.125, causal=0, wl=-1, wr=-1, dtype=0,
                ws=256, ws_bytes=1 << 30)


def _call_bwd(**kw):
    a = dict(BWD_GOOD)
    a.update(kw)
    return fa.fa_bwd(a["q"], a["k"], a["v"], a["out"], a["dout"], a["lse"], a["dq"], a["dk"],
                     a["dv"], a["B"], a["H"], a["H_kv"], a["L_q"], a["L_k"], a["D"], a["scale"],
                     a["causal"], a["wl"], a["wr"], a["dtype"], a["ws"], a["ws_bytes"], None)


def test_bwd_workspace_bytes(lib):
    # dQ accumulator (B*H*L_q*D fp32), then lse2 and delta over L_q padded to 128
    up = lambda x: (x + 255) // 256 * 256
    B, H, L_q, D = 2, 3, 130, 64
    want = up(B * H * L_q * D * 4) + 2 * up(B * H * 256 * 4)
    assert fa.fa_bwd_workspace_bytes(B, H, L_q, D) == want
    assert fa.fa_bwd_workspace_bytes(B, H, L_q, 40) == 0
    assert fa.fa_bwd_workspace_bytes(B, H, L_q, 48) > 0          # any multiple of 16
    assert fa.fa_bwd_workspace_bytes(0, H, L_q, 64) == 0


@pytest.mark.parametrize("kw,code", [
    (dict(q=0), -1), (dict(dout=0), -1), (dict(lse=0), -1), (dict(dk=0), -1), (dict(ws=0), -1),
    (dict(B=0), -2), (dict(H=4, H_kv=3), -2), (dict(L_k=-1), -2),
    (dict(D=40), -3), (dict(D=144), -3), (dict(dtype=2), -4),
    (dict(dq=8), -5), (dict(lse=2), -5), (dict(ws=128), -5),
    (dict(scale=float("nan")), -6), (dict(ws_bytes=1000), -9),
])
def test_bwd_argument_errors(lib, kw, code):
    assert _call_bwd(**kw) == code


# ------------------------------------------------------------ masked / statistics entry
def _call_ex(mask=16, mtype=1, sb=0, sh=0, sq=8, smax=0, ssum=0, **kw):
    a = dict(GOOD)
    a.update(kw)
    return fa.fa_fwd_ex(a["q"], a["k"], a["v"], a["out"], a["lse"], smax, ssum, mask, mtype,
                        sb, sh, sq, a["B"], a["H"], a["H_kv"], a["L_q"], a["L_k"], a["D"],
                        a["scale"], a["causal"], a["wl"], a["wr"], a["dtype"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(mtype=4), -6), (dict(mtype=-1), -6), (dict(sq=-1), -6), (dict(sb=-8), -6),
    (dict(mask=0), -1), (dict(smax=16, ssum=0), -1), (dict(smax=0, ssum=16), -1),
    (dict(smax=18, ssum=16), -5), (dict(q=0), -1), (dict(D=40), -3),
])
def test_ex_argument_errors(lib, kw, code):
    assert _call_ex(**kw) == code


# ------------------------------------------------------------ fp8 entry
def _call_fp8(dq=1.0, dk=1.0, dv=1.0, **kw):
    a = dict(GOOD)
    a.update(kw)
    return fa.fa_fwd_fp8(a["q"], a["k"], a["v"], a["out"], a["lse"], a["B"], a["H"], a["H_kv"],
                         a["L_q"], a["L_k"], a["D"], a["scale"], dq, dk, dv, a["causal"],
                         a["wl"], a["wr"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(D=16), -3), (dict(D=48), -3), (dict(q=0), -1), (dict(q=8), -5),
    (dict(dq=-1.0), -6), (dict(dv=float("inf")), -6), (dict(scale=-1.0), -6),
    (dict(dq=1e30, dk=1e30), -6),
])
def test_fp8_argument_errors(lib, kw, code):
    assert _call_fp8(**kw) == code


def _call_fp8_ex(mask=16, mtype=1, sb=0, sh=0, sq=8, smax=0, ssum=0, dq=1.0, dk=1.0, dv=1.0,
                 **kw):
    a = dict(GOOD)
    a.update(kw)
    return fa.fa_fwd_fp8_ex(a["q"], a["k"], a["v"], a["out"], a["lse"], smax, ssum, mask, mtype,
                            sb, sh, sq, a["B"], a["H"], a["H_kv"], a["L_q"], a["L_k"], a["D"],
                            a["scale"], dq, dk, dv, a["causal"], a["wl"], a["wr"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(mtype=4), -6), (dict(sq=-1), -6), (dict(mask=0), -1), (dict(smax=16, ssum=0), -1),
    (dict(smax=18, ssum=16), -5), (dict(D=48), -3), (dict(D=16), -3), (dict(dk=-2.0), -6),
    (dict(q=8), -5),
])
def test_fp8_ex_argument_errors(lib, kw, code):
    assert _call_fp8_ex(**kw) == code


def test_16bit_entries_refuse_the_fp8_code(lib):
    # dtype 2 is internal to fa_fwd_fp8 / fa_fwd_fp8_splitkv
    assert _call(dtype=2) == -4
    assert _call_split(dtype=2) == -4
    assert _call_static(dtype=2) == -4


def _call_fp8_split(dq=1.0, dk=1.0, dv=1.0, n_splits=2, ws=256, ws_bytes=None, **kw):
    a = dict(GOOD)
    a.update(kw)
    if ws_bytes is None:
        ws_bytes = fa.fa_splitkv_workspace_bytes(a["B"], a["H"], a["L_q"], a["D"],
                                                 max(1, min(64, n_splits)))
    return fa.fa_fwd_fp8_splitkv(a["q"], a["k"], a["v"], a["out"], a["lse"], a["B"], a["H"],
                                 a["H_kv"], a["L_q"], a["L_k"], a["D"], a["scale"], dq, dk, dv,
                                 a["causal"], a["wl"], a["wr"], n_splits, ws, ws_bytes, None)


@pytest.mark.parametrize("kw,code", [
    (dict(n_splits=0), -6), (dict(n_splits=65), -6), (dict(ws=0), -1), (dict(ws=128), -5),
    (dict(ws_bytes=100), -9), (dict(D=16), -3), (dict(D=48), -3), (dict(q=0), -1),
    (dict(q=8), -5), (dict(dq=-1.0), -6), (dict(dv=float("nan")), -6), (dict(scale=-1.0), -6),
])
def test_fp8_splitkv_argument_errors(lib, kw, code):
    assert _call_fp8_split(**kw) == code


def test_fp8_splitkv_empty_queries_is_a_no_op(lib):
    assert _call_fp8_split(L_q=0, ws=0) == 0


# ------------------------------------------------------------ host-buffer entry
def _call_host(ws=256, ws_bytes=1 << 40, n_chunks=4, **kw):
    a = dict(GOOD)
    a.update(kw)
    return fa.fa_fwd_host(a["q"], a["k"], a["v"], a["out"], a["lse"], a["B"], a["H"], a["H_kv"],
                          a["L_q"], a["L_k"], a["D"], a["scale"], a["causal"], a["wl"], a["wr"],
                          a["dtype"], ws, ws_bytes, n_chunks, None)


def test_host_workspace_bytes(lib):
    # two slots of one chunk: ceil(B*H_kv / n_chunks) K/V heads and their
    # query heads; q, k, v, out in the element type, lse fp32, 256-aligned parts
    up = lambda x: (x + 255) // 256 * 256
    B, H, H_kv, L_q, L_k, D, n = 2, 8, 2, 100, 300, 64, 3
    per = -(-(B * H_kv) // n)
    slot = 2 * up(per * 4 * L_q * D * 2) + 2 * up(per * L_k * D * 2) + up(per * 4 * L_q * 4)
    assert fa.fa_fwd_host_workspace_bytes(B, H, H_kv, L_q, L_k, D, n) == 2 * slot
    assert fa.fa_fwd_host_workspace_bytes(B, H, H_kv, L_q, L_k, 40, n) == 0
    assert fa.fa_fwd_host_workspace_bytes(B, H, 3, L_q, L_k, D, n) == 0
    assert fa.fa_fwd_host_workspace_bytes(B, H, H_kv, L_q, L_k, D, 0) == 0


@pytest.mark.parametrize("kw,code", [
    (dict(n_chunks=0), -6), (dict(ws=0), -1), (dict(ws=128), -5), (dict(ws_bytes=100), -9),
    (dict(D=40), -3), (dict(dtype=2), -4), (dict(q=0), -1), (dict(H=4, H_kv=3), -2),
    (dict(scale=float("nan")), -6),
])
def test_host_argument_errors(lib, kw, code):
    assert _call_host(**kw) == code


def _call_bwd_ex(mask=16, mtype=1, sb=0, sh=0, sq=8, **kw):
    a = dict(BWD_GOOD)
    a.update(kw)
    return fa.fa_bwd_ex(a["q"], a["k"], a["v"], a["out"], a["dout"], a["lse"], a["dq"], a["dk"],
                        a["dv"], mask, mtype, sb, sh, sq, a["B"], a["H"], a["H_kv"], a["L_q"],
                        a["L_k"], a["D"], a["scale"], a["causal"], a["wl"], a["wr"], a["dtype"],
                        a["ws"], a["ws_bytes"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(mtype=4), -6), (dict(sq=-1), -6), (dict(mask=0), -1), (dict(D=40), -3),
    (dict(q=0), -1), (dict(ws_bytes=10), -9),
])
def test_bwd_ex_argument_errors(lib, kw, code):
    assert _call_bwd_ex(**kw) == code


def test_watchdog_selftest_rejects_null(lib):
    # returns before any CUDA call
    assert fa.fa_selftest_wait_timeout(None, None) == -1


# ------------------------------------------------------------ watchdog test library
def test_product_library_has_no_test_hook(lib):
    # the withheld-copy hook exists only in lib/libfa_testhooks.so
    assert not hasattr(lib, "fa_test_set_withhold")


def test_test_library_exports_the_hook():
    import ctypes
    from exact_attention_113_b200 import build as fa_build
    if not os.path.exists(fa_build.TESTHOOKS_PATH):
        pytest.skip("watchdog test library not built (build(testhooks=True))")
    t = ctypes.CDLL(fa_build.TESTHOOKS_PATH)
    assert hasattr(t, "fa_test_set_withhold") and hasattr(t, "fa_fwd")


def test_register_check_follows_the_backward_launch_shape():
    # the build refuses instances whose register count differs from the
    # launch allocation their setmaxnreg split adds up to: 168 for the
    # forward, 80 for the D <= 64 backward (768 threads), 128 above (512)
    from exact_attention_113_b200 import build as fa_build

    def log(entries):
        return "\n".join(f"ptxas info    : Compiling entry function '{name}' for 'sm_100a'\n"
                         f"ptxas info    : Used {regs} registers, used 3 barriers"
                         for name, regs in entries)
    fwd = ("_ZN2fa13fa_fwd_kernelILi128ELi0ELb0ELb0EEEvNS_9FwdParamsE", 168)
    good = [fwd, ("_ZN2fa13fa_bwd_kernelILi64ELi0ELb0EEEvNS_9BwdParamsE", 80),
            ("_ZN2fa13fa_bwd_kernelILi16ELi1ELb1EEEvNS_9BwdParamsE", 80),
            ("_ZN2fa13fa_bwd_kernelILi128ELi0ELb0EEEvNS_9BwdParamsE", 128),
            ("_ZN2fa13fa_bwd_kernelILi80ELi1ELb0EEEvNS_9BwdParamsE", 128)]
    counts = fa_build.check_register_counts(log(good))
    assert len(counts) == len(good)
    for wrong in (("_ZN2fa13fa_bwd_kernelILi64ELi0ELb0EEEvNS_9BwdParamsE", 128),
                  ("_ZN2fa13fa_bwd_kernelILi96ELi0ELb0EEEvNS_9BwdParamsE", 80),
                  ("_ZN2fa13fa_fwd_kernelILi64ELi0ELb0ELb0EEEvNS_9FwdParamsE", 160)):
        with pytest.raises(RuntimeError, match="launch allocation"):
            fa_build.check_register_counts(log(good + [wrong]))
