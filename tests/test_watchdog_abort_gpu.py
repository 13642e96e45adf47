"""The attention kernel's own abort path on the GPU, without a fault.

The watchdog test library (lib/libfa_testhooks.so, include/fa_test_hooks.h:
the same sources as libfa.so built with FA_TEST_HOOKS and a 10 ms device wait
limit) can make the forward kernel's K producer of CTA 0 withhold the copy of
one key block.  Nothing ever completes that block's barrier phase, so the MMA
warp's bounded wait runs out: it raises the CTA's abort flag and the device
status word, every other role leaves its loop at its next wait or at the flag,
the producers let their copies in flight land, the MMA warp waits for its
issued MMAs and TMEM is freed (the review of every wait and barrier on this
path is in the design notes).  The test checks that the launch ends within
the limit's order of magnitude, that fa_get_device_status reports
FA_ERR_TIMEOUT once, and that the next, normal launch in the same context
matches the oracle.  The schedules that end differently are covered: the
two-tile ping-pong (more query tiles than SMs), the one-tile dual softmax
with its cross-warpgroup merge barrier, and the balanced pair whose receiver
gives up while its sender hands over its rows."""
from __future__ import annotations

import ctypes
import os
import time

import numpy as np
import pytest
import torch

from exact_attention_113_b200 import build as fa_build
from exact_attention_113_b200.inputs import F16, Workload, make_qkv
from tests.parity import compare, reference

pytestmark = pytest.mark.gpu
FA_OK, FA_ERR_TIMEOUT = 0, -8


@pytest.fixture(scope="module")
def hooks():
    if not os.path.exists(fa_build.TESTHOOKS_PATH) or fa_build.is_stale(fa_build.TESTHOOKS_PATH):
        fa_build.build(testhooks=True)
    lib = ctypes.CDLL(fa_build.TESTHOOKS_PATH)
    vp, i = ctypes.c_void_p, ctypes.c_int
    lib.fa_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, ctypes.c_float, i, i, i, i, vp]
    lib.fa_fwd.restype = i
    lib.fa_get_device_status.argtypes = [vp]
    lib.fa_get_device_status.restype = i
    lib.fa_test_set_withhold.argtypes = [i]
    lib.fa_test_set_withhold.restype = i
    yield lib
    lib.fa_test_set_withhold(-1)


def _launch(lib, w, q, k, v, out, lse):
    stream = torch.cuda.current_stream().cuda_stream
    st = lib.fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                    w.B, w.H, w.H_kv, w.L_q, w.L_k, w.D, w.softmax_scale, int(w.causal),
                    w.window_left, w.window_right, F16, stream)
    assert st == FA_OK
    return stream


CASES = [
    # more 128-row query tiles than SMs: two tiles per CTA (ping-pong)
    Workload(name="abort_pingpong", B=2, H=40, H_kv=40, L_q=1024, L_k=1024, D=128, dtype=F16,
             seed=6001),
    # a few tiles: one tile per CTA, keys split between two softmax warpgroups
    Workload(name="abort_dual", B=1, H=2, H_kv=2, L_q=1024, L_k=1024, D=64, dtype=F16,
             seed=6002),
    # causal, a few tiles: the balanced schedule; CTA 0 is the receiver of the
    # heaviest tile's pair (key blocks 0 .. 4), its sender hands over blocks
    # 5 .. 7 while the receiver's wait runs out
    Workload(name="abort_balanced", B=1, H=2, H_kv=2, L_q=1024, L_k=1024, D=64, dtype=F16,
             causal=True, seed=6003),
]


# block 2 is requested by the K producer warp; block 0 (the CTA's first) by
# thread 0 during set-up, before the block-wide barrier
@pytest.mark.parametrize("withheld", [2, 0])
@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_withheld_copy_ends_the_launch_with_a_timeout(hooks, w, withheld):
    q, k, v = (t.cuda() for t in make_qkv(w))
    out = torch.full_like(q, float("nan"))
    lse = torch.full((w.B, w.H, w.L_q), float("nan"), device="cuda")
    assert hooks.fa_get_device_status(None) == FA_OK       # nothing pending
    # CTA 0 covers the first query tile(s) of head 0: key blocks 0 .. 7
    assert hooks.fa_test_set_withhold(withheld) == FA_OK
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    stream = _launch(hooks, w, q, k, v, out, lse)
    assert hooks.fa_get_device_status(stream) == FA_ERR_TIMEOUT
    elapsed = time.perf_counter() - t0
    assert elapsed < 2.0, f"the aborted launch took {elapsed:.2f} s"
    assert hooks.fa_get_device_status(stream) == FA_OK     # read once, then cleared

    # the same context runs a normal launch that matches the oracle
    assert hooks.fa_test_set_withhold(-1) == FA_OK
    out.fill_(float("nan"))
    lse.fill_(float("nan"))
    stream = _launch(hooks, w, q, k, v, out, lse)
    assert hooks.fa_get_device_status(stream) == FA_OK
    ref, ref_lse, pr, heads = reference(w, *make_qkv(w))
    compare(out.float().cpu().numpy().reshape(-1, w.D), lse.cpu().numpy().reshape(-1), ref,
            ref_lse, w.dtype, w.name, pr, False, heads)
