"""The balanced one-wave schedule against the fp64 oracle.

When a problem has no more 128-row query tiles than the GPU has SMs (one
tile per CTA, a single wave) and its tiles see uneven key ranges (causal
masks, windows), the host splits every tile whose key range has more than
half the longest range's blocks between the two CTAs of a cluster pair: the
first CTA takes the first half of the blocks, the second the rest and hands
its (m, l, O) to the first through distributed shared memory; the first
merges the two as two key slices and writes the row.  The other tiles run
alone, two to a cluster.  It applies when the longest range has 4 to 1024
key blocks, some tiles are not split (uneven ranges) and all pairs fit in
one wave (2 x items x pairs <= 148 SMs).

Every shape below satisfies that (the comment gives tiles per head, the
blocks of the longest range and the cluster pairs per head), covering fp16 /
bf16, D 16 / 64 / 128, GQA, unequal query and key lengths (top-left
aligned), windows, the mask input with the softmax statistics, no lse, an
odd number of light tiles (an idle CTA), and large-variance inputs that move
the running maximum differently in the two halves."""
from __future__ import annotations

import pytest

from exact_attention_113_b200.inputs import BF16, F16, Workload
from tests.parity import check_full
from tests.test_mask_gpu import _mask, check_masked

pytestmark = pytest.mark.gpu


def _w(name, **kw):
    base = dict(B=1, H=12, H_kv=12, L_q=1024, L_k=1024, D=64, dtype=F16, causal=True, seed=9900)
    base.update(kw)
    return Workload(name=name, **base)


def test_gpt2_shape_target_gate():
    # 8 tiles, 8 blocks; heavy 4..7 split, light (0, 1) (2, 3): 6 pairs x 12 heads = 144 CTAs
    check_full(_w("bal_gpt2"))


@pytest.mark.parametrize("D", [16, 64, 128])
@pytest.mark.parametrize("dtype", [F16, BF16])
def test_head_dims_and_types(D, dtype):
    # B1 H4 L2048: 16 tiles, 16 blocks; 8 split + 4 light pairs = 12 pairs x 4 = 96 CTAs
    check_full(_w(f"bal_d{D}", H=4, H_kv=4, L_q=2048, L_k=2048, D=D, dtype=dtype,
                  seed=9910 + D + dtype), derived=True)


def test_gqa():
    # H 8 over 2 K/V heads (L_q >= 128: not packed): 8 tiles per head, 6 pairs x 8 = 96 CTAs
    check_full(_w("bal_gqa", H=8, H_kv=2, seed=9920), derived=True)


def test_unequal_lengths_and_odd_light_count():
    # L_q 1000 (8 tiles, the last 104 rows), L_k 1800: tile t sees keys 0 .. 128 t + 127;
    # 8 blocks at most, heavy 4..7, light 0..3 -> 6 pairs; L_q 640: 5 tiles, heavy 3, 4,
    # light 0, 1, 2 -> 2 + 2 pairs, the second light pair has one idle CTA
    check_full(_w("bal_uneq", H=6, H_kv=6, L_q=1000, L_k=1800, seed=9930), derived=True)
    check_full(_w("bal_odd", H=6, H_kv=6, L_q=640, L_k=640, seed=9931), derived=True)


def test_window():
    # causal with window_left 700: ranges of up to 7 blocks (the first tiles fewer)
    check_full(_w("bal_win", H=6, H_kv=6, L_q=1536, L_k=1536, window_left=700, seed=9940),
               derived=True)


def test_without_lse_and_large_values():
    check_full(_w("bal_nolse", seed=9950), with_lse=False, derived=True)
    check_full(_w("bal_std4", std=4.0, seed=9951), derived=True)


@pytest.mark.parametrize("kind", ["bool", "f32"])
def test_mask_and_statistics(kind):
    w = _w(f"bal_mask_{kind}", H=6, H_kv=6, L_q=1024, L_k=1024, seed=9960)
    check_masked(w, _mask((w.B, w.H, w.L_q, w.L_k), kind, 9970))
