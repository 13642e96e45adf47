"""Pins of the oracle's fp8 (e4m3) input path (CPU only).

  - every one of the 256 e4m3 codes decodes to torch.float8_e4m3fn's value
    (library conversion, independent of the C decoder);
  - closed points of the format: 448, the smallest subnormal 2^-9, -0, NaN;
  - attention on e4m3 codes equals attention on the same values given as
    fp16 codes (every e4m3 value is exact in fp16), so the fp8 path inherits
    the forward's pins."""
from __future__ import annotations

import numpy as np
import torch

from exact_attention_113_b200.inputs import F16, Workload, make_qkv

E4M3 = 2


def test_decode_every_code_matches_torch(orc):
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).double().numpy()
    got = orc.decode(codes.numpy(), E4M3)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_decode_closed_points(orc):
    assert orc.e4m3_to_f64(0x7E) == 448.0
    assert orc.e4m3_to_f64(0x01) == 2.0 ** -9
    assert orc.e4m3_to_f64(0x08) == 2.0 ** -6          # smallest normal
    assert orc.e4m3_to_f64(0x38) == 1.0
    v = orc.e4m3_to_f64(0x80)
    assert v == 0.0 and np.signbit(v)
    assert np.isnan(orc.e4m3_to_f64(0x7F)) and np.isnan(orc.e4m3_to_f64(0xFF))


def test_attention_on_e4m3_equals_fp16_of_same_values(orc):
    w = Workload(name="f8", B=1, H=2, H_kv=1, L_q=33, L_k=70, D=32, dtype=F16, seed=9100)
    q, k, v = make_qkv(w)
    f8 = [t.float().to(torch.float8_e4m3fn) for t in (q, k, v)]
    codes = [t.view(torch.uint8).numpy() for t in f8]
    f16 = [t.to(torch.float16).view(torch.int16).numpy().view(np.uint16) for t in f8]
    a = orc.attention_rows(*codes, E4M3, 0.2, True)
    b = orc.attention_rows(*f16, F16, 0.2, True)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
