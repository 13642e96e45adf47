"""Seeded synthetic inputs and the named workloads.

This module is the only one that both the CUDA path's callers and the CPU
oracle's callers use.  It draws random numbers and names shapes; it holds none
of the attention arithmetic.

Recipe: a CPU ``torch.Generator`` seeded per workload draws fp32 standard
normals for Q, then K, then V (in that order, each [B, H or H_kv, L, D]);
they are multiplied by ``std`` and cast to fp16 or bf16 with round-to-nearest
-even (torch's cast).  The same bytes feed the GPU and the oracle.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch

F16, BF16 = 0, 1
TORCH_DTYPE = {F16: torch.float16, BF16: torch.bfloat16}
DTYPE_NAME = {F16: "fp16", BF16: "bf16"}


@dataclasses.dataclass(frozen=True)
class Workload:
    """One attention forward problem: shapes, mask, dtype, input recipe."""
    name: str
    B: int
    H: int
    H_kv: int
    L_q: int
    L_k: int
    D: int
    dtype: int = F16
    causal: bool = False
    window_left: int = -1
    window_right: int = -1
    scale: float | None = None      # None -> 1/sqrt(D)
    std: float = 1.0
    seed: int = 0

    @property
    def softmax_scale(self) -> float:
        return self.scale if self.scale is not None else 1.0 / math.sqrt(self.D)


def make_qkv(w: Workload, device="cpu"):
    """Q [B,H,L_q,D], K and V [B,H_kv,L_k,D] for workload ``w``."""
    g = torch.Generator(device="cpu").manual_seed(int(w.seed))
    dt = TORCH_DTYPE[w.dtype]
    out = []
    for shape in ((w.B, w.H, w.L_q, w.D), (w.B, w.H_kv, w.L_k, w.D),
                  (w.B, w.H_kv, w.L_k, w.D)):
        x = torch.randn(shape, generator=g, dtype=torch.float32)
        if w.std != 1.0:
            x.mul_(w.std)
        out.append(x.to(dt).to(device))
    return tuple(out)


def make_qkv_fp8(w: Workload, device="cpu"):
    """Q, K, V of workload ``w`` as fp8 E4M3 tensors: the same seeded normals
    as make_qkv, converted to float8_e4m3fn (round to nearest)."""
    g = torch.Generator(device="cpu").manual_seed(int(w.seed))
    out = []
    for shape in ((w.B, w.H, w.L_q, w.D), (w.B, w.H_kv, w.L_k, w.D),
                  (w.B, w.H_kv, w.L_k, w.D)):
        x = torch.randn(shape, generator=g, dtype=torch.float32)
        if w.std != 1.0:
            x.mul_(w.std)
        out.append(x.to(torch.float8_e4m3fn).to(device))
    return tuple(out)


def make_dout(w: Workload, device="cpu"):
    """The upstream gradient dO [B,H,L_q,D] for a backward of workload ``w``
    (seeded N(0, 1), its own stream: seed + 7919)."""
    g = torch.Generator(device="cpu").manual_seed(int(w.seed) + 7919)
    x = torch.randn((w.B, w.H, w.L_q, w.D), generator=g, dtype=torch.float32)
    return x.to(TORCH_DTYPE[w.dtype]).to(device)


def to_bits(t: torch.Tensor) -> np.ndarray:
    """A CPU copy of an fp16/bf16 tensor as uint16 bit patterns (fp8
    tensors: uint8 codes)."""
    t = t.detach().cpu().contiguous()
    if t.element_size() == 1:
        return t.view(torch.uint8).numpy()
    return t.view(torch.int16).numpy().view(np.uint16)


def sample_rows(w: Workload, per_head_random: int = 8, seed: int = 7) -> np.ndarray:
    """Deterministic row sample for large workloads, per (b, h): rows
    0, 1, 2, 127, 128, 129, L/2, L-1 (plus 4095, 4096, 4097, 8191 when a
    left window is set) and ``per_head_random`` seeded random rows.
    Returns flattened row ids (b*H + h)*L_q + i, sorted and unique."""
    L = w.L_q
    fixed = [0, 1, 2, 127, 128, 129, L // 2, L - 1]
    if w.window_left >= 0:
        fixed += [4095, 4096, 4097, 8191]
    fixed = [i for i in fixed if 0 <= i < L]
    rng = np.random.default_rng(seed)
    ids = []
    for bh in range(w.B * w.H):
        extra = rng.integers(0, L, size=per_head_random) if L > 0 else []
        for i in sorted(set(fixed) | set(int(x) for x in extra)):
            ids.append(bh * L + i)
    return np.array(sorted(set(ids)), dtype=np.int64)


def _c(name, **kw):
    return Workload(name=name, **kw)


# The named workloads.  Seeds follow 1000 + workload index + 10*variant;
# causal and non-causal variants of one shape share their inputs.
TINY = [
    _c("tiny_noncausal", B=1, H=2, H_kv=2, L_q=128, L_k=128, D=64, scale=1 / 8, seed=1000),
    _c("tiny_causal", B=1, H=2, H_kv=2, L_q=128, L_k=128, D=64, scale=1 / 8, causal=True, seed=1000),
]
GPT2 = _c("gpt2_causal", B=1, H=12, H_kv=12, L_q=1024, L_k=1024, D=64, scale=1 / 8,
          causal=True, seed=1001)
MEMTABLE = [
    _c("memtable_fp16", B=1, H=16, H_kv=16, L_q=2048, L_k=2048, D=128, dtype=F16, seed=1002),
    _c("memtable_bf16", B=1, H=16, H_kv=16, L_q=2048, L_k=2048, D=128, dtype=BF16, seed=1012),
]
SWEEP_L = (512, 1024, 2048, 4096, 8192, 16384)
SWEEP = [
    _c(f"sweep_d{D}_l{L}_{'causal' if c else 'noncausal'}", B=4, H=48, H_kv=48,
       L_q=L, L_k=L, D=D, causal=c, seed=1003 + 10 * (SWEEP_L.index(L) + 6 * (D == 16)))
    for D in (64, 16) for L in SWEEP_L for c in (True, False)
]
GQA_WINDOW = _c("gqa_window_l16384", B=2, H=32, H_kv=8, L_q=16384, L_k=16384, D=128,
                dtype=BF16, causal=True, window_left=4096, window_right=0, std=0.5,
                seed=1004)
ROOFLINE = _c("roofline_b4h48l8192d128", B=4, H=48, H_kv=48, L_q=8192, L_k=8192,
              D=128, dtype=F16, causal=False, seed=1014)

# a smaller case of the roofline kernel for detailed profiles (400 MB of
# inputs and outputs: larger than L2, a few hundred MB on the device)
PROFILE = _c("profile_b4h48l2048d128", B=4, H=48, H_kv=48, L_q=2048, L_k=2048, D=128,
             dtype=F16, causal=False, seed=1015)

# decoding: a few query rows against a long key/value cache (split-KV shapes).
# The speculative case puts its L_q queries at the end of the cache with the
# window (query i sees keys j <= i + L_k - L_q).
DECODE = [
    _c("decode_b8h32kv8_l1_k32768_d128", B=8, H=32, H_kv=8, L_q=1, L_k=32768, D=128,
       dtype=BF16, seed=1016),
    _c("decode_b4h32kv32_l1_k16384_d64", B=4, H=32, H_kv=32, L_q=1, L_k=16384, D=64,
       dtype=F16, seed=1017),
    _c("decode_b2h16kv4_l16_k65536_d128", B=2, H=16, H_kv=4, L_q=16, L_k=65536, D=128,
       dtype=BF16, window_right=65536 - 16, seed=1018),
]

ALL = {w.name: w for w in TINY + [GPT2] + MEMTABLE + SWEEP + DECODE +
       [GQA_WINDOW, ROOFLINE, PROFILE]}
