"""Host-side logic of bench.py (CPU only): FLOP accounting against closed
forms, and the cross-rank reduction with two gloo ranks."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import bench
from exact_attention_113_b200 import inputs as W


def _w(**kw):
    base = dict(name="x", B=2, H=3, H_kv=3, L_q=100, L_k=100, D=64)
    base.update(kw)
    return W.Workload(**base)


def test_visible_pairs_closed_forms():
    L = 100
    assert bench.visible_pairs_per_head(_w()) == L * L
    assert bench.visible_pairs_per_head(_w(causal=True)) == L * (L + 1) // 2
    # causal with left window wl: row i sees min(i, wl) + 1 keys
    wl = 7
    expect = sum(min(i, wl) + 1 for i in range(L))
    assert bench.visible_pairs_per_head(_w(causal=True, window_left=wl)) == expect
    # L_q > L_k, causal: rows >= L_k see all L_k keys
    w = _w(L_q=150, L_k=100, causal=True)
    assert bench.visible_pairs_per_head(w) == 100 * 101 // 2 + 50 * 100


def test_metric_and_algorithmic_flops():
    w = _w()
    assert bench.metric_flops(w) == 4 * 2 * 3 * 100 * 100 * 64
    assert bench.algorithmic_flops(w) == bench.metric_flops(w)
    wc = _w(causal=True)
    assert bench.metric_flops(wc) == bench.metric_flops(w) / 2
    assert bench.algorithmic_flops(wc) == 4 * 64 * 2 * 3 * (100 * 101 // 2)
    rows = np.arange(2 * 3 * 100)
    assert bench.row_flops(wc, rows) == bench.algorithmic_flops(wc)


def test_gqa_window_pair_count_of_the_named_workload():
    w = W.GQA_WINDOW      # causal, wl=4096: 4097 keys per row once i >= 4096
    L, wl = w.L_q, w.window_left
    expect = sum(min(i, wl) + 1 for i in range(L))
    assert bench.visible_pairs_per_head(w) == expect == 58734592


def test_whole_job_value():
    assert bench.whole_job_value(1e12, 4, 10, 2.0) == pytest.approx(20.0)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        local_time = 1.0 + rank          # rank 1 is the slowest
        m = bench.max_over_ranks(local_time, world)
        v = bench.whole_job_value(3e12, world, 5, m)
        q.put((rank, m, v))
    finally:
        dist.destroy_process_group()


def test_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, m, v in got:
        assert m == 2.0                        # the max over ranks
        assert v == pytest.approx(3e12 * 2 * 5 / 2.0 / 1e12)


def test_roofline_bound_by_workload():
    # the long-sequence forward is tensor bound, one-query decoding HBM bound
    assert bench.roofline_bound(W.ROOFLINE, 1640.0, 6461.8) == "tensor"
    for w in W.DECODE:
        assert bench.roofline_bound(w, 1640.0, 6461.8) == "hbm", w.name
    # decoding moves the K/V cache once: 2 tensors * B*H_kv*L_k*D * 2 bytes
    w = W.DECODE[0]
    kv = 2 * w.B * w.H_kv * w.L_k * w.D * 2
    assert kv < bench.min_hbm_bytes(w) < kv * 1.01
    # an fp8 cache is read at one byte per element; the bf16 output stays 2
    assert kv // 2 < bench.min_hbm_bytes(w, 1) < kv // 2 * 1.01
    q = w.B * w.H * w.L_q * w.D
    assert bench.min_hbm_bytes(w) - bench.min_hbm_bytes(w, 1) == q + kv // 2


def test_resolve_splits():
    w = W.DECODE[0]
    assert bench.resolve_splits("0", w) == 0
    assert bench.resolve_splits("5", w) == 5
    assert 1 <= bench.resolve_splits("auto", w) <= 64


def test_exp_roof_closed_form():
    # B4 H48 L8192 non-causal: 4*48*8192^2 exponentials; at 1 GHz over 1 ms
    w = W.ROOFLINE
    r = bench.exp_roof(w, 1e-3, 1000.0)
    exps = 4 * 48 * 8192 * 8192
    assert r["exps_per_launch"] == exps
    assert abs(r["achieved_per_clk_per_sm"] - round(exps / (1e-3 * 1e9 * 148), 3)) < 1e-9
    assert abs(r["frac"] - round(exps / (1e-3 * 1e9 * 148) / 16.0, 4)) < 1e-9


def test_code_hash_ignores_comments_only():
    a = "int f(int x) {  // doubles\n  return 2 * x;\n}\n"
    b = "// a new header line\nint f(int x) {\n\n  return 2 * x;   // same code\n}\n"
    c = "int f(int x) {\n  return 3 * x;\n}\n"
    assert bench.code_hash([a]) == bench.code_hash([b])
    assert bench.code_hash([a]) != bench.code_hash([c])
    assert len(bench.kernel_source_hash()) == 16
