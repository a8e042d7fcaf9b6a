"""CUDA-graph capture of the hot path: a decode step (split kernel + combine,
caller-owned workspace), a prefill call and a backward call (three launches,
the second and third as programmatic dependents of the one before) are
captured once on static buffers and replayed with new inputs written into
those buffers.

The split plan is fixed at capture from the host-side length bound, and the
kernels read lengths and block tables from device memory on every replay, so
a replay with new contents must equal the oracle and, bit for bit, a direct
(uncaptured) call on the same inputs.
"""
import numpy as np
import pytest

from attention_tiled_exact_b200 import workloads as wl
from oracle import attention_ref as ref
from tests.helpers import assert_lse_close, assert_o_close, to_dev_bf16, to_dev_i32, to_f64

pytestmark = pytest.mark.gpu

B, HQ, HKV, D = 6, 8, 2, 128
MAX_LEN = 3000


def _step_inputs(step):
    rng = np.random.default_rng(500 + step)
    lens = rng.integers(0, MAX_LEN + 1, B).astype(np.int32)
    lens[step % B] = MAX_LEN
    cfg = wl.DecodeConfig("g", B, HQ, HKV, D, 1, 1, 600 + step)
    return wl.make_decode(cfg, kv_lens=lens)


def test_decode_step_graph_replay(lib):
    import torch
    max_blocks = (MAX_LEN + 15) // 16
    nb_max = B * max_blocks + 64
    q_s = torch.empty((B, HQ, D), dtype=torch.bfloat16, device="cuda")
    k_s = torch.zeros((nb_max, HKV, 16, D), dtype=torch.bfloat16, device="cuda")
    v_s = torch.zeros_like(k_s)
    bt_s = torch.zeros((B, max_blocks), dtype=torch.int32, device="cuda")
    sl_s = torch.zeros(B, dtype=torch.int32, device="cuda")
    o_s = torch.empty((B, HQ, D), dtype=torch.float32, device="cuda")
    l_s = torch.empty((B, HQ), dtype=torch.float32, device="cuda")

    def load(d):
        nb = d["k_pool"].shape[0]
        assert nb <= nb_max and d["block_table"].shape[1] <= max_blocks
        q_s.copy_(to_dev_bf16(d["q"]))
        k_s[:nb].copy_(to_dev_bf16(d["k_pool"]))
        v_s[:nb].copy_(to_dev_bf16(d["v_pool"]))
        bt_s.zero_()
        bt_s[:, :d["block_table"].shape[1]].copy_(to_dev_i32(d["block_table"]))
        sl_s.copy_(to_dev_i32(d["kv_lens"]))

    d0 = _step_inputs(0)
    scale = d0["scale"]
    ws = torch.empty(max(1, lib.decode_workspace_bytes(q_s, k_s, v_s, bt_s, sl_s, max_seq_len=MAX_LEN)),
                     dtype=torch.uint8, device="cuda")

    def step():
        lib.decode_paged(q_s, k_s, v_s, bt_s, sl_s, scale, max_seq_len=MAX_LEN, out=o_s, lse=l_s, workspace=ws)

    load(d0)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()  # first call outside capture: one-time kernel attribute setup
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for s in range(1, 4):
        d = _step_inputs(s)
        load(d)
        g.replay()
        torch.cuda.synchronize()
        o_graph, l_graph = to_f64(o_s), to_f64(l_s)
        O_ref, L_ref = ref.ref_decode_paged(d["q"], d["k_pool"], d["v_pool"], d["block_table"], d["kv_lens"], scale)
        assert_o_close(o_graph, O_ref, False, f"graph step {s}")
        assert_lse_close(l_graph, L_ref, f"graph step {s}")
        step()
        torch.cuda.synchronize()
        assert np.array_equal(to_f64(o_s), o_graph) and np.array_equal(to_f64(l_s), l_graph)


def test_prefill_graph_replay(lib):
    import torch
    cfg = wl.PrefillConfig("g", 2, 8, 2, 384, 384, 128, True, 700)
    q_s = torch.empty((2, 8, 384, 128), dtype=torch.bfloat16, device="cuda")
    k_s = torch.empty((2, 2, 384, 128), dtype=torch.bfloat16, device="cuda")
    v_s = torch.empty_like(k_s)
    o_s = torch.empty((2, 8, 384, 128), dtype=torch.float32, device="cuda")
    l_s = torch.empty((2, 8, 384), dtype=torch.float32, device="cuda")

    def call():
        lib.prefill(q_s, k_s, v_s, cfg.scale, True, out=o_s, lse=l_s)

    def load(seed):
        d = wl.make_prefill(wl.PrefillConfig("g", 2, 8, 2, 384, 384, 128, True, seed))
        q_s.copy_(to_dev_bf16(d["q"]))
        k_s.copy_(to_dev_bf16(d["k"]))
        v_s.copy_(to_dev_bf16(d["v"]))
        return d

    load(cfg.seed)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        call()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call()
    for seed in (701, 702):
        d = load(seed)
        g.replay()
        torch.cuda.synchronize()
        o_graph, l_graph = to_f64(o_s), to_f64(l_s)
        O_ref, L_ref = ref.ref_attention(d["q"], d["k"], d["v"], cfg.scale, True)
        assert_o_close(o_graph, O_ref, False, f"prefill graph {seed}")
        assert_lse_close(l_graph, L_ref, f"prefill graph {seed}")
        call()
        torch.cuda.synchronize()
        assert np.array_equal(to_f64(o_s), o_graph) and np.array_equal(to_f64(l_s), l_graph)


def test_backward_graph_replay(lib):
    import torch
    B_, HQ_, HKV_, S, D_ = 2, 8, 2, 300, 128
    q_s = torch.empty((B_, HQ_, S, D_), dtype=torch.bfloat16, device="cuda")
    k_s = torch.empty((B_, HKV_, S, D_), dtype=torch.bfloat16, device="cuda")
    v_s = torch.empty_like(k_s)
    do_s = torch.empty_like(q_s)
    o_s = torch.empty((B_, HQ_, S, D_), dtype=torch.float32, device="cuda")
    l_s = torch.empty((B_, HQ_, S), dtype=torch.float32, device="cuda")
    grads = [torch.empty(t.shape, dtype=torch.float32, device="cuda") for t in (q_s, k_s, v_s)]
    scale = 1.0 / np.sqrt(D_)

    def load(seed):
        q = wl.normal_bf16(seed, q_s.shape, 40)
        k = wl.normal_bf16(seed, k_s.shape, 41)
        v = wl.normal_bf16(seed, v_s.shape, 42)
        do = wl.normal_bf16(seed, do_s.shape, 43)
        r = ref.ref_attention_backward(q, k, v, do, scale, True)
        for dst, src in ((q_s, q), (k_s, k), (v_s, v), (do_s, do)):
            dst.copy_(to_dev_bf16(src))
        o_s.copy_(torch.tensor(np.asarray(r["o"], dtype=np.float32)))
        l_s.copy_(torch.tensor(np.asarray(r["lse"], dtype=np.float32)))
        return r

    load(800)
    ws = torch.empty(64 << 20, dtype=torch.uint8, device="cuda")

    def call():
        lib.prefill_backward(q_s, k_s, v_s, o_s, l_s, do_s, scale, True, dq=grads[0], dk=grads[1], dv=grads[2],
                             workspace=ws)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        call()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call()
    for seed in (801, 802):
        r = load(seed)
        g.replay()
        torch.cuda.synchronize()
        got = [to_f64(t) for t in grads]
        for x, name in zip(got, ("dq", "dk", "dv")):
            peak = float(np.abs(r[name]).max())
            assert float(np.abs(x - r[name]).max()) <= 1e-2 * peak, (seed, name)
        call()
        torch.cuda.synchronize()
        assert all(np.array_equal(to_f64(t), x) for t, x in zip(grads, got))
