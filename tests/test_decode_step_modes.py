"""Ways to run a decode step without paying a launch per kernel: the CUDA
graph pool (one captured step per static shape, the nearest replayed) and the
persistent decode kernel (resident, commanded from the host through mapped
host memory). Both compute exactly what attn_decode_paged computes for the
same buffers, batch and length bound: every step is checked against the fp64
oracle and, bit for bit, against a direct call with the same plan."""
import numpy as np
import pytest

from attention_tiled_exact_b200 import workloads as wl
from oracle import attention_ref as ref
from tests.helpers import assert_lse_close, assert_o_close, to_dev_bf16, to_dev_i32, to_f64

pytestmark = pytest.mark.gpu

MAX_BATCH, HQ, HKV, D = 12, 16, 4, 128
CAP = 3072  # tokens a table row holds


def _pool_inputs(seed):
    """One paged pool holding MAX_BATCH sequences of CAP tokens each, and q."""
    lens = np.full(MAX_BATCH, CAP, dtype=np.int32)
    d = wl.make_decode(wl.DecodeConfig("modes", MAX_BATCH, HQ, HKV, D, 1, 1, seed), kv_lens=lens)
    return d


def _steps(seed, n):
    """n steps: (batch, per-row lengths) with rows past batch at length 0."""
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(n):
        batch = int(rng.integers(1, MAX_BATCH + 1))
        lens = np.zeros(MAX_BATCH, dtype=np.int32)
        lens[:batch] = rng.integers(1, CAP + 1, batch)
        if batch > 2:
            lens[1] = 0  # an empty sequence inside the batch
        out.append((batch, lens))
    return out


def _direct(lib, q, kc, vc, bt, lens, scale, batch, max_len):
    """attn_decode_paged over the first `batch` rows with this length bound."""
    import torch
    o, lse = lib.decode_paged(q[:batch].contiguous(), kc, vc, bt[:batch].contiguous(), lens[:batch].contiguous(),
                              scale, max_seq_len=max_len, out_dtype=torch.float32)
    torch.cuda.synchronize()
    return to_f64(o), to_f64(lse)


def test_graph_pool_replays_match_direct_calls_and_the_oracle(lib):
    import torch
    d = _pool_inputs(61)
    dev = torch.device("cuda")
    q = to_dev_bf16(d["q"])
    kc, vc = to_dev_bf16(d["k_pool"]), to_dev_bf16(d["v_pool"])
    bt = to_dev_i32(d["block_table"])
    lens_s = torch.zeros(MAX_BATCH, dtype=torch.int32, device=dev)
    out = torch.zeros((MAX_BATCH, HQ, D), dtype=torch.float32, device=dev)
    lse = torch.zeros((MAX_BATCH, HQ), dtype=torch.float32, device=dev)
    pool = lib.DecodeGraphPool(q, kc, vc, bt, lens_s, out, lse, [2, 5, 12], [1024, 2048, CAP], d["scale"])
    try:
        for it, (batch, lens) in enumerate(_steps(62, 6)):
            lens_s.copy_(torch.from_numpy(lens))
            max_len = int(lens.max())
            bb, bl = pool.replay(batch, max_len)
            torch.cuda.synchronize()
            assert bb >= batch and bl >= max_len
            o, l = to_f64(out), to_f64(lse)
            O_ref, L_ref = ref.ref_decode_paged(d["q"][:batch], d["k_pool"], d["v_pool"], d["block_table"][:batch],
                                                lens[:batch], d["scale"])
            assert_o_close(o[:batch], O_ref, False, f"graph step {it}")
            assert_lse_close(l[:batch], L_ref, f"graph step {it}")
            assert (o[batch:bb] == 0).all() and np.isneginf(l[batch:bb]).all(), "padding rows"
            o2, l2 = _direct(lib, q, kc, vc, bt, lens_s, d["scale"], bb, bl)
            assert np.array_equal(o[:bb], o2) and np.array_equal(l[:bb], l2), f"graph step {it}: not bit-exact"
        with pytest.raises(lib.AttnError):
            pool.replay(MAX_BATCH + 1, 100)  # no bucket holds it
        with pytest.raises(lib.AttnError):
            pool.replay(1, CAP + 1)
    finally:
        pool.close()


def test_graph_pool_rejects_buckets_past_the_buffers(lib):
    import torch
    d = _pool_inputs(63)
    q = to_dev_bf16(d["q"])
    kc = to_dev_bf16(d["k_pool"])
    bt = to_dev_i32(d["block_table"])
    lens = torch.zeros(MAX_BATCH, dtype=torch.int32, device="cuda")
    out = torch.zeros((MAX_BATCH, HQ, D), dtype=torch.float32, device="cuda")
    for bad_b, bad_l in (([4, MAX_BATCH + 1], [1024]), ([4, 4], [1024]), ([4], [])):
        with pytest.raises(lib.AttnError):
            lib.DecodeGraphPool(q, kc, kc, bt, lens, out, None, bad_b, bad_l, d["scale"])


def _persistent_case(lib, seed, fp8=False):
    """Static buffers, steps, and each step's direct-call result (computed first:
    while the persistent kernel runs it holds the SMs)."""
    import torch
    d = _pool_inputs(seed)
    if fp8:
        for name in ("k", "v"):
            d[name + "_pool"], d[name + "_scale"] = wl.bf16_pool_to_e4m3(d[name + "_pool"])
        kc, vc = torch.from_numpy(d["k_pool"]).cuda(), torch.from_numpy(d["v_pool"]).cuda()
    else:
        kc, vc = to_dev_bf16(d["k_pool"]), to_dev_bf16(d["v_pool"])
    steps = _steps(seed + 1, 5)
    q_all = [wl.normal_bf16(seed + 10 + i, (MAX_BATCH, HQ, D)) for i in range(len(steps))]
    bt = to_dev_i32(d["block_table"])
    direct = []
    for (batch, lens), qb in zip(steps, q_all):
        o, l = lib.decode_paged(to_dev_bf16(qb[:batch]), kc, vc, bt[:batch].contiguous(), to_dev_i32(lens[:batch]),
                                d["scale"], max_seq_len=int(lens.max()), out_dtype=torch.float32,
                                k_scale=d.get("k_scale"), v_scale=d.get("v_scale"))
        torch.cuda.synchronize()
        direct.append((to_f64(o), to_f64(l)))
    return d, kc, vc, bt, steps, q_all, direct


@pytest.mark.parametrize("fp8", [False, True], ids=["bf16_cache", "fp8_cache"])
def test_persistent_decode_steps_match_direct_calls_and_the_oracle(lib, fp8):
    import torch
    d, kc, vc, bt, steps, q_all, direct = _persistent_case(lib, 71 + fp8, fp8)
    q_s = torch.zeros((MAX_BATCH, HQ, D), dtype=torch.bfloat16, device="cuda")
    lens_s = torch.zeros(MAX_BATCH, dtype=torch.int32, device="cuda")
    out = torch.zeros((MAX_BATCH, HQ, D), dtype=torch.float32, device="cuda")
    lse = torch.zeros((MAX_BATCH, HQ), dtype=torch.float32, device="cuda")
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    copies = torch.cuda.Stream()
    pd = lib.PersistentDecode(q_s, kc, vc, bt, lens_s, out, lse, d["scale"], error_flags=flags,
                              k_scale=d.get("k_scale"), v_scale=d.get("v_scale"))
    got = []
    try:
        assert pd.status == 0
        for (batch, lens), qb in zip(steps, q_all):
            with torch.cuda.stream(copies):  # copy engines only: the kernel holds the SMs
                q_s.copy_(torch.from_numpy(qb.view(np.int16)).view(torch.bfloat16).pin_memory(), non_blocking=True)
                lens_s.copy_(torch.from_numpy(lens).pin_memory(), non_blocking=True)
            copies.synchronize()
            pd.step(batch, int(lens.max()))
            with torch.cuda.stream(copies):
                o_h, l_h = out.to("cpu", non_blocking=True), lse.to("cpu", non_blocking=True)
            copies.synchronize()
            got.append((o_h.double().numpy()[:batch], l_h.double().numpy()[:batch]))
        assert pd.running
    finally:
        pd.stop()
    assert not pd.running and pd.status == 0
    assert lib.sync_error_flags(flags) == (lib.ATTN_OK, 0)
    for it, ((batch, lens), qb, (o, l), (o2, l2)) in enumerate(zip(steps, q_all, got, direct)):
        assert np.array_equal(o, o2) and np.array_equal(l, l2), f"step {it}: not bit-exact with a direct call"
        if fp8:
            O_ref, L_ref = ref.ref_decode_paged_fp8(qb[:batch], d["k_pool"], d["v_pool"], d["k_scale"], d["v_scale"],
                                                    d["block_table"][:batch], lens[:batch], d["scale"])
        else:
            O_ref, L_ref = ref.ref_decode_paged(qb[:batch], d["k_pool"], d["v_pool"], d["block_table"][:batch],
                                                lens[:batch], d["scale"])
        assert_o_close(o, O_ref, False, f"persistent step {it}")
        assert_lse_close(l, L_ref, f"persistent step {it}")


def test_persistent_decode_exits_when_idle_and_reports_it(lib):
    """With no command for its idle bound (here about a millisecond) the kernel
    exits by itself and reports ATTN_FAULT_TIMEOUT; the context stays usable."""
    import torch
    d = _pool_inputs(81)
    q_s = to_dev_bf16(d["q"])
    kc, vc = to_dev_bf16(d["k_pool"]), to_dev_bf16(d["v_pool"])
    bt = to_dev_i32(d["block_table"])
    lens_s = torch.full((MAX_BATCH,), 100, dtype=torch.int32, device="cuda")
    out = torch.zeros((MAX_BATCH, HQ, D), dtype=torch.float32, device="cuda")
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    pd = lib.PersistentDecode(q_s, kc, vc, bt, lens_s, out, None, d["scale"], idle_cycles=2_000_000,
                              error_flags=flags)
    pd.stream.synchronize()  # returns once the kernel gave up waiting
    assert not pd.running and pd.status & lib.ATTN_FAULT_TIMEOUT
    assert lib.sync_error_flags(flags)[0] == lib.ATTN_ERR_TIMEOUT
    with pytest.raises(lib.AttnError) as e:
        pd.wait(1, timeout_s=0.5)
    assert e.value.status == lib.ATTN_ERR_TIMEOUT
    o, _ = _direct(lib, q_s, kc, vc, bt, lens_s, d["scale"], MAX_BATCH, 100)  # a normal call still works
    O_ref, _ = ref.ref_decode_paged(d["q"], d["k_pool"], d["v_pool"], d["block_table"],
                                    np.full(MAX_BATCH, 100, dtype=np.int32), d["scale"])
    assert_o_close(o, O_ref, False, "decode after the persistent kernel exited")
