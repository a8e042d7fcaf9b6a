"""attn_decode_paged_noalloc: paged decode for callers that cannot allocate.

Such a caller (a host program that only holds pointers from another
component, or a loop that must not call cudaMalloc) passes inputs and outputs
only; the split partials live in a fixed array the library owns. This file is
collected last on purpose so that a run stopping at the first failure has
already run every other test. It must pass on its own in a fresh process as
well as after the other tests.
"""
import numpy as np
import pytest

from attention_tiled_exact_b200 import workloads as wl
from tests.helpers import assert_lse_close, assert_o_close, to_dev_bf16, to_dev_i32, to_f64


@pytest.mark.gpu
def test_noalloc_decode_matches_workspace_decode_twice(lib):
    import torch
    cfg = wl.DecodeConfig("noalloc", 6, 32, 8, 128, 1, 1, 21)
    lens = np.array([1, 17, 900, 4096, 5000, 12345], dtype=np.int32)
    d = wl.make_decode(cfg, kv_lens=lens)
    q, kc, vc = to_dev_bf16(d["q"]), to_dev_bf16(d["k_pool"]), to_dev_bf16(d["v_pool"])
    bt, sl = to_dev_i32(d["block_table"]), to_dev_i32(d["kv_lens"])
    max_len = int(lens.max())
    ref_o, ref_l = lib.decode_paged(q, kc, vc, bt, sl, cfg.scale, max_seq_len=max_len, num_splits=8,
                                    out_dtype=torch.float32)
    torch.cuda.synchronize()
    ref_o, ref_l = to_f64(ref_o), to_f64(ref_l)
    for call in range(2):  # the second call finds the first call's partials still in the array
        out = torch.full((cfg.batch, cfg.q_heads, 128), float("nan"), dtype=torch.float32, device="cuda")
        lse = torch.full((cfg.batch, cfg.q_heads), float("nan"), dtype=torch.float32, device="cuda")
        lib.decode_paged_noalloc(q, kc, vc, bt, sl, out, lse, cfg.scale, max_seq_len=max_len, num_splits=8)
        torch.cuda.synchronize()
        o, l = to_f64(out), to_f64(lse)
        assert_o_close(o, ref_o, False, f"noalloc call {call}")
        assert_lse_close(l, ref_l, f"noalloc call {call}")


@pytest.mark.gpu
def test_noalloc_after_a_larger_plan_and_without_allocating(lib):
    """A call with more splits over longer sequences leaves its partials in the
    shared array; a smaller call right after must not read any of them. Around
    that call neither torch's allocator nor the device's free memory moves."""
    import torch
    big_lens = np.array([30000, 17, 25000, 9000, 31000, 1], dtype=np.int32)
    small_lens = np.array([300, 1, 2000, 64, 65, 1000], dtype=np.int32)
    cfg = wl.DecodeConfig("noalloc2", 6, 32, 8, 128, 1, 1, 22)
    d_big = wl.make_decode(cfg, kv_lens=big_lens)
    d_small = wl.make_decode(wl.DecodeConfig("noalloc3", 6, 32, 8, 128, 1, 1, 23), kv_lens=small_lens)
    dev = {k: (to_dev_bf16(v) if k in ("q", "k_pool", "v_pool") else to_dev_i32(v))
           for k, v in d_big.items() if k in ("q", "k_pool", "v_pool", "block_table", "kv_lens")}
    small = {k: (to_dev_bf16(v) if k in ("q", "k_pool", "v_pool") else to_dev_i32(v))
             for k, v in d_small.items() if k in ("q", "k_pool", "v_pool", "block_table", "kv_lens")}
    out_big = torch.empty((6, 32, 128), dtype=torch.float32, device="cuda")
    lib.decode_paged_noalloc(dev["q"], dev["k_pool"], dev["v_pool"], dev["block_table"], dev["kv_lens"], out_big,
                             None, cfg.scale, max_seq_len=int(big_lens.max()), num_splits=32)
    ref_o, ref_l = lib.decode_paged(small["q"], small["k_pool"], small["v_pool"], small["block_table"],
                                    small["kv_lens"], cfg.scale, max_seq_len=int(small_lens.max()), num_splits=3,
                                    out_dtype=torch.float32)
    out = torch.full((6, 32, 128), float("nan"), dtype=torch.float32, device="cuda")
    lse = torch.full((6, 32), float("nan"), dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()
    allocated, (free, _) = torch.cuda.memory_allocated(), torch.cuda.mem_get_info()
    lib.decode_paged_noalloc(small["q"], small["k_pool"], small["v_pool"], small["block_table"], small["kv_lens"],
                             out, lse, cfg.scale, max_seq_len=int(small_lens.max()), num_splits=3)
    torch.cuda.synchronize()
    assert torch.cuda.memory_allocated() == allocated
    assert torch.cuda.mem_get_info()[0] == free
    assert_o_close(to_f64(out), to_f64(ref_o), False, "noalloc after a larger plan")
    assert_lse_close(to_f64(lse), to_f64(ref_l), "noalloc after a larger plan")


@pytest.mark.gpu
def test_noalloc_rejects_a_plan_larger_than_its_array(lib):
    import torch
    B, Hq, Hkv = 512, 64, 8
    q = torch.zeros((B, Hq, 128), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((4, Hkv, 16, 128), dtype=torch.bfloat16, device="cuda")
    bt = torch.zeros((B, 4096), dtype=torch.int32, device="cuda")
    sl = torch.ones((B,), dtype=torch.int32, device="cuda")
    out = torch.empty_like(q)
    with pytest.raises(lib.AttnError) as e:
        lib.decode_paged_noalloc(q, kc, kc, bt, sl, out, None, max_seq_len=65536, num_splits=64)
    assert e.value.status == lib.ATTN_ERR_WORKSPACE
