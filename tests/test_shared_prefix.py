"""Shared prefixes through block tables with aliased blocks ("抱infra脚", Paged
Attention: requests with the same prefix can share KV blocks).

Every sequence's first blocks point at the same physical blocks (sequence 0's
prefix), so the kernels read them once per sequence through the table. Decode
and chunked prefill must match the oracle, which gathers through the same
table, and must equal, bit for bit, the same computation over a layout where
each sequence owns a physical copy of the prefix.
"""
import numpy as np
import pytest

from attention_tiled_exact_b200 import workloads as wl
from oracle import attention_ref as ref
from tests.helpers import assert_lse_close, assert_o_close, to_dev_bf16, to_dev_i32, to_f64

pytestmark = pytest.mark.gpu

PREFIX_BLOCKS = 20  # 320 shared tokens


def _alias_prefix(d):
    """Point every sequence's first PREFIX_BLOCKS entries at sequence 0's blocks.

    Returns (aliased table, copied pools + table): the copy gives each sequence
    its own physical blocks holding the same prefix values."""
    table = d["block_table"].copy()
    aliased = table.copy()
    aliased[:, :PREFIX_BLOCKS] = table[0, :PREFIX_BLOCKS]
    kp, vp = d["k_pool"].copy(), d["v_pool"].copy()
    for b in range(1, table.shape[0]):
        kp[table[b, :PREFIX_BLOCKS]] = d["k_pool"][table[0, :PREFIX_BLOCKS]]
        vp[table[b, :PREFIX_BLOCKS]] = d["v_pool"][table[0, :PREFIX_BLOCKS]]
    return aliased, kp, vp, table


def test_decode_over_shared_prefix_blocks(lib):
    import torch
    lens = np.array([PREFIX_BLOCKS * 16 + s for s in (0, 1, 17, 300, 2000, 5)], dtype=np.int32)
    d = wl.make_decode(wl.DecodeConfig("prefix", len(lens), 8, 2, 128, 1, 1, 71), kv_lens=lens)
    aliased, kp, vp, own = _alias_prefix(d)
    q = to_dev_bf16(d["q"])
    sl = to_dev_i32(lens)
    outs = []
    for kpool, vpool, table in ((d["k_pool"], d["v_pool"], aliased), (kp, vp, own)):
        for splits in (1, 0):
            o, lse = lib.decode_paged(q, to_dev_bf16(kpool), to_dev_bf16(vpool), to_dev_i32(table), sl, d["scale"],
                                      num_splits=splits, out_dtype=torch.float32)
            torch.cuda.synchronize()
            outs.append((to_f64(o), to_f64(lse)))
    O_ref, L_ref = ref.ref_decode_paged(d["q"], d["k_pool"], d["v_pool"], aliased, lens, d["scale"])
    assert_o_close(outs[0][0], O_ref, False, "aliased prefix decode")
    assert_lse_close(outs[0][1], L_ref, "aliased prefix decode lse")
    for (oa, la), (oc, lc) in zip(outs[:2], outs[2:]):  # same split plan: aliased == copied, bit for bit
        assert np.array_equal(oa, oc) and np.array_equal(la, lc)


def test_chunked_prefill_over_shared_prefix_blocks(lib):
    import torch
    q_len = 200
    ctx = np.array([PREFIX_BLOCKS * 16 + s for s in (0, 64, 5)], dtype=np.int32)
    k_lens = (ctx + q_len).astype(np.int32)
    d = wl.make_paged_pool(73, k_lens, 2, 128)
    q = wl.normal_bf16(73, (len(ctx), 8, q_len, 128), 30)
    aliased, kp, vp, own = _alias_prefix(d)
    q_lens = np.full(len(ctx), q_len, dtype=np.int32)
    scale = 1.0 / np.sqrt(128)
    outs = []
    for kpool, vpool, table in ((d["k_pool"], d["v_pool"], aliased), (kp, vp, own)):
        o, lse = lib.prefill_paged(to_dev_bf16(q), to_dev_bf16(kpool), to_dev_bf16(vpool), to_dev_i32(table),
                                   to_dev_i32(k_lens), to_dev_i32(q_lens), scale, True, out_dtype=torch.float32)
        torch.cuda.synchronize()
        outs.append((to_f64(o), to_f64(lse)))
    O_ref, L_ref = ref.ref_prefill_paged(q, q_lens, d["k_pool"], d["v_pool"], aliased, k_lens, scale, True)
    assert_o_close(outs[0][0], O_ref, False, "aliased prefix prefill")
    assert_lse_close(outs[0][1], L_ref, "aliased prefix prefill lse")
    assert np.array_equal(outs[0][0], outs[1][0]) and np.array_equal(outs[0][1], outs[1][1])
