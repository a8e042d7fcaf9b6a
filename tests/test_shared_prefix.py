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


# ---------------------------------------------------------------------------
# attn_decode_paged_shared_prefix: the shared prefix attended once per batch
# (prefix prefill + suffix decode + log-sum-exp merge) against the fp64 oracle
# of plain decode over the aliased tables.
# ---------------------------------------------------------------------------


def _cascade(lib, d, num_splits=0, out_dtype=None, table=None, seq_lens=None, flags=None, max_seq_len=0,
             prefix_len=None):
    import torch
    o, lse = lib.decode_paged_shared_prefix(
        to_dev_bf16(d["q"]), to_dev_bf16(d["k_pool"]), to_dev_bf16(d["v_pool"]),
        to_dev_i32(d["block_table"] if table is None else table),
        to_dev_i32(d["kv_lens"] if seq_lens is None else seq_lens),
        d["prefix_len"] if prefix_len is None else prefix_len, d["scale"], max_seq_len=max_seq_len,
        num_splits=num_splits, out_dtype=out_dtype or torch.float32, error_flags=flags)
    torch.cuda.synchronize()
    return to_f64(o), to_f64(lse)


def _prefix_inputs(batch, G, prefix_len, lo, hi, seed, Hkv=2):
    cfg = wl.SharedPrefixConfig("sp", batch, G * Hkv, Hkv, 128, prefix_len, lo, hi, seed)
    return wl.make_shared_prefix_decode(cfg)


@pytest.mark.parametrize("batch,G,prefix_len,lo,hi", [
    (6, 4, 320, 0, 300),      # one prefix range
    (1, 1, 16, 0, 40),        # a single sequence, a one-block prefix
    (64, 4, 4096, 0, 700),    # the prefix cut into several key ranges
    (130, 2, 512, 0, 100),    # two 128-row blocks of queries, ragged
    (300, 8, 1024, 1, 2100),  # G = 8, three row blocks, split suffixes
    (5, 1, 2048, 17, 17),     # G = 1 (single-head items), equal suffixes
])
def test_shared_prefix_decode_matches_oracle(lib, batch, G, prefix_len, lo, hi):
    import torch
    d = _prefix_inputs(batch, G, prefix_len, lo, hi, seed=80 + G + batch)
    O_ref, L_ref = ref.ref_decode_paged(d["q"], d["k_pool"], d["v_pool"], d["block_table"], d["kv_lens"],
                                        d["scale"])
    for splits in (0, 1):
        o, lse = _cascade(lib, d, num_splits=splits)
        assert_o_close(o, O_ref, False, f"shared prefix splits={splits}")
        assert_lse_close(lse, L_ref, f"shared prefix splits={splits}")
    o16, _ = _cascade(lib, d, out_dtype=torch.bfloat16)
    assert_o_close(o16, O_ref, True, "shared prefix bf16 out")


def test_shared_prefix_reads_only_sequence_zero_prefix_entries(lib):
    """The prefix is read from sequence 0's table entries only: pointing the
    other sequences' prefix entries at a NaN spare block changes no bit of the
    result, and the mismatch is flagged (ATTN_FAULT_PREFIX_MISMATCH); aliased
    entries leave the error word clear."""
    import torch
    d = _prefix_inputs(9, 4, 640, 0, 500, seed=90)
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    o1, l1 = _cascade(lib, d, flags=flags)
    assert int(flags.item()) == 0
    table = d["block_table"].copy()
    table[1:, :640 // 16] = d["spare_ids"][0]
    o2, l2 = _cascade(lib, d, table=table, flags=flags)
    assert int(flags.item()) == lib.ATTN_FAULT_PREFIX_MISMATCH
    assert np.isfinite(o2).all() and np.array_equal(o1, o2) and np.array_equal(l1, l2)
    flags.zero_()
    table = d["block_table"].copy()
    table[8, 639 // 16] = d["spare_ids"][1]  # one entry of the last row, the last prefix block
    _cascade(lib, d, table=table, flags=flags)
    assert int(flags.item()) == lib.ATTN_FAULT_PREFIX_MISMATCH


def test_shared_prefix_filling_the_whole_table(lib):
    """prefix_len = table capacity: every suffix is empty (no suffix decode)."""
    d = _prefix_inputs(7, 2, 800, 0, 0, seed=91)
    assert d["block_table"].shape[1] == 800 // 16
    O_ref, L_ref = ref.ref_decode_paged(d["q"], d["k_pool"], d["v_pool"], d["block_table"], d["kv_lens"],
                                        d["scale"])
    o, lse = _cascade(lib, d)
    assert_o_close(o, O_ref, False, "prefix only")
    assert_lse_close(lse, L_ref, "prefix only")


def test_shared_prefix_zero_is_plain_decode(lib):
    """prefix_len = 0 runs the plain decode: identical bits."""
    import torch
    d = _prefix_inputs(5, 4, 0, 1, 900, seed=92)
    o1, l1 = _cascade(lib, d)
    o2, l2 = lib.decode_paged(to_dev_bf16(d["q"]), to_dev_bf16(d["k_pool"]), to_dev_bf16(d["v_pool"]),
                              to_dev_i32(d["block_table"]), to_dev_i32(d["kv_lens"]), d["scale"],
                              out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert np.array_equal(o1, to_f64(o2)) and np.array_equal(l1, to_f64(l2))


def test_shared_prefix_short_sequence_is_flagged(lib):
    """A sequence shorter than the prefix sets ATTN_FAULT_BAD_LENGTH; the
    other sequences are unaffected."""
    import torch
    d = _prefix_inputs(4, 4, 320, 10, 200, seed=93)
    lens = d["kv_lens"].copy()
    lens[2] = 300
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = _cascade(lib, d, seq_lens=lens, flags=flags)
    assert int(flags.item()) & lib.ATTN_FAULT_BAD_LENGTH
    assert np.isfinite(o).all()
    ok = [0, 1, 3]
    O_ref, L_ref = ref.ref_decode_paged(d["q"][ok], d["k_pool"], d["v_pool"], d["block_table"][ok],
                                        d["kv_lens"][ok], d["scale"])
    assert_o_close(o[ok], O_ref, False, "unaffected rows")
    assert_lse_close(lse[ok], L_ref, "unaffected rows")


def test_shared_prefix_graph_replay(lib):
    """Captured once with a caller-owned workspace, replayed with new own
    tokens and lengths in the static buffers (the prefix stays)."""
    import torch
    cfg = wl.SharedPrefixConfig("g", 8, 8, 2, 128, 512, 0, 600, 94)
    d0 = wl.make_shared_prefix_decode(cfg, suffix_lens=np.full(8, 600, dtype=np.int32))
    q_s = to_dev_bf16(d0["q"])
    k_s, v_s = to_dev_bf16(d0["k_pool"]), to_dev_bf16(d0["v_pool"])
    bt_s, sl_s = to_dev_i32(d0["block_table"]), to_dev_i32(d0["kv_lens"])
    o_s = torch.empty((8, 8, 128), dtype=torch.float32, device="cuda")
    l_s = torch.empty((8, 8), dtype=torch.float32, device="cuda")
    max_len = 512 + 600
    ws = torch.empty(lib.decode_shared_prefix_workspace_bytes(q_s, k_s, v_s, bt_s, sl_s, 512, max_seq_len=max_len),
                     dtype=torch.uint8, device="cuda")

    def step():
        lib.decode_paged_shared_prefix(q_s, k_s, v_s, bt_s, sl_s, 512, cfg.scale, max_seq_len=max_len, out=o_s,
                                       lse=l_s, workspace=ws)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    rng = np.random.default_rng(95)
    for it in range(3):
        lens = 512 + rng.integers(0, 601, 8).astype(np.int32)
        q_new = wl.normal_bf16(96 + it, (8, 8, 128))
        q_s.copy_(to_dev_bf16(q_new))
        sl_s.copy_(to_dev_i32(lens))
        g.replay()
        torch.cuda.synchronize()
        O_ref, L_ref = ref.ref_decode_paged(q_new, d0["k_pool"], d0["v_pool"], d0["block_table"], lens, cfg.scale)
        assert_o_close(to_f64(o_s), O_ref, False, f"replay {it}")
        assert_lse_close(to_f64(l_s), L_ref, f"replay {it}")


def test_shared_prefix_full_size_every_row(lib):
    """The bench's shared-prefix shape (64 sequences, 8192 shared tokens plus
    64..2048 own tokens, 32/8 heads), every row against the oracle."""
    from tests.oracle_all_rows import decode_all_rows
    cfg = wl.SHARED_PREFIX_DECODE
    d = wl.make_shared_prefix_decode(cfg)
    O_ref, L_ref = decode_all_rows(d["q"], d["k_pool"], d["v_pool"], d["block_table"], d["kv_lens"], d["scale"])
    o, lse = _cascade(lib, d)
    assert_o_close(o, O_ref, False, "shared prefix full size")
    assert_lse_close(lse, L_ref, "shared prefix full size lse")
