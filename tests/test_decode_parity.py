"""Paged split-KV decode and the LSE combine: CUDA path (C ABI) vs the fp64 oracle.

Also the bit-exact paging check: decode over a randomly permuted block table
must equal, bit for bit, decode over the same tokens re-laid in identity order.
NaN sentinels fill spare blocks and tail slots, so any read outside a
sequence's tokens shows up as NaN.
"""
import numpy as np
import pytest

from attention_tiled_exact_b200 import workloads as wl
from oracle import attention_ref as ref
from tests.helpers import assert_lse_close, assert_o_close, to_dev_bf16, to_dev_i32, to_f64

pytestmark = pytest.mark.gpu


def _decode(lib, d, num_splits=0, out_dtype=None, max_seq_len=0, flags=None, table=None, k_pool=None, v_pool=None):
    import torch
    q = to_dev_bf16(d["q"])
    kc = to_dev_bf16(d["k_pool"] if k_pool is None else k_pool)
    vc = to_dev_bf16(d["v_pool"] if v_pool is None else v_pool)
    bt = to_dev_i32(d["block_table"] if table is None else table)
    sl = to_dev_i32(d["kv_lens"])
    o, lse = lib.decode_paged(q, kc, vc, bt, sl, d["scale"], max_seq_len=max_seq_len, num_splits=num_splits,
                              out_dtype=out_dtype or torch.bfloat16, error_flags=flags)
    torch.cuda.synchronize()
    return to_f64(o), to_f64(lse)


def _inputs(lens, Hq=8, Hkv=2, seed=1):
    cfg = wl.DecodeConfig("t", len(lens), Hq, Hkv, 128, 1, 1, seed)
    return wl.make_decode(cfg, kv_lens=np.asarray(lens, dtype=np.int32))


@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("num_splits", [1, 0, 7])
def test_decode_matches_oracle(lib, G, num_splits):
    import torch
    lens = [1, 15, 16, 17, 200, 1000, 2049]
    d = _inputs(lens, Hq=2 * G, Hkv=2, seed=10 + G)
    O_ref, L_ref = ref.ref_decode_paged(d["q"], d["k_pool"], d["v_pool"], d["block_table"], d["kv_lens"], d["scale"])
    o, lse = _decode(lib, d, num_splits=num_splits, out_dtype=torch.float32)
    assert_o_close(o, O_ref, False, f"G={G} splits={num_splits}")
    assert_lse_close(lse, L_ref, f"G={G} splits={num_splits}")
    o16, _ = _decode(lib, d, num_splits=num_splits)
    assert_o_close(o16, O_ref, True, "bf16 out")


def test_split_count_does_not_change_the_result(lib):
    import torch
    d = _inputs([3000, 5000, 64, 4097], seed=4)
    o1, l1 = _decode(lib, d, num_splits=1, out_dtype=torch.float32)
    for s in (2, 5, 16, 64):
        o, l = _decode(lib, d, num_splits=s, out_dtype=torch.float32)
        assert np.abs(o - o1).max() < 2e-5 and np.abs(l - l1).max() < 2e-5


def test_zero_length_sequence(lib):
    import torch
    d = _inputs([0, 40, 0, 1], seed=5)
    O_ref, L_ref = ref.ref_decode_paged(d["q"], d["k_pool"], d["v_pool"], d["block_table"], d["kv_lens"], d["scale"])
    for s in (1, 0, 4):
        o, lse = _decode(lib, d, num_splits=s, out_dtype=torch.float32)
        assert (o[0] == 0).all() and np.isneginf(lse[0]).all() and np.isneginf(lse[2]).all()
        assert_o_close(o, O_ref, False, "zero length")
        assert_lse_close(lse, L_ref, "zero length")


def test_bit_exact_paging(lib):
    """Permuted block table vs identity re-layout: bitwise equal outputs."""
    d = _inputs([1, 16, 33, 500, 1234, 4000], Hq=8, Hkv=2, seed=6)
    for s in (1, 0, 3):
        o_perm, l_perm = _decode(lib, d, num_splits=s)
        kp, tbl = wl.relayout_identity(d["k_pool"], d["block_table"], d["kv_lens"])
        vp, tbl2 = wl.relayout_identity(d["v_pool"], d["block_table"], d["kv_lens"])
        assert np.array_equal(tbl, tbl2)
        o_id, l_id = _decode(lib, d, num_splits=s, table=tbl, k_pool=kp, v_pool=vp)
        assert np.array_equal(o_perm, o_id) and np.array_equal(l_perm, l_id)
        assert np.isfinite(o_perm).all()


def test_bad_block_id_is_flagged_not_read(lib):
    """An out-of-range table entry is reported in the error word and never dereferenced."""
    import torch
    d = _inputs([64, 64], Hq=4, Hkv=1, seed=7)
    table = d["block_table"].copy()
    table[1, 2] = d["num_blocks"] + 1000  # outside the pool
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = _decode(lib, d, num_splits=1, flags=flags, table=table)
    assert int(flags.item()) & lib.ATTN_FAULT_BAD_BLOCK
    assert np.isfinite(o).all()
    O_ref, L_ref = ref.ref_decode_paged(d["q"], d["k_pool"], d["v_pool"], d["block_table"], d["kv_lens"], d["scale"])
    assert_o_close(o[0], O_ref[0], True, "untouched sequence")


def test_length_beyond_table_is_flagged(lib):
    import torch
    d = _inputs([40, 20], Hq=4, Hkv=1, seed=8)
    d = dict(d)
    d["kv_lens"] = np.array([40, 10 ** 6], dtype=np.int32)
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, _ = _decode(lib, d, num_splits=1, flags=flags)
    assert int(flags.item()) & lib.ATTN_FAULT_BAD_LENGTH


def test_full_size_paged_decode_every_row(lib):
    """64 sequences, lengths U[1024, 32768], 32/8 heads, in the bench's launch
    configuration (bf16 O, automatic split plan), every row against the oracle;
    then fp32 output under the strict bound."""
    import torch
    from tests.oracle_all_rows import decode_all_rows
    cfg = wl.PAGED_DECODE
    d = wl.make_decode(cfg)
    O_ref, L_ref = decode_all_rows(d["q"], d["k_pool"], d["v_pool"], d["block_table"], d["kv_lens"], d["scale"])
    o, lse = _decode(lib, d, max_seq_len=int(d["kv_lens"].max()))
    assert_o_close(o, O_ref, True, "paged decode bf16 out")
    assert_lse_close(lse, L_ref, "paged decode")
    o32, lse32 = _decode(lib, d, max_seq_len=int(d["kv_lens"].max()), out_dtype=torch.float32)
    assert_o_close(o32, O_ref, False, "paged decode fp32 out")
    assert_lse_close(lse32, L_ref, "paged decode fp32 run")


# ----------------------------------------------------------------------------
# combine
# ----------------------------------------------------------------------------


@pytest.mark.parametrize("D", [64, 128])
def test_combine_matches_oracle(lib, D):
    import torch
    rng = np.random.default_rng(D)
    S, R = 37, 50
    po = rng.standard_normal((S, R, D)).astype(np.float32)
    pl = (rng.standard_normal((S, R)) * 3).astype(np.float32)
    pl[rng.random((S, R)) < 0.2] = -np.inf
    pl[:, 7] = -np.inf          # a row with no keys at all
    po[pl == -np.inf] = np.nan  # an empty split's partial must never be read
    spr = rng.integers(0, S + 1, size=R).astype(np.int32)
    spr[3] = 0
    for per_row in (None, spr):
        O_ref, L_ref = ref.combine_partials(po, pl, per_row)
        t_spr = None if per_row is None else to_dev_i32(per_row)
        o, l = lib.splitkv_lse_combine(torch.from_numpy(po).cuda(), torch.from_numpy(pl).cuda(), t_spr)
        torch.cuda.synchronize()
        assert_o_close(to_f64(o), O_ref, False, "combine")
        assert_lse_close(to_f64(l), L_ref, "combine")
    o16, _ = lib.splitkv_lse_combine(torch.from_numpy(po).cuda(), torch.from_numpy(pl).cuda(),
                                     out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    O_ref, _ = ref.combine_partials(po, pl)
    assert_o_close(to_f64(o16), O_ref, True, "combine bf16")


def test_combine_of_oracle_partials_equals_single_pass(lib):
    """Partials produced by the oracle on key chunks, merged on the GPU, equal one pass."""
    import torch
    rng = np.random.default_rng(3)
    q, k, v = rng.standard_normal((6, 128)), rng.standard_normal((900, 128)), rng.standard_normal((900, 128))
    cuts = [0, 100, 101, 450, 899, 900]
    parts = [ref.attention_rows(q, k[a:b], v[a:b], 0.09) for a, b in zip(cuts[:-1], cuts[1:])]
    po = np.stack([p[0] for p in parts]).astype(np.float32)
    pl = np.stack([p[1] for p in parts]).astype(np.float32)
    o, l = lib.splitkv_lse_combine(torch.from_numpy(po).cuda(), torch.from_numpy(pl).cuda())
    torch.cuda.synchronize()
    O, L = ref.attention_rows(q, k, v, 0.09)
    assert_o_close(to_f64(o), O, False, "chunks")
    assert_lse_close(to_f64(l), L, "chunks")
