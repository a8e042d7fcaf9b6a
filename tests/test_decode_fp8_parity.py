"""Paged split-KV decode over an FP8 E4M3 cache (one scale per tensor): the
CUDA path (C ABI) against the fp64 oracle, which decodes the codes exactly.

Spare blocks and the tail slots past each sequence end hold the E4M3 NaN code,
so a read outside a sequence's tokens shows up as NaN.
"""
import numpy as np
import pytest

from attention_tiled_exact_b200 import workloads as wl
from oracle import attention_ref as ref
from tests.helpers import assert_lse_close, assert_o_close, to_dev_bf16, to_dev_i32, to_f64

pytestmark = pytest.mark.gpu


def _to_dev_u8(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).to("cuda")


def _inputs(lens, Hq=8, Hkv=2, seed=1):
    cfg = wl.DecodeConfig("fp8", len(lens), Hq, Hkv, 128, 1, 1, seed)
    return wl.make_decode_fp8(cfg, kv_lens=np.asarray(lens, dtype=np.int32))


def _decode(lib, d, num_splits=0, out_dtype=None, table=None, k_pool=None, v_pool=None, as_float8=False, flags=None):
    import torch
    kc = _to_dev_u8(d["k_pool"] if k_pool is None else k_pool)
    vc = _to_dev_u8(d["v_pool"] if v_pool is None else v_pool)
    if as_float8:
        kc, vc = kc.view(torch.float8_e4m3fn), vc.view(torch.float8_e4m3fn)
    o, lse = lib.decode_paged(to_dev_bf16(d["q"]), kc, vc, to_dev_i32(d["block_table"] if table is None else table),
                              to_dev_i32(d["kv_lens"]), d["scale"], num_splits=num_splits,
                              out_dtype=out_dtype or torch.bfloat16, k_scale=d["k_scale"], v_scale=d["v_scale"],
                              error_flags=flags)
    torch.cuda.synchronize()
    return to_f64(o), to_f64(lse)


def _oracle(d, table=None):
    return ref.ref_decode_paged_fp8(d["q"], d["k_pool"], d["v_pool"], d["k_scale"], d["v_scale"],
                                    d["block_table"] if table is None else table, d["kv_lens"], d["scale"])


@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("num_splits", [1, 0, 7])
def test_fp8_decode_matches_oracle(lib, G, num_splits):
    import torch
    d = _inputs([1, 15, 16, 17, 200, 1000, 2049], Hq=2 * G, Hkv=2, seed=30 + G)
    O_ref, L_ref = _oracle(d)
    o, lse = _decode(lib, d, num_splits=num_splits, out_dtype=torch.float32)
    assert_o_close(o, O_ref, False, f"fp8 G={G} splits={num_splits}")
    assert_lse_close(lse, L_ref, f"fp8 G={G} splits={num_splits}")
    o16, _ = _decode(lib, d, num_splits=num_splits)
    assert_o_close(o16, O_ref, True, "fp8 bf16 out")


def test_fp8_float8_dtype_equals_uint8_codes(lib):
    """The same codes passed as torch.float8_e4m3fn or as uint8: identical bits."""
    d = _inputs([100, 3000, 7], seed=41)
    o1, l1 = _decode(lib, d)
    o2, l2 = _decode(lib, d, as_float8=True)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_fp8_bit_exact_paging(lib):
    """Permuted block table vs identity re-layout of the same codes: bitwise equal."""
    d = _inputs([1, 16, 33, 500, 1234, 4000], seed=42)
    for s in (1, 0, 3):
        o_perm, l_perm = _decode(lib, d, num_splits=s)
        kp, tbl = wl.relayout_identity(d["k_pool"], d["block_table"], d["kv_lens"])
        vp, tbl2 = wl.relayout_identity(d["v_pool"], d["block_table"], d["kv_lens"])
        assert np.array_equal(tbl, tbl2) and kp.dtype == np.uint8
        o_id, l_id = _decode(lib, d, num_splits=s, table=tbl, k_pool=kp, v_pool=vp)
        assert np.array_equal(o_perm, o_id) and np.array_equal(l_perm, l_id)
        assert np.isfinite(o_perm).all()


def test_fp8_zero_length_and_split_invariance(lib):
    import torch
    d = _inputs([0, 40, 0, 1, 5000], seed=43)
    O_ref, L_ref = _oracle(d)
    o1, l1 = _decode(lib, d, num_splits=1, out_dtype=torch.float32)
    assert (o1[0] == 0).all() and np.isneginf(l1[0]).all() and np.isneginf(l1[2]).all()
    assert_o_close(o1, O_ref, False, "fp8 zero length")
    assert_lse_close(l1, L_ref, "fp8 zero length")
    # P enters the tensor-core P V in fp16, rounded against each split's own
    # running max, so split counts agree to fp16 rounding of P (2^-11 relative).
    fin = np.isfinite(l1)
    for s in (2, 5, 16):
        o, l = _decode(lib, d, num_splits=s, out_dtype=torch.float32)
        assert np.array_equal(np.isneginf(l), ~fin)
        assert np.abs(o - o1).max() < 2e-4 and np.abs(l[fin] - l1[fin]).max() < 2e-5


def test_fp8_bad_block_id_is_flagged(lib):
    import torch
    d = _inputs([64, 64], Hq=4, Hkv=1, seed=44)
    table = d["block_table"].copy()
    table[1, 2] = d["num_blocks"] + 1000  # outside the pool
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, _ = _decode(lib, d, num_splits=1, table=table, flags=flags)
    assert int(flags.item()) & lib.ATTN_FAULT_BAD_BLOCK
    assert np.isfinite(o).all()


def test_fp8_full_size_every_row(lib):
    """The bench's decode shape (64 sequences of 1K-32K tokens, 32/8 heads) on an
    FP8 cache, every row against the oracle."""
    import torch
    from tests.oracle_all_rows import decode_fp8_all_rows
    cfg = wl.PAGED_DECODE
    d = wl.make_decode_fp8(cfg)
    O_ref, L_ref = decode_fp8_all_rows(d["q"], d["k_pool"], d["v_pool"], d["k_scale"], d["v_scale"],
                                       d["block_table"], d["kv_lens"], d["scale"])
    o, lse = _decode(lib, d, out_dtype=torch.float32)
    assert_o_close(o, O_ref, False, "fp8 full size")
    assert_lse_close(lse, L_ref, "fp8 full size lse")
