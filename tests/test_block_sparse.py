"""Block-sparse (BSR) attention through the block-table kernels.

A BSR pattern (query block r sees the key blocks listed for it, the
block-sparse format of the FlashInfer section of "抱infra脚") needs no kernel
of its own: with keys/values paged in 16-token blocks, query block r becomes
one batch entry of the paged prefill whose table lists the physical blocks of
its key blocks (non-causal), and a decode query's table lists its blocks.
workloads.bsr_tables builds those tables (a listed partial last key block goes
last). Both paths are checked against the oracle's BSR definition.
"""
import numpy as np
import pytest

from attention_tiled_exact_b200 import workloads as wl
from oracle import attention_ref as ref
from tests.helpers import assert_lse_close, assert_o_close, to_dev_bf16, to_dev_i32, to_f64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("Sq,Sk,R,window,extra", [
    (300, 1000, 64, 6, 4),    # ragged last query block, partial last key block
    (512, 2048, 128, 16, 8),  # full tiles
    (96, 333, 32, 2, 0),      # local window only
])
def test_block_sparse_prefill_matches_oracle(lib, Sq, Sk, R, window, extra):
    import torch
    Hq, Hkv, D = 8, 2, 128
    d = wl.make_block_sparse(70 + R, Hq, Hkv, Sq, Sk, D, R, window, extra)
    table, k_lens = wl.bsr_tables(d, Sk)
    n_rb = len(d["indptr"]) - 1
    qb = np.zeros((n_rb, Hq, R, D), dtype=np.uint16)
    q_lens = np.zeros(n_rb, dtype=np.int32)
    for r in range(n_rb):
        rows = d["q"][:, R * r:R * r + R]
        qb[r, :, :rows.shape[1]] = rows
        q_lens[r] = rows.shape[1]
    scale = 1.0 / np.sqrt(D)
    o, lse = lib.prefill_paged(to_dev_bf16(qb), to_dev_bf16(d["k_pool"]), to_dev_bf16(d["v_pool"]),
                               to_dev_i32(table), to_dev_i32(k_lens), to_dev_i32(q_lens), scale, False,
                               out_dtype=torch.float32)
    torch.cuda.synchronize()
    o, lse = to_f64(o), to_f64(lse)
    got = np.concatenate([o[r, :, :q_lens[r]] for r in range(n_rb)], axis=1)
    got_l = np.concatenate([lse[r, :, :q_lens[r]] for r in range(n_rb)], axis=1)
    O_ref, L_ref = ref.ref_block_sparse_attention(d["q"], d["k"], d["v"], d["indptr"], d["indices"], R, 16, scale)
    assert_o_close(got, O_ref, False, "bsr prefill")
    assert_lse_close(got_l, L_ref, "bsr prefill lse")


def test_block_sparse_decode_matches_oracle(lib):
    """Six decode queries over one cache, each seeing its own set of key blocks."""
    import torch
    Hq, Hkv, D, n, Sk = 8, 2, 128, 6, 2000
    d = wl.make_block_sparse(79, Hq, Hkv, n, Sk, D, 1, 8, 10)
    table, lens = wl.bsr_tables(d, Sk)
    q = np.ascontiguousarray(d["q"].transpose(1, 0, 2))  # [n, Hq, D]
    scale = 1.0 / np.sqrt(D)
    for splits in (1, 0):
        o, lse = lib.decode_paged(to_dev_bf16(q), to_dev_bf16(d["k_pool"]), to_dev_bf16(d["v_pool"]),
                                  to_dev_i32(table), to_dev_i32(lens), scale, num_splits=splits,
                                  out_dtype=torch.float32)
        torch.cuda.synchronize()
        O_ref, L_ref = ref.ref_block_sparse_attention(d["q"], d["k"], d["v"], d["indptr"], d["indices"], 1, 16,
                                                      scale)
        assert_o_close(to_f64(o), O_ref.transpose(1, 0, 2), False, f"bsr decode splits={splits}")
        assert_lse_close(to_f64(lse), L_ref.T, f"bsr decode lse splits={splits}")
