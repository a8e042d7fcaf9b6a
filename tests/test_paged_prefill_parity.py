"""Paged prefill (chunked prefill over a block-table KV cache) and the mixed
chunked-prefill + decode batch: CUDA path (C ABI) vs the fp64 oracle.

The pool's spare blocks, the tail slots past each sequence end and the unused
table entries hold NaN, so the kernel must neither read them into a score nor
multiply them into O.
"""
import numpy as np
import pytest

from attention_tiled_exact_b200 import workloads as wl
from oracle import attention_ref as ref
from tests.helpers import assert_lse_close, assert_o_close, to_dev_bf16, to_dev_i32, to_f64

pytestmark = pytest.mark.gpu


def _chunks(ctx, q_len, Hq, Hkv, D, seed, identity=False):
    ctx = np.asarray(ctx, dtype=np.int32)
    k_lens = (ctx + q_len).astype(np.int32)
    d = wl.make_paged_pool(seed, k_lens, Hkv, D, identity=identity)
    d["q"] = wl.normal_bf16(seed, (len(ctx), Hq, q_len, D), 30)
    d["q_lens"] = np.full(len(ctx), q_len, dtype=np.int32)
    d["scale"] = 1.0 / np.sqrt(D)
    return d


def _run(lib, d, out_dtype=None, flags=None, table=None):
    """One paged prefill call; without a caller's error word, its own must stay clear."""
    import torch
    own = flags is None
    if own:
        flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = lib.prefill_paged(to_dev_bf16(d["q"]), to_dev_bf16(d["k_pool"]), to_dev_bf16(d["v_pool"]),
                               to_dev_i32(d["block_table"] if table is None else table), to_dev_i32(d["kv_lens"]),
                               to_dev_i32(d["q_lens"]), d["scale"], True, out_dtype=out_dtype or torch.float32,
                               error_flags=flags)
    torch.cuda.synchronize()
    if own:
        assert lib.sync_error_flags(flags) == (lib.ATTN_OK, 0)
    return to_f64(o), to_f64(lse)


@pytest.mark.parametrize("ctx,q_len,Hq,Hkv,D", [
    ([0, 37, 64, 200], 100, 8, 2, 128),   # no context, ragged, 64-aligned, ragged tail
    ([5, 300], 257, 4, 4, 128),           # MHA (row-block pairs), odd row blocks
    ([1000, 16], 64, 16, 2, 64),          # G=8, D=64, 16-aligned context
    ([17], 1, 4, 1, 128),                 # one query row
])
def test_paged_prefill_matches_oracle(lib, ctx, q_len, Hq, Hkv, D):
    import torch
    d = _chunks(ctx, q_len, Hq, Hkv, D, seed=50 + q_len + D)
    O_ref, L_ref = ref.ref_prefill_paged(d["q"], d["q_lens"], d["k_pool"], d["v_pool"], d["block_table"],
                                         d["kv_lens"], d["scale"], True)
    o, lse = _run(lib, d)
    assert_o_close(o, O_ref, False, "paged prefill fp32")
    assert_lse_close(lse, L_ref, "paged prefill lse")
    o16, _ = _run(lib, d, out_dtype=torch.bfloat16)
    assert_o_close(o16, O_ref, True, "paged prefill bf16")


@pytest.mark.parametrize("n_seq,q_len,Hq,Hkv,D", [
    (12, 256, 8, 2, 128),   # 96 work items: sorted by cost before they are dealt to the SMs
    (260, 128, 32, 4, 64),  # 4160 work items: more than the sort takes, plain snake order
])
def test_paged_prefill_many_items(lib, n_seq, q_len, Hq, Hkv, D):
    """Variable lengths with either item order: every valid row is written once
    and matches the oracle (sampled rows), rows past q_lens[b] stay untouched."""
    import torch
    rng = np.random.default_rng(n_seq)
    d = _chunks(rng.integers(0, 300, n_seq), q_len, Hq, Hkv, D, seed=90 + n_seq)
    d["q_lens"] = rng.integers(1, q_len + 1, n_seq).astype(np.int32)
    q = to_dev_bf16(d["q"])
    out = torch.full(q.shape, 7.0, dtype=torch.float32, device="cuda")
    lse = torch.full(q.shape[:3], 7.0, dtype=torch.float32, device="cuda")
    lib.prefill_paged(q, to_dev_bf16(d["k_pool"]), to_dev_bf16(d["v_pool"]), to_dev_i32(d["block_table"]),
                      to_dev_i32(d["kv_lens"]), to_dev_i32(d["q_lens"]), d["scale"], True, out=out, lse=lse)
    torch.cuda.synchronize()
    o, l = to_f64(out), to_f64(lse)
    valid = np.arange(q_len)[None, None, :] < d["q_lens"][:, None, None]
    assert np.isfinite(l[np.broadcast_to(valid, l.shape)]).all()
    assert (l[~np.broadcast_to(valid, l.shape)] == 7.0).all() and (o[~np.broadcast_to(valid, l.shape)] == 7.0).all()
    rows = [(0, 0, 0), (n_seq - 1, Hq - 1, int(d["q_lens"][-1]) - 1)]
    for _ in range(60):
        b = int(rng.integers(n_seq))
        rows.append((b, int(rng.integers(Hq)), int(rng.integers(d["q_lens"][b]))))
    O_ref, L_ref = ref.ref_prefill_paged(d["q"], d["q_lens"], d["k_pool"], d["v_pool"], d["block_table"],
                                         d["kv_lens"], d["scale"], True, rows=rows)
    assert_o_close(np.stack([o[b, h, i] for b, h, i in rows]), O_ref, False, "many items")
    assert_lse_close(np.array([l[b, h, i] for b, h, i in rows]), L_ref, "many items lse")


def test_paged_equals_dense_bitwise(lib):
    """Same tokens, dense [B,H,S,D] layout vs identity-ordered pages: identical bits."""
    import torch
    ctx, q_len = [64, 192], 128  # 64-aligned key lengths, so the dense and paged tiles line up
    d = _chunks(ctx, q_len, 8, 2, 128, seed=7)
    o_p, l_p = _run(lib, d)
    # dense K/V gathered from the pool, padded to the longest sequence with zeros
    Sk = int(d["kv_lens"].max())
    k = np.zeros((2, 2, Sk, 128), dtype=np.uint16)
    v = np.zeros((2, 2, Sk, 128), dtype=np.uint16)
    for b in range(2):
        for h in range(2):
            n = int(d["kv_lens"][b])
            k[b, h, :n] = ref.gather_paged(d["k_pool"], d["block_table"][b], n, h)
            v[b, h, :n] = ref.gather_paged(d["v_pool"], d["block_table"][b], n, h)
    for b in range(2):  # run each sequence densely with its own key length
        n = int(d["kv_lens"][b])
        o, l = lib.prefill(to_dev_bf16(d["q"][b:b + 1]), to_dev_bf16(k[b:b + 1, :, :n]),
                           to_dev_bf16(v[b:b + 1, :, :n]), d["scale"], True, out_dtype=torch.float32)
        torch.cuda.synchronize()
        assert np.array_equal(to_f64(o)[0], o_p[b]) and np.array_equal(to_f64(l)[0], l_p[b])


def test_paged_bad_block_is_flagged(lib):
    import torch
    d = _chunks([40], 30, 4, 1, 128, seed=8)
    table = d["block_table"].copy()
    table[0, 1] = d["num_blocks"] + 7
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, _ = _run(lib, d, flags=flags, table=table)
    assert int(flags.item()) & lib.ATTN_FAULT_BAD_BLOCK
    assert np.isfinite(o).all()


def _mixed_run(lib, d, cfg, out_dtype=None):
    """One step of the mixed batch: paged prefill of the chunks, then decode of the rest."""
    import torch
    out_dtype = out_dtype or torch.float32
    kc, vc = to_dev_bf16(d["k_pool"]), to_dev_bf16(d["v_pool"])
    table = to_dev_i32(d["block_table"])
    lens = to_dev_i32(d["kv_lens"])
    nc = cfg.chunks
    o_p, l_p = lib.prefill_paged(to_dev_bf16(d["q_chunk"]), kc, vc, table[:nc], lens[:nc], None, cfg.scale, True,
                                 out_dtype=out_dtype)
    o_d, l_d = lib.decode_paged(to_dev_bf16(d["q_dec"]), kc, vc, table[nc:].contiguous(), lens[nc:].contiguous(),
                                cfg.scale, max_seq_len=int(d["kv_lens"][nc:].max()), out_dtype=out_dtype)
    torch.cuda.synchronize()
    return to_f64(o_p), to_f64(l_p), to_f64(o_d), to_f64(l_d)


def test_mixed_batch_small(lib):
    cfg = wl.MixedConfig("mixed_small", 3, 96, 0, 300, 5, 16, 600, 8, 2, 128, 11)
    d = wl.make_mixed(cfg)
    o_p, l_p, o_d, l_d = _mixed_run(lib, d, cfg)
    nc = cfg.chunks
    Op, Lp = ref.ref_prefill_paged(d["q_chunk"], [cfg.chunk_len] * nc, d["k_pool"], d["v_pool"],
                                   d["block_table"][:nc], d["kv_lens"][:nc], cfg.scale, True)
    Od, Ld = ref.ref_decode_paged(d["q_dec"], d["k_pool"], d["v_pool"], d["block_table"][nc:], d["kv_lens"][nc:],
                                  cfg.scale)
    assert_o_close(o_p, Op, False, "mixed prefill")
    assert_lse_close(l_p, Lp, "mixed prefill")
    assert_o_close(o_d, Od, False, "mixed decode")
    assert_lse_close(l_d, Ld, "mixed decode")


def test_mixed_full_size_every_row(lib):
    """8 chunks x 512 queries on context U[0, 8192] + 128 decode rows on
    U[512, 16384]: every prefill row and every decode row against the oracle
    (fp32 output, strict bound), then the bench's bf16-output step."""
    import torch
    from tests.oracle_all_rows import decode_all_rows, prefill_paged_all_rows
    cfg = wl.MIXED
    d = wl.make_mixed(cfg)
    nc = cfg.chunks
    Op, Lp = prefill_paged_all_rows(d["q_chunk"], np.full(nc, cfg.chunk_len, dtype=np.int32), d["k_pool"],
                                    d["v_pool"], d["block_table"][:nc], d["kv_lens"][:nc], cfg.scale, True)
    Od, Ld = decode_all_rows(d["q_dec"], d["k_pool"], d["v_pool"], d["block_table"][nc:], d["kv_lens"][nc:],
                             cfg.scale)
    o_p, l_p, o_d, l_d = _mixed_run(lib, d, cfg)
    assert_o_close(o_p, Op, False, "mixed prefill")
    assert_lse_close(l_p, Lp, "mixed prefill")
    assert_o_close(o_d, Od, False, "mixed decode")
    assert_lse_close(l_d, Ld, "mixed decode")
    o_p, l_p, o_d, l_d = _mixed_run(lib, d, cfg, out_dtype=torch.bfloat16)
    assert_o_close(o_p, Op, True, "mixed prefill bf16 out")
    assert_o_close(o_d, Od, True, "mixed decode bf16 out")
