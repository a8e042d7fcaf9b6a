"""Packed variable-length queries (cu_seqlens_q): a batch of chunks of
different lengths without padding ("抱infra脚", Chunked Prefill).

Sequence b owns rows cu_seqlens_q[b] .. cu_seqlens_q[b+1] - 1 of q / o
[total_q, Hq, D], its LSE lives in [Hq, total_q]. Every valid row must get
the bits the padded [B, Hq, Sq_max, D] call gives it, and match the oracle;
rows the call does not own stay untouched."""
import numpy as np
import pytest

from attention_tiled_exact_b200 import workloads as wl
from oracle import attention_ref as ref
from tests.helpers import assert_lse_close, assert_o_close, to_dev_bf16, to_dev_i32, to_f64

pytestmark = pytest.mark.gpu


def _pack(q_pad, lens):
    """[B, Hq, Sq_max, D] -> [total, Hq, D] (plus cu_seqlens)."""
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    rows = [q_pad[b, :, :lens[b]].transpose(1, 0, 2) for b in range(len(lens))]
    return np.ascontiguousarray(np.concatenate(rows, axis=0)), cu


@pytest.mark.parametrize("Hq,Hkv,D,causal", [(8, 2, 128, True), (6, 2, 64, False), (4, 4, 128, True)])
def test_packed_dense_matches_padded_and_oracle(lib, Hq, Hkv, D, causal):
    import torch
    lens_q = np.array([300, 1, 0, 513, 128], dtype=np.int32)
    lens_k = np.array([300, 700, 50, 513, 1000], dtype=np.int32)
    B, Sq, Sk = len(lens_q), int(lens_q.max()), int(lens_k.max())
    d = wl.make_prefill(wl.PrefillConfig("packed", B, Hq, Hkv, Sq, Sk, D, causal, 41 + D + Hq))
    q_pk, cu = _pack(d["q"], lens_q)
    total = int(cu[-1])
    extra = 7  # rows after the last sequence: not owned by the call
    q_pk = np.concatenate([q_pk, np.zeros((extra, Hq, D), dtype=q_pk.dtype)], axis=0)
    k, v = to_dev_bf16(d["k"]), to_dev_bf16(d["v"])
    lk = to_dev_i32(lens_k)
    o_pad, l_pad = lib.prefill(to_dev_bf16(d["q"]), k, v, d["scale"], causal, out_dtype=torch.float32,
                               seqlens_q=to_dev_i32(lens_q), seqlens_k=lk)
    out = torch.full((total + extra, Hq, D), 7.0, dtype=torch.float32, device="cuda")
    lse = torch.full((Hq, total + extra), 7.0, dtype=torch.float32, device="cuda")
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    lib.prefill(to_dev_bf16(q_pk), k, v, d["scale"], causal, out=out, lse=lse, seqlens_k=lk,
                cu_seqlens_q=to_dev_i32(cu), max_seqlen_q=Sq, error_flags=flags)
    assert lib.sync_error_flags(flags) == (lib.ATTN_OK, 0)
    o_pad, l_pad, o, l = to_f64(o_pad), to_f64(l_pad), to_f64(out), to_f64(lse)
    for b in range(B):
        r0, r1 = int(cu[b]), int(cu[b + 1])
        assert np.array_equal(o[r0:r1].transpose(1, 0, 2), o_pad[b, :, :lens_q[b]]), f"seq {b}: O bits"
        assert np.array_equal(l[:, r0:r1], l_pad[b, :, :lens_q[b]]), f"seq {b}: LSE bits"
        if r1 > r0:
            O_ref, L_ref = ref.ref_attention(d["q"][b:b + 1, :, :lens_q[b]], d["k"][b:b + 1, :, :lens_k[b]],
                                             d["v"][b:b + 1, :, :lens_k[b]], d["scale"], causal)
            assert_o_close(o[r0:r1].transpose(1, 0, 2)[None], O_ref, False, f"seq {b}")
            assert_lse_close(l[:, r0:r1][None], L_ref, f"seq {b}")
    assert (o[total:] == 7.0).all() and (l[:, total:] == 7.0).all(), "rows past total written"


def test_packed_paged_chunks_match_padded_and_oracle(lib):
    """Chunked prefill over a paged cache with chunks of different lengths."""
    import torch
    q_lens = np.array([512, 37, 200, 1, 129], dtype=np.int32)
    ctx = np.array([1000, 0, 77, 4096, 16], dtype=np.int32)
    k_lens = (ctx + q_lens).astype(np.int32)
    Hq, Hkv, D = 8, 2, 128
    pool = wl.make_paged_pool(44, k_lens, Hkv, D)
    Sq = int(q_lens.max())
    q_pad = wl.normal_bf16(44, (len(q_lens), Hq, Sq, D), 30)
    q_pk, cu = _pack(q_pad, q_lens)
    scale = 1.0 / np.sqrt(D)
    kc, vc = to_dev_bf16(pool["k_pool"]), to_dev_bf16(pool["v_pool"])
    bt, lk = to_dev_i32(pool["block_table"]), to_dev_i32(k_lens)
    o_pad, l_pad = lib.prefill_paged(to_dev_bf16(q_pad), kc, vc, bt, lk, to_dev_i32(q_lens), scale, True,
                                     out_dtype=torch.float32)
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    o_pk, l_pk = lib.prefill_paged(to_dev_bf16(q_pk), kc, vc, bt, lk, None, scale, True, out_dtype=torch.float32,
                                   cu_seqlens_q=to_dev_i32(cu), max_seqlen_q=Sq, error_flags=flags)
    assert lib.sync_error_flags(flags) == (lib.ATTN_OK, 0)
    o_pad, l_pad, o, l = to_f64(o_pad), to_f64(l_pad), to_f64(o_pk), to_f64(l_pk)
    O_ref, L_ref = ref.ref_prefill_paged(q_pad, q_lens, pool["k_pool"], pool["v_pool"], pool["block_table"], k_lens,
                                         scale, True)
    for b in range(len(q_lens)):
        r0, r1 = int(cu[b]), int(cu[b + 1])
        assert np.array_equal(o[r0:r1].transpose(1, 0, 2), o_pad[b, :, :q_lens[b]]), f"chunk {b}: O bits"
        assert np.array_equal(l[:, r0:r1], l_pad[b, :, :q_lens[b]]), f"chunk {b}: LSE bits"
        assert_o_close(o[r0:r1].transpose(1, 0, 2), O_ref[b, :, :q_lens[b]], False, f"chunk {b}")
        assert_lse_close(l[:, r0:r1], L_ref[b, :, :q_lens[b]], f"chunk {b}")
    o16, _ = lib.prefill_paged(to_dev_bf16(q_pk), kc, vc, bt, lk, None, scale, True, cu_seqlens_q=to_dev_i32(cu),
                               max_seqlen_q=Sq)
    torch.cuda.synchronize()
    o16 = to_f64(o16)
    for b in range(len(q_lens)):
        r0, r1 = int(cu[b]), int(cu[b + 1])
        assert_o_close(o16[r0:r1].transpose(1, 0, 2), O_ref[b, :, :q_lens[b]], True, f"chunk {b} bf16")


def test_packed_rejects_seqlens_q_alongside(lib):
    import torch
    q = torch.zeros((10, 2, 128), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((1, 1, 16, 128), dtype=torch.bfloat16, device="cuda")
    cu = to_dev_i32(np.array([0, 10], dtype=np.int32))
    with pytest.raises(lib.AttnError) as e:
        lib.prefill(q, k, k, None, True, cu_seqlens_q=cu, max_seqlen_q=10, seqlens_q=to_dev_i32(np.array([10])))
    assert e.value.status == lib.ATTN_ERR_INVALID_ARG
