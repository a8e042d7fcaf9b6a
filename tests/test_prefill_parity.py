"""Prefill parity: the CUDA path (through the C ABI) against the fp64 oracle.

Sizes are small enough for the oracle to finish in seconds but span several
128-row / 128-key tiles with ragged tails; the full-size workloads are checked
on every row, in the launch configuration the bench times.
"""
import numpy as np
import pytest

from attention_tiled_exact_b200 import workloads as wl
from oracle import attention_ref as ref
from tests.helpers import assert_lse_close, assert_o_close, to_dev_bf16, to_dev_i32, to_f64

pytestmark = pytest.mark.gpu


def _run(lib, d, out_dtype=None, **kw):
    """One prefill call; its error word must stay clear (no block, length or
    timeout fault: a wait that ran out would still leave a correct-looking O)."""
    import torch
    q, k, v = to_dev_bf16(d["q"]), to_dev_bf16(d["k"]), to_dev_bf16(d["v"])
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = lib.prefill(q, k, v, d["scale"], d["causal"], out_dtype=out_dtype or torch.bfloat16, error_flags=flags,
                         **kw)
    status, word = lib.sync_error_flags(flags)
    assert word == 0 and status == lib.ATTN_OK, f"error word {word:#x}"
    return to_f64(o), to_f64(lse)


def _case(B, Hq, Hkv, Sq, Sk, D, causal, seed):
    cfg = wl.PrefillConfig("t", B, Hq, Hkv, Sq, Sk, D, causal, seed)
    return wl.make_prefill(cfg)


def test_tiny_config_with_lse(lib):
    """1 x 1 x 128 x 64, non-causal, scale 1/8, seed 0; O and the per-row LSE."""
    import torch
    d = wl.make_prefill(wl.TINY)
    O_ref, L_ref = ref.ref_attention(d["q"], d["k"], d["v"], d["scale"], d["causal"])
    for dt in (torch.bfloat16, torch.float32):
        o, lse = _run(lib, d, out_dtype=dt)
        assert_o_close(o, O_ref, dt == torch.bfloat16, "tiny")
        assert_lse_close(lse, L_ref, "tiny")


CASES = [
    # B, Hq, Hkv, Sq, Sk, D, causal
    (2, 8, 2, 300, 300, 128, True),     # GQA G=4, ragged third tile
    (1, 4, 1, 256, 256, 128, True),     # MQA, exact tiles
    (1, 2, 2, 257, 257, 128, True),     # MHA (G=1: row-block pairs, odd count of row blocks)
    (1, 6, 2, 200, 333, 64, False),     # G=3 (odd), non-causal, Sk != Sq
    (1, 16, 2, 130, 400, 128, True),    # G=8, bottom-right causal with Sq < Sk
    (1, 4, 2, 300, 100, 128, True),     # Sq > Sk: the first 200 rows see no key
    (2, 4, 4, 1, 700, 128, True),       # a single query row
    (1, 4, 2, 513, 129, 64, False),     # D=64, ragged keys
]


@pytest.mark.parametrize("B,Hq,Hkv,Sq,Sk,D,causal", CASES)
def test_prefill_matches_oracle(lib, B, Hq, Hkv, Sq, Sk, D, causal):
    import torch
    d = _case(B, Hq, Hkv, Sq, Sk, D, causal, seed=100 + Sq + Sk + D)
    O_ref, L_ref = ref.ref_attention(d["q"], d["k"], d["v"], d["scale"], causal)
    o, lse = _run(lib, d, out_dtype=torch.float32)
    assert_o_close(o, O_ref, False, "fp32 out")
    assert_lse_close(lse, L_ref, "lse")
    o16, lse16 = _run(lib, d)
    assert_o_close(o16, O_ref, True, "bf16 out")
    assert np.array_equal(lse16, lse)


def test_no_keys_gives_zero_and_minus_inf(lib):
    import torch
    d = _case(1, 2, 1, 64, 0, 128, False, seed=3)
    d["k"] = d["k"][:, :, :0]
    d["v"] = d["v"][:, :, :0]
    q = to_dev_bf16(d["q"])
    k = torch.empty((1, 1, 0, 128), dtype=torch.bfloat16, device="cuda")
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = lib.prefill(q, k, k, d["scale"], False, out_dtype=torch.float32, error_flags=flags)
    assert lib.sync_error_flags(flags) == (lib.ATTN_OK, 0)
    assert (to_f64(o) == 0).all() and np.isneginf(to_f64(lse)).all()


def test_strided_inputs(lib):
    """Q/K/V/O as [B, S, H, D] buffers viewed as [B, H, S, D] (non-contiguous strides)."""
    import torch
    d = _case(2, 4, 2, 190, 190, 128, True, seed=11)
    O_ref, L_ref = ref.ref_attention(d["q"], d["k"], d["v"], d["scale"], True)
    q = to_dev_bf16(np.ascontiguousarray(d["q"].transpose(0, 2, 1, 3))).transpose(1, 2)
    k = to_dev_bf16(np.ascontiguousarray(d["k"].transpose(0, 2, 1, 3))).transpose(1, 2)
    v = to_dev_bf16(np.ascontiguousarray(d["v"].transpose(0, 2, 1, 3))).transpose(1, 2)
    out = torch.empty((2, 190, 4, 128), dtype=torch.float32, device="cuda").transpose(1, 2)
    o, lse = lib.prefill(q, k, v, d["scale"], True, out=out)
    torch.cuda.synchronize()
    assert_o_close(to_f64(o), O_ref, False, "strided")
    assert_lse_close(to_f64(lse), L_ref, "strided")


@pytest.mark.parametrize("Hq,Hkv,D,causal", [
    (8, 2, 128, True),   # GQA G=4: two query heads per item
    (8, 2, 128, False),
    (6, 2, 64, True),    # G=3 (odd): two row blocks of one head per item, D=64
])
def test_dense_varlen_padded_batch(lib, Hq, Hkv, D, causal):
    """A padded dense batch with per-sequence query and key lengths: every sequence
    matches the oracle on its own slice (bottom-right causal alignment per
    sequence), rows past seqlens_q[b] are left untouched, a key length past the
    tensor is clamped to it, and a sequence without keys gets O = 0, LSE = -inf."""
    import torch
    B, Sq, Sk = 6, 300, 420
    d = _case(B, Hq, Hkv, Sq, Sk, D, causal, seed=77 + D + Hq)
    rng = np.random.default_rng(7)
    lq = rng.integers(1, Sq + 1, B).astype(np.int32)
    lk = rng.integers(1, Sk + 1, B).astype(np.int32)
    lq[0], lk[1], lk[2], lk[3] = Sq, Sk, 0, Sk + 50  # full rows, full keys, no keys, clamped keys
    q, k, v = to_dev_bf16(d["q"]), to_dev_bf16(d["k"]), to_dev_bf16(d["v"])
    out = torch.full((B, Hq, Sq, D), 7.0, dtype=torch.float32, device="cuda")
    lse = torch.full((B, Hq, Sq), 7.0, dtype=torch.float32, device="cuda")
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    lib.prefill(q, k, v, d["scale"], causal, out=out, lse=lse, seqlens_q=to_dev_i32(lq), seqlens_k=to_dev_i32(lk),
                error_flags=flags)
    assert lib.sync_error_flags(flags) == (lib.ATTN_OK, 0)
    o, l = to_f64(out), to_f64(lse)
    for b in range(B):
        nq, nk = int(lq[b]), min(int(lk[b]), Sk)
        O_ref, L_ref = ref.ref_attention(d["q"][b:b + 1, :, :nq], d["k"][b:b + 1, :, :nk], d["v"][b:b + 1, :, :nk],
                                         d["scale"], causal)
        assert_o_close(o[b:b + 1, :, :nq], O_ref, False, f"seq {b}")
        assert_lse_close(l[b:b + 1, :, :nq], L_ref, f"seq {b} lse")
        assert (o[b, :, nq:] == 7.0).all() and (l[b, :, nq:] == 7.0).all(), f"seq {b}: rows past seqlens_q written"


def test_repeated_calls_are_deterministic(lib):
    d = _case(1, 8, 2, 384, 384, 128, True, seed=5)
    o1, l1 = _run(lib, d)
    o2, l2 = _run(lib, d)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_error_word_stays_clear(lib):
    import torch
    d = _case(1, 4, 2, 256, 256, 128, True, seed=6)
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    q, k, v = to_dev_bf16(d["q"]), to_dev_bf16(d["k"]), to_dev_bf16(d["v"])
    lib.prefill(q, k, v, d["scale"], True, error_flags=flags)
    torch.cuda.synchronize()
    assert int(flags.item()) == 0


@pytest.mark.parametrize("cfg", [wl.CAUSAL_GQA_2K, wl.CAUSAL_GQA_16K], ids=lambda c: c.name)
def test_full_size_every_row(lib, cfg):
    """The full-size workloads in the bench's launch configuration (bf16 O and
    the LSE, one call), every row of every head against the oracle; then the
    same call with fp32 output under the strict 1e-2 bound."""
    import torch
    from tests.oracle_all_rows import prefill_all_rows
    d = wl.make_prefill(cfg)
    O_ref, L_ref = prefill_all_rows(d["q"], d["k"], d["v"], d["scale"], cfg.causal)
    o16, lse16 = _run(lib, d)
    assert_o_close(o16, O_ref, True, f"{cfg.name} bf16 out")
    assert_lse_close(lse16, L_ref, cfg.name)
    del o16
    o32, lse32 = _run(lib, d, out_dtype=torch.float32)
    assert_o_close(o32, O_ref, False, f"{cfg.name} fp32 out")
    assert np.array_equal(lse32, lse16)


@pytest.mark.gpu
@pytest.mark.parametrize("B,Hq,Hkv,S,Sk,D,causal,hpc,f32,with_lse", [
    (2, 8, 2, 300, 300, 128, True, 1, False, True),
    (3, 6, 3, 200, 450, 64, False, 0, True, True),
    (1, 4, 4, 129, 129, 128, True, 2, False, False),
    (2, 4, 2, 64, 0, 128, False, 1, True, True),
])
def test_prefill_from_host_matches_the_device_call(lib, B, Hq, Hkv, S, Sk, D, causal, hpc, f32, with_lse):
    """Chunked host<->device pipeline: the same bits as one device call (each
    chunk's items compute exactly what they compute in the whole call), and
    the oracle's values."""
    import torch
    d = wl.make_prefill(wl.PrefillConfig("from_host", B, Hq, Hkv, S, max(Sk, 1), D, causal, 81 + D))
    k_bits, v_bits = d["k"][:, :, :Sk], d["v"][:, :, :Sk]
    host = lambda bits: torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).pin_memory()
    hq, hk, hv = host(d["q"]), host(k_bits), host(v_bits)
    odt = torch.float32 if f32 else torch.bfloat16
    q, k, v = torch.empty_like(hq, device="cuda"), torch.empty_like(hk, device="cuda"), torch.empty_like(hv, device="cuda")
    o = torch.empty((B, Hq, S, D), dtype=odt, device="cuda")
    lse = torch.empty((B, Hq, S), dtype=torch.float32, device="cuda") if with_lse else None
    ho = torch.full((B, Hq, S, D), 7.0, dtype=odt).pin_memory()
    hl = torch.full((B, Hq, S), 7.0, dtype=torch.float32).pin_memory() if with_lse else None
    lib.prefill_from_host(hq, hk, hv, q, k, v, o, ho, lse, hl, d["scale"], causal, kv_heads_per_chunk=hpc)
    torch.cuda.synchronize()
    o_ref, l_ref = lib.prefill(hq.cuda(), hk.cuda(), hv.cuda(), d["scale"], causal, out_dtype=odt)
    torch.cuda.synchronize()
    assert torch.equal(ho, o_ref.cpu())
    if with_lse:
        assert torch.equal(hl, l_ref.cpu())
    O, L = ref.ref_attention(d["q"], k_bits, v_bits, d["scale"], causal)
    assert_o_close(ho.double().numpy(), O, not f32, "from host")
    if with_lse:
        assert_lse_close(hl.double().numpy(), L, "from host")

