"""Seeded random shapes for every call family, each against the fp64 oracle.

The hand-picked cases elsewhere target known edges; these draw batch sizes,
head counts (every supported group size), lengths (tile multiples, off-by-one
and ragged), head dims, masks, output dtypes and paged layouts at random from
a fixed seed, so that combinations nobody listed are exercised too. Sizes stay
small enough for the oracle (at most a few hundred rows per sequence)."""
import numpy as np
import pytest

from attention_tiled_exact_b200 import workloads as wl
from oracle import attention_ref as ref
from tests.helpers import assert_lse_close, assert_o_close, to_dev_bf16, to_dev_i32, to_f64

pytestmark = pytest.mark.gpu

N_CASES = 24


def _rng(i, kind):
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([20260, kind, i])))


def _length(r):
    # tile multiples, one off either side, or anything up to 600
    base = int(r.integers(1, 5)) * 128
    return int(r.choice([base - 1, base, base + 1, int(r.integers(1, 600))]))


@pytest.mark.parametrize("i", range(N_CASES))
def test_random_dense_prefill(lib, i):
    import torch
    r = _rng(i, 1)
    G = int(r.choice([1, 2, 3, 4, 8]))
    Hkv = int(r.integers(1, 4))
    B, D = int(r.integers(1, 4)), int(r.choice([64, 128]))
    Sq, Sk = _length(r), _length(r)
    causal = bool(r.integers(0, 2))
    f32 = bool(r.integers(0, 2))
    d = wl.make_prefill(wl.PrefillConfig(f"rand{i}", B, G * Hkv, Hkv, Sq, Sk, D, causal, 1000 + i))
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = lib.prefill(to_dev_bf16(d["q"]), to_dev_bf16(d["k"]), to_dev_bf16(d["v"]), d["scale"], causal,
                         out_dtype=torch.float32 if f32 else torch.bfloat16, error_flags=flags)
    assert lib.sync_error_flags(flags) == (lib.ATTN_OK, 0)
    O, L = ref.ref_attention(d["q"], d["k"], d["v"], d["scale"], causal)
    what = f"B{B} G{G} Hkv{Hkv} Sq{Sq} Sk{Sk} D{D} causal={causal}"
    assert_o_close(to_f64(o), O, not f32, what)
    assert_lse_close(to_f64(lse), L, what)


@pytest.mark.parametrize("i", range(N_CASES))
def test_random_paged_prefill_and_decode(lib, i):
    """Chunks of random lengths over random cached contexts (chunked prefill),
    then one decode row per sequence over the same pages."""
    import torch
    r = _rng(i, 2)
    G = int(r.choice([1, 2, 4, 8]))
    Hkv, B, D = int(r.integers(1, 3)), int(r.integers(1, 6)), 128
    q_lens = r.integers(1, 300, size=B).astype(np.int32)
    ctx = r.integers(0, 900, size=B).astype(np.int32)
    k_lens = (ctx + q_lens).astype(np.int32)
    pool = wl.make_paged_pool(2000 + i, k_lens, Hkv, D)
    Sq = int(q_lens.max())
    q = wl.normal_bf16(2000 + i, (B, G * Hkv, Sq, D), 30)
    scale = 1.0 / np.sqrt(D)
    kc, vc = to_dev_bf16(pool["k_pool"]), to_dev_bf16(pool["v_pool"])
    bt, lk = to_dev_i32(pool["block_table"]), to_dev_i32(k_lens)
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = lib.prefill_paged(to_dev_bf16(q), kc, vc, bt, lk, to_dev_i32(q_lens), scale, True,
                               out_dtype=torch.float32, error_flags=flags)
    assert lib.sync_error_flags(flags) == (lib.ATTN_OK, 0)
    O, L = ref.ref_prefill_paged(q, q_lens, pool["k_pool"], pool["v_pool"], pool["block_table"], k_lens, scale, True)
    o, lse = to_f64(o), to_f64(lse)
    for b in range(B):
        assert_o_close(o[b, :, :q_lens[b]], O[b, :, :q_lens[b]], False, f"case {i} chunk {b}")
        assert_lse_close(lse[b, :, :q_lens[b]], L[b, :, :q_lens[b]], f"case {i} chunk {b}")
    # decode: one query row per sequence over all of its cached keys
    qd = wl.normal_bf16(2000 + i, (B, G * Hkv, D), 31)
    splits = int(r.choice([0, 1, 3]))
    od, ld = lib.decode_paged(to_dev_bf16(qd), kc, vc, bt, lk, scale, num_splits=splits, out_dtype=torch.float32,
                              error_flags=flags)
    assert lib.sync_error_flags(flags) == (lib.ATTN_OK, 0)
    Od, Ld = ref.ref_decode_paged(qd, pool["k_pool"], pool["v_pool"], pool["block_table"], k_lens, scale)
    assert_o_close(to_f64(od), Od, False, f"case {i} decode")
    assert_lse_close(to_f64(ld), Ld, f"case {i} decode")


@pytest.mark.parametrize("i", range(12))
def test_random_backward(lib, i):
    import torch
    r = _rng(i, 3)
    G = int(r.choice([1, 2, 4]))
    Hkv, B, D = int(r.integers(1, 3)), int(r.integers(1, 3)), int(r.choice([64, 128]))
    S = _length(r) % 400 + 1
    causal = bool(r.integers(0, 2))
    d = wl.make_prefill(wl.PrefillConfig(f"randb{i}", B, G * Hkv, Hkv, S, S, D, causal, 3000 + i))
    do = wl.normal_bf16(3000 + i, d["q"].shape, 43)
    q, k, v = to_dev_bf16(d["q"]), to_dev_bf16(d["k"]), to_dev_bf16(d["v"])
    o, lse = lib.prefill(q, k, v, d["scale"], causal, out_dtype=torch.float32)
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    grads = lib.prefill_backward(q, k, v, o, lse, to_dev_bf16(do), d["scale"], causal, error_flags=flags)
    assert lib.sync_error_flags(flags) == (lib.ATTN_OK, 0)
    want = ref.ref_attention_backward(d["q"], d["k"], d["v"], do, d["scale"], causal)
    for name, g in zip(("dq", "dk", "dv"), grads):
        err = float(np.abs(to_f64(g) - want[name]).max())
        scale_ref = float(np.abs(want[name]).max())
        assert err <= 1e-2 * scale_ref, (i, name, err, scale_ref, B, G, Hkv, S, D, causal)
