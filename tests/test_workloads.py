"""Seeded generators: reproducible, the right shapes, valid block tables, sentinels in place."""
import numpy as np

from attention_tiled_exact_b200 import workloads as wl


def test_seeded_generation_is_reproducible_and_thread_independent():
    a = wl.normal_bf16(5, (3, 1 << 20), 1, threads=1)
    b = wl.normal_bf16(5, (3, 1 << 20), 1, threads=8)
    c = wl.normal_bf16(6, (3, 1 << 20), 1)
    assert a.dtype == np.uint16 and np.array_equal(a, b) and not np.array_equal(a, c)
    x = a.astype(np.uint32) << 16
    f = x.view(np.float32)
    assert abs(f.mean()) < 5e-3 and abs(f.std() - 1) < 5e-3


def test_bf16_rounding_is_nearest_even():
    x = np.array([1.0, 1 + 2 ** -8, 1 + 3 * 2 ** -8, 1 + 2 ** -8 + 2 ** -20, -0.0, np.inf], np.float32)
    bits = wl.f32_to_bf16_bits(x)
    assert list(bits) == [0x3F80, 0x3F80, 0x3F82, 0x3F81, 0x8000, 0x7F80]


def test_prefill_shapes():
    d = wl.make_prefill(wl.TINY)
    assert d["q"].shape == (1, 1, 128, 64) and d["k"].shape == (1, 1, 128, 64)
    assert d["scale"] == 0.125 and d["causal"] is False


def test_block_table_is_a_permutation_with_nan_sentinels():
    lens = np.array([1, 15, 16, 17, 100, 33])
    d = wl.make_paged_pool(3, lens, kv_heads=2, head_dim=8, spare_blocks=5)
    t, nb = d["block_table"], d["num_blocks"]
    nblk = (lens + 15) // 16
    used = np.concatenate([t[b, :n] for b, n in enumerate(nblk)])
    assert len(np.unique(used)) == nblk.sum() and nb == nblk.sum() + 5
    assert set(used) | set(d["spare_ids"].tolist()) == set(range(nb))
    assert (used < nb).all() and (t >= 0).all() and (t < nb).all()
    for pool in (d["k_pool"], d["v_pool"]):
        assert (pool[d["spare_ids"]] == wl.BF16_NAN).all()
        for b, L in enumerate(lens):
            last = t[b, (L - 1) // 16]
            assert (pool[last, :, L % 16 or 16:] == wl.BF16_NAN).all()
            assert (pool[last, :, : (L - 1) % 16 + 1] != wl.BF16_NAN).all()
        # unused table entries point at a NaN block
        for b, n in enumerate(nblk):
            assert (pool[t[b, n:]] == wl.BF16_NAN).all()


def test_identity_relayout_keeps_logical_tokens():
    lens = np.array([3, 40, 16])
    d = wl.make_paged_pool(4, lens, kv_heads=1, head_dim=4)
    newp, newt = wl.relayout_identity(d["k_pool"], d["block_table"], lens)
    for b, L in enumerate(lens):
        for tkn in range(L):
            assert np.array_equal(newp[newt[b, tkn // 16], :, tkn % 16],
                                  d["k_pool"][d["block_table"][b, tkn // 16], :, tkn % 16])


def test_mixed_batch_shapes():
    cfg = wl.MixedConfig("m", 2, 32, 0, 64, 3, 16, 80, 4, 2, 8, 9)
    d = wl.make_mixed(cfg)
    assert d["q_chunk"].shape == (2, 4, 32, 8) and d["q_dec"].shape == (3, 4, 8)
    assert len(d["kv_lens"]) == 5
    assert np.array_equal(d["kv_lens"][:2], d["ctx_chunk"] + 32)
    assert (d["ctx_dec"] >= 16).all() and (d["ctx_dec"] <= 80).all()


def test_pair_counts():
    assert wl.causal_pairs(2048, 2048, True) == 2048 * 2049 // 2
    assert wl.causal_pairs(4, 6, True) == 3 + 4 + 5 + 6
    assert wl.causal_pairs(6, 4, True) == 0 + 0 + 1 + 2 + 3 + 4
    assert wl.causal_pairs(5, 7, False) == 35


def test_e4m3_encoder_round_trips_every_finite_code():
    """Every finite E4M3 value encodes back to its own code (+0 / -0 kept apart)."""
    from oracle import attention_ref as ref
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    vals = ref.e4m3_bits_to_f64(codes)
    assert np.array_equal(wl.e4m3_codes(vals), codes)


def test_e4m3_encoder_rounding():
    """Ties go to the even code, values past 448 saturate, NaN stays NaN."""
    x = np.array([1.0625, 1.1875, 2.0 ** -10, 3 * 2.0 ** -10, 500.0, -1e9, np.nan])
    assert [int(c) for c in wl.e4m3_codes(x)] == [0x38, 0x3A, 0x00, 0x02, 0x7E, 0xFE, 0x7F]


def test_shared_prefix_tables_alias_the_prefix_blocks():
    cfg = wl.SharedPrefixConfig("t", 7, 8, 2, 64, 96, 0, 50, 3)
    d = wl.make_shared_prefix_decode(cfg)
    t, pb = d["block_table"], 96 // 16
    assert (t[:, :pb] == t[0, :pb]).all()  # every row lists the same prefix blocks first
    own = [t[b, pb:pb + (int(s) + 15) // 16] for b, s in enumerate(d["suffix_lens"])]
    ids = np.concatenate([t[0, :pb]] + own)
    assert len(set(ids.tolist())) == len(ids)  # prefix and own blocks are distinct
    assert not set(ids.tolist()) & set(d["spare_ids"].tolist())
    assert (d["kv_lens"] == 96 + d["suffix_lens"]).all()
    for pool in (d["k_pool"], d["v_pool"]):
        assert (pool[d["spare_ids"]] == wl.BF16_NAN).all()
        for b, L in enumerate(d["kv_lens"]):
            if L % 16:
                assert (pool[t[b, (L - 1) // 16], :, L % 16:] == wl.BF16_NAN).all()
