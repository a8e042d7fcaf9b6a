"""Pins for the fp64 oracle: things other than the oracle itself that fix its results.

* brute force: pure-Python ``math.fsum`` loops on tiny inputs;
* closed forms: hand-derived fixtures under tests/golden/, one key, causal
  row 0, zero query, constant V, one dominant key, rows of P sum to 1;
* a library special case: torch's fp64 CPU ``scaled_dot_product_attention``
  with K/V repeated for GQA;
* invariants: key/value permutation, split-and-combine, paged vs contiguous,
  GQA vs repeated MHA;
* planted mistakes: mutated copies of the formula are rejected by the pins.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from oracle import attention_ref as ref
from attention_tiled_exact_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "softmax_closed_form.json")


def _nested(x):
    return np.asarray(x, dtype=np.float64).tolist()


def _rand(rng, *shape):
    return rng.standard_normal(shape)


# ----------------------------------------------------------------------------
# brute force
# ----------------------------------------------------------------------------


@pytest.mark.parametrize("B,Hq,Hkv,Sq,Sk,D,causal", [
    (1, 1, 1, 4, 4, 8, False),
    (2, 4, 2, 5, 7, 8, False),
    (2, 4, 2, 5, 7, 8, True),     # bottom-right offset 2
    (1, 3, 1, 6, 6, 4, True),     # MQA
    (1, 2, 2, 7, 5, 4, True),     # Sq > Sk: first two rows see no key
    (1, 4, 4, 1, 9, 8, False),    # decode-like
])
def test_numpy_oracle_matches_brute_force(B, Hq, Hkv, Sq, Sk, D, causal):
    rng = np.random.default_rng(1234 + Sq * Sk + D)
    q, k, v = _rand(rng, B, Hq, Sq, D), _rand(rng, B, Hkv, Sk, D), _rand(rng, B, Hkv, Sk, D)
    scale = 0.37
    O, L = ref.ref_attention(q, k, v, scale, causal)
    Ob, Lb = oracle.brute_attention(_nested(q), _nested(k), _nested(v), scale, causal)
    np.testing.assert_allclose(O, np.array(Ob), rtol=0, atol=1e-12)
    Lb = np.array(Lb)
    assert np.array_equal(np.isinf(L), np.isinf(Lb))
    fin = np.isfinite(Lb)
    np.testing.assert_allclose(L[fin], Lb[fin], rtol=0, atol=1e-12)
    if Sq > Sk and causal:
        assert np.all(O[:, :, : Sq - Sk] == 0) and np.all(np.isneginf(L[:, :, : Sq - Sk]))


# ----------------------------------------------------------------------------
# closed forms
# ----------------------------------------------------------------------------


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


@pytest.mark.parametrize("case", _golden()["attention"], ids=lambda c: c["name"])
def test_golden_attention_closed_form(case):
    O, L = ref.ref_attention(np.array(case["q"]), np.array(case["k"]), np.array(case["v"]),
                             case["scale"], case["causal"])
    np.testing.assert_allclose(O, np.array(case["expected_o"]), rtol=0, atol=1e-13)
    np.testing.assert_allclose(L, np.array(case["expected_lse"]), rtol=0, atol=1e-13)


@pytest.mark.parametrize("case", _golden()["combine"], ids=lambda c: c["name"])
def test_golden_combine_closed_form(case):
    lse = np.array([[float(x) for x in row] for row in case["part_lse"]])
    O, L = ref.combine_partials(np.array(case["part_o"]), lse)
    np.testing.assert_allclose(O, np.array(case["expected_o"]), rtol=0, atol=1e-13)
    np.testing.assert_allclose(L, np.array(case["expected_lse"]), rtol=0, atol=1e-13)


def test_single_key_returns_its_value():
    rng = np.random.default_rng(0)
    q, k, v = _rand(rng, 1, 2, 3, 16), _rand(rng, 1, 2, 1, 16), _rand(rng, 1, 2, 1, 16)
    O, L = ref.ref_attention(q, k, v, 0.25, False)
    np.testing.assert_array_equal(O, np.broadcast_to(v, O.shape))
    np.testing.assert_allclose(L[0, :, :], 0.25 * np.einsum("hsd,hd->hs", q[0], k[0, :, 0]),
                               atol=1e-14)


def test_causal_row0_is_first_value_row():
    rng = np.random.default_rng(1)
    q, k, v = _rand(rng, 2, 4, 9, 8), _rand(rng, 2, 2, 9, 8), _rand(rng, 2, 2, 9, 8)
    O, L = ref.ref_attention(q, k, v, 0.5, True)
    for h in range(4):
        np.testing.assert_array_equal(O[:, h, 0], v[:, h // 2, 0])
        np.testing.assert_allclose(L[:, h, 0], 0.5 * np.einsum("bd,bd->b", q[:, h, 0], k[:, h // 2, 0]),
                                   atol=1e-14)


def test_zero_query_gives_mean_of_visible_values():
    rng = np.random.default_rng(2)
    Sq, Sk = 5, 8
    q = np.zeros((1, 2, Sq, 8))
    k, v = _rand(rng, 1, 1, Sk, 8), _rand(rng, 1, 1, Sk, 8)
    O, L = ref.ref_attention(q, k, v, 1.0, True)
    for i in range(Sq):
        nvis = i + (Sk - Sq) + 1
        np.testing.assert_allclose(O[0, :, i], np.broadcast_to(v[0, 0, :nvis].mean(0), (2, 8)), atol=1e-14)
        np.testing.assert_allclose(L[0, :, i], math.log(nvis), atol=1e-14)


def test_constant_values_are_returned():
    rng = np.random.default_rng(3)
    q, k = _rand(rng, 1, 4, 6, 8), _rand(rng, 1, 2, 10, 8)
    row = _rand(rng, 8)
    v = np.broadcast_to(row, (1, 2, 10, 8)).copy()
    for causal in (False, True):
        O, _ = ref.ref_attention(q, k, v, 0.3, causal)
        np.testing.assert_allclose(O, np.broadcast_to(row, O.shape), atol=1e-14)


def test_dominant_key_selects_its_value():
    rng = np.random.default_rng(4)
    D = 8
    k = _rand(rng, 1, 1, 12, D) * 0.01
    q = np.zeros((1, 1, 1, D))
    q[0, 0, 0, 0] = 1.0
    k[0, 0, 7, 0] = 2000.0
    v = _rand(rng, 1, 1, 12, D)
    O, L = ref.ref_attention(q, k, v, 1.0, False)
    np.testing.assert_allclose(O[0, 0, 0], v[0, 0, 7], atol=1e-12)
    assert abs(L[0, 0, 0] - 2000.0) < 1e-9


def test_softmax_rows_sum_to_one():
    rng = np.random.default_rng(5)
    q, k = _rand(rng, 6, 8), _rand(rng, 11, 8)
    pos = ref.causal_positions(6, 11)
    for qp in (None, pos):
        p, m, l = ref.softmax_probs(q, k, 0.7, qp)
        np.testing.assert_allclose((p / l[:, None]).sum(axis=1), 1.0, atol=1e-14)
        assert np.all(p <= 1.0) and np.allclose(p.max(axis=1), 1.0)


# ----------------------------------------------------------------------------
# a library routine as a special case
# ----------------------------------------------------------------------------


@pytest.mark.parametrize("Sq,Sk,causal", [(33, 33, False), (33, 33, True), (17, 40, True), (1, 50, False)])
def test_matches_torch_sdpa_fp64(Sq, Sk, causal):
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(6 + Sq + Sk)
    B, Hq, Hkv, D = 2, 8, 2, 16
    q, k, v = _rand(rng, B, Hq, Sq, D), _rand(rng, B, Hkv, Sk, D), _rand(rng, B, Hkv, Sk, D)
    scale = 1 / math.sqrt(D)
    O, L = ref.ref_attention(q, k, v, scale, causal)
    G = Hq // Hkv
    tq = torch.from_numpy(q)
    tk = torch.from_numpy(k).repeat_interleave(G, dim=1)
    tv = torch.from_numpy(v).repeat_interleave(G, dim=1)
    mask = None
    if causal:
        i = torch.arange(Sq)[:, None] + (Sk - Sq)
        j = torch.arange(Sk)[None, :]
        mask = j <= i
    To = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask, scale=scale)
    np.testing.assert_allclose(O, To.numpy(), rtol=0, atol=1e-12)
    s = torch.einsum("bhqd,bhkd->bhqk", tq, tk) * scale
    if mask is not None:
        s = s.masked_fill(~mask, float("-inf"))
    np.testing.assert_allclose(L, torch.logsumexp(s, dim=-1).numpy(), rtol=0, atol=1e-12)


# ----------------------------------------------------------------------------
# invariants
# ----------------------------------------------------------------------------


def test_noncausal_invariant_to_key_permutation():
    rng = np.random.default_rng(7)
    q, k, v = _rand(rng, 1, 4, 9, 8), _rand(rng, 1, 2, 13, 8), _rand(rng, 1, 2, 13, 8)
    perm = rng.permutation(13)
    O1, L1 = ref.ref_attention(q, k, v, 0.4, False)
    O2, L2 = ref.ref_attention(q, k[:, :, perm], v[:, :, perm], 0.4, False)
    np.testing.assert_allclose(O1, O2, atol=1e-13)
    np.testing.assert_allclose(L1, L2, atol=1e-13)


@pytest.mark.parametrize("cuts", [[0, 5, 13], [0, 1, 2, 13], [0, 4, 4, 9, 13], [0, 13]])
def test_split_combine_equals_single_pass(cuts):
    rng = np.random.default_rng(8)
    q, k, v = _rand(rng, 3, 8), _rand(rng, 13, 8), _rand(rng, 13, 8)
    O, L = ref.attention_rows(q, k, v, 0.6)
    parts_o, parts_l = [], []
    for a, b in zip(cuts[:-1], cuts[1:]):
        o, l = ref.attention_rows(q, k[a:b], v[a:b], 0.6)
        parts_o.append(o)
        parts_l.append(l)
    Oc, Lc = ref.combine_partials(np.stack(parts_o), np.stack(parts_l))
    np.testing.assert_allclose(Oc, O, atol=1e-13)
    np.testing.assert_allclose(Lc, L, atol=1e-13)


def test_combine_respects_splits_per_row():
    rng = np.random.default_rng(9)
    po, pl = _rand(rng, 4, 3, 8), _rand(rng, 4, 3)
    pl[2:, 0] = np.nan  # never read for row 0
    O, L = ref.combine_partials(po, pl, splits_per_row=[2, 4, 1])
    O0, L0 = ref.combine_partials(po[:2, :1], pl[:2, :1])
    np.testing.assert_allclose(O[0], O0[0], atol=1e-14)
    np.testing.assert_allclose(L[2], pl[0, 2], atol=1e-14)
    np.testing.assert_allclose(O[2], po[0, 2], atol=1e-14)


def test_paged_equals_contiguous():
    lens = np.array([1, 16, 17, 40, 5])
    d = wl.make_paged_pool(11, lens, kv_heads=2, head_dim=8)
    rng = np.random.default_rng(10)
    q = wl.normal_bf16(11, (len(lens), 4, 8), 5)
    O, L = ref.ref_decode_paged(q, d["k_pool"], d["v_pool"], d["block_table"], lens, 0.35)
    for b, n in enumerate(lens):
        for kvh in range(2):
            kk = np.stack([d["k_pool"][d["block_table"][b, t // 16], kvh, t % 16] for t in range(n)])
            vv = np.stack([d["v_pool"][d["block_table"][b, t // 16], kvh, t % 16] for t in range(n)])
            for h in (2 * kvh, 2 * kvh + 1):
                o, l = ref.attention_rows(ref.bf16_bits_to_f64(q[b, h][None]), kk, vv, 0.35)
                np.testing.assert_allclose(O[b, h], o[0], atol=1e-13)
                np.testing.assert_allclose(L[b, h], l[0], atol=1e-13)
    assert np.isfinite(O).all() and np.isfinite(L).all()  # the NaN sentinels were never read
    del rng


def test_paged_prefill_equals_dense_on_gathered_keys():
    ctx = np.array([0, 20, 3])
    qlen = 6
    lens = ctx + qlen
    d = wl.make_paged_pool(12, lens, kv_heads=1, head_dim=8)
    q = wl.normal_bf16(12, (3, 2, qlen, 8), 5)
    O, L = ref.ref_prefill_paged(q, [qlen] * 3, d["k_pool"], d["v_pool"], d["block_table"], lens, 0.3, True)
    for b in range(3):
        kk = ref.gather_paged(d["k_pool"], d["block_table"][b], int(lens[b]), 0)[None, None]
        vv = ref.gather_paged(d["v_pool"], d["block_table"][b], int(lens[b]), 0)[None, None]
        Od, Ld = ref.ref_attention(q[b:b + 1], kk, vv, 0.3, True)
        np.testing.assert_allclose(O[b], Od[0], atol=1e-13)
        np.testing.assert_allclose(L[b], Ld[0], atol=1e-13)


def test_gqa_equals_repeated_mha():
    rng = np.random.default_rng(13)
    q, k, v = _rand(rng, 2, 6, 7, 8), _rand(rng, 2, 2, 7, 8), _rand(rng, 2, 2, 7, 8)
    O1, L1 = ref.ref_attention(q, k, v, 0.5, True)
    O2, L2 = ref.ref_attention(q, np.repeat(k, 3, axis=1), np.repeat(v, 3, axis=1), 0.5, True)
    np.testing.assert_array_equal(O1, O2)
    np.testing.assert_array_equal(L1, L2)


def test_rows_subset_matches_full():
    rng = np.random.default_rng(14)
    q, k, v = _rand(rng, 2, 4, 9, 8), _rand(rng, 2, 2, 12, 8), _rand(rng, 2, 2, 12, 8)
    O, L = ref.ref_attention(q, k, v, 0.5, True)
    rows = [(0, 0, 0), (1, 3, 8), (1, 2, 4)]
    Or, Lr = ref.ref_attention(q, k, v, 0.5, True, rows=rows)
    for n, (b, h, i) in enumerate(rows):
        np.testing.assert_allclose(Or[n], O[b, h, i], atol=1e-14)
        np.testing.assert_allclose(Lr[n], L[b, h, i], atol=1e-14)


def test_bf16_decode_is_exact():
    bits = np.array([0x3F80, 0xC020, 0x0001, 0x7F7F, 0x8000], dtype=np.uint16)
    vals = ref.bf16_bits_to_f64(bits)
    assert vals[0] == 1.0 and vals[1] == -2.5 and vals[2] == 2.0 ** -133
    assert vals[3] == (2 - 2 ** -7) * 2.0 ** 127 and vals[4] == 0.0 and math.copysign(1, vals[4]) < 0


# ----------------------------------------------------------------------------
# planted mistakes: each mutant of the formula must fail a pin
# ----------------------------------------------------------------------------


def _candidate(q, k, v, scale, causal, mutant):
    """A copy of the definition with one planted mistake (or none)."""
    B, Hq, Sq, D = q.shape
    Hkv, Sk = k.shape[1], k.shape[2]
    G = Hq // Hkv
    O = np.zeros((B, Hq, Sq, D))
    L = np.zeros((B, Hq, Sq))
    for b in range(B):
        for h in range(Hq):
            kvh = (h % Hkv) if mutant == "gqa_modulo" else h // G
            s = (1.0 if mutant == "no_scale" else scale) * (q[b, h] @ k[b, kvh].T)
            if causal:
                i = np.arange(Sq)[:, None] + (0 if mutant == "top_left" else Sk - Sq)
                j = np.arange(Sk)[None, :]
                s = np.where((j < i) if mutant == "strict_mask" else (j <= i), s, -np.inf)
            m = s.max(1)
            p = np.exp(s - m[:, None])
            l = p.sum(1)
            vv = v[b, kvh].T.T if mutant != "transposed_v" else v[b, kvh][::-1]
            O[b, h] = (p @ vv) / (l[:, None] if mutant != "no_norm" else 1.0)
            L[b, h] = (0 if mutant == "lse_no_max" else m) + np.log(l)
    return O, L


@pytest.mark.parametrize("mutant", ["no_scale", "top_left", "strict_mask", "gqa_modulo",
                                    "transposed_v", "no_norm", "lse_no_max"])
def test_pins_reject_planted_mistakes(mutant):
    rng = np.random.default_rng(15)
    q, k, v = _rand(rng, 1, 4, 5, 4), _rand(rng, 1, 2, 7, 4), _rand(rng, 1, 2, 7, 4)
    Ob, Lb = oracle.brute_attention(_nested(q), _nested(k), _nested(v), 0.5, True)
    Oc, Lc = _candidate(q, k, v, 0.5, True, None)
    assert np.allclose(Oc, Ob, atol=1e-12) and np.allclose(Lc, Lb, atol=1e-12)
    Om, Lm = _candidate(q, k, v, 0.5, True, mutant)
    assert not (np.allclose(Om, Ob, atol=1e-6) and np.allclose(Lm, Lb, atol=1e-6))


# ----------------------------------------------------------------------------
# FP8 E4M3 cache: the format decode and the decode oracle over it
# ----------------------------------------------------------------------------


@pytest.mark.parametrize("code,value", [
    (0x00, 0.0), (0x38, 1.0), (0x40, 2.0), (0x3C, 1.5), (0x3F, 1.875), (0x7E, 448.0), (0xFE, -448.0),
    (0x77, 240.0), (0x08, 2.0 ** -6), (0x07, 7 * 2.0 ** -9), (0x01, 2.0 ** -9), (0xB8, -1.0), (0x30, 0.5),
])
def test_e4m3_decode_hand_codes(code, value):
    """Values worked out by hand from the format: exponent bias 7, 3 mantissa bits, subnormals at e = 0."""
    assert ref.e4m3_bits_to_f64(np.array([code], dtype=np.uint8))[0] == value


def test_e4m3_decode_matches_torch_on_every_code():
    torch = pytest.importorskip("torch")
    codes = np.arange(256, dtype=np.uint8)
    t = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    o = ref.e4m3_bits_to_f64(codes)
    assert np.array_equal(np.isnan(t), np.isnan(o)) and np.isnan(o).sum() == 2  # 0x7F and 0xFF
    assert np.array_equal(t[~np.isnan(t)], o[~np.isnan(o)])
    assert np.array_equal(np.signbit(t[~np.isnan(t)]), np.signbit(o[~np.isnan(o)]))


def test_fp8_decode_oracle_matches_brute_force():
    """Tiny FP8 cache: the paged FP8 decode oracle against math.fsum loops on the
    hand-gathered, hand-dequantised keys and values of every sequence."""
    cfg = wl.DecodeConfig("t", 3, 4, 2, 8, 1, 1, 21)
    lens = np.array([5, 17, 1], dtype=np.int32)
    d = wl.make_decode_fp8(cfg, kv_lens=lens)
    O, L = ref.ref_decode_paged_fp8(d["q"], d["k_pool"], d["v_pool"], d["k_scale"], d["v_scale"],
                                    d["block_table"], lens, d["scale"])
    qf = ref.bf16_bits_to_f64(d["q"])

    def dequant(code, s):  # sign, exponent bias 7, 3 mantissa bits
        c = int(code)
        sign = -1.0 if c & 0x80 else 1.0
        e, m = (c >> 3) & 15, c & 7
        return sign * s * ((m / 8.0) * 2.0 ** -6 if e == 0 else (1 + m / 8.0) * 2.0 ** (e - 7))

    for b, Lb in enumerate(lens):
        toks = [(d["block_table"][b][t // 16], t % 16) for t in range(Lb)]
        for h in range(4):
            kvh = h // 2
            kk = [[[dequant(d["k_pool"][p, kvh, s, j], d["k_scale"]) for j in range(8)] for p, s in toks]]
            vv = [[[dequant(d["v_pool"][p, kvh, s, j], d["v_scale"]) for j in range(8)] for p, s in toks]]
            Ob, Lbr = oracle.brute_attention([[[list(qf[b, h])]]], [kk], [vv], d["scale"], False)
            assert np.allclose(O[b, h], Ob[0][0][0], atol=1e-12) and abs(L[b, h] - Lbr[0][0][0]) < 1e-12


def test_decode_over_a_shared_prefix_is_the_merge_of_prefix_and_suffix():
    """Attention over prefix + own keys equals the log-sum-exp merge of the
    attention over each part: the identity the shared-prefix decode relies on,
    checked with the oracle's decode on the full, the prefix-only and the
    suffix-only tables."""
    cfg = wl.SharedPrefixConfig("t", 5, 4, 2, 32, 48, 0, 40, 7)
    d = wl.make_shared_prefix_decode(cfg)
    t, pb = d["block_table"], 3
    O, L = ref.ref_decode_paged(d["q"], d["k_pool"], d["v_pool"], t, d["kv_lens"], d["scale"])
    Op, Lp = ref.ref_decode_paged(d["q"], d["k_pool"], d["v_pool"], t[:, :pb], np.full(5, 48), d["scale"])
    Os, Ls = ref.ref_decode_paged(d["q"], d["k_pool"], d["v_pool"], t[:, pb:], d["suffix_lens"], d["scale"])
    Om, Lm = ref.combine_partials(np.stack([Op.reshape(20, 32), Os.reshape(20, 32)]),
                                  np.stack([Lp.reshape(20), Ls.reshape(20)]))
    assert np.abs(Om - O.reshape(20, 32)).max() < 1e-12 and np.abs(Lm - L.reshape(20)).max() < 1e-12
    assert np.isneginf(Ls.reshape(20)[np.repeat(d["suffix_lens"] == 0, 4)]).all()


# ----------------------------------------------------------------------------
# backward: gradients of the definition
# ----------------------------------------------------------------------------


def _autograd_backward(q, k, v, do, scale, causal):
    """dQ, dK, dV by torch autograd in fp64 through the forward written with
    torch ops (K/V repeated over each query-head group; masked softmax)."""
    torch = pytest.importorskip("torch")
    G = q.shape[1] // k.shape[1]
    tq, tk, tv = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    kk, vv = tk.repeat_interleave(G, dim=1), tv.repeat_interleave(G, dim=1)
    s = scale * tq @ kk.transpose(-1, -2)
    Sq, Sk = q.shape[2], k.shape[2]
    if causal:
        vis = torch.arange(Sk)[None, :] <= (torch.arange(Sq) + (Sk - Sq))[:, None]
        s = s.masked_fill(~vis, float("-inf"))
    p = torch.softmax(s, dim=-1).nan_to_num(0.0)  # rows with no key: P = 0
    o = p @ vv
    o.backward(torch.tensor(do, dtype=torch.float64))
    return tq.grad.numpy(), tk.grad.numpy(), tv.grad.numpy(), o.detach().numpy()


@pytest.mark.parametrize("Hq,Hkv,Sq,Sk,causal", [
    (2, 2, 6, 6, False), (4, 2, 5, 9, True), (8, 2, 9, 4, True), (3, 1, 7, 7, True), (4, 4, 1, 12, False),
])
def test_backward_matches_torch_autograd(Hq, Hkv, Sq, Sk, causal):
    rng = np.random.default_rng(400 + Hq * Sq + Sk)
    q, do = _rand(rng, 2, Hq, Sq, 8), _rand(rng, 2, Hq, Sq, 8)
    k, v = _rand(rng, 2, Hkv, Sk, 8), _rand(rng, 2, Hkv, Sk, 8)
    r = ref.ref_attention_backward(q, k, v, do, 0.4, causal)
    dq, dk, dv, o = _autograd_backward(q, k, v, do, 0.4, causal)
    for name, a, b in (("dq", r["dq"], dq), ("dk", r["dk"], dk), ("dv", r["dv"], dv), ("o", r["o"], o)):
        assert np.abs(a - b).max() < 1e-12, name
    assert np.abs(r["delta"] - (do * o).sum(-1)).max() < 1e-12


def test_backward_matches_finite_differences():
    """Directional derivatives of f = sum(O * dO) by central differences."""
    rng = np.random.default_rng(410)
    q, do = _rand(rng, 1, 4, 5, 6), _rand(rng, 1, 4, 5, 6)
    k, v = _rand(rng, 1, 2, 7, 6), _rand(rng, 1, 2, 7, 6)
    r = ref.ref_attention_backward(q, k, v, do, 0.6, True)
    eps = 1e-5
    for name, x in (("q", q), ("k", k), ("v", v)):
        u = rng.standard_normal(x.shape)
        args_p = dict(q=q, k=k, v=v)
        args_m = dict(q=q, k=k, v=v)
        args_p[name] = x + eps * u
        args_m[name] = x - eps * u
        fp = (ref.ref_attention(args_p["q"], args_p["k"], args_p["v"], 0.6, True)[0] * do).sum()
        fm = (ref.ref_attention(args_m["q"], args_m["k"], args_m["v"], 0.6, True)[0] * do).sum()
        fd = (fp - fm) / (2 * eps)
        assert abs(fd - (r["d" + name] * u).sum()) < 1e-7 * max(1.0, abs(fd)), name


def test_backward_closed_forms():
    rng = np.random.default_rng(420)
    # one key: O = v everywhere, so dV = sum of dO over the group's rows and dQ = dK = 0
    q, do = _rand(rng, 1, 4, 6, 8), _rand(rng, 1, 4, 6, 8)
    k, v = _rand(rng, 1, 2, 1, 8), _rand(rng, 1, 2, 1, 8)
    r = ref.ref_attention_backward(q, k, v, do, 0.5, False)
    assert np.abs(r["dq"]).max() < 1e-15 and np.abs(r["dk"]).max() < 1e-15
    for kvh in range(2):
        assert np.allclose(r["dv"][0, kvh, 0], do[0, 2 * kvh:2 * kvh + 2].sum(axis=(0, 1)), atol=1e-12)
    # zero queries: uniform P over the visible keys and dK = scale * dS^T Q = 0
    q0 = np.zeros((1, 2, 5, 8))
    k, v, do = _rand(rng, 1, 2, 5, 8), _rand(rng, 1, 2, 5, 8), _rand(rng, 1, 2, 5, 8)
    r = ref.ref_attention_backward(q0, k, v, do, 0.5, True)
    assert np.abs(r["dk"]).max() == 0.0
    n_vis = np.arange(1, 6)
    for h in range(2):
        want = np.stack([(do[0, h, j:] / n_vis[j:, None]).sum(0) for j in range(5)])
        assert np.allclose(r["dv"][0, h], want, atol=1e-12)


def test_backward_gqa_is_repeated_mha_summed():
    rng = np.random.default_rng(430)
    q, do = _rand(rng, 1, 6, 5, 4), _rand(rng, 1, 6, 5, 4)
    k, v = _rand(rng, 1, 2, 8, 4), _rand(rng, 1, 2, 8, 4)
    r = ref.ref_attention_backward(q, k, v, do, 0.7, True)
    m = ref.ref_attention_backward(q, np.repeat(k, 3, axis=1), np.repeat(v, 3, axis=1), do, 0.7, True)
    assert np.allclose(r["dq"], m["dq"], atol=1e-13)
    assert np.allclose(r["dk"], m["dk"].reshape(1, 2, 3, 8, 4).sum(2), atol=1e-13)
    assert np.allclose(r["dv"], m["dv"].reshape(1, 2, 3, 8, 4).sum(2), atol=1e-13)


def _candidate_backward(q, k, v, do, scale, causal, mutant):
    """A copy of the gradient formulas with one planted mistake (or none)."""
    B, Hq, Sq, D = q.shape
    Hkv, Sk = k.shape[1], k.shape[2]
    G = Hq // Hkv
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    for b in range(B):
        for h in range(Hq):
            kvh = h // G
            s = scale * q[b, h] @ k[b, kvh].T
            if causal:
                vis = np.arange(Sk)[None, :] <= (np.arange(Sq) + Sk - Sq)[:, None]
                s = np.where(vis, s, -np.inf)
            p = np.exp(s - s.max(1, keepdims=True))
            p /= p.sum(1, keepdims=True)
            dP = do[b, h] @ v[b, kvh].T
            delta = (p * dP).sum(1, keepdims=True)
            if mutant == "no_delta":
                delta = 0.0
            dS = p * (dP + delta) if mutant == "delta_sign" else p * (dP - delta)
            dv[b, kvh] += (p @ do[b, h]) if mutant == "dv_untransposed" else (p.T @ do[b, h])
            dq[b, h] = (1.0 if mutant == "dq_no_scale" else scale) * dS @ k[b, kvh]
            dk[b, kvh] += scale * ((dS @ q[b, h]) if mutant == "dk_untransposed" else (dS.T @ q[b, h]))
    return dq, dk, dv


@pytest.mark.parametrize("mutant", ["no_delta", "delta_sign", "dv_untransposed", "dq_no_scale", "dk_untransposed"])
def test_backward_pins_reject_planted_mistakes(mutant):
    rng = np.random.default_rng(440)
    q, do = _rand(rng, 1, 4, 6, 4), _rand(rng, 1, 4, 6, 4)
    k, v = _rand(rng, 1, 2, 6, 4), _rand(rng, 1, 2, 6, 4)
    want = _autograd_backward(q, k, v, do, 0.5, True)[:3]
    good = _candidate_backward(q, k, v, do, 0.5, True, None)
    assert all(np.allclose(a, b, atol=1e-12) for a, b in zip(good, want))
    bad = _candidate_backward(q, k, v, do, 0.5, True, mutant)
    assert not all(np.allclose(a, b, atol=1e-6) for a, b in zip(bad, want))


# ----------------------------------------------------------------------------
# block-sparse (BSR) attention
# ----------------------------------------------------------------------------


def test_block_sparse_with_every_block_is_dense():
    rng = np.random.default_rng(450)
    q, k, v = _rand(rng, 4, 37, 8), _rand(rng, 2, 50, 8), _rand(rng, 2, 50, 8)
    n_rb, n_cb = 5, 4  # row blocks of 8, column blocks of 16 (the last one ragged)
    indptr = np.arange(n_rb + 1) * n_cb
    indices = np.tile(np.arange(n_cb)[::-1], n_rb)  # every block, in reverse order
    O, L = ref.ref_block_sparse_attention(q, k, v, indptr, indices, 8, 16, 0.3)
    Od, Ld = ref.ref_attention(q[None], k[None], v[None], 0.3, False)
    assert np.abs(O - Od[0]).max() < 1e-12 and np.abs(L - Ld[0]).max() < 1e-12


def test_block_sparse_is_dense_attention_over_the_gathered_blocks():
    """Each query block against the concatenation of its listed key blocks,
    through the brute-force fsum definition (a different computation)."""
    rng = np.random.default_rng(451)
    q, k, v = _rand(rng, 2, 10, 4), _rand(rng, 1, 40, 4), _rand(rng, 1, 40, 4)
    indptr = np.array([0, 2, 2, 5])  # row block 1 sees nothing
    indices = np.array([2, 0, 1, 2, 0])
    O, L = ref.ref_block_sparse_attention(q, k, v, indptr, indices, 4, 16, 0.5)
    for r in range(3):
        rows = slice(4 * r, min(4 * r + 4, 10))
        cols = indices[indptr[r]:indptr[r + 1]]
        if len(cols) == 0:
            assert (O[:, rows] == 0).all() and np.isneginf(L[:, rows]).all()
            continue
        keys = np.concatenate([np.arange(c * 16, min(c * 16 + 16, 40)) for c in cols])
        Ob, Lb = oracle.brute_attention(_nested(q[None, :, rows]), _nested(k[None][:, :, keys]),
                                        _nested(v[None][:, :, keys]), 0.5, False)
        assert np.abs(O[:, rows] - np.asarray(Ob)[0]).max() < 1e-12
        assert np.abs(L[:, rows] - np.asarray(Lb)[0]).max() < 1e-12


def test_block_sparse_via_block_tables_is_the_bsr_definition():
    """The paged-prefill oracle over the per-query-block tables of
    workloads.bsr_tables (the form the kernels take) equals the BSR
    definition, including a listed partial last key block."""
    d = wl.make_block_sparse(72, 4, 2, 70, 200, 8, 16, 3, 2)
    table, lens = wl.bsr_tables(d, 200)
    n_rb = len(d["indptr"]) - 1
    qb = np.zeros((n_rb, 4, 16, 8), dtype=np.uint16)
    q_lens = np.zeros(n_rb, dtype=np.int32)
    for r in range(n_rb):
        rows = d["q"][:, 16 * r:16 * r + 16]
        qb[r, :, :rows.shape[1]] = rows
        q_lens[r] = rows.shape[1]
    O, L = ref.ref_prefill_paged(qb, q_lens, d["k_pool"], d["v_pool"], table, lens, 0.35, False)
    Ob, Lb = ref.ref_block_sparse_attention(d["q"], d["k"], d["v"], d["indptr"], d["indices"], 16, 16, 0.35)
    got = np.concatenate([O[r, :, :q_lens[r]] for r in range(n_rb)], axis=1)
    got_l = np.concatenate([L[r, :, :q_lens[r]] for r in range(n_rb)], axis=1)
    assert (200 - 1) // 16 in set(d["indices"].tolist())  # the partial block is exercised
    assert np.abs(got - Ob).max() < 1e-12 and np.abs(got_l - Lb).max() < 1e-12


# ----------------------------------------------------------------------------
# randomised shapes (hypothesis): backward and block-sparse pins
# ----------------------------------------------------------------------------

from hypothesis import given, settings, strategies as st  # noqa: E402


@settings(max_examples=25, deadline=None)
@given(G=st.sampled_from([1, 2, 3]), Hkv=st.integers(1, 2), Sq=st.integers(1, 9), Sk=st.integers(1, 9),
       D=st.sampled_from([2, 5]), causal=st.booleans(), seed=st.integers(0, 10_000))
def test_backward_random_shapes_match_autograd(G, Hkv, Sq, Sk, D, causal, seed):
    rng = np.random.default_rng(seed)
    q, do = _rand(rng, 1, G * Hkv, Sq, D), _rand(rng, 1, G * Hkv, Sq, D)
    k, v = _rand(rng, 1, Hkv, Sk, D), _rand(rng, 1, Hkv, Sk, D)
    r = ref.ref_attention_backward(q, k, v, do, 0.7, causal)
    dq, dk, dv, _ = _autograd_backward(q, k, v, do, 0.7, causal)
    assert np.abs(r["dq"] - dq).max() < 1e-11
    assert np.abs(r["dk"] - dk).max() < 1e-11
    assert np.abs(r["dv"] - dv).max() < 1e-11


@settings(max_examples=25, deadline=None)
@given(Sq=st.integers(1, 20), Sk=st.integers(1, 40), rb=st.sampled_from([1, 4, 8]), seed=st.integers(0, 10_000))
def test_block_sparse_random_patterns_match_gathered_dense(Sq, Sk, rb, seed):
    """Random BSR patterns (possibly empty rows, any order) against dense
    attention over each row block's gathered keys."""
    rng = np.random.default_rng(seed)
    q, k, v = _rand(rng, 2, Sq, 3), _rand(rng, 1, Sk, 3), _rand(rng, 1, Sk, 3)
    n_rb, n_cb = -(-Sq // rb), -(-Sk // 16)
    lists = [rng.permutation(n_cb)[:rng.integers(0, n_cb + 1)] for _ in range(n_rb)]
    indptr = np.concatenate([[0], np.cumsum([len(c) for c in lists])])
    indices = np.concatenate(lists).astype(np.int64) if indptr[-1] else np.zeros(0, dtype=np.int64)
    O, L = ref.ref_block_sparse_attention(q, k, v, indptr, indices, rb, 16, 0.4)
    for r, cols in enumerate(lists):
        rows = slice(r * rb, min(r * rb + rb, Sq))
        if len(cols) == 0:
            assert (O[:, rows] == 0).all() and np.isneginf(L[:, rows]).all()
            continue
        keys = np.concatenate([np.arange(c * 16, min(c * 16 + 16, Sk)) for c in cols])
        Od, Ld = ref.ref_attention(q[None, :, rows], k[None][:, :, keys], v[None][:, :, keys], 0.4, False)
        assert np.abs(O[:, rows] - Od[0]).max() < 1e-12 and np.abs(L[:, rows] - Ld[0]).max() < 1e-12
