"""The all-rows harness used by the full-size parity tests gives the oracle's
own answer: on small inputs it matches the oracle's whole-problem calls to
fp64 rounding (only BLAS summation order differs), including causal chunks
whose late keys are left out, rows that see no key (Sq > Sk) and GQA groups."""
import numpy as np

from attention_tiled_exact_b200 import workloads as wl
from oracle import attention_ref as ref
from tests import oracle_all_rows as oar


def _close(a, b):
    a, b = np.asarray(a), np.asarray(b)
    assert np.array_equal(np.isneginf(a), np.isneginf(b))
    fin = np.isfinite(b)
    assert np.abs(a[fin] - b[fin]).max() <= 1e-12


def test_prefill_all_rows_equals_the_oracle():
    for (B, Hq, Hkv, Sq, Sk, D, causal, seed) in [(2, 4, 2, 600, 700, 16, True, 1), (1, 3, 1, 530, 530, 8, True, 2),
                                                  (1, 2, 2, 700, 300, 8, True, 3), (1, 2, 1, 300, 257, 8, False, 4)]:
        d = wl.make_prefill(wl.PrefillConfig("h", B, Hq, Hkv, Sq, Sk, D, causal, seed))
        O, L = oar.prefill_all_rows(d["q"], d["k"], d["v"], d["scale"], causal)
        O_ref, L_ref = ref.ref_attention(d["q"], d["k"], d["v"], d["scale"], causal)
        _close(O, O_ref)
        _close(L, L_ref)


def test_decode_and_paged_prefill_all_rows_equal_the_oracle():
    lens = np.array([1, 40, 333, 17], dtype=np.int32)
    d = wl.make_decode(wl.DecodeConfig("h", 4, 8, 2, 128, 1, 1, 5), kv_lens=lens)
    O, L = oar.decode_all_rows(d["q"], d["k_pool"], d["v_pool"], d["block_table"], lens, d["scale"])
    O_ref, L_ref = ref.ref_decode_paged(d["q"], d["k_pool"], d["v_pool"], d["block_table"], lens, d["scale"])
    _close(O, O_ref)
    _close(L, L_ref)
    k_lens = np.array([90, 300, 40], dtype=np.int32)
    q_lens = np.array([64, 64, 40], dtype=np.int32)
    p = wl.make_paged_pool(6, k_lens, 2, 32)
    q = wl.normal_bf16(6, (3, 4, 64, 32), 30)
    O, L = oar.prefill_paged_all_rows(q, q_lens, p["k_pool"], p["v_pool"], p["block_table"], k_lens, 0.2, True)
    O_ref, L_ref = ref.ref_prefill_paged(q, q_lens, p["k_pool"], p["v_pool"], p["block_table"], k_lens, 0.2, True)
    _close(O, O_ref)
    _close(L, L_ref)


def test_fp8_decode_and_backward_all_rows_equal_the_oracle():
    lens = np.array([16, 100, 5], dtype=np.int32)
    d = wl.make_decode_fp8(wl.DecodeConfig("h", 3, 4, 2, 128, 1, 1, 7), kv_lens=lens)
    O, L = oar.decode_fp8_all_rows(d["q"], d["k_pool"], d["v_pool"], d["k_scale"], d["v_scale"], d["block_table"],
                                   lens, d["scale"])
    O_ref, L_ref = ref.ref_decode_paged_fp8(d["q"], d["k_pool"], d["v_pool"], d["k_scale"], d["v_scale"],
                                            d["block_table"], lens, d["scale"])
    _close(O, O_ref)
    _close(L, L_ref)
    q = wl.normal_bf16(8, (2, 4, 50, 16), 40)
    k = wl.normal_bf16(8, (2, 2, 60, 16), 41)
    v = wl.normal_bf16(8, (2, 2, 60, 16), 42)
    do = wl.normal_bf16(8, (2, 4, 50, 16), 43)
    r = oar.backward_all_heads(q, k, v, do, 0.25, True)
    r_ref = ref.ref_attention_backward(q, k, v, do, 0.25, True)
    for name in ("dq", "dk", "dv"):
        _close(r[name], r_ref[name])
