"""Attention backward (dQ, dK, dV) through the C ABI against the fp64 oracle.

Tolerance. The kernels round P and dS to bf16 (relative error <= 2^-9) where
they enter the tensor-core products, and accumulate in fp32; the inputs are
exact bf16. Each gradient entry is a sum of terms that each carry that
relative error, so the error is bounded by 2^-9 times the sum of the terms'
magnitudes, which for these N(0, 1) inputs stays within a small multiple of
the gradient's own largest entry. The tests gate every gradient tensor at
max|d - d_ref| <= 1e-2 * max|d_ref| (and report the errors seen).
"""
import numpy as np
import pytest

from attention_tiled_exact_b200 import workloads as wl
from oracle import attention_ref as ref
from tests.helpers import to_dev_bf16, to_f64

pytestmark = pytest.mark.gpu

REL_TOL = 1e-2


def assert_grad_close(got, want, name):
    peak = float(np.abs(want).max())
    err = float(np.abs(got - want).max()) if got.size else 0.0
    print(f"{name}: max|err| {err:.3e}, max|ref| {peak:.3e}, ratio {err / max(peak, 1e-30):.2e}")
    assert np.isfinite(got).all(), name
    assert err <= REL_TOL * max(peak, 1e-6), f"{name}: max|err| {err:.3e} > {REL_TOL} x max|ref| {peak:.3e}"


def _inputs(B, Hq, Hkv, Sq, Sk, D, seed):
    q = wl.normal_bf16(seed, (B, Hq, Sq, D), 40)
    k = wl.normal_bf16(seed, (B, Hkv, Sk, D), 41)
    v = wl.normal_bf16(seed, (B, Hkv, Sk, D), 42)
    do = wl.normal_bf16(seed, (B, Hq, Sq, D), 43)
    return q, k, v, do


def _f32(x):
    import torch
    return torch.tensor(np.asarray(x, dtype=np.float32), device="cuda")


def _backward(lib, q, k, v, do, o, lse, scale, causal, grad_dtype=None, **kw):
    import torch
    dq, dk, dv = lib.prefill_backward(to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v), o, lse, to_dev_bf16(do),
                                      scale, causal, grad_dtype=grad_dtype or torch.float32, **kw)
    torch.cuda.synchronize()
    return to_f64(dq), to_f64(dk), to_f64(dv)


@pytest.mark.parametrize("B,Hq,Hkv,Sq,Sk,D,causal", [
    (1, 2, 2, 128, 128, 64, False),    # one tile each way
    (1, 2, 2, 128, 128, 128, True),    # the diagonal block alone
    (2, 8, 2, 300, 300, 128, True),    # GQA, ragged last blocks
    (1, 4, 1, 200, 456, 128, True),    # a chunk on cached context (Sq < Sk)
    (1, 4, 2, 456, 200, 64, True),     # Sq > Sk: the first rows see no key
    (2, 4, 4, 1, 777, 128, False),     # one query row
    (1, 8, 2, 513, 513, 64, True),     # G = 4, head_dim 64
    (1, 2, 1, 130, 70, 128, False),    # fewer keys than one tile
    (1, 8, 1, 2048, 128, 128, False),  # one dK/dV item, 128 dQ items: dQ CTAs on idle SMs from the start
])
def test_backward_matches_oracle(lib, B, Hq, Hkv, Sq, Sk, D, causal):
    seed = 7 * Sq + Sk + D + Hq
    q, k, v, do = _inputs(B, Hq, Hkv, Sq, Sk, D, seed)
    scale = 1.0 / np.sqrt(D)
    r = ref.ref_attention_backward(q, k, v, do, scale, causal)
    dq, dk, dv = _backward(lib, q, k, v, do, _f32(r["o"]), _f32(r["lse"]), scale, causal)
    assert_grad_close(dq, r["dq"], "dq")
    assert_grad_close(dk, r["dk"], "dk")
    assert_grad_close(dv, r["dv"], "dv")


def test_backward_after_gpu_forward(lib):
    """The path a user runs: the library's forward (bf16 and fp32 O), then the backward."""
    import torch
    B, Hq, Hkv, S, D = 2, 8, 2, 384, 128
    q, k, v, do = _inputs(B, Hq, Hkv, S, S, D, 51)
    scale = 1.0 / np.sqrt(D)
    r = ref.ref_attention_backward(q, k, v, do, scale, True)
    for out_dtype in (torch.float32, torch.bfloat16):
        o, lse = lib.prefill(to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v), scale, True, out_dtype=out_dtype)
        dq, dk, dv = _backward(lib, q, k, v, do, o, lse, scale, True)
        assert_grad_close(dq, r["dq"], f"dq ({out_dtype})")
        assert_grad_close(dk, r["dk"], f"dk ({out_dtype})")
        assert_grad_close(dv, r["dv"], f"dv ({out_dtype})")


def test_backward_bf16_gradients_and_determinism(lib):
    import torch
    q, k, v, do = _inputs(1, 4, 2, 260, 260, 128, 52)
    scale = 0.1
    r = ref.ref_attention_backward(q, k, v, do, scale, True)
    o, lse = _f32(r["o"]), _f32(r["lse"])
    g16 = _backward(lib, q, k, v, do, o, lse, scale, True, grad_dtype=torch.bfloat16)
    for got, name in zip(g16, ("dq", "dk", "dv")):
        assert_grad_close(got, r[name], name + " bf16")
    a = _backward(lib, q, k, v, do, o, lse, scale, True)
    b = _backward(lib, q, k, v, do, o, lse, scale, True)
    assert all(np.array_equal(x, y) for x, y in zip(a, b))  # no atomics: bitwise repeatable


def test_backward_strided_layout(lib):
    """[B, S, H, D] storage for every tensor (head stride D, row stride H*D)."""
    import torch
    B, Hq, Hkv, S, D = 1, 4, 2, 200, 128
    q, k, v, do = _inputs(B, Hq, Hkv, S, S, D, 53)
    scale = 1.0 / np.sqrt(D)
    r = ref.ref_attention_backward(q, k, v, do, scale, True)

    def bshd(x):
        return to_dev_bf16(np.ascontiguousarray(np.asarray(x).transpose(0, 2, 1, 3))).transpose(1, 2)

    def grad_buf(shape):
        return torch.empty((shape[0], shape[2], shape[1], shape[3]), dtype=torch.float32, device="cuda").transpose(1, 2)

    o = _f32(np.ascontiguousarray(r["o"].transpose(0, 2, 1, 3))).transpose(1, 2)
    dq, dk, dv = grad_buf(q.shape), grad_buf(k.shape), grad_buf(v.shape)
    lib.prefill_backward(bshd(q), bshd(k), bshd(v), o, _f32(r["lse"]), bshd(do), scale, True, dq=dq, dk=dk, dv=dv)
    torch.cuda.synchronize()
    assert_grad_close(to_f64(dq), r["dq"], "dq bshd")
    assert_grad_close(to_f64(dk), r["dk"], "dk bshd")
    assert_grad_close(to_f64(dv), r["dv"], "dv bshd")


def test_backward_full_size_every_head(lib):
    """The causal GQA prefill shape (4 x 32/8 heads x 2048 x 128) after the
    library's forward: every gradient of every head against the oracle."""
    import torch
    from tests.oracle_all_rows import backward_all_heads
    cfg = wl.CAUSAL_GQA_2K
    d = wl.make_prefill(cfg)
    do = wl.normal_bf16(cfg.seed, (cfg.batch, cfg.q_heads, cfg.seqlen_q, cfg.head_dim), 43)
    r = backward_all_heads(d["q"], d["k"], d["v"], do, cfg.scale, True)
    o, lse = lib.prefill(to_dev_bf16(d["q"]), to_dev_bf16(d["k"]), to_dev_bf16(d["v"]), cfg.scale, True,
                         out_dtype=torch.float32)
    dq, dk, dv = _backward(lib, d["q"], d["k"], d["v"], do, o, lse, cfg.scale, True)
    assert_grad_close(dq, r["dq"], "dq full size")
    assert_grad_close(dk, r["dk"], "dk full size")
    assert_grad_close(dv, r["dv"], "dv full size")
