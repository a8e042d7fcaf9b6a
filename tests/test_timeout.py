"""The pipeline-wait timeout path of the prefill and backward kernels.

Every mbarrier wait in those kernels is bounded. When one runs out, its CTA
stops, waits for the copies and tensor-core products it already issued (those
complete by themselves), frees its tensor memory and ORs ATTN_FAULT_TIMEOUT
into the caller's error word. The diagnostic attn_set_wait_limit shrinks the
bound to one clock cycle, so that waits give up at once: the call must report
the timeout, and a normal call afterwards on the same stream must match the
oracle (a CTA that kept its tensor memory would leave the next launch unable
to allocate any). No GPU fault is involved: the waits simply return early.
"""
import numpy as np
import pytest

from attention_tiled_exact_b200 import workloads as wl
from oracle import attention_ref as ref
from tests.helpers import assert_lse_close, assert_o_close, to_dev_bf16, to_f64


def test_status_from_flags_mapping(lib):
    assert lib.status_from_flags(0) == lib.ATTN_OK
    assert lib.status_from_flags(lib.ATTN_FAULT_TIMEOUT) == lib.ATTN_ERR_TIMEOUT
    assert lib.status_from_flags(lib.ATTN_FAULT_TIMEOUT | lib.ATTN_FAULT_BAD_BLOCK) == lib.ATTN_ERR_TIMEOUT
    for bit in (lib.ATTN_FAULT_BAD_BLOCK, lib.ATTN_FAULT_BAD_LENGTH, lib.ATTN_FAULT_PREFIX_MISMATCH):
        assert lib.status_from_flags(bit) == lib.ATTN_ERR_DEVICE_FAULT


def test_sync_error_flags_rejects_a_null_word(lib):
    import ctypes
    assert lib.LIB.attn_sync_error_flags(None, None, ctypes.byref(ctypes.c_int32(0))) == lib.ATTN_ERR_INVALID_ARG


@pytest.fixture
def short_waits(lib):
    lib.set_wait_limit(1)
    try:
        yield
    finally:
        lib.set_wait_limit(0)


def _prefill_case():
    return wl.make_prefill(wl.PrefillConfig("timeout", 2, 8, 2, 700, 700, 128, True, 31))


@pytest.mark.gpu
def test_prefill_timeout_is_reported_and_the_next_call_is_correct(lib):
    import torch
    d = _prefill_case()
    q, k, v = to_dev_bf16(d["q"]), to_dev_bf16(d["k"]), to_dev_bf16(d["v"])
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    lib.set_wait_limit(1)
    try:
        for _ in range(3):
            lib.prefill(q, k, v, d["scale"], True, error_flags=flags)
        status, word = lib.sync_error_flags(flags)
    finally:
        lib.set_wait_limit(0)
    assert word & lib.ATTN_FAULT_TIMEOUT and status == lib.ATTN_ERR_TIMEOUT
    flags.zero_()
    O_ref, L_ref = ref.ref_attention(d["q"], d["k"], d["v"], d["scale"], True)
    for _ in range(2):
        o, lse = lib.prefill(q, k, v, d["scale"], True, out_dtype=torch.float32, error_flags=flags)
        status, word = lib.sync_error_flags(flags)
        assert status == lib.ATTN_OK and word == 0
        assert_o_close(to_f64(o), O_ref, False, "prefill after a timeout")
        assert_lse_close(to_f64(lse), L_ref, "prefill after a timeout")


@pytest.mark.gpu
def test_paged_prefill_timeout_is_reported(lib, short_waits):
    import torch
    from tests.helpers import to_dev_i32
    k_lens = np.array([300, 900, 17], dtype=np.int32)
    d = wl.make_paged_pool(32, k_lens, 2, 128)
    q = wl.normal_bf16(32, (3, 8, 256, 128), 30)
    q_lens = np.array([256, 200, 17], dtype=np.int32)
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    lib.prefill_paged(to_dev_bf16(q), to_dev_bf16(d["k_pool"]), to_dev_bf16(d["v_pool"]),
                      to_dev_i32(d["block_table"]), to_dev_i32(k_lens), to_dev_i32(q_lens), None, True,
                      error_flags=flags)
    status, word = lib.sync_error_flags(flags)
    assert word & lib.ATTN_FAULT_TIMEOUT and status == lib.ATTN_ERR_TIMEOUT


@pytest.mark.gpu
def test_backward_timeout_is_reported_and_the_next_call_is_correct(lib):
    import torch
    cfg = wl.PrefillConfig("timeout_bwd", 1, 8, 2, 384, 384, 128, True, 33)
    d = wl.make_prefill(cfg)
    do = wl.normal_bf16(cfg.seed, d["q"].shape, 43)
    q, k, v, g = to_dev_bf16(d["q"]), to_dev_bf16(d["k"]), to_dev_bf16(d["v"]), to_dev_bf16(do)
    o, lse = lib.prefill(q, k, v, d["scale"], True, out_dtype=torch.float32)
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    lib.set_wait_limit(1)
    try:
        lib.prefill_backward(q, k, v, o, lse, g, d["scale"], True, error_flags=flags)
        status, word = lib.sync_error_flags(flags)
    finally:
        lib.set_wait_limit(0)
    assert word & lib.ATTN_FAULT_TIMEOUT and status == lib.ATTN_ERR_TIMEOUT
    flags.zero_()
    grads = lib.prefill_backward(q, k, v, o, lse, g, d["scale"], True, error_flags=flags)
    status, word = lib.sync_error_flags(flags)
    assert status == lib.ATTN_OK and word == 0
    r = ref.ref_attention_backward(d["q"], d["k"], d["v"], do, d["scale"], True)
    for name, t in zip(("dq", "dk", "dv"), grads):
        err = float(np.abs(to_f64(t) - r[name]).max())
        assert err <= 1e-2 * float(np.abs(r[name]).max()), (name, err)
