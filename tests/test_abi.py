"""The C-ABI library: it loads, exports every declared symbol, its structs match
the ctypes mirrors, and argument errors come back as status codes before any
GPU work (these run without a GPU)."""
import ctypes
import os
import re
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn.h")


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"ATTN_API\s+[\w\s\*]+?\b(\w+)\s*\(", src)))


def test_header_declares_the_three_calls():
    names = _declared_functions()
    for n in ("attn_prefill", "attn_decode_paged", "splitkv_lse_combine", "attn_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", lib.library_path()], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    missing = [n for n in _declared_functions() if n not in exported]
    assert not missing, missing
    for n in _declared_functions():
        assert hasattr(lib.LIB, n)


def test_library_has_no_torch_dependency(lib):
    out = subprocess.run(["ldd", lib.library_path()], capture_output=True, text=True).stdout
    assert "torch" not in out and "c10" not in out


def test_struct_layouts_match_the_header(lib):
    """Compile a C probe against attn.h and compare sizes/offsets with ctypes."""
    fields_p = [f for f, _ in lib.PrefillParams._fields_]
    fields_d = [f for f, _ in lib.DecodeParams._fields_]
    fields_b = [f for f, _ in lib.BackwardParams._fields_]
    body = ['#include <stdio.h>', '#include <stddef.h>', '#include "attn.h"', "int main(void){"]
    body.append('printf("P %zu\\n", sizeof(attn_prefill_params));')
    body.append('printf("D %zu\\n", sizeof(attn_decode_params));')
    body.append('printf("B %zu\\n", sizeof(attn_backward_params));')
    body.append('printf("C %zu\\n", sizeof(attn_persistent_cmd));')
    body.append('printf("H %zu\\n", sizeof(attn_prefill_host_io));')
    for f, _ in lib.PrefillHostIO._fields_:
        body.append(f'printf("h.{f} %zu\\n", offsetof(attn_prefill_host_io, {f}));')
    for f, _ in lib.PersistentCmd._fields_:
        body.append(f'printf("c.{f} %zu\\n", offsetof(attn_persistent_cmd, {f}));')
    for f in fields_p:
        body.append(f'printf("p.{f} %zu\\n", offsetof(attn_prefill_params, {f}));')
    for f in fields_d:
        body.append(f'printf("d.{f} %zu\\n", offsetof(attn_decode_params, {f}));')
    for f in fields_b:
        body.append(f'printf("b.{f} %zu\\n", offsetof(attn_backward_params, {f}));')
    body.append("return 0;}")
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "probe.c")
        exe = os.path.join(d, "probe")
        open(c, "w").write("\n".join(body))
        subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), c, "-o", exe], check=True)
        got = dict(line.split() for line in subprocess.run([exe], capture_output=True, text=True).stdout.splitlines())
    assert int(got["P"]) == ctypes.sizeof(lib.PrefillParams)
    assert int(got["D"]) == ctypes.sizeof(lib.DecodeParams)
    for f in fields_p:
        assert int(got[f"p.{f}"]) == getattr(lib.PrefillParams, f).offset, f
    for f in fields_d:
        assert int(got[f"d.{f}"]) == getattr(lib.DecodeParams, f).offset, f
    assert int(got["C"]) == ctypes.sizeof(lib.PersistentCmd)
    for f, _ in lib.PersistentCmd._fields_:
        assert int(got[f"c.{f}"]) == getattr(lib.PersistentCmd, f).offset, f
    assert int(got["H"]) == ctypes.sizeof(lib.PrefillHostIO)
    for f, _ in lib.PrefillHostIO._fields_:
        assert int(got[f"h.{f}"]) == getattr(lib.PrefillHostIO, f).offset, f
    assert int(got["B"]) == ctypes.sizeof(lib.BackwardParams)
    for f in fields_b:
        assert int(got[f"b.{f}"]) == getattr(lib.BackwardParams, f).offset, f


def test_status_strings(lib):
    assert lib.status_string(0) == "ok"
    assert "workspace" in lib.status_string(lib.ATTN_ERR_WORKSPACE)
    assert lib.status_string(99) == "unknown status"
    assert lib.LIB.attn_version() >= 100


def _prefill_params(lib, **kw):
    p = lib.PrefillParams()
    fake = 1 << 20  # 16-byte aligned, never dereferenced: validation fails or no device is found first
    p.q = p.k = p.v = p.o = fake
    p.batch, p.num_q_heads, p.num_kv_heads, p.head_dim, p.seqlen_q, p.seqlen_k = 1, 4, 2, 128, 16, 16
    p.q_batch_stride = p.k_batch_stride = p.v_batch_stride = p.o_batch_stride = 4 * 16 * 128
    p.q_head_stride = p.k_head_stride = p.v_head_stride = p.o_head_stride = 16 * 128
    p.q_row_stride = p.k_row_stride = p.v_row_stride = p.o_row_stride = 128
    p.scale = 0.088
    for k, v in kw.items():
        setattr(p, k, v)
    return p


@pytest.mark.parametrize("field,value,code", [
    ("head_dim", 96, 2), ("num_kv_heads", 3, 2), ("scale", float("nan"), 1), ("scale", -1.0, 1),
    ("seqlen_q", -1, 1), ("q", 0, 1), ("q", (1 << 20) + 2, 2), ("k_row_stride", 100, 2),
    ("o_dtype", 7, 1), ("num_kv_heads", 0, 1),
])
def test_prefill_rejects_bad_arguments(lib, field, value, code):
    p = _prefill_params(lib, **{field: value})
    assert lib.LIB.attn_prefill(ctypes.byref(p), None) == code


def test_prefill_paged_argument_checks(lib):
    p = _prefill_params(lib, k_cache=1 << 20)  # v_cache missing, k/v still set
    assert lib.LIB.attn_prefill(ctypes.byref(p), None) == lib.ATTN_ERR_INVALID_ARG
    p = _prefill_params(lib, k=0, v=0, k_cache=1 << 20, v_cache=1 << 20, block_table=1 << 20, seqlens_k=1 << 20,
                        max_blocks_per_seq=4, num_blocks=8, block_size=32)
    assert lib.LIB.attn_prefill(ctypes.byref(p), None) == lib.ATTN_ERR_UNSUPPORTED


def test_empty_prefill_is_a_no_op(lib):
    p = _prefill_params(lib, seqlen_q=0)
    assert lib.LIB.attn_prefill(ctypes.byref(p), None) == 0
    p = _prefill_params(lib, batch=0)
    assert lib.LIB.attn_prefill(ctypes.byref(p), None) == 0


def _decode_params(lib, **kw):
    p = lib.DecodeParams()
    fake = 1 << 20
    p.q = p.k_cache = p.v_cache = p.block_table = p.seq_lens = p.o = fake
    p.batch, p.num_q_heads, p.num_kv_heads, p.head_dim = 64, 32, 8, 128
    p.block_size, p.max_blocks_per_seq, p.num_blocks = 16, 2048, 70000
    p.max_seq_len, p.num_splits, p.scale = 32768, 0, 0.088
    for k, v in kw.items():
        setattr(p, k, v)
    return p


def test_decode_workspace_query_and_too_small(lib):
    p = _decode_params(lib)
    need = ctypes.c_size_t(0)
    assert lib.LIB.attn_decode_paged(ctypes.byref(p), None, 0, ctypes.byref(need), None) == 0
    assert need.value > 0 and need.value % 256 == 0
    rows = 64 * 32
    splits = need.value // (rows * 129 * 4)
    assert splits >= 2
    # too small: reported, nothing enqueued (the fake pointer is never touched)
    need2 = ctypes.c_size_t(0)
    st = lib.LIB.attn_decode_paged(ctypes.byref(p), ctypes.c_void_p(1 << 20), need.value - 256, ctypes.byref(need2), None)
    assert st == lib.ATTN_ERR_WORKSPACE and need2.value == need.value
    # a single split needs no workspace
    p1 = _decode_params(lib, num_splits=1)
    assert lib.LIB.attn_decode_paged(ctypes.byref(p1), None, 0, ctypes.byref(need), None) == 0
    assert need.value == 0


@pytest.mark.parametrize("field,value,code", [
    ("head_dim", 64, 2), ("num_kv_heads", 3, 2), ("num_q_heads", 24, 2), ("block_size", 32, 2),
    ("scale", 0.0, 1), ("max_blocks_per_seq", 0, 1), ("batch", -1, 1), ("q", 0, 1), ("o", (1 << 20) + 4, 2),
    ("num_splits", -2, 1), ("kv_dtype", 1, 1), ("kv_dtype", 7, 1),
])
def test_decode_rejects_bad_arguments(lib, field, value, code):
    p = _decode_params(lib, **{field: value})
    need = ctypes.c_size_t(0)
    assert lib.LIB.attn_decode_paged(ctypes.byref(p), None, 0, ctypes.byref(need), None) == code


@pytest.mark.parametrize("k_scale,v_scale,code", [
    (0.01, 0.02, 0), (0.0, 0.02, 1), (0.01, -1.0, 1), (float("inf"), 0.02, 1), (0.01, float("nan"), 1),
])
def test_decode_fp8_scales_are_checked(lib, k_scale, v_scale, code):
    """An FP8 E4M3 cache needs finite positive scales (checked before anything is enqueued)."""
    p = _decode_params(lib, kv_dtype=lib.ATTN_DTYPE_FP8_E4M3, k_scale=k_scale, v_scale=v_scale)
    need = ctypes.c_size_t(0)
    assert lib.LIB.attn_decode_paged(ctypes.byref(p), None, 0, ctypes.byref(need), None) == code


@pytest.mark.parametrize("prefix_len,code", [(-16, 1), (8, 1), (2048 * 16 + 16, 1), (4096, 0), (2048 * 16, 0)])
def test_shared_prefix_decode_checks_prefix_len(lib, prefix_len, code):
    """prefix_len must be a multiple of 16 within the table capacity."""
    p = _decode_params(lib)
    need = ctypes.c_size_t(0)
    assert lib.LIB.attn_decode_paged_shared_prefix(ctypes.byref(p), prefix_len, None, 0, ctypes.byref(need),
                                                   None) == code
    if code == 0:
        assert need.value > 0 and need.value % 256 == 0


def test_shared_prefix_decode_workspace_and_dtypes(lib):
    p = _decode_params(lib)
    need0, need = ctypes.c_size_t(0), ctypes.c_size_t(0)
    f = lib.LIB.attn_decode_paged_shared_prefix
    # prefix_len 0 is the plain decode, with its workspace size
    assert lib.LIB.attn_decode_paged(ctypes.byref(p), None, 0, ctypes.byref(need0), None) == 0
    assert f(ctypes.byref(p), 0, None, 0, ctypes.byref(need), None) == 0 and need.value == need0.value
    # a prefix needs room for its partials even with a single suffix split
    p1 = _decode_params(lib, num_splits=1)
    assert f(ctypes.byref(p1), 1024, None, 0, ctypes.byref(need), None) == 0
    assert need.value >= 64 * 32 * 129 * 4 * 2
    # too small: reported, nothing enqueued
    need2 = ctypes.c_size_t(0)
    assert f(ctypes.byref(p1), 1024, ctypes.c_void_p(1 << 20), need.value - 256, ctypes.byref(need2),
             None) == lib.ATTN_ERR_WORKSPACE and need2.value == need.value
    # the prefix runs on the bf16 prefill kernel: FP8 caches are not supported here
    p8 = _decode_params(lib, kv_dtype=lib.ATTN_DTYPE_FP8_E4M3, k_scale=0.01, v_scale=0.01)
    assert f(ctypes.byref(p8), 1024, None, 0, ctypes.byref(need), None) == lib.ATTN_ERR_UNSUPPORTED
    # ordinary decode argument checks apply first
    bad = _decode_params(lib, head_dim=64)
    assert f(ctypes.byref(bad), 1024, None, 0, ctypes.byref(need), None) == lib.ATTN_ERR_UNSUPPORTED


def _backward_params(lib, **kw):
    p = lib.BackwardParams()
    fake = 1 << 20
    for f in ("q", "k", "v", "o", "lse", "dout", "dq", "dk", "dv"):
        setattr(p, f, fake)
    p.batch, p.num_q_heads, p.num_kv_heads, p.head_dim, p.seqlen_q, p.seqlen_k = 2, 8, 2, 128, 300, 300
    for t, (bs, hs) in (("q", (8 * 300 * 128, 300 * 128)), ("do", (8 * 300 * 128, 300 * 128)),
                        ("o", (8 * 300 * 128, 300 * 128)), ("dq", (8 * 300 * 128, 300 * 128)),
                        ("k", (2 * 300 * 128, 300 * 128)), ("v", (2 * 300 * 128, 300 * 128)),
                        ("dk", (2 * 300 * 128, 300 * 128)), ("dv", (2 * 300 * 128, 300 * 128))):
        setattr(p, f"{t}_batch_stride", bs)
        setattr(p, f"{t}_head_stride", hs)
        setattr(p, f"{t}_row_stride", 128)
    p.scale, p.causal, p.o_dtype, p.grad_dtype = 0.088, 1, 0, 1
    for k, v in kw.items():
        setattr(p, k, v)
    return p


def test_backward_workspace_query(lib):
    p = _backward_params(lib)
    need = ctypes.c_size_t(0)
    f = lib.LIB.attn_prefill_backward
    assert f(ctypes.byref(p), None, 0, ctypes.byref(need), None) == 0
    assert need.value == 2 * ((2 * 8 * 384 * 4 + 255) // 256 * 256)  # rows padded to 128-row blocks
    need2 = ctypes.c_size_t(0)
    assert f(ctypes.byref(p), ctypes.c_void_p(1 << 20), need.value - 256, ctypes.byref(need2),
             None) == lib.ATTN_ERR_WORKSPACE and need2.value == need.value


@pytest.mark.parametrize("field,value,code", [
    ("head_dim", 96, 2), ("num_kv_heads", 3, 2), ("scale", float("nan"), 1), ("lse", 0, 1), ("dv", 0, 1),
    ("dq", (1 << 20) + 8, 2), ("k_row_stride", 132, 2), ("o_dtype", 2, 1), ("grad_dtype", 5, 1),
    ("dk_row_stride", 64, 1), ("seqlen_q", -1, 1),
])
def test_backward_rejects_bad_arguments(lib, field, value, code):
    p = _backward_params(lib, **{field: value})
    need = ctypes.c_size_t(0)
    assert lib.LIB.attn_prefill_backward(ctypes.byref(p), None, 0, ctypes.byref(need), None) == code


def test_combine_rejects_bad_arguments(lib):
    f = lib.LIB.splitkv_lse_combine
    assert f(1 << 20, 1 << 20, -1, 4, 128, None, 1 << 20, 0, None, None) == lib.ATTN_ERR_INVALID_ARG
    assert f(1 << 20, 1 << 20, 2, 4, 96, None, 1 << 20, 0, None, None) == lib.ATTN_ERR_UNSUPPORTED
    assert f(1 << 20, 1 << 20, 2, 4, 128, None, None, 0, None, None) == lib.ATTN_ERR_INVALID_ARG
    assert f(1 << 20, 1 << 20, 2, 0, 128, None, 1 << 20, 0, None, None) == 0


def test_product_path_has_no_cpu_fallback():
    """The package never imports the oracle; the binding refuses to load without the library."""
    pkg = os.path.join(ROOT, "attention_tiled_exact_b200")
    for fn in os.listdir(pkg):
        if fn.endswith(".py"):
            src = open(os.path.join(pkg, fn)).read()
            assert "import oracle" not in src and "from oracle" not in src, fn
    binding = open(os.path.join(pkg, "binding.py")).read()
    assert "raise ImportError" in binding


def test_prefill_from_host_argument_checks(lib):
    import ctypes
    p = lib.PrefillParams()
    p.batch, p.num_q_heads, p.num_kv_heads, p.head_dim, p.seqlen_q, p.seqlen_k = 1, 4, 2, 128, 16, 16
    p.q, p.k, p.v, p.o = (ctypes.c_void_p(4096 * (i + 1)) for i in range(4))
    for nm in ("q", "o"):
        setattr(p, f"{nm}_row_stride", 128), setattr(p, f"{nm}_head_stride", 16 * 128)
        setattr(p, f"{nm}_batch_stride", 4 * 16 * 128)
    for nm in ("k", "v"):
        setattr(p, f"{nm}_row_stride", 128), setattr(p, f"{nm}_head_stride", 16 * 128)
        setattr(p, f"{nm}_batch_stride", 2 * 16 * 128)
    p.scale = 0.1
    io = lib.PrefillHostIO()
    assert lib.LIB.attn_prefill_from_host(ctypes.byref(p), ctypes.byref(io), None) == lib.ATTN_ERR_INVALID_ARG
    io.q, io.k, io.v, io.o = (ctypes.c_void_p(8192 * (i + 1)) for i in range(4))
    io.kv_heads_per_chunk = 3  # does not divide 2
    assert lib.LIB.attn_prefill_from_host(ctypes.byref(p), ctypes.byref(io), None) == lib.ATTN_ERR_INVALID_ARG
    io.kv_heads_per_chunk = 1
    p.q_head_stride = 32 * 128  # not contiguous
    assert lib.LIB.attn_prefill_from_host(ctypes.byref(p), ctypes.byref(io), None) == lib.ATTN_ERR_UNSUPPORTED
