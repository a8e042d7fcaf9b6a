"""ctypes binding of libattn_b200.so.

Argument marshalling only: torch tensors provide device memory and the
current CUDA stream; every step of the computation runs in the library's
kernels. The names follow the C ABI declared in include/attn.h.

Importing this module loads the library and fails loudly if it is missing
(build it with ``python -m attention_tiled_exact_b200.build``). There is no
CPU fallback. With ``ATTN_B200_DEBUG_BOUNDS=1`` in the environment it loads
the debug build ``libattn_b200_debug.so`` instead, whose kernels check their
shared-memory, tensor-memory and output indices (``ATTN_FAULT_BOUNDS``).
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
DEBUG_BOUNDS = os.environ.get("ATTN_B200_DEBUG_BOUNDS", "0") not in ("", "0")
_LIB_FILE = os.path.join(HERE, "libattn_b200_debug.so" if DEBUG_BOUNDS else "libattn_b200.so")

ATTN_OK = 0
ATTN_ERR_INVALID_ARG = 1
ATTN_ERR_UNSUPPORTED = 2
ATTN_ERR_WORKSPACE = 3
ATTN_ERR_CUDA = 4
ATTN_ERR_DEVICE_FAULT = 5
ATTN_ERR_TIMEOUT = 6
ATTN_ERR_NO_DEVICE = 7

ATTN_DTYPE_BF16 = 0
ATTN_DTYPE_F32 = 1
ATTN_DTYPE_FP8_E4M3 = 2

ATTN_FAULT_TIMEOUT = 0x1
ATTN_FAULT_BAD_BLOCK = 0x2
ATTN_FAULT_BAD_LENGTH = 0x4
ATTN_FAULT_PREFIX_MISMATCH = 0x8
ATTN_FAULT_BOUNDS = 0x10

# Bounds-check sites of the debug build (attn_bounds_site_t).
BOUNDS_SITES = {
    "PREFILL_SMEM_Q": 1, "PREFILL_SMEM_KV": 2, "PREFILL_TABLE": 3, "PREFILL_TMEM_S": 4, "PREFILL_TMEM_O": 5,
    "PREFILL_SMEM_STAGE": 6, "PREFILL_SMEM_VFIX": 7, "PREFILL_OUT": 8, "DECODE_TABLE": 9, "DECODE_SMEM": 10,
    "DECODE_PARTIAL": 11, "COMBINE": 12, "BWD_SMEM": 13, "BWD_TMEM": 14, "BWD_OUT": 15,
}


def fault_site(word: int) -> int:
    """The site of the first failed bounds check recorded in an error word (0: none)."""
    return (int(word) >> 16) & 0xFF

_vp = ctypes.c_void_p
_i32 = ctypes.c_int32
_i64 = ctypes.c_int64


class PrefillParams(ctypes.Structure):
    """Mirror of ``attn_prefill_params``."""

    _fields_ = [
        ("q", _vp), ("k", _vp), ("v", _vp), ("o", _vp), ("lse", _vp),
        ("batch", _i32), ("num_q_heads", _i32), ("num_kv_heads", _i32), ("head_dim", _i32),
        ("seqlen_q", _i32), ("seqlen_k", _i32),
        ("q_batch_stride", _i64), ("q_head_stride", _i64), ("q_row_stride", _i64),
        ("k_batch_stride", _i64), ("k_head_stride", _i64), ("k_row_stride", _i64),
        ("v_batch_stride", _i64), ("v_head_stride", _i64), ("v_row_stride", _i64),
        ("o_batch_stride", _i64), ("o_head_stride", _i64), ("o_row_stride", _i64),
        ("scale", ctypes.c_float), ("causal", _i32), ("o_dtype", _i32),
        ("seqlens_q", _vp), ("seqlens_k", _vp), ("k_cache", _vp), ("v_cache", _vp),
        ("block_table", _vp), ("max_blocks_per_seq", _i32), ("num_blocks", _i32),
        ("block_size", _i32), ("error_flags", _vp), ("cu_seqlens_q", _vp), ("total_q", _i32),
    ]


class PrefillHostIO(ctypes.Structure):
    """Mirror of ``attn_prefill_host_io`` (host pointers)."""

    _fields_ = [("q", _vp), ("k", _vp), ("v", _vp), ("o", _vp), ("lse", _vp), ("kv_heads_per_chunk", _i32)]


class BackwardParams(ctypes.Structure):
    """Mirror of ``attn_backward_params``."""

    _fields_ = [
        ("q", _vp), ("k", _vp), ("v", _vp), ("o", _vp), ("lse", _vp), ("dout", _vp),
        ("dq", _vp), ("dk", _vp), ("dv", _vp),
        ("batch", _i32), ("num_q_heads", _i32), ("num_kv_heads", _i32), ("head_dim", _i32),
        ("seqlen_q", _i32), ("seqlen_k", _i32),
    ] + [(f"{t}_{d}_stride", _i64) for t in ("q", "k", "v", "o", "do", "dq", "dk", "dv")
         for d in ("batch", "head", "row")] + [
        ("scale", ctypes.c_float), ("causal", _i32), ("o_dtype", _i32), ("grad_dtype", _i32),
        ("error_flags", _vp),
    ]


class DecodeParams(ctypes.Structure):
    """Mirror of ``attn_decode_params``."""

    _fields_ = [
        ("q", _vp), ("k_cache", _vp), ("v_cache", _vp), ("block_table", _vp), ("seq_lens", _vp),
        ("o", _vp), ("lse", _vp),
        ("batch", _i32), ("num_q_heads", _i32), ("num_kv_heads", _i32), ("head_dim", _i32),
        ("block_size", _i32), ("max_blocks_per_seq", _i32), ("num_blocks", _i32),
        ("max_seq_len", _i32), ("num_splits", _i32), ("scale", ctypes.c_float), ("o_dtype", _i32),
        ("error_flags", _vp), ("kv_dtype", _i32), ("k_scale", ctypes.c_float), ("v_scale", ctypes.c_float),
    ]


class PersistentCmd(ctypes.Structure):
    """Mirror of ``attn_persistent_cmd`` (host memory shared with the persistent kernel)."""

    _fields_ = [("seq", _i32), ("batch", _i32), ("max_seq_len", _i32), ("stop", _i32), ("done", _i32),
                ("status", _i32), ("running", _i32), ("reserved", _i32)]


def _load():
    if not os.path.exists(_LIB_FILE):
        raise ImportError(f"{_LIB_FILE} is missing: build it with "
                          "`python -m attention_tiled_exact_b200.build` (needs nvcc)")
    lib = ctypes.CDLL(_LIB_FILE)
    lib.attn_prefill.argtypes = [ctypes.POINTER(PrefillParams), _vp]
    lib.attn_prefill.restype = ctypes.c_int
    lib.attn_prefill_from_host.argtypes = [ctypes.POINTER(PrefillParams), ctypes.POINTER(PrefillHostIO), _vp]
    lib.attn_prefill_from_host.restype = ctypes.c_int
    lib.attn_decode_paged.argtypes = [ctypes.POINTER(DecodeParams), _vp, ctypes.c_size_t,
                                      ctypes.POINTER(ctypes.c_size_t), _vp]
    lib.attn_decode_paged.restype = ctypes.c_int
    lib.attn_decode_paged_noalloc.argtypes = [ctypes.POINTER(DecodeParams), _vp]
    lib.attn_decode_paged_noalloc.restype = ctypes.c_int
    lib.attn_decode_paged_shared_prefix.argtypes = [ctypes.POINTER(DecodeParams), ctypes.c_int32, _vp,
                                                    ctypes.c_size_t, ctypes.POINTER(ctypes.c_size_t), _vp]
    lib.attn_decode_paged_shared_prefix.restype = ctypes.c_int
    lib.attn_prefill_backward.argtypes = [ctypes.POINTER(BackwardParams), _vp, ctypes.c_size_t,
                                          ctypes.POINTER(ctypes.c_size_t), _vp]
    lib.attn_prefill_backward.restype = ctypes.c_int
    lib.splitkv_lse_combine.argtypes = [_vp, _vp, ctypes.c_int, ctypes.c_int, ctypes.c_int, _vp, _vp,
                                        ctypes.c_int, _vp, _vp]
    lib.splitkv_lse_combine.restype = ctypes.c_int
    lib.attn_status_string.argtypes = [ctypes.c_int]
    lib.attn_status_string.restype = ctypes.c_char_p
    lib.attn_version.argtypes = []
    lib.attn_version.restype = ctypes.c_int
    lib.attn_status_from_flags.argtypes = [ctypes.c_int32]
    lib.attn_status_from_flags.restype = ctypes.c_int
    lib.attn_sync_error_flags.argtypes = [_vp, _vp, ctypes.POINTER(ctypes.c_int32)]
    lib.attn_sync_error_flags.restype = ctypes.c_int
    lib.attn_set_wait_limit.argtypes = [ctypes.c_longlong]
    lib.attn_set_wait_limit.restype = None
    lib.attn_selftest_exp2.argtypes = [_vp, _vp, _vp, ctypes.c_int, _vp]
    lib.attn_selftest_exp2.restype = ctypes.c_int
    lib.attn_debug_bounds_enabled.argtypes = []
    lib.attn_debug_bounds_enabled.restype = ctypes.c_int
    lib.attn_debug_plant_bounds.argtypes = [ctypes.c_int]
    lib.attn_debug_plant_bounds.restype = ctypes.c_int
    lib.attn_decode_persistent_workspace.argtypes = [ctypes.POINTER(DecodeParams), ctypes.POINTER(ctypes.c_size_t)]
    lib.attn_decode_persistent_workspace.restype = ctypes.c_int
    lib.attn_decode_persistent_launch.argtypes = [ctypes.POINTER(DecodeParams), _vp, _vp, ctypes.c_size_t,
                                                  ctypes.c_longlong, _vp]
    lib.attn_decode_persistent_launch.restype = ctypes.c_int
    lib.attn_decode_persistent_submit.argtypes = [_vp, ctypes.c_int32, ctypes.c_int32, ctypes.POINTER(ctypes.c_int32)]
    lib.attn_decode_persistent_submit.restype = ctypes.c_int
    lib.attn_decode_persistent_wait.argtypes = [_vp, ctypes.c_int32, ctypes.c_longlong]
    lib.attn_decode_persistent_wait.restype = ctypes.c_int
    lib.attn_decode_persistent_stop.argtypes = [_vp]
    lib.attn_decode_persistent_stop.restype = None
    i32p = ctypes.POINTER(ctypes.c_int32)
    lib.attn_decode_graph_pool_workspace.argtypes = [ctypes.POINTER(DecodeParams), i32p, ctypes.c_int, i32p,
                                                     ctypes.c_int, ctypes.POINTER(ctypes.c_size_t)]
    lib.attn_decode_graph_pool_workspace.restype = ctypes.c_int
    lib.attn_decode_graph_pool_create.argtypes = [ctypes.POINTER(DecodeParams), i32p, ctypes.c_int, i32p,
                                                  ctypes.c_int, _vp, ctypes.c_size_t, ctypes.POINTER(_vp)]
    lib.attn_decode_graph_pool_create.restype = ctypes.c_int
    lib.attn_decode_graph_pool_replay.argtypes = [_vp, ctypes.c_int32, ctypes.c_int32, _vp, i32p, i32p]
    lib.attn_decode_graph_pool_replay.restype = ctypes.c_int
    lib.attn_decode_graph_pool_destroy.argtypes = [_vp]
    lib.attn_decode_graph_pool_destroy.restype = None
    return lib


LIB = _load()


def library_path() -> str:
    return _LIB_FILE


def status_string(status: int) -> str:
    return LIB.attn_status_string(int(status)).decode()


class AttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


def _check(status: int, where: str):
    if status != ATTN_OK:
        raise AttnError(status, where)


def status_from_flags(flags: int) -> int:
    """The status an error word maps to (ATTN_ERR_TIMEOUT, ATTN_ERR_DEVICE_FAULT or ATTN_OK)."""
    return int(LIB.attn_status_from_flags(int(flags)))


def sync_error_flags(error_flags) -> tuple[int, int]:
    """Wait for the current stream, read the int32 device error word and map it.

    Returns ``(status, word)``; the word is left as it is.
    """
    _need(error_flags.dtype == torch.int32 and error_flags.is_cuda and error_flags.numel() >= 1, "int32 error word")
    word = ctypes.c_int32(0)
    st = LIB.attn_sync_error_flags(_ptr(error_flags), _stream(error_flags.device), ctypes.byref(word))
    if st == ATTN_ERR_CUDA or st == ATTN_ERR_INVALID_ARG:
        raise AttnError(st, "attn_sync_error_flags")
    return int(st), int(word.value)


def set_wait_limit(cycles: int = 0) -> None:
    """Diagnostic: clock-cycle bound of the prefill/backward pipeline waits (0 = the ~1 s default)."""
    LIB.attn_set_wait_limit(int(cycles))


def debug_bounds_enabled() -> bool:
    """True when the loaded library is the bounds-checking debug build."""
    return bool(LIB.attn_debug_bounds_enabled())


def debug_plant_bounds(site: int) -> None:
    """Debug build: kernels launched from now on report a failed check at ``site``
    (0 turns it off) while their accesses keep their real, checked indices."""
    _check(LIB.attn_debug_plant_bounds(int(site)), "attn_debug_plant_bounds")


def selftest_exp2(x):
    """Diagnostic: the prefill kernel's FMA-pipe 2^x and MUFU ex2.approx of an fp32 CUDA tensor.

    Returns ``(y_poly, y_mufu)``, fp32 tensors shaped like ``x``.
    """
    _need(x.dtype == torch.float32 and x.is_cuda and x.is_contiguous(), "contiguous fp32 CUDA tensor")
    y_poly, y_mufu = torch.empty_like(x), torch.empty_like(x)
    _check(LIB.attn_selftest_exp2(_ptr(x), _ptr(y_poly), _ptr(y_mufu), x.numel(), _stream(x.device)),
           "attn_selftest_exp2")
    return y_poly, y_mufu


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _out_code(dtype) -> int:
    if dtype == torch.bfloat16:
        return ATTN_DTYPE_BF16
    if dtype == torch.float32:
        return ATTN_DTYPE_F32
    raise TypeError("output dtype must be bfloat16 or float32")


def _need(cond, msg):
    if not cond:
        raise ValueError(msg)


# ----------------------------------------------------------------------------
# prefill
# ----------------------------------------------------------------------------


def _queries(p, q, out, lse, out_dtype, want_lse, batch, cu_seqlens_q, max_seqlen_q):
    """Fill the query / output / LSE fields of PrefillParams for a padded
    [B,Hq,Sq,D] or a packed [total_q,Hq,D] layout; returns (out, lse)."""
    if cu_seqlens_q is None:
        _need(q.dim() == 4 and q.shape[0] == batch, "q must be [B, Hq, Sq, D]")
        B, Hq, Sq, D = q.shape
        o_shape, lse_shape = (B, Hq, Sq, D), (B, Hq, Sq)
    else:
        _need(q.dim() == 3, "packed q must be [total_q, Hq, D]")
        _need(cu_seqlens_q.dtype == torch.int32 and cu_seqlens_q.is_cuda and cu_seqlens_q.is_contiguous() and
              cu_seqlens_q.numel() == batch + 1, "int32 cu_seqlens_q [B + 1]")
        _need(max_seqlen_q is not None and int(max_seqlen_q) >= 0, "max_seqlen_q (an upper bound of the rows of a sequence)")
        total, Hq, D = q.shape
        Sq = int(max_seqlen_q)
        o_shape, lse_shape = (total, Hq, D), (Hq, total)
    _need(q.dtype == torch.bfloat16 and q.is_cuda and q.stride(-1) == 1, "bf16 CUDA q, last dim contiguous")
    if out is None:
        out = torch.empty(o_shape, dtype=out_dtype, device=q.device)
    _need(tuple(out.shape) == o_shape and out.stride(-1) == 1, f"out {o_shape}")
    if lse is None and want_lse:
        lse = torch.empty(lse_shape, dtype=torch.float32, device=q.device)
    if lse is not None:
        _need(lse.is_contiguous() and lse.dtype == torch.float32 and tuple(lse.shape) == lse_shape, f"lse {lse_shape}")
    p.q, p.o, p.lse = _ptr(q), _ptr(out), _ptr(lse)
    p.num_q_heads, p.head_dim, p.seqlen_q = Hq, D, Sq
    if cu_seqlens_q is None:
        p.q_batch_stride, p.q_head_stride, p.q_row_stride = q.stride(0), q.stride(1), q.stride(2)
        p.o_batch_stride, p.o_head_stride, p.o_row_stride = out.stride(0), out.stride(1), out.stride(2)
    else:
        p.q_batch_stride, p.q_head_stride, p.q_row_stride = 0, q.stride(1), q.stride(0)
        p.o_batch_stride, p.o_head_stride, p.o_row_stride = 0, out.stride(1), out.stride(0)
        p.cu_seqlens_q, p.total_q = _ptr(cu_seqlens_q), q.shape[0]
    p.o_dtype = _out_code(out.dtype)
    return out, lse


def prefill(q, k, v, scale: float | None = None, causal: bool = False, out=None, lse=None,
            out_dtype=torch.bfloat16, want_lse: bool = True, error_flags=None, seqlens_q=None, seqlens_k=None,
            cu_seqlens_q=None, max_seqlen_q=None):
    """Tiled prefill attention. q [B,Hq,Sq,D], k/v [B,Hkv,Sk,D] bf16 CUDA tensors.

    seqlens_q / seqlens_k (int32 [B] CUDA tensors, optional): valid query rows
    and keys of each sequence of a padded batch (rows past seqlens_q[b] are
    not written).
    Packed queries: with cu_seqlens_q (int32 [B + 1] CUDA) and max_seqlen_q
    (host int), q is [total_q, Hq, D], sequence b owning rows
    cu_seqlens_q[b] .. cu_seqlens_q[b+1] - 1; O is then [total_q, Hq, D] and
    the LSE [Hq, total_q].
    Returns ``(O [B,Hq,Sq,D], LSE [B,Hq,Sq] fp32 or None)`` (padded).
    """
    _need(k.dim() == 4 and v.dim() == 4, "k, v must be 4-D [B, H, S, D]")
    B, Hkv, Sk, D = k.shape
    _need(tuple(v.shape) == tuple(k.shape) and q.shape[-1] == D, "shape mismatch")
    for t in (k, v):
        _need(t.dtype == torch.bfloat16 and t.is_cuda and t.stride(3) == 1, "bf16 CUDA, last dim contiguous")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    p = PrefillParams()
    out, lse = _queries(p, q, out, lse, out_dtype, want_lse, B, cu_seqlens_q, max_seqlen_q)
    p.k, p.v = _ptr(k), _ptr(v)
    p.batch, p.num_kv_heads, p.seqlen_k = B, Hkv, Sk
    p.k_batch_stride, p.k_head_stride, p.k_row_stride = k.stride(0), k.stride(1), k.stride(2)
    p.v_batch_stride, p.v_head_stride, p.v_row_stride = v.stride(0), v.stride(1), v.stride(2)
    p.scale, p.causal = float(scale), int(bool(causal))
    p.error_flags = _ptr(error_flags)
    for name, t in (("seqlens_q", seqlens_q), ("seqlens_k", seqlens_k)):
        if t is not None:
            _need(t.dtype == torch.int32 and t.is_cuda and t.is_contiguous() and t.numel() == B, f"int32 {name} [B]")
    p.seqlens_q, p.seqlens_k = _ptr(seqlens_q), _ptr(seqlens_k)
    _check(LIB.attn_prefill(ctypes.byref(p), _stream(q.device)), "attn_prefill")
    return out, lse


def prefill_from_host(q_host, k_host, v_host, q, k, v, o, o_host, lse=None, lse_host=None,
                      scale: float | None = None, causal: bool = False, kv_heads_per_chunk: int = 0,
                      error_flags=None):
    """Dense prefill from and to host memory, copies overlapped with compute.

    q_host / k_host / v_host (CPU bf16, pinned, contiguous [B,H,S,D]) are
    copied into the device staging tensors q / k / v (contiguous, same
    shapes); O (and the LSE, when ``lse`` is given) are computed into ``o`` /
    ``lse`` and copied back into ``o_host`` / ``lse_host``, chunk by chunk
    (one batch entry and ``kv_heads_per_chunk`` kv heads per chunk; 0 = all).
    Asynchronous on the current stream; the host tensors are ready after it
    synchronises. Returns ``(o_host, lse_host)``.
    """
    for t in (q_host, k_host, v_host, o_host) + ((lse_host,) if lse is not None else ()):
        _need(t is not None and not t.is_cuda and t.is_contiguous(), "host tensors: CPU, contiguous")
    for t in (q, k, v, o) + ((lse,) if lse is not None else ()):
        _need(t.is_cuda and t.is_contiguous(), "device tensors: CUDA, contiguous")
    _need(tuple(q_host.shape) == tuple(q.shape) and tuple(k_host.shape) == tuple(k.shape) and
          tuple(v_host.shape) == tuple(v.shape) and tuple(o_host.shape) == tuple(o.shape), "host/device shapes")
    _need(q.dtype == k.dtype == v.dtype == q_host.dtype == k_host.dtype == v_host.dtype == torch.bfloat16,
          "bf16 inputs")
    _need(o.dtype == o_host.dtype and o.dtype in (torch.bfloat16, torch.float32), "o: bf16 or fp32 on both sides")
    B, Hq, Sq, D = q.shape
    Hkv, Sk = k.shape[1], k.shape[2]
    p = PrefillParams()
    p.q, p.k, p.v, p.o = _ptr(q), _ptr(k), _ptr(v), _ptr(o)
    p.lse = _ptr(lse)
    p.batch, p.num_q_heads, p.num_kv_heads, p.head_dim, p.seqlen_q, p.seqlen_k = B, Hq, Hkv, D, Sq, Sk
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o)):
        setattr(p, f"{name}_batch_stride", t.stride(0))
        setattr(p, f"{name}_head_stride", t.stride(1))
        setattr(p, f"{name}_row_stride", t.stride(2))
    p.scale = float(scale if scale is not None else 1.0 / math.sqrt(D))
    p.causal, p.o_dtype = int(bool(causal)), _out_code(o.dtype)
    p.error_flags = _ptr(error_flags)
    io = PrefillHostIO()
    io.q, io.k, io.v, io.o = (ctypes.c_void_p(t.data_ptr()) for t in (q_host, k_host, v_host, o_host))
    io.lse = ctypes.c_void_p(lse_host.data_ptr()) if lse is not None else None
    io.kv_heads_per_chunk = int(kv_heads_per_chunk)
    _check(LIB.attn_prefill_from_host(ctypes.byref(p), ctypes.byref(io), _stream(q.device)), "attn_prefill_from_host")
    return o_host, lse_host


def _backward_params(q, k, v, o, lse, dout, dq, dk, dv, scale, causal, error_flags):
    B, Hq, Sq, D = q.shape
    Hkv, Sk = k.shape[1], k.shape[2]
    p = BackwardParams()
    p.q, p.k, p.v, p.o, p.lse, p.dout = _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout)
    p.dq, p.dk, p.dv = _ptr(dq), _ptr(dk), _ptr(dv)
    p.batch, p.num_q_heads, p.num_kv_heads, p.head_dim, p.seqlen_q, p.seqlen_k = B, Hq, Hkv, D, Sq, Sk
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("do", dout), ("dq", dq), ("dk", dk), ("dv", dv)):
        setattr(p, f"{name}_batch_stride", t.stride(0))
        setattr(p, f"{name}_head_stride", t.stride(1))
        setattr(p, f"{name}_row_stride", t.stride(2))
    p.scale = float(scale if scale is not None else 1.0 / math.sqrt(D))
    p.causal, p.o_dtype, p.grad_dtype = int(bool(causal)), _out_code(o.dtype), _out_code(dq.dtype)
    p.error_flags = _ptr(error_flags)
    return p


def prefill_backward(q, k, v, o, lse, dout, scale: float | None = None, causal: bool = False, dq=None, dk=None,
                     dv=None, grad_dtype=torch.float32, workspace=None, error_flags=None):
    """Gradients of :func:`prefill` (dense): returns ``(dQ, dK, dV)``.

    q, dout [B,Hq,Sq,D] bf16; k, v [B,Hkv,Sk,D] bf16; o [B,Hq,Sq,D] (bf16 or
    fp32) and lse [B,Hq,Sq] fp32 are the forward's outputs for the same
    inputs. The gradients are ``grad_dtype`` (fp32 or bf16) unless given.
    """
    _need(q.dim() == 4 and k.dim() == 4 and v.dim() == 4 and dout.dim() == 4 and o.dim() == 4, "4-D tensors")
    B, Hq, Sq, D = q.shape
    _need(tuple(v.shape) == tuple(k.shape) and k.shape[0] == B and k.shape[3] == D, "k/v shape")
    _need(tuple(o.shape) == tuple(q.shape) and tuple(dout.shape) == tuple(q.shape), "o/dout shape")
    for t in (q, k, v, dout):
        _need(t.dtype == torch.bfloat16 and t.is_cuda and t.stride(3) == 1, "bf16 CUDA, last dim contiguous")
    _need(o.dtype in (torch.bfloat16, torch.float32) and o.stride(3) == 1, "o bf16 or fp32")
    _need(lse.dtype == torch.float32 and lse.is_contiguous() and tuple(lse.shape) == (B, Hq, Sq), "lse [B,Hq,Sq]")
    if dq is None:
        dq = torch.empty(q.shape, dtype=grad_dtype, device=q.device)
    if dk is None:
        dk = torch.empty(k.shape, dtype=grad_dtype, device=q.device)
    if dv is None:
        dv = torch.empty(v.shape, dtype=grad_dtype, device=q.device)
    _need(dq.dtype == dk.dtype == dv.dtype, "one dtype for dq, dk, dv")
    p = _backward_params(q, k, v, o, lse, dout, dq, dk, dv, scale, causal, error_flags)
    need = ctypes.c_size_t(0)
    _check(LIB.attn_prefill_backward(ctypes.byref(p), None, 0, ctypes.byref(need), None), "attn_prefill_backward(size)")
    if workspace is None and need.value > 0:
        workspace = torch.empty(need.value, dtype=torch.uint8, device=q.device)
    ws_ptr = _ptr(workspace) if workspace is not None else ctypes.c_void_p(0)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(LIB.attn_prefill_backward(ctypes.byref(p), ws_ptr, ws_bytes, None, _stream(q.device)),
           "attn_prefill_backward")
    return dq, dk, dv


def prefill_paged(q, k_cache, v_cache, block_table, seqlens_k, seqlens_q=None, scale: float | None = None,
                  causal: bool = True, out=None, lse=None, out_dtype=torch.bfloat16, want_lse: bool = True,
                  error_flags=None, cu_seqlens_q=None, max_seqlen_q=None):
    """Prefill of query chunks against a paged KV cache (chunked prefill).

    q [B,Hq,Sq,D] bf16 (rows past seqlens_q[b] are not written), or packed
    [total_q,Hq,D] with cu_seqlens_q / max_seqlen_q as in :func:`prefill`;
    k_cache/v_cache [NB,Hkv,16,D] bf16; block_table [B,max_blocks] int32;
    seqlens_k [B] int32: cached keys of each sequence, the chunk's own keys
    included (bottom-right causal alignment). Returns ``(O, LSE)``.
    """
    _need(k_cache.dim() == 4 and v_cache.shape == k_cache.shape, "shapes")
    NB, Hkv, BS, D = k_cache.shape
    B = block_table.shape[0]
    _need(q.shape[-1] == D and k_cache.dtype == torch.bfloat16 and v_cache.dtype == torch.bfloat16,
          "bf16 caches of q's head_dim")
    _need(k_cache.is_contiguous() and v_cache.is_contiguous(), "contiguous caches")
    _need(block_table.dtype == torch.int32 and block_table.is_contiguous() and block_table.shape[0] == B,
          "int32 block table [B, max_blocks]")
    _need(seqlens_k.dtype == torch.int32 and seqlens_k.numel() == B, "int32 seqlens_k [B]")
    if seqlens_q is not None:
        _need(seqlens_q.dtype == torch.int32 and seqlens_q.numel() == B, "int32 seqlens_q [B]")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    p = PrefillParams()
    out, lse = _queries(p, q, out, lse, out_dtype, want_lse, B, cu_seqlens_q, max_seqlen_q)
    p.k_cache, p.v_cache, p.block_table = _ptr(k_cache), _ptr(v_cache), _ptr(block_table)
    p.seqlens_k, p.seqlens_q = _ptr(seqlens_k), _ptr(seqlens_q)
    p.batch, p.num_kv_heads = B, Hkv
    p.seqlen_k = block_table.shape[1] * BS  # upper bound of seqlens_k
    p.max_blocks_per_seq, p.num_blocks, p.block_size = block_table.shape[1], NB, BS
    p.scale, p.causal = float(scale), int(bool(causal))
    p.error_flags = _ptr(error_flags)
    _check(LIB.attn_prefill(ctypes.byref(p), _stream(q.device)), "attn_prefill(paged)")
    return out, lse


# ----------------------------------------------------------------------------
# decode
# ----------------------------------------------------------------------------


def _is_fp8(t) -> bool:
    return t.dtype in (torch.uint8, torch.float8_e4m3fn)


def _decode_params(q, k_cache, v_cache, block_table, seq_lens, scale, max_seq_len, num_splits, out, lse,
                   error_flags, k_scale=None, v_scale=None):
    B, Hq, D = q.shape
    NB, Hkv, BS, D2 = k_cache.shape
    p = DecodeParams()
    p.q, p.k_cache, p.v_cache = _ptr(q), _ptr(k_cache), _ptr(v_cache)
    p.block_table, p.seq_lens, p.o, p.lse = _ptr(block_table), _ptr(seq_lens), _ptr(out), _ptr(lse)
    p.batch, p.num_q_heads, p.num_kv_heads, p.head_dim = B, Hq, Hkv, D
    p.block_size, p.max_blocks_per_seq, p.num_blocks = BS, block_table.shape[1], NB
    p.max_seq_len, p.num_splits = int(max_seq_len), int(num_splits)
    p.scale = float(scale if scale is not None else 1.0 / math.sqrt(D))
    p.o_dtype = _out_code(out.dtype) if out is not None else ATTN_DTYPE_BF16
    p.error_flags = _ptr(error_flags)
    if _is_fp8(k_cache):
        p.kv_dtype = ATTN_DTYPE_FP8_E4M3
        p.k_scale, p.v_scale = float(k_scale if k_scale is not None else 1.0), float(v_scale if v_scale is not None else 1.0)
    return p


def _check_decode_inputs(q, k_cache, v_cache, block_table, seq_lens, allow_fp8=True):
    _need(q.dim() == 3 and k_cache.dim() == 4 and v_cache.shape == k_cache.shape, "shapes")
    ok_cache = k_cache.dtype == torch.bfloat16 or (allow_fp8 and _is_fp8(k_cache))
    _need(q.dtype == torch.bfloat16 and k_cache.dtype == v_cache.dtype and ok_cache,
          "bf16 q; bf16 or FP8 E4M3 caches" if allow_fp8 else "bf16 q and caches")
    _need(q.is_contiguous() and k_cache.is_contiguous() and v_cache.is_contiguous(), "contiguous q and caches")
    _need(block_table.dtype == torch.int32 and block_table.is_contiguous() and block_table.dim() == 2,
          "int32 block table [B, max_blocks]")
    _need(seq_lens.dtype == torch.int32 and seq_lens.numel() == q.shape[0], "int32 seq_lens [B]")


def decode_workspace_bytes(q, k_cache, v_cache, block_table, seq_lens, max_seq_len: int = 0,
                           num_splits: int = 0) -> int:
    """Bytes of workspace :func:`decode_paged` needs for these shapes."""
    p = _decode_params(q, k_cache, v_cache, block_table, seq_lens, None, max_seq_len, num_splits, q, None, None)
    need = ctypes.c_size_t(0)
    _check(LIB.attn_decode_paged(ctypes.byref(p), None, 0, ctypes.byref(need), None), "attn_decode_paged(size)")
    return int(need.value)


def decode_paged(q, k_cache, v_cache, block_table, seq_lens, scale: float | None = None, max_seq_len: int = 0,
                 num_splits: int = 0, out=None, lse=None, workspace=None, out_dtype=torch.bfloat16,
                 want_lse: bool = True, error_flags=None, k_scale=None, v_scale=None):
    """Flash-Decoding over a paged KV cache.

    q [B,Hq,D] bf16; k_cache/v_cache [NB,Hkv,16,D] bf16, or FP8 E4M3 codes
    (torch.uint8 or torch.float8_e4m3fn) standing for code * k_scale and
    code * v_scale; block_table [B,maxblk] int32; seq_lens [B] int32 (all
    CUDA). ``max_seq_len`` is a host-side upper bound of seq_lens used for the
    split plan (0 = table capacity). Returns ``(O [B,Hq,D], LSE [B,Hq] or None)``.
    """
    _check_decode_inputs(q, k_cache, v_cache, block_table, seq_lens)
    B, Hq, D = q.shape
    if out is None:
        out = torch.empty((B, Hq, D), dtype=out_dtype, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    p = _decode_params(q, k_cache, v_cache, block_table, seq_lens, scale, max_seq_len, num_splits, out, lse,
                       error_flags, k_scale, v_scale)
    need = ctypes.c_size_t(0)
    _check(LIB.attn_decode_paged(ctypes.byref(p), None, 0, ctypes.byref(need), None), "attn_decode_paged(size)")
    if workspace is None and need.value > 0:
        workspace = torch.empty(need.value, dtype=torch.uint8, device=q.device)
    ws_ptr = _ptr(workspace) if workspace is not None else ctypes.c_void_p(0)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(LIB.attn_decode_paged(ctypes.byref(p), ws_ptr, ws_bytes, None, _stream(q.device)),
           "attn_decode_paged")
    return out, lse


def decode_shared_prefix_workspace_bytes(q, k_cache, v_cache, block_table, seq_lens, prefix_len: int,
                                         max_seq_len: int = 0, num_splits: int = 0) -> int:
    """Bytes of workspace :func:`decode_paged_shared_prefix` needs for these shapes."""
    p = _decode_params(q, k_cache, v_cache, block_table, seq_lens, None, max_seq_len, num_splits, q, None, None)
    need = ctypes.c_size_t(0)
    _check(LIB.attn_decode_paged_shared_prefix(ctypes.byref(p), int(prefix_len), None, 0, ctypes.byref(need), None),
           "attn_decode_paged_shared_prefix(size)")
    return int(need.value)


def decode_paged_shared_prefix(q, k_cache, v_cache, block_table, seq_lens, prefix_len: int,
                               scale: float | None = None, max_seq_len: int = 0, num_splits: int = 0, out=None,
                               lse=None, workspace=None, out_dtype=torch.bfloat16, want_lse: bool = True,
                               error_flags=None):
    """:func:`decode_paged` for sequences that all start with the same
    ``prefix_len`` tokens (a multiple of 16), stored in the blocks listed
    first in sequence 0's table; the prefix is attended once per batch.

    Same tensors as :func:`decode_paged` (bf16 caches only). Returns
    ``(O [B,Hq,D], LSE [B,Hq] or None)``.
    """
    _check_decode_inputs(q, k_cache, v_cache, block_table, seq_lens, allow_fp8=False)
    B, Hq, D = q.shape
    if out is None:
        out = torch.empty((B, Hq, D), dtype=out_dtype, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    p = _decode_params(q, k_cache, v_cache, block_table, seq_lens, scale, max_seq_len, num_splits, out, lse,
                       error_flags)
    need = ctypes.c_size_t(0)
    _check(LIB.attn_decode_paged_shared_prefix(ctypes.byref(p), int(prefix_len), None, 0, ctypes.byref(need), None),
           "attn_decode_paged_shared_prefix(size)")
    if workspace is None and need.value > 0:
        workspace = torch.empty(need.value, dtype=torch.uint8, device=q.device)
    ws_ptr = _ptr(workspace) if workspace is not None else ctypes.c_void_p(0)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(LIB.attn_decode_paged_shared_prefix(ctypes.byref(p), int(prefix_len), ws_ptr, ws_bytes, None,
                                               _stream(q.device)), "attn_decode_paged_shared_prefix")
    return out, lse


def decode_paged_noalloc(q, k_cache, v_cache, block_table, seq_lens, out, lse=None, scale: float | None = None,
                         max_seq_len: int = 0, num_splits: int = 0, error_flags=None, k_scale=None, v_scale=None):
    """:func:`decode_paged` for callers that cannot allocate device memory.

    The caller passes every input and the outputs (``out`` [B,Hq,D] bf16 or
    fp32, ``lse`` [B,Hq] fp32 or None); the split partials go to a fixed 16 MiB
    array that the library owns on each GPU, so nothing is allocated here or in
    the library. Calls that overlap on the GPU race on that array.
    """
    _check_decode_inputs(q, k_cache, v_cache, block_table, seq_lens)
    _need(out is not None and tuple(out.shape) == tuple(q.shape) and out.is_contiguous(), "out [B, Hq, D]")
    p = _decode_params(q, k_cache, v_cache, block_table, seq_lens, scale, max_seq_len, num_splits, out, lse,
                       error_flags, k_scale, v_scale)
    _check(LIB.attn_decode_paged_noalloc(ctypes.byref(p), _stream(q.device)), "attn_decode_paged_noalloc")
    return out, lse


# ----------------------------------------------------------------------------
# combine
# ----------------------------------------------------------------------------


def splitkv_lse_combine(part_o, part_lse, splits_per_row=None, out=None, out_lse=None,
                        out_dtype=torch.float32):
    """Merge split partials. part_o [S, rows, D] fp32, part_lse [S, rows] fp32.

    Returns ``(O [rows, D], LSE [rows])``.
    """
    _need(part_o.dim() == 3 and part_lse.dim() == 2, "part_o [S, rows, D], part_lse [S, rows]")
    S, R, D = part_o.shape
    _need(tuple(part_lse.shape) == (S, R), "part_lse shape")
    _need(part_o.dtype == torch.float32 and part_lse.dtype == torch.float32, "fp32 partials")
    _need(part_o.is_contiguous() and part_lse.is_contiguous(), "contiguous partials")
    if splits_per_row is not None:
        _need(splits_per_row.dtype == torch.int32 and splits_per_row.numel() == R, "int32 splits_per_row [rows]")
    if out is None:
        out = torch.empty((R, D), dtype=out_dtype, device=part_o.device)
    if out_lse is None:
        out_lse = torch.empty((R,), dtype=torch.float32, device=part_o.device)
    _check(LIB.splitkv_lse_combine(_ptr(part_o), _ptr(part_lse), S, R, D, _ptr(splits_per_row), _ptr(out),
                                   _out_code(out.dtype), _ptr(out_lse), _stream(part_o.device)),
           "splitkv_lse_combine")
    return out, out_lse


# ----------------------------------------------------------------------------
# persistent decode and the decode graph pool
# ----------------------------------------------------------------------------


class PersistentDecode:
    """A resident decode kernel driven step by step from the host.

    The tensors are the static buffers every step reads and writes (as for
    :func:`decode_paged`; ``out`` and, optionally, ``lse`` are written). The
    buffers hold up to ``q.shape[0]`` sequences; ``max_seq_len`` bounds every
    step's lengths (0: the table capacity). The kernel is launched on
    ``stream`` (a non-blocking torch stream by default) and runs until
    :meth:`stop`, or until ``idle_cycles`` SM cycles pass without a step.
    While it runs it holds every SM, so kernels of other streams wait; fill
    the static buffers with copies (copy engines), not kernels.
    """

    def __init__(self, q, k_cache, v_cache, block_table, seq_lens, out, lse=None, scale=None, max_seq_len=0,
                 num_splits=0, idle_cycles=2_000_000_000, error_flags=None, k_scale=None, v_scale=None,
                 stream=None):
        _check_decode_inputs(q, k_cache, v_cache, block_table, seq_lens)
        _need(out is not None and tuple(out.shape) == tuple(q.shape) and out.is_contiguous(), "out [B, Hq, D]")
        self._keep = (q, k_cache, v_cache, block_table, seq_lens, out, lse, error_flags)
        self.params = _decode_params(q, k_cache, v_cache, block_table, seq_lens, scale, max_seq_len, num_splits,
                                     out, lse, error_flags, k_scale, v_scale)
        need = ctypes.c_size_t(0)
        _check(LIB.attn_decode_persistent_workspace(ctypes.byref(self.params), ctypes.byref(need)),
               "attn_decode_persistent_workspace")
        self.workspace = torch.empty(max(int(need.value), 256), dtype=torch.uint8, device=q.device)
        self.cmd_buf = torch.zeros(ctypes.sizeof(PersistentCmd) // 4, dtype=torch.int32, pin_memory=True)
        self.cmd = PersistentCmd.from_address(self.cmd_buf.data_ptr())
        self.stream = stream if stream is not None else torch.cuda.Stream(device=q.device)
        self._cmd_ptr = ctypes.c_void_p(self.cmd_buf.data_ptr())
        _check(LIB.attn_decode_persistent_launch(ctypes.byref(self.params), self._cmd_ptr, _ptr(self.workspace),
                                                 self.workspace.numel(), int(idle_cycles),
                                                 ctypes.c_void_p(self.stream.cuda_stream)),
               "attn_decode_persistent_launch")

    def submit(self, batch: int, max_seq_len: int = 0) -> int:
        """Start a step over the first ``batch`` sequences of the static buffers; returns its number."""
        step = ctypes.c_int32(0)
        _check(LIB.attn_decode_persistent_submit(self._cmd_ptr, int(batch), int(max_seq_len), ctypes.byref(step)),
               "attn_decode_persistent_submit")
        return int(step.value)

    def wait(self, step: int, timeout_s: float = 10.0) -> None:
        """Block the host until step ``step`` is complete (its outputs are in HBM)."""
        _check(LIB.attn_decode_persistent_wait(self._cmd_ptr, int(step), int(timeout_s * 1e6)),
               "attn_decode_persistent_wait")

    def step(self, batch: int, max_seq_len: int = 0, timeout_s: float = 10.0) -> int:
        s = self.submit(batch, max_seq_len)
        self.wait(s, timeout_s)
        return s

    @property
    def status(self) -> int:
        return int(self.cmd.status)

    @property
    def running(self) -> bool:
        return bool(self.cmd.running)

    def stop(self) -> None:
        """Ask the kernel to exit and wait for its stream."""
        LIB.attn_decode_persistent_stop(self._cmd_ptr)
        self.stream.synchronize()


class DecodeGraphPool:
    """CUDA graphs of the decode step, one per (batch bucket, length bucket).

    The tensors are the static buffers every replay reads and writes (as for
    :func:`decode_paged`); the buckets are ascending lists. :meth:`replay`
    launches the smallest bucket covering a step on the current stream; rows
    of the static buffers past the step's batch must keep seq_lens 0.
    """

    def __init__(self, q, k_cache, v_cache, block_table, seq_lens, out, lse, batch_buckets, len_buckets,
                 scale=None, num_splits=0, error_flags=None, k_scale=None, v_scale=None):
        _check_decode_inputs(q, k_cache, v_cache, block_table, seq_lens)
        _need(out is not None and tuple(out.shape) == tuple(q.shape) and out.is_contiguous(), "out [B, Hq, D]")
        self._keep = (q, k_cache, v_cache, block_table, seq_lens, out, lse, error_flags)
        self.params = _decode_params(q, k_cache, v_cache, block_table, seq_lens, scale, 0, num_splits, out, lse,
                                     error_flags, k_scale, v_scale)
        bb = (ctypes.c_int32 * len(batch_buckets))(*batch_buckets)
        lb = (ctypes.c_int32 * len(len_buckets))(*len_buckets)
        need = ctypes.c_size_t(0)
        _check(LIB.attn_decode_graph_pool_workspace(ctypes.byref(self.params), bb, len(batch_buckets), lb,
                                                    len(len_buckets), ctypes.byref(need)),
               "attn_decode_graph_pool_workspace")
        self.workspace = torch.empty(max(int(need.value), 256), dtype=torch.uint8, device=q.device)
        handle = ctypes.c_void_p(0)
        _check(LIB.attn_decode_graph_pool_create(ctypes.byref(self.params), bb, len(batch_buckets), lb,
                                                 len(len_buckets), _ptr(self.workspace), self.workspace.numel(),
                                                 ctypes.byref(handle)), "attn_decode_graph_pool_create")
        self._handle = handle

    def replay(self, batch: int, max_seq_len: int = 0):
        """Replay the bucket covering (batch, max_seq_len) on the current stream; returns that bucket."""
        bb, bl = ctypes.c_int32(0), ctypes.c_int32(0)
        _check(LIB.attn_decode_graph_pool_replay(self._handle, int(batch), int(max_seq_len),
                                                 _stream(self._keep[0].device), ctypes.byref(bb), ctypes.byref(bl)),
               "attn_decode_graph_pool_replay")
        return int(bb.value), int(bl.value)

    def close(self) -> None:
        if self._handle:
            LIB.attn_decode_graph_pool_destroy(self._handle)
            self._handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
