"""Exact scaled-dot-product attention for B200 (sm_100a).

A thin marshalling layer over the C-ABI library ``libattn_b200.so`` (every
step of the computation runs in its CUDA kernels):

* :func:`prefill` -- tiled causal / non-causal GQA prefill with online softmax;
* :func:`prefill_paged` -- the same over a block-table KV cache (chunked prefill);
* :func:`prefill_from_host` -- a dense prefill from and to host memory, its
  copies overlapped with the computation;
* :func:`prefill_backward` -- dQ, dK, dV of the dense prefill;
* :func:`decode_paged` -- split-KV decode over a block-table KV cache (bf16 or
  FP8 E4M3 cache), with :func:`decode_workspace_bytes` for its workspace;
* :func:`decode_paged_shared_prefix` -- decode of a batch sharing a prefix,
  which is attended once per batch (:func:`decode_shared_prefix_workspace_bytes`);
* :func:`decode_paged_noalloc` -- decode for callers that cannot allocate;
* :class:`PersistentDecode` -- a resident decode kernel driven step by step;
* :class:`DecodeGraphPool` -- CUDA graphs of the decode step per static shape;
* :func:`splitkv_lse_combine` -- log-sum-exp merge of split partials;
* :func:`sync_error_flags` / :func:`status_from_flags` -- the device error
  word as a status;
* :func:`debug_bounds_enabled` / :func:`debug_plant_bounds` -- the bounds-
  checking debug build (loaded with ``ATTN_B200_DEBUG_BOUNDS=1``).

The library is loaded on first use of one of these names; if it is missing
the import fails with an error that says how to build it. There is no CPU
fallback.
"""
_API = ("prefill", "prefill_paged", "prefill_from_host", "prefill_backward", "decode_paged", "decode_workspace_bytes",
        "decode_paged_shared_prefix", "decode_shared_prefix_workspace_bytes", "decode_paged_noalloc",
        "splitkv_lse_combine", "sync_error_flags", "status_from_flags", "set_wait_limit", "selftest_exp2",
        "debug_bounds_enabled", "debug_plant_bounds",
        "PersistentDecode", "DecodeGraphPool",
        "AttnError", "library_path", "status_string")


def __getattr__(name):
    if name in _API:
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)


__all__ = list(_API)
