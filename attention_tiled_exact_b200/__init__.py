"""Exact scaled-dot-product attention for B200 (sm_100a).

Three calls, each a thin marshalling layer over the C-ABI library
``libattn_b200.so`` (every step of the computation runs in its CUDA kernels):

* :func:`prefill` -- tiled causal / non-causal GQA prefill with online softmax;
* :func:`prefill_paged` -- the same over a block-table KV cache (chunked prefill);
* :func:`decode_paged` -- split-KV decode over a block-table KV cache;
* :func:`splitkv_lse_combine` -- log-sum-exp merge of split partials.

The library is loaded on first use of one of these names; if it is missing
the import fails with an error that says how to build it. There is no CPU
fallback.
"""
_API = ("prefill", "prefill_paged", "decode_paged", "decode_paged_noalloc", "splitkv_lse_combine", "decode_workspace_bytes",
        "AttnError", "library_path", "status_string")


def __getattr__(name):
    if name in _API:
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)


__all__ = list(_API)
