"""Runs the library's calls through the bounds-checking debug build and
prints one JSON line per case: the largest differences from the oracle and
the device error word.

Started by tests/test_debug_bounds.py in a child process with
ATTN_B200_DEBUG_BOUNDS=1 (the binding picks the library at import). With
``--plant`` every bounds-check site is planted in turn and the case that
reaches it is run: the word must then name that site while the outputs stay
those of the oracle (a planted check reports without changing the access).
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from attention_tiled_exact_b200 import binding as attn  # noqa: E402
from attention_tiled_exact_b200 import workloads as wl  # noqa: E402
from oracle import attention_ref as ref  # noqa: E402


def bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def i32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def f64(t):
    return t.double().cpu().numpy()


def case_prefill(flags, d_head=128, out_dtype=torch.float32):
    d = wl.make_prefill(wl.PrefillConfig("dbg_prefill", 1, 8, 2, 300, 300, d_head, True, 61 + d_head))
    o, lse = attn.prefill(bf16(d["q"]), bf16(d["k"]), bf16(d["v"]), d["scale"], True, out_dtype=out_dtype,
                          error_flags=flags)
    torch.cuda.synchronize()
    O, L = ref.ref_attention(d["q"], d["k"], d["v"], d["scale"], True)
    return np.abs(f64(o) - O).max(), np.abs(f64(lse) - L).max()


def case_prefill_bf16_out(flags):
    # bf16 output goes out through the staged tile stores
    d = wl.make_prefill(wl.PrefillConfig("dbg_prefill16", 1, 4, 2, 256, 256, 128, False, 65))
    o, lse = attn.prefill(bf16(d["q"]), bf16(d["k"]), bf16(d["v"]), d["scale"], False, error_flags=flags)
    torch.cuda.synchronize()
    O, L = ref.ref_attention(d["q"], d["k"], d["v"], d["scale"], False)
    return np.abs(f64(o) - O).max(), np.abs(f64(lse) - L).max()


def case_prefill_paged(flags):
    q_lens = np.array([200, 37], dtype=np.int32)
    k_lens = np.array([1000 + 200, 77 + 37], dtype=np.int32)  # neither a multiple of 16: ragged last blocks
    Hq, Hkv, D = 8, 2, 128
    pool = wl.make_paged_pool(67, k_lens, Hkv, D)
    q = wl.normal_bf16(67, (2, Hq, int(q_lens.max()), D), 30)
    scale = 1.0 / np.sqrt(D)
    o, lse = attn.prefill_paged(bf16(q), bf16(pool["k_pool"]), bf16(pool["v_pool"]), i32(pool["block_table"]),
                                i32(k_lens), i32(q_lens), scale, True, out_dtype=torch.float32, error_flags=flags)
    torch.cuda.synchronize()
    O, L = ref.ref_prefill_paged(q, q_lens, pool["k_pool"], pool["v_pool"], pool["block_table"], k_lens, scale,
                                 True)
    o, lse = f64(o), f64(lse)
    eo = max(np.abs(o[b, :, :q_lens[b]] - O[b, :, :q_lens[b]]).max() for b in range(2))
    el = max(np.abs(lse[b, :, :q_lens[b]] - L[b, :, :q_lens[b]]).max() for b in range(2))
    return eo, el


def case_decode(flags, fp8=False):
    cfg = wl.DecodeConfig("dbg_decode", 3, 8, 2, 128, 1, 1, 69)
    lens = np.array([700, 33, 3000], dtype=np.int32)
    d = wl.make_decode_fp8(cfg, kv_lens=lens) if fp8 else wl.make_decode(cfg, kv_lens=lens)
    kw = dict(k_scale=d["k_scale"], v_scale=d["v_scale"]) if fp8 else {}
    pools = (torch.from_numpy(d["k_pool"]).cuda(), torch.from_numpy(d["v_pool"]).cuda()) if fp8 else \
        (bf16(d["k_pool"]), bf16(d["v_pool"]))
    o, lse = attn.decode_paged(bf16(d["q"]), *pools, i32(d["block_table"]), i32(d["kv_lens"]), d["scale"],
                               num_splits=4, out_dtype=torch.float32, error_flags=flags, **kw)
    torch.cuda.synchronize()
    if fp8:
        O, L = ref.ref_decode_paged_fp8(d["q"], d["k_pool"], d["v_pool"], d["k_scale"], d["v_scale"],
                                        d["block_table"], d["kv_lens"], d["scale"])
    else:
        O, L = ref.ref_decode_paged(d["q"], d["k_pool"], d["v_pool"], d["block_table"], d["kv_lens"], d["scale"])
    return np.abs(f64(o) - O).max(), np.abs(f64(lse) - L).max()


def case_backward(flags):
    d = wl.make_prefill(wl.PrefillConfig("dbg_bwd", 1, 4, 2, 200, 200, 128, True, 71))
    do = wl.normal_bf16(71, d["q"].shape, 43)
    q, k, v = bf16(d["q"]), bf16(d["k"]), bf16(d["v"])
    o, lse = attn.prefill(q, k, v, d["scale"], True, out_dtype=torch.float32)
    grads = attn.prefill_backward(q, k, v, o, lse, bf16(do), d["scale"], True, error_flags=flags)
    torch.cuda.synchronize()
    r = ref.ref_attention_backward(d["q"], d["k"], d["v"], do, d["scale"], True)
    err = max(np.abs(f64(g) - r[n]).max() / np.abs(r[n]).max() for n, g in zip(("dq", "dk", "dv"), grads))
    return err, 0.0


CASES = {
    "prefill_d128": case_prefill,
    "prefill_d64": lambda f: case_prefill(f, 64),
    "prefill_bf16_out": case_prefill_bf16_out,
    "prefill_paged": case_prefill_paged,
    "decode": case_decode,
    "decode_fp8": lambda f: case_decode(f, True),
    "backward": case_backward,
}

# The case that reaches each site.
SITE_CASE = {
    "PREFILL_SMEM_Q": "prefill_d128", "PREFILL_SMEM_KV": "prefill_d128", "PREFILL_TABLE": "prefill_paged",
    "PREFILL_TMEM_S": "prefill_d128", "PREFILL_TMEM_O": "prefill_d128", "PREFILL_SMEM_STAGE": "prefill_bf16_out",
    "PREFILL_SMEM_VFIX": "prefill_paged", "PREFILL_OUT": "prefill_d128", "DECODE_TABLE": "decode",
    "DECODE_SMEM": "decode", "DECODE_PARTIAL": "decode", "COMBINE": "decode", "BWD_SMEM": "backward",
    "BWD_TMEM": "backward", "BWD_OUT": "backward",
}


def run(name, case, site=0):
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    attn.debug_plant_bounds(site)
    try:
        eo, el = case(flags)
    finally:
        attn.debug_plant_bounds(0)
    status, word = attn.sync_error_flags(flags)
    print(json.dumps({"case": name, "site": site, "err_o": float(eo), "err_lse": float(el), "word": int(word),
                      "status": int(status)}), flush=True)


def main():
    assert attn.debug_bounds_enabled(), "the debug library is not the one loaded"
    if "--plant" in sys.argv:
        for site_name, site in attn.BOUNDS_SITES.items():
            run(SITE_CASE[site_name], CASES[SITE_CASE[site_name]], site)
    else:
        for name, case in CASES.items():
            run(name, case)


if __name__ == "__main__":
    main()
