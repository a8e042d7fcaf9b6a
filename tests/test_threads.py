"""First calls from several host threads at once, in a fresh process: the
one-time kernel set-up (per device, under a lock) must be done exactly once
and every call must still be right."""
import os
import subprocess
import sys
import textwrap

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = textwrap.dedent("""
    import sys, threading
    sys.path.insert(0, {root!r})
    import numpy as np, torch
    from attention_tiled_exact_b200 import binding as attn, workloads as wl
    from oracle import attention_ref as ref
    torch.cuda.init()
    d = wl.make_prefill(wl.PrefillConfig("threads", 1, 8, 2, 300, 300, 128, True, 5))
    dd = wl.make_decode(wl.DecodeConfig("threads_dec", 3, 8, 2, 128, 1, 1, 6),
                        kv_lens=np.array([700, 33, 2000], dtype=np.int32))
    dev = lambda bits: torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()
    q, k, v = dev(d["q"]), dev(d["k"]), dev(d["v"])
    qd, kc, vc = dev(dd["q"]), dev(dd["k_pool"]), dev(dd["v_pool"])
    bt, sl = torch.from_numpy(dd["block_table"]).cuda(), torch.from_numpy(dd["kv_lens"]).cuda()
    torch.cuda.synchronize()
    go = threading.Barrier(8)
    out, errs = [None] * 8, []

    def work(i):
        try:
            s = torch.cuda.Stream()
            with torch.cuda.stream(s):
                go.wait()
                if i % 2 == 0:
                    o, l = attn.prefill(q, k, v, d["scale"], True, out_dtype=torch.float32)
                else:
                    o, l = attn.decode_paged(qd, kc, vc, bt, sl, dd["scale"], num_splits=3, out_dtype=torch.float32)
            s.synchronize()
            out[i] = (o.double().cpu().numpy(), l.double().cpu().numpy())
        except Exception as e:  # reported below
            errs.append(repr(e))

    ts = [threading.Thread(target=work, args=(i,)) for i in range(8)]
    [t.start() for t in ts]
    [t.join() for t in ts]
    assert not errs, errs
    Op, Lp = ref.ref_attention(d["q"], d["k"], d["v"], d["scale"], True)
    Od, Ld = ref.ref_decode_paged(dd["q"], dd["k_pool"], dd["v_pool"], dd["block_table"], dd["kv_lens"], dd["scale"])
    for i, (o, l) in enumerate(out):
        O, L = (Op, Lp) if i % 2 == 0 else (Od, Ld)
        assert np.abs(o - O).max() <= 1e-2 and np.abs(l - L).max() <= 1e-3, i
        assert np.array_equal(o, out[i % 2][0]), "same call, same bits"
    print("threads ok")
""")


@pytest.mark.gpu
def test_first_calls_from_eight_threads_in_a_fresh_process():
    r = subprocess.run([sys.executable, "-c", SCRIPT.format(root=ROOT)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and "threads ok" in r.stdout, r.stdout + r.stderr
