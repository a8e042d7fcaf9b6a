"""Every row of a full-size workload through the oracle, in reasonable time.

Plumbing for the parity tests only: the arithmetic is the oracle's own
(``attention_rows``, ``ref_decode_paged``, ``ref_prefill_paged``), called
unchanged on independent pieces of the problem, and the pieces run on a pool
of threads (NumPy and BLAS release the GIL), one BLAS thread each.

Query rows are independent in the definition, so a head's rows are cut into
chunks. Under the causal mask a chunk's rows see no key past the chunk's last
query position: those keys are left out of the call, since a masked key adds
exactly 0 to the row max, the row sum and P V (its weight is exp(-inf) = 0).
Results equal the whole-head call up to BLAS summation order (~1e-16).
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

from oracle import attention_ref as ref

ROW_CHUNK = 256


def _pool():
    return ThreadPoolExecutor(max_workers=max(1, os.cpu_count() or 1))


def _blas_single_thread():
    from threadpoolctl import threadpool_limits
    return threadpool_limits(limits=1)


def prefill_all_rows(q, k, v, scale, causal):
    """Dense prefill oracle over every (batch, head, row): O [B,Hq,Sq,D], LSE [B,Hq,Sq]."""
    B, Hq, Sq, D = q.shape
    Hkv, Sk = k.shape[1], k.shape[2]
    G = Hq // Hkv
    pos = ref.causal_positions(Sq, Sk)
    O = np.zeros((B, Hq, Sq, D))
    L = np.zeros((B, Hq, Sq))

    def run(task):
        b, h, r0 = task
        r1 = min(r0 + ROW_CHUNK, Sq)
        kend = min(Sk, int(pos[r1 - 1]) + 1) if causal else Sk
        kend = max(kend, 0)
        O[b, h, r0:r1], L[b, h, r0:r1] = ref.attention_rows(
            q[b, h, r0:r1], k[b, h // G, :kend], v[b, h // G, :kend], scale, pos[r0:r1] if causal else None)

    tasks = [(b, h, r0) for b in range(B) for h in range(Hq) for r0 in range(0, Sq, ROW_CHUNK)]
    with _blas_single_thread(), _pool() as ex:
        list(ex.map(run, tasks))
    return O, L


def decode_all_rows(q, k_pool, v_pool, block_table, seq_lens, scale):
    """Paged decode oracle over every (sequence, head): O [B,Hq,D], LSE [B,Hq]."""
    B, Hq, D = q.shape
    O = np.zeros((B, Hq, D))
    L = np.zeros((B, Hq))

    def run(b):
        rows = [(b, h) for h in range(Hq)]
        o, lse = ref.ref_decode_paged(q, k_pool, v_pool, block_table, seq_lens, scale, rows=rows)
        O[b], L[b] = o, lse

    with _blas_single_thread(), _pool() as ex:
        list(ex.map(run, range(B)))
    return O, L


def prefill_paged_all_rows(q, q_lens, k_pool, v_pool, block_table, k_lens, scale, causal):
    """Paged prefill oracle, one sequence per task: O [B,Hq,Sqm,D], LSE [B,Hq,Sqm]."""
    B, Hq, Sqm, D = q.shape
    O = np.zeros((B, Hq, Sqm, D))
    L = np.full((B, Hq, Sqm), -np.inf)

    def run(b):
        o, lse = ref.ref_prefill_paged(q[b:b + 1], q_lens[b:b + 1], k_pool, v_pool, block_table[b:b + 1],
                                       k_lens[b:b + 1], scale, causal)
        O[b], L[b] = o[0], lse[0]

    with _blas_single_thread(), _pool() as ex:
        list(ex.map(run, range(B)))
    return O, L


def decode_fp8_all_rows(q, k_pool, v_pool, k_scale, v_scale, block_table, seq_lens, scale):
    """FP8-cache decode oracle over every (sequence, head): O [B,Hq,D], LSE [B,Hq]."""
    B, Hq, D = q.shape
    O = np.zeros((B, Hq, D))
    L = np.zeros((B, Hq))

    def run(b):
        rows = [(b, h) for h in range(Hq)]
        o, lse = ref.ref_decode_paged_fp8(q, k_pool, v_pool, k_scale, v_scale, block_table, seq_lens, scale,
                                          rows=rows)
        O[b], L[b] = o, lse

    with _blas_single_thread(), _pool() as ex:
        list(ex.map(run, range(B)))
    return O, L


def backward_all_heads(q, k, v, do, scale, causal):
    """Backward oracle, one (batch, key/value head) group per task: dq, dk, dv."""
    B, Hq, Sq, D = q.shape
    Hkv, Sk = k.shape[1], k.shape[2]
    G = Hq // Hkv
    out = dict(dq=np.zeros((B, Hq, Sq, D)), dk=np.zeros((B, Hkv, Sk, D)), dv=np.zeros((B, Hkv, Sk, D)))

    def run(task):
        b, kvh = task
        hs = slice(kvh * G, (kvh + 1) * G)
        r = ref.ref_attention_backward(q[b:b + 1, hs], k[b:b + 1, kvh:kvh + 1], v[b:b + 1, kvh:kvh + 1],
                                       do[b:b + 1, hs], scale, causal)
        out["dq"][b, hs] = r["dq"][0]
        out["dk"][b, kvh] = r["dk"][0, 0]
        out["dv"][b, kvh] = r["dv"][0, 0]

    with _blas_single_thread(), _pool() as ex:
        list(ex.map(run, [(b, kvh) for b in range(B) for kvh in range(Hkv)]))
    return out
