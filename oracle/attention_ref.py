"""Plain, slow, fp64 reference for exact attention (the oracle).

TEST INFRASTRUCTURE: only tests, ``__graft_entry__.smoke()`` and the bench's
CPU-baseline / reference legs may import this module. It shares no code with
the CUDA path.

What it computes. The pages state that FlashAttention does not change the
mathematical definition of attention: tiling, online softmax and fusion reach
exactly the result of the standard computation ("推理加速" interview notes,
section FlashAttention and "它到底优化了什么"). So the oracle is that standard
computation written out, with S materialised ("抱infra脚", section "Flash
Attention 核心技术", the naive workflow S -> P -> O):

    S = scale * Q K^T          (one query head, its key/value head)
    S[i, j] = -inf             where causal and key j lies after query i
    m_i = max_j S[i, j];  P = exp(S - m);  l_i = sum_j P[i, j]
    O = P V / l;          LSE_i = m_i + ln l_i   (natural log)

* Key/value heads are shared by contiguous groups of query heads: query head h
  reads key/value head h // G with G = Hq / Hkv ("5.2 推理加速的未来趋势",
  GQA/MQA paragraph).
* Causal alignment is bottom-right: with Sq queries and Sk keys, query i sits
  at absolute position i + (Sk - Sq) and sees keys 0 .. i + (Sk - Sq). This
  is the reading for a prompt chunk appended to cached context ("抱infra脚",
  Chunked Prefill); it equals the usual top-left mask when Sq == Sk.
* A row that sees no key has O = 0 and LSE = -inf.
* Paged KV: token t of sequence b is in physical block table[b, t // 16] at
  slot t % 16 ("抱infra脚", Paged Attention: fixed-size blocks mapped through
  a block table). The oracle gathers the logical sequence, then applies the
  dense definition. It never splits the key range.
* Split-KV partials are merged with the log-sum-exp weights: with
  M = max_s LSE_s, LSE = M + ln sum_s exp(LSE_s - M) and
  O = sum_s exp(LSE_s - LSE) O_s ("GPU Kernel 调度:大模型推理的拐点 2026",
  Flash Decoding section: partial output / max / sum per chunk merged by the
  online-softmax formula, each partial carrying a log-sum-exp in FP32).

Backward. The pages count a forward and a backward kernel for FlashAttention-2
("GPU Kernel 调度:大模型推理的拐点 2026", the four-layer decomposition) and ask
that both match a reference implementation (same page, checklist item 1),
without writing the gradients out. They are the plain derivatives of the
definition above for an upstream gradient dO (per query head, with P the
normalised probabilities and masked entries 0):

    dV = P^T dO            dP = dO V^T
    D_i = sum_j P[i, j] dP[i, j]  ( = sum_d dO[i, d] O[i, d] )
    dS = P * (dP - D)      dQ = scale * dS K      dK = scale * dS^T Q

dK and dV of a key/value head sum the contributions of its G query heads.
Pins: torch autograd in fp64 through a softmax written with torch ops,
central finite differences, closed forms (one key; zero queries) and GQA vs
MHA with repeated K/V.

Block-sparse attention (BSR: query blocks see listed key blocks, the
FlashInfer abstraction, "抱infra脚", FlashInfer) is the same definition with
S = -inf outside the listed blocks. Pins: every block listed equals dense
attention, and each query block equals dense attention over its gathered
key blocks.

Pins (tests/test_oracle.py): brute-force ``math.fsum`` loops on tiny inputs,
closed forms (one key, causal row 0, zero query, constant V, hand-derived
weights), torch's fp64 CPU ``scaled_dot_product_attention`` with repeated
K/V, and invariants (key permutation, split-and-combine, paged vs contiguous,
GQA vs repeated MHA). No function here is "parity unpinned".

FP8 KV cache ("5.2 推理加速的未来趋势：新算法、新硬件、新协同", 协同层 section:
an FP8 KV cache halves its memory at almost no accuracy cost). The pages give
no format details or scale convention; the reading taken here is the OCP
E4M3 format without infinities (sign, 4 exponent bits with bias 7, 3 mantissa
bits; S.1111.111 is NaN) and one scale per tensor: a cached code c stands for
decode(c) * k_scale (keys) or decode(c) * v_scale (values). Pins: decoded
values of hand-checked codes, every code against torch's float8_e4m3fn, and
FP8 decode equal to the bf16-style definition on the dequantised values.
"""
from __future__ import annotations

import numpy as np

BLOCK_SIZE = 16


def bf16_bits_to_f64(bits) -> np.ndarray:
    """Decode bf16 bit patterns (uint16) exactly into float64."""
    u = np.asarray(bits).astype(np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def e4m3_bits_to_f64(bits) -> np.ndarray:
    """Decode FP8 E4M3 codes (uint8) exactly into float64.

    Bit 7 is the sign, bits 6..3 the exponent e (bias 7), bits 2..0 the
    mantissa m: e == 0 gives the subnormal m / 8 * 2^-6, otherwise the value
    is (1 + m / 8) * 2^(e - 7); e == 15 with m == 7 is NaN (no infinities).
    """
    b = np.asarray(bits).astype(np.int64)
    sign = np.where((b & 0x80) != 0, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = (b & 0x7).astype(np.float64)
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    return np.where((e == 15) & (b & 0x7 == 7), np.nan, sign * mag)


def _as_f64(x) -> np.ndarray:
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return bf16_bits_to_f64(x)
    return x.astype(np.float64)


def softmax_probs(q, k, scale, q_pos=None):
    """Materialised P = softmax(scale * q k^T + mask) for one head.

    ``q`` [n, D], ``k`` [Sk, D]; ``q_pos`` (absolute query positions) turns on
    the causal mask: key j is visible to query i when j <= q_pos[i].
    Returns ``(P, m, l)`` with ``m`` the row max of the masked scores and ``l``
    the row sum of exp(S - m). Rows with no visible key get P = 0, m = -inf,
    l = 0.
    """
    q = _as_f64(q)
    k = _as_f64(k)
    s = scale * (q @ k.T)
    if q_pos is not None:
        j = np.arange(k.shape[0])[None, :]
        s = np.where(j <= np.asarray(q_pos)[:, None], s, -np.inf)
    m = s.max(axis=1) if s.shape[1] else np.full(s.shape[0], -np.inf)
    empty = ~np.isfinite(m)
    m_safe = np.where(empty, 0.0, m)
    p = np.exp(s - m_safe[:, None])
    p[empty] = 0.0
    l = p.sum(axis=1)
    return p, m, l


def attention_rows(q, k, v, scale, q_pos=None):
    """Attention for a set of query rows against one key/value sequence.

    ``q`` [n, D]; ``k``, ``v`` [Sk, D]; ``q_pos`` as in :func:`softmax_probs`
    (None = no mask). Returns ``(O [n, D], LSE [n])`` in fp64.
    """
    v = _as_f64(v)
    p, m, l = softmax_probs(q, k, scale, q_pos)
    empty = l == 0.0
    l_safe = np.where(empty, 1.0, l)
    o = (p @ v) / l_safe[:, None]
    o[empty] = 0.0
    with np.errstate(divide="ignore"):
        lse = np.where(empty, -np.inf, m + np.log(l_safe))
    return o, lse


def causal_positions(seqlen_q: int, seqlen_k: int) -> np.ndarray:
    """Absolute positions of the queries under bottom-right alignment."""
    return np.arange(seqlen_q) + (seqlen_k - seqlen_q)


def ref_attention(q, k, v, scale, causal, rows=None):
    """Dense reference. Q [B,Hq,Sq,D], K/V [B,Hkv,Sk,D] (bf16 bits or floats).

    ``rows`` optionally restricts the computation to a list of
    ``(b, h, i)`` query rows; then the result is ``(O [n, D], LSE [n])``.
    Otherwise returns ``(O [B,Hq,Sq,D], LSE [B,Hq,Sq])``.
    """
    q = np.asarray(q)
    B, Hq, Sq, D = q.shape
    Hkv, Sk = np.asarray(k).shape[1], np.asarray(k).shape[2]
    if Hq % Hkv:
        raise ValueError("query heads must be a multiple of key/value heads")
    G = Hq // Hkv
    pos = causal_positions(Sq, Sk)
    if rows is not None:
        out_o = np.zeros((len(rows), D))
        out_l = np.zeros(len(rows))
        for n, (b, h, i) in enumerate(rows):
            o, lse = attention_rows(_as_f64(q[b, h, i:i + 1]), k[b, h // G], v[b, h // G], scale,
                                    pos[i:i + 1] if causal else None)
            out_o[n], out_l[n] = o[0], lse[0]
        return out_o, out_l
    O = np.zeros((B, Hq, Sq, D))
    L = np.zeros((B, Hq, Sq))
    for b in range(B):
        for h in range(Hq):
            O[b, h], L[b, h] = attention_rows(q[b, h], k[b, h // G], v[b, h // G], scale,
                                              pos if causal else None)
    return O, L


def ref_attention_backward(q, k, v, do, scale, causal):
    """Gradients of O = softmax(scale Q K^T + causal mask) V for upstream dO.

    q, do [B, Hq, Sq, D]; k, v [B, Hkv, Sk, D] (bf16 bits or floats). Returns
    a dict of fp64 arrays: dq [B, Hq, Sq, D], dk and dv [B, Hkv, Sk, D], plus
    the forward o, lse [B, Hq, Sq] and delta [B, Hq, Sq] (= rowsum(dO * O)).
    Rows that see no key contribute nothing (P = 0).
    """
    q, k, v, do = (_as_f64(x) for x in (q, k, v, do))
    B, Hq, Sq, D = q.shape
    Hkv, Sk = k.shape[1], k.shape[2]
    G = Hq // Hkv
    pos = causal_positions(Sq, Sk) if causal else None
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    o = np.zeros_like(q)
    lse = np.full((B, Hq, Sq), -np.inf)
    delta = np.zeros((B, Hq, Sq))
    for b in range(B):
        for h in range(Hq):
            kvh = h // G
            p, m, l = softmax_probs(q[b, h], k[b, kvh], scale, pos)
            seen = l > 0.0
            P = p / np.where(seen, l, 1.0)[:, None]
            with np.errstate(divide="ignore"):
                lse[b, h] = np.where(seen, m + np.log(np.where(seen, l, 1.0)), -np.inf)
            o[b, h] = P @ v[b, kvh]
            dv[b, kvh] += P.T @ do[b, h]
            dP = do[b, h] @ v[b, kvh].T
            delta[b, h] = (P * dP).sum(axis=1)
            dS = P * (dP - delta[b, h][:, None])
            dq[b, h] = scale * (dS @ k[b, kvh])
            dk[b, kvh] += scale * (dS.T @ q[b, h])
    return dict(dq=dq, dk=dk, dv=dv, o=o, lse=lse, delta=delta)


def ref_block_sparse_attention(q, k, v, indptr, indices, row_block, col_block, scale):
    """Attention with a block-sparse mask in BSR form, for one sequence.

    q [Hq, Sq, D]; k, v [Hkv, Sk, D]. Query rows are grouped in blocks of
    ``row_block`` rows and keys in blocks of ``col_block`` keys; query block r
    sees exactly the key blocks ``indices[indptr[r]:indptr[r + 1]]`` (every
    key of those blocks below Sk) and no other key. The block-sparse format
    is the FlashInfer unified abstraction ("抱infra脚", FlashInfer). Written
    out as the dense definition with S = -inf outside the mask. Returns
    O [Hq, Sq, D] and LSE [Hq, Sq] (a row with no visible key: 0 and -inf).
    """
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    Hq, Sq, D = q.shape
    Hkv, Sk = k.shape[0], k.shape[1]
    G = Hq // Hkv
    visible = np.zeros((Sq, Sk), dtype=bool)
    for i in range(Sq):
        r = i // row_block
        for c in indices[indptr[r]:indptr[r + 1]]:
            visible[i, c * col_block:min((c + 1) * col_block, Sk)] = True
    O = np.zeros((Hq, Sq, D))
    L = np.full((Hq, Sq), -np.inf)
    for h in range(Hq):
        s = scale * (q[h] @ k[h // G].T)
        s = np.where(visible, s, -np.inf)
        for i in range(Sq):
            if not visible[i].any():
                continue
            m = s[i].max()
            p = np.exp(s[i] - m)
            l = p.sum()
            O[h, i] = (p @ v[h // G]) / l
            L[h, i] = m + np.log(l)
    return O, L


def gather_paged(pool, block_table_row, length: int, kv_head: int) -> np.ndarray:
    """Logical [length, D] keys (or values) of one sequence and KV head.

    Token t comes from ``pool[block_table_row[t // 16], kv_head, t % 16]``.
    The result keeps the pool's dtype (bf16 bits stay bits).
    """
    pool = np.asarray(pool)
    t = np.arange(length)
    phys = np.asarray(block_table_row)[t // BLOCK_SIZE]
    return pool[phys, kv_head, t % BLOCK_SIZE]


def ref_decode_paged(q, k_pool, v_pool, block_table, seq_lens, scale, rows=None):
    """Decode: one query token per sequence; all ``seq_lens[b]`` cached keys visible.

    q [B, Hq, D]; pools [NB, Hkv, 16, D]. Returns O [B, Hq, D], LSE [B, Hq]
    (or, with ``rows`` = list of (b, h), arrays over those rows).
    """
    q = np.asarray(q)
    B, Hq, D = q.shape
    Hkv = np.asarray(k_pool).shape[1]
    G = Hq // Hkv
    todo = rows if rows is not None else [(b, h) for b in range(B) for h in range(Hq)]
    O = np.zeros((len(todo), D))
    L = np.zeros(len(todo))
    cache = {}
    for n, (b, h) in enumerate(todo):
        key = (b, h // G)
        if key not in cache:
            cache.clear()
            kk = gather_paged(k_pool, block_table[b], int(seq_lens[b]), h // G)
            vv = gather_paged(v_pool, block_table[b], int(seq_lens[b]), h // G)
            cache[key] = (kk, vv)
        kk, vv = cache[key]
        o, lse = attention_rows(_as_f64(q[b, h][None]), kk, vv, scale, None)
        O[n], L[n] = o[0], lse[0]
    if rows is None:
        return O.reshape(B, Hq, D), L.reshape(B, Hq)
    return O, L


def ref_decode_paged_fp8(q, k_pool, v_pool, k_scale, v_scale, block_table, seq_lens, scale, rows=None):
    """Decode over an FP8 E4M3 cache with one scale per tensor.

    Pools hold uint8 codes [NB, Hkv, 16, D]; the cached key (value) is
    decode(code) * k_scale (v_scale). Each sequence's codes are gathered and
    decoded, then the decode definition above applies unchanged. Returns O
    [B, Hq, D], LSE [B, Hq] (or arrays over ``rows`` = list of (b, h)).
    """
    q = np.asarray(q)
    B, Hq, D = q.shape
    G = Hq // np.asarray(k_pool).shape[1]
    todo = rows if rows is not None else [(b, h) for b in range(B) for h in range(Hq)]
    O = np.zeros((len(todo), D))
    L = np.zeros(len(todo))
    for n, (b, h) in enumerate(todo):
        kk = e4m3_bits_to_f64(gather_paged(k_pool, block_table[b], int(seq_lens[b]), h // G)) * float(k_scale)
        vv = e4m3_bits_to_f64(gather_paged(v_pool, block_table[b], int(seq_lens[b]), h // G)) * float(v_scale)
        o, lse = attention_rows(_as_f64(q[b, h][None]), kk, vv, scale, None)
        O[n], L[n] = o[0], lse[0]
    if rows is None:
        return O.reshape(B, Hq, D), L.reshape(B, Hq)
    return O, L


def ref_prefill_paged(q, q_lens, k_pool, v_pool, block_table, k_lens, scale, causal, rows=None):
    """Prefill of query chunks against paged keys/values.

    q [B, Hq, Sq_max, D] with ``q_lens[b]`` valid rows; sequence b has
    ``k_lens[b]`` cached keys (its own chunk included, so the chunk's queries
    sit at positions k_lens[b] - q_lens[b] + i under the causal mask).
    Returns O [B, Hq, Sq_max, D] and LSE [B, Hq, Sq_max] (rows past q_lens are
    zero / -inf), or arrays over ``rows`` = list of (b, h, i).
    """
    q = np.asarray(q)
    B, Hq, Sqm, D = q.shape
    Hkv = np.asarray(k_pool).shape[1]
    G = Hq // Hkv
    if rows is not None:
        O = np.zeros((len(rows), D))
        L = np.zeros(len(rows))
        for n, (b, h, i) in enumerate(rows):
            kk = gather_paged(k_pool, block_table[b], int(k_lens[b]), h // G)
            vv = gather_paged(v_pool, block_table[b], int(k_lens[b]), h // G)
            pos = causal_positions(int(q_lens[b]), int(k_lens[b]))[i:i + 1]
            o, lse = attention_rows(_as_f64(q[b, h, i:i + 1]), kk, vv, scale,
                                    pos if causal else None)
            O[n], L[n] = o[0], lse[0]
        return O, L
    O = np.zeros((B, Hq, Sqm, D))
    L = np.full((B, Hq, Sqm), -np.inf)
    for b in range(B):
        nq, nk = int(q_lens[b]), int(k_lens[b])
        pos = causal_positions(nq, nk)
        for kvh in range(Hkv):
            kk = gather_paged(k_pool, block_table[b], nk, kvh)
            vv = gather_paged(v_pool, block_table[b], nk, kvh)
            for h in range(kvh * G, (kvh + 1) * G):
                O[b, h, :nq], L[b, h, :nq] = attention_rows(
                    q[b, h, :nq], kk, vv, scale, pos if causal else None)
    return O, L


def combine_partials(part_o, part_lse, splits_per_row=None):
    """Merge split-KV partials by their log-sum-exp weights.

    ``part_o`` [S, rows, D] holds each split's normalised output, ``part_lse``
    [S, rows] its log-sum-exp (natural log; -inf for a split with no key).
    ``splits_per_row`` [rows] limits row r to its first splits. Returns
    ``(O [rows, D], LSE [rows])``; a row whose splits are all empty gets
    O = 0, LSE = -inf.
    """
    po = _as_f64(part_o)
    pl = _as_f64(part_lse)
    S, R, D = po.shape
    O = np.zeros((R, D))
    L = np.full(R, -np.inf)
    for r in range(R):
        n = S if splits_per_row is None else int(splits_per_row[r])
        lse = pl[:n, r]
        if n == 0 or not np.isfinite(lse).any():
            continue
        keep = np.isfinite(lse)  # an empty split (LSE = -inf) has weight 0; its output is not read
        M = lse[keep].max()
        w = np.exp(lse[keep] - M)
        L[r] = M + np.log(w.sum())
        wn = np.exp(lse[keep] - L[r])
        O[r] = (wn[:, None] * po[:n, r][keep]).sum(axis=0)
    return O, L
