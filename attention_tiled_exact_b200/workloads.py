"""Seeded synthetic inputs for the attention workloads.

This module only draws random numbers and lays them out; it holds none of the
attention arithmetic. Both the CUDA path (through the tests and the bench) and
the fp64 oracle are fed from it, so it must stay free of anything that could
make the two sides agree by construction.

Conventions:

* Random values are NumPy PCG64 standard normals drawn in float32 and rounded
  to bfloat16 by round-to-nearest-even on the bit pattern. Tensors are returned
  as ``uint16`` arrays holding bf16 bit patterns.
* Large tensors are drawn in fixed-size chunks, each from its own child of
  ``SeedSequence(seed)``, so the values do not depend on the thread count.
* Paged KV pools use 16-token blocks ``[num_blocks, kv_heads, 16, head_dim]``
  addressed through a per-sequence block table. Physical blocks are a random
  permutation over a shared pool that has spare blocks. Spare blocks and the
  unused tail slots of each sequence's last block hold NaN, and unused table
  entries point at a NaN spare block, so a kernel that reads anything it should
  not read produces NaN instead of a plausible number.

The five workloads follow the problem statement: exact attention
``O = softmax(Q K^T * scale + causal mask) V`` with key/value heads shared by
groups of query heads, prefill over contiguous ``[B, H, S, D]`` tensors, and
decode / chunked prefill over a block-table KV cache ("vLLM - Paged Attention"
section of the infra interview-prep page; "Flash Decoding" section of the GPU
kernel scheduling post).
"""
from __future__ import annotations

import concurrent.futures as _cf
import dataclasses
import math
import os

import numpy as np

BLOCK_SIZE = 16
BF16_NAN = np.uint16(0x7FC0)
_CHUNK = 1 << 22  # elements per independently seeded chunk


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round-to-nearest-even) and return the bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = ((u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)).astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        r[nan] = BF16_NAN
    return r


def normal_bf16(seed: int, shape, stream: int = 0, threads: int | None = None) -> np.ndarray:
    """iid N(0,1) values rounded to bf16, as uint16 bits.

    ``stream`` selects an independent sub-stream of ``seed`` (Q, K and V of one
    workload use streams 0, 1 and 2). The tensor is filled chunk by chunk; chunk
    ``c`` uses child ``c`` of ``SeedSequence([seed, stream])``.
    """
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    nchunks = max(1, (n + _CHUNK - 1) // _CHUNK)
    children = np.random.SeedSequence([seed, stream]).spawn(nchunks)

    def fill(c):
        lo = c * _CHUNK
        hi = min(n, lo + _CHUNK)
        if hi <= lo:
            return
        rng = np.random.Generator(np.random.PCG64(children[c]))
        out[lo:hi] = f32_to_bf16_bits(rng.standard_normal(hi - lo, dtype=np.float32))

    threads = threads or min(16, os.cpu_count() or 1)
    if nchunks == 1 or threads == 1:
        for c in range(nchunks):
            fill(c)
    else:
        with _cf.ThreadPoolExecutor(threads) as ex:
            list(ex.map(fill, range(nchunks)))
    return out.reshape(shape)


# ----------------------------------------------------------------------------
# Workload descriptions
# ----------------------------------------------------------------------------


@dataclasses.dataclass(frozen=True)
class PrefillConfig:
    """Dense prefill: Q [B,Hq,Sq,D], K/V [B,Hkv,Sk,D], bf16."""

    name: str
    batch: int
    q_heads: int
    kv_heads: int
    seqlen_q: int
    seqlen_k: int
    head_dim: int
    causal: bool
    seed: int

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)


@dataclasses.dataclass(frozen=True)
class DecodeConfig:
    """Paged decode: one query token per sequence over a block-table KV cache."""

    name: str
    batch: int
    q_heads: int
    kv_heads: int
    head_dim: int
    len_lo: int
    len_hi: int
    seed: int
    spare_blocks: int = 64

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)


@dataclasses.dataclass(frozen=True)
class SharedPrefixConfig:
    """Paged decode where every sequence starts with the same prefix_len
    tokens (stored once), followed by suffix_lo..suffix_hi tokens of its own."""

    name: str
    batch: int
    q_heads: int
    kv_heads: int
    head_dim: int
    prefix_len: int
    suffix_lo: int
    suffix_hi: int
    seed: int
    spare_blocks: int = 64

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)


@dataclasses.dataclass(frozen=True)
class MixedConfig:
    """Chunked prefill on top of cached context, plus decode rows, paged KV."""

    name: str
    chunks: int
    chunk_len: int
    chunk_ctx_lo: int
    chunk_ctx_hi: int
    decodes: int
    dec_ctx_lo: int
    dec_ctx_hi: int
    q_heads: int
    kv_heads: int
    head_dim: int
    seed: int
    spare_blocks: int = 64

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)


TINY = PrefillConfig("tiny_noncausal_b1_h1_s128_d64", 1, 1, 1, 128, 128, 64, False, 0)
CAUSAL_GQA_2K = PrefillConfig("causal_gqa_b4_h32kv8_s2048_d128", 4, 32, 8, 2048, 2048, 128, True, 1)
CAUSAL_GQA_16K = PrefillConfig("causal_gqa_b1_h32kv8_s16384_d128", 1, 32, 8, 16384, 16384, 128, True, 2)
PAGED_DECODE = DecodeConfig("paged_decode_b64_h32kv8_d128_len1k_32k", 64, 32, 8, 128, 1024, 32768, 3)
MIXED = MixedConfig("mixed_8x512chunks_ctx0_8k_plus_128dec_ctx512_16k",
                    8, 512, 0, 8192, 128, 512, 16384, 32, 8, 128, 4)

SHARED_PREFIX_DECODE = SharedPrefixConfig("shared_prefix_decode_b64_h32kv8_d128_prefix8k_own64_2k",
                                          64, 32, 8, 128, 8192, 64, 2048, 5)
WORKLOADS = {c.name: c for c in (TINY, CAUSAL_GQA_2K, CAUSAL_GQA_16K, PAGED_DECODE, MIXED,
                                  SHARED_PREFIX_DECODE)}


# ----------------------------------------------------------------------------
# Generators
# ----------------------------------------------------------------------------


def make_prefill(cfg: PrefillConfig) -> dict:
    """Contiguous Q/K/V bf16 bit arrays in [B, H, S, D] layout."""
    q = normal_bf16(cfg.seed, (cfg.batch, cfg.q_heads, cfg.seqlen_q, cfg.head_dim), 0)
    k = normal_bf16(cfg.seed, (cfg.batch, cfg.kv_heads, cfg.seqlen_k, cfg.head_dim), 1)
    v = normal_bf16(cfg.seed, (cfg.batch, cfg.kv_heads, cfg.seqlen_k, cfg.head_dim), 2)
    return dict(q=q, k=k, v=v, scale=cfg.scale, causal=cfg.causal)


def random_lengths(seed: int, n: int, lo: int, hi: int, stream: int = 10) -> np.ndarray:
    """n integers uniform in [lo, hi] (inclusive), int32."""
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, stream])))
    return rng.integers(lo, hi + 1, size=n).astype(np.int32)


def make_block_tables(seed: int, kv_lens: np.ndarray, spare_blocks: int = 64,
                      stream: int = 11, identity: bool = False):
    """Random block tables over a shared pool.

    Returns ``(block_table [B, max_blocks] int32, num_blocks, spare_ids)``.
    Logical block ``j`` of sequence ``b`` lives in physical block
    ``block_table[b, j]``. Physical ids are a random permutation of the pool
    (or the identity when ``identity``). Entries past a sequence's last block
    point at a spare block (which holds NaN).
    """
    kv_lens = np.asarray(kv_lens, dtype=np.int64)
    nblk = (kv_lens + BLOCK_SIZE - 1) // BLOCK_SIZE
    used = int(nblk.sum())
    num_blocks = used + spare_blocks
    if identity:
        perm = np.arange(num_blocks, dtype=np.int64)
    else:
        rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, stream])))
        perm = rng.permutation(num_blocks)
    spare_ids = perm[used:]
    max_blocks = max(1, int(nblk.max()) if len(nblk) else 1)
    filler = int(spare_ids[0]) if spare_blocks > 0 else 0
    table = np.full((len(kv_lens), max_blocks), filler, dtype=np.int32)
    off = 0
    for b, n in enumerate(nblk):
        table[b, :n] = perm[off:off + n]
        off += n
    return table, num_blocks, spare_ids


def make_paged_pool(seed: int, kv_lens, kv_heads: int, head_dim: int, spare_blocks: int = 64,
                    identity: bool = False, stream_base: int = 1):
    """K/V pools [NB, Hkv, 16, D] (bf16 bits) plus block tables for ``kv_lens``.

    The pools are filled with N(0,1) values; spare blocks and the tail slots of
    each sequence's last block are then overwritten with NaN.
    """
    kv_lens = np.asarray(kv_lens, dtype=np.int32)
    table, nb, spare = make_block_tables(seed, kv_lens, spare_blocks, identity=identity)
    shape = (nb, kv_heads, BLOCK_SIZE, head_dim)
    k_pool = normal_bf16(seed, shape, stream_base)
    v_pool = normal_bf16(seed, shape, stream_base + 1)
    for pool in (k_pool, v_pool):
        pool[spare] = BF16_NAN
        for b, L in enumerate(kv_lens):
            tail = int(L) % BLOCK_SIZE
            if tail:
                last = table[b, (int(L) - 1) // BLOCK_SIZE]
                pool[last, :, tail:, :] = BF16_NAN
    return dict(k_pool=k_pool, v_pool=v_pool, block_table=table, num_blocks=nb,
                kv_lens=kv_lens, spare_ids=spare)


# FP8 E4M3 (OCP, no infinities): sign bit 7, exponent bits 6..3 with bias 7,
# mantissa bits 2..0; exponent 0 is subnormal (m / 8 * 2^-6); code 0x7F is NaN.
# The non-negative finite codes 0x00..0x7E in increasing order of value:
def _e4m3_table() -> np.ndarray:
    c = np.arange(0x7F)
    e, m = c >> 3, (c & 7).astype(np.float64)
    return np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))


_E4M3_VALUES = _e4m3_table()
FP8_NAN = np.uint8(0x7F)


def e4m3_codes(x) -> np.ndarray:
    """Round values to the nearest FP8 E4M3 code (ties to the even code),
    saturating at +-448; NaN maps to the NaN code."""
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), 448.0)
    hi = np.clip(np.searchsorted(_E4M3_VALUES, a, side="left"), 0, len(_E4M3_VALUES) - 1)
    lo = np.maximum(hi - 1, 0)
    d_lo, d_hi = a - _E4M3_VALUES[lo], _E4M3_VALUES[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo).astype(np.uint8)
    code = code | (np.signbit(x).astype(np.uint8) << 7)
    return np.where(np.isnan(x), FP8_NAN, code).astype(np.uint8)


def bf16_pool_to_e4m3(pool: np.ndarray, chunk: int = 1 << 24) -> tuple:
    """Quantise a bf16 pool (uint16 bits) to E4M3 codes with one scale,
    scale = max|x| / 448 over its finite entries; NaN entries get the NaN code.

    Each of the 65536 bf16 bit patterns is rounded once (a lookup table), so
    the pool itself is only gathered through the table, chunk by chunk.
    """
    flat = pool.reshape(-1)
    starts = range(0, flat.size, chunk)

    def chunk_amax(i):
        a = flat[i:i + chunk] & np.uint16(0x7FFF)
        return int(np.where(a < np.uint16(0x7F80), a, np.uint16(0)).max()) if a.size else 0  # finite only

    with _cf.ThreadPoolExecutor(max(1, min(16, os.cpu_count() or 1))) as ex:
        amax_bits = max(ex.map(chunk_amax, starts), default=0)
    amax = float(np.array([amax_bits << 16], dtype=np.uint32).view(np.float32)[0])
    scale = amax / 448.0 if amax > 0 else 1.0
    with np.errstate(invalid="ignore"):  # the NaN patterns stay NaN
        values = (np.arange(1 << 16, dtype=np.uint32) << 16).view(np.float32).astype(np.float64)
        table = e4m3_codes(values / scale)
    out = np.empty(flat.size, dtype=np.uint8)

    def chunk_codes(i):
        np.take(table, flat[i:i + chunk], out=out[i:i + chunk])

    with _cf.ThreadPoolExecutor(max(1, min(16, os.cpu_count() or 1))) as ex:
        list(ex.map(chunk_codes, starts))
    return out.reshape(pool.shape), scale


def make_decode_fp8(cfg: DecodeConfig, kv_lens=None, identity: bool = False) -> dict:
    """Paged decode inputs with an FP8 E4M3 cache and one scale per tensor.

    The N(0,1) bf16 pools of :func:`make_decode` are quantised with
    :func:`bf16_pool_to_e4m3` (NaN sentinels in spare blocks and tail slots
    become the NaN code). Returns the make_decode dict with ``k_pool`` /
    ``v_pool`` as uint8 codes and ``k_scale`` / ``v_scale``.
    """
    d = make_decode(cfg, kv_lens=kv_lens, identity=identity)
    for name in ("k", "v"):
        d[name + "_pool"], d[name + "_scale"] = bf16_pool_to_e4m3(d[name + "_pool"])
    return d


def make_decode(cfg: DecodeConfig, kv_lens=None, identity: bool = False) -> dict:
    """Paged decode inputs: q [B, Hq, D] and a paged pool for the lengths."""
    if kv_lens is None:
        kv_lens = random_lengths(cfg.seed, cfg.batch, cfg.len_lo, cfg.len_hi)
    q = normal_bf16(cfg.seed, (cfg.batch, cfg.q_heads, cfg.head_dim), 0)
    d = make_paged_pool(cfg.seed, kv_lens, cfg.kv_heads, cfg.head_dim, cfg.spare_blocks,
                        identity=identity)
    d.update(q=q, scale=cfg.scale)
    return d


def make_shared_prefix_decode(cfg: SharedPrefixConfig, suffix_lens=None) -> dict:
    """Paged decode inputs whose sequences share their first prefix_len tokens.

    The prefix occupies prefix_len / 16 physical blocks that every row of the
    block table lists first (aliased); each sequence's own tokens follow in
    blocks of its own. Physical ids are a random permutation of the pool;
    spare blocks and the tail slots past each sequence end hold NaN. Returns
    q, k_pool, v_pool, block_table, kv_lens (= prefix_len + suffix),
    suffix_lens, prefix_len, num_blocks, spare_ids, scale.
    """
    assert cfg.prefix_len % BLOCK_SIZE == 0
    if suffix_lens is None:
        suffix_lens = random_lengths(cfg.seed, cfg.batch, cfg.suffix_lo, cfg.suffix_hi)
    suffix_lens = np.asarray(suffix_lens, dtype=np.int32)
    pb = cfg.prefix_len // BLOCK_SIZE
    own = (suffix_lens.astype(np.int64) + BLOCK_SIZE - 1) // BLOCK_SIZE
    used = pb + int(own.sum())
    num_blocks = used + cfg.spare_blocks
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([cfg.seed, 11])))
    perm = rng.permutation(num_blocks)
    spare = perm[used:]
    max_blocks = max(1, pb + (int(own.max()) if len(own) else 0))
    filler = int(spare[0]) if cfg.spare_blocks > 0 else 0
    table = np.full((len(suffix_lens), max_blocks), filler, dtype=np.int32)
    table[:, :pb] = perm[:pb]
    off = pb
    for b, n in enumerate(own):
        table[b, pb:pb + n] = perm[off:off + n]
        off += n
    shape = (num_blocks, cfg.kv_heads, BLOCK_SIZE, cfg.head_dim)
    k_pool = normal_bf16(cfg.seed, shape, 1)
    v_pool = normal_bf16(cfg.seed, shape, 2)
    kv_lens = (cfg.prefix_len + suffix_lens).astype(np.int32)
    for pool in (k_pool, v_pool):
        pool[spare] = BF16_NAN
        for b, L in enumerate(kv_lens):
            tail = int(L) % BLOCK_SIZE
            if tail:
                pool[table[b, (int(L) - 1) // BLOCK_SIZE], :, tail:, :] = BF16_NAN
    q = normal_bf16(cfg.seed, (len(suffix_lens), cfg.q_heads, cfg.head_dim), 0)
    return dict(q=q, k_pool=k_pool, v_pool=v_pool, block_table=table, kv_lens=kv_lens, suffix_lens=suffix_lens,
                prefix_len=cfg.prefix_len, num_blocks=num_blocks, spare_ids=spare, scale=cfg.scale)


def make_block_sparse(seed: int, q_heads: int, kv_heads: int, seqlen_q: int, seqlen_k: int, head_dim: int,
                      row_block: int, window: int, extra: int, spare_blocks: int = 8) -> dict:
    """A block-sparse (BSR) pattern over one sequence, with its keys/values paged.

    Query block r (``row_block`` rows) sees a window of ``window`` key blocks
    (16 keys each) around its own position plus ``extra`` random other key
    blocks, listed in random order (``indptr`` / ``indices``, logical key
    blocks). q [Hq, Sq, D], k/v [Hkv, Sk, D] are N(0,1) bf16; the pools
    [NB, Hkv, 16, D] hold logical key block c in physical block ``phys[c]``
    (a random permutation); spare blocks and the tail slots past Sk hold NaN.
    """
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, 60])))
    n_rb = -(-seqlen_q // row_block)
    n_cb = -(-seqlen_k // BLOCK_SIZE)
    indptr = [0]
    indices = []
    for r in range(n_rb):
        centre = (r * row_block * seqlen_k) // max(seqlen_q, 1) // BLOCK_SIZE
        lo = max(0, centre - window // 2)
        cols = set(range(lo, min(n_cb, lo + window)))
        others = [c for c in range(n_cb) if c not in cols]
        if others and extra:
            cols |= set(rng.choice(others, size=min(extra, len(others)), replace=False).tolist())
        cols = np.array(sorted(cols), dtype=np.int32)
        rng.shuffle(cols)
        indices.extend(cols.tolist())
        indptr.append(len(indices))
    q = normal_bf16(seed, (q_heads, seqlen_q, head_dim), 61)
    k = normal_bf16(seed, (kv_heads, seqlen_k, head_dim), 62)
    v = normal_bf16(seed, (kv_heads, seqlen_k, head_dim), 63)
    nb = n_cb + spare_blocks
    phys = rng.permutation(nb).astype(np.int32)
    pools = []
    for x in (k, v):
        pool = np.full((nb, kv_heads, BLOCK_SIZE, head_dim), BF16_NAN, dtype=np.uint16)
        for c in range(n_cb):
            t1 = min((c + 1) * BLOCK_SIZE, seqlen_k)
            pool[phys[c], :, :t1 - c * BLOCK_SIZE] = x[:, c * BLOCK_SIZE:t1]
        pools.append(pool)
    return dict(q=q, k=k, v=v, k_pool=pools[0], v_pool=pools[1], phys=phys[:n_cb], spare_ids=phys[n_cb:],
                indptr=np.array(indptr, dtype=np.int64), indices=np.array(indices, dtype=np.int32),
                row_block=row_block, num_blocks=nb)


def bsr_tables(d: dict, seqlen_k: int) -> tuple:
    """Block tables that express a BSR pattern from :func:`make_block_sparse`:
    one row per query block listing the physical blocks of its key blocks.

    The kernels mask each table row by its token count, so a partial last key
    block (Sk not a multiple of 16), when listed, is moved to the end of its
    row and the count stops at Sk. Returns ``(table [n_rb, max_n] int32,
    seqlens_k [n_rb] int32)``; unused entries point at a spare block.
    """
    indptr, indices, phys = d["indptr"], d["indices"], d["phys"]
    n_rb = len(indptr) - 1
    tail = seqlen_k % BLOCK_SIZE
    last = (seqlen_k - 1) // BLOCK_SIZE
    width = max(1, int(np.diff(indptr).max()) if n_rb else 1)
    table = np.full((n_rb, width), int(d["spare_ids"][0]), dtype=np.int32)
    lens = np.zeros(n_rb, dtype=np.int32)
    for r in range(n_rb):
        cols = [int(c) for c in indices[indptr[r]:indptr[r + 1]]]
        partial = tail and last in cols
        if partial:
            cols = [c for c in cols if c != last] + [last]
        table[r, :len(cols)] = phys[cols]
        lens[r] = BLOCK_SIZE * len(cols) - ((BLOCK_SIZE - tail) if partial else 0)
    return table, lens


def relayout_identity(pool: np.ndarray, table: np.ndarray, kv_lens) -> tuple:
    """Copy a paged pool into identity order (sequence 0's blocks first, ...).

    Returns ``(new_pool, new_table)`` holding the same logical tokens; used by
    the bit-exact paging test. Unused slots stay NaN (bf16 bits, or the E4M3
    NaN code for uint8 pools).
    """
    kv_lens = np.asarray(kv_lens, dtype=np.int64)
    nblk = (kv_lens + BLOCK_SIZE - 1) // BLOCK_SIZE
    used = int(nblk.sum())
    fill = FP8_NAN if pool.dtype == np.uint8 else BF16_NAN
    new_pool = np.full((used + 1,) + pool.shape[1:], fill, dtype=pool.dtype)
    new_table = np.full(table.shape, used, dtype=np.int32)
    off = 0
    for b, n in enumerate(nblk):
        new_pool[off:off + n] = pool[table[b, :n]]
        new_table[b, :n] = np.arange(off, off + n)
        off += n
    return new_pool, new_table


def make_mixed(cfg: MixedConfig) -> dict:
    """Mixed batch: prefill chunks on cached context plus decode rows.

    The chunk's own keys/values are already in the paged cache, so the key
    length of chunk ``b`` is ``ctx_b + chunk_len``. Queries of the chunks are
    ``[chunks, Hq, chunk_len, D]``; decode queries are ``[decodes, Hq, D]``.
    One pool holds the KV of all sequences (chunks first, then decodes).
    """
    ctx_chunk = random_lengths(cfg.seed, cfg.chunks, cfg.chunk_ctx_lo, cfg.chunk_ctx_hi, 10)
    ctx_dec = random_lengths(cfg.seed, cfg.decodes, cfg.dec_ctx_lo, cfg.dec_ctx_hi, 12)
    k_lens = np.concatenate([ctx_chunk + cfg.chunk_len, ctx_dec]).astype(np.int32)
    d = make_paged_pool(cfg.seed, k_lens, cfg.kv_heads, cfg.head_dim, cfg.spare_blocks)
    q_chunk = normal_bf16(cfg.seed, (cfg.chunks, cfg.q_heads, cfg.chunk_len, cfg.head_dim), 20)
    q_dec = normal_bf16(cfg.seed, (cfg.decodes, cfg.q_heads, cfg.head_dim), 21)
    d.update(q_chunk=q_chunk, q_dec=q_dec, ctx_chunk=ctx_chunk, ctx_dec=ctx_dec,
             chunk_len=cfg.chunk_len, scale=cfg.scale)
    return d


def causal_pairs(seqlen_q: int, seqlen_k: int, causal: bool) -> int:
    """Number of visible (query, key) pairs in one head (bottom-right causal)."""
    if not causal:
        return seqlen_q * seqlen_k
    rows = np.arange(seqlen_q, dtype=np.int64) + (seqlen_k - seqlen_q) + 1
    return int(np.clip(rows, 0, seqlen_k).sum())
