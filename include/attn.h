/*
 * attn.h -- C ABI of libattn_b200.so: exact scaled-dot-product attention on
 * B200 (sm_100a).
 *
 * The operation (all three entry points compute parts of it):
 *
 *   O = softmax(Q K^T * scale + causal mask) V,  LSE = ln sum_j exp(scale q.k_j)
 *
 * Attention keeps its mathematical definition; tiling, the online softmax and
 * kernel fusion only change how it is computed ("推理加速" interview notes,
 * section FlashAttention; "抱infra脚", section Flash Attention 核心技术).
 * Key/value heads are shared by contiguous groups of G = Hq / Hkv query heads:
 * query head h reads key/value head h / G ("5.2 推理加速的未来趋势", GQA/MQA).
 * The causal mask is aligned bottom-right: with Sq queries over Sk keys, query
 * i sees keys 0 .. i + (Sk - Sq).
 *
 * Conventions shared by every call:
 *  - Element types: Q, K, V and the KV cache are bf16; accumulation is fp32;
 *    LSE is fp32, natural log; O is bf16 or fp32 (attn_dtype_t).
 *  - Every pointer is DEVICE memory owned by the caller. The library allocates
 *    no device memory and keeps no state besides a per-device cache of the SM
 *    count and of kernel attributes, and two non-blocking streams per device
 *    (attn_decode_paged_shared_prefix, attn_prefill_from_host). Host pointers
 *    are used only where a parameter says "host".
 *  - Calls are asynchronous and stream-ordered: they validate arguments on the
 *    host, enqueue kernels on `stream` and return. Nothing synchronises.
 *  - Errors: a call returns ATTN_OK or an attn_status_t; it never aborts,
 *    traps or falls back to another implementation. Argument errors are
 *    detected on the host before anything is enqueued. Faults found on the
 *    device (a block id outside the pool, a sequence longer than its block
 *    table, a pipeline wait that ran out of time) skip the affected work and
 *    OR a bit (ATTN_FAULT_*) into the caller's optional `error_flags` word,
 *    which the caller reads after synchronising.
 *  - All entry points are thread-safe; calls on different streams may overlap.
 */
#ifndef ATTN_B200_H_
#define ATTN_B200_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ATTN_API __attribute__((visibility("default")))
#else
#define ATTN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* attn_stream_t; /* a cudaStream_t; NULL = legacy default stream */

typedef enum {
  ATTN_OK = 0,
  ATTN_ERR_INVALID_ARG = 1,   /* null pointer, bad size, inconsistent shapes */
  ATTN_ERR_UNSUPPORTED = 2,   /* head_dim not 64/128, Hq % Hkv != 0, misaligned pointer/stride */
  ATTN_ERR_WORKSPACE = 3,     /* workspace too small; *workspace_needed says how much */
  ATTN_ERR_CUDA = 4,          /* a CUDA runtime call or kernel launch failed */
  ATTN_ERR_DEVICE_FAULT = 5,  /* error_flags holds a fault bit other than ATTN_FAULT_TIMEOUT (attn_sync_error_flags) */
  ATTN_ERR_TIMEOUT = 6,       /* error_flags holds ATTN_FAULT_TIMEOUT (attn_sync_error_flags) */
  ATTN_ERR_NO_DEVICE = 7      /* no sm_100 device is current */
} attn_status_t;

typedef enum { ATTN_DTYPE_BF16 = 0, ATTN_DTYPE_F32 = 1, ATTN_DTYPE_FP8_E4M3 = 2 } attn_dtype_t;

/* Bits a kernel ORs into *error_flags. */
#define ATTN_FAULT_TIMEOUT 0x1      /* a pipeline wait exceeded its bound; the tile was abandoned */
#define ATTN_FAULT_BAD_BLOCK 0x2    /* a block-table entry was outside [0, num_blocks) */
#define ATTN_FAULT_BAD_LENGTH 0x4   /* a sequence length exceeded its block table or was negative */
#define ATTN_FAULT_PREFIX_MISMATCH 0x8 /* attn_decode_paged_shared_prefix: a table row's prefix blocks differ from row 0's */
#define ATTN_FAULT_BOUNDS 0x10      /* debug build only: an index failed its bounds check (site in bits 16..23) */
/* The site (attn_bounds_site_t) of the first failed bounds check of a debug
 * build, 0 if none; the word's other bits are the ATTN_FAULT_* flags. */
#define ATTN_FAULT_SITE(word) (((word) >> 16) & 0xff)

/*
 * Bounds-check sites of the debug build (libattn_b200_debug.so, compiled with
 * ATTN_DEBUG_BOUNDS=1). Before each of these accesses the debug kernels check
 * the computed index against the extent it must stay within; a failed check
 * skips the access (no trap), ORs ATTN_FAULT_BOUNDS into error_flags and, if
 * it is the first, records its site in bits 16..23. A skipped copy can leave a
 * pipeline wait unfinished, which then also reports ATTN_FAULT_TIMEOUT. The
 * release library carries none of these checks.
 */
typedef enum {
  ATTN_SITE_NONE = 0,
  ATTN_SITE_PREFILL_SMEM_Q = 1,      /* Q tile copy: destination inside the Q buffer */
  ATTN_SITE_PREFILL_SMEM_KV = 2,     /* K / V tile copy: ring slot inside its ring */
  ATTN_SITE_PREFILL_TABLE = 3,       /* paged prefill: block-table column < max_blocks */
  ATTN_SITE_PREFILL_TMEM_S = 4,      /* S / P columns (load, store, MMA target) inside the allocation */
  ATTN_SITE_PREFILL_TMEM_O = 5,      /* O columns (rescale, epilogue, MMA target) inside the allocation */
  ATTN_SITE_PREFILL_SMEM_STAGE = 6,  /* output staging inside the warp's staging area */
  ATTN_SITE_PREFILL_SMEM_VFIX = 7,   /* zeroing of V rows past the sequence end inside the V slot */
  ATTN_SITE_PREFILL_OUT = 8,         /* O / LSE row, head and batch inside the output tensors */
  ATTN_SITE_DECODE_TABLE = 9,        /* decode: block-table column < max_blocks */
  ATTN_SITE_DECODE_SMEM = 10,        /* decode: K / V staging inside the split's shared buffer */
  ATTN_SITE_DECODE_PARTIAL = 11,     /* decode: split index < the workspace's splits per row */
  ATTN_SITE_COMBINE = 12,            /* combine: split index < num_splits */
  ATTN_SITE_BWD_SMEM = 13,           /* backward: ring stage and per-row vectors inside shared memory */
  ATTN_SITE_BWD_TMEM = 14,           /* backward: S / dP / accumulator columns inside the allocation */
  ATTN_SITE_BWD_OUT = 15             /* backward: gradient row / vector row inside its tensor */
} attn_bounds_site_t;

/*
 * Prefill: tiled attention over a whole query block, one pass over K/V with
 * the online softmax (running row max and row sum, rescaled as the max grows)
 * and only O and LSE written back ("推理加速", FlashAttention 的核心思路 flow:
 * tile Q/K/V, load tiles on chip, attend per tile, online softmax, write the
 * final output only; "GPU Kernel 调度:大模型推理的拐点 2026", FlashAttention-3
 * paragraph: Q tiles in parallel, K/V tiles pipelined, producer/consumer roles).
 *
 * Layout (element strides; the last dimension, head_dim, is contiguous):
 *   q [batch, num_q_heads, seqlen_q, head_dim] bf16, strides q_*_stride
 *   k, v [batch, num_kv_heads, seqlen_k, head_dim] bf16, strides k_*_stride and v_*_stride
 *   o [batch, num_q_heads, seqlen_q, head_dim] o_dtype, strides o_*_stride
 *   lse [batch, num_q_heads, seqlen_q] fp32, contiguous; may be NULL
 * Requirements: head_dim in {64, 128}; num_q_heads % num_kv_heads == 0;
 * q/k/v base pointers 16-byte aligned and their batch/head/row strides
 * multiples of 8 elements (16 bytes); o 16-byte aligned with strides that are
 * multiples of 8 elements; seqlen_q, seqlen_k >= 0 (k and v may be NULL when
 * seqlen_k == 0: every row then gets O = 0, LSE = -inf); scale > 0 and finite.
 * Variable lengths in a padded dense batch: seqlens_q and seqlens_k (device,
 * [batch], each nullable) give sequence b's valid query rows (<= seqlen_q;
 * rows past it are not written) and keys (larger values are clamped to
 * seqlen_k); the causal alignment then uses the per-sequence lengths.
 *
 * Paged keys/values (chunked prefill over a KV cache, "抱infra脚" Chunked
 * Prefill and Paged Attention): set k_cache/v_cache non-NULL (then k and v
 * must be NULL). Sequence b then has seqlens_k[b] keys, token t stored at
 * k_cache[block_table[b * max_blocks_per_seq + t / block_size], kvh,
 * t % block_size, :]; the pools are contiguous
 * [num_blocks, num_kv_heads, block_size, head_dim] with block_size == 16.
 * seqlens_q (device, [batch], nullable) gives the valid query rows of each
 * sequence (<= seqlen_q; rows past it are not written); seqlens_k (device,
 * [batch]) is required in paged mode and each entry must be <=
 * max_blocks_per_seq * block_size; seqlen_k must then be the maximum of
 * seqlens_k (an upper bound is fine). The causal alignment uses the
 * per-sequence lengths.
 *
 * Packed variable-length queries (a batch of chunks of different lengths
 * without padding, "抱infra脚" Chunked Prefill): set cu_seqlens_q (device,
 * [batch + 1], nondecreasing, cu_seqlens_q[0] == 0) and total_q (host, the
 * rows of the packed tensors, >= cu_seqlens_q[batch]). Then q and o are
 * [total_q, num_q_heads, head_dim] with strides q_row_stride / q_head_stride
 * (o_row_stride / o_head_stride; the batch strides are ignored), sequence b
 * owns rows cu_seqlens_q[b] .. cu_seqlens_q[b+1] - 1, lse is [num_q_heads,
 * total_q] fp32 contiguous, and seqlen_q is an upper bound on a sequence's
 * rows (rows past it are not computed). seqlens_q must then be NULL. Keys and
 * values are dense per sequence or paged exactly as above, with the same
 * bottom-right causal alignment per sequence. A packed call gives every valid
 * row the same bits as the padded layout would.
 *
 * Block-sparse attention (BSR: query block r sees only the key blocks listed
 * for it, the block-sparse format of the FlashInfer section of "抱infra脚")
 * is this paged mode, non-causal, with one batch entry per query block whose
 * table row lists the physical blocks of its key blocks, in any order. A
 * table row is masked by its token count seqlens_k[r], so a partial block
 * (fewer than 16 valid keys) may only be the last one of a row. Decode takes
 * a BSR pattern the same way (one table row per query).
 */
typedef struct {
  const void* q;
  const void* k;
  const void* v;
  void* o;
  float* lse;
  int batch;
  int num_q_heads;
  int num_kv_heads;
  int head_dim;
  int seqlen_q;
  int seqlen_k;
  int64_t q_batch_stride, q_head_stride, q_row_stride;
  int64_t k_batch_stride, k_head_stride, k_row_stride;
  int64_t v_batch_stride, v_head_stride, v_row_stride;
  int64_t o_batch_stride, o_head_stride, o_row_stride;
  float scale;
  int causal;
  attn_dtype_t o_dtype;
  /* optional per-sequence lengths / paged KV */
  const int32_t* seqlens_q;
  const int32_t* seqlens_k;
  const void* k_cache;
  const void* v_cache;
  const int32_t* block_table;
  int max_blocks_per_seq;
  int num_blocks;
  int block_size;
  int32_t* error_flags; /* nullable */
  /* optional packed queries (see above) */
  const int32_t* cu_seqlens_q;
  int total_q;
} attn_prefill_params;

ATTN_API attn_status_t attn_prefill(const attn_prefill_params* p, attn_stream_t stream);

/*
 * attn_prefill with the inputs taken from, and the outputs returned to, HOST
 * memory, the copies overlapped with the computation: the call a serving
 * process makes when Q/K/V arrive in host memory (the inputs and outputs of
 * "推理加速" FlashAttention's flow, moved over PCIe).
 *
 * p describes a dense prefill (no paged keys, no variable or packed lengths)
 * whose DEVICE tensors q, k, v, o (and lse, nullable) are contiguous in the
 * [batch, heads, seqlen, head_dim] layout (row stride head_dim, head stride
 * seqlen * head_dim, batch stride heads * seqlen * head_dim); they are the
 * caller's staging buffers. io gives the HOST tensors in the same layouts:
 * q, k, v (read), o (and lse when p->lse is set; written); they should be
 * pinned (page-locked) for the copies to overlap. The work is cut into chunks
 * of one batch entry and kv_heads_per_chunk key/value heads (with their query
 * heads; 0 = all heads of a batch entry); kv_heads_per_chunk must divide
 * num_kv_heads. Per chunk: the inputs are copied host -> device on one of the
 * library's side streams, the prefill of that chunk runs on `stream`, and its
 * O and LSE go device -> host on a second side stream, so that chunk c + 1's
 * inputs travel while chunk c computes and chunk c - 1's outputs travel back.
 * Work enqueued on `stream` after the call starts after every copy of the
 * call has completed. Host and device buffers must not be touched until then.
 * The two side streams are the library's, shared by all threads (calls from
 * several threads are ordered on them, which is correct but serialises their
 * copies).
 * Errors: as attn_prefill, plus ATTN_ERR_INVALID_ARG for a null or
 * non-dividing io field, ATTN_ERR_UNSUPPORTED for non-contiguous device
 * tensors, paged / variable-length parameters or an O in another dtype than
 * io's layout implies (o_dtype decides the host O element size).
 */
typedef struct {
  const void* q;   /* host [batch, num_q_heads, seqlen_q, head_dim] bf16 */
  const void* k;   /* host [batch, num_kv_heads, seqlen_k, head_dim] bf16 */
  const void* v;   /* host, as k */
  void* o;         /* host [batch, num_q_heads, seqlen_q, head_dim], o_dtype */
  float* lse;      /* host [batch, num_q_heads, seqlen_q] fp32; required when p->lse is set */
  int kv_heads_per_chunk;
} attn_prefill_host_io;

ATTN_API attn_status_t attn_prefill_from_host(const attn_prefill_params* p, const attn_prefill_host_io* io,
                                              attn_stream_t stream);

/*
 * Paged decode (Flash-Decoding): one query token per sequence against its
 * whole cached context, with the key range cut into splits that run on
 * different SMs; each split produces a partial output and its log-sum-exp in
 * fp32, and a small combine kernel merges them ("GPU Kernel 调度:大模型推理的
 * 拐点 2026", Flash Decoding section; "抱infra脚", Paged Attention: fixed-size
 * blocks mapped through a block table).
 *
 * Layout:
 *   q [batch, num_q_heads, head_dim] bf16, contiguous
 *   k_cache, v_cache [num_blocks, num_kv_heads, block_size, head_dim] bf16, contiguous
 *   block_table [batch, max_blocks_per_seq] int32 (device), row-major
 *   seq_lens [batch] int32 (device): keys of each sequence, all visible
 *   o [batch, num_q_heads, head_dim] o_dtype, contiguous
 *   lse [batch, num_q_heads] fp32, nullable
 * Requirements: block_size == 16; head_dim == 128; num_q_heads % num_kv_heads
 * == 0 and num_q_heads / num_kv_heads in {1, 2, 4, 8}; 16-byte aligned
 * pointers. max_seq_len (host) is an upper bound on seq_lens (0 = use the
 * table capacity max_blocks_per_seq * block_size); it only sizes the split
 * plan. num_splits: 0 = automatic, otherwise the number of splits a sequence
 * of max_seq_len keys is cut into (1 = no split: the partials step is
 * skipped and the combine is not launched).
 *
 * Workspace: device memory of at least *workspace_needed bytes, 256-byte
 * aligned, owned by the caller, holding the fp32 partials. Pass workspace =
 * NULL to only query the size (returns ATTN_OK, enqueues nothing). If
 * workspace_bytes is too small the call returns ATTN_ERR_WORKSPACE and
 * enqueues nothing. A sequence with 0 keys gets O = 0 and LSE = -inf.
 *
 * FP8 cache ("5.2 推理加速的未来趋势：新算法、新硬件、新协同", 协同层: an FP8 KV
 * cache halves its memory at almost no accuracy cost): kv_dtype =
 * ATTN_DTYPE_FP8_E4M3 means k_cache / v_cache hold one-byte codes in the OCP
 * E4M3 format without infinities (same [num_blocks, num_kv_heads, block_size,
 * head_dim] layout), and the cached key (value) is code * k_scale (code *
 * v_scale). One scale per tensor is this library's convention (the pages give
 * none); k_scale and v_scale must be finite and > 0. kv_dtype = 0 (BF16, the
 * zero-initialised default) ignores both scales. o stays bf16 or fp32.
 */
typedef struct {
  const void* q;
  const void* k_cache;
  const void* v_cache;
  const int32_t* block_table;
  const int32_t* seq_lens;
  void* o;
  float* lse;
  int batch;
  int num_q_heads;
  int num_kv_heads;
  int head_dim;
  int block_size;
  int max_blocks_per_seq;
  int num_blocks;
  int max_seq_len;
  int num_splits;
  float scale;
  attn_dtype_t o_dtype;
  int32_t* error_flags; /* nullable */
  attn_dtype_t kv_dtype; /* ATTN_DTYPE_BF16 (0) or ATTN_DTYPE_FP8_E4M3 */
  float k_scale;         /* FP8 only */
  float v_scale;         /* FP8 only */
} attn_decode_params;

ATTN_API attn_status_t attn_decode_paged(const attn_decode_params* p, void* workspace, size_t workspace_bytes,
                                size_t* workspace_needed, attn_stream_t stream);

/*
 * Backward of attn_prefill (dense, non-paged): the gradients dQ, dK, dV of
 * O = softmax(scale Q K^T + causal mask) V for an upstream gradient dO. These
 * are the plain derivatives of that definition; the pages count one backward
 * kernel next to the forward one for FlashAttention-2 and ask both to match a
 * reference ("GPU Kernel 调度:大模型推理的拐点 2026", the four-layer
 * decomposition and checklist item 1). With P = exp(scale Q K^T - LSE)
 * (masked entries 0), per query head:
 *   dV = P^T dO;  dP = dO V^T;  D = rowsum(dO * O);  dS = P * (dP - D);
 *   dQ = scale dS K;  dK = scale dS^T Q
 * and dK, dV of a key/value head sum over its num_q_heads / num_kv_heads
 * query heads. The causal mask and its bottom-right alignment are those of
 * attn_prefill. P and dS are rebuilt tile by tile (never stored); P and dS
 * enter the tensor-core products in bf16 with fp32 accumulation.
 *
 * Layout (element strides; the last dimension contiguous):
 *   q, dout [batch, num_q_heads, seqlen_q, head_dim] bf16
 *   k, v [batch, num_kv_heads, seqlen_k, head_dim] bf16
 *   o [batch, num_q_heads, seqlen_q, head_dim] o_dtype: attn_prefill's output
 *   lse [batch, num_q_heads, seqlen_q] fp32, contiguous: attn_prefill's LSE
 *   dq like q, dk and dv like k, all grad_dtype (BF16 or F32)
 * Requirements: head_dim 64 or 128; num_q_heads % num_kv_heads == 0; every
 * pointer 16-byte aligned and every stride a multiple of 8 elements.
 * All buffers are the caller's device memory; dq, dk, dv are overwritten
 * (rows that see no key get 0). Deterministic: no atomics.
 *
 * Workspace: at least *workspace_needed bytes of device memory, 256-byte
 * aligned (two fp32 values per query row, rows padded to a multiple of 128
 * per head). workspace = NULL only queries the
 * size (returns ATTN_OK, enqueues nothing); a smaller workspace returns
 * ATTN_ERR_WORKSPACE and enqueues nothing. Asynchronous on `stream`: up to
 * three kernels, the last a programmatic dependent of the one before it
 * (capturable in a CUDA graph); work enqueued on `stream` after the call
 * starts after all of them.
 */
typedef struct {
  const void* q;
  const void* k;
  const void* v;
  const void* o;
  const float* lse;
  const void* dout;
  void* dq;
  void* dk;
  void* dv;
  int batch;
  int num_q_heads;
  int num_kv_heads;
  int head_dim;
  int seqlen_q;
  int seqlen_k;
  int64_t q_batch_stride, q_head_stride, q_row_stride;
  int64_t k_batch_stride, k_head_stride, k_row_stride;
  int64_t v_batch_stride, v_head_stride, v_row_stride;
  int64_t o_batch_stride, o_head_stride, o_row_stride;
  int64_t do_batch_stride, do_head_stride, do_row_stride;
  int64_t dq_batch_stride, dq_head_stride, dq_row_stride;
  int64_t dk_batch_stride, dk_head_stride, dk_row_stride;
  int64_t dv_batch_stride, dv_head_stride, dv_row_stride;
  float scale;
  int causal;
  attn_dtype_t o_dtype;    /* dtype of o: BF16 or F32 */
  attn_dtype_t grad_dtype; /* dtype of dq, dk, dv: BF16 or F32 */
  int32_t* error_flags;    /* nullable */
} attn_backward_params;

ATTN_API attn_status_t attn_prefill_backward(const attn_backward_params* p, void* workspace, size_t workspace_bytes,
                                             size_t* workspace_needed, attn_stream_t stream);

/*
 * attn_decode_paged for a batch whose sequences all begin with the same
 * prefix_len tokens (a shared prompt): requests with a common prefix can share
 * their KV blocks ("抱infra脚", Paged Attention), and a common prefix should
 * not be processed once per request ("抱infra脚", RadixAttention).
 *
 * The prefix's keys/values are the blocks listed first in sequence 0's table,
 * block_table[0][0 .. prefix_len / 16); the other sequences' entries for
 * those positions must alias the same blocks. They are only compared with
 * row 0's: a row that lists different blocks there sets
 * ATTN_FAULT_PREFIX_MISMATCH in error_flags, and its prefix is still taken
 * from row 0 (the result does not depend on those entries). Each
 * sequence b continues with its own blocks block_table[b][prefix_len / 16 ..]
 * up to seq_lens[b] keys. The result is what attn_decode_paged returns when
 * every sequence's first prefix_len keys/values are sequence 0's, up to fp32
 * rounding (the prefix is merged in as separate log-sum-exp partials).
 *
 * The prefix is read once per batch instead of once per sequence: all batch
 * queries of a query head run as the rows of one non-causal tcgen05 prefill
 * over the prefix (cut into up to 16 key ranges when the batch is small),
 * the split-KV decode covers each sequence's suffix, and one kernel merges
 * the partials ("GPU Kernel 调度:大模型推理的拐点 2026", Flash Decoding
 * section: partials merged by their log-sum-exp). The prefix prefill and the
 * suffix decode are independent, so the prefill runs on the library's second
 * stream of the device (forked from `stream` and joined back with events;
 * stream capture follows the fork, so the call can be captured into a CUDA
 * graph). Calls from several threads share that second stream: one of them
 * being captured while another runs eagerly makes the eager one fail with
 * ATTN_ERR_CUDA (a stream in capture takes no eager work).
 *
 * Parameters as attn_decode_paged, plus prefix_len (host): a multiple of 16
 * with 0 <= prefix_len <= max_blocks_per_seq * 16, else
 * ATTN_ERR_INVALID_ARG; 0 runs attn_decode_paged itself (with its workspace
 * size). kv_dtype must be ATTN_DTYPE_BF16 (ATTN_ERR_UNSUPPORTED otherwise).
 * max_seq_len, if given, bounds seq_lens as in attn_decode_paged. Workspace
 * rules as attn_decode_paged; the workspace is always needed (it holds the
 * prefix and suffix partials) and its size depends on the device's SM count.
 * A sequence with seq_lens[b] < prefix_len (or longer than its table) sets
 * ATTN_FAULT_BAD_LENGTH in error_flags; its suffix is then taken as empty
 * (or as the table's capacity).
 */
ATTN_API attn_status_t attn_decode_paged_shared_prefix(const attn_decode_params* p, int32_t prefix_len,
                                                       void* workspace, size_t workspace_bytes,
                                                       size_t* workspace_needed, attn_stream_t stream);

/*
 * attn_decode_paged without a workspace argument, for callers that cannot
 * allocate device memory: a host program that only receives tensor pointers
 * from another component and has no allocator of its own to pass through this
 * C ABI, or a latency-critical loop that must not call cudaMalloc (which can
 * synchronise the device). The pages have no counterpart to this call; it is a
 * deployment convenience, not part of the method.
 * Same parameters and results as attn_decode_paged. The split partials live in
 * a 16 MiB array of device memory owned by the library (held on every GPU that
 * loads the library until the process exits); nothing is allocated per call.
 * If the split plan for these shapes needs more than 16 MiB (as
 * attn_decode_paged would report through workspace_needed), the call returns
 * ATTN_ERR_WORKSPACE and enqueues nothing; a smaller num_splits lowers the need.
 * The first call on a device looks up the array's device address (once per
 * device, with that device current); make that first call before any stream
 * capture. All calls share the one array: calls whose kernels overlap on the
 * GPU, e.g. on two streams, race and must be serialised by the caller.
 * The looked-up address stays cached for the life of the process: after
 * cudaDeviceReset on a device, this call must not be used on that device
 * again (the cached address would point into the destroyed context).
 */
ATTN_API attn_status_t attn_decode_paged_noalloc(const attn_decode_params* p, attn_stream_t stream);

/*
 * Persistent decode: one resident kernel executes a stream of decode steps
 * over static buffers, commanded from the host through a small block of host
 * memory, instead of launching kernels for every step ("GPU Kernel 调度:大模型推
 * 理的拐点 2026", Persistent Kernel section: a kernel that stays resident and
 * pulls work removes the per-step launch cost that shows at small batch).
 * Every step computes exactly what attn_decode_paged computes for the same
 * buffers, batch and max_seq_len: the same split plan and kernels' arithmetic,
 * bit for bit.
 *
 * attn_persistent_cmd is host memory shared with the kernel: it must be
 * page-locked and mapped into the device (cudaHostAlloc with
 * cudaHostAllocMapped, or any pinned memory on a system with unified
 * addressing). Fields marked host are written by the caller (through
 * attn_decode_persistent_submit / _stop), fields marked device by the kernel.
 *
 * attn_decode_persistent_launch: p describes the static buffers exactly as for
 * attn_decode_paged (q, o, lse, block_table, seq_lens, caches, error_flags),
 * with p->batch the largest batch a step may have and p->max_seq_len the
 * largest bound a step may give (0: the table capacity). The call zeroes
 * *cmd, zeroes the control words of the workspace (cudaMemsetAsync on
 * `stream`) and launches the kernel cooperatively on `stream` (one CTA per
 * resident slot of every SM); it returns at once. While the kernel runs it
 * holds every SM: kernels of other streams wait, copies do not. Workspace:
 * attn_decode_persistent_workspace bytes of device memory, 256-byte aligned,
 * owned by the caller and not touched by anyone else while the kernel runs.
 * idle_cycles (> 0): the kernel exits, with ATTN_FAULT_TIMEOUT in cmd->status
 * and error_flags, after that many SM clock cycles without a command.
 *
 * A step: write its inputs (q rows, block-table rows, seq_lens) into the
 * static buffers and make them visible (e.g. synchronise the stream that
 * copied them), then attn_decode_persistent_submit(cmd, batch, max_seq_len,
 * &step) (max_seq_len 0: the launch bound), then
 * attn_decode_persistent_wait(cmd, step, timeout_us) before reading o / lse or
 * rewriting the inputs. Submit returns ATTN_ERR_INVALID_ARG while a step is
 * still running. Wait returns ATTN_OK, or ATTN_ERR_TIMEOUT when the step did
 * not finish within timeout_us or the kernel gave up. attn_decode_persistent_stop
 * asks the kernel to exit once idle; the caller then synchronises `stream`.
 * The host-side calls make no CUDA call.
 */
typedef struct {
  int32_t seq;          /* host: number of the last step submitted (1, 2, ...) */
  int32_t batch;        /* host: sequences in that step (<= the launch's batch) */
  int32_t max_seq_len;  /* host: bound of that step's seq_lens (0: the launch bound) */
  int32_t stop;         /* host: nonzero asks the kernel to exit once idle */
  int32_t done;         /* device: number of the last step completed */
  int32_t status;       /* device: ATTN_FAULT_* bits when the kernel gave up */
  int32_t running;      /* device: 1 from the kernel's start until it exits */
  int32_t reserved;
} attn_persistent_cmd;

ATTN_API attn_status_t attn_decode_persistent_workspace(const attn_decode_params* p, size_t* bytes);
ATTN_API attn_status_t attn_decode_persistent_launch(const attn_decode_params* p, attn_persistent_cmd* cmd,
                                                     void* workspace, size_t workspace_bytes, long long idle_cycles,
                                                     attn_stream_t stream);
ATTN_API attn_status_t attn_decode_persistent_submit(attn_persistent_cmd* cmd, int32_t batch, int32_t max_seq_len,
                                                     int32_t* step);
ATTN_API attn_status_t attn_decode_persistent_wait(const attn_persistent_cmd* cmd, int32_t step, long long timeout_us);
ATTN_API void attn_decode_persistent_stop(attn_persistent_cmd* cmd);

/*
 * A pool of CUDA graphs of the decode step, one per static shape ("GPU Kernel
 * 调度:大模型推理的拐点 2026", CUDA Graph section: capture the shapes a server
 * sees up front and replay the nearest one, so a step costs one graph launch
 * instead of one launch per kernel).
 *
 * attn_decode_graph_pool_create captures attn_decode_paged once for every
 * (batch bucket, length bucket) pair, over the static buffers p describes
 * (q, o, lse, block_table, seq_lens, caches and error_flags as for
 * attn_decode_paged; p->batch is the rows those buffers hold, at least the
 * largest batch bucket). Buckets are host arrays of strictly ascending
 * positive values (at most 1024 each); a length bucket is a max_seq_len bound
 * (up to the table capacity). workspace: at least attn_decode_graph_pool_workspace
 * bytes of device memory, 256-byte aligned, owned by the caller and shared by
 * every graph of the pool. The capture runs on an internal stream and does
 * not touch the buffers.
 *
 * attn_decode_graph_pool_replay(pool, batch, max_seq_len, stream, ...) launches
 * the graph of the smallest batch bucket >= batch and the smallest length
 * bucket >= max_seq_len (0: the largest), and reports the chosen bucket in
 * *bucket_batch / *bucket_len (nullable). The graph reads the buffers as they
 * are when it runs: the caller has written this step's q rows, table rows and
 * seq_lens, and keeps seq_lens of the rows from batch up to the bucket's batch
 * at 0 (those rows get O = 0, LSE = -inf). The result is attn_decode_paged
 * with batch = the bucket's batch and max_seq_len = the bucket's length, bit
 * for bit. ATTN_ERR_INVALID_ARG when no bucket covers the step. Replays share
 * the workspace: replays that overlap on the GPU race.
 */
typedef struct attn_decode_graph_pool attn_decode_graph_pool;

ATTN_API attn_status_t attn_decode_graph_pool_workspace(const attn_decode_params* p, const int32_t* batch_buckets,
                                                        int n_batch, const int32_t* len_buckets, int n_len,
                                                        size_t* bytes);
ATTN_API attn_status_t attn_decode_graph_pool_create(const attn_decode_params* p, const int32_t* batch_buckets,
                                                     int n_batch, const int32_t* len_buckets, int n_len,
                                                     void* workspace, size_t workspace_bytes,
                                                     attn_decode_graph_pool** pool);
ATTN_API attn_status_t attn_decode_graph_pool_replay(attn_decode_graph_pool* pool, int32_t batch, int32_t max_seq_len,
                                                     attn_stream_t stream, int32_t* bucket_batch, int32_t* bucket_len);
ATTN_API void attn_decode_graph_pool_destroy(attn_decode_graph_pool* pool);

/*
 * Split-KV log-sum-exp combine ("GPU Kernel 调度:大模型推理的拐点 2026",
 * Flash Decoding section: partials merged with the online-softmax formula,
 * each carrying a log-sum-exp accumulated in FP32). For each row r:
 *   n = splits_per_row ? splits_per_row[r] : num_splits   (0 <= n <= num_splits)
 *   M = max_{s<n} part_lse[s][r];  LSE = M + ln sum_{s<n} exp(part_lse[s][r] - M)
 *   O[r] = sum_{s<n} exp(part_lse[s][r] - LSE) * part_o[s][r][:]
 * A split with LSE = -inf has weight 0 (its part_o is not read); a row with
 * no finite LSE gets O = 0, LSE = -inf.
 * Layout: part_o [num_splits, rows, head_dim] fp32, part_lse [num_splits, rows]
 * fp32, splits_per_row [rows] int32 (device, nullable), out_o [rows, head_dim]
 * in out_dtype, out_lse [rows] fp32 (nullable). head_dim in {64, 128};
 * 16-byte aligned pointers.
 */
ATTN_API attn_status_t splitkv_lse_combine(const float* part_o, const float* part_lse, int num_splits, int rows,
                                  int head_dim, const int32_t* splits_per_row, void* out_o,
                                  attn_dtype_t out_dtype, float* out_lse, attn_stream_t stream);

/*
 * Error word helpers. The kernels OR ATTN_FAULT_* bits into a caller's
 * error_flags word instead of aborting; these turn the word into a status.
 * attn_status_from_flags: ATTN_ERR_TIMEOUT if ATTN_FAULT_TIMEOUT is set, else
 * ATTN_ERR_DEVICE_FAULT if any bit is set, else ATTN_OK.
 * attn_sync_error_flags: waits for `stream` (cudaStreamSynchronize), copies
 * the device word error_flags to *flags_out (nullable, host) and returns
 * attn_status_from_flags of it; ATTN_ERR_INVALID_ARG for a NULL word,
 * ATTN_ERR_CUDA if the copy or the synchronisation failed. The word is left
 * as it is (the caller clears it before reusing it).
 */
ATTN_API attn_status_t attn_status_from_flags(int32_t flags);
ATTN_API attn_status_t attn_sync_error_flags(const int32_t* error_flags, attn_stream_t stream, int32_t* flags_out);

/*
 * Diagnostics (not part of the method; for tests and bring-up).
 *
 * attn_set_wait_limit: the clock-cycle bound of every pipeline wait in the
 * prefill and backward kernels launched after the call (process-wide;
 * cycles <= 0 restores the default of 2e9 cycles, about one second). A wait
 * that runs out makes its CTA stop, wait for the copies and tensor-core
 * products it already issued (those waits keep their own ~1 s bound), free
 * its tensor memory and OR ATTN_FAULT_TIMEOUT into error_flags; the outputs of
 * that call are then undefined. A tiny bound exercises that path on purpose.
 *
 * attn_selftest_exp2: y_poly[i] = the prefill kernel's FMA-pipe 2^x[i] (a
 * cubic on the reduced argument; relative error about 7.5e-5 for x in
 * [-125, 127], inputs below -126 clamped to -126) and, if y_mufu is not NULL,
 * y_mufu[i] = the MUFU ex2.approx.ftz result, for 0 <= i < n. x, y_poly,
 * y_mufu: device fp32 arrays of n elements. Asynchronous on `stream`.
 */
ATTN_API void attn_set_wait_limit(long long cycles);
ATTN_API attn_status_t attn_selftest_exp2(const float* x, float* y_poly, float* y_mufu, int n, attn_stream_t stream);

/*
 * attn_debug_bounds_enabled: 1 in the debug build (bounds checks compiled
 * in), 0 in the release library.
 *
 * attn_debug_plant_bounds: debug build only. Every kernel launched after the
 * call reports a failed check at `site` (attn_bounds_site_t) each time it
 * reaches that site, as if its index were out of range, while the access
 * itself still uses the real, checked index: it shows that the site's check
 * is wired and recorded, without touching anything out of range. site 0 turns
 * it off. Process-wide. The release library returns ATTN_ERR_UNSUPPORTED.
 */
ATTN_API int attn_debug_bounds_enabled(void);
ATTN_API attn_status_t attn_debug_plant_bounds(int site);

/* Static, human-readable name of a status code. */
ATTN_API const char* attn_status_string(attn_status_t status);

/* Library version: major * 10000 + minor * 100 + patch. */
ATTN_API int attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_B200_H_ */
