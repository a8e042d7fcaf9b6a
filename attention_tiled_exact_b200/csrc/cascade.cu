// Decode over a prefix that every sequence of the batch shares (cascade).
//
// What it computes: exactly what attn_decode_paged computes when the first
// prefix_len tokens of every sequence are the same tokens: paged KV blocks
// can be shared by requests with a common prefix ("抱infra脚", Paged
// Attention), and a common prompt prefix should not be processed again for
// every request ("抱infra脚", RadixAttention). The plain decode reads the
// shared blocks once per sequence; here they are read once per batch.
//
// Attention over the concatenation of two key ranges is the log-sum-exp merge
// of the attention over each range (the split-KV identity of Flash-Decoding,
// "GPU Kernel 调度:大模型推理的拐点 2026", Flash Decoding section). So:
//   1. prefix: all G * N decode queries of one key/value head (its G query
//      heads times the N sequences) are the rows of one non-causal prefill
//      problem over the prefix keys, on the tcgen05 prefill kernel: the
//      prefix K/V tiles are loaded once per kv head instead of once per
//      sequence and query head, q.k / p.v become full 128-row tensor-core
//      tiles, and the problem is an MHA one (one query "head" per kv head).
//      The prefix keys are cut into S ranges that run as S batch entries, S
//      chosen so that the work items fill the GPU; each range gives a partial
//      (O, LSE). q is copied into the workspace in that layout, once per
//      range: [S][kv head][g * N + n][D] for query head kvh * G + g of
//      sequence n;
//   2. suffix: the split-KV decode over each sequence's own tokens past the
//      prefix (block table entries from prefix_len / 16 on, lengths
//      seq_lens[b] - prefix_len), giving one more partial per row;
//   3. merge: one warp per (sequence, head) row combines the S prefix
//      partials with the suffix decode's split partials (the decode's own
//      combine is not run).
// A small kernel before step 1 writes the suffix lengths (flagging sequences
// shorter than the prefix), the per-range prefix lengths and the q copies,
// and flags table rows whose prefix entries differ from row 0's.
#include <cuda_bf16.h>
#include <stdint.h>
#include <string.h>

#include "internal.h"
#include "sm100_ptx.cuh"

namespace attn {

namespace cascade {

constexpr int MAX_RANGES = 16;      // prefix key ranges (batch entries of the prefix prefill)
constexpr int MIN_RANGE_BLOCKS = 16;  // at least 256 prefix keys per range

__global__ void __launch_bounds__(256)
    prepare_kernel(const int32_t* __restrict__ seq_lens, int batch, int prefix_len, int suffix_cap,
                   int32_t* __restrict__ suffix_lens, int32_t* __restrict__ range_lens, int ranges, int range_len,
                   const uint4* __restrict__ q, uint4* __restrict__ q_rep, int hq, int row_vecs,
                   const int32_t* __restrict__ block_table, int max_blocks, int32_t* __restrict__ error_flags) {
  const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long stride = (long long)gridDim.x * blockDim.x;
  // Every row's prefix entries must alias row 0's (the prefix is read from
  // row 0 only): a row that lists other blocks there is flagged.
  const int prefix_blocks = prefix_len / 16;
  bool mismatch = false;
  for (long long i = tid + prefix_blocks; i < (long long)batch * prefix_blocks; i += stride) {
    const long long b = i / prefix_blocks;
    const int j = (int)(i - b * prefix_blocks);
    mismatch |= block_table[b * max_blocks + j] != block_table[j];
  }
  if (mismatch && error_flags) atomicOr(error_flags, ATTN_FAULT_PREFIX_MISMATCH);
  for (long long i = tid; i < batch; i += stride) {
    const int L = seq_lens[i];
    int s = L - prefix_len;
    if (L < prefix_len || s > suffix_cap) {
      if (error_flags) atomicOr(error_flags, ATTN_FAULT_BAD_LENGTH);
      s = s < 0 ? 0 : suffix_cap;
    }
    suffix_lens[i] = s;
  }
  for (long long i = tid; i < ranges; i += stride) {
    const int rest = prefix_len - (int)i * range_len;
    range_lens[i] = rest < range_len ? rest : range_len;
  }
  // q [N][hq][D] -> q_rep[s][h][n][D] (h = kvh * G + g): a transpose of
  // D-element rows, repeated for every range.
  const long long q_vecs = (long long)batch * hq * row_vecs;
  for (long long i = tid; i < ranges * q_vecs; i += stride) {
    const long long j = i % q_vecs;
    const long long t = j / row_vecs;
    const int c = (int)(j - t * row_vecs);
    const long long h = t / batch, n = t - h * batch;
    q_rep[i] = q[(n * hq + h) * row_vecs + c];
  }
}

// One warp per row r = b * hq + h, over all partials of the row:
//  - prefix range s < ranges: O at pre_o[(s * rows + h * n_seq + b) * HD],
//    LSE at pre_lse[s * rows + h * n_seq + b] (the prefill's [range][kv head]
//    [g * N + n] row order);
//  - the suffix (when suf_o is not NULL), of n = max(1, ceil(L / T)) splits
//    for suffix length L = suffix_lens[b] (at most max_splits): with n == 1
//    the decode wrote it to suf_o[r * HD] / suf_lse[r], else its split i is
//    at part_o[(i * rows + r) * HD] / part_lse[i * rows + r] (the decode's own
//    combine is not run: this kernel merges its splits with the prefix).
// A partial with LSE -inf has weight 0 and is not read.
template <int HD>
__global__ void __launch_bounds__(256)
    merge_kernel(const float* __restrict__ pre_o, const float* __restrict__ pre_lse, int ranges, int n_seq, int hq,
                 const float* __restrict__ suf_o, const float* __restrict__ suf_lse,
                 const float* __restrict__ part_o, const float* __restrict__ part_lse,
                 const int32_t* __restrict__ suffix_lens, int split_tokens, int max_splits, void* out_o, int out_f32,
                 float* __restrict__ out_lse) {
  constexpr int PER = HD / 32;
  constexpr float LOG2E = 1.4426950408889634f;
  const int rows = n_seq * hq;
  const int r = blockIdx.x * (blockDim.x / 32) + warp_id();
  const int lane = lane_id();
  if (r >= rows) return;
  const int b = r / hq, h = r - b * hq;
  int ns = 0;  // suffix partials of this row
  if (suf_o) {
    const int L = suffix_lens[b];
    ns = L > 0 ? (L + split_tokens - 1) / split_tokens : 1;
    ns = ns < 1 ? 1 : (ns > max_splits ? max_splits : ns);
    if (ns > 1 && !part_o) ns = 1;
  }
  const int total = ranges + ns;
  auto lse_of = [&](int s) -> float {
    if (s < ranges) return pre_lse[(long long)s * rows + (long long)h * n_seq + b];
    return ns == 1 ? suf_lse[r] : part_lse[(long long)(s - ranges) * rows + r];
  };
  auto o_of = [&](int s) -> const float* {
    if (s < ranges) return pre_o + ((long long)s * rows + (long long)h * n_seq + b) * HD;
    return ns == 1 ? suf_o + (long long)r * HD : part_o + ((long long)(s - ranges) * rows + r) * HD;
  };
  // The partials' LSEs, lanes strided over them (32 at a time): max, then
  // the sum of exp(lse - max).
  float M = -INFINITY;
  for (int s = lane; s < total; s += 32) M = fmaxf(M, lse_of(s));
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  float out[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) out[i] = 0.f;
  float lse = -INFINITY;
  if (M != -INFINITY) {
    float sum = 0.f;
    for (int s = lane; s < total; s += 32) sum += ex2_approx((lse_of(s) - M) * LOG2E);  // exp(-inf) = 0
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    lse = M + logf(sum);
    for (int s0 = 0; s0 < total; s0 += 32) {
      // Lane j holds partial s0 + j's weight; every lane reads its slice of
      // each partial's O (weight 0: not read).
      const float ls = s0 + lane < total ? lse_of(s0 + lane) : -INFINITY;
      const float wl = ls == -INFINITY ? 0.f : ex2_approx((ls - lse) * LOG2E);
      const int n = total - s0 < 32 ? total - s0 : 32;
      for (int j = 0; j < n; ++j) {
        const float wgt = __shfl_sync(0xffffffffu, wl, j);
        if (wgt == 0.f) continue;  // warp-uniform
        const float* src = o_of(s0 + j) + lane * PER;
#pragma unroll
        for (int i = 0; i < PER; i += 2) {
          const float2 x = *reinterpret_cast<const float2*>(src + i);
          out[i] = fmaf(wgt, x.x, out[i]);
          out[i + 1] = fmaf(wgt, x.y, out[i + 1]);
        }
      }
    }
  }
  if (out_f32) {
    float* dst = reinterpret_cast<float*>(out_o) + (long long)r * HD + lane * PER;
#pragma unroll
    for (int i = 0; i < PER; i += 2) *reinterpret_cast<float2*>(dst + i) = make_float2(out[i], out[i + 1]);
  } else {
    __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(out_o) + (long long)r * HD + lane * PER;
#pragma unroll
    for (int i = 0; i < PER; i += 2)
      *reinterpret_cast<__nv_bfloat162*>(dst + i) = __floats2bfloat162_rn(out[i], out[i + 1]);
  }
  if (lane == 0 && out_lse) out_lse[r] = lse;
}

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

}  // namespace cascade

// Prefix work items of the prefill kernel for one key range: the problem has
// one query head per kv head with G * N rows, and the kernel pairs row blocks
// of a head into one item.
static long long prefix_items_per_range(const attn_decode_params& p) {
  const long long rows = (long long)p.batch * (p.num_q_heads / p.num_kv_heads);
  const long long row_blocks = (rows + 127) / 128;
  return ((row_blocks + 1) / 2) * p.num_kv_heads;
}

CascadePlan plan_cascade(const attn_decode_params& p, int prefix_len) {
  using namespace cascade;
  CascadePlan c;
  memset(&c, 0, sizeof(c));
  c.prefix_len = prefix_len;
  const int prefix_blocks = prefix_len / 16;
  const long long items = prefix_items_per_range(p);
  long long r = items > 0 ? device_sm_count() / items : 1;
  if (r > prefix_blocks / MIN_RANGE_BLOCKS) r = prefix_blocks / MIN_RANGE_BLOCKS;
  if (r > MAX_RANGES) r = MAX_RANGES;
  if (r < 1) r = 1;
  const int range_blocks = (prefix_blocks + (int)r - 1) / (int)r;
  c.range_blocks = range_blocks;
  c.ranges = range_blocks > 0 ? (prefix_blocks + range_blocks - 1) / range_blocks : 0;
  c.suffix_cap = (p.max_blocks_per_seq - prefix_blocks) * 16;

  // The suffix decode: same tables shifted by the prefix blocks, lengths from
  // the workspace, partial output in fp32.
  c.suffix = p;
  c.suffix.block_table = p.block_table ? p.block_table + prefix_blocks : nullptr;
  int bound = c.suffix_cap;
  if (p.max_seq_len > 0 && p.max_seq_len - prefix_len < bound) bound = p.max_seq_len - prefix_len;
  c.suffix.max_seq_len = bound > 0 ? bound : 1;
  c.suffix.o_dtype = ATTN_DTYPE_F32;
  c.suffix_plan = plan_decode(c.suffix);

  const size_t rows = (size_t)p.batch * p.num_q_heads, D = p.head_dim;
  size_t off = 0;
  c.off_suffix_lens = off;
  off += align256((size_t)p.batch * 4);
  c.off_range_lens = off;
  off += align256((size_t)MAX_RANGES * 4);
  c.off_q_rep = off;
  off += align256((size_t)c.ranges * rows * D * 2);
  c.off_pre_o = off;
  off += align256((size_t)c.ranges * rows * D * 4);
  c.off_pre_lse = off;
  off += align256((size_t)c.ranges * rows * 4);
  c.off_suf_o = off;
  off += align256(rows * D * 4);
  c.off_suf_lse = off;
  off += align256(rows * 4);
  c.off_decode = off;
  off += c.suffix_plan.workspace_bytes;
  c.workspace_bytes = off;
  return c;
}

attn_status_t launch_cascade(const attn_decode_params& p, const CascadePlan& c, void* workspace,
                             cudaStream_t stream) {
  using namespace cascade;
  if (p.batch == 0) return ATTN_OK;
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  int32_t* suffix_lens = reinterpret_cast<int32_t*>(ws + c.off_suffix_lens);
  int32_t* range_lens = reinterpret_cast<int32_t*>(ws + c.off_range_lens);
  __nv_bfloat16* q_rep = reinterpret_cast<__nv_bfloat16*>(ws + c.off_q_rep);
  float* pre_o = reinterpret_cast<float*>(ws + c.off_pre_o);
  float* pre_lse = reinterpret_cast<float*>(ws + c.off_pre_lse);
  float* suf_o = reinterpret_cast<float*>(ws + c.off_suf_o);
  float* suf_lse = reinterpret_cast<float*>(ws + c.off_suf_lse);
  const long long rows = (long long)p.batch * p.num_q_heads;
  const int D = p.head_dim;

  const int G = p.num_q_heads / p.num_kv_heads;
  {
    const int row_vecs = D * 2 / 16;
    const long long work = c.ranges * rows * row_vecs;
    long long blocks = (work + 255) / 256;
    const long long cap = 4LL * device_sm_count();
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    prepare_kernel<<<(int)blocks, 256, 0, stream>>>(p.seq_lens, p.batch, c.prefix_len, c.suffix_cap, suffix_lens,
                                                   range_lens, c.ranges, c.range_blocks * 16,
                                                   reinterpret_cast<const uint4*>(p.q), reinterpret_cast<uint4*>(q_rep),
                                                   p.num_q_heads, row_vecs, p.block_table, p.max_blocks_per_seq,
                                                   p.error_flags);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  }

  // 1. prefix: batch entry s = key range s; query "head" kvh holds the G * N
  // rows of kv head kvh's query heads.
  attn_prefill_params pp;
  memset(&pp, 0, sizeof(pp));
  pp.q = q_rep;
  pp.o = pre_o;
  pp.lse = pre_lse;
  pp.batch = c.ranges;
  pp.num_q_heads = p.num_kv_heads;
  pp.num_kv_heads = p.num_kv_heads;
  pp.head_dim = D;
  pp.seqlen_q = G * p.batch;
  pp.seqlen_k = c.range_blocks * 16;
  pp.q_batch_stride = rows * D;
  pp.q_head_stride = (long long)G * p.batch * D;
  pp.q_row_stride = D;
  pp.o_batch_stride = rows * D;
  pp.o_head_stride = (long long)G * p.batch * D;
  pp.o_row_stride = D;
  pp.scale = p.scale;
  pp.causal = 0;
  pp.o_dtype = ATTN_DTYPE_F32;
  pp.seqlens_k = range_lens;
  pp.k_cache = p.k_cache;
  pp.v_cache = p.v_cache;
  pp.block_table = p.block_table;  // row 0; range s starts at entry s * range_blocks
  pp.max_blocks_per_seq = c.range_blocks;
  pp.num_blocks = p.num_blocks;
  pp.block_size = 16;
  pp.error_flags = p.error_flags;
  // The prefix prefill (short, latency-bound items on up to one CTA per SM)
  // and the suffix decode (memory-bound) are independent: the prefill runs on
  // a side stream, launched first, and the decode's CTAs take the SMs it
  // leaves and those it frees; the merge waits for both. (Capping the
  // prefill to a third or fewer of the SMs was slower, measured.) Without a
  // side stream or events they run one after the other on `stream`.
  const bool has_suffix = c.suffix_cap > 0;
  cudaStream_t side = has_suffix ? side_stream() : nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
  if (side && (cudaEventCreateWithFlags(&fork, cudaEventDisableTiming) != cudaSuccess ||
               cudaEventCreateWithFlags(&join, cudaEventDisableTiming) != cudaSuccess ||
               cudaEventRecord(fork, stream) != cudaSuccess || cudaStreamWaitEvent(side, fork, 0) != cudaSuccess)) {
    cudaGetLastError();
    side = nullptr;
  }
  auto release = [&]() {
    if (fork) cudaEventDestroy(fork);
    if (join) cudaEventDestroy(join);
  };
  attn_status_t st = launch_prefill(pp, side ? side : stream);
  if (st == ATTN_OK && side && (cudaEventRecord(join, side) != cudaSuccess)) {
    cudaGetLastError();
    st = ATTN_ERR_CUDA;
  }
  if (st != ATTN_OK) {
    release();
    return st;
  }

  // 2. suffix decode (skipped when the prefix fills every table row).
  // Its splits stay in the decode workspace: the merge below combines them
  // with the prefix ranges in one pass.
  const float* part_o = nullptr;
  const float* part_lse = nullptr;
  if (has_suffix) {
    attn_decode_params ps = c.suffix;
    ps.seq_lens = suffix_lens;
    ps.o = suf_o;
    ps.lse = suf_lse;
    st = launch_decode(ps, c.suffix_plan, ws + c.off_decode, stream, /*combine=*/false);
    if (st != ATTN_OK) {
      if (side) cudaStreamWaitEvent(stream, join, 0);
      release();
      return st;
    }
    if (c.suffix_plan.max_splits > 1) {
      const size_t po = (size_t)c.suffix_plan.max_splits * rows * D * sizeof(float);
      part_o = reinterpret_cast<const float*>(ws + c.off_decode);
      part_lse = reinterpret_cast<const float*>(ws + c.off_decode + align256(po));
    }
  }

  if (side) {
    const bool joined = cudaStreamWaitEvent(stream, join, 0) == cudaSuccess;
    release();
    if (!joined) {
      cudaGetLastError();
      return ATTN_ERR_CUDA;
    }
  }

  // 3. merge: prefix ranges and suffix splits of every row.
  const int warps = 8;
  const int grid = (int)((rows + warps - 1) / warps);
  merge_kernel<128><<<grid, warps * 32, 0, stream>>>(
      pre_o, pre_lse, c.ranges, p.batch, p.num_q_heads, has_suffix ? suf_o : nullptr,
      has_suffix ? suf_lse : nullptr, part_o, part_lse, suffix_lens, c.suffix_plan.split_tokens,
      c.suffix_plan.max_splits, p.o, p.o_dtype == ATTN_DTYPE_F32, p.lse);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace attn
