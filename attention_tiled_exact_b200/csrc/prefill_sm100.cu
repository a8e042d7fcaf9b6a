// Tiled exact-attention prefill for sm_100a.
//
// What it computes: O = softmax(Q K^T * scale + causal mask) V and the row
// log-sum-exp, for bf16 Q/K/V with fp32 accumulation. The computation follows
// the FlashAttention recipe the pages describe: Q, K and V are cut into tiles
// that are brought on chip, S = Q K^T and P V are computed tile by tile, and an
// online softmax keeps a running row max and row sum so that only the final O
// is written back ("推理加速" interview notes, FlashAttention 的核心思路;
// "抱infra脚", Flash Attention 核心技术: tiling, online softmax, fusion).
// Q tiles run in parallel and K/V tiles are pipelined through shared memory by
// a producer, with the matrix products and the softmax in different warps
// ("GPU Kernel 调度:大模型推理的拐点 2026", FlashAttention-2/3 paragraph).
//
// B200 design (one persistent CTA per SM, 384 threads = three warpgroups):
//   * two Q tiles of 128 rows per CTA. For GQA with an even group size the two
//     tiles are two query heads of one key/value head on the same rows, so both
//     tiles need exactly the same key range; otherwise they are two row blocks
//     of one head. Every K/V block is loaded once for both tiles.
//   * keys advance in blocks of 128, so every S MMA is a full-rate
//     M=128 x N=128 instruction. Each tile owns 128 TMEM columns for S; P
//     (bf16 pairs) overwrites their first 64 columns and feeds P V from TMEM.
//   * the two tiles ping-pong: one thread (warp 9) issues every MMA in the
//     order P_0 V_i, S_0(i+1), P_1 V_i, S_1(i+1), so the tensor core works on
//     one tile's products while the other tile's softmax runs.
//   * warp 8 (TMA): loads the Q tiles (the next work item's Q is prefetched
//     into L2 one item ahead) and streams K and V blocks through two-stage
//     shared-memory rings (128-byte swizzle) in the order the MMAs use them.
//   * warps 0-3 / 4-7 (softmax, one warpgroup per tile, one thread per row):
//     read S, mask (diagonal and tail blocks only), update the running max,
//     p = 2^(s*scale*log2e - m), running sum, write P to TMEM. The running max
//     is only moved when it grows by more than 2^8 (which keeps O and the row
//     sum consistent); then O is rescaled in TMEM (the previous P V has
//     completed by the time S of the next block is signalled). The same warps
//     run the epilogue: O / l staged in swizzled shared memory and written by
//     TMA tile stores, LSE = (m + log2 l) * ln 2.
//   * TMEM: S_0 / P_0 cols [0,128), S_1 / P_1 [128,256), O_0 [256,256+D),
//     O_1 [384,384+D).
//   * every mbarrier wait is bounded; on a timeout the CTA raises a flag in
//     shared memory, all roles stop, in-flight copies and MMAs are drained
//     (again bounded), tensor memory is freed, and ATTN_FAULT_TIMEOUT is ORed
//     into the caller's error word.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "exp2_poly.cuh"
#include "bounds_check.cuh"
#include "internal.h"
#include "sm100_ptx.cuh"

namespace attn {
namespace prefill {

constexpr int BM = 128;            // query rows per Q tile
constexpr int BK = 128;            // keys per block
constexpr int NUM_THREADS = 384;   // warpgroups: softmax tile 0, softmax tile 1, {TMA, MMA, idle, idle}
constexpr int SOFTMAX_WARPS = 8;
constexpr int TMA_WARP = 8;
constexpr int MMA_WARP = 9;        // issues every MMA (and owns the TMEM allocation)
constexpr int KSTAGES = 2;         // K blocks in flight
constexpr int VSTAGES = 2;         // V blocks in flight
// Register split. The block is launched with REG_LAUNCH registers per thread
// (384 threads x 168 = 64512 registers); the third warpgroup gives registers
// back and the two softmax warpgroups take them: 2*128*216 + 128*72 = 64512.
// The host refuses to launch unless the compiled kernel uses exactly
// REG_LAUNCH registers, so the split can never ask for more than the block has.
constexpr int REG_LAUNCH = 168;
constexpr int REG_SOFTMAX = 216;
constexpr int REG_OTHER = 72;
static_assert(2 * 128 * REG_SOFTMAX + 128 * REG_OTHER == NUM_THREADS * REG_LAUNCH, "register split");
constexpr uint32_t TMEM_COLS = 512;
constexpr float RESCALE_THRESHOLD = 8.0f;        // log2 units: rescale only when the max grows by > 2^8
// Variable-length launches with at most SORT_MAX_ITEMS items sort the items by
// cost before the snake assignment; a CTA then keeps at most LIST_MAX of them.
constexpr int SORT_MAX_ITEMS = 4096;
constexpr int LIST_MAX = 64;

// Division by a runtime constant d for dividends in [0, 2^31): with
// l = ceil(log2 d), p = 31 + l and m = ceil(2^p / d), n / d = (n * m) >> p
// exactly (m * d - 2^p < d <= 2^l, so n * (m * d - 2^p) < 2^p). Set up on the
// host; one 64-bit multiply and a shift on the device.
struct FastDiv {
  unsigned long long m;
  int p, d;
  __host__ void init(int divisor) {
    d = divisor;
    int l = 0;
    while ((1ll << l) < (long long)divisor) ++l;
    p = 31 + l;
    m = ((1ull << p) + (unsigned long long)divisor - 1) / (unsigned long long)divisor;
  }
  __device__ __forceinline__ int div(int n) const { return (int)(((unsigned long long)(unsigned)n * m) >> p); }
};

struct Args {
  int batch, hq, hkv, group, seqlen_q, seqlen_k;
  FastDiv fd_outer, fd_mid, fd_inner;  // item decode: per-row-block count, then the two inner factors
  float scale_log2;
  int causal;
  int pair_heads;
  int n_row_blocks;
  const int32_t* seqlens_q;
  const int32_t* seqlens_k;
  const int32_t* cu_seqlens_q;  // packed queries: sequence b's rows are [cu[b], cu[b+1]) of total_q
  int total_q;
  void* o;
  float* lse;
  int o_f32;
  int o_tma;  // O rows of a full 32-row warp slice go out through the tm_o tile store
  int sort_items;  // order items by cost (variable lengths) instead of row block
  long long o_bs, o_hs, o_rs;
  long long lse_rows;  // rows per (batch, head) of the LSE tensor: seqlen_q, or total_q when packed
  int32_t* error_flags;
  long long wait_limit;  // cycle bound of every pipeline wait
  int planted;           // debug build: bounds-check site reported as failed
  long long out_rows;    // rows per (batch, head) of O: seqlen_q, or total_q when packed
  // paged keys/values (PAGED kernels only)
  const int32_t* block_table;
  int max_blocks;
  int num_blocks;
};

template <int D>
struct Layout {
  static constexpr int CHUNKS = D / 64;           // 64-column (128-byte) boxes per row
  static constexpr int Q_TILE = BM * D * 2;       // bytes
  static constexpr int KV_TILE = BK * D * 2;
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = Q_OFF + 2 * Q_TILE;
  static constexpr int V_OFF = K_OFF + KSTAGES * KV_TILE;
  // Output staging: one 128-byte-swizzled box of 32 rows x 128 bytes per
  // softmax warp.
  static constexpr int W_STAGE = 32 * 128;
  static constexpr int O_OFF = V_OFF + VSTAGES * KV_TILE;
  static constexpr int BAR_OFF = O_OFF + SOFTMAX_WARPS * W_STAGE;
  // q_full, q_empty, k_full[K], k_empty[K], v_full[V], v_empty[V], s_full[2], p_full[2], o_full[2], mma_done
  static constexpr int NUM_BARS = 2 + 2 * KSTAGES + 2 * VSTAGES + 2 + 2 + 2 + 1;
  static constexpr int MISC_OFF = BAR_OFF + NUM_BARS * 8;  // tmem address, abort flag, item count
  static constexpr int LIST_OFF = MISC_OFF + 16;            // this CTA's items when they are sorted
  static constexpr int BYTES = LIST_OFF + LIST_MAX * 4;
  static_assert(SORT_MAX_ITEMS * 8 <= KSTAGES * KV_TILE, "item sort scratch lives in the K ring");
  static constexpr int SMEM_BYTES = BYTES + 1024;  // slack for 1024-byte alignment
};

struct Work {
  int b, kvh;
  int qoff, qb;  // the sequence's first row and batch coordinate in the Q / O / LSE tensors
  int head[2];
  int row0[2];
  int active[2];
  int n_kv[2];  // key blocks of BK each
  int sq, sk;
};

__device__ __forceinline__ Work decode_work(const Args& a, int item) {
  Work w;
  if (a.pair_heads) {
    // fd_outer: batch * hkv * pairs, fd_mid: pairs, fd_inner: hkv
    const int pairs = a.fd_mid.d;
    const int q0 = a.fd_outer.div(item);
    const int rb = a.n_row_blocks - 1 - q0;  // heaviest (causal) row blocks first
    int r = item - q0 * a.fd_outer.d;
    const int q1 = a.fd_mid.div(r);
    const int pair = r - q1 * pairs;
    r = q1;
    w.b = a.fd_inner.div(r);
    w.kvh = r - w.b * a.hkv;
    w.head[0] = w.kvh * a.group + 2 * pair;
    w.head[1] = w.head[0] + 1;
    w.row0[0] = w.row0[1] = rb * BM;
  } else {
    // fd_outer: batch * hq, fd_mid: hq, fd_inner: group
    const int npairs = (a.n_row_blocks + 1) / 2;
    const int q0 = a.fd_outer.div(item);
    const int p = npairs - 1 - q0;
    const int r = item - q0 * a.fd_outer.d;
    w.b = a.fd_mid.div(r);
    const int h = r - w.b * a.hq;
    w.kvh = a.fd_inner.div(h);
    w.head[0] = w.head[1] = h;
    w.row0[0] = 2 * p * BM;
    w.row0[1] = (2 * p + 1) * BM;
  }
  if (a.cu_seqlens_q) {  // packed: rows [s0, s1) of the [total_q, Hq, D] tensors
    int s0 = a.cu_seqlens_q[w.b], s1 = a.cu_seqlens_q[w.b + 1];
    s0 = min(max(s0, 0), a.total_q);
    s1 = min(max(s1, s0), a.total_q);
    w.qoff = s0;
    w.qb = 0;
    w.sq = s1 - s0;
  } else {
    w.qoff = 0;
    w.qb = w.b;
    w.sq = a.seqlens_q ? a.seqlens_q[w.b] : a.seqlen_q;
  }
  w.sk = a.seqlens_k ? a.seqlens_k[w.b] : a.seqlen_k;
  if (w.sq > a.seqlen_q) w.sq = a.seqlen_q;
  if (w.sq < 0) w.sq = 0;
  if (w.sk < 0) w.sk = 0;
  if (a.block_table && w.sk > a.max_blocks * 16) w.sk = a.max_blocks * 16;  // flagged by the producer
  if (!a.block_table && w.sk > a.seqlen_k) w.sk = a.seqlen_k;  // dense keys end at the tensor's length
  for (int t = 0; t < 2; ++t) {
    w.active[t] = w.row0[t] < w.sq;
    int kend = w.sk;
    if (a.causal) {
      const int last_row = min(w.row0[t] + BM, w.sq) - 1;
      const int lim = last_row + (w.sk - w.sq) + 1;  // keys [0, lim) visible to the tile's last row
      kend = max(0, min(w.sk, lim));
    }
    w.n_kv[t] = w.active[t] ? (kend + BK - 1) / BK : 0;
  }
  return w;
}

// The k-th work item of CTA c in boustrophedon order over heaviest-first
// items: c, 2G-1-c, 2G+c, 4G-1-c, ... (G = gridDim.x), which pairs heavy and
// light causal items on every CTA. Returns -1 past the end.
__device__ __forceinline__ int snake_item(int k, int n_items) {
  const int G = gridDim.x, c = blockIdx.x;
  const int item = k * G + ((k & 1) ? (G - 1 - c) : c);
  return item < n_items ? item : -1;
}

// Variable-length work: every CTA sorts all items by cost, largest first
// (bitonic sort of (cost, ~item) keys in shared scratch, all threads), and
// keeps the ones at its snake positions in the sorted list. Cost is the
// item's key-block count plus a fixed per-item overhead of about 1.4 blocks
// (epilogue and pipeline refill, measured). The scratch is the K ring, which
// no copy has touched yet; a proxy fence orders these writes before the
// first TMA writes there.
__device__ void order_items(const Args& a, int n_items, unsigned long long* keys, int* list, int* n_mine) {
  int np2 = 1;
  while (np2 < n_items) np2 <<= 1;
  for (int i = threadIdx.x; i < np2; i += blockDim.x) {
    unsigned long long key = 0;  // padding sorts last
    if (i < n_items) {
      const Work w = decode_work(a, i);
      const int n = (w.active[0] || w.active[1]) ? max(w.n_kv[0], w.n_kv[1]) : 0;
      const unsigned cost = (unsigned)n * 8u + 11u;
      key = ((unsigned long long)cost << 32) | (unsigned long long)(~(unsigned)i);  // ties: lower item first
    }
    keys[i] = key;
  }
  __syncthreads();
  for (int k = 2; k <= np2; k <<= 1)
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < np2; i += blockDim.x) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const unsigned long long x = keys[i], y = keys[ixj];
          if (((i & k) == 0) ? (x < y) : (x > y)) {  // descending overall
            keys[i] = y;
            keys[ixj] = x;
          }
        }
      }
      __syncthreads();
    }
  if (threadIdx.x == 0) {
    int n = 0;
    for (int k = 0, pos; (pos = snake_item(k, n_items)) >= 0 && n < LIST_MAX; ++k)
      list[n++] = (int)(~(unsigned)(keys[pos] & 0xffffffffull));
    *n_mine = n;
  }
  fence_proxy_async_smem();
  __syncthreads();
}

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Exponentials of one row block of scores (s[]), their sum, and the packed
// bf16 P stored to TMEM 16 columns at a time. EMU8: in every 8 consecutive
// pairs, a spread-out EMU8 of them take exp2 on the FMA pipe (exp2_poly2), the
// rest on MUFU. MASKED: masked scores are -inf; the polynomial clamps its
// input, so its results are then replaced by an exact 0 (MUFU gives 0 itself).
template <int EMU8, bool MASKED = false>
__device__ __forceinline__ void exp_pack_store(const float (&s)[BK], float sl2, float m_off, uint32_t tP,
                                               float2& acc) {
  const float2 sc2 = make_float2(sl2, sl2);
  const float2 mo2 = make_float2(-m_off, -m_off);
  float2 a0 = make_float2(0.f, 0.f), a1 = a0, a2 = a0, a3 = a0;
#pragma unroll
  for (int ch = 0; ch < BK / 32; ++ch) {
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int c = ch * 32 + 2 * i;
      const float2 x = __ffma2_rn(make_float2(s[c], s[c + 1]), sc2, mo2);
      float2 pr;
      if (((i * EMU8) & 7) < EMU8) {
        pr = exp2_poly2(x);
        if (MASKED) {
          pr.x = x.x == -INFINITY ? 0.f : pr.x;
          pr.y = x.y == -INFINITY ? 0.f : pr.y;
        }
      } else {
        pr.x = ex2_approx(x.x);
        pr.y = ex2_approx(x.y);
      }
      if ((i & 3) == 0) a0 = __fadd2_rn(a0, pr);
      if ((i & 3) == 1) a1 = __fadd2_rn(a1, pr);
      if ((i & 3) == 2) a2 = __fadd2_rn(a2, pr);
      if ((i & 3) == 3) a3 = __fadd2_rn(a3, pr);
      pk[i] = pack_bf16x2(pr.x, pr.y);
    }
    tmem_st16(tP + ch * 16, pk);
  }
  acc = __fadd2_rn(__fadd2_rn(a0, a1), __fadd2_rn(a2, a3));
}

template <uint32_t N>
__device__ __forceinline__ void regs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <uint32_t N>
__device__ __forceinline__ void regs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// Epilogue of one warp's 32 rows through shared memory and tile stores.
// Lane l owns row l: its O row (TMEM lane) is scaled by inv_l, converted and
// written into a 128-byte-swizzled box (16-byte unit u of row l lands at unit
// u ^ (l & 7), so the 32 lanes' stores hit all banks), then lane 0 issues one
// tile store per 32-row x 128-byte box. A staging area holds one box, so a
// row goes out in D / 64 (bf16) or D / 32 (fp32) rounds; before a staging
// area is rewritten, lane 0 waits until the previous store has read it.
template <int D, bool F32>
__device__ __forceinline__ void store_rows_tma(const CUtensorMap* tm_o, uint8_t* stage, uint32_t tO, bool has_keys,
                                               float inv_l, int row0, int head, int b) {
  constexpr int COLS = F32 ? 32 : 64;  // columns per 128-byte box
  constexpr int BOXES = D / COLS;
  constexpr int PER_ROUND = 1;
  const int lane = lane_id();
  const int sw = lane & 7;
#pragma unroll
  for (int b0 = 0; b0 < BOXES; b0 += PER_ROUND) {
    if (lane == 0) bulk_wait_group_read0();
    __syncwarp();
#pragma unroll
    for (int bb = 0; bb < PER_ROUND; ++bb) {
      uint8_t* row = stage + bb * 4096 + lane * 128;
#pragma unroll
      for (int h = 0; h < COLS / 32; ++h) {
        const int c = (b0 + bb) * (COLS / 32) + h;  // 32-column TMEM chunk
        uint32_t o[32];
        if (has_keys) {  // warp-uniform: every lane issues the collective load
          tmem_ld32(tO + c * 32, o);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int k = 0; k < 32; ++k) o[k] = 0u;
        }
        if constexpr (F32) {
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            uint4 v;
            v.x = __float_as_uint(__uint_as_float(o[4 * u + 0]) * inv_l);
            v.y = __float_as_uint(__uint_as_float(o[4 * u + 1]) * inv_l);
            v.z = __float_as_uint(__uint_as_float(o[4 * u + 2]) * inv_l);
            v.w = __float_as_uint(__uint_as_float(o[4 * u + 3]) * inv_l);
            *reinterpret_cast<uint4*>(row + ((u ^ sw) << 4)) = v;
          }
        } else {
#pragma unroll
          for (int u4 = 0; u4 < 4; ++u4) {
            const int u = h * 4 + u4;
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(o[8 * u4 + 0]) * inv_l, __uint_as_float(o[8 * u4 + 1]) * inv_l);
            v.y = pack_bf16x2(__uint_as_float(o[8 * u4 + 2]) * inv_l, __uint_as_float(o[8 * u4 + 3]) * inv_l);
            v.z = pack_bf16x2(__uint_as_float(o[8 * u4 + 4]) * inv_l, __uint_as_float(o[8 * u4 + 5]) * inv_l);
            v.w = pack_bf16x2(__uint_as_float(o[8 * u4 + 6]) * inv_l, __uint_as_float(o[8 * u4 + 7]) * inv_l);
            *reinterpret_cast<uint4*>(row + ((u ^ sw) << 4)) = v;
          }
        }
      }
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
#pragma unroll
      for (int bb = 0; bb < PER_ROUND; ++bb) tma_store_4d(tm_o, stage + bb * 4096, (b0 + bb) * COLS, row0, head, b);
      bulk_commit_group();
    }
  }
}

// All lanes of the warp get the same answer (a timeout seen by one lane is
// seen by all), so warp-collective instructions after it stay converged.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, long long limit) {
  return __all_sync(0xffffffffu, mbar_wait_bounded(bar, parity, abort_flag, limit));
}

// Persistent: CTA c processes work items in the snake order of snake_item
// (items are numbered heaviest first). All barrier phases run on per-CTA
// counters that continue across items, so the next item's Q load and first S
// MMA overlap this item's tail.
// PAGED: K and V come from a pool of 16-token blocks [num_blocks, Hkv, 16, D]
// addressed through the block table; the K/V tensor maps then cover the pool.
template <int D, int EMU8, bool PAGED>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    prefill_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                       const Args args, int n_items) {
  using L = Layout<D>;
  static_assert(EMU8 >= 0 && EMU8 <= 8, "EMU8");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
  uint64_t* q_full = bars;
  uint64_t* q_empty = q_full + 1;
  uint64_t* k_full = q_empty + 1;
  uint64_t* k_empty = k_full + KSTAGES;
  uint64_t* v_full = k_empty + KSTAGES;
  uint64_t* v_empty = v_full + VSTAGES;
  // Per tile. S of block i+1 is issued only after P of block i has arrived,
  // so neither side can run a phase ahead and a parity wait never aliases.
  uint64_t* s_full = v_empty + VSTAGES;
  uint64_t* p_full = s_full + 2;
  uint64_t* o_full = p_full + 2;
  uint64_t* mma_done = o_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4);

  const int warp = warp_id();
  const int lane = lane_id();

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);  // the item's last S MMA has read Q
    for (int s = 0; s < KSTAGES; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < VSTAGES; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[t], 128);
      mbar_init(&o_full[t], 1);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == MMA_WARP) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  int* item_list = reinterpret_cast<int*>(smem + L::LIST_OFF);
  int* n_mine = reinterpret_cast<int*>(smem + L::MISC_OFF + 8);
  if (args.sort_items)
    order_items(args, n_items, reinterpret_cast<unsigned long long*>(smem + L::K_OFF), item_list, n_mine);
  // The k-th item of this CTA (-1 past its last).
  auto cta_item = [&](int k) -> int {
    if (args.sort_items) return k < *n_mine ? item_list[k] : -1;
    return snake_item(k, n_items);
  };

  if (warp >= SOFTMAX_WARPS) {
    regs_dec<REG_OTHER>();
    if (warp == TMA_WARP && lane == 0) {
      // ---------------------------------------------------------------- producer
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      int nk = 0, nv = 0;  // K / V blocks issued so far (all items)
      int nq = 0;          // items whose Q was loaded
      bool ok = true;
      for (int kk_item = 0, item; ok && (item = cta_item(kk_item)) >= 0; ++kk_item) {
        const Work w = decode_work(args, item);
        const int n_kv = max(w.n_kv[0], w.n_kv[1]);
        if (!w.active[0] && !w.active[1]) continue;
        if (PAGED && args.seqlens_k[w.b] > args.max_blocks * 16 && args.error_flags)
          atomicOr(args.error_flags, ATTN_FAULT_BAD_LENGTH);
        // Q tiles: wait until the last S MMA of the previous item has read them.
        if (nq > 0 && !mbar_wait_bounded(q_empty, (nq - 1) & 1, abort_flag, args.wait_limit)) break;
        mbar_arrive_expect_tx(q_full, (w.active[0] + w.active[1]) * L::Q_TILE);
        for (int t = 0; t < 2; ++t) {
          if (!w.active[t]) continue;
          for (int c = 0; c < L::CHUNKS; ++c) {
            const int off = L::Q_OFF + t * L::Q_TILE + c * (BM * 128);
            if (ATTN_IN_BOUNDS(off >= L::Q_OFF && off + BM * 128 <= L::Q_OFF + 2 * L::Q_TILE,
                               ATTN_SITE_PREFILL_SMEM_Q, args.error_flags, args.planted))
              tma_load_4d(smem + off, &tm_q, q_full, c * 64, w.qoff + w.row0[t], w.head[t], w.qb);
          }
        }
        ++nq;
        // Bring the next item's Q tiles into L2 now, so that its shared-memory
        // load at the end of this item does not wait on HBM.
        {
          const int nxt = cta_item(kk_item + 1);
          if (nxt >= 0) {
            const Work wn = decode_work(args, nxt);
            for (int t = 0; t < 2; ++t) {
              if (!wn.active[t]) continue;
              for (int c = 0; c < L::CHUNKS; ++c)
                tma_prefetch_l2_4d(&tm_q, c * 64, wn.qoff + wn.row0[t], wn.head[t], wn.qb);
            }
          }
        }
        const int32_t* table = PAGED ? args.block_table + (long long)w.b * args.max_blocks : nullptr;
        // Paged: the physical cache blocks of key block blk, read from the
        // table once for K and V and all before any copy is issued (the copies
        // are ordered memory operations, so reading the table between them
        // would expose one global-load latency per cache block). A block past
        // the sequence end, or a table entry outside the pool (flagged), is
        // read from one past the pool's last block, which TMA fills with zeros.
        int phys[BK / 16];
        auto fetch_table = [&](int blk) {
          if constexpr (PAGED) {
            int e[BK / 16];
#pragma unroll
            for (int j = 0; j < BK / 16; ++j) {
              const int tok = blk * BK + j * 16;
              e[j] = args.num_blocks;
              if (tok < w.sk && ATTN_IN_BOUNDS((tok >> 4) < args.max_blocks, ATTN_SITE_PREFILL_TABLE,
                                               args.error_flags, args.planted))
                e[j] = table[tok >> 4];
            }
#pragma unroll
            for (int j = 0; j < BK / 16; ++j) {
              const int tok = blk * BK + j * 16;
              const bool good = e[j] >= 0 && e[j] < args.num_blocks;
              if (tok < w.sk && !good && args.error_flags) atomicOr(args.error_flags, ATTN_FAULT_BAD_BLOCK);
              phys[j] = good ? e[j] : args.num_blocks;
            }
          }
        };
        auto load = [&](bool is_v, int blk) -> bool {
          int& cnt = is_v ? nv : nk;
          const int stages = is_v ? VSTAGES : KSTAGES;
          uint64_t* full = is_v ? v_full : k_full;
          uint64_t* empty = is_v ? v_empty : k_empty;
          const int s = cnt % stages;
          if (cnt >= stages && !mbar_wait_bounded(&empty[s], ((cnt / stages) - 1) & 1, abort_flag, args.wait_limit))
            return false;
          mbar_arrive_expect_tx(&full[s], L::KV_TILE);
          const int ring = is_v ? L::V_OFF : L::K_OFF;
          uint8_t* dst = smem + ring + s * L::KV_TILE;
          const CUtensorMap* tm = is_v ? &tm_v : &tm_k;
          if constexpr (!PAGED) {
            for (int c = 0; c < L::CHUNKS; ++c)
              if (ATTN_IN_BOUNDS(s >= 0 && s < stages && (s * L::KV_TILE + c * (BK * 128) + BK * 128 <=
                                                          stages * L::KV_TILE),
                                 ATTN_SITE_PREFILL_SMEM_KV, args.error_flags, args.planted))
                tma_load_4d(dst + c * (BK * 128), tm, &full[s], c * 64, blk * BK, w.kvh, w.b);
          } else {
            for (int j = 0; j < BK / 16; ++j)
              for (int c = 0; c < L::CHUNKS; ++c)
                if (ATTN_IN_BOUNDS(s >= 0 && s < stages && (s * L::KV_TILE + c * (BK * 128) + j * (16 * 128) +
                                                                16 * 128 <= stages * L::KV_TILE),
                                   ATTN_SITE_PREFILL_SMEM_KV, args.error_flags, args.planted))
                  tma_load_4d(dst + c * (BK * 128) + j * (16 * 128), tm, &full[s], c * 64, 0, w.kvh, phys[j]);
          }
          ++cnt;
          return true;
        };
        // The tensor core consumes K_0, V_0, K_1, V_1, ...; each load first
        // waits for the block two back in its ring to be released.
        for (int i = 0; i < n_kv && ok; ++i) {
          fetch_table(i);
          ok = load(false, i);
          if (ok) ok = load(true, i);
        }
      }
      // Drain: wait for the last copy issued into each slot (a slot's earlier
      // copy completed before its empty barrier let the next one start), so no
      // copy is in flight when the CTA exits. On the abort path the consumers
      // have stopped, but every copy issued still lands by itself, so these
      // waits ignore the abort flag.
      for (int i = max(0, nk - KSTAGES); i < nk; ++i) mbar_wait_drain(&k_full[i % KSTAGES], (i / KSTAGES) & 1);
      for (int i = max(0, nv - VSTAGES); i < nv; ++i) mbar_wait_drain(&v_full[i % VSTAGES], (i / VSTAGES) & 1);
      if (nq > 0) mbar_wait_drain(q_full, (nq - 1) & 1);
    } else if (warp == MMA_WARP && lane == 0) {
      // ---------------------------------------------------------------- MMA issuer (both tiles)
      // One thread issues every MMA in the fixed order S_0(0), S_1(0), then per
      // block i: P_0 V_i, S_0(i+1), P_1 V_i, S_1(i+1). The tensor core runs them
      // in that order, so tile 1's products fill the pipe while tile 0's
      // softmax works and the other way round.
      constexpr uint32_t ID_S = instr_desc_bf16(BM, BK, 0);
      constexpr uint32_t ID_PV = instr_desc_bf16(BM, D, 1);
      // Shared-memory descriptors as low words (start address, leading byte
      // offset) over one common high word (stride 1024 bytes, 128-byte
      // swizzle); each MMA adds its k-step offset as an immediate.
      const uint32_t hi = sw128_desc_hi(1024);
      const uint32_t q_lo = sw128_desc_lo(smem_addr(smem + L::Q_OFF), 16);       // K-major
      const uint32_t k_lo = sw128_desc_lo(smem_addr(smem + L::K_OFF), 16);       // K-major
      const uint32_t v_lo = sw128_desc_lo(smem_addr(smem + L::V_OFF), BK * 128);  // MN-major
      const uint32_t id_s = ID_S, id_pv = ID_PV;
      // S_t = Q_t K^T for the K block in ring position kg.
      auto issue_s = [&](int t, int kg) {
        const uint32_t qa = q_lo + (uint32_t)((t * L::Q_TILE) >> 4);
        const uint32_t ka = k_lo + (uint32_t)(((kg % KSTAGES) * L::KV_TILE) >> 4);
        const uint32_t d = tmem_base + t * 128;
        if (!ATTN_IN_BOUNDS(t >= 0 && t < 2 && t * 128 + BK <= 256, ATTN_SITE_PREFILL_TMEM_S, args.error_flags,
                            args.planted))
          return;
        static_for<0, D / 16>([&](auto c) {
          constexpr int kk = decltype(c)::value;
          constexpr uint32_t a_off = ((kk >> 2) * (BM * 128) + (kk & 3) * 32) >> 4;
          constexpr uint32_t b_off = ((kk >> 2) * (BK * 128) + (kk & 3) * 32) >> 4;
          mma_ss_lo<a_off, b_off>(d, qa, ka, hi, id_s, kk > 0 ? 1u : 0u);
        });
      };
      // O_t (+)= P_t V, P from TMEM (bf16 pairs over S_t's first BK / 2
      // columns), V in ring position vg.
      auto issue_pv = [&](int t, int vg, bool first) {
        const uint32_t va = v_lo + (uint32_t)(((vg % VSTAGES) * L::KV_TILE) >> 4);
        const uint32_t d = tmem_base + 256 + t * 128, a = tmem_base + t * 128;
        if (!ATTN_IN_BOUNDS(t >= 0 && t < 2 && 256 + t * 128 + D <= (int)TMEM_COLS, ATTN_SITE_PREFILL_TMEM_O,
                            args.error_flags, args.planted))
          return;
        static_for<0, BK / 16>([&](auto c) {
          constexpr int kk = decltype(c)::value;
          constexpr uint32_t b_off = (kk * 16 * 128) >> 4;
          mma_ts_lo<kk * 8, b_off>(d, a, va, hi, id_pv, (!first || kk > 0) ? 1u : 0u);
        });
      };
      int gb[2] = {0, 0};  // each tile's blocks so far (all items): S / P barrier phases
      int kb = 0;          // K / V blocks loaded before the current item (both rings advance alike)
      int nq = 0;          // active items so far (Q phases)
      bool ok = true;
      for (int kk_item = 0, item; ok && (item = cta_item(kk_item)) >= 0; ++kk_item) {
        const Work w = decode_work(args, item);
        if (!w.active[0] && !w.active[1]) continue;
        const int n_kv = max(w.n_kv[0], w.n_kv[1]);
        // S of block i for every tile that has it; then K_i can be released.
        auto s_blocks = [&](int i) -> bool {
          const int kg = kb + i;
          if (!mbar_wait_bounded(&k_full[kg % KSTAGES], (kg / KSTAGES) & 1, abort_flag, args.wait_limit)) return false;
          tc_fence_after();
          for (int t = 0; t < 2; ++t) {
            if (i >= w.n_kv[t]) continue;
            issue_s(t, kg);
            mma_commit(&s_full[t]);
          }
          mma_commit(&k_empty[kg % KSTAGES]);
          if (i == n_kv - 1) mma_commit(q_empty);  // the item's last S MMA has been issued
          return true;
        };
        ok = mbar_wait_bounded(q_full, nq & 1, abort_flag, args.wait_limit);
        if (ok && n_kv == 0) {
          // Every row of the item sees no key: no K/V block was loaded and no
          // MMA reads Q. Hand the Q buffer back at once (the epilogue writes
          // O = 0 and LSE = -inf without tensor memory).
          mma_commit(q_empty);
        } else if (ok) {
          ok = s_blocks(0);
        }
        for (int i = 0; i < n_kv && ok; ++i) {
          const int vg = kb + i;  // V_i is the (kb + i)-th V block
          ok = mbar_wait_bounded(&v_full[vg % VSTAGES], (vg / VSTAGES) & 1, abort_flag, args.wait_limit);
          const bool next = i + 1 < n_kv;
          const int kg = kb + i + 1;
          if (ok && next) ok = mbar_wait_bounded(&k_full[kg % KSTAGES], (kg / KSTAGES) & 1, abort_flag, args.wait_limit);
          for (int t = 0; t < 2 && ok; ++t) {
            if (i >= w.n_kv[t]) continue;
            ok = mbar_wait_bounded(&p_full[t], (gb[t] + i) & 1, abort_flag, args.wait_limit);
            if (!ok) break;
            tc_fence_after();
            issue_pv(t, vg, i == 0);
            if (i == w.n_kv[t] - 1) mma_commit(&o_full[t]);
            // S_t(i+1) overwrites the P just read: MMAs from one thread run
            // in issue order.
            if (i + 1 < w.n_kv[t]) {
              issue_s(t, kg);
              mma_commit(&s_full[t]);
            }
          }
          if (!ok) break;
          mma_commit(&v_empty[vg % VSTAGES]);
          if (next) {
            mma_commit(&k_empty[kg % KSTAGES]);
            if (i + 1 == n_kv - 1) mma_commit(q_empty);
          }
        }
        gb[0] += w.n_kv[0];
        gb[1] += w.n_kv[1];
        kb += n_kv;
        ++nq;
      }
      // Wait until every MMA issued has completed before tensor memory can be
      // released (on the abort path too: the issued MMAs finish by themselves).
      mma_commit(mma_done);
      mbar_wait_drain(mma_done, 0);
    }
  } else {
    regs_inc<REG_SOFTMAX>();
    // ---------------------------------------------------------------- softmax + epilogue
    const int t = warp >> 2;
    const int sub = warp & 3;
    const int r = sub * 32 + lane;  // row within the tile == TMEM lane
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(sub * 32) << 16);
    const uint32_t tS = lane_base + t * 128;
    const uint32_t tO = lane_base + 256 + t * 128;
    const float sl2 = args.scale_log2;
    // This warp's S / P and O columns stay inside the allocation.
    const bool s_cols = ATTN_IN_BOUNDS(t >= 0 && t < 2 && t * 128 + BK <= 256, ATTN_SITE_PREFILL_TMEM_S,
                                       args.error_flags, args.planted);
    const bool o_cols = ATTN_IN_BOUNDS(t >= 0 && t < 2 && 256 + t * 128 + D <= (int)TMEM_COLS,
                                       ATTN_SITE_PREFILL_TMEM_O, args.error_flags, args.planted);
    (void)s_cols;
    (void)o_cols;
    int gb = 0;  // this tile's blocks so far (all items)
    int kb = 0;  // K / V blocks loaded before the current item
    int nf = 0;  // items this tile finished (o_full phases)
    bool ok = true;
    for (int kk_item = 0, item; ok && (item = cta_item(kk_item)) >= 0; ++kk_item) {
      const Work w = decode_work(args, item);
      if (!w.active[0] && !w.active[1]) continue;
      const int n_kv = max(w.n_kv[0], w.n_kv[1]);
      const int nt = w.n_kv[t];
      if (!w.active[t]) {
        kb += n_kv;
        continue;
      }
      // Paged: the item's last V block may hold rows past the sequence end
      // (tail slots of a partly filled cache block); they are zeroed in shared
      // memory before this tile's last P V, because 0 * NaN would poison O.
      const bool v_fix = PAGED && nt == n_kv && nt > 0 && (w.sk & 15) != 0 && nt * BK > w.sk;
      const int qrow = w.row0[t] + r;
      const int qpos = qrow + (w.sk - w.sq);  // absolute position (bottom-right causal)
      float m2 = -INFINITY;  // running max of s * scale * log2(e)
      float l = 0.f;         // running sum of 2^(s*scale*log2e - m2)
      for (int i = 0; i < nt; ++i) {
        const int g = gb + i;
        ok = warp_wait(&s_full[t], g & 1, abort_flag, args.wait_limit);
        if (!ok) break;
        tc_fence_after();
        uint32_t sb[BK];
#pragma unroll
        for (int c = 0; c < BK / 32; ++c)
          if (s_cols) tmem_ld32(tS + c * 32, &sb[c * 32]);
        tmem_ld_wait();
        float s[BK];
#pragma unroll
        for (int c = 0; c < BK; ++c) s[c] = __uint_as_float(sb[c]);
        const int k0 = i * BK;
        const bool need_mask = (k0 + BK > w.sk) || (args.causal && (k0 + BK - 1 > w.row0[t] + (w.sk - w.sq)));
        if (need_mask) {
          const int lim = args.causal ? min(w.sk, qpos + 1) : w.sk;  // keys [0, lim) visible
#pragma unroll
          for (int c = 0; c < BK; ++c)
            if (k0 + c >= lim) s[c] = -INFINITY;
        }
        // Row max: eight independent max3 chains.
        float am[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) am[k] = fmaxf(s[k], s[k + 8]);
#pragma unroll
        for (int c = 16; c < BK; c += 16)
#pragma unroll
          for (int k = 0; k < 8; ++k) am[k] = max3f(am[k], s[c + k], s[c + k + 8]);
        const float mx = max3f(max3f(am[0], am[1], am[2]), max3f(am[3], am[4], am[5]), fmaxf(am[6], am[7]));
        const float m_new = fmaxf(m2, mx * sl2);
        const bool upd = (m_new - m2) > RESCALE_THRESHOLD;  // false when both are -inf (NaN compare)
        const float alpha = upd ? ex2_approx(m2 - m_new) : 1.f;
        if (upd) m2 = m_new;
        const float m_off = (m2 == -INFINITY) ? 0.f : m2;
        if (i > 0 && __any_sync(0xffffffffu, upd) && o_cols) {
          // Rescale O in place. Its last writer, P V of the previous block,
          // has completed: the commit that signalled this S tracks every
          // earlier MMA of the issuer.
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(tO + c * 32, o);
            tmem_ld_wait();
#pragma unroll
            for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
            tmem_st32(tO + c * 32, o);
          }
        }
        float2 acc = make_float2(0.f, 0.f);
        if (!s_cols) {
        } else if (need_mask) {
          exp_pack_store<EMU8, true>(s, sl2, m_off, tS, acc);
        } else {
          exp_pack_store<EMU8>(s, sl2, m_off, tS, acc);
        }
        l = l * alpha + (acc.x + acc.y);
        if (v_fix && i == nt - 1) {
          const int vg = kb + i, vs = vg % VSTAGES;
          ok = warp_wait(&v_full[vs], (vg / VSTAGES) & 1, abort_flag, args.wait_limit);
          if (!ok) {
            tmem_st_wait();  // this block's P stores, before tensor memory can be freed
            break;
          }
          uint8_t* vblk = smem + L::V_OFF + vs * L::KV_TILE;
          const int r0 = w.sk - k0;  // first row past the sequence end
          const int units = (BK - r0) * L::CHUNKS * 8;  // 16-byte units to clear
          for (int u = r; u < units; u += 128) {
            const int unit = u & 7, rc = u >> 3;
            const int row = r0 + rc % (BK - r0), c = rc / (BK - r0);
            const int off = c * (BK * 128) + row * 128 + unit * 16;
            if (ATTN_IN_BOUNDS(vs >= 0 && vs < VSTAGES && row >= 0 && row < BK && off >= 0 && off + 16 <= L::KV_TILE,
                               ATTN_SITE_PREFILL_SMEM_VFIX, args.error_flags, args.planted))
              *reinterpret_cast<uint4*>(vblk + off) = make_uint4(0u, 0u, 0u, 0u);
          }
          fence_proxy_async_smem();
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&p_full[t]);
      }
      gb += nt;
      kb += n_kv;
      if (!ok) break;
      // ------------------------------------------------------------ epilogue
      // 1 / l and the LSE need no TMEM: done while the last P V runs.
      const bool store = qrow < w.sq;
      const bool empty = !(l > 0.f);
      const float inv_l = empty ? 0.f : 1.f / l;
      // The row, head and batch coordinates of this row's O and LSE (rows
      // past the sequence end are not stored).
      const bool out_ok =
          !store || ATTN_IN_BOUNDS(w.qoff + qrow >= 0 && w.qoff + qrow < args.out_rows && w.head[t] >= 0 &&
                                       w.head[t] < args.hq && w.qb >= 0 && w.qb < (args.cu_seqlens_q ? 1 : args.batch),
                                   ATTN_SITE_PREFILL_OUT, args.error_flags, args.planted);
      if (args.lse && store && out_ok) {
        const float lse = empty ? -INFINITY : (m2 + log2f(l)) * 0.69314718055994530942f;
        args.lse[((long long)w.qb * args.hq + w.head[t]) * args.lse_rows + w.qoff + qrow] = lse;
      }
      const bool has_keys = nt > 0;
      if (has_keys) {
        ok = warp_wait(&o_full[t], nf & 1, abort_flag, args.wait_limit);
        ++nf;
        if (!ok) break;
      }
      const long long obase = (long long)w.qb * args.o_bs + (long long)w.head[t] * args.o_hs +
                              (long long)(w.qoff + qrow) * args.o_rs;
      if (has_keys) tc_fence_after();
      if (args.o_tma && w.row0[t] + sub * 32 + 32 <= w.sq) {  // warp-uniform
        uint8_t* stage = smem + L::O_OFF + warp * L::W_STAGE;
        const int r0 = w.qoff + w.row0[t] + sub * 32;
        // The warp's staging area (one 4 KB box per round) and its 32 output
        // rows.
        if (ATTN_IN_BOUNDS(warp >= 0 && warp < SOFTMAX_WARPS &&
                               L::O_OFF + (warp + 1) * L::W_STAGE <= L::BAR_OFF && 4096 <= L::W_STAGE &&
                               r0 >= 0 && r0 + 32 <= args.out_rows,
                           ATTN_SITE_PREFILL_SMEM_STAGE, args.error_flags, args.planted)) {
          if (args.o_f32)
            store_rows_tma<D, true>(&tm_o, stage, tO, has_keys && o_cols, inv_l, r0, w.head[t], w.qb);
          else
            store_rows_tma<D, false>(&tm_o, stage, tO, has_keys && o_cols, inv_l, r0, w.head[t], w.qb);
        }
        continue;
      }
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        if (has_keys && o_cols) {  // warp-uniform: every lane issues the collective load
          tmem_ld32(tO + c * 32, o);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int k = 0; k < 32; ++k) o[k] = 0u;
        }
        if (!store || !out_ok) continue;
        if (args.o_f32) {
          float* dst = reinterpret_cast<float*>(args.o) + obase + c * 32;
#pragma unroll
          for (int k = 0; k < 32; k += 4) {
            float4 v = make_float4(__uint_as_float(o[k]) * inv_l, __uint_as_float(o[k + 1]) * inv_l,
                                   __uint_as_float(o[k + 2]) * inv_l, __uint_as_float(o[k + 3]) * inv_l);
            *reinterpret_cast<float4*>(dst + k) = v;
          }
        } else {
          __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(args.o) + obase + c * 32;
#pragma unroll
          for (int k = 0; k < 32; k += 8) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(o[k + 0]) * inv_l, __uint_as_float(o[k + 1]) * inv_l);
            v.y = pack_bf16x2(__uint_as_float(o[k + 2]) * inv_l, __uint_as_float(o[k + 3]) * inv_l);
            v.z = pack_bf16x2(__uint_as_float(o[k + 4]) * inv_l, __uint_as_float(o[k + 5]) * inv_l);
            v.w = pack_bf16x2(__uint_as_float(o[k + 6]) * inv_l, __uint_as_float(o[k + 7]) * inv_l);
            *reinterpret_cast<uint4*>(dst + k) = v;
          }
        }
      }
      // The next item's first P V overwrites O_t only after this thread's
      // next p_full arrival, which follows these loads (tcgen05.wait::ld).
    }
    // Tile stores still in flight must finish before the CTA exits.
    if (lane == 0) bulk_wait_group0();
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag && args.error_flags) atomicOr(args.error_flags, ATTN_FAULT_TIMEOUT);
  if (warp == MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
  // The driver entry point is process-wide; a function-local static is
  // initialised once, thread-safely.
  static const EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<EncodeTiledFn>(ptr);
    cudaGetLastError();
    return nullptr;
  }();
  return fn;
}

// 4-D map over [d3][d2][d1][d0 = head_dim] with byte strides s1..s3, box
// (128 bytes of d0, box_rows, 1, 1), 128-byte swizzle, zero fill out of bounds.
static bool encode_4d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t d3,
                      uint64_t s1, uint64_t s2, uint64_t s3, uint32_t box_rows, bool f32 = false) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {d0, d1, d2, d3};
  cuuint64_t strides[3] = {s1, s2, s3};
  cuuint32_t box[4] = {f32 ? 32u : 64u, box_rows, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
                  const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D, int EMU8, bool PAGED>
static attn_status_t launch_variant(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                    const CUtensorMap& to, const Args& a, int items, cudaStream_t stream) {
  using L = Layout<D>;
  static_assert(L::SMEM_BYTES <= 232448, "shared memory budget");
  auto kern = prefill_fwd_kernel<D, EMU8, PAGED>;
  static DeviceOnce setup;
  const attn_status_t st = setup.run([&]() -> attn_status_t {
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) {
      cudaGetLastError();
      return ATTN_ERR_CUDA;
    }
    // The in-kernel register split assumes exactly REG_LAUNCH registers per
    // thread at launch; anything else could make setmaxnreg.inc wait forever.
    if (fa.numRegs != REG_LAUNCH) return ATTN_ERR_UNSUPPORTED;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM_BYTES) != cudaSuccess) {
      cudaGetLastError();
      return ATTN_ERR_CUDA;
    }
    return ATTN_OK;
  });
  if (st != ATTN_OK) return st;
  const int grid = items < device_sm_count() ? items : device_sm_count();
  Args ak = a;
  // Sort only when lengths vary per sequence and every CTA's share fits its list.
  ak.sort_items = (a.seqlens_q || a.seqlens_k || a.cu_seqlens_q) && items <= SORT_MAX_ITEMS &&
                  (items + grid - 1) / grid <= LIST_MAX;
  kern<<<grid, NUM_THREADS, L::SMEM_BYTES, stream>>>(tq, tk, tv, to, ak, items);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace prefill

attn_status_t launch_prefill(const attn_prefill_params& p, cudaStream_t stream) {
  using namespace prefill;
  if (p.batch == 0 || p.seqlen_q == 0 || p.num_q_heads == 0) return ATTN_OK;
  const bool paged = p.k_cache != nullptr;
  const int D = p.head_dim;
  // Packed queries ([total_q, Hq, D] rows addressed through cu_seqlens_q) are
  // one "batch" of total_q rows to the tensor maps.
  const bool packed = p.cu_seqlens_q != nullptr;
  const uint64_t q_rows = packed ? (uint64_t)p.total_q : (uint64_t)p.seqlen_q;
  const uint64_t q_batches = packed ? 1 : (uint64_t)p.batch;
  const int64_t q_bs = packed ? p.q_row_stride * (int64_t)p.total_q : p.q_batch_stride;
  const int64_t o_bs = packed ? p.o_row_stride * (int64_t)p.total_q : p.o_batch_stride;
  CUtensorMap tq, tk, tv;
  if (!encode_4d(&tq, p.q, D, q_rows, p.num_q_heads, q_batches, p.q_row_stride * 2, p.q_head_stride * 2, q_bs * 2,
                 BM))
    return ATTN_ERR_CUDA;
  if (paged) {
    // Pools [num_blocks, Hkv, 16, D]: one 16-row box per cache block and D chunk.
    const uint64_t row = (uint64_t)D * 2, blk = 16 * row, nb = blk * p.num_kv_heads;
    if (!encode_4d(&tk, p.k_cache, D, 16, p.num_kv_heads, p.num_blocks, row, blk, nb, 16) ||
        !encode_4d(&tv, p.v_cache, D, 16, p.num_kv_heads, p.num_blocks, row, blk, nb, 16))
      return ATTN_ERR_CUDA;
  } else if (p.seqlen_k > 0) {
    if (!encode_4d(&tk, p.k, D, p.seqlen_k, p.num_kv_heads, p.batch, p.k_row_stride * 2, p.k_head_stride * 2,
                   p.k_batch_stride * 2, BK) ||
        !encode_4d(&tv, p.v, D, p.seqlen_k, p.num_kv_heads, p.batch, p.v_row_stride * 2, p.v_head_stride * 2,
                   p.v_batch_stride * 2, BK))
      return ATTN_ERR_CUDA;
  } else {
    tk = tq;  // no keys: nothing is loaded through these maps
    tv = tq;
  }

  Args a;
  memset(&a, 0, sizeof(a));
  a.batch = p.batch;
  a.hq = p.num_q_heads;
  a.hkv = p.num_kv_heads;
  a.group = p.num_q_heads / p.num_kv_heads;
  a.seqlen_q = p.seqlen_q;
  a.seqlen_k = p.seqlen_k;
  a.scale_log2 = p.scale * 1.4426950408889634f;
  a.causal = p.causal ? 1 : 0;
  a.pair_heads = (a.group % 2 == 0) ? 1 : 0;
  if (a.pair_heads) {
    a.fd_outer.init(p.batch * p.num_kv_heads * (a.group / 2));
    a.fd_mid.init(a.group / 2);
    a.fd_inner.init(p.num_kv_heads);
  } else {
    a.fd_outer.init(p.batch * p.num_q_heads);
    a.fd_mid.init(p.num_q_heads);
    a.fd_inner.init(a.group);
  }
  a.n_row_blocks = (p.seqlen_q + BM - 1) / BM;
  a.seqlens_q = p.seqlens_q;
  a.seqlens_k = p.seqlens_k;
  a.cu_seqlens_q = p.cu_seqlens_q;
  a.total_q = packed ? p.total_q : 0;
  a.lse_rows = packed ? p.total_q : p.seqlen_q;
  a.o = p.o;
  a.lse = p.lse;
  a.o_f32 = p.o_dtype == ATTN_DTYPE_F32;
  a.o_bs = o_bs;
  a.o_hs = p.o_head_stride;
  a.o_rs = p.o_row_stride;
  // O goes out through tile stores when its map encodes (the API's alignment
  // rules make that the normal case); otherwise every row is stored directly.
  const int esz = a.o_f32 ? 4 : 2;
  CUtensorMap to;
  a.o_tma = encode_4d(&to, p.o, D, q_rows, p.num_q_heads, q_batches, p.o_row_stride * esz, p.o_head_stride * esz,
                      o_bs * esz, 32, a.o_f32 != 0)
                ? 1
                : 0;
  if (!a.o_tma) to = tq;  // never read
  a.error_flags = p.error_flags;
  a.wait_limit = pipeline_wait_limit();
  a.planted = planted_bounds_site();
  a.out_rows = a.lse_rows;
  if (paged) {
    a.block_table = p.block_table;
    a.max_blocks = p.max_blocks_per_seq;
    a.num_blocks = p.num_blocks;
  }
  long long items;
  if (a.pair_heads)
    items = (long long)a.n_row_blocks * p.batch * p.num_kv_heads * (a.group / 2);
  else
    items = (long long)((a.n_row_blocks + 1) / 2) * p.batch * p.num_q_heads;
  if (items <= 0) return ATTN_OK;
  if (items > 0x7fffffffLL) return ATTN_ERR_INVALID_ARG;

  // A quarter of the exponentials go to the FMA-pipe polynomial (measured best
  // on B200 for head_dim 128: the MUFU pipe is the scarcer resource).
  if (paged) {
    if (D == 128) return launch_variant<128, 2, true>(tq, tk, tv, to, a, (int)items, stream);
    return launch_variant<64, 2, true>(tq, tk, tv, to, a, (int)items, stream);
  }
  if (D == 128) return launch_variant<128, 2, false>(tq, tk, tv, to, a, (int)items, stream);
  return launch_variant<64, 2, false>(tq, tk, tv, to, a, (int)items, stream);
}

}  // namespace attn
