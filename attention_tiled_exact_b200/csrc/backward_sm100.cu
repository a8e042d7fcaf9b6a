// Backward of exact attention for sm_100a: dQ, dK, dV from Q, K, V, the
// forward's O and LSE, and the upstream gradient dO.
//
// What it computes (the plain derivatives of O = softmax(scale Q K^T + mask) V;
// FlashAttention-2 has one forward and one backward kernel, "GPU Kernel 调度:
// 大模型推理的拐点 2026", the four-layer decomposition): per query head, with
// P = exp(scale Q K^T - LSE) (masked entries 0),
//     dV = P^T dO,   dP = dO V^T,   D_i = rowsum(dO * O)_i,
//     dS = P * (dP - D),   dQ = scale dS K,   dK = scale dS^T Q,
// dK and dV of a key/value head summing its G query heads. Nothing of size
// Sq x Sk goes to HBM: P and dS are rebuilt tile by tile from Q, K and the
// forward's LSE, exactly as the forward builds S tile by tile.
//
// Three launches:
//   * prep (one CTA per (batch, head, 128-row block), 16-byte loads, four
//     rows of a thread in flight): -D = -rowsum(dO * O) and -LSE log2(e)
//     (-inf for rows that see no key, so that their P is exactly 0), padded
//     to whole 128-row blocks;
//   * dK/dV kernel, persistent (one CTA per SM over the (batch, kv head,
//     128-key block j) items, heaviest first): K_j and V_j stay in shared
//     memory for the item; for every query head of the group and every query
//     block i that sees block j, TMA streams Q_i and dO_i through a two-stage
//     ring and one thread issues
//         S^T = K_j Q_i^T, dP^T = V_j dO_i^T          (tcgen05, fp32 in TMEM)
//     two warpgroups (one key row per thread, the TMEM lane; 64 query columns
//     each) turn them into P^T = exp2(S^T scale log2 e - LSE log2 e) and
//     dS^T = P^T (dP^T - D), written back into TMEM as bf16, and the thread
//     issues
//         dV += P^T dO_i, dK += dS^T Q_i              (A from TMEM)
//     into two accumulators that stay in TMEM for the item;
//   * dQ kernel, persistent over the (batch, query head, 128-query block i)
//     items: Q_i and dO_i stay in shared memory for the item, K_j and V_j
//     stream, S and dP are recomputed the same way and dQ += dS K_j
//     accumulates in TMEM. It is launched as a programmatic dependent of the
//     dK/dV kernel, whose results it does not read, so that its CTAs start on
//     the SMs the dK/dV kernel's last items leave.
// dQ is recomputed rather than accumulated with atomics from the dK/dV
// kernel (7 products per tile pair instead of 5): the result is
// deterministic, and TMEM has no room for a fifth 128-column accumulator
// next to S^T, dP^T, dK and dV.
//
// Every operand form here is one the forward kernel also uses: K-major A and
// B from shared memory for S-like products, A from TMEM with an MN-major B
// tile (rows of the tile = the reduction) for the accumulating products.
// Every mbarrier wait is bounded; on a timeout the CTA stops, drains and
// reports ATTN_FAULT_TIMEOUT.
#include <cuda.h>
#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include "bounds_check.cuh"
#include "internal.h"
#include "sm100_ptx.cuh"

namespace attn {

namespace bwd {

constexpr int BM = 128;              // rows of every tile (queries or keys)
constexpr int EW_WARPS = 8;          // two elementwise warpgroups, one per 64-column half
constexpr int TMA_WARP = 8;
constexpr int MMA_WARP = 9;
constexpr int NUM_THREADS = 320;
static_assert(TMA_WARP == EW_WARPS && MMA_WARP == EW_WARPS + 1 && NUM_THREADS == (EW_WARPS + 2) * 32, "warp roles");
constexpr uint32_t TMEM_COLS = 512;
constexpr float LOG2E = 1.4426950408889634f;

struct Args {
  int batch, hq, hkv, group, seqlen_q, seqlen_k, n_qb, n_kb;
  int causal;
  float scale, scale_log2;
  // Per query row, padded to whole 128-row blocks: [B, Hq, n_qb * 128],
  // both negated so that the elementwise step is one packed FMA and one
  // packed add per pair.
  const float* lse2;   // -LSE * log2(e); -inf where the row sees no key and past Sq
  const float* delta;  // -rowsum(dO * O); 0 past Sq
  void* dq;
  void* dk;
  void* dv;
  long long dq_bs, dq_hs, dq_rs, dk_bs, dk_hs, dk_rs, dv_bs, dv_hs, dv_rs;
  int grad_f32;
  int32_t* error_flags;
  long long wait_limit;  // cycle bound of every pipeline wait
  int planted;           // debug build: bounds-check site reported as failed
};

// dK/dV kernel shared memory: K_j and V_j resident; a two-stage ring of
// (Q_i, dO_i) pairs with that query block's -LSE log2 e and -D per column.
template <int D>
struct KvLayout {
  static constexpr int CHUNKS = D / 64;  // 64-column (128-byte) boxes per row
  static constexpr int TILE = BM * D * 2;
  static constexpr int K_OFF = 0;
  static constexpr int V_OFF = TILE;
  static constexpr int RING_OFF = 2 * TILE;            // stage s: Q at + 2 s TILE, dO at + (2 s + 1) TILE
  static constexpr int VEC_OFF = RING_OFF + 4 * TILE;  // [stage][lse2, delta][BM] floats
  static constexpr int BAR_OFF = VEC_OFF + 2 * 2 * BM * 4;
  // a_full, a_empty, ring_full[2], ring_empty[2], s_full, dp_full, p_full, ds_full, acc_full, mma_done
  static constexpr int NUM_BARS = 12;
  static constexpr int MISC_OFF = BAR_OFF + NUM_BARS * 8;  // tmem address, abort flag
  static constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;  // + slack for 1024-byte alignment
};

// dQ kernel shared memory: Q_i and dO_i resident; K_j in a three-slot ring
// (S_j is issued two steps ahead and dQ += dS_j K_j reads K_j last), V_j in a
// two-slot ring.
template <int D>
struct QLayout {
  static constexpr int CHUNKS = D / 64;
  static constexpr int TILE = BM * D * 2;
  static constexpr int K_SLOTS = 3;
  static constexpr int V_SLOTS = 2;
  static constexpr int Q_OFF = 0;
  static constexpr int DO_OFF = TILE;
  static constexpr int K_OFF = 2 * TILE;
  static constexpr int V_OFF = K_OFF + K_SLOTS * TILE;
  static constexpr int BAR_OFF = V_OFF + V_SLOTS * TILE;
  // a_full, a_empty, k_full[3], k_empty[3], v_full[2], v_empty[2], sdp_full, ps_full, acc_full, mma_done
  static constexpr int NUM_BARS = 2 + 2 * K_SLOTS + 2 * V_SLOTS + 4;
  static constexpr int MISC_OFF = BAR_OFF + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;
};

// Tensor memory (512 columns). Every S-like product is one 128 x 128 tile
// (N = 128: a tcgen05.mma of N = 64 costs nearly as long as one of N = 128,
// measured), so the buffers are whole tiles:
//   dK/dV kernel: S^T and dP^T of a step alternate between buffers X (0) and
//   Y (128); dV at 256, dK at 256 + D. The S^T buffer then holds P^T (bf16
//   pairs) over the first 32 columns of each 64-column half and dS^T over the
//   last 32.
//   dQ kernel: S and dP of step t are products 2t and 2t + 1, product p in
//   buffer p mod 3 (columns 0, 128, 256); dQ at 384. The dP buffer then holds
//   dS (bf16 pairs) over the first 32 columns of each half.
constexpr uint32_t COL_ACC_KV = 256, COL_ACC_Q = 384;

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, long long limit) {
  return __all_sync(0xffffffffu, mbar_wait_bounded(bar, parity, abort_flag, limit));
}

// Contiguous global -> shared copy completing on an mbarrier (no multicast).
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_addr(dst)),
               "l"(src), "r"(bytes), "r"(smem_addr(bar))
               : "memory");
}

// Four consecutive floats from shared memory (32-bit shared address). Not
// ordered against the mbarrier waits by a memory clobber: every use sits after
// the wait that made the data visible, in the same thread, and volatile asm
// keeps its place among the other volatile asm statements.
__device__ __forceinline__ float4 lds_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
  return v;
}

// Stores one 32-column slice of a gradient row (fp32 or bf16).
__device__ __forceinline__ void store_slice(void* base, long long off, int col0, const float* x, int f32) {
  if (f32) {
    float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(base) + off + col0);
#pragma unroll
    for (int k = 0; k < 8; ++k) dst[k] = make_float4(x[4 * k], x[4 * k + 1], x[4 * k + 2], x[4 * k + 3]);
  } else {
    uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(base) + off + col0);
#pragma unroll
    for (int k = 0; k < 4; ++k)
      dst[k] = make_uint4(pack_bf16x2(x[8 * k], x[8 * k + 1]), pack_bf16x2(x[8 * k + 2], x[8 * k + 3]),
                          pack_bf16x2(x[8 * k + 4], x[8 * k + 5]), pack_bf16x2(x[8 * k + 6], x[8 * k + 7]));
  }
}

// X (128 x 128) = A (BM x D) * B (BM x D)^T over head_dim, both operands
// K-major 128-row tiles.
template <int D>
__device__ __forceinline__ void issue_s(uint32_t d_col, uint32_t a_lo, uint32_t b_lo, uint32_t hi, uint32_t idesc) {
  static_for<0, D / 16>([&](auto c) {
    constexpr int kk = decltype(c)::value;
    constexpr uint32_t off = ((kk >> 2) * (BM * 128) + (kk & 3) * 32) >> 4;
    mma_ss_lo<off, off>(d_col, a_lo, b_lo, hi, idesc, kk > 0 ? 1u : 0u);
  });
}

// ACC += X (bf16 pairs in TMEM: half h's 64 reduction rows over columns
// a_col + 64 h + [0, 32)) * B (128 reduction rows x D, MN-major), both halves.
__device__ __forceinline__ void issue_acc(uint32_t d_col, uint32_t a_col, uint32_t b_lo, uint32_t hi,
                                          uint32_t idesc, bool first) {
  static_for<0, 8>([&](auto c) {
    constexpr int kk = decltype(c)::value;   // 16-row step of B
    constexpr int a_off = (kk >> 2) * 64 + (kk & 3) * 8;
    constexpr uint32_t b_off = (kk * 16 * 128) >> 4;
    mma_ts_lo<a_off, b_off>(d_col, a_col, b_lo, hi, idesc, (first && kk == 0) ? 0u : 1u);
  });
}

// The work of one CTA.
struct Work {
  int b, kvh, h;   // h: the query head (dQ kernel)
  int blk;         // the resident 128-row block (keys: j; queries: i)
  int first;       // first streamed block
  int per_head;    // streamed blocks per query head
  int n_steps;     // total streamed blocks (dK/dV kernel: G heads x per_head)
};

template <bool KV>
__device__ __forceinline__ Work decode_work(const Args& a, int item) {
  Work w;
  const int off = a.seqlen_k - a.seqlen_q;  // bottom-right causal alignment
  if constexpr (KV) {
    // Key block 0 first: under the causal mask it has the most query blocks.
    const int bh = item % (a.batch * a.hkv);
    w.blk = item / (a.batch * a.hkv);
    w.b = bh / a.hkv;
    w.kvh = bh - w.b * a.hkv;
    w.h = 0;
    // Query block i sees key block j when its last query (i BM + BM - 1) sits
    // at or after the block's first key: i BM + BM - 1 + off >= j BM.
    int first = 0;
    if (a.causal) {
      const int x = w.blk * BM - off - (BM - 1);
      first = x > 0 ? (x + BM - 1) / BM : 0;
    }
    w.first = first;
    w.per_head = a.n_qb > first ? a.n_qb - first : 0;
    w.n_steps = a.group * w.per_head;
  } else {
    // The last query block first: under the causal mask it sees the most keys.
    const int bh = item % (a.batch * a.hq);
    w.blk = a.n_qb - 1 - item / (a.batch * a.hq);
    w.b = bh / a.hq;
    w.h = bh - w.b * a.hq;
    w.kvh = w.h / a.group;
    int n = a.n_kb;
    if (a.causal) {
      const int last = w.blk * BM + BM - 1 + off;  // the block's last query sees keys 0..last
      const int nb = last >= 0 ? last / BM + 1 : 0;
      n = nb < n ? nb : n;
    }
    w.first = 0;
    w.per_head = n;
    w.n_steps = n;
  }
  return w;
}

// Stores this warpgroup's half of the columns of n_out accumulators of its
// rows (gradient rows past the sequence end are not written).
template <int D, bool KV>
__device__ __forceinline__ void store_grads(const Args& a, const Work& w, uint32_t lane_base, uint32_t col_acc,
                                            int half, int row_pos, bool has_acc) {
  const bool row_ok = row_pos < (KV ? a.seqlen_k : a.seqlen_q);
  const int n_out = KV ? 2 : 1;
  for (int o = 0; o < n_out; ++o) {
    // dK/dV kernel: o = 0 -> dV (unscaled), o = 1 -> dK (scale); dQ kernel: dQ (scale).
    const bool is_dv = KV && o == 0;
    void* base = KV ? (is_dv ? a.dv : a.dk) : a.dq;
    const long long row_off =
        KV ? (is_dv ? (long long)w.b * a.dv_bs + (long long)w.kvh * a.dv_hs + (long long)row_pos * a.dv_rs
                    : (long long)w.b * a.dk_bs + (long long)w.kvh * a.dk_hs + (long long)row_pos * a.dk_rs)
           : (long long)w.b * a.dq_bs + (long long)w.h * a.dq_hs + (long long)row_pos * a.dq_rs;
    const float mul = is_dv ? 1.f : a.scale;
#pragma unroll 1
    for (int cc = half * (D / 64); cc < (half + 1) * (D / 64); ++cc) {
      float x[32];
      if (has_acc) {
        uint32_t v[32];
        tmem_ld32(lane_base + col_acc + o * D + cc * 32, v);
        tmem_ld_wait();
#pragma unroll
        for (int k = 0; k < 32; ++k) x[k] = __uint_as_float(v[k]) * mul;
      } else {
#pragma unroll
        for (int k = 0; k < 32; ++k) x[k] = 0.f;  // no visible pair: the gradient is 0
      }
      if (row_ok && ATTN_IN_BOUNDS(w.b >= 0 && w.b < a.batch && (KV ? w.kvh < a.hkv : w.h < a.hq),
                                   ATTN_SITE_BWD_OUT, a.error_flags, a.planted))
        store_slice(base, row_off, cc * 32, x, a.grad_f32);
    }
  }
}

// ---------------------------------------------------------------------------
// dK / dV: persistent, one CTA per SM over the (batch, kv head, 128-key
// block j) items in a heaviest-first snake (as the dQ kernel). K_j and V_j
// stay in shared memory for the item while (Q_i, dO_i) of every query head of
// the group and every query block i that sees block j stream through; the
// ring, TMEM and barrier phases continue across items, so the next item's
// K_j / V_j load starts once the current item's last S^T and dP^T have read
// theirs and the finished item's dK / dV store overlaps the next item's first
// products. Per step t (one (head, i)):
//   S^T = K_j Q_i^T into buffer SB (X for even t, Y for odd), dP^T = V_j dO_i^T
//   into the other buffer DB;
//   phase 1 (elementwise, one key row per thread, each warpgroup 64 query
//   columns): P^T = 2^(S^T scale log2 e - LSE log2 e), written as bf16 over
//   the first 32 columns of its half of SB and kept in registers;
//   dV += P^T dO_i as soon as every warp has written P^T;
//   phase 2: dS^T = P^T (dP^T - D) over the last 32 columns of its half of SB;
//   then S^T of step t + 1 goes into DB (free: dP^T was read), dK += dS^T Q_i,
//   and dP^T of step t + 1 into SB (after dV and dK read it: MMAs from one
//   thread run in issue order).
// So the next step's S^T is computed while this step's dK accumulates, and
// phase 1 of the next step overlaps the tensor core's dK and dP^T.
template <int D>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const Args a, int n_items) {
  using L = KvLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
  uint64_t* a_full = bars;        // the item's K_j, V_j
  uint64_t* a_empty = bars + 1;   // the item's last S^T and dP^T have read them
  uint64_t* ring_full = bars + 2;
  uint64_t* ring_empty = bars + 4;
  uint64_t* s_full = bars + 6;    // S^T of the step is in TMEM
  uint64_t* dp_full = bars + 7;   // dP^T of the step is in TMEM
  uint64_t* p_full = bars + 8;    // every elementwise warp wrote P^T
  uint64_t* ds_full = bars + 9;   // every elementwise warp wrote dS^T
  uint64_t* acc_full = bars + 10; // the item's dK and dV are complete
  uint64_t* mma_done = bars + 11;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4);
  const int warp = warp_id();
  const int lane = lane_id();
  // The k-th item of this CTA (-1 past its last).
  auto cta_item = [&](int k) -> int {
    const int G = gridDim.x, c = blockIdx.x;
    const long long it = (long long)k * G + ((k & 1) ? (G - 1 - c) : c);
    return it < n_items ? (int)it : -1;
  };

  if (threadIdx.x == 0) {
    mbar_init(a_full, 1);
    mbar_init(a_empty, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&ring_full[s], 1);
      mbar_init(&ring_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(dp_full, 1);
    mbar_init(p_full, EW_WARPS);
    mbar_init(ds_full, EW_WARPS);
    mbar_init(acc_full, 1);
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
  // The dQ kernel, launched as a programmatic dependent, may now be scheduled:
  // its CTAs take the SMs this grid's CTAs leave when they finish.
  if (threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // Padded per-row vectors of query block i of head h of batch b.
  auto vec_row = [&](int b, int h, int i) { return (((long long)b * a.hq + h) * a.n_qb + i) * BM; };
  auto sb_col = [](int t) { return (uint32_t)((t & 1) * 128); };        // S^T, then P^T / dS^T, of item step t
  auto db_col = [](int t) { return (uint32_t)(128 - (t & 1) * 128); };  // dP^T of item step t

  if (warp == TMA_WARP) {
    if (lane == 0) {
      // ---------------------------------------------------------------- producer
      float* vec = reinterpret_cast<float*>(smem + L::VEC_OFF);
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      int g = 0, na = 0;  // ring steps and K/V loads issued so far (all items)
      bool ok = true;
      for (int kk = 0, item; ok && (item = cta_item(kk)) >= 0; ++kk) {
        const Work w = decode_work<true>(a, item);
        if (w.n_steps == 0) continue;
        if (na > 0 && !mbar_wait_bounded(a_empty, (na - 1) & 1, abort_flag, a.wait_limit)) break;
        mbar_arrive_expect_tx(a_full, 2 * L::TILE);
        for (int c = 0; c < L::CHUNKS; ++c) {
          tma_load_4d(smem + L::K_OFF + c * (BM * 128), &tm_k, a_full, c * 64, w.blk * BM, w.kvh, w.b);
          tma_load_4d(smem + L::V_OFF + c * (BM * 128), &tm_v, a_full, c * 64, w.blk * BM, w.kvh, w.b);
        }
        ++na;
        for (int t = 0; t < w.n_steps; ++t, ++g) {
          const int s = g & 1;
          if (g >= 2 && !mbar_wait_bounded(&ring_empty[s], ((g >> 1) - 1) & 1, abort_flag, a.wait_limit)) {
            ok = false;
            break;
          }
          const int h = w.kvh * a.group + t / w.per_head, blk = w.first + t % w.per_head;
          uint8_t* b0 = smem + L::RING_OFF + (2 * s) * L::TILE;
          uint8_t* b1 = b0 + L::TILE;
          // The stage's two tiles and its per-row vectors stay inside the ring
          // and the vector area.
          if (!ATTN_IN_BOUNDS(s >= 0 && s < 2 && L::RING_OFF + (2 * s + 2) * L::TILE <= L::VEC_OFF &&
                                  L::VEC_OFF + (2 * s + 2) * BM * 4 <= L::BAR_OFF,
                              ATTN_SITE_BWD_SMEM, a.error_flags, a.planted))
            continue;
          // The step's per-column LSE and D ride on the same barrier.
          mbar_arrive_expect_tx(&ring_full[s], 2 * L::TILE + 2 * BM * 4);
          const long long vr = vec_row(w.b, h, blk);
          if (!ATTN_IN_BOUNDS(h >= 0 && h < a.hq && blk >= 0 && blk < a.n_qb, ATTN_SITE_BWD_OUT, a.error_flags,
                              a.planted))
            continue;
          bulk_load(vec + (2 * s) * BM, a.lse2 + vr, BM * 4, &ring_full[s]);
          bulk_load(vec + (2 * s + 1) * BM, a.delta + vr, BM * 4, &ring_full[s]);
          for (int c = 0; c < L::CHUNKS; ++c) {
            tma_load_4d(b0 + c * (BM * 128), &tm_q, &ring_full[s], c * 64, blk * BM, h, w.b);
            tma_load_4d(b1 + c * (BM * 128), &tm_do, &ring_full[s], c * 64, blk * BM, h, w.b);
          }
        }
      }
      // Drain: no copy may be in flight when the CTA exits: the last K/V load
      // and the last two ring steps (earlier copies completed before their
      // slot was released); on the abort path they still land by themselves,
      // so these waits ignore the abort flag.
      if (na > 0) mbar_wait_drain(a_full, (na - 1) & 1);
      for (int u = g - 2 > 0 ? g - 2 : 0; u < g; ++u) mbar_wait_drain(&ring_full[u & 1], (u >> 1) & 1);
    }
  } else if (warp == MMA_WARP) {
    if (lane == 0) {
      // ---------------------------------------------------------------- MMA issuer
      constexpr uint32_t ID_S = instr_desc_bf16(BM, BM, 0);   // both operands K-major, N = 128
      constexpr uint32_t ID_ACC = instr_desc_bf16(BM, D, 1);  // B MN-major
      const uint32_t hi = sw128_desc_hi(1024);
      const uint32_t k_lo = sw128_desc_lo(smem_addr(smem + L::K_OFF), 16);
      const uint32_t v_lo = sw128_desc_lo(smem_addr(smem + L::V_OFF), 16);
      const uint32_t ring_k = sw128_desc_lo(smem_addr(smem + L::RING_OFF), 16);        // K-major
      const uint32_t ring_mn = sw128_desc_lo(smem_addr(smem + L::RING_OFF), BM * 128);  // MN-major
      const uint32_t id_s = ID_S, id_acc = ID_ACC;
      const uint32_t tDV = tmem_base + COL_ACC_KV, tDK = tDV + D;
      int gt = 0, na = 0;  // steps and items with work so far (all phases)
      bool ok = true;
      for (int kk = 0, item; ok && (item = cta_item(kk)) >= 0; ++kk) {
        const Work w = decode_work<true>(a, item);
        const int n = w.n_steps;
        if (n == 0) continue;
        // Ring stage addresses of item step t's streamed tiles: which = 0 (Q) or 1 (dO).
        auto b_k = [&](int t, int which) {
          return ring_k + (uint32_t)(((2 * ((gt + t) & 1) + which) * L::TILE) >> 4);
        };
        auto b_m = [&](int t, int which) {
          return ring_mn + (uint32_t)(((2 * ((gt + t) & 1) + which) * L::TILE) >> 4);
        };
        auto wait_ring = [&](int t) {
          const int g = gt + t;
          return mbar_wait_bounded(&ring_full[g & 1], (g >> 1) & 1, abort_flag, a.wait_limit);
        };
        auto issue_st = [&](int t) {  // S^T = K Q^T
          issue_s<D>(tmem_base + sb_col(t), k_lo, b_k(t, 0), hi, id_s);
          mma_commit(s_full);
        };
        auto issue_dpt = [&](int t) {  // dP^T = V dO^T
          issue_s<D>(tmem_base + db_col(t), v_lo, b_k(t, 1), hi, id_s);
          mma_commit(dp_full);
          if (t == n - 1) mma_commit(a_empty);  // the item's last S^T and dP^T: K_j, V_j are free
        };
        ok = mbar_wait_bounded(a_full, na & 1, abort_flag, a.wait_limit);
        if (ok) ok = wait_ring(0);
        if (ok) {
          tc_fence_after();
          issue_st(0);
          issue_dpt(0);
        }
        for (int t = 0; t < n && ok; ++t) {
          const bool next = t + 1 < n;
          ok = mbar_wait_bounded(p_full, (gt + t) & 1, abort_flag, a.wait_limit);
          if (!ok) break;
          tc_fence_after();
          issue_acc(tDV, tmem_base + sb_col(t), b_m(t, 1), hi, id_acc, t == 0);  // dV += P^T dO
          ok = mbar_wait_bounded(ds_full, (gt + t) & 1, abort_flag, a.wait_limit);
          if (!ok) break;
          tc_fence_after();
          if (next) {
            ok = wait_ring(t + 1);
            if (!ok) break;
            tc_fence_after();
            issue_st(t + 1);  // into DB(t): its dP^T was read by phase 2
          }
          issue_acc(tDK, tmem_base + sb_col(t) + 32, b_m(t, 0), hi, id_acc, t == 0);  // dK += dS^T Q
          mma_commit(&ring_empty[(gt + t) & 1]);  // step t's tiles and vectors are free once these have run
          if (next) issue_dpt(t + 1);              // into SB(t), after dV and dK read it
        }
        if (!ok) break;
        mma_commit(acc_full);
        gt += n;
        ++na;
      }
      // Every MMA issued must have completed before tensor memory is released
      // (on the abort path too: they finish by themselves).
      mma_commit(mma_done);
      mbar_wait_drain(mma_done, 0);
    }
  } else {
    // ------------------------------------------------------------------ elementwise + epilogue
    const int wq = warp & 3;
    const int half = warp >> 2;      // this warpgroup's 64 query columns
    const int r = wq * 32 + lane;    // key row == TMEM lane
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(wq * 32) << 16);
    const int off = a.seqlen_k - a.seqlen_q;
    const float sl2 = a.scale_log2;
    const float* vec = reinterpret_cast<const float*>(smem + L::VEC_OFF);
    const float2 sl2x2 = make_float2(sl2, sl2);
    const bool cols_ok = ATTN_IN_BOUNDS(half >= 0 && half < 2 && COL_ACC_KV + 2 * D <= TMEM_COLS,
                                        ATTN_SITE_BWD_TMEM, a.error_flags, a.planted);
    (void)cols_ok;
    int gt = 0, na = 0;  // steps and items with work so far (all phases)
    bool ok = true;
    for (int kk = 0, item; ok && (item = cta_item(kk)) >= 0; ++kk) {
      const Work w = decode_work<true>(a, item);
      const int n = w.n_steps;
      const int row_pos = w.blk * BM + r;  // key position
      for (int t = 0; t < n && ok; ++t) {
        const int g = gt + t;
        const int s = g & 1;
        const int blk = w.first + t % w.per_head;
        // Query column c (query blk BM + c, at position blk BM + c + off) sees
        // this key when c >= c_lim.
        const int c_lim = row_pos < a.seqlen_k ? (a.causal ? row_pos - off - blk * BM : -BM) : BM;
        // The producer's LSE / D copies complete on the stage's full barrier.
        ok = warp_wait(&ring_full[s], (g >> 1) & 1, abort_flag, a.wait_limit);
        if (!ok) break;
        const uint32_t lse_a = smem_addr(vec + (2 * s) * BM) + (uint32_t)(half * 64 * 4);
        const uint32_t delta_a = smem_addr(vec + (2 * s + 1) * BM) + (uint32_t)(half * 64 * 4);
        const uint32_t tS = lane_base + sb_col(t) + half * 64, tD = lane_base + db_col(t) + half * 64;
        // The whole half is visible on all but the diagonal and ragged tiles.
        const bool all_vis = c_lim <= half * 64;
        // ---- phase 1: P^T
        ok = warp_wait(s_full, g & 1, abort_flag, a.wait_limit);
        if (!ok) break;
        tc_fence_after();
        float p[64];
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          uint32_t sv[32];
          if (cols_ok) tmem_ld32(tS + cc * 32, sv);
          tmem_ld_wait();
          uint32_t pk[16];
#pragma unroll
          for (int gg = 0; gg < 2; ++gg) {  // 16 columns at a time: their -LSE log2 e loaded first
            float4 lv[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) lv[q] = lds_f4(lse_a + (uint32_t)(cc * 32 + gg * 16 + 4 * q) * 4u);
#pragma unroll
            for (int j = 0; j < 16; j += 2) {
              const int jj = gg * 16 + j;
              const float4 l4 = lv[j >> 2];
              const float2 nl = (j & 2) ? make_float2(l4.z, l4.w) : make_float2(l4.x, l4.y);
              const float2 x = __ffma2_rn(make_float2(__uint_as_float(sv[jj]), __uint_as_float(sv[jj + 1])), sl2x2, nl);
              float2 pp = make_float2(ex2_approx(x.x), ex2_approx(x.y));
              if (!all_vis) {
                const int c = half * 64 + cc * 32 + jj;
                pp.x = c >= c_lim ? pp.x : 0.f;
                pp.y = c + 1 >= c_lim ? pp.y : 0.f;
              }
              p[cc * 32 + jj] = pp.x;
              p[cc * 32 + jj + 1] = pp.y;
              pk[jj / 2] = pack_bf16x2(pp.x, pp.y);
            }
          }
          // bf16 pairs over the first 32 columns of this half, read already.
          if (cols_ok) tmem_st16(tS + cc * 16, pk);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full);
        // ---- phase 2: dS^T
        ok = warp_wait(dp_full, g & 1, abort_flag, a.wait_limit);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          uint32_t dv[32];
          if (cols_ok) tmem_ld32(tD + cc * 32, dv);
          tmem_ld_wait();
          uint32_t dk[16];
#pragma unroll
          for (int gg = 0; gg < 2; ++gg) {
            float4 nd4[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) nd4[q] = lds_f4(delta_a + (uint32_t)(cc * 32 + gg * 16 + 4 * q) * 4u);
#pragma unroll
            for (int j = 0; j < 16; j += 2) {
              const int jj = gg * 16 + j;
              const float4 d4 = nd4[j >> 2];
              const float2 nd = (j & 2) ? make_float2(d4.z, d4.w) : make_float2(d4.x, d4.y);
              const float2 ds = __fmul2_rn(make_float2(p[cc * 32 + jj], p[cc * 32 + jj + 1]),
                                           __fadd2_rn(make_float2(__uint_as_float(dv[jj]), __uint_as_float(dv[jj + 1])), nd));
              dk[jj / 2] = pack_bf16x2(ds.x, ds.y);
            }
          }
          // bf16 pairs over the last 32 columns of this half of SB (its S^T was
          // read in phase 1).
          if (cols_ok) tmem_st16(tS + 32 + cc * 16, dk);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(ds_full);
      }
      if (!ok) break;
      // ---- epilogue: each warpgroup stores half of the columns of its rows
      if (n > 0) {
        ok = warp_wait(acc_full, na & 1, abort_flag, a.wait_limit);
        if (!ok) break;
        tc_fence_after();
      }
      // The next item's first dV / dK products overwrite the accumulators
      // after this warp's next p_full / ds_full arrivals, which follow these
      // loads.
      store_grads<D, true>(a, w, lane_base, COL_ACC_KV, half, row_pos, n > 0 && cols_ok);
      gt += n;
      na += n > 0 ? 1 : 0;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag && a.error_flags) atomicOr(a.error_flags, ATTN_FAULT_TIMEOUT);
  if (warp == MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// dQ: persistent, one CTA per SM; CTA c takes the items (batch, query head,
// 128-query block i) c, 2G-1-c, 2G+c, ... of the heaviest-first numbering
// (G CTAs), so heavy and light causal blocks pair up on every CTA. Q_i and
// dO_i stay in shared memory for the item while K_j, V_j stream; the rings,
// the TMEM allocation and the barrier phases continue across items, so an
// item's first K/V blocks are already under way while the previous item ends,
// and its Q_i / dO_i load starts as soon as the previous item's last S and dP
// have read theirs. Per step t (key block j = t):
//   S_t = Q_i K_j^T (product 2t) and dP_t = dO_i V_j^T (product 2t + 1), product
//   p into TMEM buffer p mod 3; the elementwise warps (one query row per
//   thread, each warpgroup 64 key columns) write dS_t = P_t (dP_t - D) as
//   bf16 over the dP buffer; dQ += dS_t K_j.
// Issue order after step t's elementwise work: dP_{t+1} (into S_t's buffer,
// read already), dQ += dS_t K_j, S_{t+2} (into dP_t's buffer, after the
// accumulation read it). S is two steps ahead and dP one, so the tensor core
// runs dQ and S while the elementwise warps work on the next step. The next
// item's first dQ product overwrites the accumulator only after the
// elementwise warps (which also store it) have finished the previous item.
template <int D>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do, const Args a,
                  int n_items) {
  using L = QLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
  uint64_t* a_full = bars;                      // the item's Q_i, dO_i
  uint64_t* a_empty = bars + 1;                 // the item's last S and dP have read them
  uint64_t* k_full = bars + 2;                  // [K_SLOTS]
  uint64_t* k_empty = k_full + L::K_SLOTS;      // [K_SLOTS]
  uint64_t* v_full = k_empty + L::K_SLOTS;      // [V_SLOTS]
  uint64_t* v_empty = v_full + L::V_SLOTS;      // [V_SLOTS]
  uint64_t* sdp_full = v_empty + L::V_SLOTS;    // S and dP of the step are in TMEM
  uint64_t* ps_full = sdp_full + 1;             // every elementwise warp wrote dS
  uint64_t* acc_full = ps_full + 1;             // the item's dQ is complete
  uint64_t* mma_done = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4);
  const int warp = warp_id();
  const int lane = lane_id();
  // The k-th item of this CTA (-1 past its last).
  auto cta_item = [&](int k) -> int {
    const int G = gridDim.x, c = blockIdx.x;
    const long long it = (long long)k * G + ((k & 1) ? (G - 1 - c) : c);
    return it < n_items ? (int)it : -1;
  };

  if (threadIdx.x == 0) {
    mbar_init(a_full, 1);
    mbar_init(a_empty, 1);
    for (int s = 0; s < L::K_SLOTS; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < L::V_SLOTS; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    mbar_init(sdp_full, 1);
    mbar_init(ps_full, EW_WARPS);
    mbar_init(acc_full, 1);
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
  auto buf_col = [](int p) { return (uint32_t)((p % 3) * 128); };  // TMEM buffer of product p of an item

  if (warp == TMA_WARP) {
    if (lane == 0) {
      // ---------------------------------------------------------------- producer
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      // K_u then V_u for every item's blocks u = 0, 1, ... in ring order;
      // each load waits for the block a whole ring back to be released, and
      // an item's Q_i, dO_i wait for the previous item's last S and dP.
      int nk = 0, nv = 0, na = 0;  // K, V and Q/dO loads issued so far (all items)
      bool ok = true;
      for (int kk = 0, item; ok && (item = cta_item(kk)) >= 0; ++kk) {
        const Work w = decode_work<false>(a, item);
        if (w.n_steps == 0) continue;
        if (na > 0 && !mbar_wait_bounded(a_empty, (na - 1) & 1, abort_flag, a.wait_limit)) break;
        mbar_arrive_expect_tx(a_full, 2 * L::TILE);
        for (int c = 0; c < L::CHUNKS; ++c) {
          tma_load_4d(smem + L::Q_OFF + c * (BM * 128), &tm_q, a_full, c * 64, w.blk * BM, w.h, w.b);
          tma_load_4d(smem + L::DO_OFF + c * (BM * 128), &tm_do, a_full, c * 64, w.blk * BM, w.h, w.b);
        }
        ++na;
        for (int u = 0; u < w.n_steps; ++u) {
          const int ks = nk % L::K_SLOTS, vs = nv % L::V_SLOTS;
          if (nk >= L::K_SLOTS &&
              !mbar_wait_bounded(&k_empty[ks], ((nk / L::K_SLOTS) - 1) & 1, abort_flag, a.wait_limit)) {
            ok = false;
            break;
          }
          if (ATTN_IN_BOUNDS(ks >= 0 && ks < L::K_SLOTS && L::K_OFF + (ks + 1) * L::TILE <= L::V_OFF,
                             ATTN_SITE_BWD_SMEM, a.error_flags, a.planted)) {
            mbar_arrive_expect_tx(&k_full[ks], L::TILE);
            for (int c = 0; c < L::CHUNKS; ++c)
              tma_load_4d(smem + L::K_OFF + ks * L::TILE + c * (BM * 128), &tm_k, &k_full[ks], c * 64, u * BM,
                          w.kvh, w.b);
          }
          ++nk;
          if (nv >= L::V_SLOTS &&
              !mbar_wait_bounded(&v_empty[vs], ((nv / L::V_SLOTS) - 1) & 1, abort_flag, a.wait_limit)) {
            ok = false;
            break;
          }
          if (ATTN_IN_BOUNDS(vs >= 0 && vs < L::V_SLOTS && L::V_OFF + (vs + 1) * L::TILE <= L::BAR_OFF,
                             ATTN_SITE_BWD_SMEM, a.error_flags, a.planted)) {
            mbar_arrive_expect_tx(&v_full[vs], L::TILE);
            for (int c = 0; c < L::CHUNKS; ++c)
              tma_load_4d(smem + L::V_OFF + vs * L::TILE + c * (BM * 128), &tm_v, &v_full[vs], c * 64, u * BM,
                          w.kvh, w.b);
          }
          ++nv;
        }
      }
      // Drain: the last copy into each slot and of Q/dO (earlier ones
      // completed before their slot was released); the waits ignore the
      // abort flag.
      if (na > 0) mbar_wait_drain(a_full, (na - 1) & 1);
      for (int u = nk - L::K_SLOTS > 0 ? nk - L::K_SLOTS : 0; u < nk; ++u)
        mbar_wait_drain(&k_full[u % L::K_SLOTS], (u / L::K_SLOTS) & 1);
      for (int u = nv - L::V_SLOTS > 0 ? nv - L::V_SLOTS : 0; u < nv; ++u)
        mbar_wait_drain(&v_full[u % L::V_SLOTS], (u / L::V_SLOTS) & 1);
    }
  } else if (warp == MMA_WARP) {
    if (lane == 0) {
      // ---------------------------------------------------------------- MMA issuer
      constexpr uint32_t ID_S = instr_desc_bf16(BM, BM, 0);
      constexpr uint32_t ID_ACC = instr_desc_bf16(BM, D, 1);
      const uint32_t hi = sw128_desc_hi(1024);
      const uint32_t q_lo = sw128_desc_lo(smem_addr(smem + L::Q_OFF), 16);
      const uint32_t do_lo = sw128_desc_lo(smem_addr(smem + L::DO_OFF), 16);
      const uint32_t k_k = sw128_desc_lo(smem_addr(smem + L::K_OFF), 16);          // K-major
      const uint32_t k_mn = sw128_desc_lo(smem_addr(smem + L::K_OFF), BM * 128);   // MN-major
      const uint32_t v_k = sw128_desc_lo(smem_addr(smem + L::V_OFF), 16);
      const uint32_t id_s = ID_S, id_acc = ID_ACC;
      const uint32_t tDQ = tmem_base + COL_ACC_Q;
      int kb = 0;  // K / V blocks of the CTA's earlier items (ring positions)
      int gt = 0;  // steps of the CTA's earlier items (sdp / ps phases)
      int na = 0;  // items with work so far (a_full / acc_full phases)
      bool ok = true;
      for (int kk = 0, item; ok && (item = cta_item(kk)) >= 0; ++kk) {
        const Work w = decode_work<false>(a, item);
        const int n = w.n_steps;
        if (n == 0) continue;
        // Ring position u of this item's block u is kb + u.
        auto kslot = [&](int u) { return (uint32_t)((((kb + u) % L::K_SLOTS) * L::TILE) >> 4); };
        auto vslot = [&](int u) { return (uint32_t)((((kb + u) % L::V_SLOTS) * L::TILE) >> 4); };
        auto wait_k = [&](int u) {
          const int g = kb + u;
          return mbar_wait_bounded(&k_full[g % L::K_SLOTS], (g / L::K_SLOTS) & 1, abort_flag, a.wait_limit);
        };
        auto wait_v = [&](int u) {
          const int g = kb + u;
          return mbar_wait_bounded(&v_full[g % L::V_SLOTS], (g / L::V_SLOTS) & 1, abort_flag, a.wait_limit);
        };
        auto issue_sq = [&](int u) { issue_s<D>(tmem_base + buf_col(2 * u), q_lo, k_k + kslot(u), hi, id_s); };
        auto issue_dp = [&](int u) {  // then the step's S and dP are complete once this has run
          issue_s<D>(tmem_base + buf_col(2 * u + 1), do_lo, v_k + vslot(u), hi, id_s);
          mma_commit(sdp_full);
          mma_commit(&v_empty[(kb + u) % L::V_SLOTS]);
          if (u == n - 1) mma_commit(a_empty);  // the item's last S and dP: Q_i, dO_i are free
        };
        ok = mbar_wait_bounded(a_full, na & 1, abort_flag, a.wait_limit);
        if (ok) ok = wait_k(0);
        if (ok) {
          tc_fence_after();
          issue_sq(0);
          ok = wait_v(0);
        }
        if (ok) {
          tc_fence_after();
          issue_dp(0);
          if (n > 1) {
            ok = wait_k(1);
            if (ok) {
              tc_fence_after();
              issue_sq(1);
            }
          }
        }
        for (int t = 0; t < n && ok; ++t) {
          ok = mbar_wait_bounded(ps_full, (gt + t) & 1, abort_flag, a.wait_limit);
          if (!ok) break;
          tc_fence_after();
          if (t + 1 < n) {
            ok = wait_v(t + 1);
            if (!ok) break;
            tc_fence_after();
            issue_dp(t + 1);  // into S_t's buffer, read by step t's elementwise work
          }
          issue_acc(tDQ, tmem_base + buf_col(2 * t + 1), k_mn + kslot(t), hi, id_acc, t == 0);  // dQ += dS K
          mma_commit(&k_empty[(kb + t) % L::K_SLOTS]);  // K_t's last reader
          if (t + 2 < n) {
            ok = wait_k(t + 2);
            if (!ok) break;
            tc_fence_after();
            issue_sq(t + 2);  // into dP_t's buffer, after the accumulation read dS_t
          }
        }
        if (!ok) break;
        mma_commit(acc_full);
        kb += n;
        gt += n;
        ++na;
      }
      mma_commit(mma_done);
      mbar_wait_drain(mma_done, 0);
    }
  } else {
    // ------------------------------------------------------------------ elementwise + epilogue
    const int wq = warp & 3;
    const int half = warp >> 2;      // this warpgroup's 64 key columns
    const int r = wq * 32 + lane;    // query row == TMEM lane
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(wq * 32) << 16);
    const int off = a.seqlen_k - a.seqlen_q;
    const float sl2 = a.scale_log2;
    const float2 sl2x2 = make_float2(sl2, sl2);
    const bool cols_ok = ATTN_IN_BOUNDS(half >= 0 && half < 2 && COL_ACC_Q + D <= TMEM_COLS, ATTN_SITE_BWD_TMEM,
                                        a.error_flags, a.planted);
    (void)cols_ok;
    int gt = 0;  // steps of earlier items (sdp / ps phases)
    int na = 0;  // items with work so far (acc_full phases)
    bool ok = true;
    for (int kk = 0, item; ok && (item = cta_item(kk)) >= 0; ++kk) {
      const Work w = decode_work<false>(a, item);
      const int n = w.n_steps;
      const int row_pos = w.blk * BM + r;  // query position
      float nlse_r = -INFINITY, ndelta_r = 0.f;
      {
        const long long vr = (((long long)w.b * a.hq + w.h) * a.n_qb + w.blk) * BM + r;  // padded: -inf / 0 past Sq
        if (ATTN_IN_BOUNDS(w.h >= 0 && w.h < a.hq && w.blk >= 0 && w.blk < a.n_qb && r >= 0 && r < BM,
                           ATTN_SITE_BWD_OUT, a.error_flags, a.planted)) {
          nlse_r = a.lse2[vr];
          ndelta_r = a.delta[vr];
        }
      }
      const float2 nl = make_float2(nlse_r, nlse_r), nd = make_float2(ndelta_r, ndelta_r);
      for (int t = 0; t < n && ok; ++t) {
        // Key column c (key t BM + c) is visible when c < c_lim: below Sk and,
        // causal, at most row_pos + off.
        int c_lim = a.seqlen_k - t * BM;
        if (a.causal) {
          const int cl = row_pos + off - t * BM + 1;
          c_lim = cl < c_lim ? cl : c_lim;
        }
        const bool all_vis = c_lim >= half * 64 + 64;
        const uint32_t tS = lane_base + buf_col(2 * t) + half * 64, tD = lane_base + buf_col(2 * t + 1) + half * 64;
        ok = warp_wait(sdp_full, (gt + t) & 1, abort_flag, a.wait_limit);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          uint32_t sv[32], dv[32];
          if (cols_ok) {
            tmem_ld32(tS + cc * 32, sv);
            tmem_ld32(tD + cc * 32, dv);
          }
          tmem_ld_wait();
          uint32_t dk[16];
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            // P = 2^(S scale log2 e - LSE log2 e); dS = P (dP - D).
            const float2 x = __ffma2_rn(make_float2(__uint_as_float(sv[j]), __uint_as_float(sv[j + 1])), sl2x2, nl);
            float2 pp = make_float2(ex2_approx(x.x), ex2_approx(x.y));
            if (!all_vis) {
              const int c = half * 64 + cc * 32 + j;
              pp.x = c < c_lim ? pp.x : 0.f;
              pp.y = c + 1 < c_lim ? pp.y : 0.f;
            }
            const float2 ds =
                __fmul2_rn(pp, __fadd2_rn(make_float2(__uint_as_float(dv[j]), __uint_as_float(dv[j + 1])), nd));
            dk[j / 2] = pack_bf16x2(ds.x, ds.y);
          }
          // bf16 pairs over this half's first 32 columns of the dP buffer, read already.
          if (cols_ok) tmem_st16(tD + cc * 16, dk);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(ps_full);
      }
      if (!ok) break;
      if (n > 0) {
        ok = warp_wait(acc_full, na & 1, abort_flag, a.wait_limit);
        if (!ok) break;
        tc_fence_after();
      }
      // The next item's first dQ product overwrites the accumulator after
      // this warp's next ps_full arrival, which follows these loads.
      store_grads<D, false>(a, w, lane_base, COL_ACC_Q, half, row_pos, n > 0 && cols_ok);
      gt += n;
      na += n > 0 ? 1 : 0;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag && a.error_flags) atomicOr(a.error_flags, ATTN_FAULT_TIMEOUT);
  if (warp == MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
  // This grid may have started before the dK/dV grid ended; it ends only
  // after that grid, so that work after the call on the stream follows both.
  if (threadIdx.x == 0) asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Per query row, padded to whole 128-row blocks: -D = -rowsum(dO * O) and
// -LSE * log2(e) (-inf for rows that see no key and for padding rows, whose D
// is 0). One CTA per (batch, head, 128-row block); D / 8 threads share a row,
// each with 16-byte loads of 8 elements, and every thread issues the loads of
// UNR rows (and their LSE) before it reduces any of them, so that enough bytes
// are in flight to keep HBM busy.
template <int D, bool OF32>
__global__ void __launch_bounds__(256)
    bwd_prep_kernel(const void* o, long long o_bs, long long o_hs, long long o_rs, const __nv_bfloat16* dout,
                    long long do_bs, long long do_hs, long long do_rs, const float* lse, int hq, int seqlen_q,
                    int n_qb, float* lse2, float* delta) {
  constexpr int TPR = D / 8;         // threads per row: 16 (head_dim 128) or 8 (64)
  constexpr int RPP = 256 / TPR;     // rows per pass: 16 or 32
  constexpr int PASSES = BM / RPP;   // 8 or 4
  constexpr int UNR = 4;
  static_assert(PASSES % UNR == 0, "whole unrolled groups");
  const int qb = (int)(blockIdx.x % (unsigned)n_qb);
  const int bh = (int)(blockIdx.x / (unsigned)n_qb);
  const int h = bh % hq, b = bh / hq;
  const int sub = threadIdx.x % TPR, r0 = threadIdx.x / TPR;
  // Padded row (bh n_qb + qb) BM + r == blockIdx.x BM + r.
  float* lse2_blk = lse2 + (long long)blockIdx.x * BM;
  float* delta_blk = delta + (long long)blockIdx.x * BM;
  const __nv_bfloat16* drow = dout + b * do_bs + h * do_hs + sub * 8;
  const float* lrow = lse + (long long)bh * seqlen_q;
#pragma unroll
  for (int p0 = 0; p0 < PASSES; p0 += UNR) {
    uint4 dv[UNR], ov[UNR], ov2[UNR];
    float lv[UNR];
#pragma unroll
    for (int u = 0; u < UNR; ++u) {
      const int q = qb * BM + (p0 + u) * RPP + r0;
      dv[u] = ov[u] = ov2[u] = make_uint4(0u, 0u, 0u, 0u);
      lv[u] = 0.f;
      if (q < seqlen_q) {
        dv[u] = __ldg(reinterpret_cast<const uint4*>(drow + q * do_rs));
        if constexpr (OF32) {
          const float* orow = reinterpret_cast<const float*>(o) + b * o_bs + h * o_hs + q * o_rs + sub * 8;
          ov[u] = __ldcs(reinterpret_cast<const uint4*>(orow));
          ov2[u] = __ldcs(reinterpret_cast<const uint4*>(orow + 4));
        } else {
          const __nv_bfloat16* orow =
              reinterpret_cast<const __nv_bfloat16*>(o) + b * o_bs + h * o_hs + q * o_rs + sub * 8;
          ov[u] = __ldcs(reinterpret_cast<const uint4*>(orow));
        }
        if (sub == 0) lv[u] = __ldg(lrow + q);
      }
    }
#pragma unroll
    for (int u = 0; u < UNR; ++u) {
      const uint32_t dw[4] = {dv[u].x, dv[u].y, dv[u].z, dv[u].w};
      float of[8];
      if constexpr (OF32) {
        of[0] = __uint_as_float(ov[u].x), of[1] = __uint_as_float(ov[u].y);
        of[2] = __uint_as_float(ov[u].z), of[3] = __uint_as_float(ov[u].w);
        of[4] = __uint_as_float(ov2[u].x), of[5] = __uint_as_float(ov2[u].y);
        of[6] = __uint_as_float(ov2[u].z), of[7] = __uint_as_float(ov2[u].w);
      } else {
        const uint32_t ow[4] = {ov[u].x, ov[u].y, ov[u].z, ov[u].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ow[e]));
          of[2 * e] = f.x, of[2 * e + 1] = f.y;
        }
      }
      float acc = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&dw[e]));
        acc = fmaf(f.x, of[2 * e], acc);
        acc = fmaf(f.y, of[2 * e + 1], acc);
      }
#pragma unroll
      for (int sh = TPR / 2; sh >= 1; sh >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, sh);
      const int r = (p0 + u) * RPP + r0;
      if (sub == 0) {
        const bool live = qb * BM + r < seqlen_q;
        const float l = lv[u];
        lse2_blk[r] = live && l != -INFINITY ? -l * LOG2E : -INFINITY;
        delta_blk[r] = live ? -acc : 0.f;
      }
    }
  }
}

}  // namespace bwd

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
typedef CUresult (*BwdEncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static BwdEncodeFn bwd_encode_fn() {
  static const BwdEncodeFn fn = []() -> BwdEncodeFn {  // process-wide; initialised once, thread-safely
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<BwdEncodeFn>(ptr);
    cudaGetLastError();
    return nullptr;
  }();
  return fn;
}

// bf16 [d3][d2][d1][d0 = head_dim] with element strides s1..s3; box of 64
// columns x 128 rows, 128-byte swizzle, zero fill out of bounds.
static bool bwd_map(CUtensorMap* map, const void* base, int D, int rows, int heads, int batch, int64_t rs, int64_t hs,
                    int64_t bs) {
  BwdEncodeFn fn = bwd_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)rows, (cuuint64_t)heads, (cuuint64_t)batch};
  cuuint64_t strides[3] = {(cuuint64_t)rs * 2, (cuuint64_t)hs * 2, (cuuint64_t)bs * 2};
  cuuint32_t box[4] = {64u, (cuuint32_t)bwd::BM, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Two fp32 values per query row, rows padded to whole 128-row blocks.
static size_t padded_rows(const attn_backward_params& p) {
  return (size_t)p.batch * p.num_q_heads * ((p.seqlen_q + bwd::BM - 1) / bwd::BM) * bwd::BM;
}

size_t backward_workspace_bytes(const attn_backward_params& p) {
  const size_t n = padded_rows(p) * sizeof(float);
  return 2 * ((n + 255) / 256 * 256);
}

template <int D, bool KV>
static attn_status_t launch_bwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                const CUtensorMap& tdo, const bwd::Args& a, long long grid, bool dependent,
                                cudaStream_t stream) {
  constexpr int SMEM = KV ? bwd::KvLayout<D>::SMEM_BYTES : bwd::QLayout<D>::SMEM_BYTES;
  static_assert(SMEM <= 232448, "shared memory budget");
  auto kern = [] {
    if constexpr (KV) return bwd::bwd_dkdv_kernel<D>;
    else return bwd::bwd_dq_kernel<D>;
  }();
  static DeviceOnce setup;  // the shared-memory attribute, once per device
  const attn_status_t st = setup.run([&]() -> attn_status_t {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM) != cudaSuccess) {
      cudaGetLastError();
      return ATTN_ERR_CUDA;
    }
    return ATTN_OK;
  });
  if (st != ATTN_OK) return st;
  if (grid <= 0) return ATTN_OK;
  if (grid > 0x7fffffffLL) return ATTN_ERR_INVALID_ARG;
  // Persistent: at most one CTA per SM over all items (grid = the item count).
  const long long ctas = grid < device_sm_count() ? grid : device_sm_count();
  if (!dependent) {
    kern<<<(unsigned)ctas, bwd::NUM_THREADS, SMEM, stream>>>(tq, tk, tv, tdo, a, (int)grid);
  } else {
    // The dQ kernel reads nothing the dK/dV kernel writes: as a programmatic
    // dependent of the dK/dV launch right before it, its CTAs start on the
    // SMs the dK/dV kernel's last items leave idle instead of after the grid.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)ctas);
    cfg.blockDim = dim3(bwd::NUM_THREADS);
    cfg.dynamicSmemBytes = SMEM;
    cfg.stream = stream;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, tq, tk, tv, tdo, a, (int)grid) != cudaSuccess) return ATTN_ERR_CUDA;
  }
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

attn_status_t launch_backward(const attn_backward_params& p, void* workspace, cudaStream_t stream) {
  if (p.batch == 0 || p.num_q_heads == 0 || (p.seqlen_q == 0 && p.seqlen_k == 0)) return ATTN_OK;
  const int D = p.head_dim;
  const size_t n = padded_rows(p);
  const int n_qb = (p.seqlen_q + bwd::BM - 1) / bwd::BM;
  float* lse2 = reinterpret_cast<float*>(workspace);
  float* delta = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(workspace) + (n * 4 + 255) / 256 * 256);
  const bool o_f32 = p.o_dtype == ATTN_DTYPE_F32;
  if (n > 0) {
    // One CTA per (batch, head, 128-row block): n / 128 of them.
    const long long blocks = (long long)(n / bwd::BM);
    if (blocks > 0x7fffffffLL) return ATTN_ERR_INVALID_ARG;
    auto prep = [&](auto kern) {
      kern<<<(unsigned)blocks, 256, 0, stream>>>(p.o, p.o_batch_stride, p.o_head_stride, p.o_row_stride,
                                                  reinterpret_cast<const __nv_bfloat16*>(p.dout), p.do_batch_stride,
                                                  p.do_head_stride, p.do_row_stride, p.lse, p.num_q_heads,
                                                  p.seqlen_q, n_qb, lse2, delta);
    };
    if (D == 128)
      o_f32 ? prep(bwd::bwd_prep_kernel<128, true>) : prep(bwd::bwd_prep_kernel<128, false>);
    else
      o_f32 ? prep(bwd::bwd_prep_kernel<64, true>) : prep(bwd::bwd_prep_kernel<64, false>);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  }
  // Tensor maps need at least one row; an empty side is never loaded.
  const int sq_map = p.seqlen_q > 0 ? p.seqlen_q : 1, sk_map = p.seqlen_k > 0 ? p.seqlen_k : 1;
  CUtensorMap tq, tk, tv, tdo;
  if (!bwd_map(&tq, p.q, D, sq_map, p.num_q_heads, p.batch, p.q_row_stride, p.q_head_stride, p.q_batch_stride) ||
      !bwd_map(&tdo, p.dout, D, sq_map, p.num_q_heads, p.batch, p.do_row_stride, p.do_head_stride,
               p.do_batch_stride) ||
      !bwd_map(&tk, p.k, D, sk_map, p.num_kv_heads, p.batch, p.k_row_stride, p.k_head_stride, p.k_batch_stride) ||
      !bwd_map(&tv, p.v, D, sk_map, p.num_kv_heads, p.batch, p.v_row_stride, p.v_head_stride, p.v_batch_stride))
    return ATTN_ERR_CUDA;
  bwd::Args a;
  memset(&a, 0, sizeof(a));
  a.batch = p.batch;
  a.hq = p.num_q_heads;
  a.hkv = p.num_kv_heads;
  a.group = p.num_q_heads / p.num_kv_heads;
  a.seqlen_q = p.seqlen_q;
  a.seqlen_k = p.seqlen_k;
  a.n_qb = (p.seqlen_q + bwd::BM - 1) / bwd::BM;
  a.n_kb = (p.seqlen_k + bwd::BM - 1) / bwd::BM;
  a.causal = p.causal ? 1 : 0;
  a.scale = p.scale;
  a.scale_log2 = p.scale * bwd::LOG2E;
  a.lse2 = lse2;
  a.delta = delta;
  a.dq = p.dq;
  a.dk = p.dk;
  a.dv = p.dv;
  a.dq_bs = p.dq_batch_stride;
  a.dq_hs = p.dq_head_stride;
  a.dq_rs = p.dq_row_stride;
  a.dk_bs = p.dk_batch_stride;
  a.dk_hs = p.dk_head_stride;
  a.dk_rs = p.dk_row_stride;
  a.dv_bs = p.dv_batch_stride;
  a.dv_hs = p.dv_head_stride;
  a.dv_rs = p.dv_row_stride;
  a.grad_f32 = p.grad_dtype == ATTN_DTYPE_F32;
  a.error_flags = p.error_flags;
  a.wait_limit = pipeline_wait_limit();
  a.planted = planted_bounds_site();
  const long long kv_items = (long long)a.n_kb * p.batch * p.num_kv_heads;
  const long long q_items = (long long)a.n_qb * p.batch * p.num_q_heads;
  attn_status_t st;
  if (D == 128) {
    st = launch_bwd<128, true>(tq, tk, tv, tdo, a, kv_items, false, stream);
    if (st == ATTN_OK) st = launch_bwd<128, false>(tq, tk, tv, tdo, a, q_items, kv_items > 0, stream);
  } else {
    st = launch_bwd<64, true>(tq, tk, tv, tdo, a, kv_items, false, stream);
    if (st == ATTN_OK) st = launch_bwd<64, false>(tq, tk, tv, tdo, a, q_items, kv_items > 0, stream);
  }
  // The dQ kernel is a dependent only of this call's dK/dV launch (a kernel
  // before the call may trigger its dependents early, and the prep kernel's
  // results must be complete before the dQ kernel reads them).
  return st;
}

}  // namespace attn
