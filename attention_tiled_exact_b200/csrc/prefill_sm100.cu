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
// B200 design (one CTA per SM, 320 threads):
//   * two Q tiles of 128 rows per CTA. For GQA with an even group size the two
//     tiles are two query heads of one key/value head on the same rows, so both
//     tiles need exactly the same K/V range; otherwise they are two row blocks
//     of one head. K/V tiles are loaded once for both.
//   * warp 8 (TMA): loads the Q tiles and streams K_j, V_j tiles (128 keys)
//     into a ring of shared-memory slots with cp.async.bulk.tensor, 128-byte
//     swizzle, completion on mbarriers.
//   * warp 9 (MMA): one thread issues tcgen05.mma. S_t = Q_t K_j^T (M=128,
//     N=128, K=head_dim) lands in tensor memory; O_t += P_t V_j reads P_t from
//     tensor memory (or shared memory in the reference variant) and V_j from
//     shared memory. The issue order PV_0(j), S_0(j+1), PV_1(j), S_1(j+1) lets
//     one tile's softmax overlap the other tile's matrix products.
//   * warps 0-3 / 4-7 (softmax, one warpgroup per tile, one thread per row):
//     read S from tensor memory, mask (diagonal and tail tiles only), update the
//     running max, p = 2^(s*scale*log2e - m), running sum, write P (bf16) back
//     to tensor memory, and rescale O in tensor memory when the max grew by
//     more than 2^8 (otherwise the stale max is kept, which leaves O and the
//     row sum consistent). The same warps run the epilogue: O / l -> global,
//     LSE = (m + log2 l) * ln 2.
//   * tensor memory: S_0 cols [0,128), S_1 [128,256), O_0 [256,256+D),
//     O_1 [384,384+D); P_t (bf16 pairs) overwrites the first 64 columns of S_t.
//   * every mbarrier wait is bounded; on a timeout the CTA raises a flag in
//     shared memory, all roles stop, in-flight copies and MMAs are drained
//     (again bounded), tensor memory is freed, and ATTN_FAULT_TIMEOUT is ORed
//     into the caller's error word.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include "internal.h"
#include "sm100_ptx.cuh"

namespace attn {
namespace prefill {

constexpr int BM = 128;            // query rows per Q tile
constexpr int BN = 128;            // keys per K/V tile
constexpr int NUM_THREADS = 320;   // 8 softmax warps + TMA warp + MMA warp
constexpr int TMA_WARP = 8;
constexpr int MMA_WARP = 9;
constexpr uint32_t TMEM_COLS = 512;
constexpr long long WAIT_LIMIT = 2000000000LL;  // cycles (~1 s)
constexpr float RESCALE_THRESHOLD = 8.0f;        // log2 units: rescale only when the max grows by > 2^8

struct Args {
  int batch, hq, hkv, group, seqlen_q, seqlen_k;
  float scale_log2;
  int causal;
  int pair_heads;
  int n_row_blocks;
  const int32_t* seqlens_q;
  const int32_t* seqlens_k;
  void* o;
  float* lse;
  int o_f32;
  long long o_bs, o_hs, o_rs;
  // paged keys/values
  int paged;
  const int32_t* block_table;
  int max_blocks_per_seq;
  int num_blocks;
  int32_t* error_flags;
};

template <int D, int NSTAGE, bool P_TMEM>
struct Layout {
  static constexpr int CHUNKS = D / 64;               // 64-column (128-byte) boxes per row
  static constexpr int Q_TILE = BM * D * 2;           // bytes
  static constexpr int KV_TILE = BN * D * 2;
  static constexpr int P_TILE = BM * BN * 2;
  static constexpr int Q_OFF = 0;
  static constexpr int KV_OFF = Q_OFF + 2 * Q_TILE;
  static constexpr int P_OFF = KV_OFF + NSTAGE * KV_TILE;
  static constexpr int BAR_OFF = P_OFF + (P_TMEM ? 0 : 2 * P_TILE);
  // barriers: q_full, kv_full[NSTAGE], kv_empty[NSTAGE], s_full[2], p_full[2], o_full[2], mma_done
  static constexpr int NUM_BARS = 1 + 2 * NSTAGE + 2 + 2 + 2 + 1;
  static constexpr int MISC_OFF = BAR_OFF + NUM_BARS * 8;
  static constexpr int BYTES = MISC_OFF + 16;
  static constexpr int SMEM_BYTES = BYTES + 1024;  // slack for 1024-byte alignment
};

struct Work {
  int b, kvh;
  int head[2];
  int row0[2];
  int active[2];
  int n_kv[2];
  int sq, sk;
};

__device__ __forceinline__ Work decode_work(const Args& a, int item) {
  Work w;
  if (a.pair_heads) {
    const int pairs = a.group / 2;
    const int per_rb = a.batch * a.hkv * pairs;
    const int rb = a.n_row_blocks - 1 - item / per_rb;  // heaviest (causal) row blocks first
    int r = item % per_rb;
    const int pair = r % pairs;
    r /= pairs;
    w.kvh = r % a.hkv;
    w.b = r / a.hkv;
    w.head[0] = w.kvh * a.group + 2 * pair;
    w.head[1] = w.head[0] + 1;
    w.row0[0] = w.row0[1] = rb * BM;
  } else {
    const int npairs = (a.n_row_blocks + 1) / 2;
    const int per = a.batch * a.hq;
    const int p = npairs - 1 - item / per;
    const int r = item % per;
    const int h = r % a.hq;
    w.b = r / a.hq;
    w.kvh = h / a.group;
    w.head[0] = w.head[1] = h;
    w.row0[0] = 2 * p * BM;
    w.row0[1] = (2 * p + 1) * BM;
  }
  w.sq = a.seqlens_q ? a.seqlens_q[w.b] : a.seqlen_q;
  w.sk = a.seqlens_k ? a.seqlens_k[w.b] : a.seqlen_k;
  if (w.sq > a.seqlen_q) w.sq = a.seqlen_q;
  if (w.sq < 0) w.sq = 0;
  if (w.sk < 0) w.sk = 0;
  for (int t = 0; t < 2; ++t) {
    w.active[t] = w.row0[t] < w.sq;
    int kend = w.sk;
    if (a.causal) {
      const int last_row = min(w.row0[t] + BM, w.sq) - 1;
      const int lim = last_row + (w.sk - w.sq) + 1;  // keys [0, lim) visible to the tile's last row
      kend = max(0, min(w.sk, lim));
    }
    w.n_kv[t] = w.active[t] ? (kend + BN - 1) / BN : 0;
  }
  return w;
}

template <int D, int NSTAGE, bool P_TMEM>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    prefill_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const Args args) {
  using L = Layout<D, NSTAGE, P_TMEM>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = bars + 1 + NSTAGE;
  uint64_t* s_full = bars + 1 + 2 * NSTAGE;
  uint64_t* p_full = s_full + 2;
  uint64_t* o_full = p_full + 2;
  uint64_t* mma_done = o_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4);

  const int warp = warp_id();
  const int lane = lane_id();

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
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

  const Work w = decode_work(args, blockIdx.x);
  const int n_kv = max(w.n_kv[0], w.n_kv[1]);

  if (warp == TMA_WARP) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      const uint32_t q_bytes = (w.active[0] + w.active[1]) * L::Q_TILE;
      mbar_arrive_expect_tx(q_full, q_bytes);
      for (int t = 0; t < 2; ++t) {
        if (!w.active[t]) continue;
        for (int c = 0; c < L::CHUNKS; ++c)
          tma_load_4d(smem + L::Q_OFF + t * L::Q_TILE + c * (BM * 128), &tm_q, q_full, c * 64, w.row0[t],
                      w.head[t], w.b);
      }
      int issued = 0;
      bool ok = true;
      for (int i = 0; i < 2 * n_kv && ok; ++i) {
        const int j = i >> 1;
        const int s = i % NSTAGE;
        if (i >= NSTAGE) ok = mbar_wait_bounded(&kv_empty[s], ((i / NSTAGE) - 1) & 1, abort_flag, WAIT_LIMIT);
        if (!ok) break;
        mbar_arrive_expect_tx(&kv_full[s], L::KV_TILE);
        const CUtensorMap* tm = (i & 1) ? &tm_v : &tm_k;
        for (int c = 0; c < L::CHUNKS; ++c)
          tma_load_4d(smem + L::KV_OFF + s * L::KV_TILE + c * (BN * 128), tm, &kv_full[s], c * 64, j * BN,
                      w.kvh, w.b);
        issued = i + 1;
      }
      // Drain: wait for the last copy issued into each slot, so no copy is in
      // flight when the CTA exits (matters only on the abort path).
      for (int i = max(0, issued - NSTAGE); i < issued; ++i)
        mbar_wait_bounded(&kv_full[i % NSTAGE], (i / NSTAGE) & 1, abort_flag, WAIT_LIMIT);
      if (w.active[0] || w.active[1]) mbar_wait_bounded(q_full, 0, abort_flag, WAIT_LIMIT);
    }
  } else if (warp == MMA_WARP) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t ID_S = instr_desc_bf16(BM, BN, 0);
      constexpr uint32_t ID_PV = instr_desc_bf16(BM, D, 1);
      const uint32_t q_smem = smem_addr(smem + L::Q_OFF);
      const uint32_t kv_smem = smem_addr(smem + L::KV_OFF);
      auto issue_s = [&](int t, int j) {
        const uint32_t qa = q_smem + t * L::Q_TILE;
        const uint32_t ka = kv_smem + ((2 * j) % NSTAGE) * L::KV_TILE;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (BM * 128) + (kk & 3) * 32;
          mma_ss(tmem_base + t * 128, smem_desc_sw128(qa + off, 16, 1024), smem_desc_sw128(ka + off, 16, 1024),
                 ID_S, kk > 0);
        }
      };
      auto issue_pv = [&](int t, int j) {
        const uint32_t va = kv_smem + ((2 * j + 1) % NSTAGE) * L::KV_TILE;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          const uint64_t bdesc = smem_desc_sw128(va + kk * 16 * 128, BN * 128, 1024);
          if constexpr (P_TMEM) {
            mma_ts(tmem_base + 256 + t * 128, tmem_base + t * 128 + kk * 8, bdesc, ID_PV, (j > 0) || (kk > 0));
          } else {
            const uint32_t pa = smem_addr(smem + L::P_OFF + t * L::P_TILE) + (kk >> 2) * (BM * 128) + (kk & 3) * 32;
            mma_ss(tmem_base + 256 + t * 128, smem_desc_sw128(pa, 16, 1024), bdesc, ID_PV, (j > 0) || (kk > 0));
          }
        }
      };
      bool ok = true;
      if (n_kv > 0) {
        ok = mbar_wait_bounded(q_full, 0, abort_flag, WAIT_LIMIT) &&
             mbar_wait_bounded(&kv_full[0], 0, abort_flag, WAIT_LIMIT);
        if (ok) {
          tc_fence_after();
          for (int t = 0; t < 2; ++t)
            if (w.n_kv[t] > 0) {
              issue_s(t, 0);
              mma_commit(&s_full[t]);
            }
          mma_commit(&kv_empty[0]);
        }
      }
      for (int j = 0; j < n_kv && ok; ++j) {
        const int iv = 2 * j + 1, ik = 2 * j + 2;
        ok = mbar_wait_bounded(&kv_full[iv % NSTAGE], (iv / NSTAGE) & 1, abort_flag, WAIT_LIMIT);
        bool k_ready = false;
        for (int t = 0; t < 2 && ok; ++t) {
          if (j >= w.n_kv[t]) continue;
          ok = mbar_wait_bounded(&p_full[t], j & 1, abort_flag, WAIT_LIMIT);
          if (!ok) break;
          tc_fence_after();
          issue_pv(t, j);
          if (j == w.n_kv[t] - 1) {
            mma_commit(&o_full[t]);
          } else {
            if (!k_ready) {
              ok = mbar_wait_bounded(&kv_full[ik % NSTAGE], (ik / NSTAGE) & 1, abort_flag, WAIT_LIMIT);
              if (!ok) break;
              tc_fence_after();
              k_ready = true;
            }
            issue_s(t, j + 1);
            mma_commit(&s_full[t]);
          }
        }
        if (!ok) break;
        mma_commit(&kv_empty[iv % NSTAGE]);
        if (k_ready) mma_commit(&kv_empty[ik % NSTAGE]);
      }
      // Wait until every MMA issued above has completed before tensor memory
      // can be released (bounded; matters on the abort path).
      mma_commit(mma_done);
      mbar_wait_bounded(mma_done, 0, abort_flag, WAIT_LIMIT);
    }
  } else {
    // ---------------------------------------------------------------- softmax + epilogue
    const int t = warp >> 2;
    const int sub = warp & 3;
    const int r = sub * 32 + lane;  // row within the tile == TMEM lane
    if (w.active[t]) {
      const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(sub * 32) << 16);
      const uint32_t tS = lane_base + t * 128;
      const uint32_t tO = lane_base + 256 + t * 128;
      const int qrow = w.row0[t] + r;
      const int qpos = qrow + (w.sk - w.sq);  // absolute position (bottom-right causal)
      const float sl2 = args.scale_log2;
      float m2 = -INFINITY;  // running max of s * scale * log2(e)
      float l = 0.f;         // running sum of 2^(s*scale*log2e - m2)
      bool ok = true;
      for (int j = 0; j < w.n_kv[t]; ++j) {
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(&s_full[t], j & 1, abort_flag, WAIT_LIMIT));
        if (!ok) break;
        tc_fence_after();
        uint32_t sb[BN];
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) tmem_ld32(tS + c * 32, &sb[c * 32]);
        tmem_ld_wait();
        float s[BN];
#pragma unroll
        for (int c = 0; c < BN; ++c) s[c] = __uint_as_float(sb[c]);
        const int k0 = j * BN;
        const bool need_mask = (k0 + BN > w.sk) || (args.causal && (k0 + BN - 1 > w.row0[t] + (w.sk - w.sq)));
        if (need_mask) {
          const int lim = args.causal ? min(w.sk, qpos + 1) : w.sk;  // keys [0, lim) visible
#pragma unroll
          for (int c = 0; c < BN; ++c)
            if (k0 + c >= lim) s[c] = -INFINITY;
        }
        float mx = s[0];
#pragma unroll
        for (int c = 1; c < BN; ++c) mx = fmaxf(mx, s[c]);
        const float m_new = fmaxf(m2, mx * sl2);
        const bool upd = (m_new - m2) > RESCALE_THRESHOLD;  // false when both are -inf (NaN compare)
        const float alpha = upd ? ex2_approx(m2 - m_new) : 1.f;
        if (upd) m2 = m_new;
        const float m_off = (m2 == -INFINITY) ? 0.f : m2;
        float rs = 0.f;
#pragma unroll
        for (int c = 0; c < BN; ++c) {
          s[c] = ex2_approx(fmaf(s[c], sl2, -m_off));
          rs += s[c];
        }
        l = l * alpha + rs;
        if (j > 0 && __any_sync(0xffffffffu, upd)) {
          // O_t is stable here: PV(j-1) completed before S(j) was signalled.
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(tO + c * 32, o);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(tO + c * 32, o);
          }
          tmem_st_wait();
        }
        if constexpr (P_TMEM) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t pk[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) pk[i] = pack_bf16x2(s[h * 64 + 2 * i], s[h * 64 + 2 * i + 1]);
            tmem_st32(tS + h * 32, pk);
          }
          tmem_st_wait();
        } else {
          // P row r into the 128-byte-swizzled K-major tile: 16-byte unit u of a
          // 128-byte row sits at unit (u ^ (r % 8)).
          uint8_t* prow = smem + L::P_OFF + t * L::P_TILE + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
          for (int u = 0; u < BN / 8; ++u) {
            const int chunk = u >> 3, uu = u & 7;
            uint4 v;
            v.x = pack_bf16x2(s[u * 8 + 0], s[u * 8 + 1]);
            v.y = pack_bf16x2(s[u * 8 + 2], s[u * 8 + 3]);
            v.z = pack_bf16x2(s[u * 8 + 4], s[u * 8 + 5]);
            v.w = pack_bf16x2(s[u * 8 + 6], s[u * 8 + 7]);
            *reinterpret_cast<uint4*>(prow + chunk * (BM * 128) + ((uu ^ (r & 7)) * 16)) = v;
          }
          fence_proxy_async_smem();
        }
        tc_fence_before();
        mbar_arrive(&p_full[t]);
      }
      // ------------------------------------------------------------ epilogue
      const bool has_keys = w.n_kv[t] > 0;
      if (ok && has_keys) ok = __all_sync(0xffffffffu, mbar_wait_bounded(&o_full[t], 0, abort_flag, WAIT_LIMIT));
      if (ok) {
        const bool store = qrow < w.sq;
        const bool empty = !(l > 0.f);
        const float inv_l = empty ? 0.f : 1.f / l;
        const long long obase =
            (long long)w.b * args.o_bs + (long long)w.head[t] * args.o_hs + (long long)qrow * args.o_rs;
        if (args.lse && store) {
          const float lse = empty ? -INFINITY : (m2 + log2f(l)) * 0.69314718055994530942f;
          args.lse[((long long)w.b * args.hq + w.head[t]) * args.seqlen_q + qrow] = lse;
        }
        if (has_keys) tc_fence_after();
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          if (has_keys) {  // warp-uniform: every lane issues the collective load
            tmem_ld32(tO + c * 32, o);
            tmem_ld_wait();
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = 0u;
          }
          if (!store) continue;
          if (args.o_f32) {
            float* dst = reinterpret_cast<float*>(args.o) + obase + c * 32;
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
              float4 v = make_float4(__uint_as_float(o[i]) * inv_l, __uint_as_float(o[i + 1]) * inv_l,
                                     __uint_as_float(o[i + 2]) * inv_l, __uint_as_float(o[i + 3]) * inv_l);
              *reinterpret_cast<float4*>(dst + i) = v;
            }
          } else {
            __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(args.o) + obase + c * 32;
#pragma unroll
            for (int i = 0; i < 32; i += 8) {
              uint4 v;
              v.x = pack_bf16x2(__uint_as_float(o[i + 0]) * inv_l, __uint_as_float(o[i + 1]) * inv_l);
              v.y = pack_bf16x2(__uint_as_float(o[i + 2]) * inv_l, __uint_as_float(o[i + 3]) * inv_l);
              v.z = pack_bf16x2(__uint_as_float(o[i + 4]) * inv_l, __uint_as_float(o[i + 5]) * inv_l);
              v.w = pack_bf16x2(__uint_as_float(o[i + 6]) * inv_l, __uint_as_float(o[i + 7]) * inv_l);
              *reinterpret_cast<uint4*>(dst + i) = v;
            }
          }
        }
      }
    }
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
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// 4-D bf16 map over [d3][d2][d1][d0 = head_dim] with byte strides s1..s3, box
// (64, box_rows, 1, 1), 128-byte swizzle, zero fill out of bounds.
static bool encode_4d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t d3,
                      uint64_t s1, uint64_t s2, uint64_t s3, uint32_t box_rows) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {d0, d1, d2, d3};
  cuuint64_t strides[3] = {s1, s2, s3};
  cuuint32_t box[4] = {64, box_rows, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D, int NSTAGE, bool P_TMEM>
static attn_status_t launch_variant(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                    const Args& a, int items, cudaStream_t stream) {
  using L = Layout<D, NSTAGE, P_TMEM>;
  static_assert(L::SMEM_BYTES <= 232448, "shared memory budget");
  auto kern = prefill_fwd_kernel<D, NSTAGE, P_TMEM>;
  static bool configured = false;  // per process; the attribute is per function
  if (!configured) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM_BYTES) != cudaSuccess)
      return ATTN_ERR_CUDA;
    configured = true;
  }
  kern<<<items, NUM_THREADS, L::SMEM_BYTES, stream>>>(tq, tk, tv, a);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace prefill

// Debug knob: ATTN_PREFILL_P_SMEM=1 selects the variant that stages P in
// shared memory (a second, independently laid out path for cross-checking).
static int prefill_p_in_smem() {
  const char* e = getenv("ATTN_PREFILL_P_SMEM");
  return (e && e[0] == '1') ? 1 : 0;
}

attn_status_t launch_prefill(const attn_prefill_params& p, cudaStream_t stream) {
  using namespace prefill;
  if (p.batch == 0 || p.seqlen_q == 0 || p.num_q_heads == 0) return ATTN_OK;
  if (p.k_cache != nullptr) return ATTN_ERR_UNSUPPORTED;  // paged prefill: not in this build yet
  const int D = p.head_dim;
  CUtensorMap tq, tk, tv;
  if (!encode_4d(&tq, p.q, D, p.seqlen_q, p.num_q_heads, p.batch, p.q_row_stride * 2, p.q_head_stride * 2,
                 p.q_batch_stride * 2, BM))
    return ATTN_ERR_CUDA;
  if (p.seqlen_k > 0) {
    if (!encode_4d(&tk, p.k, D, p.seqlen_k, p.num_kv_heads, p.batch, p.k_row_stride * 2, p.k_head_stride * 2,
                   p.k_batch_stride * 2, BN) ||
        !encode_4d(&tv, p.v, D, p.seqlen_k, p.num_kv_heads, p.batch, p.v_row_stride * 2, p.v_head_stride * 2,
                   p.v_batch_stride * 2, BN))
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
  a.n_row_blocks = (p.seqlen_q + BM - 1) / BM;
  a.seqlens_q = p.seqlens_q;
  a.seqlens_k = p.seqlens_k;
  a.o = p.o;
  a.lse = p.lse;
  a.o_f32 = p.o_dtype == ATTN_DTYPE_F32;
  a.o_bs = p.o_batch_stride;
  a.o_hs = p.o_head_stride;
  a.o_rs = p.o_row_stride;
  a.error_flags = p.error_flags;
  long long items;
  if (a.pair_heads)
    items = (long long)a.n_row_blocks * p.batch * p.num_kv_heads * (a.group / 2);
  else
    items = (long long)((a.n_row_blocks + 1) / 2) * p.batch * p.num_q_heads;
  if (items <= 0) return ATTN_OK;
  if (items > 0x7fffffffLL) return ATTN_ERR_INVALID_ARG;

  const bool p_smem = prefill_p_in_smem() != 0;
  if (D == 128) {
    if (p_smem) return launch_variant<128, 2, false>(tq, tk, tv, a, (int)items, stream);
    return launch_variant<128, 4, true>(tq, tk, tv, a, (int)items, stream);
  }
  if (p_smem) return launch_variant<64, 4, false>(tq, tk, tv, a, (int)items, stream);
  return launch_variant<64, 6, true>(tq, tk, tv, a, (int)items, stream);
}

}  // namespace attn
