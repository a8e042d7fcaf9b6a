// Split-KV paged decode and the log-sum-exp combine, for sm_100a.
//
// What they compute: one query token per sequence attends to all of that
// sequence's cached keys, which live in 16-token blocks of a shared pool
// addressed through a per-sequence block table ("抱infra脚", Paged Attention).
// The key range is cut into splits handled by different CTAs; each split
// yields its normalised partial output and log-sum-exp in fp32, and a small
// kernel merges them with the online-softmax formula ("GPU Kernel 调度:大模型推
// 理的拐点 2026", Flash Decoding section).
//
// Decode kernel (grid = splits x kv_heads x batch, 4 warps per CTA):
//   * one CTA serves all G = Hq/Hkv query heads of one key/value head, so each
//     K/V block is read from HBM once for the whole group;
//   * each warp walks every 4th block of the split; blocks are gathered through
//     the block table with coalesced 16-byte cp.async copies (a warp moves a
//     4 KB K block and a 4 KB V block per step, 512 contiguous bytes per
//     instruction) into a 3-stage per-warp shared-memory ring;
//   * q.k: lane (half h, chunk c) holds 8 head_dim elements of 8 tokens; partial
//     dot products for all G heads use packed fp32 FMAs, then a transposing
//     butterfly over the 16 lanes of a half-warp finishes them with 8G/16
//     values per lane;
//   * online softmax per head with the running max kept stale until it grows by
//     more than 2^8 (O and the row sum stay consistent); p is exchanged through
//     shared memory; O accumulates p * v with packed fp32 FMAs;
//   * masked tokens (past the sequence end, or a block whose table entry is out
//     of range) get p = 0 and their values are never multiplied in, so stale or
//     NaN cache contents cannot leak into the result;
//   * the 4 warps' states are merged in shared memory; a sequence with a single
//     split writes O and LSE directly, otherwise the split writes its partial.
// Combine kernel: one warp per (sequence, query head) row, 16-byte loads.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "internal.h"
#include "sm100_ptx.cuh"

namespace attn {
namespace decode {

constexpr int D = 128;
constexpr int BS = 16;          // tokens per cache block
constexpr int WARPS = 4;
constexpr int NST = 3;          // per-warp pipeline stages
constexpr int BLOCK_BYTES = BS * D * 2;  // 4 KB
constexpr float RESCALE_THRESHOLD = 8.0f;
constexpr float LN2 = 0.69314718055994530942f;

struct Args {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k_cache;
  const __nv_bfloat16* v_cache;
  const int32_t* block_table;
  const int32_t* seq_lens;
  void* o;
  float* lse;
  int o_f32;
  float* part_o;
  float* part_lse;
  int batch, hq, hkv, max_blocks, num_blocks, split_tokens;
  float scale_log2;
  int32_t* error_flags;
};

template <int G>
struct Smem {
  uint8_t kv[WARPS][NST][2][BLOCK_BYTES];  // 96 KB
  float sc[WARPS][G][BS];                  // scores (log2 units)
  float p[WARPS][2][BS / 2][G];            // probabilities, [token parity][token / 2][head]
  float alpha[WARPS][G];
};

template <int G>
struct MergeSmem {
  float m[WARPS][G];
  float l[WARPS][G];
  float o[WARPS][G][D];
};

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ float2 bf16x2_to_float2(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

// Sequence length clamped to the block table's capacity (flagging a fault).
__device__ __forceinline__ int checked_len(const Args& a, int b) {
  int L = a.seq_lens[b];
  if (L < 0 || L > a.max_blocks * BS) {
    if (a.error_flags) atomicOr(a.error_flags, ATTN_FAULT_BAD_LENGTH);
    L = L < 0 ? 0 : a.max_blocks * BS;
  }
  return L;
}

template <int G>
__global__ void __launch_bounds__(WARPS * 32)
    decode_split_kernel(const Args a) {
  static_assert(G == 1 || G == 2 || G == 4 || G == 8, "group size");
  constexpr int NF = (G >= 2) ? G / 2 : 1;  // scores per lane after the reduction
  extern __shared__ __align__(128) uint8_t smem_raw[];
  Smem<G>& sm = *reinterpret_cast<Smem<G>*>(smem_raw);

  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int warp = warp_id(), lane = lane_id();
  const int hw = lane >> 4, c = lane & 15;  // half-warp, 16-byte chunk of head_dim

  const int T = a.split_tokens;
  int L = checked_len(a, b);
  if (L > (int)gridDim.x * T) {  // longer than the caller's max_seq_len bound
    if (a.error_flags && split == 0 && threadIdx.x == 0) atomicOr(a.error_flags, ATTN_FAULT_BAD_LENGTH);
    L = gridDim.x * T;
  }
  const int n_splits = max(1, (L + T - 1) / T);
  if (split >= n_splits) return;
  const int t_begin = split * T;
  const int t_end = min(L, t_begin + T);
  const int blk_begin = t_begin / BS;
  const int blk_end = (t_end + BS - 1) / BS;
  const int32_t* table = a.block_table + (long long)b * a.max_blocks;

  // q for the G heads: this lane's 8 elements (chunk c), as 4 pairs per head.
  float2 q2[G][4];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const uint4 raw =
        *reinterpret_cast<const uint4*>(a.q + ((long long)b * a.hq + kvh * G + g) * D + c * 8);
    q2[g][0] = bf16x2_to_float2(raw.x);
    q2[g][1] = bf16x2_to_float2(raw.y);
    q2[g][2] = bf16x2_to_float2(raw.z);
    q2[g][3] = bf16x2_to_float2(raw.w);
  }

  float2 o2[G][4];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int m = 0; m < 4; ++m) o2[g][m] = make_float2(0.f, 0.f);
  float m_run = -INFINITY, l_run = 0.f;  // meaningful in lanes g < G (head g)

  // This warp's blocks: blk_begin + warp, + WARPS, ...
  const int n_mine = (blk_end - blk_begin - warp + WARPS - 1) / WARPS;
  auto block_of = [&](int n) { return blk_begin + warp + n * WARPS; };
  auto phys_of = [&](int blk, bool& valid) {
    const int ph = table[blk];
    valid = (ph >= 0) && (ph < a.num_blocks);
    return ph;
  };
  auto issue = [&](int n) {
    if (n < n_mine) {
      bool valid;
      const int ph = phys_of(block_of(n), valid);
      if (valid) {
        const long long off = ((long long)ph * a.hkv + kvh) * (BS * D);
        const uint8_t* ksrc = reinterpret_cast<const uint8_t*>(a.k_cache + off);
        const uint8_t* vsrc = reinterpret_cast<const uint8_t*>(a.v_cache + off);
        uint8_t* kdst = sm.kv[warp][n % NST][0];
        uint8_t* vdst = sm.kv[warp][n % NST][1];
#pragma unroll
        for (int i = 0; i < 8; ++i) cp_async16(kdst + (i * 32 + lane) * 16, ksrc + (i * 32 + lane) * 16);
#pragma unroll
        for (int i = 0; i < 8; ++i) cp_async16(vdst + (i * 32 + lane) * 16, vsrc + (i * 32 + lane) * 16);
      }
    }
    cp_async_commit();
  };

#pragma unroll
  for (int s = 0; s < NST - 1; ++s) issue(s);

  for (int n = 0; n < n_mine; ++n) {
    issue(n + NST - 1);
    cp_async_wait<NST - 1>();
    __syncwarp();
    const int blk = block_of(n);
    bool valid;
    phys_of(blk, valid);
    if (!valid && lane == 0 && a.error_flags) atomicOr(a.error_flags, ATTN_FAULT_BAD_BLOCK);
    const int tok0 = blk * BS;
    const int n_valid = valid ? min(BS, t_end - tok0) : 0;  // tokens of this block inside the split
    const uint8_t* kblk = sm.kv[warp][n % NST][0];
    const uint8_t* vblk = sm.kv[warp][n % NST][1];

    // ---- partial q.k for 8 tokens (2i + hw) x G heads over this lane's 8 elements
    float v[8 * G];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint4 kr = *reinterpret_cast<const uint4*>(kblk + (2 * i + hw) * (D * 2) + c * 16);
      const float2 k0 = bf16x2_to_float2(kr.x), k1 = bf16x2_to_float2(kr.y), k2 = bf16x2_to_float2(kr.z),
                   k3 = bf16x2_to_float2(kr.w);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float2 acc = __fmul2_rn(q2[g][0], k0);
        acc = __ffma2_rn(q2[g][1], k1, acc);
        acc = __ffma2_rn(q2[g][2], k2, acc);
        acc = __ffma2_rn(q2[g][3], k3, acc);
        v[i * G + g] = acc.x + acc.y;
      }
    }
    // ---- transposing butterfly over the 16 lanes of the half-warp
    {
      int n_cur = 8 * G;
#pragma unroll
      for (int mask = 8; mask >= 1; mask >>= 1) {
        if (n_cur >= 2) {
          const int half = n_cur / 2;
          const bool up = (c & mask) != 0;
#pragma unroll
          for (int k = 0; k < 8 * G / 2; ++k) {
            if (k < half) {
              const float send = up ? v[k] : v[half + k];
              const float keep = up ? v[half + k] : v[k];
              v[k] = keep + __shfl_xor_sync(0xffffffffu, send, mask);
            }
          }
          n_cur = half;
        } else {
          v[0] += __shfl_xor_sync(0xffffffffu, v[0], mask);
        }
      }
    }
    // lane holds NF finished scores, global index base + k -> token 2*(idx/G) + hw, head idx%G
    const int base = (G >= 2) ? NF * c : (c >> 1);
#pragma unroll
    for (int k = 0; k < NF; ++k) {
      const int idx = base + k;
      const int tk = 2 * (idx / G) + hw;
      const int g = idx % G;
      const float s = (tk < n_valid) ? v[k] * a.scale_log2 : -INFINITY;
      sm.sc[warp][g][tk] = s;
    }
    __syncwarp();
    // ---- online softmax, lane g owns head g
    if (lane < G) {
      float s[BS];
#pragma unroll
      for (int t4 = 0; t4 < BS / 4; ++t4) {
        const float4 x = *reinterpret_cast<const float4*>(&sm.sc[warp][lane][t4 * 4]);
        s[t4 * 4 + 0] = x.x;
        s[t4 * 4 + 1] = x.y;
        s[t4 * 4 + 2] = x.z;
        s[t4 * 4 + 3] = x.w;
      }
      float bm = s[0];
#pragma unroll
      for (int t = 1; t < BS; ++t) bm = fmaxf(bm, s[t]);
      const float m_new = fmaxf(m_run, bm);
      const bool upd = (m_new - m_run) > RESCALE_THRESHOLD;
      const float alpha = upd ? ex2_approx(m_run - m_new) : 1.f;
      if (upd) m_run = m_new;
      const float mo = (m_run == -INFINITY) ? 0.f : m_run;
      float rs = 0.f;
#pragma unroll
      for (int t = 0; t < BS; ++t) {
        const float p = ex2_approx(s[t] - mo);
        rs += p;
        sm.p[warp][t & 1][t >> 1][lane] = p;
      }
      l_run = l_run * alpha + rs;
      sm.alpha[warp][lane] = alpha;
    }
    __syncwarp();
    // ---- O += p * v
    {
      float al[G];
      bool any = false;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        al[g] = sm.alpha[warp][g];
        any |= (al[g] != 1.f);
      }
      if (any) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float2 a2 = make_float2(al[g], al[g]);
#pragma unroll
          for (int m = 0; m < 4; ++m) o2[g][m] = __fmul2_rn(o2[g][m], a2);
        }
      }
      const bool full = (n_valid == BS);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int tk = 2 * i + hw;
        uint4 vr = *reinterpret_cast<const uint4*>(vblk + tk * (D * 2) + c * 16);
        if (!full && tk >= n_valid) vr = make_uint4(0u, 0u, 0u, 0u);  // never multiply masked values in
        const float2 v0 = bf16x2_to_float2(vr.x), v1 = bf16x2_to_float2(vr.y), v2 = bf16x2_to_float2(vr.z),
                     v3 = bf16x2_to_float2(vr.w);
        float pg[G];
#pragma unroll
        for (int g = 0; g < G; ++g) pg[g] = sm.p[warp][hw][i][g];
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float2 p2 = make_float2(pg[g], pg[g]);
          o2[g][0] = __ffma2_rn(p2, v0, o2[g][0]);
          o2[g][1] = __ffma2_rn(p2, v1, o2[g][1]);
          o2[g][2] = __ffma2_rn(p2, v2, o2[g][2]);
          o2[g][3] = __ffma2_rn(p2, v3, o2[g][3]);
        }
      }
    }
    __syncwarp();  // the slot is refilled by the next issue
  }
  cp_async_wait<0>();

  // ---- merge the two half-warps (disjoint tokens, same running max)
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      o2[g][m].x += __shfl_xor_sync(0xffffffffu, o2[g][m].x, 16);
      o2[g][m].y += __shfl_xor_sync(0xffffffffu, o2[g][m].y, 16);
    }
  __syncthreads();  // the KV ring is reused for the merge
  MergeSmem<G>& mg = *reinterpret_cast<MergeSmem<G>*>(smem_raw);
  if (lane < G) {
    mg.m[warp][lane] = m_run;
    mg.l[warp][lane] = l_run;
  }
  if (hw == 0) {
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float4* dst = reinterpret_cast<float4*>(&mg.o[warp][g][c * 8]);
      dst[0] = make_float4(o2[g][0].x, o2[g][0].y, o2[g][1].x, o2[g][1].y);
      dst[1] = make_float4(o2[g][2].x, o2[g][2].y, o2[g][3].x, o2[g][3].y);
    }
  }
  __syncthreads();

  // ---- merge the 4 warps: thread d handles column d of every head
  const int d = threadIdx.x;
#pragma unroll
  for (int g = 0; g < G; ++g) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) M = fmaxf(M, mg.m[w][g]);
    const float Ms = (M == -INFINITY) ? 0.f : M;
    float lsum = 0.f, acc = 0.f;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) {
      const float wt = ex2_approx(mg.m[w][g] - Ms);
      lsum += wt * mg.l[w][g];
      acc += wt * mg.o[w][g][d];
    }
    const bool empty = !(lsum > 0.f);
    const float out = empty ? 0.f : acc / lsum;
    const float lse = empty ? -INFINITY : (M + log2f(lsum)) * LN2;
    const long long row = (long long)b * a.hq + kvh * G + g;
    if (n_splits == 1) {
      if (a.o_f32)
        reinterpret_cast<float*>(a.o)[row * D + d] = out;
      else
        reinterpret_cast<__nv_bfloat16*>(a.o)[row * D + d] = __float2bfloat16_rn(out);
      if (d == 0 && a.lse) a.lse[row] = lse;
    } else {
      const long long rows = (long long)a.batch * a.hq;
      a.part_o[((long long)split * rows + row) * D + d] = out;
      if (d == 0) a.part_lse[(long long)split * rows + row] = lse;
    }
  }
}

}  // namespace decode

// ---------------------------------------------------------------------------
// Combine
// ---------------------------------------------------------------------------
namespace combine {

// One warp per row. Row r's split count is splits_per_row[r] when given,
// else num_splits when seq_lens is NULL (standalone call), else (decode path)
// n = max(1, ceil(L / split_tokens)) from its sequence length; on the decode
// path rows with n == 1 were written by the decode kernel and are skipped.
template <int HD>
__global__ void __launch_bounds__(256) lse_combine_kernel(const float* __restrict__ part_o,
                                                          const float* __restrict__ part_lse, int num_splits,
                                                          int rows, const int32_t* __restrict__ splits_per_row,
                                                          const int32_t* __restrict__ seq_lens, int split_tokens,
                                                          int max_len, int rows_per_seq, void* out_o, int out_f32,
                                                          float* out_lse) {
  constexpr int PER = HD / 32;  // floats per lane
  const int row = blockIdx.x * (blockDim.x / 32) + warp_id();
  const int lane = lane_id();
  if (row >= rows) return;
  int n;
  if (splits_per_row) {  // standalone call with per-row counts
    n = min(max(splits_per_row[row], 0), num_splits);
  } else if (seq_lens == nullptr) {  // standalone call: every row has num_splits partials
    n = num_splits;
  } else {  // decode path
    int L = seq_lens[row / rows_per_seq];
    L = min(max(L, 0), max_len);
    n = max(1, (L + split_tokens - 1) / split_tokens);
    if (n == 1) return;
    n = min(n, num_splits);
  }
  constexpr float LOG2E = 1.4426950408889634f;
  // max and sum of exp over the splits, lanes strided over s
  float M = -INFINITY;
  for (int s = lane; s < n; s += 32) M = fmaxf(M, part_lse[(long long)s * rows + row]);
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  float out[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) out[i] = 0.f;
  float lse = -INFINITY;
  if (M != -INFINITY) {
    float sum = 0.f;
    for (int s = lane; s < n; s += 32) sum += ex2_approx((part_lse[(long long)s * rows + row] - M) * LOG2E);
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    lse = M + logf(sum);
    for (int s = 0; s < n; ++s) {
      const float ls = part_lse[(long long)s * rows + row];
      if (ls == -INFINITY) continue;  // weight 0: its partial is not read
      const float wgt = ex2_approx((ls - lse) * LOG2E);
      const float* src = part_o + ((long long)s * rows + row) * HD + lane * PER;
      if constexpr (PER == 4) {
        const float4 x = *reinterpret_cast<const float4*>(src);
        out[0] = fmaf(wgt, x.x, out[0]);
        out[1] = fmaf(wgt, x.y, out[1]);
        out[2] = fmaf(wgt, x.z, out[2]);
        out[3] = fmaf(wgt, x.w, out[3]);
      } else {
        const float2 x = *reinterpret_cast<const float2*>(src);
        out[0] = fmaf(wgt, x.x, out[0]);
        out[1] = fmaf(wgt, x.y, out[1]);
      }
    }
  }
  if (out_f32) {
    float* dst = reinterpret_cast<float*>(out_o) + (long long)row * HD + lane * PER;
#pragma unroll
    for (int i = 0; i < PER; ++i) dst[i] = out[i];
  } else {
    __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(out_o) + (long long)row * HD + lane * PER;
#pragma unroll
    for (int i = 0; i < PER; i += 2) *reinterpret_cast<uint32_t*>(dst + i) = pack_bf16x2(out[i], out[i + 1]);
  }
  if (lane == 0 && out_lse) out_lse[row] = lse;
}

}  // namespace combine

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
static int env_int(const char* name, int dflt) {
  const char* e = getenv(name);
  return (e && *e) ? atoi(e) : dflt;
}

DecodePlan plan_decode(const attn_decode_params& p) {
  DecodePlan plan;
  const int cap = p.max_blocks_per_seq * decode::BS;
  const int max_len = (p.max_seq_len > 0 && p.max_seq_len < cap) ? p.max_seq_len : cap;
  const int unit = decode::BS * decode::WARPS;  // 64 tokens
  int T;
  const int forced = env_int("ATTN_DECODE_SPLIT_TOKENS", 0);
  if (forced > 0) {
    T = forced;
  } else if (p.num_splits > 0) {
    T = (max_len + p.num_splits - 1) / p.num_splits;
  } else {
    // Enough CTAs for many waves (good balance across sequences of mixed
    // lengths) while each split still streams at least 512 tokens.
    const long long pairs = (long long)p.batch * p.num_kv_heads;
    const long long target = 32LL * device_sm_count();
    long long per_seq = (target + pairs - 1) / pairs;
    if (per_seq < 1) per_seq = 1;
    T = (int)((max_len + per_seq - 1) / per_seq);
    if (T < 512) T = 512;
  }
  T = ((T + unit - 1) / unit) * unit;
  if (T <= 0) T = unit;
  plan.split_tokens = T;
  plan.max_splits = max_len > 0 ? (max_len + T - 1) / T : 1;
  if (plan.max_splits < 1) plan.max_splits = 1;
  const size_t rows = (size_t)p.batch * p.num_q_heads;
  size_t bytes = 0;
  if (plan.max_splits > 1) {
    const size_t po = plan.max_splits * rows * p.head_dim * sizeof(float);
    const size_t pl = plan.max_splits * rows * sizeof(float);
    bytes = ((po + 255) / 256) * 256 + ((pl + 255) / 256) * 256;
  }
  plan.workspace_bytes = bytes;
  return plan;
}

template <int G>
static attn_status_t launch_decode_g(const decode::Args& a, const DecodePlan& plan, cudaStream_t stream) {
  auto kern = decode::decode_split_kernel<G>;
  const int smem = (int)sizeof(decode::Smem<G>);
  static_assert(sizeof(decode::MergeSmem<G>) <= sizeof(decode::Smem<G>), "merge buffer fits");
  static bool configured = false;
  if (!configured) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return ATTN_ERR_CUDA;
    configured = true;
  }
  dim3 grid(plan.max_splits, a.hkv, a.batch);
  kern<<<grid, decode::WARPS * 32, smem, stream>>>(a);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

attn_status_t launch_decode(const attn_decode_params& p, const DecodePlan& plan, void* workspace,
                            cudaStream_t stream) {
  if (p.batch == 0) return ATTN_OK;
  decode::Args a;
  a.q = reinterpret_cast<const __nv_bfloat16*>(p.q);
  a.k_cache = reinterpret_cast<const __nv_bfloat16*>(p.k_cache);
  a.v_cache = reinterpret_cast<const __nv_bfloat16*>(p.v_cache);
  a.block_table = p.block_table;
  a.seq_lens = p.seq_lens;
  a.o = p.o;
  a.lse = p.lse;
  a.o_f32 = p.o_dtype == ATTN_DTYPE_F32;
  const size_t rows = (size_t)p.batch * p.num_q_heads;
  a.part_o = reinterpret_cast<float*>(workspace);
  const size_t po = plan.max_splits * rows * p.head_dim * sizeof(float);
  a.part_lse = plan.max_splits > 1
                   ? reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(workspace) + ((po + 255) / 256) * 256)
                   : nullptr;
  a.batch = p.batch;
  a.hq = p.num_q_heads;
  a.hkv = p.num_kv_heads;
  a.max_blocks = p.max_blocks_per_seq;
  a.num_blocks = p.num_blocks;
  a.split_tokens = plan.split_tokens;
  a.scale_log2 = p.scale * 1.4426950408889634f;
  a.error_flags = p.error_flags;
  attn_status_t st;
  switch (p.num_q_heads / p.num_kv_heads) {
    case 1: st = launch_decode_g<1>(a, plan, stream); break;
    case 2: st = launch_decode_g<2>(a, plan, stream); break;
    case 4: st = launch_decode_g<4>(a, plan, stream); break;
    case 8: st = launch_decode_g<8>(a, plan, stream); break;
    default: return ATTN_ERR_UNSUPPORTED;
  }
  if (st != ATTN_OK || plan.max_splits <= 1) return st;
  return launch_combine(a.part_o, a.part_lse, plan.max_splits, (int)rows, p.head_dim, nullptr, p.seq_lens,
                        plan.split_tokens, p.num_q_heads, p.o, p.o_dtype, p.lse, stream);
}

attn_status_t launch_combine(const float* part_o, const float* part_lse, int num_splits, int rows, int head_dim,
                             const int32_t* splits_per_row, const int32_t* seq_lens, int split_tokens,
                             int rows_per_seq, void* out_o, attn_dtype_t out_dtype, float* out_lse,
                             cudaStream_t stream) {
  if (rows == 0) return ATTN_OK;
  const int warps = 8;
  const int grid = (rows + warps - 1) / warps;
  const int max_len = num_splits * split_tokens;
  if (head_dim == 128)
    combine::lse_combine_kernel<128><<<grid, warps * 32, 0, stream>>>(
        part_o, part_lse, num_splits, rows, splits_per_row, seq_lens, split_tokens, max_len, rows_per_seq, out_o,
        out_dtype == ATTN_DTYPE_F32, out_lse);
  else
    combine::lse_combine_kernel<64><<<grid, warps * 32, 0, stream>>>(
        part_o, part_lse, num_splits, rows, splits_per_row, seq_lens, split_tokens, max_len, rows_per_seq, out_o,
        out_dtype == ATTN_DTYPE_F32, out_lse);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace attn
