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
//   * q.k on the warp-level tensor cores (mma.sync m16n8k16, fp32 accumulate):
//     the G query heads are the rows of A (zero-padded to 16), the block's 16
//     tokens the columns of B, with head_dim permuted identically on both
//     sides so that each thread reads its K row slice as contiguous 16-byte
//     loads; the online softmax of a head then runs on its 4 lanes with
//     shuffles, the running max kept stale until it grows by more than 2^8 (O
//     and the row sum stay consistent);
//   * O += p * v: for bf16 caches on the CUDA cores in fp32 (p goes through
//     shared memory to lanes holding 8 head_dim elements of 8 tokens, packed
//     fp32 FMAs); for FP8 caches also on the tensor cores with P kept in
//     registers as fp16 (the score fragments of the two 8-token tiles form
//     the A fragment of one k = 16 step), which keeps the FP8 kernel on the
//     memory bound instead of the instruction bound;
//   * masked tokens (past the sequence end, or a block whose table entry is out
//     of range) get p = 0 and their values are never multiplied in, so stale or
//     NaN cache contents cannot leak into the result;
//   * the 4 warps' states are merged in shared memory; a sequence with a single
//     split writes O and LSE directly, otherwise the split writes its partial.
//   * FP8 cache (E4M3 codes, one scale per tensor): blocks are 2 KB, pairs of
//     codes are widened exactly to fp16 with cvt.rn.f16x2.e4m3x2, the key
//     scale multiplies the scores and the value scale O once at the end.
// Combine kernel: one warp per (sequence, query head) row, 16-byte loads.
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <string.h>
#include <stdint.h>

#include "bounds_check.cuh"
#include "internal.h"
#include "sm100_ptx.cuh"

namespace attn {
namespace decode {

constexpr int D = 128;
constexpr int BS = 16;          // tokens per cache block
constexpr int WARPS = 4;
// Per-warp pipeline stages: an FP8 block is half the bytes of a bf16 one, so
// its kernel keeps one more stage in flight per warp.
template <bool FP8>
constexpr int stages() {
  return FP8 ? 4 : 3;
}
constexpr int BLOCK_BYTES = BS * D * 2;  // 4 KB
constexpr float RESCALE_THRESHOLD = 8.0f;
constexpr float LN2 = 0.69314718055994530942f;

struct Args {
  const __nv_bfloat16* q;
  const uint8_t* k_cache;  // bf16 elements, or E4M3 codes for the FP8 kernels
  const uint8_t* v_cache;
  float k_scale, v_scale;  // FP8 only
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
  int planted;  // debug build: bounds-check site reported as failed
};

template <int G, bool FP8 = false>
struct Smem {
  uint8_t kv[WARPS][stages<FP8>()][2][FP8 ? BLOCK_BYTES / 2 : BLOCK_BYTES];  // 96 KB (bf16) / 64 KB (FP8)
  float p[WARPS][2][BS / 2][G];  // bf16 caches: probabilities, [token parity][token / 2][head]
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

// Two E4M3 codes (low byte = first element) widened exactly to fp32: every
// E4M3 value, subnormals included, is a normal fp16 value.
__device__ __forceinline__ float2 e4m3x2_to_float2(uint32_t w) {
  uint32_t h2;
  asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}" : "=r"(h2) : "r"(w));
  __half2 h;
  memcpy(&h, &h2, 4);
  return __half22float2(h);
}

// D(16x8, fp32) += A(16x16) * B(16x8), warp-level tensor-core MMA with bf16 or
// fp16 operands (two packed elements per register).
template <bool F16>
__device__ __forceinline__ void mma_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  if constexpr (F16)
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%0,%1,%2,%3};"
                 : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  else
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%0,%1,%2,%3};"
                 : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t w) {
  uint32_t h2;
  asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}" : "=r"(h2) : "r"(w));
  return h2;
}

__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t w) {
  const float2 f = bf16x2_to_float2(w);
  __half2 h = __floats2half2_rn(f.x, f.y);
  uint32_t r;
  memcpy(&r, &h, 4);
  return r;
}

// Eight cache elements of one row (this lane's head_dim chunk) as fp32 pairs.
template <bool FP8>
__device__ __forceinline__ void load_row8(const uint8_t* row, int c, bool zero, float2 (&x)[4]) {
  if constexpr (FP8) {
    uint2 r = *reinterpret_cast<const uint2*>(row + c * 8);
    if (zero) r = make_uint2(0u, 0u);
    x[0] = e4m3x2_to_float2(r.x & 0xffffu);
    x[1] = e4m3x2_to_float2(r.x >> 16);
    x[2] = e4m3x2_to_float2(r.y & 0xffffu);
    x[3] = e4m3x2_to_float2(r.y >> 16);
  } else {
    uint4 r = *reinterpret_cast<const uint4*>(row + c * 16);
    if (zero) r = make_uint4(0u, 0u, 0u, 0u);
    x[0] = bf16x2_to_float2(r.x);
    x[1] = bf16x2_to_float2(r.y);
    x[2] = bf16x2_to_float2(r.z);
    x[3] = bf16x2_to_float2(r.w);
  }
}

// Sequence length clamped to the block table's capacity (flagging a fault).
// A 32-bit or 16-byte load of an input that the host may rewrite between the
// steps of the persistent decode kernel (q, the block table, the lengths):
// there it bypasses L1 (__ldcg), which is not coherent with those writes; the
// per-launch kernels keep L1 (a block-table entry sits on the path to every
// copy, and an L1 hit keeps that short).
template <bool COHERENT, typename T>
__device__ __forceinline__ T ld_input(const T* p) {
  if constexpr (COHERENT) return __ldcg(p);
  return *p;
}

template <bool COHERENT = false>
__device__ __forceinline__ int checked_len(const Args& a, int b) {
  int L = ld_input<COHERENT>(a.seq_lens + b);
  if (L < 0 || L > a.max_blocks * BS) {
    if (a.error_flags) atomicOr(a.error_flags, ATTN_FAULT_BAD_LENGTH);
    L = L < 0 ? 0 : a.max_blocks * BS;
  }
  return L;
}

// q.k on the warp-level tensor cores. The G query heads are the rows
// of A (padded to 16 with zeros), the block's 16 tokens the columns of B (two
// n = 8 tiles), head_dim the reduction in 8 steps of 16. Inside a step, the
// reduction index that thread t holds (2t, 2t+1, 2t+8, 2t+9) is mapped to the
// physical elements 32 t + 4 step + (0, 1, 2, 3) in both A and B (a dot
// product does not depend on the order of its terms), so each thread reads
// its K row as 32 contiguous elements. Scores land with head = lane / 4 and
// tokens 8 n + 2 (lane % 4) + (0, 1): the softmax of a head runs on its 4
// lanes with shuffles.
// MMA_PV: O += P V on the tensor cores as well. P stays in
// registers (the score fragments of the two 8-token tiles form the A fragment
// of one k = 16 step), V is the B operand with head_dim permuted so that n-tile
// j, column n reads element 16 n + j: each thread then gathers its 4 token rows
// (2t, 2t+1, 2t+8, 2t+9) as 16 contiguous elements and holds the output of
// head lane / 4 for the 32 contiguous elements 32 (lane % 4) + 0..31.
// One (split, kv head, sequence) task of the split-KV decode, by one CTA of
// WARPS warps (all threads call it together; smem_raw holds Smem<G, FP8>).
// max_splits is the plan's split count: a longer sequence is cut there.
template <int G, bool FP8, bool MMA_PV, bool COHERENT = false>
__device__ __forceinline__ void split_task(const Args& a, int split, int kvh, int b, int max_splits,
                                           uint8_t* smem_raw) {
  static_assert(G == 1 || G == 2 || G == 4 || G == 8, "group size");
  constexpr int ELEM = FP8 ? 1 : 2;              // bytes per cache element
  constexpr int ROW = D * ELEM;                  // bytes per cached token row
  constexpr int CHUNKS16 = BS * ROW / (16 * 32);  // 16-byte copies per lane per block
  Smem<G, FP8>& sm = *reinterpret_cast<Smem<G, FP8>*>(smem_raw);
  constexpr int NST = stages<FP8>();

  const int warp = warp_id(), lane = lane_id();
  const int hw = lane >> 4, c = lane & 15;  // half-warp, 16-byte chunk of head_dim

  const int T = a.split_tokens;
  int L = checked_len<COHERENT>(a, b);
  if (L > max_splits * T) {  // longer than the caller's max_seq_len bound
    if (a.error_flags && split == 0 && threadIdx.x == 0) atomicOr(a.error_flags, ATTN_FAULT_BAD_LENGTH);
    L = max_splits * T;
  }
  const int n_splits = max(1, (L + T - 1) / T);
  if (split >= n_splits) return;
  const int t_begin = split * T;
  const int t_end = min(L, t_begin + T);
  const int blk_begin = t_begin / BS;
  const int blk_end = (t_end + BS - 1) / BS;
  const int32_t* table = a.block_table + (long long)b * a.max_blocks;

  // A fragments of q (head lane / 4, elements 32 (lane % 4) + 4 step + (0, 1)
  // and (2, 3)); rows past G and rows 8..15 are zero. fp16 operands for FP8
  // caches (every E4M3 value is exact in fp16), bf16 otherwise.
  uint32_t qa[8][2];
  {
    const int gq = lane >> 2, tq = lane & 3;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      uint4 r = make_uint4(0u, 0u, 0u, 0u);
      if (gq < G)
        r = ld_input<COHERENT>(reinterpret_cast<const uint4*>(a.q + ((long long)b * a.hq + kvh * G + gq) * D + 32 * tq + 8 * w));
      qa[2 * w][0] = FP8 ? bf16x2_to_f16x2(r.x) : r.x;
      qa[2 * w][1] = FP8 ? bf16x2_to_f16x2(r.y) : r.y;
      qa[2 * w + 1][0] = FP8 ? bf16x2_to_f16x2(r.z) : r.z;
      qa[2 * w + 1][1] = FP8 ? bf16x2_to_f16x2(r.w) : r.w;
    }
  }

  float2 o2[G][4];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int m = 0; m < 4; ++m) o2[g][m] = make_float2(0.f, 0.f);
  float ot[16][2];  // MMA_PV: O of head lane / 4, element 32 (lane % 4) + 16 j + nt in ot[nt][j]
#pragma unroll
  for (int nt = 0; nt < 16; ++nt) ot[nt][0] = ot[nt][1] = 0.f;
  float zpad[2] = {0.f, 0.f};  // rows 8..15 of the MMA accumulator: padding, always zero
  // Running max / sum of head g, replicated in its lanes 4g .. 4g+3.
  float m_run = -INFINITY, l_run = 0.f;

  // This warp's blocks: blk_begin + warp, + WARPS, ...
  const int n_mine = (blk_end - blk_begin - warp + WARPS - 1) / WARPS;
  auto block_of = [&](int n) { return blk_begin + warp + n * WARPS; };
  auto phys_of = [&](int blk, bool& valid) {
    if (!ATTN_IN_BOUNDS(blk >= 0 && blk < a.max_blocks, ATTN_SITE_DECODE_TABLE, a.error_flags, a.planted)) {
      valid = false;
      return -1;
    }
    const int ph = ld_input<COHERENT>(table + blk);
    valid = (ph >= 0) && (ph < a.num_blocks);
    return ph;
  };
  auto issue = [&](int n) {
    if (n < n_mine) {
      bool valid;
      const int ph = phys_of(block_of(n), valid);
      [[maybe_unused]] constexpr int SLOT = (int)sizeof(sm.kv[0][0][0]);
      if (valid && ATTN_IN_BOUNDS(warp >= 0 && warp < WARPS && n % NST >= 0 && ((CHUNKS16 - 1) * 32 + 31) * 16 + 16 <= SLOT,
                                  ATTN_SITE_DECODE_SMEM, a.error_flags, a.planted)) {
        const long long off = ((long long)ph * a.hkv + kvh) * (BS * ROW);  // bytes
        const uint8_t* ksrc = a.k_cache + off;
        const uint8_t* vsrc = a.v_cache + off;
        uint8_t* kdst = sm.kv[warp][n % NST][0];
        uint8_t* vdst = sm.kv[warp][n % NST][1];
#pragma unroll
        for (int i = 0; i < CHUNKS16; ++i) cp_async16(kdst + (i * 32 + lane) * 16, ksrc + (i * 32 + lane) * 16);
#pragma unroll
        for (int i = 0; i < CHUNKS16; ++i) cp_async16(vdst + (i * 32 + lane) * 16, vsrc + (i * 32 + lane) * 16);
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

    // ---- S = q K^T on the tensor cores, then the online softmax per head on its 4 lanes
    const int gq = lane >> 2, tq = lane & 3;
    float cacc[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
      for (int j = 0; j < 4; ++j) cacc[nt][j] = 0.f;
      const uint8_t* krow = kblk + (8 * nt + gq) * ROW + 32 * tq * ELEM;
      uint32_t kw[8 * ELEM];  // this thread's 32 elements of the token row
#pragma unroll
      for (int v4 = 0; v4 < 2 * ELEM; ++v4) {
        const uint4 r = *reinterpret_cast<const uint4*>(krow + 16 * v4);
        kw[4 * v4 + 0] = r.x;
        kw[4 * v4 + 1] = r.y;
        kw[4 * v4 + 2] = r.z;
        kw[4 * v4 + 3] = r.w;
      }
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        uint32_t b0, b1;
        if constexpr (FP8) {
          b0 = e4m3x2_to_f16x2(kw[ks] & 0xffffu);
          b1 = e4m3x2_to_f16x2(kw[ks] >> 16);
        } else {
          b0 = kw[2 * ks];
          b1 = kw[2 * ks + 1];
        }
        mma_16816<FP8>(cacc[nt], qa[ks][0], 0u, qa[ks][1], 0u, b0, b1);
      }
    }
    const float sl2 = FP8 ? a.scale_log2 * a.k_scale : a.scale_log2;  // cached key = code * k_scale
    float sc[4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int tk = 8 * nt + 2 * tq + j;
        sc[2 * nt + j] = (tk < n_valid) ? cacc[nt][j] * sl2 : -INFINITY;
      }
    float bm = fmaxf(fmaxf(sc[0], sc[1]), fmaxf(sc[2], sc[3]));
    bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 1));
    bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 2));
    const float m_new = fmaxf(m_run, bm);
    const bool upd = (m_new - m_run) > RESCALE_THRESHOLD;
    const float alpha = upd ? ex2_approx(m_run - m_new) : 1.f;
    if (upd) m_run = m_new;
    const float mo = (m_run == -INFINITY) ? 0.f : m_run;
    float pr[4], rs = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      pr[j] = ex2_approx(sc[j] - mo);
      rs += pr[j];
    }
    rs += __shfl_xor_sync(0xffffffffu, rs, 1);
    rs += __shfl_xor_sync(0xffffffffu, rs, 2);
    l_run = l_run * alpha + rs;
    if constexpr (MMA_PV) {
      if (alpha != 1.f) {
#pragma unroll
        for (int nt = 0; nt < 16; ++nt) {
          ot[nt][0] *= alpha;
          ot[nt][1] *= alpha;
        }
      }
      // A = P (head gq, tokens 2t, 2t+1 | 8+2t, 8+2t+1); padding heads are zero.
      uint32_t pa0 = 0u, pa2 = 0u;
      if (gq < G) {
        if constexpr (FP8) {
          __half2 h0 = __floats2half2_rn(pr[0], pr[1]), h2 = __floats2half2_rn(pr[2], pr[3]);
          memcpy(&pa0, &h0, 4);
          memcpy(&pa2, &h2, 4);
        } else {
          pa0 = pack_bf16x2(pr[0], pr[1]);
          pa2 = pack_bf16x2(pr[2], pr[3]);
        }
      }
      // B = V: rows 2t, 2t+1, 2t+8, 2t+9 (masked rows read as zero), elements 16 gq .. 16 gq + 15.
      constexpr int WPR = 4 * ELEM;  // 32-bit words per 16-element row slice
      uint32_t vr[4][WPR];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int tk = 2 * tq + (r & 1) + 8 * (r >> 1);
        const bool keep = tk < n_valid;
#pragma unroll
        for (int v4 = 0; v4 < ELEM; ++v4) {
          uint4 x = *reinterpret_cast<const uint4*>(vblk + tk * ROW + 16 * gq * ELEM + 16 * v4);
          if (!keep) x = make_uint4(0u, 0u, 0u, 0u);
          vr[r][4 * v4 + 0] = x.x;
          vr[r][4 * v4 + 1] = x.y;
          vr[r][4 * v4 + 2] = x.z;
          vr[r][4 * v4 + 3] = x.w;
        }
      }
#pragma unroll
      for (int nt = 0; nt < 16; ++nt) {
        uint32_t b0, b1;
        if constexpr (FP8) {  // byte nt of the two rows -> one E4M3 pair -> fp16 pair
          const int w = nt >> 2, j = nt & 3;
          const uint32_t sel = (uint32_t)(j | ((j + 4) << 4));
          b0 = e4m3x2_to_f16x2(__byte_perm(vr[0][w], vr[1][w], sel));
          b1 = e4m3x2_to_f16x2(__byte_perm(vr[2][w], vr[3][w], sel));
        } else {  // half nt of the two rows -> one bf16 pair
          const int w = nt >> 1;
          const uint32_t sel = (nt & 1) ? 0x7632u : 0x5410u;
          b0 = __byte_perm(vr[0][w], vr[1][w], sel);
          b1 = __byte_perm(vr[2][w], vr[3][w], sel);
        }
        float acc[4] = {ot[nt][0], ot[nt][1], zpad[0], zpad[1]};
        mma_16816<FP8>(acc, pa0, 0u, pa2, 0u, b0, b1);
        ot[nt][0] = acc[0];
        ot[nt][1] = acc[1];
      }
    } else {
      if (gq < G) {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int tk = 8 * nt + 2 * tq + j;
            sm.p[warp][tk & 1][tk >> 1][gq] = pr[2 * nt + j];
          }
        if (tq == 0) sm.alpha[warp][gq] = alpha;
      }
      __syncwarp();
    }

    // ---- O += p * v (CUDA cores)
    if constexpr (!MMA_PV) {
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
        float2 vx[4];
        load_row8<FP8>(vblk + tk * ROW, c, !full && tk >= n_valid, vx);  // never multiply masked values in
        const float2 v0 = vx[0], v1 = vx[1], v2 = vx[2], v3 = vx[3];
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
  if constexpr (FP8) {  // cached value = code * v_scale: applied to O once
    const float2 vs = make_float2(a.v_scale, a.v_scale);
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int m = 0; m < 4; ++m) o2[g][m] = __fmul2_rn(o2[g][m], vs);
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
      ot[nt][0] *= a.v_scale;
      ot[nt][1] *= a.v_scale;
    }
  }

  // ---- merge the two half-warps (disjoint tokens, same running max)
  if constexpr (!MMA_PV) {
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        o2[g][m].x += __shfl_xor_sync(0xffffffffu, o2[g][m].x, 16);
        o2[g][m].y += __shfl_xor_sync(0xffffffffu, o2[g][m].y, 16);
      }
  }
  __syncthreads();  // the KV ring is reused for the merge
  MergeSmem<G>& mg = *reinterpret_cast<MergeSmem<G>*>(smem_raw);
  if ((lane & 3) == 0 && (lane >> 2) < G) {
    mg.m[warp][lane >> 2] = m_run;
    mg.l[warp][lane >> 2] = l_run;
  }
  if constexpr (MMA_PV) {
    if ((lane >> 2) < G) {
      float* dst = &mg.o[warp][lane >> 2][32 * (lane & 3)];
#pragma unroll
      for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4)
          *reinterpret_cast<float4*>(dst + 16 * j + 4 * q4) =
              make_float4(ot[4 * q4][j], ot[4 * q4 + 1][j], ot[4 * q4 + 2][j], ot[4 * q4 + 3][j]);
    }
  } else if (hw == 0) {
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
      if (ATTN_IN_BOUNDS(split >= 0 && split < max_splits && row >= 0 && row < rows, ATTN_SITE_DECODE_PARTIAL,
                         a.error_flags, a.planted)) {
        a.part_o[((long long)split * rows + row) * D + d] = out;
        if (d == 0) a.part_lse[(long long)split * rows + row] = lse;
      }
    }
  }
}

template <int G, bool FP8, bool MMA_PV>
__global__ void __launch_bounds__(WARPS * 32)
    decode_split_kernel(const Args a) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  split_task<G, FP8, MMA_PV>(a, blockIdx.x, blockIdx.y, blockIdx.z, gridDim.x, smem_raw);
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
__device__ __forceinline__ void combine_row(int row, const float* __restrict__ part_o,
                                            const float* __restrict__ part_lse, int num_splits, int rows,
                                            const int32_t* __restrict__ splits_per_row,
                                            const int32_t* __restrict__ seq_lens, int split_tokens, int max_len,
                                            int rows_per_seq, void* out_o, int out_f32, float* out_lse,
                                            int32_t* flags = nullptr, int planted = 0) {
  constexpr int PER = HD / 32;  // floats per lane
  const int lane = lane_id();
  int n;
  if (splits_per_row) {  // standalone call with per-row counts
    n = min(max(__ldcg(splits_per_row + row), 0), num_splits);
  } else if (seq_lens == nullptr) {  // standalone call: every row has num_splits partials
    n = num_splits;
  } else {  // decode path
    int L = __ldcg(seq_lens + row / rows_per_seq);
    L = min(max(L, 0), max_len);
    n = max(1, (L + split_tokens - 1) / split_tokens);
    if (n == 1) return;
    n = min(n, num_splits);
  }
  constexpr float LOG2E = 1.4426950408889634f;
  // max and sum of exp over the splits, lanes strided over s
  float M = -INFINITY;
  for (int s = lane; s < n; s += 32) M = fmaxf(M, __ldcg(part_lse + (long long)s * rows + row));
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  float out[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) out[i] = 0.f;
  float lse = -INFINITY;
  if (M != -INFINITY) {
    float sum = 0.f;
    for (int s = lane; s < n; s += 32) sum += ex2_approx((__ldcg(part_lse + (long long)s * rows + row) - M) * LOG2E);
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    lse = M + logf(sum);
    for (int s = 0; s < n; ++s) {
      if (!ATTN_IN_BOUNDS(s < num_splits, ATTN_SITE_COMBINE, flags, planted)) break;
      const float ls = __ldcg(part_lse + (long long)s * rows + row);
      if (ls == -INFINITY) continue;  // weight 0: its partial is not read
      const float wgt = ex2_approx((ls - lse) * LOG2E);
      const float* src = part_o + ((long long)s * rows + row) * HD + lane * PER;
      if constexpr (PER == 4) {
        const float4 x = __ldcg(reinterpret_cast<const float4*>(src));
        out[0] = fmaf(wgt, x.x, out[0]);
        out[1] = fmaf(wgt, x.y, out[1]);
        out[2] = fmaf(wgt, x.z, out[2]);
        out[3] = fmaf(wgt, x.w, out[3]);
      } else {
        const float2 x = __ldcg(reinterpret_cast<const float2*>(src));
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

template <int HD>
__global__ void __launch_bounds__(256) lse_combine_kernel(const float* __restrict__ part_o,
                                                          const float* __restrict__ part_lse, int num_splits,
                                                          int rows, const int32_t* __restrict__ splits_per_row,
                                                          const int32_t* __restrict__ seq_lens, int split_tokens,
                                                          int max_len, int rows_per_seq, void* out_o, int out_f32,
                                                          float* out_lse, int32_t* flags, int planted) {
  const int row = blockIdx.x * (blockDim.x / 32) + warp_id();
  if (row >= rows) return;
  combine_row<HD>(row, part_o, part_lse, num_splits, rows, splits_per_row, seq_lens, split_tokens, max_len,
                  rows_per_seq, out_o, out_f32, out_lse, flags, planted);
}

}  // namespace combine

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
static int env_int(const char* name, int dflt) {
  const char* e = getenv(name);
  return (e && *e) ? atoi(e) : dflt;
}

namespace decode {

// Tokens per split (a multiple of 64) and the number of splits a sequence of
// max_len keys is cut into. num_splits > 0 fixes the count; forced > 0 fixes
// the tokens; otherwise enough CTAs for many waves (good balance across
// sequences of mixed lengths) while each split still streams at least 512
// tokens. The same arithmetic runs on the host (attn_decode_paged) and in the
// persistent decode kernel, so both cut a step identically.
__host__ __device__ inline void split_plan(int batch, int hkv, int max_len, int num_splits, int sm_count, int forced,
                                           int* split_tokens, int* max_splits) {
  const int unit = BS * WARPS;  // 64 tokens
  int T;
  if (forced > 0) {
    T = forced;
  } else if (num_splits > 0) {
    T = (max_len + num_splits - 1) / num_splits;
  } else {
    const long long pairs = (long long)batch * hkv;
    const long long target = 32LL * sm_count;
    long long per_seq = pairs > 0 ? (target + pairs - 1) / pairs : 1;
    if (per_seq < 1) per_seq = 1;
    T = (int)((max_len + per_seq - 1) / per_seq);
    if (T < 512) T = 512;
  }
  T = ((T + unit - 1) / unit) * unit;
  if (T <= 0) T = unit;
  int n = max_len > 0 ? (max_len + T - 1) / T : 1;
  *split_tokens = T;
  *max_splits = n < 1 ? 1 : n;
}

// Bytes of the partials (O then LSE, each 256-byte aligned) for a plan.
__host__ __device__ inline size_t partial_bytes(int max_splits, size_t rows, int head_dim, size_t* lse_offset) {
  if (max_splits <= 1) {
    if (lse_offset) *lse_offset = 0;
    return 0;
  }
  const size_t po = (size_t)max_splits * rows * head_dim * sizeof(float);
  const size_t pl = (size_t)max_splits * rows * sizeof(float);
  if (lse_offset) *lse_offset = ((po + 255) / 256) * 256;
  return ((po + 255) / 256) * 256 + ((pl + 255) / 256) * 256;
}

}  // namespace decode

DecodePlan plan_decode(const attn_decode_params& p) {
  DecodePlan plan;
  const int cap = p.max_blocks_per_seq * decode::BS;
  const int max_len = (p.max_seq_len > 0 && p.max_seq_len < cap) ? p.max_seq_len : cap;
  decode::split_plan(p.batch, p.num_kv_heads, max_len, p.num_splits, device_sm_count(),
                     env_int("ATTN_DECODE_SPLIT_TOKENS", 0), &plan.split_tokens, &plan.max_splits);
  plan.workspace_bytes =
      decode::partial_bytes(plan.max_splits, (size_t)p.batch * p.num_q_heads, p.head_dim, nullptr);
  return plan;
}

// The split kernel's one-time set-up (its shared-memory attribute), once per device.
template <int G, bool FP8>
static attn_status_t setup_decode_g() {
  auto kern = decode::decode_split_kernel<G, FP8, FP8>;  // P V on the tensor cores for FP8 caches
  const int smem = (int)sizeof(decode::Smem<G, FP8>);
  static DeviceOnce setup;
  return setup.run([&]() -> attn_status_t {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) {
      cudaGetLastError();
      return ATTN_ERR_CUDA;
    }
    return ATTN_OK;
  });
}

attn_status_t prepare_decode(const attn_decode_params& p) {
  const bool fp8 = p.kv_dtype == ATTN_DTYPE_FP8_E4M3;
  switch (p.num_q_heads / p.num_kv_heads) {
    case 1: return fp8 ? setup_decode_g<1, true>() : setup_decode_g<1, false>();
    case 2: return fp8 ? setup_decode_g<2, true>() : setup_decode_g<2, false>();
    case 4: return fp8 ? setup_decode_g<4, true>() : setup_decode_g<4, false>();
    case 8: return fp8 ? setup_decode_g<8, true>() : setup_decode_g<8, false>();
    default: return ATTN_ERR_UNSUPPORTED;
  }
}

template <int G, bool FP8>
static attn_status_t launch_decode_g(const decode::Args& a, const DecodePlan& plan, cudaStream_t stream) {
  auto kern = decode::decode_split_kernel<G, FP8, FP8>;  // P V on the tensor cores for FP8 caches
  const int smem = (int)sizeof(decode::Smem<G, FP8>);
  static_assert(sizeof(decode::MergeSmem<G>) <= sizeof(decode::Smem<G, FP8>), "merge buffer fits");
  const attn_status_t st = setup_decode_g<G, FP8>();
  if (st != ATTN_OK) return st;
  dim3 grid(plan.max_splits, a.hkv, a.batch);
  kern<<<grid, decode::WARPS * 32, smem, stream>>>(a);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

attn_status_t launch_decode(const attn_decode_params& p, const DecodePlan& plan, void* workspace,
                            cudaStream_t stream, bool combine) {
  if (p.batch == 0) return ATTN_OK;
  decode::Args a;
  a.q = reinterpret_cast<const __nv_bfloat16*>(p.q);
  a.k_cache = reinterpret_cast<const uint8_t*>(p.k_cache);
  a.v_cache = reinterpret_cast<const uint8_t*>(p.v_cache);
  const bool fp8 = p.kv_dtype == ATTN_DTYPE_FP8_E4M3;
  a.k_scale = fp8 ? p.k_scale : 1.f;
  a.v_scale = fp8 ? p.v_scale : 1.f;
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
  a.planted = planted_bounds_site();
  attn_status_t st;
  switch (p.num_q_heads / p.num_kv_heads) {
    case 1: st = fp8 ? launch_decode_g<1, true>(a, plan, stream) : launch_decode_g<1, false>(a, plan, stream); break;
    case 2: st = fp8 ? launch_decode_g<2, true>(a, plan, stream) : launch_decode_g<2, false>(a, plan, stream); break;
    case 4: st = fp8 ? launch_decode_g<4, true>(a, plan, stream) : launch_decode_g<4, false>(a, plan, stream); break;
    case 8: st = fp8 ? launch_decode_g<8, true>(a, plan, stream) : launch_decode_g<8, false>(a, plan, stream); break;
    default: return ATTN_ERR_UNSUPPORTED;
  }
  if (st != ATTN_OK || plan.max_splits <= 1 || !combine) return st;
  return launch_combine(a.part_o, a.part_lse, plan.max_splits, (int)rows, p.head_dim, nullptr, p.seq_lens,
                        plan.split_tokens, p.num_q_heads, p.o, p.o_dtype, p.lse, stream, p.error_flags);
}

attn_status_t launch_combine(const float* part_o, const float* part_lse, int num_splits, int rows, int head_dim,
                             const int32_t* splits_per_row, const int32_t* seq_lens, int split_tokens,
                             int rows_per_seq, void* out_o, attn_dtype_t out_dtype, float* out_lse,
                             cudaStream_t stream, int32_t* error_flags) {
  if (rows == 0) return ATTN_OK;
  const int planted = planted_bounds_site();
  const int warps = 8;
  const int grid = (rows + warps - 1) / warps;
  const int max_len = num_splits * split_tokens;
  if (head_dim == 128)
    combine::lse_combine_kernel<128><<<grid, warps * 32, 0, stream>>>(
        part_o, part_lse, num_splits, rows, splits_per_row, seq_lens, split_tokens, max_len, rows_per_seq, out_o,
        out_dtype == ATTN_DTYPE_F32, out_lse, error_flags, planted);
  else
    combine::lse_combine_kernel<64><<<grid, warps * 32, 0, stream>>>(
        part_o, part_lse, num_splits, rows, splits_per_row, seq_lens, split_tokens, max_len, rows_per_seq, out_o,
        out_dtype == ATTN_DTYPE_F32, out_lse, error_flags, planted);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Persistent decode: one resident kernel runs a stream of decode steps over
// static buffers, commanded from the host through a block of host memory that
// is mapped into the device ("GPU Kernel 调度:大模型推理的拐点 2026", Persistent
// Kernel section: a resident kernel pulls work instead of paying a launch per
// step). A step is the same computation as attn_decode_paged: the same split
// plan, the same split task per (split, kv head, sequence) and the same
// log-sum-exp combine, so its results are bit for bit those of a launch.
//
//   * CTA 0 polls the command block (system-scope acquire loads) for the next
//     step number, or a stop request, and posts the step's batch and length
//     bound in a mailbox in device memory; the other CTAs wait on the mailbox.
//   * every CTA takes (split, kv head, sequence) tasks in turn; the CTA whose
//     split is the last one of its (sequence, kv head) to finish merges that
//     group's partials (a per-group counter, no grid-wide barrier).
//   * the last CTA to finish the step writes its number back to the command
//     block (system-scope release).
//   * every wait is bounded: with no command for idle_limit cycles (or, for the
//     other CTAs, no mailbox post for idle_limit + wait_limit) the kernel exits,
//     raising ATTN_FAULT_TIMEOUT in the command block's status and error_flags.
// ---------------------------------------------------------------------------
namespace decode {

// Words of the command block (attn_persistent_cmd) and of the mailbox.
enum { CMD_SEQ = 0, CMD_BATCH, CMD_MAXLEN, CMD_STOP, CMD_DONE, CMD_STATUS, CMD_RUNNING };
enum { MB_STEP = 0, MB_BATCH, MB_MAXLEN, MB_STATE, MB_DONE_CTAS, MB_COUNTERS = 8 };
enum { ST_WAIT = 0, ST_RUN, ST_STOP, ST_IDLE };

struct PersistArgs {
  Args base;           // static buffers; batch, split_tokens and the partials are set per step
  int* cmd;            // device address of the host command block
  float* partials;     // workspace: the partials of the largest step
  int* sync;           // workspace: mailbox, finished-CTA count, per-(sequence, kv head) counters
  int max_batch, cap_len, num_splits, sm_count, forced;
  long long idle_limit, wait_limit;
};

__device__ __forceinline__ int ld_acquire_sys(const int* p) {
  int v;
  asm volatile("ld.acquire.sys.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_sys(int* p, int v) {
  asm volatile("st.release.sys.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_gpu(int* p, int v) {
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

template <int G, bool FP8>
__global__ void __launch_bounds__(WARPS * 32) decode_persistent_kernel(const PersistArgs pa) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  __shared__ int s_state, s_batch, s_maxlen, s_last;
  int* const cmd = pa.cmd;
  int* const sync = pa.sync;
  const int hkv = pa.base.hkv, hq = pa.base.hq;
  if (blockIdx.x == 0 && threadIdx.x == 0) st_release_sys(cmd + CMD_RUNNING, 1);
  for (int step = 1;; ++step) {
    // ---- the step's command
    if (threadIdx.x == 0) {
      int state = ST_WAIT, batch = 0, maxlen = 0;
      const long long t0 = clock64();
      if (blockIdx.x == 0) {
        while (state == ST_WAIT) {
          if (ld_acquire_sys(cmd + CMD_SEQ) >= step) {
            state = ST_RUN;
            batch = ld_acquire_sys(cmd + CMD_BATCH);
            maxlen = ld_acquire_sys(cmd + CMD_MAXLEN);
          } else if (ld_acquire_sys(cmd + CMD_STOP)) {
            state = ST_STOP;
          } else if (clock64() - t0 > pa.idle_limit) {
            state = ST_IDLE;
          } else {
            __nanosleep(256);
          }
        }
        sync[MB_BATCH] = batch;
        sync[MB_MAXLEN] = maxlen;
        sync[MB_STATE] = state;
        st_release_gpu(sync + MB_STEP, step);
      } else {
        while (ld_acquire_gpu(sync + MB_STEP) < step) {
          if (clock64() - t0 > pa.idle_limit + pa.wait_limit) {
            state = ST_IDLE;
            break;
          }
          __nanosleep(256);
        }
        if (state == ST_WAIT) {
          state = ld_acquire_gpu(sync + MB_STATE);
          batch = ld_acquire_gpu(sync + MB_BATCH);
          maxlen = ld_acquire_gpu(sync + MB_MAXLEN);
        }
      }
      s_state = state;
      s_batch = batch;
      s_maxlen = maxlen;
    }
    __syncthreads();
    if (s_state != ST_RUN) {
      if (threadIdx.x == 0 && s_state == ST_IDLE) {
        atomicOr(cmd + CMD_STATUS, ATTN_FAULT_TIMEOUT);
        if (pa.base.error_flags) atomicOr(pa.base.error_flags, ATTN_FAULT_TIMEOUT);
      }
      if (blockIdx.x == 0 && threadIdx.x == 0) {
        __threadfence_system();
        st_release_sys(cmd + CMD_RUNNING, 0);
      }
      break;
    }
    // ---- the step: the split plan of attn_decode_paged for this batch and bound
    int batch = s_batch, maxlen = s_maxlen;
    if (batch < 0 || batch > pa.max_batch) {
      if (threadIdx.x == 0 && blockIdx.x == 0 && pa.base.error_flags)
        atomicOr(pa.base.error_flags, ATTN_FAULT_BAD_LENGTH);
      batch = batch < 0 ? 0 : pa.max_batch;
    }
    if (maxlen <= 0 || maxlen > pa.cap_len) maxlen = pa.cap_len;
    int T, nsplit;
    split_plan(batch, hkv, maxlen, pa.num_splits, pa.sm_count, pa.forced, &T, &nsplit);
    Args a = pa.base;
    a.batch = batch;
    a.split_tokens = T;
    size_t lse_off = 0;
    partial_bytes(nsplit, (size_t)batch * hq, D, &lse_off);
    a.part_o = pa.partials;
    a.part_lse = nsplit > 1 ? reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(pa.partials) + lse_off) : nullptr;
    const int tasks = nsplit * hkv * batch;
    for (int t = blockIdx.x; t < tasks; t += gridDim.x) {
      const int split = t % nsplit, r = t / nsplit, kvh = r % hkv, b = r / hkv;
      split_task<G, FP8, FP8, true>(a, split, kvh, b, nsplit, smem_raw);
      __syncthreads();  // shared memory is refilled by the next task
      if (nsplit == 1) continue;
      int L = __ldcg(a.seq_lens + b);  // clamped exactly as split_task clamps it
      L = L < 0 ? 0 : (L > a.max_blocks * BS ? a.max_blocks * BS : L);
      if (L > nsplit * T) L = nsplit * T;
      const int n = max(1, (L + T - 1) / T);
      if (n == 1 || split >= n) continue;  // O written directly, or an empty split
      if (threadIdx.x == 0) {
        __threadfence();  // this split's partial, before its arrival
        s_last = atomicAdd(sync + MB_COUNTERS + b * hkv + kvh, 1) == n - 1;
      }
      __syncthreads();
      if (s_last) {  // every split of (b, kvh) has arrived: merge its G rows
        __threadfence();
        for (int g = warp_id(); g < G; g += WARPS)
          combine::combine_row<D>((b * hq) + kvh * G + g, a.part_o, a.part_lse, nsplit, batch * hq, nullptr,
                                  a.seq_lens, T, nsplit * T, hq, a.o, a.o_f32, a.lse, a.error_flags, a.planted);
        if (threadIdx.x == 0) sync[MB_COUNTERS + b * hkv + kvh] = 0;  // ready for the next step
      }
      __syncthreads();
    }
    // ---- the last CTA out reports the step
    if (threadIdx.x == 0) {
      __threadfence();
      if (atomicAdd(sync + MB_DONE_CTAS, 1) == (int)gridDim.x - 1) {
        sync[MB_DONE_CTAS] = 0;
        __threadfence_system();
        st_release_sys(cmd + CMD_DONE, step);
      }
    }
  }
}

}  // namespace decode

// Workspace of the persistent decode: the partials of the largest step (any
// batch up to p.batch at the length bound), then the mailbox and counters.
static void persistent_layout(const attn_decode_params& p, int cap_len, size_t* sync_off, size_t* total) {
  size_t part = 0;
  const int sms = device_sm_count();
  const int forced = env_int("ATTN_DECODE_SPLIT_TOKENS", 0);
  for (int b = 1; b <= p.batch; ++b) {
    int T, n;
    decode::split_plan(b, p.num_kv_heads, cap_len, p.num_splits, sms, forced, &T, &n);
    const size_t need = decode::partial_bytes(n, (size_t)b * p.num_q_heads, p.head_dim, nullptr);
    if (need > part) part = need;
  }
  *sync_off = (part + 255) / 256 * 256;
  const size_t words = decode::MB_COUNTERS + (size_t)p.batch * p.num_kv_heads;
  *total = *sync_off + (words * sizeof(int) + 255) / 256 * 256;
}

static int persistent_cap_len(const attn_decode_params& p) {
  const int cap = p.max_blocks_per_seq * decode::BS;
  return (p.max_seq_len > 0 && p.max_seq_len < cap) ? p.max_seq_len : cap;
}

size_t decode_persistent_workspace_bytes(const attn_decode_params& p) {
  size_t off, total;
  persistent_layout(p, persistent_cap_len(p), &off, &total);
  return total;
}

template <int G, bool FP8>
static attn_status_t launch_persistent_g(const decode::PersistArgs& pa, cudaStream_t stream) {
  auto kern = decode::decode_persistent_kernel<G, FP8>;
  const int smem = (int)sizeof(decode::Smem<G, FP8>);
  static DeviceOnce setup;  // the shared-memory attribute, once per device
  attn_status_t st = setup.run([&]() -> attn_status_t {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) {
      cudaGetLastError();
      return ATTN_ERR_CUDA;
    }
    return ATTN_OK;
  });
  if (st != ATTN_OK) return st;
  // Every CTA must be resident at once (CTAs wait on CTA 0's mailbox): a
  // cooperative launch of as many CTAs as fit.
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, decode::WARPS * 32, smem) != cudaSuccess ||
      per_sm < 1) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  const int grid = per_sm * pa.sm_count;
  void* args[] = {const_cast<decode::PersistArgs*>(&pa)};
  if (cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(kern), dim3(grid), dim3(decode::WARPS * 32), args,
                                  smem, stream) != cudaSuccess) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  return ATTN_OK;
}

attn_status_t launch_decode_persistent(const attn_decode_params& p, int32_t* cmd_dev, void* workspace,
                                       long long idle_cycles, cudaStream_t stream) {
  const int cap_len = persistent_cap_len(p);
  size_t sync_off, total;
  persistent_layout(p, cap_len, &sync_off, &total);
  int* sync = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(workspace) + sync_off);
  if (cudaMemsetAsync(sync, 0, total - sync_off, stream) != cudaSuccess) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  decode::PersistArgs pa;
  memset(&pa, 0, sizeof(pa));
  decode::Args& a = pa.base;
  a.q = reinterpret_cast<const __nv_bfloat16*>(p.q);
  a.k_cache = reinterpret_cast<const uint8_t*>(p.k_cache);
  a.v_cache = reinterpret_cast<const uint8_t*>(p.v_cache);
  const bool fp8 = p.kv_dtype == ATTN_DTYPE_FP8_E4M3;
  a.k_scale = fp8 ? p.k_scale : 1.f;
  a.v_scale = fp8 ? p.v_scale : 1.f;
  a.block_table = p.block_table;
  a.seq_lens = p.seq_lens;
  a.o = p.o;
  a.lse = p.lse;
  a.o_f32 = p.o_dtype == ATTN_DTYPE_F32;
  a.hq = p.num_q_heads;
  a.hkv = p.num_kv_heads;
  a.max_blocks = p.max_blocks_per_seq;
  a.num_blocks = p.num_blocks;
  a.scale_log2 = p.scale * 1.4426950408889634f;
  a.error_flags = p.error_flags;
  a.planted = planted_bounds_site();
  pa.cmd = cmd_dev;
  pa.partials = reinterpret_cast<float*>(workspace);
  pa.sync = sync;
  pa.max_batch = p.batch;
  pa.cap_len = cap_len;
  pa.num_splits = p.num_splits;
  pa.sm_count = device_sm_count();
  pa.forced = env_int("ATTN_DECODE_SPLIT_TOKENS", 0);
  pa.idle_limit = idle_cycles;
  pa.wait_limit = 2000000000LL;
  switch (p.num_q_heads / p.num_kv_heads) {
    case 1: return fp8 ? launch_persistent_g<1, true>(pa, stream) : launch_persistent_g<1, false>(pa, stream);
    case 2: return fp8 ? launch_persistent_g<2, true>(pa, stream) : launch_persistent_g<2, false>(pa, stream);
    case 4: return fp8 ? launch_persistent_g<4, true>(pa, stream) : launch_persistent_g<4, false>(pa, stream);
    case 8: return fp8 ? launch_persistent_g<8, true>(pa, stream) : launch_persistent_g<8, false>(pa, stream);
    default: return ATTN_ERR_UNSUPPORTED;
  }
}

}  // namespace attn
