// Projection GEMMs of the block stack on the 5th-generation tensor cores.
//
//   out = epilogue(A @ W^T),  A [M, K] bf16 (activations), W [N, K] bf16 (weights)
//
// "从文本到聊天模型" §5.4 (c_q/c_k/c_v), §5.3 (residual add of c_proj), §5.7
// (c_fc + relu^2, c_proj), §5.8 (lm_head, cross-entropy); soft-cap from
// "Nanochat与nanoGPT对比：关键升级" §1.
//
// Design (one CTA per SM, persistent over output tiles):
//   warp 0      TMA producer: 128x64 A and 256x64 W tiles, 128-byte swizzle,
//               into a 4-stage shared-memory ring (48 KB per stage);
//   warp 1      allocates 512 TMEM columns; one thread issues
//               tcgen05.mma.cta_group::1.kind::f16 (M=128, N=256, K=16) into one of
//               two 256-column fp32 accumulators and commits stage releases;
//   CTA pairs   (16-bit K-major operands, M > 128): a cluster of two CTAs
//               computes 256x256 tiles with tcgen05.mma.cta_group::2 (M=256).
//               Each CTA loads its own 128 rows of A and 128 of the 256 W rows
//               (6 stages of 32 KB), both halves signalling rank 0's barrier;
//               rank 0 issues the MMAs and commits to the barriers of both
//               CTAs; each CTA's tensor memory receives its 128 rows x 256
//               columns, and its epilogue warps hand the accumulator back to
//               rank 0.  Every W byte loaded into shared memory then serves
//               256 rows instead of 128.
//   warps 2..9  epilogue: tcgen05.ld of the accumulator (a warp may only read
//               the 32 TMEM lanes = tile rows its warp index mod 4 selects, so
//               two warps share each lane quarter and split the 256 columns),
//               fused epilogue op; results are staged per warp in a 4 KB
//               swizzled shared-memory tile and written by a TMA tensor store
//               (a TMA reduce-add for the fp32 residual); then hand the
//               accumulator back.
// e4m3 operands (dynamic tensorwise FP8, "Nanochat与nanoGPT对比" §1 table, FP8
// row): the same pipeline with tcgen05.mma kind::f8f6f4.  A 128-byte swizzle
// row then holds 128 elements instead of 64, so a stage covers K = 128 with the
// same byte layout, descriptors and four MMAs (K = 32 each); the epilogue
// scales the fp32 accumulator by 1 / (s_a s_w) before its fused op.
// Tiles are visited with the N index fastest so consecutive CTAs share one A
// row-block and the weight matrix stays resident in L2.
// Every mbarrier wait is bounded; on timeout the CTA records NC_DEV_TIMEOUT,
// drains its in-flight copies and MMAs, frees its tensor memory and exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "nc_half.cuh"
#include "nc_internal.h"
#include "nc_ptx.cuh"

namespace nc {
namespace gemm {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;  // one 128-byte swizzle row of bf16
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BN * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int NUM_ACC = 2;
constexpr int TMEM_COLS = 512;  // NUM_ACC * BN
constexpr int EPI_WARPS = 8;  // two per TMEM lane quarter, each owning half the columns
constexpr int NUM_THREADS = 64 + 32 * EPI_WARPS;
constexpr int EPI_COLS = BN / 2;  // columns per epilogue warp
constexpr int STG_BYTES = 32 * 128;  // per epilogue warp: 32 rows x 128 B staging tile
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + EPI_WARPS * STG_BYTES + 1024 /*align*/ +
                           256 /*barriers*/;
constexpr uint32_t IDESC_BF16 = idesc_f32acc(BM, BN, false);
constexpr uint32_t IDESC_F16 = idesc_f32acc(BM, BN, true);
// CTA pairs (16-bit K-major operands): one MMA of M = 256 rows over two SMs.
// Each CTA loads its 128 rows of A and 128 of the tile's 256 rows of W, so a
// stage is 32 KB and the same ring space holds six of them; each CTA's tensor
// memory receives the full 256 columns of its own 128 rows.
constexpr int PAIR_STAGES = 6;
constexpr int PAIR_B_BYTES = (BN / 2) * BK * 2;
constexpr int PAIR_STAGE_BYTES = A_BYTES + PAIR_B_BYTES;
static_assert(PAIR_STAGES * PAIR_STAGE_BYTES <= STAGES * STAGE_BYTES, "pair ring fits the tile ring");
constexpr int MAX_STAGES = PAIR_STAGES > STAGES ? PAIR_STAGES : STAGES;
constexpr uint32_t IDESC_PAIR_BF16 = idesc_f32acc(2 * BM, BN, false);
constexpr uint32_t IDESC_PAIR_F16 = idesc_f32acc(2 * BM, BN, true);
constexpr uint32_t IDESC_E4M3 = idesc_e4m3_f32acc(BM, BN);

// Dequantisation factors of an e4m3 product, 1 / (s_a s_w), for the q, k and v
// column ranges of the QKV projection (all three equal elsewhere).
struct Dq {
  float q, k, v;
};

__device__ __forceinline__ void scale32(uint32_t (&r)[32], float f) {
#pragma unroll
  for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * f);
}

struct Smem {  // barrier block placed after the tile ring and the staging tiles
  uint64_t full[MAX_STAGES];
  uint64_t empty[MAX_STAGES];
  uint64_t tmem_full[NUM_ACC];
  uint64_t tmem_empty[NUM_ACC];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(Smem) <= 256, "barrier block");

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Soft-cap l = cap * tanh(z / cap) written as cap - 2 cap / (1 + e^(2z/cap)),
// plus p = exp(l - cap) = exp(-2 cap / (1 + e^(2z/cap))): three MUFU operations
// per logit.  The limits are exact (z -> +inf: l = cap; z -> -inf: l = -cap).
struct SoftCap {
  float k_in;   // 2 log2(e) / cap
  float two_cap;
  float cap;
  float k_out;  // -2 cap log2(e)
  __device__ __forceinline__ explicit SoftCap(float c)
      : k_in(2.0f * 1.4426950408889634f / c), two_cap(2.0f * c), cap(c),
        k_out(-2.0f * c * 1.4426950408889634f) {}
  __device__ __forceinline__ float apply(float z, float& p) const {
    const float r = rcp_approx(1.0f + ex2_approx(z * k_in));
    p = ex2_approx(k_out * r);
    return fmaf(-two_cap, r, cap);
  }
  __device__ __forceinline__ float apply(float z) const {
    const float r = rcp_approx(1.0f + ex2_approx(z * k_in));
    return fmaf(-two_cap, r, cap);
  }
};

// Row r (0..31) of a warp's staging tile: 128 bytes written as eight 16-byte
// chunks at the positions the TMA 128-byte swizzle expects (chunk j of row r
// lives at chunk j ^ (r % 8)); a warp's 32 stores of one chunk hit 8 distinct
// 16-byte bank groups, the minimum of 4 wavefronts for 512 bytes.
__device__ __forceinline__ void stage_row(uint8_t* stg, int r, const uint32_t (&w)[32]) {
#pragma unroll
  for (int j = 0; j < 8; ++j)
    *reinterpret_cast<uint4*>(stg + r * 128 + ((j ^ (r & 7)) << 4)) =
        make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
}

// Half of row r: 64 bytes into chunks [c0, c0 + 4) of the swizzled row.
__device__ __forceinline__ void stage_half_row(uint8_t* stg, int r, int c0, const uint32_t (&w)[16]) {
#pragma unroll
  for (int j = 0; j < 4; ++j)
    *reinterpret_cast<uint4*>(stg + r * 128 + (((c0 + j) ^ (r & 7)) << 4)) =
        make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
}

// Hand the warp's staging tile to TMA: store (or add into the fp32 destination)
// the 32-row box whose top-left element is (row0, col0).  Lane 0 waits until
// TMA has read the tile before anyone reuses the buffer.
template <bool REDUCE>
__device__ __forceinline__ void flush_issue(const CUtensorMap* map, uint8_t* stg, int col0, int row0,
                                            uint32_t lane) {
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    if constexpr (REDUCE)
      tma_reduce_add_2d(map, smem_u32(stg), col0, row0);
    else
      tma_store_2d(map, smem_u32(stg), col0, row0);
    bulk_commit();
  }
}

// The staging tile may be rewritten once TMA has read it.
__device__ __forceinline__ void flush_wait(uint32_t lane) {
  if (lane == 0) bulk_wait_read0();
  __syncwarp();
}

template <bool REDUCE>
__device__ __forceinline__ void flush_stage(const CUtensorMap* map, uint8_t* stg, int col0, int row0,
                                            uint32_t lane) {
  flush_issue<REDUCE>(map, stg, col0, row0, lane);
  flush_wait(lane);
}

// Epilogue of one 32-column chunk for the CE path (partial sums; logits are
// written directly when asked for).
__device__ __forceinline__ void epilogue_ce_chunk(const uint32_t (&r)[32], int row, int col0,
                                                  const EpiParams& ep, float& ce_sum, float& ce_tl,
                                                  int target) {
  // Soft-capped logits l lie in (-cap, cap): exp(l - cap) never overflows, so
  // the per-tile partial sums combine by plain addition.
  const SoftCap sc(ep.cap);
  float v[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    float p;
    v[i] = sc.apply(__uint_as_float(r[i]), p);
    ce_sum += p;
  }
  const int rel = target - col0;
  if (rel >= 0 && rel < 32) {
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (i == rel) ce_tl = v[i];
  }
  if (ep.store_logits) {
    float4* o = reinterpret_cast<float4*>(reinterpret_cast<float*>(ep.out) + (int64_t)row * ep.ldo + col0);
#pragma unroll
    for (int j = 0; j < 8; ++j) o[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
  }
}

// fp32 epilogues (residual add, plain store, soft-cap): 32-column chunks.  The
// TMEM load of chunk c+1 overlaps the TMA read of chunk c.
template <int EPI, bool SC>
__device__ __forceinline__ void epilogue_f32_half(uint32_t taddr, const CUtensorMap* tmC, uint8_t* stg,
                                                  int n0, int row0, int N, const EpiParams& ep,
                                                  uint32_t lane, float dq) {
  uint32_t r[32];
  if (n0 < N) {
    tmem_ld_32x32b_x32(taddr, r);
    tmem_wait_ld();
  }
#pragma unroll 1
  for (int c = 0; c < EPI_COLS / 32; ++c) {
    const int col0 = n0 + c * 32;
    if (col0 >= N) break;  // warp-uniform
    if constexpr (SC) scale32(r, dq);
    if (ep.alpha_ptr) scale32(r, *ep.alpha_ptr);
    else if (ep.alpha != 0.0f) scale32(r, ep.alpha);
    if constexpr (EPI == EPI_SOFTCAP_F32) {
      const SoftCap sc(ep.cap);
#pragma unroll
      for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(sc.apply(__uint_as_float(r[i])));
    }
    if (c > 0) flush_wait(lane);  // previous chunk read out of the staging tile
    stage_row(stg, (int)lane, r);
    flush_issue<EPI == EPI_RESID_F32>(tmC, stg, col0, row0, lane);
    if (c + 1 < EPI_COLS / 32 && col0 + 32 < N) {
      tmem_ld_32x32b_x32(taddr + (c + 1) * 32, r);
      tmem_wait_ld();
    }
  }
  flush_wait(lane);
}

// 16-bit epilogues (plain store, relu^2): 64-column chunks (128 B per row).
// The TMEM loads of chunk c+1 overlap the TMA read of chunk c.
// With SC (e4m3 operands) the relu^2 epilogue also keeps the running maximum
// of its outputs in *om (bits; fp32 before the 16-bit rounding).
template <int EPI, bool F16, bool SC = false>
__device__ __forceinline__ void epilogue_16_half(uint32_t taddr, const CUtensorMap* tmC, uint8_t* stg,
                                                 int n0, int row0, int N, uint32_t lane, float dq = 1.0f,
                                                 uint32_t* om = nullptr) {
  uint32_t r[2][32];
  if (n0 < N) {
    tmem_ld_32x32b_x32(taddr, r[0]);
    tmem_ld_32x32b_x32(taddr + 32, r[1]);
    tmem_wait_ld();
  }
#pragma unroll 1
  for (int c = 0; c < EPI_COLS / 64; ++c) {
    const int col0 = n0 + c * 64;
    if (col0 >= N) break;  // warp-uniform
    uint32_t w[32];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        float a = __uint_as_float(r[h][2 * i]), b = __uint_as_float(r[h][2 * i + 1]);
        if constexpr (SC) {
          a *= dq;
          b *= dq;
        }
        if constexpr (EPI == EPI_RELU2_16) {
          a = fmaxf(a, 0.0f);
          b = fmaxf(b, 0.0f);
          a *= a;
          b *= b;
        }
        if (om) *om = max(*om, max(__float_as_uint(a) & 0x7FFFFFFFu, __float_as_uint(b) & 0x7FFFFFFFu));
        w[16 * h + i] = Half<F16>::pack2(a, b);
      }
    if (c + 1 < EPI_COLS / 64 && col0 + 64 < N) {
      tmem_ld_32x32b_x32(taddr + (c + 1) * 64, r[0]);
      tmem_ld_32x32b_x32(taddr + (c + 1) * 64 + 32, r[1]);
    }
    if (c > 0) flush_wait(lane);
    stage_row(stg, (int)lane, w);
    flush_issue<false>(tmC, stg, col0, row0, lane);
    tmem_wait_ld();
  }
  flush_wait(lane);
}

// Backward epilogues with a 16-bit output that depend on the row (and column):
//   EPI_CE_BWD_16     the accumulator is the recomputed logit z; with l the
//                     soft-capped logit, p = exp(l - lse_row) its probability:
//                     out = (p - [col == target]) (1 - (l / cap)^2), 0 for rows
//                     whose target is -1 (the gradient of the summed
//                     cross-entropy with respect to z);
//   EPI_RELU2_BWD_16  the accumulator is dL/dh for h = relu(u)^2 (saved, 16-bit,
//                     in ep.aux): out = dL/du = acc * 2 sqrt(h).
// 64-column chunks, staged and stored by TMA like epilogue_16_half.
template <int EPI, bool F16>
__device__ __forceinline__ void epilogue_16_rowdep(uint32_t taddr, const CUtensorMap* tmC, uint8_t* stg, int n0,
                                                   int row0, int row, int M, int N, const EpiParams& ep,
                                                   uint32_t lane) {
  const bool live = row < M;
  int target = -1;
  float f = 0.0f;  // exp(cap - lse_row): p = exp(l - cap) f
  const SoftCap sc(ep.cap);
  if constexpr (EPI == EPI_CE_BWD_16) {
    if (live) {
      target = ep.targets[row];
      const float lse = ep.row_lse[row] + (ep.ce_target ? ep.ce_target[row] : 0.0f);
      f = ex2_approx((ep.cap - lse) * 1.4426950408889634f);
    }
  }
  const float inv_cap2 = 1.0f / (ep.cap * ep.cap);
#pragma unroll 1
  for (int c = 0; c < EPI_COLS / 64; ++c) {
    const int col0 = n0 + c * 64;
    if (col0 >= N) break;  // warp-uniform
    uint32_t r[2][32];
    tmem_ld_32x32b_x32(taddr + c * 64, r[0]);
    tmem_ld_32x32b_x32(taddr + c * 64 + 32, r[1]);
    tmem_wait_ld();
    uint32_t hv[32];  // RELU2_BWD: the saved h of these 64 columns
    if constexpr (EPI == EPI_RELU2_BWD_16) {
      if (live) {
        const uint4* hp = reinterpret_cast<const uint4*>(ep.aux + (int64_t)row * ep.ld_aux + col0);
        const int nv = N - col0;  // columns of this chunk inside the row (a multiple of 8)
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint4 u = 8 * j < nv ? __ldg(hp + j) : make_uint4(0u, 0u, 0u, 0u);
          hv[4 * j] = u.x;
          hv[4 * j + 1] = u.y;
          hv[4 * j + 2] = u.z;
          hv[4 * j + 3] = u.w;
        }
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) hv[j] = 0u;
      }
    }
    uint32_t w[32];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        float g[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float acc = __uint_as_float(r[h][2 * i + e]);
          if constexpr (EPI == EPI_CE_BWD_16) {
            float pc;
            const float l = sc.apply(acc, pc);
            const int col = col0 + 32 * h + 2 * i + e;
            const float p = pc * f - (col == target ? 1.0f : 0.0f);
            g[e] = target >= 0 ? p * (1.0f - l * l * inv_cap2) : 0.0f;
          } else {
            const float2 hh = Half<F16>::unpack2(hv[16 * h + i]);
            g[e] = acc * 2.0f * sqrtf(e == 0 ? hh.x : hh.y);
          }
        }
        w[16 * h + i] = Half<F16>::pack2(g[0], g[1]);
      }
    if (c > 0) flush_wait(lane);
    stage_row(stg, (int)lane, w);
    flush_issue<false>(tmC, stg, col0, row0, lane);
  }
  flush_wait(lane);
}

// QKV projection epilogue for one head of HD columns: q and k heads get RoPE
// (pair (u_i, u_{i+HD/2}) rotated by t * theta_i) and RMSNorm over the head
// ("Nanochat与nanoGPT对比" §1: QK-norm after RoPE); v heads are stored as is.
// The rotation preserves the head's norm, so pass 1 takes the RMS straight from
// the fp32 accumulator.  Pass 2 rotates 32-pair groups; the first halves of the
// pairs fill the staging tile (columns [0, HD/2) of the head) while the second
// halves wait in registers, then take its place for columns [HD/2, HD).
template <bool F16, int HD, bool SC>
__device__ __forceinline__ void epilogue_qkv_head(uint32_t taddr, const CUtensorMap* tmC, uint8_t* stg,
                                                  int row, int col0, int row0, int M,
                                                  const EpiParams& ep, uint32_t lane, const Dq& dqs,
                                                  uint32_t* om) {
  constexpr int G = HD / 64;  // 32-pair groups per head (1 or 2)
  const int head = col0 / HD;
  if (head >= ep.H + ep.Hkv) {  // v head (warp-uniform): plain 16-bit store
    epilogue_16_half<EPI_STORE_16, F16, SC>(taddr, tmC, stg, col0, row0, col0 + HD, lane, dqs.v, om);
    return;
  }
  const float dq = head < ep.H ? dqs.q : dqs.k;
  float ss = 0.0f;
#pragma unroll
  for (int c = 0; c < HD / 64; ++c) {  // two 32-column loads per wait
    uint32_t r0[32], r1[32];
    tmem_ld_32x32b_x32(taddr + c * 64, r0);
    tmem_ld_32x32b_x32(taddr + c * 64 + 32, r1);
    tmem_wait_ld();
    float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      s4[i & 3] = fmaf(__uint_as_float(r0[i]), __uint_as_float(r0[i]), s4[i & 3]);
      s4[i & 3] = fmaf(__uint_as_float(r1[i]), __uint_as_float(r1[i]), s4[i & 3]);
    }
    ss += (s4[0] + s4[1]) + (s4[2] + s4[3]);
  }
  // e4m3: the head's values are dq * acc, so its mean square is dq^2 ss / HD
  const float rs = SC ? rsqrtf(ss * (dq * dq) * (1.0f / HD) + ep.eps) * dq : rsqrtf(ss * (1.0f / HD) + ep.eps);
  const int t = ep.pos0 + (row < M ? row : 0) % ep.T;
  const float* cs = ep.rope + (int64_t)t * (HD / 2);
  const float* sn = ep.rope + ((int64_t)(ep.rope_T > 0 ? ep.rope_T : ep.T) + t) * (HD / 2);
  // Pass 2 runs twice: first the rotated first halves u'_i (columns [0, HD/2)),
  // then -- re-reading TMEM -- the second halves u'_{i+HD/2}, so no half has to
  // be held in registers across a TMA store.
#pragma unroll 1
  for (int part = 0; part < 2; ++part) {
#pragma unroll
    for (int g = 0; g < G; ++g) {
      uint32_t ra[32], rb[32];
      tmem_ld_32x32b_x32(taddr + g * 32, ra);
      tmem_ld_32x32b_x32(taddr + HD / 2 + g * 32, rb);
      tmem_wait_ld();
      uint32_t w[16];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float4 c4 = __ldg(reinterpret_cast<const float4*>(cs + g * 32) + j);
        const float4 s4 = __ldg(reinterpret_cast<const float4*>(sn + g * 32) + j);
        const float cc[4] = {c4.x, c4.y, c4.z, c4.w};
        const float sv[4] = {s4.x, s4.y, s4.z, s4.w};
        float v[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float a = __uint_as_float(ra[4 * j + e]), b = __uint_as_float(rb[4 * j + e]);
          v[e] = (part == 0 ? (a * cc[e] - b * sv[e]) : (a * sv[e] + b * cc[e])) * rs;
        }
        w[2 * j] = Half<F16>::pack2(v[0], v[1]);
        w[2 * j + 1] = Half<F16>::pack2(v[2], v[3]);
      }
      // HD = 128: each part is one 64-column chunk (groups at chunks 0-3, 4-7);
      // HD = 64: one chunk holds both parts (first halves 0-3, second 4-7).
      stage_half_row(stg, (int)lane, HD == 128 ? 4 * g : 4 * part, w);
    }
    if constexpr (HD == 128) flush_stage<false>(tmC, stg, col0 + 64 * part, row0, lane);
  }
  if constexpr (HD == 64) flush_stage<false>(tmC, stg, col0, row0, lane);
}

// The same for a projection whose q and k rows were pair-interleaved by the
// weight cast: inside each q/k head, column 2p holds u_p and column 2p+1 holds
// u_{p+HD/2}, so every 64-column chunk carries 32 whole RoPE pairs and is
// rotated, normalised and stored on its own (output in the same interleaved
// order, for q and k alike -- attention scores are unchanged by a common
// permutation of the head dimension).
// v head of the QKV projection with a value embedding (full nanochat forward,
// "Nanochat与nanoGPT对比" §1, value-residual note): v + gate[g] * table[token]
// for kv head g, the table row read in fp32 and added to the fp32 accumulator.
template <bool F16, int HD, bool SC>
__device__ __forceinline__ void epilogue_v_embed(uint32_t taddr, const CUtensorMap* tmC, uint8_t* stg,
                                                 int row, int col0, int row0, int M, const EpiParams& ep,
                                                 uint32_t lane, float dq, uint32_t* om) {
  const int g = col0 / HD - ep.H - ep.Hkv;  // kv head
  int tok = row < M ? ep.tokens[row] : 0;
  if (tok < 0 || tok >= ep.V) tok = 0;  // flagged by the embedding kernel
  const float4* ve = reinterpret_cast<const float4*>(ep.ve + (int64_t)tok * ep.Hkv * HD + (int64_t)g * HD);
  const float gate = ep.ve_gate[g];
#pragma unroll 1
  for (int c = 0; c < HD / 64; ++c) {
    uint32_t r0[32], r1[32];
    tmem_ld_32x32b_x32(taddr + c * 64, r0);
    tmem_ld_32x32b_x32(taddr + c * 64 + 32, r1);
    tmem_wait_ld();
    if constexpr (SC) {
      scale32(r0, dq);
      scale32(r1, dq);
    }
    uint32_t w[32];
#pragma unroll
    for (int j = 0; j < 16; ++j) {  // columns 4j .. 4j+3 of this 64-column chunk
      const float4 e = __ldg(ve + c * 16 + j);
      const uint32_t* src = j < 8 ? r0 : r1;
      const int k = (j & 7) * 4;
      const float v0 = fmaf(gate, e.x, __uint_as_float(src[k])), v1 = fmaf(gate, e.y, __uint_as_float(src[k + 1]));
      const float v2 = fmaf(gate, e.z, __uint_as_float(src[k + 2])), v3 = fmaf(gate, e.w, __uint_as_float(src[k + 3]));
      *om = max(*om, max(max(__float_as_uint(v0) & 0x7FFFFFFFu, __float_as_uint(v1) & 0x7FFFFFFFu),
                         max(__float_as_uint(v2) & 0x7FFFFFFFu, __float_as_uint(v3) & 0x7FFFFFFFu)));
      w[2 * j] = Half<F16>::pack2(v0, v1);
      w[2 * j + 1] = Half<F16>::pack2(v2, v3);
    }
    if (c > 0) flush_wait(lane);
    stage_row(stg, (int)lane, w);
    flush_issue<false>(tmC, stg, col0 + 64 * c, row0, lane);
  }
  flush_wait(lane);
}

template <bool F16, int HD, bool SC>
__device__ __forceinline__ void epilogue_qkv_head_il(uint32_t taddr, const CUtensorMap* tmC,
                                                     uint8_t* stg, int row, int col0, int row0, int M,
                                                     const EpiParams& ep, uint32_t lane, const Dq& dqs,
                                                     uint32_t* om) {
  const int head = col0 / HD;
  if (head >= ep.H + ep.Hkv) {  // v head (warp-uniform)
    if (ep.ve)
      epilogue_v_embed<F16, HD, SC>(taddr, tmC, stg, row, col0, row0, M, ep, lane, dqs.v, om);
    else  // plain 16-bit store
      epilogue_16_half<EPI_STORE_16, F16, SC>(taddr, tmC, stg, col0, row0, col0 + HD, lane, dqs.v, om);
    return;
  }
  const float dq = head < ep.H ? dqs.q : dqs.k;
  float ss = 0.0f;
#pragma unroll
  for (int c = 0; c < HD / 64; ++c) {
    uint32_t r0[32], r1[32];
    tmem_ld_32x32b_x32(taddr + c * 64, r0);
    tmem_ld_32x32b_x32(taddr + c * 64 + 32, r1);
    tmem_wait_ld();
    float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      s4[i & 3] = fmaf(__uint_as_float(r0[i]), __uint_as_float(r0[i]), s4[i & 3]);
      s4[i & 3] = fmaf(__uint_as_float(r1[i]), __uint_as_float(r1[i]), s4[i & 3]);
    }
    ss += (s4[0] + s4[1]) + (s4[2] + s4[3]);
  }
  // e4m3: the head's values are dq * acc, so its mean square is dq^2 ss / HD
  const float rs = SC ? rsqrtf(ss * (dq * dq) * (1.0f / HD) + ep.eps) * dq : rsqrtf(ss * (1.0f / HD) + ep.eps);
  if (ep.rstd_out && row < M) ep.rstd_out[(int64_t)row * (ep.H + ep.Hkv) + head] = rs;
  const int t = ep.pos0 + (row < M ? row : 0) % ep.T;
  const int rt = ep.rope_T > 0 ? ep.rope_T : ep.T;
  const float* cs = ep.rope + (int64_t)t * (HD / 2);
  const float* sn = ep.rope + ((int64_t)rt + t) * (HD / 2);
  // pair-major copy: the warp's 32 rows are consecutive positions, so each
  // load of one pair's (cos, sin) reads one contiguous run of the table
  const float2* cp = ep.rope_pairs ? ep.rope_pairs + t : nullptr;
#pragma unroll 1
  for (int c = 0; c < HD / 64; ++c) {  // pairs 32c .. 32c+31
    uint32_t r0[32], r1[32];
    tmem_ld_32x32b_x32(taddr + c * 64, r0);
    tmem_ld_32x32b_x32(taddr + c * 64 + 32, r1);
    tmem_wait_ld();
    uint32_t w[32];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      float cc[4], sv[4];
      if (cp) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 v = __ldg(cp + (int64_t)(c * 32 + 4 * j + e) * rt);
          cc[e] = v.x;
          sv[e] = v.y;
        }
      } else {
        const float4 c4 = __ldg(reinterpret_cast<const float4*>(cs + c * 32) + j);
        const float4 s4 = __ldg(reinterpret_cast<const float4*>(sn + c * 32) + j);
        cc[0] = c4.x, cc[1] = c4.y, cc[2] = c4.z, cc[3] = c4.w;
        sv[0] = s4.x, sv[1] = s4.y, sv[2] = s4.z, sv[3] = s4.w;
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int pp = 4 * j + e;  // pair within the chunk
        const uint32_t* src = pp < 16 ? r0 : r1;
        const int kk = pp & 15;
        const float a = __uint_as_float(src[2 * kk]), b = __uint_as_float(src[2 * kk + 1]);
        w[pp] = Half<F16>::pack2((a * cc[e] - b * sv[e]) * rs, (a * sv[e] + b * cc[e]) * rs);
      }
    }
    if (c > 0) flush_wait(lane);
    stage_row(stg, (int)lane, w);
    flush_issue<false>(tmC, stg, col0 + 64 * c, row0, lane);
  }
  flush_wait(lane);
}

// EPI: epilogue selector; F16: 16-bit operands (and 16-bit outputs) fp16
// instead of bf16; HD: head size of the QKV epilogues (0 otherwise); FP8:
// e4m3 operands (16-bit outputs still in the F16 format).
// LAY: operand layout (GEMM_NT, GEMM_NN, GEMM_TN).  An MN-major operand is
// loaded as boxes of 64 K rows x 64 MN elements (128 bytes, swizzled); the
// descriptor then steps 64-element MN blocks by the box size and 8-row K
// groups by 1024 bytes, and each MMA of K = 16 advances 16 rows (2048 bytes).
template <int EPI, bool F16, int HD, bool FP8, int LAY = GEMM_NT, bool PAIR = false>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmC, int M, int N, int K, EpiParams ep,
                uint32_t* dev_status, uint64_t limit_ns) {
  constexpr bool A_MN = LAY == GEMM_TN, B_MN = LAY != GEMM_NT;
  static_assert(!(FP8 && LAY != GEMM_NT), "e4m3 operands are K-major");
  static_assert(!PAIR || !FP8, "CTA pairs: 16-bit operands");
  constexpr uint32_t IDESC = (PAIR ? (F16 ? IDESC_PAIR_F16 : IDESC_PAIR_BF16)
                                   : (FP8 ? IDESC_E4M3 : (F16 ? IDESC_F16 : IDESC_BF16))) |
                             (A_MN ? (1u << 15) : 0u) | (B_MN ? (1u << 16) : 0u);
  constexpr int NST = PAIR ? PAIR_STAGES : STAGES;            // ring stages
  constexpr int SBYTES = PAIR ? PAIR_STAGE_BYTES : STAGE_BYTES;  // bytes of one stage in this CTA
  constexpr int TM = PAIR ? 2 * BM : BM;                      // rows of one output tile
  constexpr int MN_BOX = 64 * BK * 2;  // bytes of one MN-major box
  constexpr int KE = FP8 ? 2 * BK : BK;  // elements per 128-byte swizzle row
  extern __shared__ uint8_t smem_raw[];
  uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  uint8_t* staging = tiles + STAGES * STAGE_BYTES;  // EPI_WARPS x STG_BYTES
  Smem* sm = reinterpret_cast<Smem*>(staging + EPI_WARPS * STG_BYTES);

  const uint32_t warp = warp_id_sync();
  const uint32_t lane = lane_id();
  // With CTA pairs both CTAs of cluster c walk the same tiles; rank 0 issues
  // the MMAs, and each rank owns rows [rank * BM, rank * BM + BM) of a tile.
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const int tile0 = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int tstride = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  const int num_m = (M + TM - 1) / TM;
  const int num_n = (N + BN - 1) / BN;
  // Split-K (residual-add epilogue only): tile t covers K slice t / (num_m * num_n).
  const int ksplit = (EPI == EPI_RESID_F32 && ep.ksplit > 1) ? ep.ksplit : 1;
  const int num_mn = num_m * num_n;
  const int num_tiles = num_mn * ksplit;
  const int num_kb = (K + KE - 1) / KE;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(smem_u32(&sm->full[s]), 1);
      mbar_init(smem_u32(&sm->empty[s]), 1);
    }
    for (int a = 0; a < NUM_ACC; ++a) {
      mbar_init(smem_u32(&sm->tmem_full[a]), 1);
      mbar_init(smem_u32(&sm->tmem_empty[a]), PAIR ? 2 * EPI_WARPS : EPI_WARPS);
    }
    mbar_init(smem_u32(&sm->drain), 1);
    sm->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc_pair(smem_u32(&sm->tmem_base), TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(&sm->tmem_base), TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) cluster_sync();  // both CTAs' barriers are initialised
  tc_fence_after();
  const uint32_t tmem_base = sm->tmem_base;
  const WaitCtl ctl{&sm->abort_flag, dev_status, limit_ns};

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer
      int stage = 0;
      uint32_t phase = 0;
      uint32_t outstanding = 0;  // bit s: stage s has a load this thread issued
      uint32_t out_phase = 0;    // bit s: phase of that load
      bool ok = true;
      for (int tile = tile0; tile < num_tiles && ok; tile += tstride) {
        const int mn = tile % num_mn, ks = tile / num_mn;
        const int m0 = (mn / num_n) * TM;
        const int n0 = (mn % num_n) * BN;
        const int kb_end = (ks + 1) * num_kb / ksplit;
        for (int kb = ks * num_kb / ksplit; kb < kb_end; ++kb) {
          const uint32_t eb = smem_u32(&sm->empty[stage]);
          if (!(PAIR ? mbar_wait_cluster(eb, phase ^ 1u, ctl) : mbar_wait(eb, phase ^ 1u, ctl))) {
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(&sm->full[stage]);
          uint8_t* a_dst = tiles + stage * SBYTES;
          if constexpr (PAIR) {
            // Both halves complete on rank 0's barrier, which expects the bytes
            // of both CTAs.
            const uint32_t fb0 = mapa_shared(fb, 0);
            if (rank == 0) mbar_arrive_expect_tx(fb, 2 * SBYTES);
            const int ma = m0 + (int)rank * BM, nb = n0 + (int)rank * (BN / 2);  // this CTA's rows of A and W
            if constexpr (A_MN) {
#pragma unroll
              for (int i = 0; i < BM / 64; ++i)
                tma_load_2d_pair(smem_u32(a_dst + i * MN_BOX), &tmA, ma + 64 * i, kb * BK, fb0);
            } else {
              tma_load_2d_pair(smem_u32(a_dst), &tmA, kb * KE, ma, fb0);
            }
            if constexpr (B_MN) {
#pragma unroll
              for (int i = 0; i < BN / 2 / 64; ++i)
                tma_load_2d_pair(smem_u32(a_dst + A_BYTES + i * MN_BOX), &tmB, nb + 64 * i, kb * BK, fb0);
            } else {
              tma_load_2d_pair(smem_u32(a_dst + A_BYTES), &tmB, kb * KE, nb, fb0);
            }
          } else {
          mbar_arrive_expect_tx(fb, STAGE_BYTES);
          if constexpr (A_MN) {
#pragma unroll
            for (int i = 0; i < BM / 64; ++i) tma_load_2d(smem_u32(a_dst + i * MN_BOX), &tmA, m0 + 64 * i, kb * BK, fb);
          } else {
            tma_load_2d(smem_u32(a_dst), &tmA, kb * KE, m0, fb);
          }
          if constexpr (B_MN) {
#pragma unroll
            for (int i = 0; i < BN / 64; ++i)
              tma_load_2d(smem_u32(a_dst + A_BYTES + i * MN_BOX), &tmB, n0 + 64 * i, kb * BK, fb);
          } else {
            tma_load_2d(smem_u32(a_dst + A_BYTES), &tmB, kb * KE, n0, fb);
          }
          }
          outstanding |= 1u << stage;
          out_phase = (out_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == NST) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if ((!ok || sm->abort_flag) && rank == 0) {
        // Let every copy this thread started land before the CTA exits (with
        // CTA pairs, rank 0's barriers also count the peer's copies, and the
        // closing cluster barrier keeps both CTAs resident until then).
        int zero = 0;
        const WaitCtl drain_ctl{&zero, nullptr, limit_ns};
        for (int s = 0; s < NST; ++s)
          if (outstanding & (1u << s))
            mbar_wait(smem_u32(&sm->full[s]), (out_phase >> s) & 1u, drain_ctl);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ---------------- UMMA issuer (rank 0 of a pair issues for both CTAs)
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      // Arrive on a barrier of this CTA and, with CTA pairs, on the same
      // barrier of the peer once the MMAs issued so far are done.
      auto commit = [&](uint64_t* bar) {
        if constexpr (PAIR) {
          umma_commit_pair(smem_u32(bar));
          umma_commit_pair(mapa_shared(smem_u32(bar), 1));
        } else {
          umma_commit(smem_u32(bar));
        }
      };
      for (int tile = tile0; tile < num_tiles && ok; tile += tstride) {
        const uint32_t teb = smem_u32(&sm->tmem_empty[acc]);
        if (!(PAIR ? mbar_wait_cluster(teb, acc_phase ^ 1u, ctl) : mbar_wait(teb, acc_phase ^ 1u, ctl))) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        const int ks = tile / num_mn;
        const int kb_begin = ks * num_kb / ksplit, kb_end = (ks + 1) * num_kb / ksplit;
        for (int kb = kb_begin; kb < kb_end; ++kb) {
          if (!mbar_wait(smem_u32(&sm->full[stage]), phase, ctl)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(tiles + stage * SBYTES);
          const uint32_t b_addr = a_addr + A_BYTES;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {  // 32 bytes of each row (K-major) or 16 rows (MN-major) per MMA
            const uint64_t adesc = A_MN ? sw128_desc(a_addr + k * 2048, MN_BOX, 1024) : sw128_kmajor_desc(a_addr + k * 32);
            const uint64_t bdesc = B_MN ? sw128_desc(b_addr + k * 2048, MN_BOX, 1024) : sw128_kmajor_desc(b_addr + k * 32);
            const uint32_t accum = (kb != kb_begin || k != 0) ? 1u : 0u;
            if constexpr (PAIR)
              umma_f16_pair(d_tmem, adesc, bdesc, IDESC, accum);
            else if constexpr (FP8)
              umma_f8(d_tmem, adesc, bdesc, IDESC, accum);
            else
              umma_f16(d_tmem, adesc, bdesc, IDESC, accum);
          }
          commit(&sm->empty[stage]);
          if (++stage == NST) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        commit(&sm->tmem_full[acc]);
        if (++acc == NUM_ACC) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      // Wait until every MMA this thread issued has completed.
      if constexpr (PAIR)
        umma_commit_pair(smem_u32(&sm->drain));
      else
        umma_commit(smem_u32(&sm->drain));
      int zero = 0;
      WaitCtl drain_ctl{&zero, nullptr, limit_ns};
      mbar_wait(smem_u32(&sm->drain), 0, drain_ctl);
    }
  } else {
    // ---------------- epilogue warps
    const uint32_t quarter = warp & 3u;
    const int half = (int)(warp - 2) / 4;  // which half of the tile's columns
    const int row_in_tile = quarter * 32 + lane;
    uint8_t* stg = staging + (warp - 2) * STG_BYTES;  // this warp's staging tile
    Dq dqs{1.0f, 1.0f, 1.0f};
    // max |16-bit output| (bits): the fp16 range check, and with e4m3 operands
    // the relu^2 output's amax for ep.amax_out
    uint32_t om = 0;
    if constexpr (FP8) {  // 1 / (s_a s_w) from the tensors' amax values
      const float sa = e4m3_scale(__ldg(ep.amax_a));
      dqs.q = 1.0f / (sa * e4m3_scale(__ldg(ep.amax_b)));
      if constexpr (EPI == EPI_QKV_ROPE || EPI == EPI_QKV_ROPE_IL) {
        dqs.k = 1.0f / (sa * e4m3_scale(__ldg(ep.amax_b + 1)));
        dqs.v = 1.0f / (sa * e4m3_scale(__ldg(ep.amax_b + 2)));
      } else {
        dqs.k = dqs.v = dqs.q;
      }
    }
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = tile0; tile < num_tiles; tile += tstride) {
      const int m_blk = (tile % num_mn) / num_n;
      const int n_blk = (tile % num_mn) % num_n;
      const int m0 = m_blk * TM + (int)rank * BM;  // this CTA's first row
      const int n0 = n_blk * BN + half * EPI_COLS;  // this warp's first column
      const int row = m0 + row_in_tile;
      if constexpr (EPI == EPI_QKV_ROPE || EPI == EPI_QKV_ROPE_IL) {
        // This row's cos/sin lines are known before the accumulator is ready:
        // pull them into L1 while the MMAs run (q and k heads only).
        if (row < M && n0 < N && n0 / HD < ep.H + ep.Hkv && !(EPI == EPI_QKV_ROPE_IL && ep.rope_pairs)) {
          const int t = ep.pos0 + row % ep.T;
          const int rt = ep.rope_T > 0 ? ep.rope_T : ep.T;
          const char* cl = reinterpret_cast<const char*>(ep.rope + (int64_t)t * (HD / 2));
          const char* sl = reinterpret_cast<const char*>(ep.rope + ((int64_t)rt + t) * (HD / 2));
#pragma unroll
          for (int l = 0; l < HD * 2 / 128; ++l) {
            asm volatile("prefetch.global.L1 [%0];" ::"l"(cl + 128 * l));
            asm volatile("prefetch.global.L1 [%0];" ::"l"(sl + 128 * l));
          }
        }
      }
      const uint32_t tfb = smem_u32(&sm->tmem_full[acc]);
      if (!(PAIR ? mbar_wait_cluster(tfb, acc_phase, ctl) : mbar_wait(tfb, acc_phase, ctl))) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((quarter * 32u) << 16) + acc * BN + half * EPI_COLS;
      const int row0 = m0 + (int)quarter * 32;  // first tile row of this warp
      float ce_sum = 0.0f, ce_tl = 0.0f;
      int target = -1;
      if constexpr (EPI == EPI_QKV_ROPE || EPI == EPI_QKV_ROPE_IL) {
#pragma unroll 1
        for (int hh = 0; hh < EPI_COLS / HD; ++hh) {
          const int col0 = n0 + hh * HD;
          if (col0 >= N) break;  // warp-uniform
          if constexpr (EPI == EPI_QKV_ROPE)
            epilogue_qkv_head<F16, HD, FP8>(taddr + hh * HD, &tmC, stg, row, col0, row0, M, ep, lane, dqs, &om);
          else
            epilogue_qkv_head_il<F16, HD, FP8>(taddr + hh * HD, &tmC, stg, row, col0, row0, M, ep, lane, dqs,
                                               &om);
        }
      } else if constexpr (EPI == EPI_STORE_16 || EPI == EPI_RELU2_16) {
        epilogue_16_half<EPI, F16, FP8>(taddr, &tmC, stg, n0, row0, N, lane, dqs.q, &om);
      } else if constexpr (EPI == EPI_CE_BWD_16 || EPI == EPI_RELU2_BWD_16) {
        epilogue_16_rowdep<EPI, F16>(taddr, &tmC, stg, n0, row0, row, M, N, ep, lane);
      } else if constexpr (EPI == EPI_CE_PARTIAL) {
        if (row < M) target = ep.targets ? ep.targets[row] : -1;
#pragma unroll 1
        for (int c = 0; c < EPI_COLS / 32; ++c) {
          const int col0 = n0 + c * 32;
          if (col0 >= N) break;  // warp-uniform
          uint32_t r[32];
          tmem_ld_32x32b_x32(taddr + c * 32, r);
          tmem_wait_ld();
          if constexpr (FP8) scale32(r, dqs.q);
          if (row < M) epilogue_ce_chunk(r, row, col0, ep, ce_sum, ce_tl, target);
        }
      } else {
        epilogue_f32_half<EPI, FP8>(taddr, &tmC, stg, n0, row0, N, ep, lane, dqs.q);
      }
      if constexpr (EPI == EPI_CE_PARTIAL) {
        if (row < M) {
          ep.ce_partial[(int64_t)row * (2 * num_n) + 2 * n_blk + half] = ce_sum;
          if (target >= n0 && target < n0 + EPI_COLS && target < N) ep.ce_target[row] = ce_tl;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {  // the accumulator is free again (rank 0 of a pair counts both CTAs)
        if constexpr (PAIR)
          mbar_arrive_cluster(mapa_shared(smem_u32(&sm->tmem_empty[acc]), 0));
        else
          mbar_arrive(smem_u32(&sm->tmem_empty[acc]));
      }
      if (++acc == NUM_ACC) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
    if constexpr (EPI == EPI_STORE_16 || EPI == EPI_RELU2_16 || EPI == EPI_QKV_ROPE || EPI == EPI_QKV_ROPE_IL) {
      om = __reduce_max_sync(0xFFFFFFFFu, om);
      // fp16 saturates above 65504 (0x477FE000 as fp32 bits): flag it
      if constexpr (F16)
        if (lane == 0 && om > 0x477FE000u && dev_status) atomicOr(dev_status, NC_DEV_F16_RANGE);
      if constexpr (FP8 && EPI == EPI_RELU2_16)
        if (ep.amax_out && lane == 0) fold_amax(ep.amax_out, stored_abs_bits<F16>(om));
    }
    if (lane == 0) bulk_wait0();  // every TMA store / reduce of this warp has landed
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  // With CTA pairs neither CTA may leave while the other can still reach its
  // shared memory, barriers or tensor memory.
  if constexpr (PAIR) cluster_sync();
  tc_fence_after();
  if (warp == 1) {
    if constexpr (PAIR)
      tmem_dealloc_pair(tmem_base, TMEM_COLS);
    else
      tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------- host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 16-bit row-major [rows, cols] with row stride `ld` elements; box = 64 x box_rows.
static bool make_map(CUtensorMap* map, const void* ptr, int64_t rows, int64_t cols, int64_t ld,
                     int box_rows, bool f16) {
  const uint64_t dims[2] = {(uint64_t)cols, (uint64_t)rows};
  const uint64_t strides[1] = {(uint64_t)(ld * 2)};
  const uint32_t box[2] = {(uint32_t)BK, (uint32_t)box_rows};
  return encode_tensor_map(map, f16, 2, ptr, dims, strides, box);
}

// 8-bit row-major [rows, cols] with row stride `ld` bytes; box = 128 x box_rows.
static bool make_map_u8(CUtensorMap* map, const void* ptr, int64_t rows, int64_t cols, int64_t ld,
                        int box_rows) {
  const uint64_t dims[2] = {(uint64_t)cols, (uint64_t)rows};
  const uint64_t strides[1] = {(uint64_t)ld};
  const uint32_t box[2] = {(uint32_t)(2 * BK), (uint32_t)box_rows};
  return encode_tensor_map_u8(map, 2, ptr, dims, strides, box);
}

// Persistent grid: one CTA (or CTA pair) per SM that can hold one.  With CTA
// pairs the grid is the number of two-CTA clusters the device can keep
// resident at once (queried once per device), times two.
template <int EPI, bool F16, int HD, bool FP8, int LAY = GEMM_NT, bool PAIR = false>
static cudaError_t launch_t(const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& mc, int M,
                            int N, int K, const EpiParams& ep, uint32_t* dev_status, uint64_t limit_ns,
                            cudaStream_t stream) {
  auto kern = gemm_kernel<EPI, F16, HD, FP8, LAY, PAIR>;
  static bool attr_done[64] = {};
  static int pair_slots[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_done[dev]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    if constexpr (PAIR) {
      cudaLaunchConfig_t q = {};
      cudaLaunchAttribute qa[1];
      qa[0].id = cudaLaunchAttributeClusterDimension;
      qa[0].val.clusterDim.x = 2;
      qa[0].val.clusterDim.y = 1;
      qa[0].val.clusterDim.z = 1;
      q.gridDim = dim3(2 * 148);
      q.blockDim = dim3(NUM_THREADS);
      q.dynamicSmemBytes = SMEM_BYTES;
      q.attrs = qa;
      q.numAttrs = 1;
      int clusters = 0;
      e = cudaOccupancyMaxActiveClusters(&clusters, kern, &q);
      if (e != cudaSuccess) return e;
      if (clusters < 1) return cudaErrorInvalidConfiguration;
      pair_slots[dev] = clusters;
    }
    attr_done[dev] = true;
  }
  const int tm = PAIR ? 2 * BM : BM;
  const int tiles = ((M + tm - 1) / tm) * ((N + BN - 1) / BN) * (EPI == EPI_RESID_F32 && ep.ksplit > 1 ? ep.ksplit : 1);
  if constexpr (PAIR) {
    const int clusters = tiles < pair_slots[dev] ? tiles : pair_slots[dev];
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 2;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2 * clusters);
    cfg.blockDim = dim3(NUM_THREADS);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.stream = stream;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, ma, mb, mc, M, N, K, ep, dev_status, limit_ns);
  } else {
    const int sms = device_sm_count();
    const int grid = tiles < sms ? tiles : sms;
    kern<<<grid, NUM_THREADS, SMEM_BYTES, stream>>>(ma, mb, mc, M, N, K, ep, dev_status, limit_ns);
    return cudaGetLastError();
  }
}

template <bool F16, bool FP8, bool PAIR = false>
static cudaError_t dispatch(int epi, const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& mc,
                            int M, int N, int K, const EpiParams& ep, uint32_t* st, uint64_t lim,
                            cudaStream_t s) {
  switch (epi) {
    case EPI_STORE_16: return launch_t<EPI_STORE_16, F16, 0, FP8, GEMM_NT, PAIR>(ma, mb, mc, M, N, K, ep, st, lim, s);
    case EPI_RELU2_16: return launch_t<EPI_RELU2_16, F16, 0, FP8, GEMM_NT, PAIR>(ma, mb, mc, M, N, K, ep, st, lim, s);
    case EPI_RESID_F32: return launch_t<EPI_RESID_F32, F16, 0, FP8, GEMM_NT, PAIR>(ma, mb, mc, M, N, K, ep, st, lim, s);
    case EPI_STORE_F32: return launch_t<EPI_STORE_F32, F16, 0, FP8, GEMM_NT, PAIR>(ma, mb, mc, M, N, K, ep, st, lim, s);
    case EPI_SOFTCAP_F32: return launch_t<EPI_SOFTCAP_F32, F16, 0, FP8, GEMM_NT, PAIR>(ma, mb, mc, M, N, K, ep, st, lim, s);
    case EPI_CE_PARTIAL: return launch_t<EPI_CE_PARTIAL, F16, 0, FP8, GEMM_NT, PAIR>(ma, mb, mc, M, N, K, ep, st, lim, s);
    case EPI_CE_BWD_16:
      if constexpr (FP8) return cudaErrorInvalidValue;
      else return launch_t<EPI_CE_BWD_16, F16, 0, false, GEMM_NT, PAIR>(ma, mb, mc, M, N, K, ep, st, lim, s);
    case EPI_QKV_ROPE:
      if constexpr (FP8) return cudaErrorInvalidValue;  // the interleaved form only
      else
        return ep.D == 128 ? launch_t<EPI_QKV_ROPE, F16, 128, false, GEMM_NT, PAIR>(ma, mb, mc, M, N, K, ep, st, lim, s)
                           : launch_t<EPI_QKV_ROPE, F16, 64, false, GEMM_NT, PAIR>(ma, mb, mc, M, N, K, ep, st, lim, s);
    case EPI_QKV_ROPE_IL:
      return ep.D == 128 ? launch_t<EPI_QKV_ROPE_IL, F16, 128, FP8, GEMM_NT, PAIR>(ma, mb, mc, M, N, K, ep, st, lim, s)
                         : launch_t<EPI_QKV_ROPE_IL, F16, 64, FP8, GEMM_NT, PAIR>(ma, mb, mc, M, N, K, ep, st, lim, s);
    default: return cudaErrorInvalidValue;
  }
}

template <bool F16, int LAY, bool PAIR>
static cudaError_t dispatch_layout(int epi, const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& mc,
                                   int M, int N, int K, const EpiParams& ep, uint32_t* st, uint64_t lim,
                                   cudaStream_t s) {
  switch (epi) {
    case EPI_STORE_16: return launch_t<EPI_STORE_16, F16, 0, false, LAY, PAIR>(ma, mb, mc, M, N, K, ep, st, lim, s);
    case EPI_STORE_F32: return launch_t<EPI_STORE_F32, F16, 0, false, LAY, PAIR>(ma, mb, mc, M, N, K, ep, st, lim, s);
    case EPI_RESID_F32: return launch_t<EPI_RESID_F32, F16, 0, false, LAY, PAIR>(ma, mb, mc, M, N, K, ep, st, lim, s);
    case EPI_RELU2_BWD_16:
      return launch_t<EPI_RELU2_BWD_16, F16, 0, false, LAY, PAIR>(ma, mb, mc, M, N, K, ep, st, lim, s);
    default: return cudaErrorInvalidValue;
  }
}

// One thread waits for a phase that never completes; the bounded wait gives
// up after limit_ns and records NC_DEV_TIMEOUT.
__global__ void selftest_wait_kernel(uint32_t* dev_status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const WaitCtl ctl{&abort_flag, dev_status, limit_ns};
    (void)mbar_wait(smem_u32(&bar), 0, ctl);
  }
  __syncthreads();
}

}  // namespace gemm

static bool encode_any(CUtensorMap* map, CUtensorMapDataType dt, int rank, const void* base,
                       const uint64_t* dims, const uint64_t* strides, const uint32_t* box);

bool encode_tensor_map(CUtensorMap* map, bool f16, int rank, const void* base, const uint64_t* dims,
                       const uint64_t* strides, const uint32_t* box) {
  return encode_any(map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank,
                    base, dims, strides, box);
}

bool encode_tensor_map_u8(CUtensorMap* map, int rank, const void* base, const uint64_t* dims,
                          const uint64_t* strides, const uint32_t* box) {
  return encode_any(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, rank, base, dims, strides, box);
}

bool encode_tensor_map_f32(CUtensorMap* map, int rank, const void* base, const uint64_t* dims,
                           const uint64_t* strides, const uint32_t* box) {
  return encode_any(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, rank, base, dims, strides, box);
}

static bool encode_any(CUtensorMap* map, CUtensorMapDataType dt, int rank, const void* base,
                       const uint64_t* dims, const uint64_t* strides, const uint32_t* box) {
  gemm::EncodeTiledFn enc = gemm::get_encode_fn();
  if (!enc || rank < 1 || rank > 5) return false;
  cuuint64_t d[5], st[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
  }
  for (int i = 0; i + 1 < rank; ++i) st[i] = strides[i];
  const CUresult r = enc(map, dt, (cuuint32_t)rank, const_cast<void*>(base), d, st, bx, es,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

nc_status selftest_wait_launch(uint32_t* dev_status, uint64_t limit_ns, cudaStream_t stream) {
  gemm::selftest_wait_kernel<<<1, 32, 0, stream>>>(dev_status, limit_ns);
  return cudaGetLastError() == cudaSuccess ? NC_OK : NC_ERR_CUDA;
}

int gemm_ce_partials_per_row(int N) { return 2 * ((N + gemm::BN - 1) / gemm::BN); }

// Output tile map for the TMA stores of the epilogue: 32 rows x 128 bytes
// (64 16-bit or 32 fp32 columns), the box one epilogue warp stages.
static bool make_out_map(CUtensorMap* mc, int epi, int M, int N, bool f16, const EpiParams& ep) {
  memset(mc, 0, sizeof(*mc));
  if (epi == EPI_CE_PARTIAL) return true;
  const uint64_t dims[2] = {(uint64_t)N, (uint64_t)M};
  const bool out16 = (epi == EPI_STORE_16 || epi == EPI_RELU2_16 || epi == EPI_QKV_ROPE ||
                      epi == EPI_QKV_ROPE_IL || epi == EPI_CE_BWD_16 || epi == EPI_RELU2_BWD_16);
  const uint64_t strides[1] = {(uint64_t)ep.ldo * (out16 ? 2 : 4)};
  const uint32_t box[2] = {out16 ? 64u : 32u, 32u};
  return out16 ? encode_tensor_map(mc, f16, 2, ep.out, dims, strides, box)
               : encode_tensor_map_f32(mc, 2, ep.out, dims, strides, box);
}

static nc_status check_epi(int epi, int K, int ke, const EpiParams& ep) {
  if (epi < EPI_STORE_16 || epi > EPI_RELU2_BWD_16) return NC_ERR_INVALID_ARG;
  if (epi == EPI_CE_BWD_16 && (!ep.targets || !ep.row_lse)) return NC_ERR_INVALID_ARG;
  if (epi == EPI_RELU2_BWD_16 && (!ep.aux || ep.ld_aux % 8)) return NC_ERR_INVALID_ARG;
  if ((epi == EPI_QKV_ROPE || epi == EPI_QKV_ROPE_IL) && (ep.D != 64 && ep.D != 128)) return NC_ERR_SHAPE;
  if (ep.ksplit > 1 && (epi != EPI_RESID_F32 || ep.ksplit > (K + ke - 1) / ke)) return NC_ERR_INVALID_ARG;
  return NC_OK;
}

nc_status gemm_launch(const uint16_t* a, int64_t lda, const uint16_t* w, int64_t ldw, int M, int N,
                      int K, int epi, bool f16, const EpiParams& ep, uint32_t* dev_status,
                      cudaStream_t stream, uint64_t limit_ns) {
  using namespace gemm;
  if (nc_status s = check_epi(epi, K, BK, ep)) return s;
  CUtensorMap ma, mb, mc;
  if (!make_map(&ma, a, M, K, lda, BM, f16)) return NC_ERR_CUDA;
  // CTA pairs for every product with more than one 128-row block (no split K).
  const bool pair = M > BM && ep.ksplit <= 1;
  if (!make_map(&mb, w, N, K, ldw, pair ? BN / 2 : BN, f16)) return NC_ERR_CUDA;
  if (!make_out_map(&mc, epi, M, N, f16, ep)) return NC_ERR_CUDA;
  cudaError_t e;
  if (pair)
    e = f16 ? dispatch<true, false, true>(epi, ma, mb, mc, M, N, K, ep, dev_status, limit_ns, stream)
            : dispatch<false, false, true>(epi, ma, mb, mc, M, N, K, ep, dev_status, limit_ns, stream);
  else
    e = f16 ? dispatch<true, false>(epi, ma, mb, mc, M, N, K, ep, dev_status, limit_ns, stream)
            : dispatch<false, false>(epi, ma, mb, mc, M, N, K, ep, dev_status, limit_ns, stream);
  return e == cudaSuccess ? NC_OK : NC_ERR_CUDA;
}

// MN-major operand given as [K rows, MN cols] with row stride `ld` elements;
// box = 64 MN elements x 64 K rows.
static bool make_map_mn(CUtensorMap* map, const void* ptr, int64_t k_rows, int64_t mn_cols, int64_t ld, bool f16) {
  const uint64_t dims[2] = {(uint64_t)mn_cols, (uint64_t)k_rows};
  const uint64_t strides[1] = {(uint64_t)(ld * 2)};
  const uint32_t box[2] = {64u, (uint32_t)gemm::BK};
  return encode_tensor_map(map, f16, 2, ptr, dims, strides, box);
}

nc_status gemm_launch_layout(const uint16_t* a, int64_t lda, const uint16_t* w, int64_t ldw, int M, int N, int K,
                             int epi, bool f16, int layout, const EpiParams& ep, uint32_t* dev_status,
                             cudaStream_t stream, uint64_t limit_ns) {
  using namespace gemm;
  if (layout == GEMM_NT) return gemm_launch(a, lda, w, ldw, M, N, K, epi, f16, ep, dev_status, stream, limit_ns);
  if (layout != GEMM_NN && layout != GEMM_TN) return NC_ERR_INVALID_ARG;
  if (epi != EPI_STORE_16 && epi != EPI_STORE_F32 && epi != EPI_RESID_F32 && epi != EPI_RELU2_BWD_16)
    return NC_ERR_INVALID_ARG;
  if (nc_status s = check_epi(epi, K, BK, ep)) return s;
  CUtensorMap ma, mb, mc;
  // CTA pairs for the weight gradients (GEMM_TN) with more than one 128-row
  // block; the GEMM_NN products measured 6 % slower per clock on pairs
  const bool pair = layout == GEMM_TN && M > BM;
  const bool ok_a = layout == GEMM_TN ? make_map_mn(&ma, a, K, M, lda, f16) : make_map(&ma, a, M, K, lda, BM, f16);
  if (!ok_a || !make_map_mn(&mb, w, K, N, ldw, f16)) return NC_ERR_CUDA;
  if (!make_out_map(&mc, epi, M, N, f16, ep)) return NC_ERR_CUDA;
  cudaError_t e;
#define NC_LAYOUT_CASE(L, P)                                                                           \
  (f16 ? dispatch_layout<true, L, P>(epi, ma, mb, mc, M, N, K, ep, dev_status, limit_ns, stream)        \
       : dispatch_layout<false, L, P>(epi, ma, mb, mc, M, N, K, ep, dev_status, limit_ns, stream))
  if (layout == GEMM_NN)
    e = pair ? NC_LAYOUT_CASE(GEMM_NN, true) : NC_LAYOUT_CASE(GEMM_NN, false);
  else
    e = pair ? NC_LAYOUT_CASE(GEMM_TN, true) : NC_LAYOUT_CASE(GEMM_TN, false);
#undef NC_LAYOUT_CASE
  return e == cudaSuccess ? NC_OK : NC_ERR_CUDA;
}

nc_status gemm_launch_e4m3(const uint8_t* a, int64_t lda, const uint8_t* w, int64_t ldw, int M, int N, int K,
                           int epi, bool f16, const EpiParams& ep, uint32_t* dev_status, cudaStream_t stream,
                           uint64_t limit_ns) {
  using namespace gemm;
  if (nc_status s = check_epi(epi, K, 2 * BK, ep)) return s;
  if (epi == EPI_QKV_ROPE || !ep.amax_a || !ep.amax_b || K % 16 || lda % 16 || ldw % 16)
    return NC_ERR_INVALID_ARG;
  CUtensorMap ma, mb, mc;
  if (!make_map_u8(&ma, a, M, K, lda, BM)) return NC_ERR_CUDA;
  if (!make_map_u8(&mb, w, N, K, ldw, BN)) return NC_ERR_CUDA;
  if (!make_out_map(&mc, epi, M, N, f16, ep)) return NC_ERR_CUDA;
  const cudaError_t e = f16 ? dispatch<true, true>(epi, ma, mb, mc, M, N, K, ep, dev_status, limit_ns, stream)
                            : dispatch<false, true>(epi, ma, mb, mc, M, N, K, ep, dev_status, limit_ns, stream);
  return e == cudaSuccess ? NC_OK : NC_ERR_CUDA;
}

}  // namespace nc
