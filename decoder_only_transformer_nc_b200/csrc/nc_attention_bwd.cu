// Attention backward on the 5th-generation tensor cores ("从文本到聊天模型"
// §6.5: loss.backward() of the training step, through the windowed causal GQA
// attention of §5.5).  Per head, with scale s = 1/sqrt(D), the weights P are
// recomputed from the forward's log-sum-exp:
//   P = exp(s Q K^T - lse),  dV = P^T dO,  dP = dO V^T,
//   dS = P o (dP - Delta) with Delta_i = sum_d dO_i O_i,
//   dQ = s dS K,  dK = s dS^T Q.
// Two kernels, so that no sum needs atomics (dK and dV sum over the query
// heads of their kv group):
//   attn_bwd_kv_kernel  one CTA per (128 keys, kv head, batch row): S^T = K Q^T
//                       and dP^T = V dO^T into tensor memory, P^T and dS^T
//                       written back over them as 16-bit values, then
//                       dV += P^T dO and dK += dS^T Q with the A operand read
//                       from tensor memory; loops over the query heads of the
//                       group and the query tiles that see these keys;
//   attn_bwd_q_kernel   one CTA per (128 queries, head, batch row): S = Q K^T
//                       and dP = dO V^T, dS written back over dP, dQ += dS K;
//                       loops over the key tiles inside the window.
// Each 128-column score tile is computed and consumed in two halves of 64
// columns, each with its own four softmax warps (one per TMEM lane quarter),
// so the tensor core works on one half while the softmax warps of the other
// run; the streamed tiles (Q, dO or K, V) pass through a two-stage ring.
// Warp 0 issues the TMA loads (128-byte swizzle, boxes of 64 dims x 128
// tokens), warp 1 owns 512 TMEM columns and issues tcgen05.mma; warps 2..9
// are the softmax warps and, at the end, the epilogue.  Every mbarrier wait is
// bounded: on timeout the CTA records NC_DEV_TIMEOUT and winds down.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "nc_half.cuh"
#include "nc_internal.h"
#include "nc_ptx.cuh"


namespace nc {
namespace attn_bwd {

constexpr int BT = 128;  // tokens of a tile (the CTA's own, and each streamed one)
constexpr int NST = 2;   // ring stages
constexpr int ATOM = BT * 128;  // box: 64 dims x 128 tokens
constexpr int NUM_THREADS = 320;
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 32 lanes x 16 consecutive 32-bit columns from registers (thread i -> lane
// base + i).
__device__ __forceinline__ void tmem_st_x16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32"
      " [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// 32 lanes x 16 consecutive 32-bit columns into registers.
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32"
      " {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

// 32 lanes x 8 consecutive 32-bit columns from registers.
__device__ __forceinline__ void tmem_st_x8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[0]),
               "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}

template <int D>
struct Geo {
  static constexpr int KA = D / 64;               // 64-dim boxes per token row
  static constexpr int TILE = KA * ATOM;          // one [128 tokens x D] tile
  static constexpr int STAGE = 2 * TILE;          // a stage: tiles of two tensors
  static constexpr int OFF_RING = 2 * TILE;       // after the CTA's own two tiles
  static constexpr int OFF_LD = OFF_RING + NST * STAGE;  // per stage: lse * log2e, delta of 128 queries
  static constexpr int OFF_BAR = OFF_LD + NST * 2 * BT * 4;
  static constexpr int SMEM_BYTES = OFF_BAR + 256 + 1024;  // + barriers, + 1024-byte alignment
};

struct Bars {
  uint64_t fixed_full;       // the CTA's own two tiles (K, V or Q, dO)
  uint64_t ring_full[NST];   // streamed units of a stage
  uint64_t ring_empty[NST];
  uint64_t ld_full[NST];     // lse / delta vectors of a stage (kv kernel)
  uint64_t s_full[2];        // scores and dP of column half h of a tile in tensor memory
  uint64_t p_full[2];        // their 16-bit products written back
  uint64_t acc_full;
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

// K-major operand (rows = tokens from row0, K = dims): the MMA's 16 dims k.
__device__ __forceinline__ uint64_t kmajor(uint32_t tile, int row0, int k) {
  return sw128_kmajor_desc(tile + (k >> 2) * ATOM + row0 * 128 + (k & 3) * 32);
}
// MN-major operand (K = tokens, N = dims): the MMA's 16 tokens from row0.
__device__ __forceinline__ uint64_t mnmajor(uint32_t tile, int row0) {
  return sw128_desc(tile + row0 * 128, ATOM, 1024);
}

// Items, heaviest first: kv CTAs for the first key tiles see the most queries
// (causal), q CTAs for the last query tiles see the most keys.
struct KvItem {
  int b, g, k0, t0, nt;  // query tiles [t0, t0 + nt) of each head of the group
};
__device__ __forceinline__ KvItem kv_item(int idx, int B, int Hkv, int T, int W) {
  KvItem it;
  const int per = B * Hkv;
  const int kt = idx / per, r = idx % per;
  it.b = r / Hkv;
  it.g = r % Hkv;
  it.k0 = kt * BT;
  const int k_last = min(T - 1, it.k0 + BT - 1);
  it.t0 = it.k0 / BT;
  it.nt = min(T - 1, k_last + W - 1) / BT - it.t0 + 1;
  return it;
}
struct QItem {
  int b, h, q0, t0, nt;  // key tiles [t0, t0 + nt)
};
__device__ __forceinline__ QItem q_item(int idx, int B, int H, int T, int W) {
  QItem it;
  const int per = B * H;
  const int nqt = (T + BT - 1) / BT;
  const int qt = nqt - 1 - idx / per, r = idx % per;
  it.b = r / H;
  it.h = r % H;
  it.q0 = qt * BT;
  const int q_last = min(T - 1, it.q0 + BT - 1);
  it.t0 = max(0, it.q0 - W + 1) / BT;
  it.nt = q_last / BT - it.t0 + 1;
  return it;
}

// Let every TMA load this thread started land before the CTA exits.
__device__ __forceinline__ void drain_loads(const Bars* bar, int n_issued, uint64_t limit_ns) {
  int zero = 0;
  const WaitCtl dctl{&zero, nullptr, limit_ns};
  mbar_wait(smem_u32(&bar->fixed_full), 0, dctl);
  for (int u = n_issued - NST < 0 ? 0 : n_issued - NST; u < n_issued; ++u)
    mbar_wait(smem_u32(&bar->ring_full[u % NST]), (uint32_t)(u / NST) & 1u, dctl);
}

__device__ __forceinline__ void init_bars(Bars* bar) {
  mbar_init(smem_u32(&bar->fixed_full), 1);
  for (int s = 0; s < NST; ++s) {
    mbar_init(smem_u32(&bar->ring_full[s]), 1);
    mbar_init(smem_u32(&bar->ring_empty[s]), 1);
    mbar_init(smem_u32(&bar->ld_full[s]), 32);
  }
  for (int h = 0; h < 2; ++h) {
    mbar_init(smem_u32(&bar->s_full[h]), 1);
    mbar_init(smem_u32(&bar->p_full[h]), 4);
  }
  mbar_init(smem_u32(&bar->acc_full), 1);
  mbar_init(smem_u32(&bar->drain), 1);
  bar->abort_flag = 0;
  fence_mbar_init();
}

// The MMA issuer's schedule, the same in both kernels: for each streamed tile
// i and column half h, first the products that read half h of tile i - 1
// (`grads(i - 1, h)`, once its 16-bit results are written), then the two score
// products of half h of tile i (`scores(i, h)`) over the same columns; the
// tensor core executes in issue order, so the former have read them by then.
template <class Scores, class Grads>
__device__ __forceinline__ bool mma_schedule(Bars* bar, int n, const WaitCtl& ctl, Scores scores, Grads grads) {
  for (int i = 0; i < n; ++i) {
    if (!mbar_wait(smem_u32(&bar->ring_full[i % NST]), (uint32_t)(i / NST) & 1u, ctl)) return false;
    tc_fence_after();
    for (int h = 0; h < 2; ++h) {
      if (i > 0) {
        if (!mbar_wait(smem_u32(&bar->p_full[h]), (uint32_t)(i - 1) & 1u, ctl)) return false;
        tc_fence_after();
        grads(i - 1, h);
        if (h == 1) umma_commit(smem_u32(&bar->ring_empty[(i - 1) % NST]));
      }
      scores(i, h);
      umma_commit(smem_u32(&bar->s_full[h]));
    }
  }
  for (int h = 0; h < 2 && n > 0; ++h) {
    if (!mbar_wait(smem_u32(&bar->p_full[h]), (uint32_t)(n - 1) & 1u, ctl)) return false;
    tc_fence_after();
    grads(n - 1, h);
  }
  umma_commit(smem_u32(&bar->acc_full));
  return true;
}

// 4-byte asynchronous copy global -> shared (zero when !in).
__device__ __forceinline__ void cp_async4(float* dst, const float* src, bool in) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(in ? 4 : 0)
               : "memory");
}
// Arrive on `bar` once this thread's earlier asynchronous copies have landed.
__device__ __forceinline__ void cp_async_arrive(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

template <int D, bool F16>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    attn_bwd_kv_kernel(const __grid_constant__ CUtensorMap tmQKV, const __grid_constant__ CUtensorMap tmDO,
                       const float* __restrict__ lse, const float* __restrict__ delta_t,
                       uint16_t* __restrict__ dqkv, int64_t ldqkv, int B, int T, int H, int Hkv, int W,
                       float scale, uint32_t* dev_status, uint64_t limit_ns) {
  using G = Geo<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  const uint32_t s_base = smem_u32(sm);
  const uint32_t sK = s_base, sV = s_base + G::TILE;
  auto sQt = [&](int st) { return s_base + G::OFF_RING + st * G::STAGE; };
  auto sDOt = [&](int st) { return s_base + G::OFF_RING + st * G::STAGE + G::TILE; };
  float* sLD = reinterpret_cast<float*>(sm + G::OFF_LD);  // [stage][lse | delta][128]
  Bars* bar = reinterpret_cast<Bars*>(sm + G::OFF_BAR);
  const uint32_t warp = warp_id_sync();
  const uint32_t lane = lane_id();
  const KvItem it = kv_item(blockIdx.x, B, Hkv, T, W);
  const int Gq = H / Hkv;
  const int n = Gq * it.nt;  // streamed tiles: (query head of the group, 128 queries)

  if (threadIdx.x == 0) init_bars(bar);
  if (warp == 1) {
    tmem_alloc(smem_u32(&bar->tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar->tmem_base;
  const WaitCtl ctl{&bar->abort_flag, dev_status, limit_ns};
  // tensor memory: S^T / P^T [0, 128), dP^T / dS^T [128, 256), dV, dK accumulators
  const uint32_t tS = tmem, tP = tmem + 128, tdV = tmem + 256, tdK = tmem + 256 + D;

  if (warp == 0) {
    // ---------------- producer: K, V once; per tile Q, dO (TMA) and the 128
    // queries' lse and delta (asynchronous 4-byte copies, four per lane)
    bool ok = true;
    int n_issued = 0;
    if (lane == 0) {
      prefetch_tmap(&tmQKV);
      prefetch_tmap(&tmDO);
      const uint32_t fb = smem_u32(&bar->fixed_full);
      mbar_arrive_expect_tx(fb, 2 * G::TILE);
      for (int a = 0; a < G::KA; ++a) {
        tma_load_4d(sK + a * ATOM, &tmQKV, a * 64, H + it.g, it.k0, it.b, fb);
        tma_load_4d(sV + a * ATOM, &tmQKV, a * 64, H + Hkv + it.g, it.k0, it.b, fb);
      }
    }
    for (int i = 0; i < n; ++i) {
      const int st = i % NST;
      const int hq = it.g * Gq + i / it.nt, q0 = (it.t0 + i % it.nt) * BT;
      const bool freed = mbar_wait(smem_u32(&bar->ring_empty[st]), ((uint32_t)(i / NST) & 1u) ^ 1u, ctl);
      if (__any_sync(0xffffffffu, !freed)) {
        ok = false;
        break;
      }
      if (lane == 0) {
        const uint32_t rb = smem_u32(&bar->ring_full[st]);
        mbar_arrive_expect_tx(rb, G::STAGE);
        for (int a = 0; a < G::KA; ++a) {
          tma_load_4d(sQt(st) + a * ATOM, &tmQKV, a * 64, hq, q0, it.b, rb);
          tma_load_4d(sDOt(st) + a * ATOM, &tmDO, a * 64, hq, q0, it.b, rb);
        }
      }
      ++n_issued;
      float* l = sLD + st * 2 * BT;
      for (int r = (int)lane; r < BT; r += 32) {
        const int iq = q0 + r;
        const bool in = iq < T;
        const int64_t m = (int64_t)it.b * T + (in ? iq : 0);
        cp_async4(l + r, lse + m * H + hq, in);
        cp_async4(l + BT + r, delta_t + ((int64_t)it.b * H + hq) * T + (in ? iq : 0), in);
      }
      cp_async_arrive(smem_u32(&bar->ld_full[st]));
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    if (lane == 0 && (!ok || bar->abort_flag)) drain_loads(bar, n_issued, limit_ns);
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer
      constexpr uint32_t IS = idesc_f32acc(128, 64, F16);     // a 64-column half of S^T or dP^T
      constexpr uint32_t IG = idesc_f32acc_bmn(128, D, F16);  // dV, dK: B = the tile, MN-major
      if (mbar_wait(smem_u32(&bar->fixed_full), 0, ctl)) {
        tc_fence_after();
        auto scores = [&](int i, int h) {
          const int st = i % NST;
#pragma unroll
          for (int k = 0; k < D / 16; ++k)
            umma_f16(tS + 64 * h, kmajor(sK, 0, k), kmajor(sQt(st), 64 * h, k), IS, k > 0 ? 1u : 0u);
#pragma unroll
          for (int k = 0; k < D / 16; ++k)
            umma_f16(tP + 64 * h, kmajor(sV, 0, k), kmajor(sDOt(st), 64 * h, k), IS, k > 0 ? 1u : 0u);
        };
        // dV += P^T dO and dK += dS^T Q over the 64 queries of half h of tile i
        auto grads = [&](int i, int h) {
          const int st = i % NST;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t acc = (i > 0 || h > 0 || kk > 0) ? 1u : 0u;
            umma_f16_ts(tdV, tS + 64 * h + 8 * kk, mnmajor(sDOt(st), 64 * h + 16 * kk), IG, acc);
            umma_f16_ts(tdK, tP + 64 * h + 8 * kk, mnmajor(sQt(st), 64 * h + 16 * kk), IG, acc);
          }
        };
        mma_schedule(bar, n, ctl, scores, grads);
      }
      umma_commit(smem_u32(&bar->drain));
      int zero = 0;
      const WaitCtl dctl{&zero, nullptr, limit_ns};
      mbar_wait(smem_u32(&bar->drain), 0, dctl);
    }
  } else {
    // ---------------- softmax warps: lane quarter `quarter` (32 keys), query half h
    const uint32_t quarter = warp & 3u;
    const int h = (int)(warp - 2) / 4;
    const uint32_t lane_off = (quarter * 32u) << 16;
    const int j = it.k0 + (int)(quarter * 32 + lane);  // this thread's key
    const int jhi = j < T ? min(T - 1, j + W - 1) : -1;  // it is seen by queries [j, jhi]
    bool ok = true;
    for (int i = 0; i < n && ok; ++i) {
      const int st = i % NST;
      const int q0 = (it.t0 + i % it.nt) * BT;
      bool got = mbar_wait(smem_u32(&bar->s_full[h]), (uint32_t)i & 1u, ctl);
      got = got && mbar_wait(smem_u32(&bar->ld_full[st]), (uint32_t)(i / NST) & 1u, ctl);
      if (__any_sync(0xffffffffu, !got)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float* l = sLD + st * 2 * BT;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {  // 16 queries at a time
        const int qb = 64 * h + 16 * c;  // first query of this chunk within the tile
        uint32_t rs[16], rp[16];
        tmem_ld_32x32b_x16(tS + lane_off + qb, rs);
        tmem_ld_32x32b_x16(tP + lane_off + qb, rp);
        // the chunk's lse and delta, the same for every lane (broadcast reads)
        float lv[16], dl[16];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float4 a = reinterpret_cast<const float4*>(l + qb)[q];
          const float4 b = reinterpret_cast<const float4*>(l + BT + qb)[q];
          lv[4 * q] = a.x, lv[4 * q + 1] = a.y, lv[4 * q + 2] = a.z, lv[4 * q + 3] = a.w;
          dl[4 * q] = b.x, dl[4 * q + 1] = b.y, dl[4 * q + 2] = b.z, dl[4 * q + 3] = b.w;
        }
        const int lo = j - q0 - qb, hi = jhi - q0 - qb;  // visible e: lo <= e <= hi
        tmem_wait_ld();
        uint32_t wp[8], wd[8];
#pragma unroll
        for (int e = 0; e < 16; e += 2) {
          float p[2], d[2];
#pragma unroll
          for (int v = 0; v < 2; ++v) {
            const bool vis = e + v >= lo && e + v <= hi;
            // exp(s x - lse) in base 2
            const float pv = vis ? ex2(fmaf(__uint_as_float(rs[e + v]), scale, -lv[e + v]) * kLog2e) : 0.0f;
            p[v] = pv;
            d[v] = pv * (__uint_as_float(rp[e + v]) - dl[e + v]);
          }
          wp[e / 2] = Half<F16>::pack2(p[0], p[1]);
          wd[e / 2] = Half<F16>::pack2(d[0], d[1]);
        }
        // 16-bit P^T and dS^T over the columns this chunk's scores came from
        tmem_st_x8(tS + lane_off + 64 * h + 8 * c, wp);
        tmem_st_x8(tP + lane_off + 64 * h + 8 * c, wd);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bar->p_full[h]));
    }
    // ---------------- epilogue: dV and s dK of this warp's 32 keys, dims [h D/2, (h+1) D/2)
    if (ok) ok = !__any_sync(0xffffffffu, !mbar_wait(smem_u32(&bar->acc_full), 0, ctl));
    if (ok) {
      tc_fence_after();
      uint16_t* rowp = dqkv + ((int64_t)it.b * T + (j < T ? j : 0)) * ldqkv;
#pragma unroll 1
      for (int c = 0; c < D / 64; ++c) {
        const int d0 = h * (D / 2) + 32 * c;
        uint32_t rv[32], rk[32];
        tmem_ld_32x32b_x32(tdV + lane_off + d0, rv);
        tmem_ld_32x32b_x32(tdK + lane_off + d0, rk);
        tmem_wait_ld();
        if (j < T) {
          uint4* ov = reinterpret_cast<uint4*>(rowp + (int64_t)(H + Hkv + it.g) * D + d0);
          uint4* ok4 = reinterpret_cast<uint4*>(rowp + (int64_t)(H + it.g) * D + d0);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 v, k;
            v.x = Half<F16>::pack2(__uint_as_float(rv[8 * q + 0]), __uint_as_float(rv[8 * q + 1]));
            v.y = Half<F16>::pack2(__uint_as_float(rv[8 * q + 2]), __uint_as_float(rv[8 * q + 3]));
            v.z = Half<F16>::pack2(__uint_as_float(rv[8 * q + 4]), __uint_as_float(rv[8 * q + 5]));
            v.w = Half<F16>::pack2(__uint_as_float(rv[8 * q + 6]), __uint_as_float(rv[8 * q + 7]));
            k.x = Half<F16>::pack2(__uint_as_float(rk[8 * q + 0]) * scale, __uint_as_float(rk[8 * q + 1]) * scale);
            k.y = Half<F16>::pack2(__uint_as_float(rk[8 * q + 2]) * scale, __uint_as_float(rk[8 * q + 3]) * scale);
            k.z = Half<F16>::pack2(__uint_as_float(rk[8 * q + 4]) * scale, __uint_as_float(rk[8 * q + 5]) * scale);
            k.w = Half<F16>::pack2(__uint_as_float(rk[8 * q + 6]) * scale, __uint_as_float(rk[8 * q + 7]) * scale);
            ov[q] = v;
            ok4[q] = k;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

template <int D, bool F16>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    attn_bwd_q_kernel(const __grid_constant__ CUtensorMap tmQKV, const __grid_constant__ CUtensorMap tmDO,
                      const float* __restrict__ lse,
                      const float* __restrict__ delta_t, uint16_t* __restrict__ dqkv, int64_t ldqkv, int B, int T,
                      int H, int Hkv, int W, float scale, uint32_t* dev_status, uint64_t limit_ns) {
  using G = Geo<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  const uint32_t s_base = smem_u32(sm);
  const uint32_t sQ = s_base, sDO = s_base + G::TILE;
  auto sKt = [&](int st) { return s_base + G::OFF_RING + st * G::STAGE; };
  auto sVt = [&](int st) { return s_base + G::OFF_RING + st * G::STAGE + G::TILE; };
  Bars* bar = reinterpret_cast<Bars*>(sm + G::OFF_BAR);
  const uint32_t warp = warp_id_sync();
  const uint32_t lane = lane_id();
  const QItem it = q_item(blockIdx.x, B, H, T, W);
  const int g = it.h / (H / Hkv);  // kv head
  const int n = it.nt;              // key tiles

  if (threadIdx.x == 0) init_bars(bar);
  if (warp == 1) {
    tmem_alloc(smem_u32(&bar->tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar->tmem_base;
  const WaitCtl ctl{&bar->abort_flag, dev_status, limit_ns};
  // tensor memory: S halves [0, 128), dP / dS halves [128, 256), dQ accumulator
  const uint32_t tS = tmem, tP = tmem + 128, tdQ = tmem + 256;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- producer: Q, dO once; K, V per unit
      prefetch_tmap(&tmQKV);
      prefetch_tmap(&tmDO);
      const uint32_t fb = smem_u32(&bar->fixed_full);
      mbar_arrive_expect_tx(fb, 2 * G::TILE);
      for (int a = 0; a < G::KA; ++a) {
        tma_load_4d(sQ + a * ATOM, &tmQKV, a * 64, it.h, it.q0, it.b, fb);
        tma_load_4d(sDO + a * ATOM, &tmDO, a * 64, it.h, it.q0, it.b, fb);
      }
      bool ok = true;
      int n_issued = 0;
      for (int i = 0; i < n; ++i) {
        const int st = i % NST;
        if (!mbar_wait(smem_u32(&bar->ring_empty[st]), ((uint32_t)(i / NST) & 1u) ^ 1u, ctl)) {
          ok = false;
          break;
        }
        const uint32_t rb = smem_u32(&bar->ring_full[st]);
        mbar_arrive_expect_tx(rb, G::STAGE);
        const int k0 = (it.t0 + i) * BT;
        for (int a = 0; a < G::KA; ++a) {
          tma_load_4d(sKt(st) + a * ATOM, &tmQKV, a * 64, H + g, k0, it.b, rb);
          tma_load_4d(sVt(st) + a * ATOM, &tmQKV, a * 64, H + Hkv + g, k0, it.b, rb);
        }
        ++n_issued;
      }
      if (!ok || bar->abort_flag) drain_loads(bar, n_issued, limit_ns);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer
      constexpr uint32_t IS = idesc_f32acc(128, 64, F16);     // a 64-column half of S or dP
      constexpr uint32_t IG = idesc_f32acc_bmn(128, D, F16);  // dQ: B = the K tile, MN-major
      if (mbar_wait(smem_u32(&bar->fixed_full), 0, ctl)) {
        tc_fence_after();
        auto scores = [&](int i, int h) {
          const int st = i % NST;
#pragma unroll
          for (int k = 0; k < D / 16; ++k)
            umma_f16(tS + 64 * h, kmajor(sQ, 0, k), kmajor(sKt(st), 64 * h, k), IS, k > 0 ? 1u : 0u);
#pragma unroll
          for (int k = 0; k < D / 16; ++k)
            umma_f16(tP + 64 * h, kmajor(sDO, 0, k), kmajor(sVt(st), 64 * h, k), IS, k > 0 ? 1u : 0u);
        };
        // dQ += dS K over the 64 keys of half h of tile i
        auto grads = [&](int i, int h) {
          const int st = i % NST;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_f16_ts(tdQ, tP + 64 * h + 8 * kk, mnmajor(sKt(st), 64 * h + 16 * kk), IG,
                    (i > 0 || h > 0 || kk > 0) ? 1u : 0u);
        };
        mma_schedule(bar, n, ctl, scores, grads);
      }
      umma_commit(smem_u32(&bar->drain));
      int zero = 0;
      const WaitCtl dctl{&zero, nullptr, limit_ns};
      mbar_wait(smem_u32(&bar->drain), 0, dctl);
    }
  } else {
    // ---------------- softmax warps: lane quarter `quarter` (32 queries), key half h
    const uint32_t quarter = warp & 3u;
    const int h = (int)(warp - 2) / 4;
    const uint32_t lane_off = (quarter * 32u) << 16;
    const int i_q = it.q0 + (int)(quarter * 32 + lane);  // this thread's query
    const bool q_in = i_q < T;
    // it sees keys [jlo, jhi] (none when past the sequence)
    const int jlo = q_in ? max(0, i_q - W + 1) : 1, jhi = q_in ? i_q : 0;
    const float c1 = scale * kLog2e;
    const float lse2 = q_in ? lse[((int64_t)it.b * T + i_q) * H + it.h] * kLog2e : 0.0f;
    const float dlt = q_in ? delta_t[((int64_t)it.b * H + it.h) * T + i_q] : 0.0f;
    bool ok = true;
    for (int i = 0; i < n && ok; ++i) {
      const int k0 = (it.t0 + i) * BT + 64 * h;  // first key of this half
      if (__any_sync(0xffffffffu, !mbar_wait(smem_u32(&bar->s_full[h]), (uint32_t)i & 1u, ctl))) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        uint32_t rs[32], rp[32];
        tmem_ld_32x32b_x32(tS + lane_off + 64 * h + 32 * c, rs);
        tmem_ld_32x32b_x32(tP + lane_off + 64 * h + 32 * c, rp);
        tmem_wait_ld();
        const int ka = k0 + 32 * c;                    // first key of this chunk
        uint32_t wd[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          float d[2];
#pragma unroll
          for (int v = 0; v < 2; ++v) {
            const int jk = ka + e + v;
            const bool vis = jk >= jlo && jk <= jhi;
            const float pv = vis ? ex2(fmaf(__uint_as_float(rs[e + v]), c1, -lse2)) : 0.0f;
            d[v] = pv * (__uint_as_float(rp[e + v]) - dlt);
          }
          wd[e / 2] = Half<F16>::pack2(d[0], d[1]);
        }
        tmem_st_x16(tP + lane_off + 64 * h + 16 * c, wd);  // 16-bit dS over its dP columns
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bar->p_full[h]));
    }
    // ---------------- epilogue: s dQ of this warp's 32 queries, dims [h D/2, (h+1) D/2)
    if (ok) ok = !__any_sync(0xffffffffu, !mbar_wait(smem_u32(&bar->acc_full), 0, ctl));
    if (ok) {
      tc_fence_after();
      uint16_t* rowp = dqkv + ((int64_t)it.b * T + (q_in ? i_q : 0)) * ldqkv + (int64_t)it.h * D;
#pragma unroll 1
      for (int c = 0; c < D / 64; ++c) {
        const int d0 = h * (D / 2) + 32 * c;
        uint32_t rq[32];
        tmem_ld_32x32b_x32(tdQ + lane_off + d0, rq);
        tmem_wait_ld();
        if (q_in) {
          uint4* o4 = reinterpret_cast<uint4*>(rowp + d0);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 v;
            v.x = Half<F16>::pack2(__uint_as_float(rq[8 * q + 0]) * scale, __uint_as_float(rq[8 * q + 1]) * scale);
            v.y = Half<F16>::pack2(__uint_as_float(rq[8 * q + 2]) * scale, __uint_as_float(rq[8 * q + 3]) * scale);
            v.z = Half<F16>::pack2(__uint_as_float(rq[8 * q + 4]) * scale, __uint_as_float(rq[8 * q + 5]) * scale);
            v.w = Half<F16>::pack2(__uint_as_float(rq[8 * q + 6]) * scale, __uint_as_float(rq[8 * q + 7]) * scale);
            o4[q] = v;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// delta_t[b, h, t] = sum_d dO[b, t, h, d] O[b, t, h, d]; D / 8 lanes per
// (token, head), 16 bytes of each tensor per lane.
template <int D, bool F16>
__global__ void __launch_bounds__(256) delta_kernel(const uint16_t* __restrict__ dO, const uint16_t* __restrict__ O,
                                                    float* __restrict__ delta_t, int B, int T, int H) {
  constexpr int LPH = D / 8;  // lanes per head
  const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t unit = gid / LPH;  // (token, head)
  const bool active = unit < (int64_t)B * T * H;
  float s = 0.0f;
  if (active) {
    const uint4 a = *reinterpret_cast<const uint4*>(dO + gid * 8);
    const uint4 o = *reinterpret_cast<const uint4*>(O + gid * 8);
    const uint32_t av[4] = {a.x, a.y, a.z, a.w}, ov[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 x = Half<F16>::unpack2(av[e]), y = Half<F16>::unpack2(ov[e]);
      s = fmaf(x.x, y.x, fmaf(x.y, y.y, s));
    }
  }
#pragma unroll
  for (int off = LPH / 2; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if (active && gid % LPH == 0) {
    const int64_t m = unit / H;
    const int h = (int)(unit % H);
    const int b = (int)(m / T), t = (int)(m % T);
    delta_t[((int64_t)b * H + h) * T + t] = s;
  }
}

// 4-D map over a [B, T, heads, D] 16-bit tensor with `row_stride` elements
// between consecutive tokens; box = 64 dims x 1 head x `rows` tokens x 1 row.
static bool make_map(CUtensorMap* map, const void* base, int B, int T, int heads, int D, int64_t row_stride,
                     int rows, bool f16) {
  const uint64_t dims[4] = {(uint64_t)D, (uint64_t)heads, (uint64_t)T, (uint64_t)B};
  const uint64_t strides[3] = {(uint64_t)D * 2, (uint64_t)row_stride * 2, (uint64_t)T * (uint64_t)row_stride * 2};
  const uint32_t box[4] = {64, 1, (uint32_t)rows, 1};
  return encode_tensor_map(map, f16, 4, base, dims, strides, box);
}

template <int D, bool F16>
static nc_status launch_t(const uint16_t* qkv, int64_t ldqkv, const uint16_t* dO, const float* lse,
                          const float* delta_t, uint16_t* dqkv, int B, int T, int H, int Hkv, int W,
                          uint32_t* dev_status, uint64_t limit_ns, cudaStream_t stream) {
  using G = Geo<D>;
  static bool attr_done[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return NC_ERR_CUDA;
  if (!attr_done[dev]) {
    if (cudaFuncSetAttribute(attn_bwd_kv_kernel<D, F16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             G::SMEM_BYTES) != cudaSuccess ||
        cudaFuncSetAttribute(attn_bwd_q_kernel<D, F16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             G::SMEM_BYTES) != cudaSuccess)
      return NC_ERR_CUDA;
    attr_done[dev] = true;
  }
  CUtensorMap mqkv, mdo;
  if (!make_map(&mqkv, qkv, B, T, H + 2 * Hkv, D, ldqkv, BT, F16) ||
      !make_map(&mdo, dO, B, T, H, D, (int64_t)H * D, BT, F16))
    return NC_ERR_CUDA;
  const float scale = 1.0f / sqrtf((float)D);
  const int nt = (T + BT - 1) / BT;
  attn_bwd_kv_kernel<D, F16><<<nt * B * Hkv, NUM_THREADS, G::SMEM_BYTES, stream>>>(
      mqkv, mdo, lse, delta_t, dqkv, ldqkv, B, T, H, Hkv, W, scale, dev_status, limit_ns);
  if (cudaGetLastError() != cudaSuccess) return NC_ERR_CUDA;
  attn_bwd_q_kernel<D, F16><<<nt * B * H, NUM_THREADS, G::SMEM_BYTES, stream>>>(
      mqkv, mdo, lse, delta_t, dqkv, ldqkv, B, T, H, Hkv, W, scale, dev_status, limit_ns);
  return cudaGetLastError() == cudaSuccess ? NC_OK : NC_ERR_CUDA;
}

}  // namespace attn_bwd

nc_status attn_bwd_launch(const uint16_t* qkv, int64_t ldqkv, const uint16_t* o, const uint16_t* dO,
                          const float* lse, float* delta, uint16_t* dqkv, int B, int T, int H, int Hkv, int D,
                          int window, bool f16, cudaStream_t stream, uint32_t* dev_status, uint64_t limit_ns) {
  using namespace attn_bwd;
  if (B == 0 || T == 0) return NC_OK;
  if (D != 64 && D != 128) return NC_ERR_SHAPE;
  if (ldqkv % 8) return NC_ERR_ALIGNMENT;  // TMA: 16-byte token stride
  const int64_t threads = (int64_t)B * T * H * (D / 8);
  const unsigned grid = (unsigned)((threads + 255) / 256);
  if (D == 128) {
    if (f16)
      delta_kernel<128, true><<<grid, 256, 0, stream>>>(dO, o, delta, B, T, H);
    else
      delta_kernel<128, false><<<grid, 256, 0, stream>>>(dO, o, delta, B, T, H);
  } else {
    if (f16)
      delta_kernel<64, true><<<grid, 256, 0, stream>>>(dO, o, delta, B, T, H);
    else
      delta_kernel<64, false><<<grid, 256, 0, stream>>>(dO, o, delta, B, T, H);
  }
  if (cudaGetLastError() != cudaSuccess) return NC_ERR_CUDA;
  const int W = (window <= 0 || window > T) ? T : window;
  if (D == 128)
    return f16 ? launch_t<128, true>(qkv, ldqkv, dO, lse, delta, dqkv, B, T, H, Hkv, W, dev_status, limit_ns, stream)
               : launch_t<128, false>(qkv, ldqkv, dO, lse, delta, dqkv, B, T, H, Hkv, W, dev_status, limit_ns, stream);
  return f16 ? launch_t<64, true>(qkv, ldqkv, dO, lse, delta, dqkv, B, T, H, Hkv, W, dev_status, limit_ns, stream)
             : launch_t<64, false>(qkv, ldqkv, dO, lse, delta, dqkv, B, T, H, Hkv, W, dev_status, limit_ns, stream);
}

}  // namespace nc
