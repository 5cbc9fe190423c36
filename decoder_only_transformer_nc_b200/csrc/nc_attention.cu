// Causal sliding-window attention with GQA on the 5th-generation tensor cores
// ("从文本到聊天模型" §5.4-5.5; window pattern and GQA from "Nanochat与nanoGPT对比：
// 关键升级" §1).
//
//   o[b,i,h,:] = sum_{j visible} softmax_j(q[b,i,h,:].k[b,j,g,:] / sqrt(D)) v[b,j,g,:]
//   visible: j <= i and i - j < W;  g = h / (H / Hkv)
//
// Work items are (128-query block, head, batch row).  The grid holds one CTA
// per item, but a running CTA cancels the launch of a CTA that has not started
// and takes its item (cluster launch control), so in effect one CTA per SM
// runs and items go to whichever SM frees up first.  Warp roles:
//   warp 0     TMA: the item's Q tile, then K and V tiles of 128 keys into two
//              2-slot rings (4-D tensor maps over [B, T, heads, D]: tokens past
//              T read as zeros, so tiles never leak into the next sequence).
//              A K slot is released as soon as its S = Q K^T has completed and a
//              V slot after its P V, so the next K tile loads while the softmax
//              of the current one runs;
//   warp 1     owns 512 TMEM columns; one thread issues S = Q K^T (M=128,
//              N=128 keys) into one of two S buffers, then O += P V (A = P read
//              from tensor memory, B = V read MN-major from shared memory) into
//              one of two O accumulators (item n uses accumulator n & 1);
//   warps 2-9  softmax: each TMEM lane quarter (32 query rows, one per thread)
//              is served by two warps that own 64 of the tile's 128 keys; they
//              swap partial row maxima (and, at the end, row sums) through
//              shared memory.  Mask the window/causal edge only on tiles that
//              straddle it (one visible-column interval per row), online
//              softmax in fp32 with exp2, write P (16-bit, two keys per
//              column) back over the first half of its own S columns, where
//              the P V product reads it (the S that next overwrites the buffer
//              is issued after that product); O is rescaled in TMEM only
//              when the running row maximum grows by more than 2^8 in the
//              exponent (P stays <= 256, exact in fp16).  The output O / l of
//              an item is written after the first tile of the next item has
//              gone to the MMA warp, so neither the last P V nor the store
//              stalls the softmax: staged in shared memory, TMA-stored.
// Only key tiles intersecting [q0 - W + 1, q0 + 127] are visited.
// Every wait is bounded; on timeout the CTA records NC_DEV_TIMEOUT, drains
// its copies and MMAs, frees its tensor memory and exits.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>

#include "nc_half.cuh"
#include "nc_internal.h"
#include "nc_ptx.cuh"

namespace nc {
namespace attn {

constexpr int BQ = 128;   // query rows per work item
constexpr int BKV = 128;  // keys per tile
constexpr int SM_WARPS = 8;  // softmax warps: two per TMEM lane quarter, 64 keys each
constexpr int NUM_THREADS = 64 + 32 * SM_WARPS;
constexpr int ATOM = 128 * 128;  // bytes of one [128 rows][64 x 16-bit] swizzle tile
constexpr float kRescaleLog2 = 8.0f;

template <int D>
struct Geo {
  static constexpr int KA = D / 64;                  // 64-wide swizzle atoms along D
  static constexpr int Q_BYTES = KA * ATOM;
  static constexpr int KV_STAGE = 2 * KA * ATOM;     // K then V
  static constexpr int P_BYTES = (BKV / 64) * ATOM;  // [128 rows][128 keys]
  static constexpr int OFF_KV = Q_BYTES;
  static constexpr int OFF_P = OFF_KV + 2 * KV_STAGE;
  static constexpr int OFF_BAR = OFF_P + 2 * P_BYTES;
  static constexpr int OFF_X = OFF_BAR + 512;       // row-statistics exchange [2 slots][2 halves][128]
  static constexpr int SMEM_BYTES = OFF_X + 2 * 2 * 128 * 4;
};

struct Bars {
  uint32_t next_item[2][4];  // work-request answers (16 B each, 16-byte aligned)
  uint64_t next_full[2];     // answer n & 1 has landed
  uint64_t next_empty[2];    // every role has read answer n & 1
  uint64_t q_full, q_empty;
  uint64_t k_full[2], k_empty[2];
  uint64_t v_full[2], v_empty[2];
  uint64_t s_full[2], s_free[2];
  uint64_t p_full[2], p_free[2];
  uint64_t o_free[2];  // O accumulator n & 1 has been read out for item n
  uint64_t xbar[4];  // per lane quarter: both column halves posted their row statistics
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(Bars) <= 512, "barrier block");
constexpr int kNextReaders = 2 + SM_WARPS;  // TMA thread, MMA thread, softmax warps

// Dynamic work distribution.  The grid has one CTA per work item.  While a
// CTA works on an item it asks the hardware scheduler to cancel the launch of
// a CTA that has not started yet (cluster launch control) and, if that
// succeeds, takes over that CTA's item next.  Items are thus handed out in
// launch order to whichever SM frees up first, while each SM keeps its
// barriers, tensor memory and pipelines across items.  One request is in
// flight at a time and none is issued after one has failed.
__device__ __forceinline__ void next_item_request(uint32_t answer, uint32_t bar) {
  asm volatile("clusterlaunchcontrol.try_cancel.async.shared::cta.mbarrier::complete_tx::bytes.b128 [%0], [%1];"
               ::"r"(answer), "r"(bar)
               : "memory");
}

// Item index carried by an answer, or -1 when no launch was cancelled.
__device__ __forceinline__ int next_item_decode(uint32_t answer, int n_items) {
  uint32_t got = 0, x = 0, y = 0, z = 0;
  asm volatile(
      "{\n\t"
      ".reg .pred p;\n\t"
      ".reg .b128 r;\n\t"
      "ld.shared.b128 r, [%4];\n\t"
      "clusterlaunchcontrol.query_cancel.is_canceled.pred.b128 p, r;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t"
      "@p clusterlaunchcontrol.query_cancel.get_first_ctaid.v4.b32.b128 {%1, %2, %3, _}, r;\n\t"
      "}"
      : "+r"(got), "+r"(x), "+r"(y), "+r"(z)
      : "r"(answer)
      : "memory");
  return (got && (int)x < n_items) ? (int)x : -1;
}

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

struct Item {
  int b, h, q0, kt0, n_tiles;
};

// Items are numbered with the query block fastest (last block first), then the
// head, then the batch row.  They are handed out in about that order, so the
// CTAs running at the same time cover all query blocks of a few heads (each
// head's K/V is fetched from HBM about once and then served from L2), and
// within a head the longest items go first, which keeps the tail short.
__device__ __forceinline__ Item item_of(int idx, int B, int H, int T, int W) {
  const int n_qb = (T + BQ - 1) / BQ;
  Item it;
  const int qb = n_qb - 1 - idx % n_qb;
  idx /= n_qb;
  it.h = idx % H;
  it.b = idx / H;
  it.q0 = qb * BQ;
  const int lo = max(0, it.q0 - W + 1);
  const int hi = min(T, it.q0 + BQ) - 1;
  it.kt0 = lo / BKV;
  it.n_tiles = hi / BKV - it.kt0 + 1;
  return it;
}

template <int D, bool F16>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                   uint16_t* __restrict__ out, int B,
                   int T, int H, int Hkv, int W, float scale_log2, uint32_t* dev_status,
                   uint64_t limit_ns, float* __restrict__ amax, float* __restrict__ lse_out) {
  using G = Geo<D>;
  constexpr uint32_t IDESC_S = idesc_f32acc(BQ, BKV, F16);
  constexpr uint32_t IDESC_PV = idesc_f32acc_bmn(BQ, D, F16);
  constexpr uint32_t TMEM_COLS = 512;
  constexpr uint32_t O_COL = 2 * BKV;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // The swizzled tiles need a 1024-byte aligned base; the dynamic window starts
  // aligned in practice.  If it ever does not, fail cleanly instead of faulting.
  if ((smem_u32(smem_raw) & 1023u) != 0) {
    if (threadIdx.x == 0 && dev_status) atomicOr(dev_status, NC_DEV_SMEM_ALIGN);
    return;
  }
  uint8_t* sm = smem_raw;
  float* xval = reinterpret_cast<float*>(sm + G::OFF_X);
  Bars* bar = reinterpret_cast<Bars*>(sm + G::OFF_BAR);
  const uint32_t s_q = smem_u32(sm);
  const uint32_t s_kv = s_q + G::OFF_KV;
  const uint32_t s_p = s_q + G::OFF_P;

  const uint32_t warp = warp_id_sync();
  const uint32_t lane = lane_id();
  const int n_qb = (T + BQ - 1) / BQ;
  const int n_items = B * H * n_qb;
  const int group = H / Hkv;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&bar->next_full[i]), 1);
      mbar_init(smem_u32(&bar->next_empty[i]), kNextReaders);
    }
    mbar_init(smem_u32(&bar->q_full), 1);
    mbar_init(smem_u32(&bar->q_empty), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&bar->k_full[i]), 1);
      mbar_init(smem_u32(&bar->k_empty[i]), 1);
      mbar_init(smem_u32(&bar->v_full[i]), 1);
      mbar_init(smem_u32(&bar->v_empty[i]), 1);
      mbar_init(smem_u32(&bar->s_full[i]), 1);
      mbar_init(smem_u32(&bar->s_free[i]), SM_WARPS);
      mbar_init(smem_u32(&bar->p_full[i]), SM_WARPS);
      mbar_init(smem_u32(&bar->p_free[i]), 1);
    }
    mbar_init(smem_u32(&bar->o_free[0]), SM_WARPS);
    mbar_init(smem_u32(&bar->o_free[1]), SM_WARPS);
    for (int i = 0; i < 4; ++i) mbar_init(smem_u32(&bar->xbar[i]), 2);
    mbar_init(smem_u32(&bar->drain), 1);
    bar->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&bar->tmem_base), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar->tmem_base;
  const WaitCtl ctl{&bar->abort_flag, dev_status, limit_ns};

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer
      uint32_t outstanding = 0, out_phase = 0;  // bits 0,1: K slots; bit 2: Q; bits 3,4: V slots
      int g = 0;
      bool ok = true;
      bool asked = false;  // a work request is in flight (answer slot ask_slot, phase ask_phase)
      int ask_slot = 0;
      uint32_t ask_phase = 0;
      int idx = blockIdx.x;
      for (int n = 0; idx >= 0 && ok; ++n) {
        const Item it = item_of(idx, B, H, T, W);
        const int gh = it.h / group;
        const int ns = n & 1;
        // Ask for the next item now; the answer is read once this item is loaded.
        if (!mbar_wait(smem_u32(&bar->next_empty[ns]), ((uint32_t)(n >> 1) & 1) ^ 1, ctl)) break;
        mbar_arrive_expect_tx(smem_u32(&bar->next_full[ns]), 16);
        next_item_request(smem_u32(&bar->next_item[ns][0]), smem_u32(&bar->next_full[ns]));
        asked = true;
        ask_slot = ns;
        ask_phase = (uint32_t)(n >> 1) & 1;
        if (!mbar_wait(smem_u32(&bar->q_empty), (n & 1) ^ 1, ctl)) break;
        mbar_arrive_expect_tx(smem_u32(&bar->q_full), G::Q_BYTES);
        for (int a = 0; a < G::KA; ++a)
          tma_load_4d(s_q + a * ATOM, &tmQ, a * 64, it.h, it.q0, it.b, smem_u32(&bar->q_full));
        outstanding |= 4u;
        out_phase = (out_phase & ~4u) | ((uint32_t)(n & 1) << 2);
        // V runs one tile behind K (K0, K1, V0, K2, V1, ...): a K load waits only
        // for the S two tiles back, never for a P V.
        for (int j = 0; j <= it.n_tiles; ++j) {
          if (j < it.n_tiles) {
            const int gk = g + j;
            const int st = gk & 1;
            const uint32_t use = (uint32_t)(gk >> 1);
            if (!mbar_wait(smem_u32(&bar->k_empty[st]), (use & 1) ^ 1, ctl)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(smem_u32(&bar->k_full[st]), G::KA * ATOM);
            for (int a = 0; a < G::KA; ++a)
              tma_load_4d(s_kv + st * G::KV_STAGE + a * ATOM, &tmK, a * 64, gh, (it.kt0 + j) * BKV, it.b,
                          smem_u32(&bar->k_full[st]));
            outstanding |= 1u << st;
            out_phase = (out_phase & ~(1u << st)) | ((use & 1) << st);
          }
          if (j > 0) {
            const int gv = g + j - 1;
            const int st = gv & 1;
            const uint32_t use = (uint32_t)(gv >> 1);
            if (!mbar_wait(smem_u32(&bar->v_empty[st]), (use & 1) ^ 1, ctl)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(smem_u32(&bar->v_full[st]), G::KA * ATOM);
            for (int a = 0; a < G::KA; ++a)
              tma_load_4d(s_kv + st * G::KV_STAGE + (G::KA + a) * ATOM, &tmV, a * 64, gh,
                          (it.kt0 + j - 1) * BKV, it.b, smem_u32(&bar->v_full[st]));
            outstanding |= 8u << st;
            out_phase = (out_phase & ~(8u << st)) | ((use & 1) << (3 + st));
          }
        }
        g += it.n_tiles;
        if (!ok) break;
        if (!mbar_wait(smem_u32(&bar->next_full[ns]), (uint32_t)(n >> 1) & 1, ctl)) break;
        asked = false;
        idx = next_item_decode(smem_u32(&bar->next_item[ns][0]), n_items);
        fence_proxy_async_smem();
        mbar_arrive(smem_u32(&bar->next_empty[ns]));
      }
      if (!ok || bar->abort_flag) {
        int zero = 0;
        const WaitCtl dctl{&zero, nullptr, limit_ns};
        if (asked) mbar_wait(smem_u32(&bar->next_full[ask_slot]), ask_phase, dctl);
        for (int st = 0; st < 2; ++st) {
          if (outstanding & (1u << st)) mbar_wait(smem_u32(&bar->k_full[st]), (out_phase >> st) & 1u, dctl);
          if (outstanding & (8u << st))
            mbar_wait(smem_u32(&bar->v_full[st]), (out_phase >> (3 + st)) & 1u, dctl);
        }
        if (outstanding & 4u) mbar_wait(smem_u32(&bar->q_full), (out_phase >> 2) & 1u, dctl);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer
      int g = 0;
      bool ok = true;
      int idx = blockIdx.x;
      for (int n = 0; idx >= 0 && ok; ++n) {
        const Item it = item_of(idx, B, H, T, W);
        if (!mbar_wait(smem_u32(&bar->q_full), n & 1, ctl)) break;
        tc_fence_after();
        for (int j = 0; j <= it.n_tiles && ok; ++j) {
          if (j < it.n_tiles) {
            const int gj = g + j;
            const int sb = gj & 1;
            const uint32_t use = (uint32_t)(gj >> 1);
            if (!mbar_wait(smem_u32(&bar->k_full[sb]), use & 1, ctl) ||
                !mbar_wait(smem_u32(&bar->s_free[sb]), (use & 1) ^ 1, ctl)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t kbase = s_kv + sb * G::KV_STAGE;
#pragma unroll
            for (int k = 0; k < D / 16; ++k) {
              const uint32_t off = (k >> 2) * ATOM + (k & 3) * 32;
              umma_f16(tmem + sb * BKV, sw128_kmajor_desc(s_q + off), sw128_kmajor_desc(kbase + off),
                       IDESC_S, k > 0 ? 1u : 0u);
            }
            umma_commit(smem_u32(&bar->s_full[sb]));
            umma_commit(smem_u32(&bar->k_empty[sb]));
            if (j == it.n_tiles - 1) umma_commit(smem_u32(&bar->q_empty));
          }
          if (j > 0) {
            const int gp = g + j - 1;
            const int pb = gp & 1;
            const uint32_t use = (uint32_t)(gp >> 1);
            if (!mbar_wait(smem_u32(&bar->p_full[pb]), use & 1, ctl) ||
                !mbar_wait(smem_u32(&bar->v_full[pb]), use & 1, ctl)) {
              ok = false;
              break;
            }
            if (j == 1 && !mbar_wait(smem_u32(&bar->o_free[n & 1]), ((uint32_t)(n >> 1) & 1) ^ 1, ctl)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t vbase = s_kv + pb * G::KV_STAGE + G::KA * ATOM;
            // P (16-bit, two keys per column) sits over the first 32 columns of
            // each key half of S buffer pb
#pragma unroll
            for (int k = 0; k < BKV / 16; ++k) {
              const uint64_t bdesc = sw128_desc(vbase + k * 2048, ATOM, 1024);
              umma_f16_ts(tmem + O_COL + (n & 1) * D, tmem + pb * BKV + 64 * (k >> 2) + 8 * (k & 3), bdesc, IDESC_PV,
                      (j > 1 || k > 0) ? 1u : 0u);
            }
            umma_commit(smem_u32(&bar->p_free[pb]));
            umma_commit(smem_u32(&bar->v_empty[pb]));
          }
        }
        g += it.n_tiles;
        if (!ok) break;
        const int ns = n & 1;
        if (!mbar_wait(smem_u32(&bar->next_full[ns]), (uint32_t)(n >> 1) & 1, ctl)) break;
        idx = next_item_decode(smem_u32(&bar->next_item[ns][0]), n_items);
        fence_proxy_async_smem();
        mbar_arrive(smem_u32(&bar->next_empty[ns]));
      }
      umma_commit(smem_u32(&bar->drain));
      int zero = 0;
      const WaitCtl dctl{&zero, nullptr, limit_ns};
      mbar_wait(smem_u32(&bar->drain), 0, dctl);
    }
  } else {
    // ---------------- softmax / correction / epilogue
    const uint32_t quarter = warp & 3u;
    const int half = (int)(warp - 2) / 4;  // which 64 keys of each tile (and D/2 of O)
    const int r = (int)(quarter * 32 + lane);
    const uint32_t lane_off = (quarter * 32u) << 16;
    const float thresh = kRescaleLog2 / scale_log2;  // in raw score units
    constexpr int KC = BKV / 2;                       // keys per warp and tile
    constexpr int DC = D / 2;                         // O columns per warp
    uint32_t xphase = 0;  // exchanges done by this warp (same count in its partner)
    // Post v for this row, wait for the partner half, return the partner's value.
    auto exchange = [&](float v, bool& ok_) -> float {
      const int slot = xphase & 1;
      xval[(slot * 2 + half) * 128 + r] = v;
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bar->xbar[quarter]));
      const bool got = mbar_wait(smem_u32(&bar->xbar[quarter]), xphase & 1u, ctl);
      ++xphase;
      if (__any_sync(0xffffffffu, !got)) {
        ok_ = false;
        return 0.0f;
      }
      return xval[(slot * 2 + (half ^ 1)) * 128 + r];
    };
    // The output of item n is written while item n + 1 runs: once the first
    // tile of n + 1 has been handed to the MMA warp, the last P V of n has had
    // a tile's worth of softmax time to land in O buffer n & 1, and the TMA
    // store stages in the P buffer of n's last tile, which the next tile of
    // n + 1 does not use.
    struct Pending {
      int b, h, q0, gl, ob;
      float l, m;
    };
    Pending pend{};
    bool has_pend = false;
    uint32_t store_busy = 0;  // P buffers a TMA store of this warp may still be reading
    uint32_t om = 0;          // max |output| of this thread's rows (bits), for *amax
    auto track = [&](float a) { om = max(om, __float_as_uint(a) & 0x7FFFFFFFu); };
    auto finish = [&](const Pending& pd, bool& ok_) {
      const float lsum = pd.l + exchange(pd.l, ok_);  // full row sum
      if (!ok_) return;
      if (__any_sync(0xffffffffu,
                     !mbar_wait(smem_u32(&bar->p_free[pd.gl & 1]), (uint32_t)(pd.gl >> 1) & 1, ctl))) {
        ok_ = false;
        return;
      }
      tc_fence_after();
      const float inv = lsum > 0.0f ? 1.0f / lsum : 0.0f;
      // natural log-sum-exp of the row's scaled scores (kept for the backward)
      if (lse_out && half == 0 && pd.q0 + r < T)
        lse_out[((int64_t)pd.b * T + pd.q0 + r) * H + pd.h] = pd.m * (scale_log2 * 0.6931471805599453f) + logf(lsum);
      const uint32_t ocol = O_COL + pd.ob * D + half * DC;
      uint32_t rr[DC / 32][32];
#pragma unroll
      for (int c = 0; c < DC / 32; ++c) tmem_ld_32x32b_x32(tmem + lane_off + ocol + c * 32, rr[c]);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bar->o_free[pd.ob]));
      if constexpr (D == 128) {
        // Stage this warp's 32 rows x 64 columns in the P buffer of the item's
        // last tile (only this warp writes these rows of this half) and let
        // TMA write them to out.
        uint8_t* sbase = sm + G::OFF_P + (pd.gl & 1) * G::P_BYTES + half * ATOM;
        uint8_t* srow = sbase + r * 128;
        if (store_busy & (1u << (pd.gl & 1))) {  // an earlier output store still reads this buffer
          if (lane == 0) bulk_wait_read0();
          __syncwarp();
          store_busy = 0;
        }
        if (amax && pd.q0 + r < T) {
#pragma unroll
          for (int c = 0; c < DC / 32; ++c)
#pragma unroll
            for (int e = 0; e < 32; ++e) track(__uint_as_float(rr[c][e]) * inv);
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          uint4 pk;
          const int c = q >> 2, e0 = (q & 3) * 8;
          pk.x = Half<F16>::pack2(__uint_as_float(rr[c][e0 + 0]) * inv, __uint_as_float(rr[c][e0 + 1]) * inv);
          pk.y = Half<F16>::pack2(__uint_as_float(rr[c][e0 + 2]) * inv, __uint_as_float(rr[c][e0 + 3]) * inv);
          pk.z = Half<F16>::pack2(__uint_as_float(rr[c][e0 + 4]) * inv, __uint_as_float(rr[c][e0 + 5]) * inv);
          pk.w = Half<F16>::pack2(__uint_as_float(rr[c][e0 + 6]) * inv, __uint_as_float(rr[c][e0 + 7]) * inv);
          *reinterpret_cast<uint4*>(srow + ((q ^ (r & 7)) << 4)) = pk;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_4d(&tmO, smem_u32(sbase + quarter * 32 * 128), half * DC, pd.h, pd.q0 + (int)quarter * 32,
                       pd.b);
          bulk_commit();
        }
        store_busy |= 1u << (pd.gl & 1);
      } else {
        const int i = pd.q0 + r;
        if (i < T) {
          if (amax) {
#pragma unroll
            for (int c = 0; c < DC / 32; ++c)
#pragma unroll
              for (int e = 0; e < 32; ++e) track(__uint_as_float(rr[c][e]) * inv);
          }
          uint16_t* orow = out + (((int64_t)pd.b * T + i) * H + pd.h) * D + half * DC;
#pragma unroll
          for (int q = 0; q < DC / 8; ++q) {
            uint4 pk;
            const int c = q >> 2, e0 = (q & 3) * 8;
            pk.x = Half<F16>::pack2(__uint_as_float(rr[c][e0 + 0]) * inv, __uint_as_float(rr[c][e0 + 1]) * inv);
            pk.y = Half<F16>::pack2(__uint_as_float(rr[c][e0 + 2]) * inv, __uint_as_float(rr[c][e0 + 3]) * inv);
            pk.z = Half<F16>::pack2(__uint_as_float(rr[c][e0 + 4]) * inv, __uint_as_float(rr[c][e0 + 5]) * inv);
            pk.w = Half<F16>::pack2(__uint_as_float(rr[c][e0 + 6]) * inv, __uint_as_float(rr[c][e0 + 7]) * inv);
            reinterpret_cast<uint4*>(orow)[q] = pk;
          }
        }
      }
    };
    int g = 0;
    bool ok = true;
    int idx = blockIdx.x;
    for (int n = 0; idx >= 0 && ok; ++n) {
      const Item it = item_of(idx, B, H, T, W);
      const int i = it.q0 + r;  // this thread's query position
      const uint32_t ocol = O_COL + (n & 1) * D + half * DC;
      float m_used = -INFINITY, l = 0.0f;
      for (int j = 0; j < it.n_tiles; ++j) {
        const int gj = g + j;
        const int sb = gj & 1;
        const uint32_t use = (uint32_t)(gj >> 1);
        if (__any_sync(0xffffffffu, !mbar_wait(smem_u32(&bar->s_full[sb]), use & 1, ctl))) {
          ok = false;
          break;
        }
        tc_fence_after();
        float s[KC];
        {
          uint32_t rr[KC / 32][32];
#pragma unroll
          for (int c = 0; c < KC / 32; ++c)
            tmem_ld_32x32b_x32(tmem + lane_off + sb * BKV + half * KC + c * 32, rr[c]);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < KC / 32; ++c)
#pragma unroll
            for (int e = 0; e < 32; ++e) s[c * 32 + e] = __uint_as_float(rr[c][e]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bar->s_free[sb]));

        const int k0 = (it.kt0 + j) * BKV + half * KC;  // first key of this warp's columns
        const bool full = (k0 + KC - 1 <= it.q0) && (it.q0 + BQ - 1 - k0 < W);
        if (!full) {
          // visible columns of this row: lo <= c <= hi  (j <= i and i - j < W)
          const int lo = i - W + 1 - k0;
          const int hi = i - k0;
#pragma unroll
          for (int c = 0; c < KC; ++c) s[c] = (c >= lo && c <= hi) ? s[c] : -INFINITY;
        }
        float mx8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) mx8[e] = s[e];
#pragma unroll
        for (int c = 8; c < KC; ++c) mx8[c & 7] = fmaxf(mx8[c & 7], s[c]);
        float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                         fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
        mx = fmaxf(mx, exchange(mx, ok));  // both halves now hold the row maximum
        if (!ok) break;
        const float m_new = fmaxf(m_used, mx);
        bool need = false;
        if (m_used == -INFINITY) {
          m_used = m_new;  // O and l are still zero for this row
        } else if (m_new > m_used + thresh) {
          need = true;
        }
        if (__any_sync(0xffffffffu, need)) {
          // Rescale this warp's half of the O row; the previous P V must have landed.
          const int gp = gj - 1;
          const bool landed = mbar_wait(smem_u32(&bar->p_free[gp & 1]), (uint32_t)(gp >> 1) & 1, ctl);
          if (__any_sync(0xffffffffu, !landed)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const float alpha = need ? ex2f((m_used - m_new) * scale_log2) : 1.0f;
#pragma unroll 1
          for (int c = 0; c < DC / 32; ++c) {
            uint32_t rr[32];
            tmem_ld_32x32b_x32(tmem + lane_off + ocol + c * 32, rr);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) rr[e] = __float_as_uint(__uint_as_float(rr[e]) * alpha);
            tmem_st_32x32b_x32(tmem + lane_off + ocol + c * 32, rr);
          }
          tmem_wait_st();
          if (need) {
            l *= alpha;
            m_used = m_new;
          }
        }
        const float ms = (m_used == -INFINITY) ? 0.0f : m_used * scale_log2;
        // P goes back over the first 32 columns of this warp's half of S
        // buffer sb (two 16-bit values per column), already read into s[]; the
        // MMA warp issues the S that next overwrites the buffer only after the
        // P V that reads it.
        float ls8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};  // 8 independent sums
        uint32_t pk[KC / 2];
#pragma unroll
        for (int c = 0; c < KC / 8; ++c) {
          float p[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            p[e] = ex2f(fmaf(s[c * 8 + e], scale_log2, -ms));
            ls8[e] += p[e];
          }
#pragma unroll
          for (int e = 0; e < 4; ++e) pk[4 * c + e] = Half<F16>::pack2(p[2 * e], p[2 * e + 1]);
        }
        l += ((ls8[0] + ls8[1]) + (ls8[2] + ls8[3])) + ((ls8[4] + ls8[5]) + (ls8[6] + ls8[7]));
        tmem_st_32x32b_x32(tmem + lane_off + sb * BKV + half * KC, pk);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bar->p_full[sb]));
        if (j == 0 && has_pend) {
          has_pend = false;
          finish(pend, ok);
          if (!ok) break;
        }
      }
      if (!ok) break;
      pend = Pending{it.b, it.h, it.q0, g + it.n_tiles - 1, n & 1, l, m_used};
      has_pend = true;
      g += it.n_tiles;
      const int ns = n & 1;
      if (__any_sync(0xffffffffu, !mbar_wait(smem_u32(&bar->next_full[ns]), (uint32_t)(n >> 1) & 1, ctl))) {
        ok = false;
        break;
      }
      idx = next_item_decode(smem_u32(&bar->next_item[ns][0]), n_items);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bar->next_empty[ns]));
    }
    if (ok && has_pend) finish(pend, ok);
    if (amax) {
      om = __reduce_max_sync(0xFFFFFFFFu, om);
      if (lane == 0) fold_amax(amax, stored_abs_bits<F16>(om));
    }
    if (lane == 0) bulk_wait0();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, TMEM_COLS);
}

// 4-D map over a [B, T, heads, D] 16-bit tensor with `row_stride` elements
// between consecutive tokens; box = 64 dims x 1 head x 128 tokens x 1 row.
static bool make_map4(CUtensorMap* map, const void* base, int B, int T, int heads, int D,
                      int64_t row_stride, bool f16) {
  const uint64_t dims[4] = {(uint64_t)D, (uint64_t)heads, (uint64_t)T, (uint64_t)B};
  const uint64_t strides[3] = {(uint64_t)D * 2, (uint64_t)row_stride * 2,
                               (uint64_t)T * (uint64_t)row_stride * 2};
  const uint32_t box[4] = {64, 1, (uint32_t)BKV, 1};
  return encode_tensor_map(map, f16, 4, base, dims, strides, box);
}

template <int D, bool F16>
static nc_status launch_t(const uint16_t* q, const uint16_t* k, const uint16_t* v, uint16_t* out,
                          int B, int T, int H, int Hkv, int W, int64_t q_stride, int64_t kv_stride,
                          uint32_t* dev_status, cudaStream_t stream, float* amax, float* lse) {
  using G = Geo<D>;
  static bool attr_done[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_done[dev]) {
    if (cudaFuncSetAttribute(attn_tc_kernel<D, F16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             G::SMEM_BYTES) != cudaSuccess)
      return NC_ERR_CUDA;
    attr_done[dev] = true;
  }
  CUtensorMap mq, mk, mv, mo;
  if (!make_map4(&mq, q, B, T, H, D, q_stride, F16) || !make_map4(&mk, k, B, T, Hkv, D, kv_stride, F16) ||
      !make_map4(&mv, v, B, T, Hkv, D, kv_stride, F16))
    return NC_ERR_CUDA;
  memset(&mo, 0, sizeof(mo));
  if (D == 128) {  // out [B, T, H, D]: boxes of 64 dims x 32 tokens (one softmax warp's rows)
    const uint64_t dims[4] = {(uint64_t)D, (uint64_t)H, (uint64_t)T, (uint64_t)B};
    const uint64_t strides[3] = {(uint64_t)D * 2, (uint64_t)H * D * 2, (uint64_t)T * H * D * 2};
    const uint32_t box[4] = {64, 1, 32, 1};
    if (!encode_tensor_map(&mo, F16, 4, out, dims, strides, box)) return NC_ERR_CUDA;
  }
  // One CTA per work item; running CTAs take over the items of CTAs that have
  // not started (see next_item_request), so about one CTA per SM ever runs.
  const int grid = B * H * ((T + BQ - 1) / BQ);
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)D);
  attn_tc_kernel<D, F16><<<grid, NUM_THREADS, G::SMEM_BYTES, stream>>>(
      mq, mk, mv, mo, out, B, T, H, Hkv, W, scale_log2, dev_status, kWaitLimitNs, amax, lse);
  return cudaGetLastError() == cudaSuccess ? NC_OK : NC_ERR_CUDA;
}

}  // namespace attn

nc_status attention_launch(const uint16_t* q, const uint16_t* k, const uint16_t* v, uint16_t* out,
                           int B, int T, int H, int Hkv, int D, int window, int64_t q_stride,
                           int64_t kv_stride, bool f16, uint32_t* dev_status, cudaStream_t stream,
                           float* amax, float* lse) {
  if (lse)  // the backward's log-sum-exp: the run-to-run reproducible kernel
    return attention_lse_launch(q, k, v, out, B, T, H, Hkv, D, window, q_stride, kv_stride, f16, dev_status,
                                stream, amax, lse);
  if (D != 64 && D != 128) return NC_ERR_SHAPE;
  if (B == 0 || T == 0) return NC_OK;
  const int W = (window <= 0 || window > T) ? T : window;
  if (D == 128)
    return f16 ? attn::launch_t<128, true>(q, k, v, out, B, T, H, Hkv, W, q_stride, kv_stride, dev_status, stream,
                                           amax, lse)
               : attn::launch_t<128, false>(q, k, v, out, B, T, H, Hkv, W, q_stride, kv_stride, dev_status,
                                            stream, amax, lse);
  return f16 ? attn::launch_t<64, true>(q, k, v, out, B, T, H, Hkv, W, q_stride, kv_stride, dev_status, stream,
                                        amax, lse)
             : attn::launch_t<64, false>(q, k, v, out, B, T, H, Hkv, W, q_stride, kv_stride, dev_status, stream,
                                         amax, lse);
}

}  // namespace nc
