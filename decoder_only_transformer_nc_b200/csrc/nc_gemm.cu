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
//   warps 2..5  epilogue: tcgen05.ld of the accumulator (each warp owns the 32
//               TMEM lanes = tile rows its warp index selects), fused epilogue
//               op, direct global stores; then hand the accumulator back.
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
constexpr int NUM_THREADS = 192;
constexpr int EPI_WARPS = 4;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;
constexpr uint32_t IDESC = idesc_bf16_f32(BM, BN);

struct Smem {  // barrier block placed after the tile ring
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tmem_full[NUM_ACC];
  uint64_t tmem_empty[NUM_ACC];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(Smem) <= 256, "barrier block");

template <int EPI>
__device__ __forceinline__ void epilogue_chunk(const uint32_t (&r)[32], int row, int col0, int N,
                                               const EpiParams& ep, float& ce_sum, float& ce_tl,
                                               int target) {
  float v[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
  if constexpr (EPI == EPI_STORE_BF16 || EPI == EPI_RELU2_BF16) {
    if constexpr (EPI == EPI_RELU2_BF16) {
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float t = fmaxf(v[i], 0.0f);
        v[i] = t * t;
      }
    }
    __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(ep.out) + (int64_t)row * ep.ldo + col0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint4 pk;
      __nv_bfloat162 h0 = __floats2bfloat162_rn(v[8 * j + 0], v[8 * j + 1]);
      __nv_bfloat162 h1 = __floats2bfloat162_rn(v[8 * j + 2], v[8 * j + 3]);
      __nv_bfloat162 h2 = __floats2bfloat162_rn(v[8 * j + 4], v[8 * j + 5]);
      __nv_bfloat162 h3 = __floats2bfloat162_rn(v[8 * j + 6], v[8 * j + 7]);
      pk.x = *reinterpret_cast<uint32_t*>(&h0);
      pk.y = *reinterpret_cast<uint32_t*>(&h1);
      pk.z = *reinterpret_cast<uint32_t*>(&h2);
      pk.w = *reinterpret_cast<uint32_t*>(&h3);
      reinterpret_cast<uint4*>(o)[j] = pk;
    }
  } else if constexpr (EPI == EPI_RESID_F32) {
    float* o = reinterpret_cast<float*>(ep.out) + (int64_t)row * ep.ldo + col0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      float4 x = reinterpret_cast<float4*>(o)[j];
      x.x += v[4 * j + 0];
      x.y += v[4 * j + 1];
      x.z += v[4 * j + 2];
      x.w += v[4 * j + 3];
      reinterpret_cast<float4*>(o)[j] = x;
    }
  } else if constexpr (EPI == EPI_STORE_F32 || EPI == EPI_SOFTCAP_F32) {
    if constexpr (EPI == EPI_SOFTCAP_F32) {
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = ep.cap * tanhf(v[i] / ep.cap);
    }
    float* o = reinterpret_cast<float*>(ep.out) + (int64_t)row * ep.ldo + col0;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      reinterpret_cast<float4*>(o)[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
  } else if constexpr (EPI == EPI_CE_PARTIAL) {
    // Soft-capped logits l in (-cap, cap): exp(l - cap) never overflows, so the
    // per-tile partial sums combine by plain addition.
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const float l = ep.cap * tanhf(v[i] / ep.cap);
      v[i] = l;
      ce_sum += __expf(l - ep.cap);
    }
    const int rel = target - col0;
    if (rel >= 0 && rel < 32) {
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (i == rel) ce_tl = v[i];
    }
    if (ep.store_logits) {
      float* o = reinterpret_cast<float*>(ep.out) + (int64_t)row * ep.ldo + col0;
#pragma unroll
      for (int j = 0; j < 8; ++j)
        reinterpret_cast<float4*>(o)[j] =
            make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
    }
  }
}

template <int EPI>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                int M, int N, int K, EpiParams ep, uint32_t* dev_status, uint64_t limit_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  Smem* sm = reinterpret_cast<Smem*>(tiles + STAGES * STAGE_BYTES);

  const uint32_t warp = warp_id_sync();
  const uint32_t lane = lane_id();
  const int num_m = (M + BM - 1) / BM;
  const int num_n = (N + BN - 1) / BN;
  const int num_tiles = num_m * num_n;
  const int num_kb = (K + BK - 1) / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&sm->full[s]), 1);
      mbar_init(smem_u32(&sm->empty[s]), 1);
    }
    for (int a = 0; a < NUM_ACC; ++a) {
      mbar_init(smem_u32(&sm->tmem_full[a]), 1);
      mbar_init(smem_u32(&sm->tmem_empty[a]), EPI_WARPS);
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
    tmem_alloc(smem_u32(&sm->tmem_base), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
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
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int m0 = (tile / num_n) * BM;
        const int n0 = (tile % num_n) * BN;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(smem_u32(&sm->empty[stage]), phase ^ 1u, ctl)) {
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(&sm->full[stage]);
          mbar_arrive_expect_tx(fb, STAGE_BYTES);
          uint8_t* a_dst = tiles + stage * STAGE_BYTES;
          tma_load_2d(smem_u32(a_dst), &tmA, kb * BK, m0, fb);
          tma_load_2d(smem_u32(a_dst + A_BYTES), &tmB, kb * BK, n0, fb);
          outstanding |= 1u << stage;
          out_phase = (out_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok || sm->abort_flag) {
        // Let every copy this thread started land before the CTA exits.
        int zero = 0;
        const WaitCtl drain_ctl{&zero, nullptr, limit_ns};
        for (int s = 0; s < STAGES; ++s)
          if (outstanding & (1u << s))
            mbar_wait(smem_u32(&sm->full[s]), (out_phase >> s) & 1u, drain_ctl);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- UMMA issuer
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        if (!mbar_wait(smem_u32(&sm->tmem_empty[acc]), acc_phase ^ 1u, ctl)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(smem_u32(&sm->full[stage]), phase, ctl)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(tiles + stage * STAGE_BYTES);
          const uint32_t b_addr = a_addr + A_BYTES;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t adesc = sw128_kmajor_desc(a_addr + k * 32);
            const uint64_t bdesc = sw128_kmajor_desc(b_addr + k * 32);
            umma_bf16(d_tmem, adesc, bdesc, IDESC, (kb | k) != 0 ? 1u : 0u);
          }
          umma_commit(smem_u32(&sm->empty[stage]));
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(smem_u32(&sm->tmem_full[acc]));
        if (++acc == NUM_ACC) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      // Wait until every MMA this thread issued has completed.
      umma_commit(smem_u32(&sm->drain));
      int zero = 0;
      WaitCtl drain_ctl{&zero, nullptr, limit_ns};
      mbar_wait(smem_u32(&sm->drain), 0, drain_ctl);
    }
  } else {
    // ---------------- epilogue warps
    const uint32_t quarter = warp & 3u;
    const int row_in_tile = quarter * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      const int m_blk = tile / num_n;
      const int n_blk = tile % num_n;
      const int m0 = m_blk * BM;
      const int n0 = n_blk * BN;
      if (!mbar_wait(smem_u32(&sm->tmem_full[acc]), acc_phase, ctl)) break;
      tc_fence_after();
      const int row = m0 + row_in_tile;
      const uint32_t taddr = tmem_base + ((quarter * 32u) << 16) + acc * BN;
      float ce_sum = 0.0f, ce_tl = 0.0f;
      int target = -1;
      if constexpr (EPI == EPI_CE_PARTIAL) {
        if (row < M) target = ep.targets ? ep.targets[row] : -1;
      }
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        const int col0 = n0 + c * 32;
        if (col0 >= N) break;  // warp-uniform
        uint32_t r[32];
        tmem_ld_32x32b_x32(taddr + c * 32, r);
        tmem_wait_ld();
        if (row < M) epilogue_chunk<EPI>(r, row, col0, N, ep, ce_sum, ce_tl, target);
      }
      if constexpr (EPI == EPI_CE_PARTIAL) {
        if (row < M) {
          ep.ce_partial[(int64_t)row * num_n + n_blk] = ce_sum;
          if (target >= n0 && target < n0 + BN && target < N) ep.ce_target[row] = ce_tl;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sm->tmem_empty[acc]));
      if (++acc == NUM_ACC) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, TMEM_COLS);
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

// bf16 row-major [rows, cols] with row stride `ld` elements; box = 64 x box_rows.
static bool make_map(CUtensorMap* map, const void* ptr, int64_t rows, int64_t cols, int64_t ld,
                     int box_rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(ld * 2)};
  cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int EPI>
static cudaError_t launch_t(const CUtensorMap& ma, const CUtensorMap& mb, int M, int N, int K,
                            const EpiParams& ep, uint32_t* dev_status, uint64_t limit_ns,
                            cudaStream_t stream) {
  static bool attr_done[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_done[dev]) {
    cudaError_t e = cudaFuncSetAttribute(gemm_kernel<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_done[dev] = true;
  }
  const int tiles = ((M + BM - 1) / BM) * ((N + BN - 1) / BN);
  const int sms = device_sm_count();
  const int grid = tiles < sms ? tiles : sms;
  gemm_kernel<EPI><<<grid, NUM_THREADS, SMEM_BYTES, stream>>>(ma, mb, M, N, K, ep, dev_status,
                                                              limit_ns);
  return cudaGetLastError();
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

nc_status selftest_wait_launch(uint32_t* dev_status, uint64_t limit_ns, cudaStream_t stream) {
  gemm::selftest_wait_kernel<<<1, 32, 0, stream>>>(dev_status, limit_ns);
  return cudaGetLastError() == cudaSuccess ? NC_OK : NC_ERR_CUDA;
}

int gemm_num_n_tiles(int N) { return (N + gemm::BN - 1) / gemm::BN; }

nc_status gemm_launch(const uint16_t* a, int64_t lda, const uint16_t* w, int64_t ldw, int M, int N,
                      int K, int epi, const EpiParams& ep, uint32_t* dev_status,
                      cudaStream_t stream, uint64_t limit_ns) {
  using namespace gemm;
  CUtensorMap ma, mb;
  if (!make_map(&ma, a, M, K, lda, BM)) return NC_ERR_CUDA;
  if (!make_map(&mb, w, N, K, ldw, BN)) return NC_ERR_CUDA;
  cudaError_t e;
  switch (epi) {
    case EPI_STORE_BF16: e = launch_t<EPI_STORE_BF16>(ma, mb, M, N, K, ep, dev_status, limit_ns, stream); break;
    case EPI_RELU2_BF16: e = launch_t<EPI_RELU2_BF16>(ma, mb, M, N, K, ep, dev_status, limit_ns, stream); break;
    case EPI_RESID_F32: e = launch_t<EPI_RESID_F32>(ma, mb, M, N, K, ep, dev_status, limit_ns, stream); break;
    case EPI_STORE_F32: e = launch_t<EPI_STORE_F32>(ma, mb, M, N, K, ep, dev_status, limit_ns, stream); break;
    case EPI_SOFTCAP_F32: e = launch_t<EPI_SOFTCAP_F32>(ma, mb, M, N, K, ep, dev_status, limit_ns, stream); break;
    case EPI_CE_PARTIAL: e = launch_t<EPI_CE_PARTIAL>(ma, mb, M, N, K, ep, dev_status, limit_ns, stream); break;
    default: return NC_ERR_INVALID_ARG;
  }
  return e == cudaSuccess ? NC_OK : NC_ERR_CUDA;
}

}  // namespace nc
