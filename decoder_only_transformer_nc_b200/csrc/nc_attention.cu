// Causal sliding-window attention with GQA ("从文本到聊天模型" §5.4-5.5;
// window pattern and GQA from "Nanochat与nanoGPT对比：关键升级" §1).
//
//   o[b,i,h,:] = sum_{j visible} softmax_j(q[b,i,h,:].k[b,j,g,:] / sqrt(D)) v[b,j,g,:]
//   visible: j <= i and i - j < W;  g = h / (H / Hkv)
//
// One CTA per (128-query block, head, batch row); 8 warps x 16 query rows.
// K/V tiles of 64 keys are double-buffered in shared memory with cp.async
// (XOR-swizzled 16-byte chunks, conflict-free ldmatrix).  Only the key tiles
// that intersect [q0 - W + 1, q0 + 127] are visited, so short-window layers
// cost O(T * W) instead of O(T^2); the mask is evaluated only on tiles that
// straddle the causal diagonal or the window edge.  Online softmax in fp32
// registers (exp2 with the 1/sqrt(D) * log2(e) scale folded in); P is reused
// from the score registers as the bf16 A operand of P.V.
#include <cuda_runtime.h>

#include <cstdint>

#include "nc_half.cuh"
#include "nc_internal.h"

namespace nc {
namespace attn {

constexpr int BQ = 128;
constexpr int BKV = 64;
constexpr int NWARPS = 8;
constexpr int NTHREADS = NWARPS * 32;

template <int D>
struct Geo {
  static constexpr int ROW_BYTES = D * 2;
  static constexpr int CHUNKS = D / 8;  // 16-byte chunks per row
  static constexpr int Q_BYTES = BQ * ROW_BYTES;
  static constexpr int KV_BYTES = BKV * ROW_BYTES;
  static constexpr int SMEM_BYTES = Q_BYTES + 4 * KV_BYTES;  // Q + 2x K + 2x V
};

// Byte offset of 16-byte chunk `chunk` of row `row`: the chunk index is XOR-ed
// with the row's low 3 bits so the 8 rows of one ldmatrix hit 8 distinct banks.
template <int D>
__device__ __forceinline__ uint32_t swz(int row, int chunk) {
  return (uint32_t)(row * Geo<D>::ROW_BYTES + ((chunk ^ (row & 7)) << 4));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;  // 0 source bytes -> zero fill
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

template <bool F16>
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  if constexpr (F16) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
}

// Copies `rows` token rows (D bf16 each) starting at token r0 into a swizzled
// tile; rows at or beyond T are zero-filled.
template <int D>
__device__ __forceinline__ void load_tile(uint32_t s_base, const uint16_t* g, int64_t stride, int r0,
                                          int rows, int T) {
  constexpr int CH = Geo<D>::CHUNKS;
  const int chunks = rows * CH;
  for (int c = threadIdx.x; c < chunks; c += NTHREADS) {
    const int r = c / CH;
    const int ch = c % CH;
    const int tok = r0 + r;
    const bool valid = tok < T;
    const uint16_t* src = g + (int64_t)(valid ? tok : 0) * stride + ch * 8;
    cp_async16(s_base + swz<D>(r, ch), src, valid);
  }
}

// F16: q, k, v, P and the output in fp16 (else bf16).
template <int D, bool F16>
__global__ void __launch_bounds__(NTHREADS, 1)
    attn_fwd_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
                    const uint16_t* __restrict__ v, uint16_t* __restrict__ out, int T, int H,
                    int Hkv, int W, int64_t q_stride, int64_t kv_stride, float scale_log2) {
  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t s_q = (uint32_t)__cvta_generic_to_shared(smem);
  constexpr int KV_BYTES = Geo<D>::KV_BYTES;
  constexpr int KSTEPS = D / 16;  // k-steps of Q.K^T
  constexpr int NT = D / 8;       // 8-wide output column tiles
  const uint32_t s_k0 = s_q + Geo<D>::Q_BYTES;
  const uint32_t s_v0 = s_k0 + 2 * KV_BYTES;

  const int n_qb = (T + BQ - 1) / BQ;
  const int qb = n_qb - 1 - (int)blockIdx.x;  // longest rows first
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int g = h / (H / Hkv);
  const int q0 = qb * BQ;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int qw0 = q0 + warp * 16;

  const uint16_t* qg = q + (int64_t)b * T * q_stride + (int64_t)h * D;
  const uint16_t* kg = k + (int64_t)b * T * kv_stride + (int64_t)g * D;
  const uint16_t* vg = v + (int64_t)b * T * kv_stride + (int64_t)g * D;

  const int lo = max(0, q0 - W + 1);
  const int hi = min(T, q0 + BQ) - 1;
  const int kt0 = lo / BKV;
  const int kt1 = hi / BKV;
  const int n_tiles = kt1 - kt0 + 1;

  load_tile<D>(s_q, qg + (int64_t)q0 * q_stride, q_stride, 0, BQ, T - q0);
  load_tile<D>(s_k0, kg, kv_stride, kt0 * BKV, BKV, T);
  load_tile<D>(s_v0, vg, kv_stride, kt0 * BKV, BKV, T);
  cp_async_commit();

  uint32_t qa[KSTEPS][4];
  float o[NT][4];
#pragma unroll
  for (int i = 0; i < NT; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.0f;
  float m_run[2] = {-INFINITY, -INFINITY};
  float l_run[2] = {0.0f, 0.0f};

  const int gq = lane >> 2;  // row within the 8-row group
  const int tq = lane & 3;   // column pair within the 8-column n-tile

  for (int it = 0; it < n_tiles; ++it) {
    const int buf = it & 1;
    if (it + 1 < n_tiles) {
      const int nb = buf ^ 1;
      load_tile<D>(s_k0 + nb * KV_BYTES, kg, kv_stride, (kt0 + it + 1) * BKV, BKV, T);
      load_tile<D>(s_v0 + nb * KV_BYTES, vg, kv_stride, (kt0 + it + 1) * BKV, BKV, T);
    }
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();

    if (it == 0) {
#pragma unroll
      for (int kk = 0; kk < KSTEPS; ++kk) {
        const int r = warp * 16 + (lane & 15);
        const int ch = 2 * kk + (lane >> 4);
        ldsm_x4(s_q + swz<D>(r, ch), qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3]);
      }
    }

    const int k0 = (kt0 + it) * BKV;
    // Warp-uniform: does any (row, key) pair of this warp fall inside the window?
    const bool skip = (k0 > qw0 + 15) || (qw0 - (k0 + BKV - 1) >= W);
    if (!skip) {
      const uint32_t s_k = s_k0 + buf * KV_BYTES;
      const uint32_t s_v = s_v0 + buf * KV_BYTES;
      float s[8][4];
#pragma unroll
      for (int n = 0; n < 8; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.0f;
#pragma unroll
      for (int kk = 0; kk < KSTEPS; ++kk) {
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const int key = 16 * jj + (lane & 7) + ((lane >> 4) << 3);
          const int ch = 2 * kk + ((lane >> 3) & 1);
          uint32_t b0, b1, b2, b3;
          ldsm_x4(s_k + swz<D>(key, ch), b0, b1, b2, b3);
          mma16816<F16>(s[2 * jj], qa[kk], b0, b1);
          mma16816<F16>(s[2 * jj + 1], qa[kk], b2, b3);
        }
      }
      const bool need_mask = !((k0 + BKV - 1 <= qw0) && (qw0 + 15 - k0 < W) && (k0 + BKV <= T));
      if (need_mask) {
#pragma unroll
        for (int n = 0; n < 8; ++n) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int i = qw0 + gq + ((e >> 1) << 3);
            const int j = k0 + 8 * n + 2 * tq + (e & 1);
            const bool vis = (j <= i) && (i - j < W) && (j < T);
            if (!vis) s[n][e] = -INFINITY;
          }
        }
      }
      // online softmax, rows gq (e = 0,1) and gq + 8 (e = 2,3)
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        float mx = -INFINITY;
#pragma unroll
        for (int n = 0; n < 8; ++n) mx = fmaxf(mx, fmaxf(s[n][2 * r], s[n][2 * r + 1]));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        const float m_new = fmaxf(m_run[r], mx);
        const float ms = (m_new == -INFINITY) ? 0.0f : m_new * scale_log2;
        const float alpha = exp2f(m_run[r] * scale_log2 - ms);
        float rs = 0.0f;
#pragma unroll
        for (int n = 0; n < 8; ++n) {
          const float p0 = exp2f(s[n][2 * r] * scale_log2 - ms);
          const float p1 = exp2f(s[n][2 * r + 1] * scale_log2 - ms);
          s[n][2 * r] = p0;
          s[n][2 * r + 1] = p1;
          rs += p0 + p1;
        }
        l_run[r] = l_run[r] * alpha + rs;
        m_run[r] = m_new;
#pragma unroll
        for (int dn = 0; dn < NT; ++dn) {
          o[dn][2 * r] *= alpha;
          o[dn][2 * r + 1] *= alpha;
        }
      }
      // O += P V
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        uint32_t pa[4];
        pa[0] = Half<F16>::pack2(s[2 * kk][0], s[2 * kk][1]);
        pa[1] = Half<F16>::pack2(s[2 * kk][2], s[2 * kk][3]);
        pa[2] = Half<F16>::pack2(s[2 * kk + 1][0], s[2 * kk + 1][1]);
        pa[3] = Half<F16>::pack2(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
        for (int dn = 0; dn < NT / 2; ++dn) {
          const int key = 16 * kk + (lane & 7) + (((lane >> 3) & 1) << 3);
          const int ch = 2 * dn + (lane >> 4);
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(s_v + swz<D>(key, ch), b0, b1, b2, b3);
          mma16816<F16>(o[2 * dn], pa, b0, b1);
          mma16816<F16>(o[2 * dn + 1], pa, b2, b3);
        }
      }
    }
    __syncthreads();
  }

  // normalise and store
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    float l = l_run[r];
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    const float inv = l > 0.0f ? 1.0f / l : 0.0f;
    const int i = qw0 + gq + 8 * r;
    if (i < T) {
      uint16_t* orow = out + ((int64_t)b * T + i) * ((int64_t)H * D) + (int64_t)h * D;
#pragma unroll
      for (int dn = 0; dn < NT; ++dn) {
        *reinterpret_cast<uint32_t*>(orow + 8 * dn + 2 * tq) =
            Half<F16>::pack2(o[dn][2 * r] * inv, o[dn][2 * r + 1] * inv);
      }
    }
  }
}

}  // namespace attn

template <int D, bool F16>
static cudaError_t attn_launch_t(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                 uint16_t* out, int B, int T, int H, int Hkv, int W,
                                 int64_t q_stride, int64_t kv_stride, cudaStream_t stream) {
  using namespace attn;
  static bool attr_done[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_done[dev]) {
    cudaError_t e = cudaFuncSetAttribute(attn_fwd_kernel<D, F16>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Geo<D>::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_done[dev] = true;
  }
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)D);
  dim3 grid((T + BQ - 1) / BQ, H, B);
  attn_fwd_kernel<D, F16><<<grid, NTHREADS, Geo<D>::SMEM_BYTES, stream>>>(
      q, k, v, out, T, H, Hkv, W, q_stride, kv_stride, scale_log2);
  return cudaGetLastError();
}

nc_status attention_launch(const uint16_t* q, const uint16_t* k, const uint16_t* v, uint16_t* out,
                           int B, int T, int H, int Hkv, int D, int window, int64_t q_stride,
                           int64_t kv_stride, bool f16, cudaStream_t stream) {
  if (D != 64 && D != 128) return NC_ERR_SHAPE;
  if (B == 0 || T == 0) return NC_OK;
  const int W = (window <= 0 || window > T) ? T : window;
  cudaError_t e;
  if (D == 128)
    e = f16 ? attn_launch_t<128, true>(q, k, v, out, B, T, H, Hkv, W, q_stride, kv_stride, stream)
            : attn_launch_t<128, false>(q, k, v, out, B, T, H, Hkv, W, q_stride, kv_stride, stream);
  else
    e = f16 ? attn_launch_t<64, true>(q, k, v, out, B, T, H, Hkv, W, q_stride, kv_stride, stream)
            : attn_launch_t<64, false>(q, k, v, out, B, T, H, Hkv, W, q_stride, kv_stride, stream);
  return e == cudaSuccess ? NC_OK : NC_ERR_CUDA;
}

}  // namespace nc
