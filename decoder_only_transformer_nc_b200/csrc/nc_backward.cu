// Backward of the block stack ("从文本到聊天模型" §6.5: the training step's
// loss.backward() after the forward's loss): the row kernels.  The projections' dgrad / wgrad products run on the tcgen05 GEMM
// (nc_gemm.cu, GEMM_NN / GEMM_TN layouts; soft-cap + cross-entropy and relu^2
// backward in its epilogues).
//
// Every gradient here is of the SUM of the token losses; the caller folds the
// 1 / (number of counted targets) of the mean into the weight gradients, so the
// 16-bit intermediate gradients stay O(1) per token.
//
// The attention backward runs on tcgen05 in nc_attention_bwd.cu.
#include <cuda_runtime.h>

#include <cstdint>

#include "nc_half.cuh"
#include "nc_internal.h"
#include "nc_ptx.cuh"

namespace nc {
namespace bwd {

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

// ---------------------------------------------------------------- RMSNorm
// y = x r, r = (mean(x^2) + eps)^(-1/2):  dx = r (dy - y mean(dy y))
// = r dy - x r^3 mean(dy x).  dx_acc (+)= that; dx16 = the new dx_acc in 16-bit.
template <bool F16>
__global__ void __launch_bounds__(256) rmsnorm_bwd_kernel(const float* __restrict__ x, const float* __restrict__ dy,
                                                          float* __restrict__ dx_acc, uint16_t* __restrict__ dx16,
                                                          int M, int C, float eps, int accumulate) {
  const int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= M) return;
  const float4* xr = reinterpret_cast<const float4*>(x + (int64_t)row * C);
  const float4* gr = reinterpret_cast<const float4*>(dy + (int64_t)row * C);
  float4* dr = reinterpret_cast<float4*>(dx_acc + (int64_t)row * C);
  uint2* hr = reinterpret_cast<uint2*>(dx16 + (int64_t)row * C);
  const int n4 = C >> 2;
  float ss = 0.0f, sg = 0.0f;
  for (int i = lane; i < n4; i += 32) {
    const float4 a = xr[i], g = gr[i];
    ss += a.x * a.x + a.y * a.y + a.z * a.z + a.w * a.w;
    sg += a.x * g.x + a.y * g.y + a.z * g.z + a.w * g.w;
  }
  ss = warp_sum(ss);
  sg = warp_sum(sg);
  const float r = rsqrtf(ss / (float)C + eps);
  const float k = r * r * r * sg / (float)C;  // dx = r dy - x r^3 mean(dy x)
  for (int i = lane; i < n4; i += 32) {
    const float4 a = xr[i], g = gr[i];
    float4 o = make_float4(fmaf(r, g.x, -k * a.x), fmaf(r, g.y, -k * a.y), fmaf(r, g.z, -k * a.z),
                           fmaf(r, g.w, -k * a.w));
    if (accumulate) {
      const float4 p = dr[i];
      o = make_float4(o.x + p.x, o.y + p.y, o.z + p.z, o.w + p.w);
    }
    dr[i] = o;
    hr[i] = make_uint2(Half<F16>::pack2(o.x, o.y), Half<F16>::pack2(o.z, o.w));
  }
}

// ---------------------------------------------------------------- QK-norm + RoPE
// One warp per (row, q/k head).  In: g = dL/d(normalised q or k) (16-bit, in
// place in dqkv), y = the saved normalised head (qkv), r = its saved QK-norm
// factor.  du = r (g - y mean(g y)) is the gradient before the norm; the
// pair-interleaved columns (2p, 2p+1) hold (u_p, u_{p+D/2}) rotated forward by
// t theta_p, so the gradient before RoPE is the inverse rotation of du.
template <bool F16>
__global__ void __launch_bounds__(256) qk_bwd_kernel(uint16_t* __restrict__ dqkv, const uint16_t* __restrict__ qkv,
                                                     int64_t ld, const float* __restrict__ rstd,
                                                     const float* __restrict__ rope, int rope_T, int M, int T,
                                                     int heads, int D) {
  const int64_t wid = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= (int64_t)M * heads) return;
  const int row = (int)(wid / heads), hh = (int)(wid % heads);
  const int per = D / 32;  // elements per lane: 4 (D = 128) or 2 (D = 64), whole pairs
  const int64_t base = (int64_t)row * ld + (int64_t)hh * D + lane * per;
  float g[4], y[4];
#pragma unroll
  for (int e = 0; e < 4; e += 2) {
    if (e < per) {
      const float2 a = Half<F16>::unpack2(*reinterpret_cast<const uint32_t*>(dqkv + base + e));
      const float2 b = Half<F16>::unpack2(*reinterpret_cast<const uint32_t*>(qkv + base + e));
      g[e] = a.x;
      g[e + 1] = a.y;
      y[e] = b.x;
      y[e + 1] = b.y;
    } else {
      g[e] = g[e + 1] = y[e] = y[e + 1] = 0.0f;
    }
  }
  float s = 0.0f;
#pragma unroll
  for (int e = 0; e < 4; ++e) s += g[e] * y[e];
  s = warp_sum(s) / (float)D;
  const float r = rstd[(int64_t)row * heads + hh];
  const int t = row % T;
  const float* cs = rope + (int64_t)t * (D / 2);
  const float* sn = rope + ((int64_t)rope_T + t) * (D / 2);
#pragma unroll
  for (int e = 0; e < 4; e += 2) {
    if (e < per) {
      const int p = (lane * per + e) >> 1;  // pair index
      const float da = r * (g[e] - y[e] * s), db = r * (g[e + 1] - y[e + 1] * s);
      const float c = cs[p], sv = sn[p];
      *reinterpret_cast<uint32_t*>(dqkv + base + e) = Half<F16>::pack2(da * c + db * sv, db * c - da * sv);
    }
  }
}

// ---------------------------------------------------------------- small kernels
// dwte[token[m]] += alpha dx[m] (alpha read from device memory); one warp per row.
__global__ void __launch_bounds__(256) embedding_bwd_kernel(const int32_t* __restrict__ tokens,
                                                            const float* __restrict__ dx, float* __restrict__ dwte,
                                                            int M, int C, int V, const float* __restrict__ alpha_p) {
  const int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= M) return;
  const float alpha = *alpha_p;
  const int tok = tokens[row];
  if (tok < 0 || tok >= V) return;  // flagged by the forward's embedding kernel
  const float* src = dx + (int64_t)row * C;
  float* dst = dwte + (int64_t)tok * C;
  for (int c = lane; c < C; c += 32) atomicAdd(dst + c, alpha * src[c]);
}

// The QKV weight gradient, computed in the packed row order of the forward's
// weight (q and k rows pair-interleaved within each head), added with factor
// alpha to the three fp32 gradients in the weights' own row order.
__global__ void __launch_bounds__(256) qkv_grad_scatter_kernel(const float* __restrict__ packed, float* __restrict__ gq,
                                                               float* __restrict__ gk, float* __restrict__ gv,
                                                               int H, int Hkv, int D, int C, float alpha) {
  const int64_t n4 = (int64_t)(H + 2 * Hkv) * D * C / 4;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t e = i * 4;
    const int64_t R = e / C, col = e - R * C;  // packed row
    const int hd = (int)(R / D), jj = (int)(R % D);
    float* dst;
    int64_t orow;
    if (hd < H + Hkv) {  // q or k head: packed row jj holds source row (jj >> 1) + (jj & 1) D/2
      const int src = (jj >> 1) + (jj & 1) * (D / 2);
      if (hd < H) {
        dst = gq;
        orow = (int64_t)hd * D + src;
      } else {
        dst = gk;
        orow = (int64_t)(hd - H) * D + src;
      }
    } else {
      dst = gv;
      orow = (int64_t)(hd - H - Hkv) * D + jj;
    }
    const float4 p = *reinterpret_cast<const float4*>(packed + e);
    float4* o = reinterpret_cast<float4*>(dst + orow * C + col);
    float4 q = *o;
    q.x = fmaf(alpha, p.x, q.x);
    q.y = fmaf(alpha, p.y, q.y);
    q.z = fmaf(alpha, p.z, q.z);
    q.w = fmaf(alpha, p.w, q.w);
    *o = q;
  }
}

}  // namespace bwd

nc_status rmsnorm_bwd_launch(const float* x, const float* dy, float* dx_acc, uint16_t* dx16, int M, int C, float eps,
                             bool accumulate, bool f16, cudaStream_t stream) {
  if (M == 0) return NC_OK;
  if (C % 4) return NC_ERR_SHAPE;
  const int grid = (M + 7) / 8;
  if (f16)
    bwd::rmsnorm_bwd_kernel<true><<<grid, 256, 0, stream>>>(x, dy, dx_acc, dx16, M, C, eps, accumulate ? 1 : 0);
  else
    bwd::rmsnorm_bwd_kernel<false><<<grid, 256, 0, stream>>>(x, dy, dx_acc, dx16, M, C, eps, accumulate ? 1 : 0);
  return cudaGetLastError() == cudaSuccess ? NC_OK : NC_ERR_CUDA;
}

nc_status qk_bwd_launch(uint16_t* dqkv, const uint16_t* qkv, int64_t ld, const float* rstd, const float* rope,
                        int rope_T, int M, int T, int H, int Hkv, int D, bool f16, cudaStream_t stream) {
  const int64_t warps = (int64_t)M * (H + Hkv);
  if (warps == 0) return NC_OK;
  if (D != 64 && D != 128) return NC_ERR_SHAPE;
  const unsigned grid = (unsigned)((warps + 7) / 8);
  if (f16)
    bwd::qk_bwd_kernel<true><<<grid, 256, 0, stream>>>(dqkv, qkv, ld, rstd, rope, rope_T, M, T, H + Hkv, D);
  else
    bwd::qk_bwd_kernel<false><<<grid, 256, 0, stream>>>(dqkv, qkv, ld, rstd, rope, rope_T, M, T, H + Hkv, D);
  return cudaGetLastError() == cudaSuccess ? NC_OK : NC_ERR_CUDA;
}

nc_status embedding_bwd_launch(const int32_t* tokens, const float* dx, float* dwte, int M, int C, int V,
                               const float* alpha, cudaStream_t stream) {
  if (M == 0) return NC_OK;
  bwd::embedding_bwd_kernel<<<(M + 7) / 8, 256, 0, stream>>>(tokens, dx, dwte, M, C, V, alpha);
  return cudaGetLastError() == cudaSuccess ? NC_OK : NC_ERR_CUDA;
}

nc_status qkv_grad_scatter_launch(const float* packed, float* gq, float* gk, float* gv, int H, int Hkv, int D, int C,
                                  float alpha, cudaStream_t stream) {
  const int64_t n4 = (int64_t)(H + 2 * Hkv) * D * C / 4;
  if (n4 == 0) return NC_OK;
  const int64_t want = (n4 + 255) / 256;
  const int grid = (int)(want < 148 * 8 ? want : 148 * 8);
  bwd::qkv_grad_scatter_kernel<<<grid, 256, 0, stream>>>(packed, gq, gk, gv, H, Hkv, D, C, alpha);
  return cudaGetLastError() == cudaSuccess ? NC_OK : NC_ERR_CUDA;
}

}  // namespace nc
