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
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
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


// ---------------------------------------------------------------- extras
// Backward of the further terms of the full nanochat forward ("Nanochat与
// nanoGPT对比" §1: smear, residual lambdas with x0, value embeddings, backout).
// Parameter gradients are of the mean loss: every sum over tokens is scaled by
// *inv (1 / counted targets) and added into the caller's fp32 gradient.

// Sum over the block of v (all threads get it); red: 32 floats of shared memory.
__device__ __forceinline__ float block_sum(float v, float* red) {
  v = warp_sum(v);
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[w] = v;
  __syncthreads();
  v = lane < (int)(blockDim.x >> 5) ? red[lane] : 0.0f;
  return warp_sum(v);
}

// out0 += sign * inv * sum(a . b0), out1 += sign * inv * sum(a . b1) (b1 may be
// null); n4 float4 elements.
__global__ void __launch_bounds__(256) dots_kernel(const float4* __restrict__ a, const float4* __restrict__ b0,
                                                   const float4* __restrict__ b1, int64_t n4,
                                                   const float* __restrict__ inv, float sign,
                                                   float* __restrict__ out0, float* __restrict__ out1) {
  __shared__ float red[32];
  float s0 = 0.0f, s1 = 0.0f;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (int64_t)gridDim.x * blockDim.x) {
    const float4 x = a[i], y = b0[i];
    s0 = fmaf(x.x, y.x, fmaf(x.y, y.y, fmaf(x.z, y.z, fmaf(x.w, y.w, s0))));
    if (b1) {
      const float4 z = b1[i];
      s1 = fmaf(x.x, z.x, fmaf(x.y, z.y, fmaf(x.z, z.z, fmaf(x.w, z.w, s1))));
    }
  }
  s0 = block_sum(s0, red);
  if (b1) s1 = block_sum(s1, red);
  if (threadIdx.x == 0) {
    const float f = sign * *inv;
    atomicAdd(out0, f * s0);
    if (b1) atomicAdd(out1, f * s1);
  }
}

// The stream gradient through "x_in = lam_r x + lam_0 x0" and the backout
// subtraction, in place: acc0 += lam_0 d; d = lam_r d - lam_sub sub + add;
// then the 16-bit copy (when dx16).  Null pointers drop their term.
template <bool F16>
__global__ void __launch_bounds__(256) mix_bwd_kernel(float4* __restrict__ dx, float4* __restrict__ acc0,
                                                      const float4* __restrict__ sub, const float4* __restrict__ add,
                                                      const float* __restrict__ lam_r, const float* __restrict__ lam_0,
                                                      const float* __restrict__ lam_sub, uint2* __restrict__ dx16,
                                                      int64_t n4) {
  const float lr = lam_r ? *lam_r : 1.0f, l0 = lam_0 ? *lam_0 : 0.0f, ls = lam_sub ? *lam_sub : 0.0f;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (int64_t)gridDim.x * blockDim.x) {
    float4 d = dx[i];
    if (acc0) {
      float4 c = acc0[i];
      c = make_float4(fmaf(l0, d.x, c.x), fmaf(l0, d.y, c.y), fmaf(l0, d.z, c.z), fmaf(l0, d.w, c.w));
      acc0[i] = c;
    }
    d = make_float4(lr * d.x, lr * d.y, lr * d.z, lr * d.w);
    if (sub) {
      const float4 b = sub[i];
      d = make_float4(fmaf(-ls, b.x, d.x), fmaf(-ls, b.y, d.y), fmaf(-ls, b.z, d.z), fmaf(-ls, b.w, d.w));
    }
    if (add) {
      const float4 b = add[i];
      d = make_float4(d.x + b.x, d.y + b.y, d.z + b.z, d.w + b.w);
    }
    dx[i] = d;
    if (dx16) dx16[i] = make_uint2(Half<F16>::pack2(d.x, d.y), Half<F16>::pack2(d.z, d.w));
  }
}

// Value embedding of one layer, v += gate[g] ve[token] per kv head g:
// dve[token] += inv gate[g] dv and dgate[g] += inv sum dv . ve[token].  Block
// (g, chunk of tokens); each warp walks tokens, each lane D/32 dims of the head.
template <bool F16>
__global__ void __launch_bounds__(256) ve_bwd_kernel(const uint16_t* __restrict__ dqkv, int64_t ld,
                                                     const int32_t* __restrict__ tokens,
                                                     const float* __restrict__ table, const float* __restrict__ gate,
                                                     float* __restrict__ dtable, float* __restrict__ dgate, int M,
                                                     int H, int Hkv, int D, int V, const float* __restrict__ inv) {
  __shared__ float red[32];
  const int g = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int warps = blockDim.x >> 5;
  const float f = *inv, fg = f * gate[g];
  float s = 0.0f;
  for (int m = blockIdx.y * warps + warp; m < M; m += gridDim.y * warps) {
    const int tok = tokens[m];
    if (tok < 0 || tok >= V) continue;  // flagged by the forward's embedding kernel
    const uint16_t* dv = dqkv + (int64_t)m * ld + (int64_t)(H + Hkv + g) * D;
    const float* ve = table + ((int64_t)tok * Hkv + g) * D;
    float* dve = dtable + ((int64_t)tok * Hkv + g) * D;
    for (int d = 2 * lane; d < D; d += 64) {
      const float2 v = Half<F16>::unpack2(*reinterpret_cast<const uint32_t*>(dv + d));
      s = fmaf(v.x, ve[d], fmaf(v.y, ve[d + 1], s));
      atomicAdd(dve + d, fg * v.x);
      atomicAdd(dve + d + 1, fg * v.y);
    }
  }
  s = block_sum(s, red);
  if (threadIdx.x == 0) atomicAdd(dgate + g, f * s);
}

// Smear, x_t = e_t + sig(e_t . w) e_{t-1} within each row of T tokens (w the
// gate weight rounded to bf16, as the forward uses it): one warp per token m
// writes de_m = dx_m + g_{m+1} dx_{m+1} + dz_m w and dz_m = (dx_m . e_{m-1})
// g_m (1 - g_m), from the embeddings e = wte[token].
__device__ __forceinline__ float smear_gate_of(const float* e, const float* w, int C, int lane) {
  float z = 0.0f;
  for (int c = lane; c < C; c += 32) z = fmaf(e[c], __bfloat162float(__float2bfloat16_rn(w[c])), z);
  z = warp_sum(z);
  return 1.0f / (1.0f + expf(-z));
}

__global__ void __launch_bounds__(256) smear_bwd_kernel(const int32_t* __restrict__ tokens,
                                                        const float* __restrict__ wte, const float* __restrict__ w,
                                                        const float* __restrict__ dx, float* __restrict__ de,
                                                        float* __restrict__ dz, int M, int T, int C, int V) {
  const int m = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (m >= M) return;
  auto row = [&](int mm) {
    int tok = tokens[mm];
    if (tok < 0 || tok >= V) tok = 0;
    return wte + (int64_t)tok * C;
  };
  const int t = m % T;
  const float* e = row(m);
  float dzm = 0.0f;
  if (t > 0) {
    const float g = smear_gate_of(e, w, C, lane);
    const float* ep = row(m - 1);
    const float* d = dx + (int64_t)m * C;
    float s = 0.0f;
    for (int c = lane; c < C; c += 32) s = fmaf(d[c], ep[c], s);
    dzm = warp_sum(s) * g * (1.0f - g);
  }
  const float gn = (t + 1 < T) ? smear_gate_of(row(m + 1), w, C, lane) : 0.0f;
  const float* d = dx + (int64_t)m * C;
  const float* dn = dx + (int64_t)(t + 1 < T ? m + 1 : m) * C;
  float* o = de + (int64_t)m * C;
  for (int c = lane; c < C; c += 32)
    o[c] = fmaf(dzm, __bfloat162float(__float2bfloat16_rn(w[c])), fmaf(gn, dn[c], d[c]));
  if (lane == 0) dz[m] = dzm;
}

// dw[c] += inv sum_m dz_m e_m[c]: block (256 columns, chunk of tokens).
__global__ void __launch_bounds__(256) smear_weight_grad_kernel(const int32_t* __restrict__ tokens,
                                                                const float* __restrict__ wte,
                                                                const float* __restrict__ dz, float* __restrict__ dw,
                                                                int M, int C, int V, const float* __restrict__ inv) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= C) return;
  const int per = (M + gridDim.y - 1) / gridDim.y;
  const int m0 = blockIdx.y * per, m1 = min(M, m0 + per);
  float s = 0.0f;
  for (int m = m0; m < m1; ++m) {
    int tok = tokens[m];
    if (tok < 0 || tok >= V) tok = 0;
    s = fmaf(dz[m], wte[(int64_t)tok * C + c], s);
  }
  atomicAdd(dw + c, *inv * s);
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

nc_status dots_launch(const float* a, const float* b0, const float* b1, int64_t n, const float* inv, float sign,
                      float* out0, float* out1, cudaStream_t stream) {
  if (n == 0) return NC_OK;
  if (n % 4) return NC_ERR_SHAPE;
  bwd::dots_kernel<<<2 * 148, 256, 0, stream>>>(reinterpret_cast<const float4*>(a), reinterpret_cast<const float4*>(b0),
                                                 reinterpret_cast<const float4*>(b1), n / 4, inv, sign, out0, out1);
  return cudaGetLastError() == cudaSuccess ? NC_OK : NC_ERR_CUDA;
}

nc_status mix_bwd_launch(float* dx, float* acc0, const float* sub, const float* add, const float* lam_r,
                         const float* lam_0, const float* lam_sub, uint16_t* dx16, int64_t n, bool f16,
                         cudaStream_t stream) {
  if (n == 0) return NC_OK;
  if (n % 4) return NC_ERR_SHAPE;
  const int64_t n4 = n / 4;
  const int grid = (int)std::min<int64_t>((n4 + 255) / 256, 148 * 16);
  auto* d4 = reinterpret_cast<float4*>(dx);
  auto* a4 = reinterpret_cast<float4*>(acc0);
  auto* s4 = reinterpret_cast<const float4*>(sub);
  auto* p4 = reinterpret_cast<const float4*>(add);
  auto* h2 = reinterpret_cast<uint2*>(dx16);
  if (f16)
    bwd::mix_bwd_kernel<true><<<grid, 256, 0, stream>>>(d4, a4, s4, p4, lam_r, lam_0, lam_sub, h2, n4);
  else
    bwd::mix_bwd_kernel<false><<<grid, 256, 0, stream>>>(d4, a4, s4, p4, lam_r, lam_0, lam_sub, h2, n4);
  return cudaGetLastError() == cudaSuccess ? NC_OK : NC_ERR_CUDA;
}

nc_status ve_bwd_launch(const uint16_t* dqkv, int64_t ld, const int32_t* tokens, const float* table, const float* gate,
                        float* dtable, float* dgate, int M, int H, int Hkv, int D, int V, const float* inv, bool f16,
                        cudaStream_t stream) {
  if (M == 0) return NC_OK;
  if (D % 2) return NC_ERR_SHAPE;
  const dim3 grid(Hkv, 64);
  if (f16)
    bwd::ve_bwd_kernel<true><<<grid, 256, 0, stream>>>(dqkv, ld, tokens, table, gate, dtable, dgate, M, H, Hkv, D, V, inv);
  else
    bwd::ve_bwd_kernel<false><<<grid, 256, 0, stream>>>(dqkv, ld, tokens, table, gate, dtable, dgate, M, H, Hkv, D, V, inv);
  return cudaGetLastError() == cudaSuccess ? NC_OK : NC_ERR_CUDA;
}

nc_status smear_bwd_launch(const int32_t* tokens, const float* wte, const float* w, const float* dx, float* de,
                           float* dz, float* dw, int M, int T, int C, int V, const float* inv, cudaStream_t stream) {
  if (M == 0) return NC_OK;
  bwd::smear_bwd_kernel<<<(M + 7) / 8, 256, 0, stream>>>(tokens, wte, w, dx, de, dz, M, T, C, V);
  if (cudaGetLastError() != cudaSuccess) return NC_ERR_CUDA;
  const dim3 grid((C + 255) / 256, 64);
  bwd::smear_weight_grad_kernel<<<grid, 256, 0, stream>>>(tokens, wte, dz, dw, M, C, V, inv);
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
