// Backward of the block stack ("从文本到聊天模型" §6.5: the training step's
// loss.backward() after the forward's loss): the row kernels and the attention
// backward.  The projections' dgrad / wgrad products run on the tcgen05 GEMM
// (nc_gemm.cu, GEMM_NN / GEMM_TN layouts; soft-cap + cross-entropy and relu^2
// backward in its epilogues).
//
// Every gradient here is of the SUM of the token losses; the caller folds the
// 1 / (number of counted targets) of the mean into the weight gradients, so the
// 16-bit intermediate gradients stay O(1) per token.
//
// Attention backward (per head, window W, scale 1/sqrt(D), P recomputed from
// the forward's log-sum-exp):  dV = P^T dO,  dP = dO V^T,
// dS = P o (dP - Delta) with Delta_i = sum_d dO_i O_i,  dQ = scale dS K,
// dK = scale dS^T Q.  Two kernels, so that no sum needs atomics:
//   attn_bwd_dq_kernel    one CTA per (64 queries, head, row): loops over the
//                         key tiles inside the window;
//   attn_bwd_dkdv_kernel  one CTA per (64 keys, kv head, row): loops over the
//                         query heads of its group and the query tiles that see
//                         these keys.
// Both use the warp-level mma.sync.m16n8k16 tensor-core path (fp32
// accumulation) with 16-bit tiles staged in padded shared memory and read by
// ldmatrix; each warp owns 16 rows of the CTA's tile.
#include <cuda_runtime.h>

#include <cstdint>

#include "nc_half.cuh"
#include "nc_internal.h"
#include "nc_mma.cuh"
#include "nc_ptx.cuh"

namespace nc {
namespace bwd {

using namespace wmma16;

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
// Delta[m, h] = sum_d dO[m, h, d] O[m, h, d]
template <bool F16>
__global__ void __launch_bounds__(256) attn_delta_kernel(const uint16_t* __restrict__ dO, const uint16_t* __restrict__ O,
                                                         float* __restrict__ delta, int M, int H, int D) {
  const int64_t wid = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= (int64_t)M * H) return;
  const int64_t base = wid * D;
  float s = 0.0f;
  for (int d = lane * 2; d < D; d += 64) {
    const float2 a = Half<F16>::unpack2(*reinterpret_cast<const uint32_t*>(dO + base + d));
    const float2 b = Half<F16>::unpack2(*reinterpret_cast<const uint32_t*>(O + base + d));
    s += a.x * b.x + a.y * b.y;
  }
  s = warp_sum(s);
  if (lane == 0) delta[wid] = s;
}

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

// ---------------------------------------------------------------- attention backward
constexpr int BLK = 64;        // rows of a tile (queries or keys)
constexpr int NTH = 128;       // 4 warps x 16 rows
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// rows [row0, row0 + 64) of a 16-bit [rows, D] view (row stride ld elements,
// head column offset col) into a padded shared tile; rows >= T are zeros.
template <int D, int LD>
__device__ __forceinline__ void stage_tile(uint16_t* dst, const uint16_t* src, int64_t ld, int64_t row_base,
                                           int row0, int T) {
  constexpr int CH = D / 8;  // 16-byte chunks per row
  for (int i = threadIdx.x; i < BLK * CH; i += NTH) {
    const int r = i / CH, c = i % CH;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (row0 + r < T) v = *reinterpret_cast<const uint4*>(src + (row_base + row0 + r) * ld + c * 8);
    *reinterpret_cast<uint4*>(dst + r * LD + c * 8) = v;
  }
}

// The same with 16-byte cp.async copies (rows >= T zero-filled), so the load
// of the next tile overlaps the products of the current one.
template <int D, int LD>
__device__ __forceinline__ void stage_tile_async(uint16_t* dst, const uint16_t* src, int64_t ld, int64_t row_base,
                                                 int row0, int T) {
  constexpr int CH = D / 8;
  for (int i = threadIdx.x; i < BLK * CH; i += NTH) {
    const int r = i / CH, c = i % CH;
    const bool valid = row0 + r < T;
    const uint16_t* g = src + (row_base + (valid ? row0 + r : 0)) * ld + c * 8;
    cp_async16(dst + r * LD + c * 8, g, valid);
  }
}

// S (16 x 64 per warp) = A_tile[rows w*16..] . B_tile^T over D, both [row][D] tiles.
template <int D, int LD, bool F16>
__device__ __forceinline__ void tile_dots(float (&acc)[8][4], uint32_t a_base, uint32_t b_base, int wrow, int lane) {
#pragma unroll
  for (int nt = 0; nt < 8; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[nt][e] = 0.0f;
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    uint32_t a[4];
    load_a<LD>(a, a_base, wrow, kk * 16, lane);
#pragma unroll
    for (int np = 0; np < 4; ++np) {
      uint32_t b[4];
      load_b_nk<LD>(b, b_base, np * 16, kk * 16, lane);
      mma16816<F16>(acc[2 * np], a, b[0], b[1]);
      mma16816<F16>(acc[2 * np + 1], a, b[2], b[3]);
    }
  }
}

// out (16 x D per warp) += X (16 x 64, C-fragments) . Y_tile (64 x D, stored [k][d]).
template <int D, int LD, bool F16>
__device__ __forceinline__ void tile_accum(float (&out)[D / 8][4], const float (&x)[8][4], uint32_t y_base, int lane) {
#pragma unroll
  for (int kc = 0; kc < 4; ++kc) {  // 16 of the 64 contraction rows
    uint32_t a[4];
    a[0] = Half<F16>::pack2(x[2 * kc][0], x[2 * kc][1]);
    a[1] = Half<F16>::pack2(x[2 * kc][2], x[2 * kc][3]);
    a[2] = Half<F16>::pack2(x[2 * kc + 1][0], x[2 * kc + 1][1]);
    a[3] = Half<F16>::pack2(x[2 * kc + 1][2], x[2 * kc + 1][3]);
#pragma unroll
    for (int dp = 0; dp < D / 16; ++dp) {
      uint32_t b[4];
      load_b_kn<LD>(b, y_base, kc * 16, dp * 16, lane);
      mma16816<F16>(out[2 * dp], a, b[0], b[1]);
      mma16816<F16>(out[2 * dp + 1], a, b[2], b[3]);
    }
  }
}

// Write a warp's 16 x D fp32 fragment rows (row0 + g, row0 + g + 8) as 16-bit.
template <int D, bool F16>
__device__ __forceinline__ void store_rows(const float (&acc)[D / 8][4], uint16_t* dst, int64_t ld, int64_t row_base,
                                           int row0, int T, int lane, float f) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int r = row0 + g + 8 * half;
    if (r >= T) continue;
    uint16_t* p = dst + (row_base + r) * ld;
#pragma unroll
    for (int nt = 0; nt < D / 8; ++nt)
      *reinterpret_cast<uint32_t*>(p + nt * 8 + 2 * t) =
          Half<F16>::pack2(acc[nt][2 * half] * f, acc[nt][2 * half + 1] * f);
  }
}

template <int D, bool F16>
__global__ void __launch_bounds__(NTH, 1)
    attn_bwd_dq_kernel(const uint16_t* __restrict__ qkv, int64_t ldqkv, const uint16_t* __restrict__ dO,
                       const float* __restrict__ lse, const float* __restrict__ delta, uint16_t* __restrict__ dqkv,
                       int T, int H, int Hkv, int W, float scale) {
  constexpr int LD = D + 8;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint16_t* sQ = reinterpret_cast<uint16_t*>(smem_raw);
  uint16_t* sdO = sQ + BLK * LD;
  uint16_t* sKV = sdO + BLK * LD;  // two buffers of (K tile, V tile)
  const int q0 = blockIdx.x * BLK, h = blockIdx.y, b = blockIdx.z;
  const int g = h / (H / Hkv);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t rb = (int64_t)b * T;
  const int64_t HD = (int64_t)H * D;
  stage_tile<D, LD>(sQ, qkv + (int64_t)h * D, ldqkv, rb, q0, T);
  stage_tile<D, LD>(sdO, dO + (int64_t)h * D, HD, rb, q0, T);
  const int ra = q0 + warp * 16 + (lane >> 2), rbw = ra + 8;  // this thread's two query rows
  const float lse_a = ra < T ? lse[(rb + ra) * H + h] : 0.0f, lse_b = rbw < T ? lse[(rb + rbw) * H + h] : 0.0f;
  const float dl_a = ra < T ? delta[(rb + ra) * H + h] : 0.0f, dl_b = rbw < T ? delta[(rb + rbw) * H + h] : 0.0f;
  const float c1 = scale * kLog2e;
  float dq[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) dq[i][e] = 0.0f;
  const int q_last = min(T - 1, q0 + BLK - 1);
  const int kt_lo = max(0, q0 - W + 1) / BLK, kt_hi = q_last / BLK;
  const uint32_t bq = smem_u32(sQ), bdo = smem_u32(sdO);
  auto issue = [&](int kt) {  // K and V tiles of key tile kt into buffer kt & 1
    uint16_t* dst = sKV + (kt & 1) * 2 * BLK * LD;
    stage_tile_async<D, LD>(dst, qkv + (int64_t)(H + g) * D, ldqkv, rb, kt * BLK, T);
    stage_tile_async<D, LD>(dst + BLK * LD, qkv + (int64_t)(H + Hkv + g) * D, ldqkv, rb, kt * BLK, T);
    cp_async_commit();
  };
  issue(kt_lo);
  for (int kt = kt_lo; kt <= kt_hi; ++kt) {
    const int k0 = kt * BLK;
    if (kt < kt_hi) {
      issue(kt + 1);
      cp_async_wait<1>();  // this tile's group has landed; the next one may still be in flight
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const uint32_t bk = smem_u32(sKV + (kt & 1) * 2 * BLK * LD), bv = bk + BLK * LD * 2;
    float s[8][4], dp[8][4];
    tile_dots<D, LD, F16>(s, bq, bk, warp * 16, lane);
    tile_dots<D, LD, F16>(dp, bdo, bv, warp * 16, lane);
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = e < 2 ? ra : rbw;
        const int j = k0 + nt * 8 + 2 * (lane & 3) + (e & 1);
        const bool vis = i < T && j <= i && i - j < W;
        const float p = vis ? ex2f(fmaf(s[nt][e], c1, -(e < 2 ? lse_a : lse_b) * kLog2e)) : 0.0f;
        s[nt][e] = p * (dp[nt][e] - (e < 2 ? dl_a : dl_b));  // dS / scale
      }
    tile_accum<D, LD, F16>(dq, s, bk, lane);
    __syncthreads();  // buffer kt & 1 is refilled by the issue of tile kt + 2
  }
  store_rows<D, F16>(dq, dqkv + (int64_t)h * D, ldqkv, rb, q0 + warp * 16, T, lane, scale);
}

template <int D, bool F16>
__global__ void __launch_bounds__(NTH, 1)
    attn_bwd_dkdv_kernel(const uint16_t* __restrict__ qkv, int64_t ldqkv, const uint16_t* __restrict__ dO,
                         const float* __restrict__ lse, const float* __restrict__ delta, uint16_t* __restrict__ dqkv,
                         int T, int H, int Hkv, int W, float scale) {
  constexpr int LD = D + 8;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint16_t* sK = reinterpret_cast<uint16_t*>(smem_raw);
  uint16_t* sV = sK + BLK * LD;
  uint16_t* sQD = sV + BLK * LD;                            // two buffers of (Q tile, dO tile)
  float* sLD = reinterpret_cast<float*>(sQD + 4 * BLK * LD);  // two buffers of ([BLK] lse, [BLK] delta)
  const int k0 = blockIdx.x * BLK, g = blockIdx.y, b = blockIdx.z;
  const int G = H / Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t rb = (int64_t)b * T;
  const int64_t HD = (int64_t)H * D;
  stage_tile<D, LD>(sK, qkv + (int64_t)(H + g) * D, ldqkv, rb, k0, T);
  stage_tile<D, LD>(sV, qkv + (int64_t)(H + Hkv + g) * D, ldqkv, rb, k0, T);
  const int ja = k0 + warp * 16 + (lane >> 2), jb = ja + 8;  // this thread's two key rows
  const float c1 = scale * kLog2e;
  float dk[D / 8][4], dv[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) dk[i][e] = dv[i][e] = 0.0f;
  const int k_last = min(T - 1, k0 + BLK - 1);
  const int qt_lo = k0 / BLK, qt_hi = min(T - 1, k_last + W - 1) / BLK;
  const uint32_t bk = smem_u32(sK), bv = smem_u32(sV);
  const int nq = qt_hi - qt_lo + 1, n_it = G * nq;  // iterations: (head of the group, query tile)
  auto issue = [&](int it) {  // Q, dO tiles and lse, delta of iteration it into buffer it & 1
    const int h = g * G + it / nq, q0 = (qt_lo + it % nq) * BLK;
    uint16_t* dst = sQD + (it & 1) * 2 * BLK * LD;
    stage_tile_async<D, LD>(dst, qkv + (int64_t)h * D, ldqkv, rb, q0, T);
    stage_tile_async<D, LD>(dst + BLK * LD, dO + (int64_t)h * D, HD, rb, q0, T);
    float* l = sLD + (it & 1) * 2 * BLK;
    for (int i = threadIdx.x; i < BLK; i += NTH) {
      const bool in = q0 + i < T;
      const int64_t r = (rb + (in ? q0 + i : 0)) * H + h;
      cp_async4(l + i, lse + r, in);
      cp_async4(l + BLK + i, delta + r, in);
    }
    cp_async_commit();
  };
  if (n_it > 0) issue(0);
  for (int it = 0; it < n_it; ++it) {
    {
      const int q0 = (qt_lo + it % nq) * BLK;
      if (it + 1 < n_it) {
        issue(it + 1);
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      __syncthreads();
      const uint32_t bq = smem_u32(sQD + (it & 1) * 2 * BLK * LD), bdo = bq + BLK * LD * 2;
      const float* sL = sLD + (it & 1) * 2 * BLK;
      float s[8][4], dp[8][4];
      tile_dots<D, LD, F16>(s, bk, bq, warp * 16, lane);   // S^T: keys x queries
      tile_dots<D, LD, F16>(dp, bv, bdo, warp * 16, lane); // dP^T
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int jq = nt * 8 + 2 * (lane & 3) + (e & 1);  // query within the tile
          const int i = q0 + jq;
          const int j = e < 2 ? ja : jb;
          const bool vis = i < T && j < T && j <= i && i - j < W;
          const float p = vis ? ex2f(fmaf(s[nt][e], c1, -sL[jq] * kLog2e)) : 0.0f;
          s[nt][e] = p;                              // P^T
          dp[nt][e] = p * (dp[nt][e] - sL[BLK + jq]);  // dS^T / scale
        }
      tile_accum<D, LD, F16>(dv, s, bdo, lane);
      tile_accum<D, LD, F16>(dk, dp, bq, lane);
      __syncthreads();  // buffer it & 1 is refilled by the issue of iteration it + 2
    }
  }
  store_rows<D, F16>(dk, dqkv + (int64_t)(H + g) * D, ldqkv, rb, k0 + warp * 16, T, lane, scale);
  store_rows<D, F16>(dv, dqkv + (int64_t)(H + Hkv + g) * D, ldqkv, rb, k0 + warp * 16, T, lane, 1.0f);
}

template <int D, bool F16>
static nc_status attn_bwd_t(const uint16_t* qkv, int64_t ldqkv, const uint16_t* dO, const float* lse,
                            const float* delta, uint16_t* dqkv, int B, int T, int H, int Hkv, int W,
                            cudaStream_t stream) {
  constexpr int LD = D + 8;
  const int smem_q = 6 * BLK * LD * 2;                  // Q, dO, and two (K, V) buffers
  const int smem_k = 6 * BLK * LD * 2 + 4 * BLK * 4;    // K, V, two (Q, dO) and two (lse, delta) buffers
  static bool attr_done[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_done[dev]) {
    if (cudaFuncSetAttribute(attn_bwd_dq_kernel<D, F16>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_q) !=
            cudaSuccess ||
        cudaFuncSetAttribute(attn_bwd_dkdv_kernel<D, F16>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_k) !=
            cudaSuccess)
      return NC_ERR_CUDA;
    attr_done[dev] = true;
  }
  const float scale = 1.0f / sqrtf((float)D);
  const dim3 gq((T + BLK - 1) / BLK, H, B), gk((T + BLK - 1) / BLK, Hkv, B);
  attn_bwd_dq_kernel<D, F16><<<gq, NTH, smem_q, stream>>>(qkv, ldqkv, dO, lse, delta, dqkv, T, H, Hkv, W, scale);
  if (cudaGetLastError() != cudaSuccess) return NC_ERR_CUDA;
  attn_bwd_dkdv_kernel<D, F16><<<gk, NTH, smem_k, stream>>>(qkv, ldqkv, dO, lse, delta, dqkv, T, H, Hkv, W, scale);
  return cudaGetLastError() == cudaSuccess ? NC_OK : NC_ERR_CUDA;
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

nc_status attn_bwd_launch(const uint16_t* qkv, int64_t ldqkv, const uint16_t* o, const uint16_t* dO,
                          const float* lse, float* delta, uint16_t* dqkv, int B, int T, int H, int Hkv, int D,
                          int window, bool f16, cudaStream_t stream) {
  if (B == 0 || T == 0) return NC_OK;
  if (D != 64 && D != 128) return NC_ERR_SHAPE;
  const int M = B * T;
  const int64_t warps = (int64_t)M * H;
  if (f16)
    bwd::attn_delta_kernel<true><<<(unsigned)((warps + 7) / 8), 256, 0, stream>>>(dO, o, delta, M, H, D);
  else
    bwd::attn_delta_kernel<false><<<(unsigned)((warps + 7) / 8), 256, 0, stream>>>(dO, o, delta, M, H, D);
  if (cudaGetLastError() != cudaSuccess) return NC_ERR_CUDA;
  const int W = (window <= 0 || window > T) ? T : window;
  if (D == 128)
    return f16 ? bwd::attn_bwd_t<128, true>(qkv, ldqkv, dO, lse, delta, dqkv, B, T, H, Hkv, W, stream)
               : bwd::attn_bwd_t<128, false>(qkv, ldqkv, dO, lse, delta, dqkv, B, T, H, Hkv, W, stream);
  return f16 ? bwd::attn_bwd_t<64, true>(qkv, ldqkv, dO, lse, delta, dqkv, B, T, H, Hkv, W, stream)
             : bwd::attn_bwd_t<64, false>(qkv, ldqkv, dO, lse, delta, dqkv, B, T, H, Hkv, W, stream);
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
