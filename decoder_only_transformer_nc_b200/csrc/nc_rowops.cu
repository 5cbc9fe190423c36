// Bandwidth-bound steps of the forward: weight cast, embedding gather,
// parameter-free RMSNorm, RoPE table, fused RoPE + QK-norm, fused soft-cap +
// log-softmax + NLL, and the loss reductions.  Each kernel reads and writes
// every byte once with 8- or 16-byte coalesced accesses; reductions are warp
// shuffles in a fixed order, so results are run-to-run deterministic.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "nc_half.cuh"
#include "nc_internal.h"

namespace nc {
namespace {

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ---------------------------------------------------------------- weight cast

constexpr int kMaxCastSegs = 160;  // 4.0 KB of kernel parameters: one launch up to 26 layers
struct CastBatch {
  const float* src[kMaxCastSegs];
  uint16_t* dst[kMaxCastSegs];
  int64_t gstart[kMaxCastSegs + 1];  // prefix sums in groups of 8 elements
  uint8_t pair_rows[kMaxCastSegs];   // segment rows pair-interleaved within perm_d-row blocks
  int nseg;
  int perm_cols, perm_d;
};

// Each fp32 weight is rounded to bf16 (nearest even).  With F16 that bf16
// value is then stored in an fp16 container: exact for |w| >= 2^-14 (every
// bf16 value with 8 significant bits fits fp16's 11), nearest fp16 subnormal
// below that (absolute change <= 2^-25).
template <bool F16>
__device__ __forceinline__ uint32_t cast_pair(float a, float b) {
  if constexpr (F16) {
    const float ra = __bfloat162float(__float2bfloat16_rn(a));
    const float rb = __bfloat162float(__float2bfloat16_rn(b));
    return Half<true>::pack2(ra, rb);
  } else {
    return Half<false>::pack2(a, b);
  }
}

template <bool F16>
__global__ void __launch_bounds__(256) cast_kernel(const __grid_constant__ CastBatch cb) {
  const int64_t total = cb.gstart[cb.nseg];
  for (int64_t g = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; g < total;
       g += (int64_t)gridDim.x * blockDim.x) {
    int lo = 0, hi = cb.nseg - 1;  // last segment with gstart <= g
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (cb.gstart[mid] <= g) lo = mid; else hi = mid - 1;
    }
    const int64_t off = (g - cb.gstart[lo]) * 8;  // destination element offset
    int64_t soff = off;
    if (cb.pair_rows[lo]) {  // destination row 2j(+1) of a block reads source row j (+ d/2)
      const int64_t row = off / cb.perm_cols, col = off - row * cb.perm_cols;
      const int64_t blk = row / cb.perm_d, jj = row - blk * cb.perm_d;
      const int64_t srow = blk * cb.perm_d + (jj >> 1) + (jj & 1) * (cb.perm_d / 2);
      soff = srow * cb.perm_cols + col;
    }
    const float4* s = reinterpret_cast<const float4*>(cb.src[lo] + soff);
    const float4 a = __ldcs(s);
    const float4 b = __ldcs(s + 1);
    uint4 o;
    o.x = cast_pair<F16>(a.x, a.y);
    o.y = cast_pair<F16>(a.z, a.w);
    o.z = cast_pair<F16>(b.x, b.y);
    o.w = cast_pair<F16>(b.z, b.w);
    *reinterpret_cast<uint4*>(cb.dst[lo] + off) = o;
  }
}

// ---------------------------------------------------------------- embedding

__global__ void __launch_bounds__(256) embedding_kernel(const int32_t* __restrict__ tokens,
                                                        const float* __restrict__ wte,
                                                        float* __restrict__ x, int M, int C, int V,
                                                        uint32_t* dev_status) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= M) return;
  int tok = tokens[warp];
  if (tok < 0 || tok >= V) {
    if (lane == 0 && dev_status) atomicOr(dev_status, NC_DEV_TOKEN_RANGE);
    tok = 0;
  }
  const float4* src = reinterpret_cast<const float4*>(wte + (int64_t)tok * C);
  float4* dst = reinterpret_cast<float4*>(x + (int64_t)warp * C);
  for (int i = lane; i < C / 4; i += 32) dst[i] = src[i];
}

// Embedding with the smear term of the full nanochat forward ("Nanochat与nanoGPT
// 对比" §1, smear note): x_t = e_t + sigmoid(gate . e_t) e_{t-1} with e = wte[idx],
// gate's fp32 weights taken at their bf16 values, position 0 of a row
// unchanged.  One warp per token; the gate dot product is a warp reduction in
// fp32.  x0 (optional) receives a copy of the result.
template <bool SMEAR>
__global__ void __launch_bounds__(256) embedding_extra_kernel(const int32_t* __restrict__ tokens,
                                                              const float* __restrict__ wte,
                                                              const float* __restrict__ gate,
                                                              float* __restrict__ x, float* __restrict__ x0,
                                                              int M, int C, int V, int T,
                                                              uint32_t* dev_status) {
  const int m = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (m >= M) return;
  int tok = tokens[m];
  if (tok < 0 || tok >= V) {
    if (lane == 0 && dev_status) atomicOr(dev_status, NC_DEV_TOKEN_RANGE);
    tok = 0;
  }
  const float4* e = reinterpret_cast<const float4*>(wte + (int64_t)tok * C);
  float4* dst = reinterpret_cast<float4*>(x + (int64_t)m * C);
  float4* dst0 = x0 ? reinterpret_cast<float4*>(x0 + (int64_t)m * C) : nullptr;
  const int n4 = C / 4;
  if constexpr (SMEAR) {
    const bool has_prev = (m % T) != 0;
    int ptok = has_prev ? tokens[m - 1] : 0;
    if (ptok < 0 || ptok >= V) ptok = 0;  // flagged by that token's own warp
    const float4* ep = reinterpret_cast<const float4*>(wte + (int64_t)ptok * C);
    const float4* g4 = reinterpret_cast<const float4*>(gate);
    float dot = 0.0f;
    for (int i = lane; i < n4; i += 32) {
      const float4 a = e[i], g = g4[i];
      dot = fmaf(a.x, __bfloat162float(__float2bfloat16_rn(g.x)), dot);
      dot = fmaf(a.y, __bfloat162float(__float2bfloat16_rn(g.y)), dot);
      dot = fmaf(a.z, __bfloat162float(__float2bfloat16_rn(g.z)), dot);
      dot = fmaf(a.w, __bfloat162float(__float2bfloat16_rn(g.w)), dot);
    }
    dot = warp_sum(dot);
    const float sg = has_prev ? 1.0f / (1.0f + expf(-dot)) : 0.0f;
    for (int i = lane; i < n4; i += 32) {
      float4 a = e[i];
      if (has_prev) {
        const float4 b = ep[i];
        a.x = fmaf(sg, b.x, a.x);
        a.y = fmaf(sg, b.y, a.y);
        a.z = fmaf(sg, b.z, a.z);
        a.w = fmaf(sg, b.w, a.w);
      }
      dst[i] = a;
      if (dst0) dst0[i] = a;
    }
  } else {
    for (int i = lane; i < n4; i += 32) {
      const float4 a = e[i];
      dst[i] = a;
      if (dst0) dst0[i] = a;
    }
  }
}

// ---------------------------------------------------------------- RMSNorm

// One warp per row; the row is held in registers (C <= 32 * 4 * NV).  With
// amax != NULL the largest |stored value| is folded into *amax (the e4m3
// quantisation of the output that follows).
template <int NV, bool F16>
__global__ void __launch_bounds__(256) rmsnorm_kernel(const float* __restrict__ x,
                                                      uint16_t* __restrict__ out, int M, int C,
                                                      float eps, float* __restrict__ amax) {
  const int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= M) return;
  const float4* xr = reinterpret_cast<const float4*>(x + (int64_t)row * C);
  const int n4 = C >> 2;
  float4 v[NV];
  float ss = 0.0f;
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int i = j * 32 + lane;
    v[j] = i < n4 ? xr[i] : make_float4(0.f, 0.f, 0.f, 0.f);
    ss += v[j].x * v[j].x + v[j].y * v[j].y + v[j].z * v[j].z + v[j].w * v[j].w;
  }
  ss = warp_sum(ss);
  const float r = rsqrtf(ss / (float)C + eps);
  uint2* o = reinterpret_cast<uint2*>(out + (int64_t)row * C);
  uint32_t om = 0;
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int i = j * 32 + lane;
    if (i < n4) {
      const float a = v[j].x * r, b = v[j].y * r, c = v[j].z * r, d = v[j].w * r;
      o[i] = make_uint2(Half<F16>::pack2(a, b), Half<F16>::pack2(c, d));
      if (amax)
        om = max(max(om, max(__float_as_uint(a) & 0x7FFFFFFFu, __float_as_uint(b) & 0x7FFFFFFFu)),
                 max(__float_as_uint(c) & 0x7FFFFFFFu, __float_as_uint(d) & 0x7FFFFFFFu));
    }
  }
  if (amax) {
    om = __reduce_max_sync(0xFFFFFFFFu, om);
    if (lane == 0) fold_amax(amax, stored_abs_bits<F16>(om));
  }
}

// Two-pass variant for wide rows.
template <bool F16>
__global__ void __launch_bounds__(256) rmsnorm_wide_kernel(const float* __restrict__ x,
                                                           uint16_t* __restrict__ out, int M, int C,
                                                           float eps, float* __restrict__ amax) {
  const int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= M) return;
  const float4* xr = reinterpret_cast<const float4*>(x + (int64_t)row * C);
  const int n4 = C >> 2;
  float ss = 0.0f;
  for (int i = lane; i < n4; i += 32) {
    const float4 a = xr[i];
    ss += a.x * a.x + a.y * a.y + a.z * a.z + a.w * a.w;
  }
  ss = warp_sum(ss);
  const float r = rsqrtf(ss / (float)C + eps);
  uint2* o = reinterpret_cast<uint2*>(out + (int64_t)row * C);
  uint32_t om = 0;
  for (int i = lane; i < n4; i += 32) {
    const float4 a = xr[i];
    const float p = a.x * r, q = a.y * r, u = a.z * r, w = a.w * r;
    o[i] = make_uint2(Half<F16>::pack2(p, q), Half<F16>::pack2(u, w));
    om = max(max(om, max(__float_as_uint(p) & 0x7FFFFFFFu, __float_as_uint(q) & 0x7FFFFFFFu)),
             max(__float_as_uint(u) & 0x7FFFFFFFu, __float_as_uint(w) & 0x7FFFFFFFu));
  }
  if (amax) {
    om = __reduce_max_sync(0xFFFFFFFFu, om);
    if (lane == 0) fold_amax(amax, stored_abs_bits<F16>(om));
  }
}

// RMSNorm fused with the residual-stream terms of the full nanochat forward
// ("Nanochat与nanoGPT对比" §1: per-layer resid_lambdas + x0, backout).  Per row:
// u = x; x_keep = u (optional); u = lam_r u + lam_0 x0 (optional); u = u -
// lam_sub x_sub (optional); x = u (write_back); out = u / sqrt(mean(u^2) + eps).
// One warp per row; the row is held in registers (C <= 32 * 4 * NV), or streamed
// twice when NV == 0.
template <int NV, bool F16>
__global__ void __launch_bounds__(256) rmsnorm_mix_kernel(float* __restrict__ x,
                                                          const float* __restrict__ x0,
                                                          const float* __restrict__ lam_r,
                                                          const float* __restrict__ lam_0,
                                                          float* __restrict__ x_keep,
                                                          const float* __restrict__ x_sub,
                                                          const float* __restrict__ lam_sub, int write_back,
                                                          uint16_t* __restrict__ out, int M, int C,
                                                          float eps) {
  const int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= M) return;
  const int64_t base = (int64_t)row * C;
  const int n4 = C >> 2;
  const float lr = x0 ? *lam_r : 1.0f, l0 = x0 ? *lam_0 : 0.0f;
  const float ls = x_sub ? *lam_sub : 0.0f;
  float4* xr = reinterpret_cast<float4*>(x + base);
  auto mix = [&](int i) -> float4 {
    float4 u = xr[i];
    if (x_keep) reinterpret_cast<float4*>(x_keep + base)[i] = u;
    if (x0) {
      const float4 b = reinterpret_cast<const float4*>(x0 + base)[i];
      u = make_float4(fmaf(lr, u.x, l0 * b.x), fmaf(lr, u.y, l0 * b.y), fmaf(lr, u.z, l0 * b.z),
                      fmaf(lr, u.w, l0 * b.w));
    }
    if (x_sub) {
      const float4 b = reinterpret_cast<const float4*>(x_sub + base)[i];
      u = make_float4(fmaf(-ls, b.x, u.x), fmaf(-ls, b.y, u.y), fmaf(-ls, b.z, u.z), fmaf(-ls, b.w, u.w));
    }
    if (write_back) xr[i] = u;
    return u;
  };
  uint2* o = reinterpret_cast<uint2*>(out + base);
  if constexpr (NV > 0) {
    // All loads of the row are issued before any arithmetic, so each lane keeps
    // up to 2 NV 16-byte reads in flight.
    float4 v[NV], b[NV];
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      const int i = j * 32 + lane;
      v[j] = i < n4 ? xr[i] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    const float* other = x0 ? x0 : x_sub;
    if (other) {
#pragma unroll
      for (int j = 0; j < NV; ++j) {
        const int i = j * 32 + lane;
        b[j] = i < n4 ? reinterpret_cast<const float4*>(other + base)[i] : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    if (x_keep) {
#pragma unroll
      for (int j = 0; j < NV; ++j) {
        const int i = j * 32 + lane;
        if (i < n4) reinterpret_cast<float4*>(x_keep + base)[i] = v[j];
      }
    }
    if (x0) {
#pragma unroll
      for (int j = 0; j < NV; ++j)
        v[j] = make_float4(fmaf(lr, v[j].x, l0 * b[j].x), fmaf(lr, v[j].y, l0 * b[j].y),
                           fmaf(lr, v[j].z, l0 * b[j].z), fmaf(lr, v[j].w, l0 * b[j].w));
    }
    if (x_sub) {
      if (x0) {  // both terms: x_sub is read now (not in the forward, which never combines them)
#pragma unroll
        for (int j = 0; j < NV; ++j) {
          const int i = j * 32 + lane;
          b[j] = i < n4 ? reinterpret_cast<const float4*>(x_sub + base)[i] : make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
#pragma unroll
      for (int j = 0; j < NV; ++j)
        v[j] = make_float4(fmaf(-ls, b[j].x, v[j].x), fmaf(-ls, b[j].y, v[j].y), fmaf(-ls, b[j].z, v[j].z),
                           fmaf(-ls, b[j].w, v[j].w));
    }
    float ss = 0.0f;
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      const int i = j * 32 + lane;
      if (write_back && i < n4) xr[i] = v[j];
      ss += v[j].x * v[j].x + v[j].y * v[j].y + v[j].z * v[j].z + v[j].w * v[j].w;
    }
    ss = warp_sum(ss);
    const float r = rsqrtf(ss / (float)C + eps);
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      const int i = j * 32 + lane;
      if (i < n4)
        o[i] = make_uint2(Half<F16>::pack2(v[j].x * r, v[j].y * r), Half<F16>::pack2(v[j].z * r, v[j].w * r));
    }
  } else {
    // Wide rows: pass 1 forms u (written back, or kept nowhere) and its sum of
    // squares; pass 2 re-reads u from x when written back, else forms it again
    // (x_keep only in pass 1).
    float ss = 0.0f;
    for (int i = lane; i < n4; i += 32) {
      const float4 u = mix(i);
      ss += u.x * u.x + u.y * u.y + u.z * u.z + u.w * u.w;
    }
    ss = warp_sum(ss);
    const float r = rsqrtf(ss / (float)C + eps);
    __syncwarp();
    for (int i = lane; i < n4; i += 32) {
      float4 u = xr[i];
      if (!write_back) {
        if (x0) {
          const float4 b = reinterpret_cast<const float4*>(x0 + base)[i];
          u = make_float4(fmaf(lr, u.x, l0 * b.x), fmaf(lr, u.y, l0 * b.y), fmaf(lr, u.z, l0 * b.z),
                          fmaf(lr, u.w, l0 * b.w));
        }
        if (x_sub) {
          const float4 b = reinterpret_cast<const float4*>(x_sub + base)[i];
          u = make_float4(fmaf(-ls, b.x, u.x), fmaf(-ls, b.y, u.y), fmaf(-ls, b.z, u.z), fmaf(-ls, b.w, u.w));
        }
      }
      o[i] = make_uint2(Half<F16>::pack2(u.x * r, u.y * r), Half<F16>::pack2(u.z * r, u.w * r));
    }
  }
}

// ---------------------------------------------------------------- RoPE

// Threads [0, T D/2) write the [2][T][D/2] table in its order; with `pairs`,
// threads [T D/2, T D) write the [D/2][T] (cos, sin) copy in its own order, so
// both stores are coalesced.  Both compute the same fp64 angle.
__global__ void rope_table_kernel(float* __restrict__ table, int T, int D, double base,
                                  float2* __restrict__ pairs) {
  const int half = D / 2;
  const int n = T * half;
  int idx = blockIdx.x * blockDim.x + threadIdx.x;
  const bool pair_major = idx >= n;
  if (pair_major) idx -= n;
  if (idx >= n || (pair_major && !pairs)) return;
  const int t = pair_major ? idx % T : idx / half;
  const int i = pair_major ? idx / T : idx % half;
  const double theta = pow(base, -2.0 * (double)i / (double)D);
  const double ang = (double)t * theta;
  const float c = (float)cos(ang), s = (float)sin(ang);
  if (pair_major) {
    pairs[idx] = make_float2(c, s);
  } else {
    table[idx] = c;
    table[(int64_t)n + idx] = s;
  }
}

// One group of D/4 lanes per (token, head).  Lane l of the group holds the
// bf16 pairs at dims (2l, 2l+1) and (D/2+2l, D/2+2l+1), i.e. both members of
// the RoPE pairs 2l and 2l+1, so the rotation needs no shuffles; the per-head
// sum of squares is a shuffle reduction inside the group.
template <int D, bool F16>
__global__ void __launch_bounds__(256) rope_qknorm_kernel(uint16_t* __restrict__ q,
                                                          uint16_t* __restrict__ k,
                                                          const float* __restrict__ table, int M,
                                                          int T, int H, int Hkv, int64_t q_stride,
                                                          int64_t k_stride, float eps) {
  constexpr int LPH = D / 4;  // lanes per head
  constexpr int HALF = D / 2;
  const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t unit = gid / LPH;  // (token, head) index
  const int l = (int)(gid % LPH);
  const int heads = H + Hkv;
  const bool active = unit < (int64_t)M * heads;
  const int64_t m = active ? unit / heads : 0;
  const int j = active ? (int)(unit - m * heads) : 0;
  const int t = (int)(m % T);
  uint16_t* p = j < H ? q + m * q_stride + (int64_t)j * D : k + m * k_stride + (int64_t)(j - H) * D;
  float ra0 = 0.f, ra1 = 0.f, rb0 = 0.f, rb1 = 0.f;
  if (active) {
    const float2 a = Half<F16>::unpack2(*reinterpret_cast<const uint32_t*>(p + 2 * l));
    const float2 b = Half<F16>::unpack2(*reinterpret_cast<const uint32_t*>(p + HALF + 2 * l));
    const float2 c = *reinterpret_cast<const float2*>(table + (int64_t)t * HALF + 2 * l);
    const float2 s = *reinterpret_cast<const float2*>(table + (int64_t)T * HALF + (int64_t)t * HALF + 2 * l);
    ra0 = a.x * c.x - b.x * s.x;
    rb0 = a.x * s.x + b.x * c.x;
    ra1 = a.y * c.y - b.y * s.y;
    rb1 = a.y * s.y + b.y * c.y;
  }
  float ss = ra0 * ra0 + ra1 * ra1 + rb0 * rb0 + rb1 * rb1;
#pragma unroll
  for (int o = LPH / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if (active) {
    const float r = rsqrtf(ss / (float)D + eps);
    *reinterpret_cast<uint32_t*>(p + 2 * l) = Half<F16>::pack2(ra0 * r, ra1 * r);
    *reinterpret_cast<uint32_t*>(p + HALF + 2 * l) = Half<F16>::pack2(rb0 * r, rb1 * r);
  }
}

// ---------------------------------------------------------------- cross-entropy

// Block-wide sum in a fixed order (warp shuffles, then warp 0 over the partials).
__device__ __forceinline__ float block_sum(float v, float* red) {
  v = warp_sum(v);
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[w] = v;
  __syncthreads();
  if (w == 0) {
    float t = lane < (int)(blockDim.x >> 5) ? red[lane] : 0.0f;
    t = warp_sum(t);
    if (lane == 0) red[32] = t;
  }
  __syncthreads();
  const float r = red[32];
  __syncthreads();
  return r;
}

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

// l = cap * tanh(z / cap) = cap - 2 cap r with r = 1 / (1 + e^(2z/cap)), and
// exp(l - cap) = e^(-2 cap r): three MUFU operations per logit, exact limits.
__device__ __forceinline__ float softcap_p(float z, float k_in, float cap, float k_out, float& p) {
  const float r = rcp_approx(1.0f + ex2_approx(z * k_in));
  p = ex2_approx(k_out * r);
  return fmaf(-2.0f * cap, r, cap);
}

// One CTA per row.  Soft-capped logits lie in (-cap, cap), so
// logsumexp(l) = cap + log(sum exp(l - cap)) needs no running maximum.
__global__ void __launch_bounds__(256) softcap_ce_kernel(const float* __restrict__ z,
                                                         const int32_t* __restrict__ targets,
                                                         float* capped_out,
                                                         float* __restrict__ token_loss, int V,
                                                         float cap, uint32_t* dev_status) {
  __shared__ float red[33];
  const int64_t row = blockIdx.x;
  const float4* zr = reinterpret_cast<const float4*>(z + row * V);
  float4* cr = capped_out ? reinterpret_cast<float4*>(capped_out + row * V) : nullptr;
  const float k_in = 2.0f * 1.4426950408889634f / cap;
  const float k_out = -2.0f * cap * 1.4426950408889634f;
  float s = 0.0f;
  for (int i = threadIdx.x; i < V / 4; i += blockDim.x) {
    float4 a = __ldcs(zr + i);
    float p0, p1, p2, p3;
    a.x = softcap_p(a.x, k_in, cap, k_out, p0);
    a.y = softcap_p(a.y, k_in, cap, k_out, p1);
    a.z = softcap_p(a.z, k_in, cap, k_out, p2);
    a.w = softcap_p(a.w, k_in, cap, k_out, p3);
    s += (p0 + p1) + (p2 + p3);
    if (cr) cr[i] = a;
  }
  s = block_sum(s, red);
  if (threadIdx.x == 0) {
    const int y = targets[row];
    float nll = 0.0f;
    if (y >= 0 && y < V) {
      float unused;
      const float ly = softcap_p(z[row * V + y], k_in, cap, k_out, unused);
      nll = cap + logf(s) - ly;
    } else if (y != -1 && dev_status) {
      atomicOr(dev_status, NC_DEV_TARGET_RANGE);
    }
    token_loss[row] = nll;
  }
}

// Combines the per-tile partial sums written by the lm_head GEMM epilogue:
// one warp per row, fixed summation order.
__global__ void __launch_bounds__(256) ce_finalize_kernel(const float* __restrict__ partial,
                                                          int n_tiles,
                                                          const float* __restrict__ target_logit,
                                                          const int32_t* __restrict__ targets,
                                                          float* __restrict__ token_loss, int M,
                                                          int V, float cap, uint32_t* dev_status) {
  const int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= M) return;
  const float* pr = partial + (int64_t)row * n_tiles;
  float s = 0.0f;
  for (int i = lane; i < n_tiles; i += 32) s += pr[i];
  s = warp_sum(s);
  if (lane == 0) {
    const int y = targets[row];
    float nll = 0.0f;
    if (y >= 0 && y < V) {
      nll = cap + logf(s) - target_logit[row];
    } else if (y != -1 && dev_status) {
      atomicOr(dev_status, NC_DEV_TARGET_RANGE);
    }
    token_loss[row] = nll;
  }
}

// Single CTA, fixed-order reduction in fp64: mean over valid targets.
__global__ void __launch_bounds__(1024) loss_mean_kernel(const float* __restrict__ token_loss,
                                                         const int32_t* __restrict__ targets, int M,
                                                         int V, float* loss, float* inv_count) {
  __shared__ double rs[32];
  __shared__ int rc[32];
  double s = 0.0;
  int c = 0;
  for (int i = threadIdx.x; i < M; i += blockDim.x) {
    const int y = targets[i];
    if (y >= 0 && y < V) {
      s += (double)token_loss[i];
      ++c;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    s += __shfl_xor_sync(0xffffffffu, s, o);
    c += __shfl_xor_sync(0xffffffffu, c, o);
  }
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    rs[w] = s;
    rc[w] = c;
  }
  __syncthreads();
  if (w == 0) {
    const int nw = blockDim.x >> 5;
    s = lane < nw ? rs[lane] : 0.0;
    c = lane < nw ? rc[lane] : 0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      s += __shfl_xor_sync(0xffffffffu, s, o);
      c += __shfl_xor_sync(0xffffffffu, c, o);
    }
    if (lane == 0) {
      loss[0] = c > 0 ? (float)(s / (double)c) : __int_as_float(0x7fc00000);
      if (inv_count) inv_count[0] = c > 0 ? (float)(1.0 / (double)c) : 0.0f;
    }
  }
}

inline nc_status last_error() { return cudaGetLastError() == cudaSuccess ? NC_OK : NC_ERR_CUDA; }

}  // namespace

nc_status cast_launch(const CastSeg* segs, int nseg, bool f16, cudaStream_t stream, int perm_cols,
                      int perm_d) {
  for (int base = 0; base < nseg; base += kMaxCastSegs) {
    CastBatch cb;
    cb.nseg = nseg - base < kMaxCastSegs ? nseg - base : kMaxCastSegs;
    cb.perm_cols = perm_cols;
    cb.perm_d = perm_d;
    cb.gstart[0] = 0;
    for (int i = 0; i < cb.nseg; ++i) {
      cb.src[i] = segs[base + i].src;
      cb.dst[i] = segs[base + i].dst;
      cb.gstart[i + 1] = cb.gstart[i] + segs[base + i].n / 8;
      cb.pair_rows[i] = segs[base + i].pair_rows ? 1 : 0;
      if (cb.pair_rows[i] && (perm_cols <= 0 || perm_cols % 8 || perm_d < 2 || perm_d % 2)) return NC_ERR_INVALID_ARG;
    }
    const int64_t groups = cb.gstart[cb.nseg];
    if (groups == 0) continue;
    const int64_t want = (groups + 255) / 256;
    const int grid = (int)(want < 148 * 16 ? want : 148 * 16);
    if (f16)
      cast_kernel<true><<<grid, 256, 0, stream>>>(cb);
    else
      cast_kernel<false><<<grid, 256, 0, stream>>>(cb);
    if (cudaGetLastError() != cudaSuccess) return NC_ERR_CUDA;
  }
  return NC_OK;
}

nc_status embedding_launch(const int32_t* tokens, const float* wte, float* x, int M, int C, int V,
                           uint32_t* dev_status, cudaStream_t stream) {
  if (M == 0) return NC_OK;
  const int grid = (M + 7) / 8;
  embedding_kernel<<<grid, 256, 0, stream>>>(tokens, wte, x, M, C, V, dev_status);
  return last_error();
}

nc_status embedding_extra_launch(const int32_t* tokens, const float* wte, const float* smear_gate,
                                 float* x, float* x0, int M, int C, int V, int T, uint32_t* dev_status,
                                 cudaStream_t stream) {
  if (M == 0) return NC_OK;
  const int grid = (M + 7) / 8;
  if (smear_gate)
    embedding_extra_kernel<true><<<grid, 256, 0, stream>>>(tokens, wte, smear_gate, x, x0, M, C, V, T, dev_status);
  else
    embedding_extra_kernel<false><<<grid, 256, 0, stream>>>(tokens, wte, nullptr, x, x0, M, C, V, T, dev_status);
  return last_error();
}

template <bool F16>
static void rmsnorm_mix_dispatch(float* x, const float* x0, const float* lr, const float* l0, float* keep,
                                 const float* sub, const float* ls, int wb, uint16_t* out, int M, int C,
                                 float eps, cudaStream_t stream) {
  const int grid = (M + 7) / 8;
  if (C <= 32 * 4 * 4)
    rmsnorm_mix_kernel<4, F16><<<grid, 256, 0, stream>>>(x, x0, lr, l0, keep, sub, ls, wb, out, M, C, eps);
  else if (C <= 32 * 4 * 8)
    rmsnorm_mix_kernel<8, F16><<<grid, 256, 0, stream>>>(x, x0, lr, l0, keep, sub, ls, wb, out, M, C, eps);
  else if (C <= 32 * 4 * 16)
    rmsnorm_mix_kernel<16, F16><<<grid, 256, 0, stream>>>(x, x0, lr, l0, keep, sub, ls, wb, out, M, C, eps);
  else
    rmsnorm_mix_kernel<0, F16><<<grid, 256, 0, stream>>>(x, x0, lr, l0, keep, sub, ls, wb, out, M, C, eps);
}

nc_status rmsnorm_mix_launch(float* x, const float* x0, const float* lam_r, const float* lam_0,
                             float* x_keep, const float* x_sub, const float* lam_sub, bool write_back,
                             uint16_t* out, int M, int C, float eps, bool f16, cudaStream_t stream) {
  if (M == 0) return NC_OK;
  if (f16)
    rmsnorm_mix_dispatch<true>(x, x0, lam_r, lam_0, x_keep, x_sub, lam_sub, write_back ? 1 : 0, out, M, C, eps,
                               stream);
  else
    rmsnorm_mix_dispatch<false>(x, x0, lam_r, lam_0, x_keep, x_sub, lam_sub, write_back ? 1 : 0, out, M, C,
                                eps, stream);
  return last_error();
}

template <bool F16>
static void rmsnorm_dispatch(const float* x, uint16_t* out, int M, int C, float eps, float* amax,
                             cudaStream_t stream) {
  const int grid = (M + 7) / 8;
  if (C <= 32 * 4 * 4)
    rmsnorm_kernel<4, F16><<<grid, 256, 0, stream>>>(x, out, M, C, eps, amax);
  else if (C <= 32 * 4 * 8)
    rmsnorm_kernel<8, F16><<<grid, 256, 0, stream>>>(x, out, M, C, eps, amax);
  else if (C <= 32 * 4 * 16)
    rmsnorm_kernel<16, F16><<<grid, 256, 0, stream>>>(x, out, M, C, eps, amax);
  else
    rmsnorm_wide_kernel<F16><<<grid, 256, 0, stream>>>(x, out, M, C, eps, amax);
}

nc_status rmsnorm_launch(const float* x, uint16_t* out, int M, int C, float eps, bool f16,
                         cudaStream_t stream, float* amax) {
  if (M == 0) return NC_OK;
  if (f16)
    rmsnorm_dispatch<true>(x, out, M, C, eps, amax, stream);
  else
    rmsnorm_dispatch<false>(x, out, M, C, eps, amax, stream);
  return last_error();
}

nc_status rope_table_launch(float* table, int T, int D, float base, cudaStream_t stream, float2* pairs) {
  const int n = T * (D / 2) * (pairs ? 2 : 1);
  if (n == 0) return NC_OK;
  rope_table_kernel<<<(n + 255) / 256, 256, 0, stream>>>(table, T, D, (double)base, pairs);
  return last_error();
}

nc_status rope_qknorm_launch(uint16_t* q, uint16_t* k, const float* table, int B, int T, int H,
                             int Hkv, int D, int64_t q_stride, int64_t k_stride, float eps, bool f16,
                             cudaStream_t stream) {
  const int64_t M = (int64_t)B * T;
  const int64_t threads = M * (H + Hkv) * (D / 4);
  if (threads == 0) return NC_OK;
  const unsigned grid = (unsigned)((threads + 255) / 256);
  if (D == 128 && f16)
    rope_qknorm_kernel<128, true><<<grid, 256, 0, stream>>>(q, k, table, (int)M, T, H, Hkv, q_stride, k_stride, eps);
  else if (D == 128)
    rope_qknorm_kernel<128, false><<<grid, 256, 0, stream>>>(q, k, table, (int)M, T, H, Hkv, q_stride, k_stride, eps);
  else if (D == 64 && f16)
    rope_qknorm_kernel<64, true><<<grid, 256, 0, stream>>>(q, k, table, (int)M, T, H, Hkv, q_stride, k_stride, eps);
  else if (D == 64)
    rope_qknorm_kernel<64, false><<<grid, 256, 0, stream>>>(q, k, table, (int)M, T, H, Hkv, q_stride, k_stride, eps);
  else
    return NC_ERR_SHAPE;
  return last_error();
}

nc_status softcap_ce_launch(const float* z, const int32_t* targets, float* capped_out,
                            float* token_loss, int M, int V, float cap, uint32_t* dev_status,
                            cudaStream_t stream) {
  if (M == 0) return NC_OK;
  softcap_ce_kernel<<<M, 256, 0, stream>>>(z, targets, capped_out, token_loss, V, cap, dev_status);
  return last_error();
}

nc_status ce_finalize_launch(const float* partial, int n_tiles, const float* target_logit,
                             const int32_t* targets, float* token_loss, int M, int V, float cap,
                             uint32_t* dev_status, cudaStream_t stream) {
  if (M == 0) return NC_OK;
  ce_finalize_kernel<<<(M + 7) / 8, 256, 0, stream>>>(partial, n_tiles, target_logit, targets,
                                                      token_loss, M, V, cap, dev_status);
  return last_error();
}

nc_status loss_mean_launch(const float* token_loss, const int32_t* targets, int M, int V,
                           float* loss, cudaStream_t stream, float* inv_count) {
  loss_mean_kernel<<<1, 1024, 0, stream>>>(token_loss, targets, M, V, loss, inv_count);
  return last_error();
}

}  // namespace nc
