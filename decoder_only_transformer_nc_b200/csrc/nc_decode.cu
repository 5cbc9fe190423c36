// KV-cache inference: cache append and the attention of one new position per
// row over the cached keys ("从文本到聊天模型" §10.1-10.4: the prompt's keys and
// values are kept per layer, and each further token attends over them instead
// of recomputing the whole prefix).
//
// Cache of one layer: [B][T_max][2][Hkv][D] 16-bit -- for each row and position
// the k heads (after RoPE and QK-norm, in the pair-interleaved order the
// forward's QKV epilogue produces) followed by the v heads.  q uses the same
// order, so q . k is unchanged.
//
// Decode attention is bound by reading the cached K/V.  Grid (split, kv head,
// row): each CTA takes a chunk of 64 (or more) consecutive visible keys of
// [lo, pos] for all query heads of one kv group (GQA: the group's heads share
// every K/V row the CTA reads).  It copies the chunk's K and V head slices into
// shared memory with 16-byte asynchronous copies, all in flight at once, then
// four warps stride over the keys with every lane holding D/32 dimensions.
// Softmax is the exact online form in fp32 (log2 domain).  Each CTA leaves
// (m, l, o) per head; a second kernel merges the splits.
#include <cuda_runtime.h>

#include <cstdint>

#include "nc_half.cuh"
#include "nc_internal.h"
#include "nc_mma.cuh"

namespace nc {
namespace {

constexpr int kMaxSplits = 32;
constexpr int kWarps = 4;

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float warp_allsum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__global__ void __launch_bounds__(256) kv_append_kernel(const uint4* __restrict__ qkv, int64_t ldq16,
                                                        int col16, int width16, uint4* __restrict__ cache,
                                                        int M, int T, int T_max, int pos0) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (int64_t)M * width16) return;
  const int m = (int)(idx / width16);
  const int c = (int)(idx - (int64_t)m * width16);
  const int b = m / T, t = pos0 + m % T;
  cache[((int64_t)b * T_max + t) * width16 + c] = qkv[(int64_t)m * ldq16 + col16 + c];
}

// DW: dimensions per lane (D / 32); G: query heads per kv head.  The CTA first
// copies the K and V head slices of its chunk of keys (kChunk rows of D 16-bit
// values each) into shared memory with 16-byte asynchronous copies, all in
// flight at once, then computes from there.
template <int DW, int G, bool F16>
__global__ void __launch_bounds__(kWarps * 32) decode_attn_kernel(const uint16_t* __restrict__ q, int64_t ldq,
                                                                  const uint16_t* __restrict__ cache,
                                                                  float* __restrict__ partial, int H, int Hkv,
                                                                  int T_max, int lo, int hi, int chunk,
                                                                  float scale_log2, const int* __restrict__ pos_dev,
                                                                  int W) {
  constexpr int D = DW * 32;
  const int s = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (pos_dev) {  // position from device memory (a graph replays the step): clamp to the cache
    hi = min(max(*pos_dev, 0), T_max - 1);
    lo = max(hi - W + 1, 0);
  }
  const int k_begin = lo + s * chunk;
  const int n = min(k_begin + chunk, hi + 1) - k_begin;  // keys of this CTA (<= kChunk)
  if (n <= 0) return;  // a split past the context (fixed-size grid only)

  extern __shared__ __align__(16) uint16_t kv_s[];  // [n][2][D]: k then v of each key
  {
    constexpr int PARTS = 2 * D / 8;  // 16-byte pieces per key (k and v)
    const int64_t row_stride = 2 * (int64_t)Hkv * D;
    const uint16_t* base = cache + ((int64_t)b * T_max + k_begin) * row_stride;
    for (int e = threadIdx.x; e < n * PARTS; e += kWarps * 32) {
      const int r = e / PARTS, part = e - r * PARTS;
      const int kv = part / (D / 8), off = (part % (D / 8)) * 8;
      const uint16_t* src = base + r * row_stride + (int64_t)(kv * Hkv + g) * D + off;
      const uint32_t dst = (uint32_t)__cvta_generic_to_shared(kv_s + (r * 2 + kv) * D + off);
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  }

  float qv[G][DW];
#pragma unroll
  for (int i = 0; i < G; ++i) {
    const uint16_t* qp = q + (int64_t)b * ldq + (int64_t)(g * G + i) * D + lane * DW;
#pragma unroll
    for (int d = 0; d < DW; d += 2) {
      const float2 f = Half<F16>::unpack2(*reinterpret_cast<const uint32_t*>(qp + d));
      qv[i][d] = f.x;
      qv[i][d + 1] = f.y;
    }
  }
  float m[G], l[G], o[G][DW];
#pragma unroll
  for (int i = 0; i < G; ++i) {
    m[i] = -INFINITY;
    l[i] = 0.0f;
#pragma unroll
    for (int d = 0; d < DW; ++d) o[i][d] = 0.0f;
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  __syncthreads();

  // Keys in groups of four per warp: four independent dot-product reductions,
  // then one max / rescale for the group, so the online softmax's dependency
  // chain is per group rather than per key.
  constexpr int U = 4;
  for (int r0 = warp * U; r0 < n; r0 += kWarps * U) {
    float kf[U][DW], vf[U][DW];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int r = r0 + u < n ? r0 + u : r0;  // past the end: a valid row, masked below
      const uint16_t* kr = kv_s + (r * 2) * D + lane * DW;
#pragma unroll
      for (int d = 0; d < DW; d += 2) {
        const float2 kk = Half<F16>::unpack2(*reinterpret_cast<const uint32_t*>(kr + d));
        const float2 vv = Half<F16>::unpack2(*reinterpret_cast<const uint32_t*>(kr + D + d));
        kf[u][d] = kk.x;
        kf[u][d + 1] = kk.y;
        vf[u][d] = vv.x;
        vf[u][d + 1] = vv.y;
      }
    }
#pragma unroll
    for (int i = 0; i < G; ++i) {
      float sc[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        float dot = 0.0f;
#pragma unroll
        for (int d = 0; d < DW; ++d) dot = fmaf(qv[i][d], kf[u][d], dot);
        sc[u] = dot;
      }
#pragma unroll
      for (int o2 = 16; o2 > 0; o2 >>= 1)
#pragma unroll
        for (int u = 0; u < U; ++u) sc[u] += __shfl_xor_sync(0xffffffffu, sc[u], o2);
      float mx = m[i];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        sc[u] = r0 + u < n ? sc[u] * scale_log2 : -INFINITY;
        mx = fmaxf(mx, sc[u]);
      }
      const float a = ex2(m[i] - mx);  // 0 on the first group (m = -inf)
      float ps = 0.0f, pv[DW];
#pragma unroll
      for (int d = 0; d < DW; ++d) pv[d] = 0.0f;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const float p = ex2(sc[u] - mx);  // 0 for the masked tail
        ps += p;
#pragma unroll
        for (int d = 0; d < DW; ++d) pv[d] = fmaf(p, vf[u][d], pv[d]);
      }
      l[i] = fmaf(l[i], a, ps);
#pragma unroll
      for (int d = 0; d < DW; ++d) o[i][d] = fmaf(o[i][d], a, pv[d]);
      m[i] = mx;
    }
  }
  // merge the four warps (reusing the K/V staging area), then write this
  // split's (m, l, o) per head
  __syncthreads();
  float* sm_ml = reinterpret_cast<float*>(kv_s);          // [kWarps][G][2]
  float* sm_o = sm_ml + kWarps * G * 2;                    // [kWarps][G][D]
#pragma unroll
  for (int i = 0; i < G; ++i) {
    if (lane == 0) {
      sm_ml[(warp * G + i) * 2] = m[i];
      sm_ml[(warp * G + i) * 2 + 1] = l[i];
    }
#pragma unroll
    for (int d = 0; d < DW; ++d) sm_o[(warp * G + i) * D + lane * DW + d] = o[i][d];
  }
  __syncthreads();
  for (int e = threadIdx.x; e < G * D; e += kWarps * 32) {
    const int i = e / D, d = e - i * D;
    float mm = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) mm = fmaxf(mm, sm_ml[(w * G + i) * 2]);
    float ll = 0.0f, oo = 0.0f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float mw = sm_ml[(w * G + i) * 2];
      const float f = mw == -INFINITY ? 0.0f : ex2(mw - mm);
      ll = fmaf(sm_ml[(w * G + i) * 2 + 1], f, ll);
      oo = fmaf(sm_o[(w * G + i) * D + d], f, oo);
    }
    float* dst = partial + (((int64_t)b * H + g * G + i) * kMaxSplits + s) * (2 + D);
    if (d == 0) {
      dst[0] = mm;
      dst[1] = ll;
    }
    dst[2 + d] = oo;
  }
}

// One block per (row, head); thread d merges dimension d over the splits.
template <bool F16>
__global__ void decode_combine_kernel(const float* __restrict__ partial, uint16_t* __restrict__ out, int H, int D,
                                      int splits, const int* __restrict__ pos_dev, int T_max, int W, int chunk) {
  const int bh = blockIdx.x;
  const int d = threadIdx.x;
  if (pos_dev) {  // the same split count the attention kernel used
    const int hi = min(max(*pos_dev, 0), T_max - 1), lo = max(hi - W + 1, 0);
    splits = (hi - lo + 1 + chunk - 1) / chunk;
  }
  const float* p = partial + (int64_t)bh * kMaxSplits * (2 + D);
  // every split's (m, l, o[d]) read up front: independent loads, one round trip
  float ms[kMaxSplits], ls[kMaxSplits], os[kMaxSplits];
#pragma unroll
  for (int s = 0; s < kMaxSplits; ++s) {
    if (s < splits) {
      const float* q = p + s * (2 + D);
      ms[s] = q[0];
      ls[s] = q[1];
      os[s] = q[2 + d];
    } else {
      ms[s] = -INFINITY;
      ls[s] = 0.0f;
      os[s] = 0.0f;
    }
  }
  float mm = -INFINITY;
#pragma unroll
  for (int s = 0; s < kMaxSplits; ++s) mm = fmaxf(mm, ms[s]);
  float ll = 0.0f, oo = 0.0f;
#pragma unroll
  for (int s = 0; s < kMaxSplits; ++s) {
    const float f = ms[s] == -INFINITY ? 0.0f : ex2(ms[s] - mm);
    ll = fmaf(ls[s], f, ll);
    oo = fmaf(os[s], f, oo);
  }
  const float v = ll > 0.0f ? oo / ll : 0.0f;
  const float v1 = __shfl_down_sync(0xffffffffu, v, 1);  // blockDim = D, a multiple of 32
  if ((d & 1) == 0) *reinterpret_cast<uint32_t*>(out + (int64_t)bh * D + d) = Half<F16>::pack2(v, v1);
}

// Finish of the split-K QKV projection of a decode step: acc [B, (H + 2 Hkv) D]
// fp32 (q and k columns in the pair-interleaved order of the packed weights:
// columns 2i, 2i+1 of a head are the RoPE pair (u_i, u_{i+D/2})).  q and k heads
// are rotated by pos * theta_i and RMS-normalised over the head ("Nanochat与
// nanoGPT对比" §1: QK-norm after RoPE); v heads are converted.  Every head goes
// to qkv [B, (H + 2 Hkv) D] 16-bit; k and v heads also to the layer's cache at
// position pos.  One warp per (row, head); lane l holds columns 4l .. 4l+3
// (D = 128) or 2l, 2l+1 (D = 64).
template <int DW, bool F16>
__global__ void __launch_bounds__(256) qkv_finish_kernel(const float* __restrict__ acc, uint16_t* __restrict__ qkv,
                                                         uint16_t* __restrict__ cache, const float* __restrict__ rope,
                                                         int rope_T, int pos, int B, int H, int Hkv, int T_max,
                                                         float eps, const int* __restrict__ pos_dev,
                                                         uint32_t* __restrict__ dev_status, DecodeVe ve) {
  constexpr int D = DW * 32;
  bool store_cache = true;
  if (pos_dev) {  // a replayed graph step: refuse a position past the cache
    const int p = *pos_dev;
    store_cache = p >= 0 && p < T_max;
    if (!store_cache && blockIdx.x == 0 && threadIdx.x == 0 && dev_status) atomicOr(dev_status, NC_DEV_POSITION);
    pos = min(max(p, 0), T_max - 1);
  }
  const int heads = H + 2 * Hkv;
  const int wid = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= B * heads) return;
  const int b = wid / heads, hd = wid - b * heads;
  const float* src = acc + ((int64_t)b * heads + hd) * D + lane * DW;
  float v[DW];
#pragma unroll
  for (int d = 0; d < DW; ++d) v[d] = src[d];
  if (hd < H + Hkv) {  // q or k head: RoPE on the adjacent pairs, then the head's RMSNorm
    const float* cs = rope + (int64_t)pos * (D / 2);
    const float* sn = rope + ((int64_t)rope_T + pos) * (D / 2);
    float ss = 0.0f;
#pragma unroll
    for (int p = 0; p < DW / 2; ++p) {
      const int i = lane * (DW / 2) + p;  // pair index
      const float c = cs[i], sv = sn[i];
      const float a = v[2 * p], bb = v[2 * p + 1];
      v[2 * p] = a * c - bb * sv;
      v[2 * p + 1] = a * sv + bb * c;
      ss = fmaf(v[2 * p], v[2 * p], ss);
      ss = fmaf(v[2 * p + 1], v[2 * p + 1], ss);
    }
    const float r = rsqrtf(warp_allsum(ss) * (1.0f / D) + eps);
#pragma unroll
    for (int d = 0; d < DW; ++d) v[d] *= r;
  } else if (ve.table) {  // v head with a value embedding: v + gate[g] * table[token], kv head g
    const int g = hd - H - Hkv;
    int tok = ve.tokens[b];
    if (tok < 0 || tok >= ve.V) tok = 0;  // flagged by the embedding kernel
    const float* e = ve.table + ((int64_t)tok * Hkv + g) * D + lane * DW;
    const float gt = ve.gate[g];
#pragma unroll
    for (int d = 0; d < DW; ++d) v[d] = fmaf(gt, e[d], v[d]);
  }
  uint32_t pk[DW / 2];
  float vmax = 0.0f;
#pragma unroll
  for (int p = 0; p < DW / 2; ++p) {
    pk[p] = Half<F16>::pack2(v[2 * p], v[2 * p + 1]);
    vmax = fmaxf(vmax, fmaxf(fabsf(v[2 * p]), fabsf(v[2 * p + 1])));
  }
  if (F16 && dev_status && vmax > 65504.0f) atomicOr(dev_status, NC_DEV_F16_RANGE);
  uint16_t* dst = qkv + ((int64_t)b * heads + hd) * D + lane * DW;
  uint16_t* cdst = (hd >= H && store_cache) ? cache + ((int64_t)b * T_max + pos) * 2 * Hkv * D + (int64_t)(hd - H) * D + lane * DW
                           : nullptr;
  if constexpr (DW == 4) {
    const uint2 w2 = make_uint2(pk[0], pk[1]);
    *reinterpret_cast<uint2*>(dst) = w2;
    if (cdst) *reinterpret_cast<uint2*>(cdst) = w2;
  } else {
    *reinterpret_cast<uint32_t*>(dst) = pk[0];
    if (cdst) *reinterpret_cast<uint32_t*>(cdst) = pk[0];
  }
}

// relu(acc)^2 -> 16-bit ("从文本到聊天模型" §5.7), for the split-K c_fc of a decode step.
template <bool F16>
__global__ void relu2_finish_kernel(const float4* __restrict__ acc, uint2* __restrict__ out, int64_t n4,
                                    uint32_t* __restrict__ dev_status) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n4) return;
  float4 a = acc[i];
  a.x = fmaxf(a.x, 0.f);
  a.y = fmaxf(a.y, 0.f);
  a.z = fmaxf(a.z, 0.f);
  a.w = fmaxf(a.w, 0.f);
  a.x *= a.x;
  a.y *= a.y;
  a.z *= a.z;
  a.w *= a.w;
  if (F16 && dev_status && fmaxf(fmaxf(a.x, a.y), fmaxf(a.z, a.w)) > 65504.0f) atomicOr(dev_status, NC_DEV_F16_RANGE);
  out[i] = make_uint2(Half<F16>::pack2(a.x, a.y), Half<F16>::pack2(a.z, a.w));
}

template <int DW, bool F16>
nc_status decode_dispatch(const uint16_t* q, int64_t ldq, const uint16_t* cache, float* partial, int B, int H,
                          int Hkv, int T_max, int lo, int hi, int splits, int chunk, float scale_log2,
                          cudaStream_t stream, const int* pos_dev, int W) {
  const dim3 grid(splits, Hkv, B);
  constexpr int D = DW * 32;
  // staging of the chunk's K/V rows, reused for the warps' merge
  const int G = H / Hkv;
  const size_t stage = (size_t)chunk * 2 * D * 2, merge = (size_t)kWarps * G * (2 + D) * 4;
  const size_t smem = stage > merge ? stage : merge;
  switch (H / Hkv) {
    case 1:
      if (smem > 48 * 1024 &&
          cudaFuncSetAttribute(decode_attn_kernel<DW, 1, F16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)smem) != cudaSuccess)
        return NC_ERR_CUDA;
      decode_attn_kernel<DW, 1, F16><<<grid, kWarps * 32, smem, stream>>>(q, ldq, cache, partial, H, Hkv, T_max, lo,
                                                                       hi, chunk, scale_log2, pos_dev, W);
      break;
    case 2:
      if (smem > 48 * 1024 &&
          cudaFuncSetAttribute(decode_attn_kernel<DW, 2, F16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)smem) != cudaSuccess)
        return NC_ERR_CUDA;
      decode_attn_kernel<DW, 2, F16><<<grid, kWarps * 32, smem, stream>>>(q, ldq, cache, partial, H, Hkv, T_max, lo,
                                                                       hi, chunk, scale_log2, pos_dev, W);
      break;
    case 4:
      if (smem > 48 * 1024 &&
          cudaFuncSetAttribute(decode_attn_kernel<DW, 4, F16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)smem) != cudaSuccess)
        return NC_ERR_CUDA;
      decode_attn_kernel<DW, 4, F16><<<grid, kWarps * 32, smem, stream>>>(q, ldq, cache, partial, H, Hkv, T_max, lo,
                                                                       hi, chunk, scale_log2, pos_dev, W);
      break;
    case 8:
      if (smem > 48 * 1024 &&
          cudaFuncSetAttribute(decode_attn_kernel<DW, 8, F16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)smem) != cudaSuccess)
        return NC_ERR_CUDA;
      decode_attn_kernel<DW, 8, F16><<<grid, kWarps * 32, smem, stream>>>(q, ldq, cache, partial, H, Hkv, T_max, lo,
                                                                       hi, chunk, scale_log2, pos_dev, W);
      break;
    default:
      return NC_ERR_SHAPE;
  }
  return cudaGetLastError() == cudaSuccess ? NC_OK : NC_ERR_CUDA;
}


// ---------------------------------------------------------------- skinny GEMM
// The projections of a decode step: out (+)= A W^T with A [M <= 32, K] (the
// step's rows) and W [N, K] streamed once.  Each CTA (4 warps) owns 64 output
// features and one slice of K; each warp multiplies all 32 rows by its 16
// features with mma.sync m16n8k16 (fp32 accumulation), over 128-wide K chunks
// that cp.async double-buffers in shared memory (rows >= M and columns >= K
// zero-filled).  Slices of K are summed by fp32 atomic adds into `out` (which
// holds the residual stream, or zeros), so their order is not fixed; with a
// single slice the CTA stores (optionally soft-capped) values instead.
constexpr int SK_M = 32, SK_N = 64, SK_KC = 128, SK_LD = SK_KC + 8, SK_THREADS = 128;
constexpr int SK_BUF = (SK_M + SK_N) * SK_LD;  // 16-bit elements per buffer

template <bool F16, int MODE>  // MODE 0: atomic add, 1: store, 2: soft-capped store
__global__ void __launch_bounds__(SK_THREADS) skinny_gemm_kernel(const uint16_t* __restrict__ A, int64_t lda,
                                                                 const uint16_t* __restrict__ W, int64_t ldw,
                                                                 float* __restrict__ out, int64_t ldo, int M, int N,
                                                                 int K, int kslice, float cap) {
  using namespace wmma16;
  extern __shared__ __align__(16) uint16_t sk_smem[];
  const int n0 = blockIdx.x * SK_N;
  const int k_begin = blockIdx.y * kslice, k_end = min(K, k_begin + kslice);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nchunks = (k_end - k_begin + SK_KC - 1) / SK_KC;
  auto issue = [&](int c) {
    uint16_t* sa = sk_smem + (c & 1) * SK_BUF;
    uint16_t* sw = sa + SK_M * SK_LD;
    const int k0 = k_begin + c * SK_KC;
    for (int i = threadIdx.x; i < (SK_M + SK_N) * (SK_KC / 8); i += SK_THREADS) {
      const int r = i / (SK_KC / 8), ch = i % (SK_KC / 8);
      const int k = k0 + ch * 8;
      if (r < SK_M) {
        const bool v = r < M && k < k_end;
        cp_async16(sa + r * SK_LD + ch * 8, A + (int64_t)(v ? r : 0) * lda + (v ? k : 0), v);
      } else {
        const int n = n0 + r - SK_M;
        const bool v = n < N && k < k_end;
        cp_async16(sw + (r - SK_M) * SK_LD + ch * 8, W + (int64_t)(v ? n : 0) * ldw + (v ? k : 0), v);
      }
    }
    cp_async_commit();
  };
  float acc[2][2][4];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[mt][nt][e] = 0.0f;
  if (nchunks > 0) issue(0);
  for (int c = 0; c < nchunks; ++c) {
    if (c + 1 < nchunks) {
      issue(c + 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const uint32_t sa = smem_u32(sk_smem + (c & 1) * SK_BUF), sw = sa + SK_M * SK_LD * 2;
#pragma unroll
    for (int kk = 0; kk < SK_KC / 16; ++kk) {
      uint32_t a0[4], a1[4], b[4];
      load_a<SK_LD>(a0, sa, 0, kk * 16, lane);
      load_a<SK_LD>(a1, sa, 16, kk * 16, lane);
      load_b_nk<SK_LD>(b, sw, warp * 16, kk * 16, lane);
      mma16816<F16>(acc[0][0], a0, b[0], b[1]);
      mma16816<F16>(acc[0][1], a0, b[2], b[3]);
      mma16816<F16>(acc[1][0], a1, b[0], b[1]);
      mma16816<F16>(acc[1][1], a1, b[2], b[3]);
    }
    __syncthreads();  // buffer c & 1 is refilled by the issue of chunk c + 2
  }
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        const int r = mt * 16 + g + 8 * hr;
        const int col = n0 + warp * 16 + nt * 8 + 2 * t;
        if (r >= M || col >= N) continue;
        float* p = out + (int64_t)r * ldo + col;
        const float v0 = acc[mt][nt][2 * hr], v1 = acc[mt][nt][2 * hr + 1];
        if constexpr (MODE == 0) {
          atomicAdd(p, v0);
          if (col + 1 < N) atomicAdd(p + 1, v1);
        } else {
          const float o0 = MODE == 2 ? cap * tanhf(v0 / cap) : v0;
          const float o1 = MODE == 2 ? cap * tanhf(v1 / cap) : v1;
          p[0] = o0;
          if (col + 1 < N) p[1] = o1;
        }
      }
}

}  // namespace

int decode_attention_max_splits() { return kMaxSplits; }

nc_status qkv_finish_launch(const float* acc, uint16_t* qkv, uint16_t* cache, const float* rope, int rope_T,
                            int pos, int B, int H, int Hkv, int D, int T_max, float eps, bool f16,
                            cudaStream_t stream, const int* pos_dev, uint32_t* dev_status, DecodeVe ve) {
  const int warps = B * (H + 2 * Hkv);
  if (warps == 0) return NC_OK;
  const unsigned grid = (unsigned)((warps + 7) / 8);
  if (D == 128)
    f16 ? qkv_finish_kernel<4, true><<<grid, 256, 0, stream>>>(acc, qkv, cache, rope, rope_T, pos, B, H, Hkv, T_max, eps,
                                                               pos_dev, dev_status, ve)
        : qkv_finish_kernel<4, false><<<grid, 256, 0, stream>>>(acc, qkv, cache, rope, rope_T, pos, B, H, Hkv, T_max,
                                                                eps, pos_dev, dev_status, ve);
  else if (D == 64)
    f16 ? qkv_finish_kernel<2, true><<<grid, 256, 0, stream>>>(acc, qkv, cache, rope, rope_T, pos, B, H, Hkv, T_max, eps,
                                                               pos_dev, dev_status, ve)
        : qkv_finish_kernel<2, false><<<grid, 256, 0, stream>>>(acc, qkv, cache, rope, rope_T, pos, B, H, Hkv, T_max,
                                                                eps, pos_dev, dev_status, ve);
  else
    return NC_ERR_SHAPE;
  return cudaGetLastError() == cudaSuccess ? NC_OK : NC_ERR_CUDA;
}

// *pos += 1: the end of a decode step whose position lives in device memory.
__global__ void pos_advance_kernel(int* pos) {
  if (threadIdx.x == 0) *pos += 1;
}

nc_status pos_advance_launch(int* pos, cudaStream_t stream) {
  pos_advance_kernel<<<1, 32, 0, stream>>>(pos);
  return cudaGetLastError() == cudaSuccess ? NC_OK : NC_ERR_CUDA;
}

// The embedding of a decode step's tokens with the further terms of the full
// nanochat forward ("Nanochat与nanoGPT对比" §1): smear (gate != NULL) mixes in
// the embedding of the token at the row's previous position, read from the
// per-position token record hist [B][T_max], where this step also writes its
// own token; x0 (!= NULL) keeps a copy of the result for the residual lambdas.
// One warp per row; the gate's weight enters as bf16, as in the whole forward.
__global__ void __launch_bounds__(256) decode_embedding_kernel(const int32_t* __restrict__ tokens,
                                                               int32_t* __restrict__ hist,
                                                               const float* __restrict__ wte,
                                                               const float* __restrict__ gate, float* __restrict__ x,
                                                               float* __restrict__ x0, int B, int C, int V, int T_max,
                                                               int pos, const int* __restrict__ pos_dev,
                                                               uint32_t* __restrict__ dev_status) {
  const int b = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (b >= B) return;
  bool in_cache = true;
  if (pos_dev) {  // flagged (NC_DEV_POSITION) by the QKV finish of the same step
    const int p = *pos_dev;
    in_cache = p >= 0 && p < T_max;
    pos = min(max(p, 0), T_max - 1);
  }
  int tok = tokens[b];
  if (tok < 0 || tok >= V) {
    if (lane == 0 && dev_status) atomicOr(dev_status, NC_DEV_TOKEN_RANGE);
    tok = 0;
  }
  const float4* e = reinterpret_cast<const float4*>(wte + (int64_t)tok * C);
  float4* dst = reinterpret_cast<float4*>(x + (int64_t)b * C);
  float4* dst0 = x0 ? reinterpret_cast<float4*>(x0 + (int64_t)b * C) : nullptr;
  const int n4 = C / 4;
  const bool has_prev = gate && pos > 0;
  float sg = 0.0f;
  const float4* ep = e;
  if (gate) {
    if (lane == 0 && in_cache) hist[(int64_t)b * T_max + pos] = tok;
    int ptok = has_prev ? hist[(int64_t)b * T_max + pos - 1] : 0;
    if (ptok < 0 || ptok >= V) ptok = 0;
    ep = reinterpret_cast<const float4*>(wte + (int64_t)ptok * C);
    const float4* g4 = reinterpret_cast<const float4*>(gate);
    float dot = 0.0f;
    for (int i = lane; i < n4; i += 32) {
      const float4 a = e[i], g = g4[i];
      dot = fmaf(a.x, __bfloat162float(__float2bfloat16_rn(g.x)), dot);
      dot = fmaf(a.y, __bfloat162float(__float2bfloat16_rn(g.y)), dot);
      dot = fmaf(a.z, __bfloat162float(__float2bfloat16_rn(g.z)), dot);
      dot = fmaf(a.w, __bfloat162float(__float2bfloat16_rn(g.w)), dot);
    }
    dot = warp_allsum(dot);
    sg = has_prev ? 1.0f / (1.0f + expf(-dot)) : 0.0f;
  }
  for (int i = lane; i < n4; i += 32) {
    float4 a = e[i];
    if (has_prev) {
      const float4 p = ep[i];
      a.x = fmaf(sg, p.x, a.x);
      a.y = fmaf(sg, p.y, a.y);
      a.z = fmaf(sg, p.z, a.z);
      a.w = fmaf(sg, p.w, a.w);
    }
    dst[i] = a;
    if (dst0) dst0[i] = a;
  }
}

nc_status decode_embedding_launch(const int32_t* tokens, int32_t* hist, const float* wte, const float* smear_gate,
                                  float* x, float* x0, int B, int C, int V, int T_max, int pos, const int* pos_dev,
                                  uint32_t* dev_status, cudaStream_t stream) {
  if (B == 0) return NC_OK;
  if (C % 4 || (smear_gate && !hist)) return NC_ERR_SHAPE;
  const unsigned grid = (unsigned)((B + 7) / 8);
  decode_embedding_kernel<<<grid, 256, 0, stream>>>(tokens, hist, wte, smear_gate, x, x0, B, C, V, T_max, pos,
                                                    pos_dev, dev_status);
  return cudaGetLastError() == cudaSuccess ? NC_OK : NC_ERR_CUDA;
}

nc_status skinny_gemm_launch(const uint16_t* a, int64_t lda, const uint16_t* w, int64_t ldw, float* out,
                             int64_t ldo, int M, int N, int K, int mode, float cap, bool f16, cudaStream_t stream) {
  if (M < 1 || M > SK_M || N < 1 || K < 8 || K % 8 || lda % 8 || ldw % 8) return NC_ERR_SHAPE;
  const int ntiles = (N + SK_N - 1) / SK_N;
  const int max_slices = (K + SK_KC - 1) / SK_KC;
  int slices = 1;
  if (mode == 0) {  // about four CTAs per SM
    slices = (4 * device_sm_count() + ntiles - 1) / ntiles;
    slices = slices < 1 ? 1 : (slices > max_slices ? max_slices : slices);
  }
  const int kslice = ((K + slices - 1) / slices + SK_KC - 1) / SK_KC * SK_KC;
  slices = (K + kslice - 1) / kslice;
  const dim3 grid(ntiles, slices);
  const int smem = 2 * SK_BUF * 2;
  static bool attr_done[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_done[dev]) {
    if (cudaFuncSetAttribute(skinny_gemm_kernel<true, 0>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) ||
        cudaFuncSetAttribute(skinny_gemm_kernel<true, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) ||
        cudaFuncSetAttribute(skinny_gemm_kernel<false, 0>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) ||
        cudaFuncSetAttribute(skinny_gemm_kernel<false, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem))
      return NC_ERR_CUDA;
    attr_done[dev] = true;
  }
  if (mode == 0) {
    if (f16)
      skinny_gemm_kernel<true, 0><<<grid, SK_THREADS, smem, stream>>>(a, lda, w, ldw, out, ldo, M, N, K, kslice, cap);
    else
      skinny_gemm_kernel<false, 0><<<grid, SK_THREADS, smem, stream>>>(a, lda, w, ldw, out, ldo, M, N, K, kslice, cap);
  } else if (mode == 2) {
    if (f16)
      skinny_gemm_kernel<true, 2><<<grid, SK_THREADS, smem, stream>>>(a, lda, w, ldw, out, ldo, M, N, K, kslice, cap);
    else
      skinny_gemm_kernel<false, 2><<<grid, SK_THREADS, smem, stream>>>(a, lda, w, ldw, out, ldo, M, N, K, kslice, cap);
  } else {
    return NC_ERR_INVALID_ARG;
  }
  return cudaGetLastError() == cudaSuccess ? NC_OK : NC_ERR_CUDA;
}

nc_status relu2_finish_launch(const float* acc, uint16_t* out, int64_t n, bool f16, cudaStream_t stream,
                              uint32_t* dev_status) {
  if (n == 0) return NC_OK;
  if (n % 4) return NC_ERR_SHAPE;
  const int64_t n4 = n / 4;
  const unsigned grid = (unsigned)((n4 + 255) / 256);
  if (f16)
    relu2_finish_kernel<true><<<grid, 256, 0, stream>>>(reinterpret_cast<const float4*>(acc),
                                                        reinterpret_cast<uint2*>(out), n4, dev_status);
  else
    relu2_finish_kernel<false><<<grid, 256, 0, stream>>>(reinterpret_cast<const float4*>(acc),
                                                         reinterpret_cast<uint2*>(out), n4, dev_status);
  return cudaGetLastError() == cudaSuccess ? NC_OK : NC_ERR_CUDA;
}

nc_status kv_append_launch(const uint16_t* qkv, int64_t ldq, int col0, int width, uint16_t* cache, int M, int T,
                           int T_max, int pos0, cudaStream_t stream) {
  if (M == 0) return NC_OK;
  if (ldq % 8 || col0 % 8 || width % 8) return NC_ERR_SHAPE;
  const int64_t n = (int64_t)M * (width / 8);
  kv_append_kernel<<<(unsigned)((n + 255) / 256), 256, 0, stream>>>(
      reinterpret_cast<const uint4*>(qkv), ldq / 8, col0 / 8, width / 8, reinterpret_cast<uint4*>(cache), M, T,
      T_max, pos0);
  return cudaGetLastError() == cudaSuccess ? NC_OK : NC_ERR_CUDA;
}

nc_status decode_attention_launch(const uint16_t* q, int64_t ldq, const uint16_t* cache, float* partial,
                                  uint16_t* out, int B, int H, int Hkv, int D, int T_max, int pos, int W, bool f16,
                                  cudaStream_t stream, const int* pos_dev) {
  if (B == 0) return NC_OK;
  if ((D != 64 && D != 128) || H % Hkv != 0) return NC_ERR_SHAPE;
  const int Wc = W <= 0 || W > T_max ? T_max : W;
  int lo = pos - W + 1 > 0 ? pos - W + 1 : 0;
  int n_keys = pos - lo + 1;
  // chunks of 64 keys (32 KB of K/V staging at D = 128), more when the window
  // needs more than kMaxSplits of them
  int chunk = (n_keys + kMaxSplits - 1) / kMaxSplits;
  chunk = chunk < 64 ? 64 : (chunk + 15) / 16 * 16;
  int splits = (n_keys + chunk - 1) / chunk;
  if (pos_dev) {  // position known on the device only: the fixed grid of kMaxSplits chunks of 64
    if (T_max > kMaxSplits * 64) return NC_ERR_SHAPE;
    chunk = 64;
    splits = kMaxSplits;
    lo = 0;
    pos = 0;
  }
  if ((size_t)chunk * 2 * D * 2 > 200 * 1024) return NC_ERR_SHAPE;  // T_max beyond the staging
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)D);
  nc_status s;
  if (D == 128)
    s = f16 ? decode_dispatch<4, true>(q, ldq, cache, partial, B, H, Hkv, T_max, lo, pos, splits, chunk, scale_log2,
                                       stream, pos_dev, Wc)
            : decode_dispatch<4, false>(q, ldq, cache, partial, B, H, Hkv, T_max, lo, pos, splits, chunk,
                                        scale_log2, stream, pos_dev, Wc);
  else
    s = f16 ? decode_dispatch<2, true>(q, ldq, cache, partial, B, H, Hkv, T_max, lo, pos, splits, chunk, scale_log2,
                                       stream, pos_dev, Wc)
            : decode_dispatch<2, false>(q, ldq, cache, partial, B, H, Hkv, T_max, lo, pos, splits, chunk,
                                        scale_log2, stream, pos_dev, Wc);
  if (s != NC_OK) return s;
  if (f16)
    decode_combine_kernel<true><<<B * H, D, 0, stream>>>(partial, out, H, D, splits, pos_dev, T_max, Wc, chunk);
  else
    decode_combine_kernel<false><<<B * H, D, 0, stream>>>(partial, out, H, D, splits, pos_dev, T_max, Wc, chunk);
  return cudaGetLastError() == cudaSuccess ? NC_OK : NC_ERR_CUDA;
}

}  // namespace nc
