// Dynamic tensorwise e4m3 quantisation ("Nanochat与nanoGPT对比：关键升级" §1,
// architecture table, FP8-training row: dynamic, tensor-level FP8; e4m3 is the
// forward format).  For every tensor x of a batch:
//
//   amax = max |x|,  s = 448 / max(amax, 1e-12)  (fp32),  q = e4m3(fp32(x * s))
//
// with round-to-nearest-even, saturating conversion.  A launch covers a batch
// of tensors ("segments"), each with its own amax slot.  Blocks are dealt to
// segments in proportion to their size, CHUNK elements per block, so a block
// reads one contiguous piece of one tensor.  Two launches:
//   amax pass      each block reduces its piece to one value and folds it into
//                  the segment's slot with one atomicMax on the bit pattern of
//                  |x| (non-negative floats order like their bits; a NaN
//                  pattern orders above every number and so propagates);
//   quantise pass  each block reads its slot (final: the previous launch has
//                  ended), forms s and converts 16 elements per thread and step.
// The q and k weight segments may be written with the RoPE-pair row order of
// the QKV projection (destination row 2j / 2j+1 of each head block takes source
// row j / j + D/2), as the 16-bit weight cast does.  Slots must hold 0 before
// the amax pass.
#include <cuda_runtime.h>

#include <cstdint>

#include "nc_half.cuh"
#include "nc_internal.h"

namespace nc {
namespace fp8 {

constexpr int kThreads = 256;
constexpr int kVec = 16;   // elements per thread and step (16 codes = one 16-byte store)
constexpr int kSteps = 8;  // steps per block
constexpr int64_t kChunk = (int64_t)kThreads * kVec * kSteps;  // 32768 elements per block
constexpr int kMaxSegs = 112;

struct SegBatch {
  const void* src[kMaxSegs];
  uint8_t* dst[kMaxSegs];
  int64_t n[kMaxSegs];
  int32_t bstart[kMaxSegs + 1];  // first block of each segment
  int16_t slot[kMaxSegs];
  uint8_t pair_rows[kMaxSegs];
  float* amax;  // slot array
  int nseg;
  int perm_cols, perm_d;
};

// 16 consecutive source elements as fp32.
template <int SRC>
__device__ __forceinline__ void load16(const void* base, int64_t e, float (&v)[16]) {
  if constexpr (SRC == FP8_SRC_F32) {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(base) + e);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float4 f = p[j];
      v[4 * j] = f.x;
      v[4 * j + 1] = f.y;
      v[4 * j + 2] = f.z;
      v[4 * j + 3] = f.w;
    }
  } else {
    const uint4* p = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(base) + e);
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const uint4 u = p[j];
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = Half<SRC == FP8_SRC_F16>::unpack2(w[i]);
        v[8 * j + 2 * i] = f.x;
        v[8 * j + 2 * i + 1] = f.y;
      }
    }
  }
}

// Segment of this block: the last one whose first block is <= blockIdx.x.
__device__ __forceinline__ int block_segment(const SegBatch& sb) {
  int lo = 0, hi = sb.nseg - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (sb.bstart[mid] <= (int)blockIdx.x) lo = mid; else hi = mid - 1;
  }
  return lo;
}

template <int SRC>
__global__ void __launch_bounds__(kThreads) amax_kernel(const __grid_constant__ SegBatch sb) {
  const int seg = block_segment(sb);
  const int64_t n = sb.n[seg];
  const int64_t base = (int64_t)(blockIdx.x - sb.bstart[seg]) * kChunk;
  uint32_t m = 0;  // max of |x| as a bit pattern
#pragma unroll 2
  for (int s = 0; s < kSteps; ++s) {
    const int64_t e = base + ((int64_t)s * kThreads + threadIdx.x) * kVec;
    if (e < n) {
      float v[16];
      load16<SRC>(sb.src[seg], e, v);
#pragma unroll
      for (int i = 0; i < 16; ++i) m = max(m, __float_as_uint(v[i]) & 0x7FFFFFFFu);
    }
  }
  m = __reduce_max_sync(0xFFFFFFFFu, m);
  __shared__ uint32_t wm[kThreads / 32];
  if ((threadIdx.x & 31) == 0) wm[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
#pragma unroll
    for (int w = 1; w < kThreads / 32; ++w) m = max(m, wm[w]);
    atomicMax(reinterpret_cast<unsigned int*>(sb.amax + sb.slot[seg]), m);
  }
}

template <int SRC>
__global__ void __launch_bounds__(kThreads) quantize_kernel(const __grid_constant__ SegBatch sb) {
  const int seg = block_segment(sb);
  const int64_t n = sb.n[seg];
  const int64_t base = (int64_t)(blockIdx.x - sb.bstart[seg]) * kChunk;
  const float s = e4m3_scale(sb.amax[sb.slot[seg]]);
  const bool perm = sb.pair_rows[seg] != 0;
#pragma unroll 2
  for (int st = 0; st < kSteps; ++st) {
    const int64_t e = base + ((int64_t)st * kThreads + threadIdx.x) * kVec;  // destination offset
    if (e >= n) break;
    int64_t se = e;
    if (perm) {  // 16 elements of one row (perm_cols % 16 == 0)
      const int64_t row = e / sb.perm_cols, col = e - row * sb.perm_cols;
      const int64_t blk = row / sb.perm_d, jj = row - blk * sb.perm_d;
      se = (blk * sb.perm_d + (jj >> 1) + (jj & 1) * (sb.perm_d / 2)) * sb.perm_cols + col;
    }
    float v[16];
    load16<SRC>(sb.src[seg], se, v);
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      w[i] = (uint32_t)e4m3x2(v[4 * i] * s, v[4 * i + 1] * s) |
             ((uint32_t)e4m3x2(v[4 * i + 2] * s, v[4 * i + 3] * s) << 16);
    *reinterpret_cast<uint4*>(sb.dst[seg] + e) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

}  // namespace fp8

nc_status fp8_quantize_launch(const Fp8Seg* segs, int nseg, int src_kind, float* amax, bool do_amax,
                              cudaStream_t stream, int perm_cols, int perm_d) {
  using namespace fp8;
  if (nseg < 0 || (nseg > 0 && !amax) || src_kind < FP8_SRC_F32 || src_kind > FP8_SRC_F16)
    return NC_ERR_INVALID_ARG;
  for (int base = 0; base < nseg; base += kMaxSegs) {
    SegBatch sb;
    sb.nseg = nseg - base < kMaxSegs ? nseg - base : kMaxSegs;
    sb.amax = amax;
    sb.perm_cols = perm_cols;
    sb.perm_d = perm_d;
    sb.bstart[0] = 0;
    int64_t blocks = 0;
    for (int i = 0; i < sb.nseg; ++i) {
      const Fp8Seg& g = segs[base + i];
      if (g.n < 0 || g.n % kVec || g.slot < 0 || g.slot > 32767) return NC_ERR_INVALID_ARG;
      if (g.pair_rows && (perm_cols <= 0 || perm_cols % kVec || perm_d < 2 || perm_d % 2 ||
                          g.n % ((int64_t)perm_cols * perm_d)))
        return NC_ERR_INVALID_ARG;
      sb.src[i] = g.src;
      sb.dst[i] = g.dst;
      sb.n[i] = g.n;
      sb.slot[i] = (int16_t)g.slot;
      sb.pair_rows[i] = g.pair_rows ? 1 : 0;
      blocks += (g.n + kChunk - 1) / kChunk;
      if (blocks > 0x7FFFFFFF) return NC_ERR_SHAPE;
      sb.bstart[i + 1] = (int32_t)blocks;
    }
    // empty segments own no block; the search above then never selects them
    if (blocks == 0) continue;
    const int grid = (int)blocks;
    if (do_amax) {
      switch (src_kind) {
        case FP8_SRC_F32: amax_kernel<FP8_SRC_F32><<<grid, kThreads, 0, stream>>>(sb); break;
        case FP8_SRC_BF16: amax_kernel<FP8_SRC_BF16><<<grid, kThreads, 0, stream>>>(sb); break;
        default: amax_kernel<FP8_SRC_F16><<<grid, kThreads, 0, stream>>>(sb); break;
      }
      if (cudaGetLastError() != cudaSuccess) return NC_ERR_CUDA;
    }
    switch (src_kind) {
      case FP8_SRC_F32: quantize_kernel<FP8_SRC_F32><<<grid, kThreads, 0, stream>>>(sb); break;
      case FP8_SRC_BF16: quantize_kernel<FP8_SRC_BF16><<<grid, kThreads, 0, stream>>>(sb); break;
      default: quantize_kernel<FP8_SRC_F16><<<grid, kThreads, 0, stream>>>(sb); break;
    }
    if (cudaGetLastError() != cudaSuccess) return NC_ERR_CUDA;
  }
  return NC_OK;
}

}  // namespace nc
