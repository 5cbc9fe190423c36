// Loss head that needs no caller-provided or runtime-allocated scratch.
//
// Some callers cannot hand this library a scratch buffer: code embedded in a
// host application whose memory manager owns the whole device budget, or code
// on a latency-critical path where cudaMalloc's implicit device-wide
// synchronisation is not acceptable.  For them, nc_lm_head_loss_static runs
// the lm_head projection with the soft-cap + cross-entropy epilogue exactly
// like the forward pass does, but keeps the per-tile partial sums and the
// target logits in the fixed device array below instead of in a workspace.
//
// The array is a file-scope __device__ variable: every GPU that loads this
// library holds it (kStaticBytes) until the process exits.  Host code must not
// pass the array's name to a kernel -- on the host that name is only a
// stand-in symbol, not a device address -- so the device address is looked
// up with cudaGetSymbolAddress once per device (with that device current) and
// cached.  The cached address belongs to the device's primary context: after
// cudaDeviceReset destroys that context the address is stale, so a process
// that resets a device must not call this entry point on it again.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "nc_internal.h"

namespace nc {
namespace {

constexpr int kMaxRows = 8192;  // M limit
constexpr int kMaxVocab = 32768;
constexpr int kMaxPartials = 256;  // partial sums per row at V = 32768
constexpr size_t kPartialFloats = (size_t)kMaxRows * kMaxPartials;
constexpr size_t kStaticBytes = (kPartialFloats + kMaxRows) * sizeof(float);  // 8.4 MB

// partials [kMaxRows][kMaxPartials] followed by target logits [kMaxRows].
static __device__ __align__(256) float g_loss_scratch[kPartialFloats + kMaxRows];
static_assert(sizeof(g_loss_scratch) == kStaticBytes, "scratch size");

std::mutex g_mu;
float* g_scratch_ptr[64] = {};

// Device address of g_loss_scratch on the current device (nullptr on failure).
float* scratch_address() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_loss_scratch) != cudaSuccess) return nullptr;
    g_scratch_ptr[dev] = static_cast<float*>(p);
  }
  return g_scratch_ptr[dev];
}

}  // namespace
}  // namespace nc

using namespace nc;

extern "C" nc_status nc_lm_head_loss_static(const uint16_t* a, const uint16_t* w_lm,
                                            const int32_t* targets, int M, int C, int V, float cap,
                                            nc_dtype dtype, float* token_loss, float* loss,
                                            uint32_t* dev_status, void* stream) {
  if (!a || !w_lm || !targets || !token_loss || M < 1 || C < 8 || V < 64 || !(cap > 0.0f) ||
      (dtype != NC_F16 && dtype != NC_BF16))
    return NC_ERR_INVALID_ARG;
  if (M > kMaxRows || V > kMaxVocab || gemm_ce_partials_per_row(V) > kMaxPartials || C % 8 != 0 ||
      V % 64 != 0)
    return NC_ERR_SHAPE;
  if (!aligned16(a) || !aligned16(w_lm)) return NC_ERR_ALIGNMENT;
  if (!device_is_sm100()) return NC_ERR_UNSUPPORTED_DEVICE;
  float* scratch = scratch_address();
  if (!scratch) return NC_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int n_tiles = gemm_ce_partials_per_row(V);
  // Every (row, partial) slot is rewritten by the GEMM and the target logit of
  // every row with a valid target is rewritten too (rows without one are never
  // read), so nothing has to be cleared between calls.
  float* partial = scratch;
  float* target_logit = scratch + (size_t)M * n_tiles;
  EpiParams ep{};
  ep.out = nullptr;
  ep.ldo = V;
  ep.cap = cap;
  ep.store_logits = 0;
  ep.ce_partial = partial;
  ep.ce_target = target_logit;
  ep.targets = targets;
  nc_status s = gemm_launch(a, C, w_lm, C, M, V, C, EPI_CE_PARTIAL, dtype == NC_F16, ep, dev_status, st);
  if (s != NC_OK) return s;
  s = ce_finalize_launch(partial, n_tiles, target_logit, targets, token_loss, M, V, cap, dev_status, st);
  if (s != NC_OK) return s;
  if (loss) s = loss_mean_launch(token_loss, targets, M, V, loss, st);
  return s;
}
