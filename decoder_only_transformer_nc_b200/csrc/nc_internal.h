// Declarations shared by the translation units of the library (not part of
// the public ABI, which is include/nc.h).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "nc.h"

namespace nc {

// Default bound of every in-kernel wait: two seconds of wall time.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// Epilogue selectors of the GEMM (the first five equal nc_epilogue).
enum : int {
  EPI_STORE_16 = NC_EPI_STORE_16,
  EPI_RELU2_16 = NC_EPI_RELU2_16,
  EPI_RESID_F32 = NC_EPI_RESID_F32,
  EPI_STORE_F32 = NC_EPI_STORE_F32,
  EPI_SOFTCAP_F32 = NC_EPI_SOFTCAP_F32,
  EPI_CE_PARTIAL = 5,   // soft-cap, per-tile sum of exp(l - cap), target logit
  EPI_QKV_ROPE = 6,     // q/k heads: RoPE + per-head RMSNorm; v heads: plain store
  EPI_QKV_ROPE_IL = 7,  // as EPI_QKV_ROPE with q/k head dims pair-interleaved (see nc_forward)
  EPI_CE_BWD_16 = 8,    // backward of soft-cap + cross-entropy from the recomputed logits:
                        //   out16 = (exp(l - lse_row) - [col == target]) (1 - (l / cap)^2)
  EPI_RELU2_BWD_16 = 9, // out16 = acc * 2 sqrt(h) with h = relu(u)^2 the saved 16-bit output
};

// Operand layouts of the GEMM.  NT: a [M, K], w [N, K] (both K contiguous);
// NN: a [M, K], w given as [K, N] (dgrad: dX = dY W with W stored [N_out, K_in]);
// TN: a given as [K, M], w given as [K, N] (wgrad: dW = dY^T X over the tokens).
enum : int { GEMM_NT = 0, GEMM_NN = 1, GEMM_TN = 2 };

struct EpiParams {
  void* out;                // 16-bit or fp32 output (or logits for EPI_CE_PARTIAL)
  int64_t ldo;              // output row stride in elements
  float cap;                // soft-cap
  int store_logits;         // EPI_CE_PARTIAL: also write capped logits to out
  float* ce_partial;        // EPI_CE_PARTIAL: [M, gemm_ce_partials_per_row(N)]
  float* ce_target;         // EPI_CE_PARTIAL: [M], l[m, y_m] (written by one tile)
  const int32_t* targets;   // EPI_CE_PARTIAL: [M]
  const float* rope;        // EPI_QKV_ROPE: [2][T][D/2] cos, sin
  int T;                    // EPI_QKV_ROPE: positions per sequence (row m is at pos0 + m % T)
  int pos0;                 // EPI_QKV_ROPE: position of the first row of each sequence
  int rope_T;               // EPI_QKV_ROPE: positions in the rope table (0: T)
  const float2* rope_pairs;  // EPI_QKV_ROPE_IL: the same angles as [D/2][rope_T] (cos, sin)
                            //   pairs, so a warp's 32 consecutive positions read one line
                            //   per pair; null: read `rope`
  int ksplit;               // EPI_RESID_F32: K is split into this many slices, each tile of a
                            //   slice adding its partial product into out (0 or 1: no split;
                            //   the fp32 sums then depend on the order the slices land)
  int H, Hkv, D;            // EPI_QKV_ROPE: head counts and head size
  float eps;                // EPI_QKV_ROPE: RMSNorm epsilon
  const int32_t* tokens;    // EPI_QKV_ROPE_IL with value embedding: [M] token ids
  const float* ve;          //   [V, Hkv*D] table of this layer (NULL: none)
  const float* ve_gate;     //   [Hkv] gates
  int V;                    //   vocabulary size (ids outside [0, V) read row 0)
  const float* amax_a;      // e4m3 operands: [1] amax of A, and
  const float* amax_b;      //   [1] amax of W ([3]: q, k, v parts for EPI_QKV_ROPE*); the
                            //   epilogue scales the product by 1 / (s_a s_w),
                            //   s = 448 / max(amax, 1e-12)
  float* amax_out;          // EPI_RELU2_16 with e4m3 operands: fold max |stored output| into
                            //   this slot (the quantisation of the output that follows)
  float alpha;              // fp32 epilogues: acc is multiplied by alpha first (0: by 1)
  const float* alpha_ptr;   //   or by *alpha_ptr (device), when given
  const float* row_lse;     // EPI_CE_BWD_16: [M] log-sum-exp of each row's capped logits (plus
                            //   ce_target[row] when ce_target is given: the forward's token
                            //   loss plus target logit)
  const uint16_t* aux;      // EPI_RELU2_BWD_16: h [M, ld_aux] (16-bit)
  int64_t ld_aux;
  float* rstd_out;          // EPI_QKV_ROPE_IL: [M, H + Hkv] the QK-norm factor of each q/k head
};

// ---- device / argument helpers (nc_api.cu)
int device_sm_count();
bool device_is_sm100();
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ---- GEMM (nc_gemm.cu)
// Number of soft-cap/CE partial sums the EPI_CE_PARTIAL epilogue writes per row.
int gemm_ce_partials_per_row(int N);
// a [M, K] (row stride lda) and w [N, K] (row stride ldw) are 16-bit in format
// `f16` (true: fp16, false: bf16); 16-bit outputs use the same format.
nc_status gemm_launch(const uint16_t* a, int64_t lda, const uint16_t* w, int64_t ldw, int M, int N,
                      int K, int epi, bool f16, const EpiParams& ep, uint32_t* dev_status,
                      cudaStream_t stream, uint64_t limit_ns = kWaitLimitNs);

// The same with e4m3 operands a [M, K] (row stride lda bytes) and w [N, K]
// (row stride ldw bytes), tcgen05 kind::f8f6f4; ep.amax_a / ep.amax_b give the
// tensorwise scales.  16-bit outputs are in format `f16`.  K % 16 == 0.
nc_status gemm_launch_e4m3(const uint8_t* a, int64_t lda, const uint8_t* w, int64_t ldw, int M, int N, int K,
                           int epi, bool f16, const EpiParams& ep, uint32_t* dev_status, cudaStream_t stream,
                           uint64_t limit_ns = kWaitLimitNs);

// 16-bit GEMM in one of the GEMM_* layouts (see above); lda / ldw are the row
// strides of a and w as given.  GEMM_NN and GEMM_TN take EPI_STORE_16,
// EPI_STORE_F32, EPI_RESID_F32 and EPI_RELU2_BWD_16.
nc_status gemm_launch_layout(const uint16_t* a, int64_t lda, const uint16_t* w, int64_t ldw, int M, int N, int K,
                             int epi, bool f16, int layout, const EpiParams& ep, uint32_t* dev_status,
                             cudaStream_t stream, uint64_t limit_ns = kWaitLimitNs);

nc_status selftest_wait_launch(uint32_t* dev_status, uint64_t limit_ns, cudaStream_t stream);

// ---- backward (nc_backward.cu); gradients of the summed token losses
// dx_acc (+)= RMSNorm backward of x with upstream dy; dx16 = dx_acc in 16-bit.
nc_status rmsnorm_bwd_launch(const float* x, const float* dy, float* dx_acc, uint16_t* dx16, int M, int C, float eps,
                             bool accumulate, bool f16, cudaStream_t stream);
// In place on the q and k columns of dqkv: QK-norm backward, then inverse RoPE
// (pair-interleaved columns), from the saved normalised qkv and QK-norm factors.
nc_status qk_bwd_launch(uint16_t* dqkv, const uint16_t* qkv, int64_t ld, const float* rstd, const float* rope,
                        int rope_T, int M, int T, int H, int Hkv, int D, bool f16, cudaStream_t stream);
// dq, dk, dv (into the q / k / v columns of dqkv) from qkv, o, dO [M, H*D], the
// forward's lse [M, H]; delta [M, H] is scratch.
// Attention backward (nc_attention_bwd.cu): delta is scratch of B*T*H floats
// (Delta_i per head, [B][H][T]); dq | dk | dv written in qkv's layout.
nc_status attn_bwd_launch(const uint16_t* qkv, int64_t ldqkv, const uint16_t* o, const uint16_t* dO,
                          const float* lse, float* delta, uint16_t* dqkv, int B, int T, int H, int Hkv, int D,
                          int window, bool f16, cudaStream_t stream, uint32_t* dev_status = nullptr,
                          uint64_t limit_ns = kWaitLimitNs);
// Backward of the further forward terms (nc_backward.cu).
nc_status dots_launch(const float* a, const float* b0, const float* b1, int64_t n, const float* inv, float sign,
                      float* out0, float* out1, cudaStream_t stream);
nc_status mix_bwd_launch(float* dx, float* acc0, const float* sub, const float* add, const float* lam_r,
                         const float* lam_0, const float* lam_sub, uint16_t* dx16, int64_t n, bool f16,
                         cudaStream_t stream);
nc_status ve_bwd_launch(const uint16_t* dqkv, int64_t ld, const int32_t* tokens, const float* table, const float* gate,
                        float* dtable, float* dgate, int M, int H, int Hkv, int D, int V, const float* inv, bool f16,
                        cudaStream_t stream);
nc_status smear_bwd_launch(const int32_t* tokens, const float* wte, const float* w, const float* dx, float* de,
                           float* dz, float* dw, int M, int T, int C, int V, const float* inv, cudaStream_t stream);
nc_status embedding_bwd_launch(const int32_t* tokens, const float* dx, float* dwte, int M, int C, int V,
                               const float* alpha, cudaStream_t stream);
nc_status qkv_grad_scatter_launch(const float* packed, float* gq, float* gk, float* gv, int H, int Hkv, int D, int C,
                                  float alpha, cudaStream_t stream);

// ---- dynamic tensorwise e4m3 quantisation (nc_fp8.cu)
enum { FP8_SRC_F32 = 0, FP8_SRC_BF16 = 1, FP8_SRC_F16 = 2 };
struct Fp8Seg {
  const void* src;         // source tensor (element type: the launch's src_kind)
  uint8_t* dst;            // e4m3 codes, n bytes
  int64_t n;               // elements, multiple of 16
  int slot;                // amax slot (index into the launch's amax array)
  bool pair_rows = false;  // destination rows in the QKV RoPE-pair order (perm_cols, perm_d)
};
// amax pass (when do_amax; slots must hold 0) then quantise pass over every
// segment.  Source pointers 16-byte aligned.
nc_status fp8_quantize_launch(const Fp8Seg* segs, int nseg, int src_kind, float* amax, bool do_amax,
                              cudaStream_t stream, int perm_cols = 0, int perm_d = 0);

// TMA tensor map with 128-byte swizzling: dims innermost first, strides in
// bytes for dims 1..rank-1.  Element type: fp16 if f16, else bf16; the _f32
// variant maps fp32 data.
bool encode_tensor_map(CUtensorMap* map, bool f16, int rank, const void* base, const uint64_t* dims,
                       const uint64_t* strides, const uint32_t* box);
bool encode_tensor_map_u8(CUtensorMap* map, int rank, const void* base, const uint64_t* dims,
                          const uint64_t* strides, const uint32_t* box);
bool encode_tensor_map_f32(CUtensorMap* map, int rank, const void* base, const uint64_t* dims,
                           const uint64_t* strides, const uint32_t* box);

// ---- attention (nc_attention.cu; with lse, nc_attention_lse.cu)
// When `lse` is given ([B, T, H] fp32 row log-sum-exp, for the backward) the
// launch goes to the kernel whose outputs are bit-reproducible run to run.
nc_status attention_launch(const uint16_t* q, const uint16_t* k, const uint16_t* v, uint16_t* out,
                           int B, int T, int H, int Hkv, int D, int window, int64_t q_stride,
                           int64_t kv_stride, bool f16, uint32_t* dev_status, cudaStream_t stream,
                           float* amax = nullptr, float* lse = nullptr);
nc_status attention_lse_launch(const uint16_t* q, const uint16_t* k, const uint16_t* v, uint16_t* out,
                               int B, int T, int H, int Hkv, int D, int window, int64_t q_stride,
                               int64_t kv_stride, bool f16, uint32_t* dev_status, cudaStream_t stream,
                               float* amax, float* lse);

// ---- elementwise / row kernels (nc_rowops.cu)
struct CastSeg {
  const float* src;
  uint16_t* dst;
  int64_t n;          // multiple of 8
  bool pair_rows = false;  // rows reordered within each block of perm_d rows (see below)
};
// fp32 -> bf16 (round to nearest even); with f16 the bf16 value is stored as fp16.
// Segments flagged pair_rows are [rows, perm_cols] matrices whose rows are
// reordered inside every block of perm_d rows so that the RoPE partners j and
// j + perm_d/2 become neighbours: destination row 2j <- source row j,
// destination row 2j+1 <- source row j + perm_d/2.
nc_status cast_launch(const CastSeg* segs, int nseg, bool f16, cudaStream_t stream, int perm_cols = 0,
                      int perm_d = 0);
nc_status embedding_launch(const int32_t* tokens, const float* wte, float* x, int M, int C, int V,
                           uint32_t* dev_status, cudaStream_t stream);
// Embedding with the smear term (gate may be NULL: plain lookup) and an optional
// copy of the result into x0.  T: positions per row (row m is at m % T).
nc_status embedding_extra_launch(const int32_t* tokens, const float* wte, const float* smear_gate,
                                 float* x, float* x0, int M, int C, int V, int T, uint32_t* dev_status,
                                 cudaStream_t stream);
// RMSNorm of u, where per row u = x, then (x_keep: x_keep = u), then (x0: u =
// lam_r[0] u + lam_0[0] x0), then (x_sub: u = u - lam_sub[0] x_sub); with
// write_back the row of x becomes u.  Scalars are read from device memory.
nc_status rmsnorm_mix_launch(float* x, const float* x0, const float* lam_r, const float* lam_0,
                             float* x_keep, const float* x_sub, const float* lam_sub, bool write_back,
                             uint16_t* out, int M, int C, float eps, bool f16, cudaStream_t stream);
// ---- KV-cache decode (nc_decode.cu)
// Copies the k|v columns [col0, col0 + width) of the M rows of qkv (row stride
// ldq) into a layer's cache [B][T_max][width]: row m goes to (m / T, pos0 + m % T).
nc_status kv_append_launch(const uint16_t* qkv, int64_t ldq, int col0, int width, uint16_t* cache, int M, int T,
                           int T_max, int pos0, cudaStream_t stream);
// Attention of one query position `pos` per row over the cached keys [lo, pos],
// lo = max(0, pos - W + 1): q [B, H*D] (row stride ldq), cache [B][T_max][2][Hkv][D]
// -> out [B, H*D] (16-bit).  `partial` holds splits x (2 + D) fp32 per (b, h).
nc_status decode_attention_launch(const uint16_t* q, int64_t ldq, const uint16_t* cache, float* partial,
                                  uint16_t* out, int B, int H, int Hkv, int D, int T_max, int pos, int W,
                                  bool f16, cudaStream_t stream,
                                  const int* pos_dev = nullptr);
// Decode projections (M <= 32 rows): mode 0 adds A W^T into out (fp32 atomic
// adds of K-slice partial sums; out holds the residual stream or zeros), mode 2
// stores cap * tanh(A W^T / cap) (one slice).
nc_status skinny_gemm_launch(const uint16_t* a, int64_t lda, const uint16_t* w, int64_t ldw, float* out,
                             int64_t ldo, int M, int N, int K, int mode, float cap, bool f16, cudaStream_t stream);
// With pos_dev, the kernels of a decode step read the position from device
// memory (clamped to the cache for their reads; the cache write refuses a
// position past it) and the attention runs on a fixed grid, so a
// captured graph of the step can be replayed; pos_advance_launch adds one to it.
nc_status pos_advance_launch(int* pos, cudaStream_t stream);
// Upper bound of the per-(b, h) splits decode_attention_launch uses.
int decode_attention_max_splits();
// From the fp32 split-K sum of a decode step's QKV projection: RoPE at `pos` and
// QK-norm of q and k heads (pair-interleaved columns), 16-bit qkv, and k|v heads
// into the layer's cache at `pos`.  A device position outside [0, T_max) writes
// no cache entry and sets NC_DEV_POSITION in dev_status.
// With ve.table set, each v head g also gets ve.gate[g] * ve.table[token][g]
// (the value embedding of the full nanochat forward; table [V][Hkv][D] fp32).
struct DecodeVe {
  const int32_t* tokens;
  const float* table;
  const float* gate;
  int V;
};
nc_status qkv_finish_launch(const float* acc, uint16_t* qkv, uint16_t* cache, const float* rope, int rope_T,
                            int pos, int B, int H, int Hkv, int D, int T_max, float eps, bool f16,
                            cudaStream_t stream, const int* pos_dev = nullptr, uint32_t* dev_status = nullptr,
                            DecodeVe ve = DecodeVe{});
// The token embedding of a decode step at `pos` (or *pos_dev) with smear
// (smear_gate != NULL: reads the previous position's token from hist [B][T_max]
// and records this step's token there) and an optional copy into x0 [B, C].
nc_status decode_embedding_launch(const int32_t* tokens, int32_t* hist, const float* wte, const float* smear_gate,
                                  float* x, float* x0, int B, int C, int V, int T_max, int pos, const int* pos_dev,
                                  uint32_t* dev_status, cudaStream_t stream);
// out = relu(acc)^2 as 16-bit (n elements, n % 4 == 0); an fp16 value past
// 65504 sets NC_DEV_F16_RANGE in dev_status.
nc_status relu2_finish_launch(const float* acc, uint16_t* out, int64_t n, bool f16, cudaStream_t stream,
                              uint32_t* dev_status = nullptr);

nc_status rmsnorm_launch(const float* x, uint16_t* out, int M, int C, float eps, bool f16,
                         cudaStream_t stream,
                         float* amax = nullptr);
// table [2][T][D/2] (cos, sin); pairs, when given, the same values as [D/2][T] float2.
nc_status rope_table_launch(float* table, int T, int D, float base, cudaStream_t stream, float2* pairs = nullptr);
// The pair-major copy kept right after a [2][T][D/2] table in the library's own buffers.
inline float2* rope_pairs_of(float* table, int T, int D) {
  return reinterpret_cast<float2*>(table + (size_t)T * D);
}
nc_status rope_qknorm_launch(uint16_t* q, uint16_t* k, const float* table, int B, int T, int H,
                             int Hkv, int D, int64_t q_stride, int64_t k_stride, float eps, bool f16,
                             cudaStream_t stream);
nc_status softcap_ce_launch(const float* z, const int32_t* targets, float* capped_out,
                            float* token_loss, int M, int V, float cap, uint32_t* dev_status,
                            cudaStream_t stream);
nc_status ce_finalize_launch(const float* partial, int n_tiles, const float* target_logit,
                             const int32_t* targets, float* token_loss, int M, int V, float cap,
                             uint32_t* dev_status, cudaStream_t stream);
// loss = mean token loss over targets in [0, V); inv_count (optional) = 1 / that count (0 if none).
nc_status loss_mean_launch(const float* token_loss, const int32_t* targets, int M, int V,
                           float* loss, cudaStream_t stream, float* inv_count = nullptr);

}  // namespace nc
