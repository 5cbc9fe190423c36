// Public C ABI (include/nc.h): argument checks, workspace layout and the
// launch sequence of the forward pass.
//
// Forward ("从文本到聊天模型" §5; block internals from "Nanochat与nanoGPT对比：
// 关键升级" §1), all on the caller's stream:
//   RoPE table; fp32 -> bf16 weight cast (Wq|Wk|Wv packed as one [(H+2Hkv)D, C]
//   matrix per layer, the rows of every q and k head reordered so that the
//   RoPE partners u_j and u_{j+D/2} are neighbours; q and k therefore leave the
//   QKV GEMM with the same pair-interleaved head layout, which leaves q.k and
//   hence attention unchanged); embedding gather;
//   per layer: RMSNorm -> QKV GEMM -> RoPE+QK-norm -> attention (layer window)
//              -> c_proj GEMM with residual add -> RMSNorm -> c_fc GEMM with
//              ReLU^2 -> c_proj GEMM with residual add;
//   final RMSNorm -> lm_head GEMM whose epilogue applies the soft-cap and
//   reduces each 256-column tile to sum(exp(l - cap)) (+ the target logit)
//   -> per-row combine to NLL -> fixed-order mean.
// The residual stream stays fp32; matmul operands are bf16 with fp32
// accumulation.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "nc_internal.h"

namespace nc {

namespace {
struct DevInfo {
  int sms = 0;
  bool sm100 = false;
  bool init = false;
};
DevInfo g_dev[64];
std::mutex g_dev_mu;

const DevInfo* dev_info() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DevInfo& d = g_dev[dev];
  if (!d.init) {
    cudaDeviceProp p;
    if (cudaGetDeviceProperties(&p, dev) != cudaSuccess) return nullptr;
    d.sms = p.multiProcessorCount;
    d.sm100 = (p.major == 10 && p.minor == 0);
    d.init = true;
  }
  return &d;
}
}  // namespace

int device_sm_count() {
  const DevInfo* d = dev_info();
  return d ? d->sms : 148;
}
bool device_is_sm100() {
  const DevInfo* d = dev_info();
  return d && d->sm100;
}

}  // namespace nc

using namespace nc;

namespace {

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool config_ok(const nc_config* c) {
  if (!c) return false;
  if (c->n_layer < 1 || c->d_model < 64 || c->n_head < 1 || c->n_kv_head < 1) return false;
  if (c->n_head % c->n_kv_head != 0) return false;
  if (c->head_dim != 64 && c->head_dim != 128) return false;
  if (c->vocab < 64 || c->vocab % 64 != 0) return false;
  if (c->seq_len < 1 || c->short_window < 1) return false;
  if (c->d_model % 64 != 0) return false;
  if ((int64_t)c->n_head * c->head_dim % 64 != 0) return false;
  if (!(c->softcap > 0.0f) || !(c->norm_eps >= 0.0f) || !(c->rope_base > 1.0f)) return false;
  if (c->act_dtype != NC_F16 && c->act_dtype != NC_BF16) return false;
  if ((c->extras & ~NC_EXTRA_ALL) != 0) return false;
  if ((c->fp8 & ~NC_FP8_ALL) != 0) return false;
  const size_t plen = strnlen(c->window_pattern, sizeof(c->window_pattern));
  if (plen == 0 || plen >= sizeof(c->window_pattern)) return false;
  for (size_t i = 0; i < plen; ++i)
    if (c->window_pattern[i] != 'S' && c->window_pattern[i] != 'L') return false;
  return true;
}

// Workspace layout of nc_forward.  Offsets are 256-byte aligned.
struct WsLayout {
  size_t status, rope, wqkv, wo, wfc, wmp, wlm, x, a, qkv, o, h, part, tgt, tl, x0, xmid, a8, amax, total;
  size_t wqkv_elems, wo_elems, wfc_elems, wmp_elems;  // per layer
};

// FP8 amax slots of a forward: per layer the weights c_q, c_k, c_v (adjacent:
// the QKV product reads three), attention c_proj, c_fc, MLP c_proj, then the
// LM head; after them per layer the activations entering the QKV, attention
// c_proj, c_fc and MLP c_proj products, then the one entering the LM head.
inline int amax_w_slot(int l, int which) { return 6 * l + which; }
inline int amax_wlm_slot(int L) { return 6 * L; }
inline int amax_a_slot(int L, int l, int which) { return 6 * L + 1 + 4 * l + which; }
inline int amax_alm_slot(int L) { return 10 * L + 1; }
inline int amax_slots(int L) { return 10 * L + 2; }

WsLayout ws_layout(const nc_config* c, int B, int T, bool own_weights = true) {
  WsLayout L;
  const size_t M = (size_t)B * T;
  const size_t C = c->d_model, D = c->head_dim, H = c->n_head, Hkv = c->n_kv_head, V = c->vocab;
  const size_t nqkv = (H + 2 * Hkv) * D;
  L.wqkv_elems = nqkv * C;
  L.wo_elems = C * H * D;
  L.wfc_elems = 4 * C * C;
  L.wmp_elems = C * 4 * C;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  L.status = take(256);
  const size_t wb = (c->fp8 & NC_FP8_BLOCK) ? 1 : 2;    // bytes per block weight element
  const size_t lb = (c->fp8 & NC_FP8_LM_HEAD) ? 1 : 2;  // ... per LM-head element
  if (own_weights) {  // else the 16-bit weights and the RoPE table live in a session
    L.rope = take((size_t)T * D * sizeof(float) * 2);  // [2][T][D/2] and the pair-major copy
    L.wqkv = take(c->n_layer * L.wqkv_elems * wb);
    L.wo = take(c->n_layer * L.wo_elems * wb);
    L.wfc = take(c->n_layer * L.wfc_elems * wb);
    L.wmp = take(c->n_layer * L.wmp_elems * wb);
    L.wlm = take(V * C * lb);
  } else {
    L.rope = L.wqkv = L.wo = L.wfc = L.wmp = L.wlm = 0;
  }
  L.x = take(M * C * 4);
  L.a = take(M * C * 2);
  L.qkv = take(M * nqkv * 2);
  L.o = take(M * H * D * 2);
  L.h = take(M * 4 * C * 2);
  L.part = take(M * (size_t)gemm_ce_partials_per_row((int)V) * 4);
  L.tgt = take(M * 4);
  L.tl = take(M * 4);
  L.x0 = (c->extras & NC_EXTRA_RESID_LAMBDAS) ? take(M * C * 4) : 0;
  L.xmid = (c->extras & NC_EXTRA_BACKOUT) ? take(M * C * 4) : 0;
  // e4m3 codes of the activation entering the current product (the widest is
  // the MLP c_proj input, 4C), and the amax slots
  const size_t widest = std::max(4 * C, H * D);
  L.a8 = c->fp8 ? take(M * widest) : 0;
  L.amax = c->fp8 ? take((size_t)amax_slots(c->n_layer) * 4) : 0;
  L.total = off;
  return L;
}

// KV-cache session: the 16-bit weights and the RoPE table (cast and built once
// by nc_prefill), the cache of every layer, the token of every position (smear
// reads the previous one), and the scratch of one decode step (B rows; x0 and
// x_mid for the residual lambdas and backout).  Offsets are 256-byte aligned.
struct SessionLayout {
  size_t status, rope, wqkv, wo, wfc, wmp, wlm, cache, hist, x, a, qkv, o, h, part, acc, x0, xmid, total;
  size_t wqkv_elems, wo_elems, wfc_elems, wmp_elems, cache_layer_elems;
};

SessionLayout session_layout(const nc_config* c, int B, int T_max) {
  SessionLayout L;
  const size_t C = c->d_model, D = c->head_dim, H = c->n_head, Hkv = c->n_kv_head, V = c->vocab;
  const size_t nqkv = (H + 2 * Hkv) * D, Bs = (size_t)B;
  L.wqkv_elems = nqkv * C;
  L.wo_elems = C * H * D;
  L.wfc_elems = 4 * C * C;
  L.wmp_elems = C * 4 * C;
  L.cache_layer_elems = Bs * T_max * 2 * Hkv * D;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  L.status = take(256);
  L.rope = take((size_t)T_max * D * sizeof(float) * 2);  // [2][T_max][D/2] and the pair-major copy
  L.wqkv = take(c->n_layer * L.wqkv_elems * 2);
  L.wo = take(c->n_layer * L.wo_elems * 2);
  L.wfc = take(c->n_layer * L.wfc_elems * 2);
  L.wmp = take(c->n_layer * L.wmp_elems * 2);
  L.wlm = take(V * C * 2);
  L.cache = take(c->n_layer * L.cache_layer_elems * 2);
  L.hist = (c->extras & NC_EXTRA_SMEAR) ? take(Bs * T_max * 4) : 0;
  L.x = take(Bs * C * 4);
  L.a = take(Bs * C * 2);
  L.qkv = take(Bs * nqkv * 2);
  L.o = take(Bs * H * D * 2);
  L.h = take(Bs * 4 * C * 2);
  L.part = take(Bs * H * (size_t)decode_attention_max_splits() * (2 + D) * 4);
  L.acc = take(Bs * (nqkv > 4 * C ? nqkv : 4 * C) * 4);  // fp32 split-K sums of QKV, then c_fc
  L.x0 = (c->extras & NC_EXTRA_RESID_LAMBDAS) ? take(Bs * C * 4) : 0;
  L.xmid = (c->extras & NC_EXTRA_BACKOUT) ? take(Bs * C * 4) : 0;
  L.total = off;
  return L;
}

// Where nc_prefill puts what a later decode step reads.
struct SessionRef {
  uint8_t* base;
  int T_max;
};

inline cudaStream_t S(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// Brackets each launch of the forward with a caller-provided pair of events.
struct Tracer {
  nc_trace* t;
  cudaStream_t st;
  int n = 0;
  bool dry;  // count launches only
  bool begin(int kind) {
    if (!t) return true;
    if (!dry && n < t->capacity) {
      if (t->kinds) t->kinds[n] = kind;
      return cudaEventRecord(static_cast<cudaEvent_t>(t->events[2 * n]), st) == cudaSuccess;
    }
    return true;
  }
  bool end() {
    if (!t) return true;
    bool ok = true;
    if (!dry && n < t->capacity)
      ok = cudaEventRecord(static_cast<cudaEvent_t>(t->events[2 * n + 1]), st) == cudaSuccess;
    ++n;
    return ok;
  }
};

// Number of kernel launches of one forward.
int forward_launch_count(const nc_config* c, bool targets, bool loss, bool logits) {
  int n = 3 + c->n_layer * 7 + 1;  // rope table, cast, embedding; layers; final norm
  if (c->fp8 & NC_FP8_BLOCK) n += 4 * c->n_layer;  // activation quantisations
  if (targets) n += 2 + (loss ? 1 : 0);
  else if (logits) n += 1;
  if ((c->fp8 & NC_FP8_LM_HEAD) && (targets || logits)) n += 1;
  return n;
}

nc_status device_ok() {
  return device_is_sm100() ? NC_OK : NC_ERR_UNSUPPORTED_DEVICE;
}

}  // namespace

extern "C" {

int nc_version(void) { return 101; }

const char* nc_status_string(nc_status s) {
  switch (s) {
    case NC_OK: return "ok";
    case NC_ERR_INVALID_ARG: return "invalid argument";
    case NC_ERR_CONFIG: return "invalid configuration";
    case NC_ERR_SHAPE: return "unsupported shape";
    case NC_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case NC_ERR_WORKSPACE: return "workspace too small";
    case NC_ERR_TOKEN_RANGE: return "token or target id out of range";
    case NC_ERR_TIMEOUT: return "bounded device wait ran out";
    case NC_ERR_UNSUPPORTED_DEVICE: return "device is not sm_100";
    case NC_ERR_CUDA: return "CUDA runtime error";
    case NC_ERR_F16_RANGE: return "an fp16 activation saturated at +-65504";
  }
  return "unknown status";
}

nc_status nc_init_config(nc_config* out, int depth, int aspect_ratio, int head_dim, int n_kv_head,
                         int seq_len, int vocab) {
  if (!out || depth < 1 || aspect_ratio < 1 || head_dim < 1 || n_kv_head < 0 || seq_len < 4 ||
      vocab < 1)
    return NC_ERR_INVALID_ARG;
  nc_config c;
  memset(&c, 0, sizeof(c));
  c.n_layer = depth;
  c.d_model = depth * aspect_ratio;
  c.head_dim = head_dim;
  c.n_head = c.d_model / head_dim;
  c.n_kv_head = n_kv_head > 0 ? n_kv_head : c.n_head;
  c.vocab = vocab;
  c.seq_len = seq_len;
  c.short_window = seq_len / 4;
  strcpy(c.window_pattern, "SSSL");
  c.softcap = 15.0f;
  c.norm_eps = 1e-6f;
  c.rope_base = 10000.0f;
  c.act_dtype = NC_F16;
  *out = c;
  return config_ok(&c) ? NC_OK : NC_ERR_CONFIG;
}

nc_status nc_check_config(const nc_config* cfg) {
  if (!cfg) return NC_ERR_INVALID_ARG;
  return config_ok(cfg) ? NC_OK : NC_ERR_CONFIG;
}

int nc_layer_window(const nc_config* cfg, int layer) {
  if (!config_ok(cfg) || layer < 0 || layer >= cfg->n_layer) return -1;
  const size_t plen = strlen(cfg->window_pattern);
  char kind = cfg->window_pattern[layer % plen];
  if (layer == cfg->n_layer - 1) kind = 'L';
  return kind == 'L' ? cfg->seq_len : cfg->short_window;
}

int nc_layer_value_embed(const nc_config* cfg, int layer) {
  if (!config_ok(cfg) || layer < 0 || layer >= cfg->n_layer) return -1;
  return (cfg->n_layer - 1 - layer) % 2 == 0 ? 1 : 0;
}

size_t nc_workspace_bytes(const nc_config* cfg, int B, int T) {
  if (!config_ok(cfg) || B < 1 || T < 1 || T > cfg->seq_len) return 0;
  return ws_layout(cfg, B, T).total;
}

double nc_forward_flops(const nc_config* cfg, int B, int T) {
  if (!config_ok(cfg) || B < 1 || T < 1) return 0.0;
  const double M = (double)B * T, C = cfg->d_model, D = cfg->head_dim, H = cfg->n_head,
               Hkv = cfg->n_kv_head, V = cfg->vocab;
  const double per_layer_proj = 2.0 * M * C * (H + 2 * Hkv) * D + 2.0 * M * H * D * C + 16.0 * M * C * C;
  double f = cfg->n_layer * per_layer_proj + 2.0 * M * C * V;
  for (int l = 0; l < cfg->n_layer; ++l) {
    const int W = nc_layer_window(cfg, l);
    double keys = 0.0;  // sum over query positions of visible keys
    for (int i = 0; i < T; ++i) keys += (double)(i + 1 < W ? i + 1 : W);
    f += 4.0 * D * H * B * keys;  // QK^T and PV, 2 flops per multiply-add each
  }
  return f;
}

nc_status nc_get_status(const void* dev_status, void* stream) {
  if (!dev_status) return NC_ERR_INVALID_ARG;
  uint32_t st = 0;
  if (cudaStreamSynchronize(S(stream)) != cudaSuccess) return NC_ERR_CUDA;
  if (cudaMemcpy(&st, dev_status, sizeof(st), cudaMemcpyDeviceToHost) != cudaSuccess)
    return NC_ERR_CUDA;
  if (st & NC_DEV_TIMEOUT) return NC_ERR_TIMEOUT;
  if (st & NC_DEV_SMEM_ALIGN) return NC_ERR_CUDA;
  if (st & NC_DEV_POSITION) return NC_ERR_SHAPE;
  if (st & NC_DEV_F16_RANGE) return NC_ERR_F16_RANGE;
  if (st & (NC_DEV_TOKEN_RANGE | NC_DEV_TARGET_RANGE)) return NC_ERR_TOKEN_RANGE;
  return NC_OK;
}

inline bool dtype_ok(int d) { return d == NC_F16 || d == NC_BF16; }

nc_status nc_cast_weights(const float* src, uint16_t* dst, int64_t n, nc_dtype container,
                          void* stream) {
  if (!src || !dst || n < 0 || n % 8 != 0 || !dtype_ok(container)) return NC_ERR_INVALID_ARG;
  if (!aligned16(src) || !aligned16(dst)) return NC_ERR_ALIGNMENT;
  if (nc_status s = device_ok()) return s;
  CastSeg seg{src, dst, n};
  return cast_launch(&seg, 1, container == NC_F16, S(stream));
}

nc_status nc_embedding(const int32_t* tokens, const float* wte, float* x, int M, int C, int V,
                       uint32_t* dev_status, void* stream) {
  if (!tokens || !wte || !x || M < 0 || C < 4 || C % 4 != 0 || V < 1) return NC_ERR_INVALID_ARG;
  if (!aligned16(wte) || !aligned16(x)) return NC_ERR_ALIGNMENT;
  if (nc_status s = device_ok()) return s;
  return embedding_launch(tokens, wte, x, M, C, V, dev_status, S(stream));
}

nc_status nc_rmsnorm(const float* x, uint16_t* out, int M, int C, float eps, nc_dtype dtype,
                     void* stream) {
  if (!x || !out || M < 0 || C < 8 || C % 8 != 0 || !(eps >= 0.0f) || !dtype_ok(dtype))
    return NC_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(out)) return NC_ERR_ALIGNMENT;
  if (nc_status s = device_ok()) return s;
  return rmsnorm_launch(x, out, M, C, eps, dtype == NC_F16, S(stream));
}

nc_status nc_rope_table(float* table, int T, int D, float base, void* stream) {
  if (!table || T < 1 || D < 2 || D % 2 != 0 || !(base > 1.0f)) return NC_ERR_INVALID_ARG;
  if (nc_status s = device_ok()) return s;
  return rope_table_launch(table, T, D, base, S(stream));
}

nc_status nc_rope_qknorm(uint16_t* q, uint16_t* k, const float* table, int B, int T, int H, int Hkv,
                         int D, int64_t q_row_stride, int64_t k_row_stride, float eps,
                         nc_dtype dtype, void* stream) {
  if (!q || !k || !table || B < 0 || T < 1 || H < 1 || Hkv < 1 || !dtype_ok(dtype))
    return NC_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return NC_ERR_SHAPE;
  if (q_row_stride < (int64_t)H * D || k_row_stride < (int64_t)Hkv * D || q_row_stride % 8 ||
      k_row_stride % 8)
    return NC_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(table)) return NC_ERR_ALIGNMENT;
  if (nc_status s = device_ok()) return s;
  return rope_qknorm_launch(q, k, table, B, T, H, Hkv, D, q_row_stride, k_row_stride, eps,
                            dtype == NC_F16, S(stream));
}

nc_status nc_attention_strided(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                               uint16_t* out, int B, int T, int H, int Hkv, int D, int window,
                               int64_t q_row_stride, int64_t kv_row_stride, nc_dtype dtype,
                               void* stream) {
  if (!q || !k || !v || !out || B < 0 || T < 0 || H < 1 || Hkv < 1 || H % Hkv != 0 ||
      !dtype_ok(dtype))
    return NC_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return NC_ERR_SHAPE;
  if (q_row_stride < (int64_t)H * D || kv_row_stride < (int64_t)Hkv * D || q_row_stride % 8 ||
      kv_row_stride % 8)
    return NC_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return NC_ERR_ALIGNMENT;
  if (nc_status s = device_ok()) return s;
  return attention_launch(q, k, v, out, B, T, H, Hkv, D, window, q_row_stride, kv_row_stride,
                          dtype == NC_F16, nullptr, S(stream));
}

nc_status nc_attention_lse(const uint16_t* q, const uint16_t* k, const uint16_t* v, uint16_t* out, float* lse,
                           int B, int T, int H, int Hkv, int D, int window, int64_t q_row_stride,
                           int64_t kv_row_stride, nc_dtype dtype, void* stream) {
  if (!q || !k || !v || !out || !lse || B < 0 || T < 0 || H < 1 || Hkv < 1 || H % Hkv != 0 || !dtype_ok(dtype))
    return NC_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return NC_ERR_SHAPE;
  if (q_row_stride < (int64_t)H * D || kv_row_stride < (int64_t)Hkv * D || q_row_stride % 8 || kv_row_stride % 8)
    return NC_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return NC_ERR_ALIGNMENT;
  if (nc_status s = device_ok()) return s;
  return attention_launch(q, k, v, out, B, T, H, Hkv, D, window, q_row_stride, kv_row_stride, dtype == NC_F16,
                          nullptr, S(stream), nullptr, lse);
}

nc_status nc_attention_backward(const uint16_t* qkv, const uint16_t* o, const uint16_t* dO, const float* lse,
                                float* delta, uint16_t* dqkv, int B, int T, int H, int Hkv, int D, int window,
                                nc_dtype dtype, void* stream) {
  if (!qkv || !o || !dO || !lse || !delta || !dqkv || B < 0 || T < 0 || H < 1 || Hkv < 1 || H % Hkv != 0 ||
      !dtype_ok(dtype))
    return NC_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return NC_ERR_SHAPE;
  if (!aligned16(qkv) || !aligned16(o) || !aligned16(dO) || !aligned16(dqkv)) return NC_ERR_ALIGNMENT;
  if (nc_status s = device_ok()) return s;
  return attn_bwd_launch(qkv, (int64_t)(H + 2 * Hkv) * D, o, dO, lse, delta, dqkv, B, T, H, Hkv, D, window,
                         dtype == NC_F16, S(stream));
}

nc_status nc_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v, uint16_t* out, int B,
                       int T, int H, int Hkv, int D, int window, nc_dtype dtype, void* stream) {
  return nc_attention_strided(q, k, v, out, B, T, H, Hkv, D, window, (int64_t)H * D,
                              (int64_t)Hkv * D, dtype, stream);
}

nc_status nc_linear(const uint16_t* a, const uint16_t* w, void* out, int M, int N, int K,
                    int64_t ldo, nc_epilogue epilogue, float cap, nc_dtype dtype,
                    uint32_t* dev_status, void* stream) {
  if (!a || !w || !out || M < 0 || N < 32 || K < 8 || !dtype_ok(dtype)) return NC_ERR_INVALID_ARG;
  if ((int)epilogue < 0 || (int)epilogue > (int)NC_EPI_SOFTCAP_F32) return NC_ERR_INVALID_ARG;
  if (N % 32 != 0 || K % 8 != 0 || ldo < N || ldo % 8 != 0) return NC_ERR_SHAPE;
  if (epilogue == NC_EPI_SOFTCAP_F32 && !(cap > 0.0f)) return NC_ERR_INVALID_ARG;
  if (!aligned16(a) || !aligned16(w) || !aligned16(out)) return NC_ERR_ALIGNMENT;
  if (nc_status s = device_ok()) return s;
  if (M == 0) return NC_OK;
  EpiParams ep{};
  ep.out = out;
  ep.ldo = ldo;
  ep.cap = cap;
  return gemm_launch(a, K, w, K, M, N, K, (int)epilogue, dtype == NC_F16, ep, dev_status, S(stream));
}

nc_status nc_linear_dgrad(const uint16_t* dy, const uint16_t* w, void* dx, int M, int N, int K,
                          nc_epilogue epilogue, nc_dtype dtype, uint32_t* dev_status, void* stream) {
  if (!dy || !w || !dx || M < 0 || N < 8 || K < 8 || !dtype_ok(dtype)) return NC_ERR_INVALID_ARG;
  if (epilogue != NC_EPI_STORE_16 && epilogue != NC_EPI_STORE_F32) return NC_ERR_INVALID_ARG;
  if (N % 8 != 0 || K % 8 != 0) return NC_ERR_SHAPE;
  if (!aligned16(dy) || !aligned16(w) || !aligned16(dx)) return NC_ERR_ALIGNMENT;
  if (nc_status s = device_ok()) return s;
  if (M == 0) return NC_OK;
  EpiParams ep{};
  ep.out = dx;
  ep.ldo = K;
  // dx = dy . w: contraction over N, output columns K; w [N, K] is the MN-major operand
  return gemm_launch_layout(dy, N, w, K, M, K, N, (int)epilogue, dtype == NC_F16, GEMM_NN, ep, dev_status, S(stream));
}

nc_status nc_linear_wgrad(const uint16_t* dy, const uint16_t* x, float* dw, int M, int N, int K, float alpha,
                          nc_dtype dtype, uint32_t* dev_status, void* stream) {
  if (!dy || !x || !dw || M < 1 || N < 8 || K < 8 || !dtype_ok(dtype)) return NC_ERR_INVALID_ARG;
  if (N % 8 != 0 || K % 8 != 0) return NC_ERR_SHAPE;
  if (!aligned16(dy) || !aligned16(x) || !aligned16(dw)) return NC_ERR_ALIGNMENT;
  if (nc_status s = device_ok()) return s;
  if (alpha == 0.0f) return NC_OK;  // nothing to add
  EpiParams ep{};
  ep.out = dw;
  ep.ldo = K;
  ep.alpha = alpha;
  const int tiles = ((N + 127) / 128) * ((K + 255) / 256);
  const int nkb = (M + 63) / 64;
  int ks = (8 * device_sm_count() + tiles - 1) / tiles;
  ks = std::min(ks, std::max(1, nkb / 16));
  ep.ksplit = std::max(ks, 1);
  return gemm_launch_layout(dy, N, x, K, N, K, M, EPI_RESID_F32, dtype == NC_F16, GEMM_TN, ep, dev_status, S(stream));
}

nc_status nc_fp8_quantize(const void* x, nc_dtype src_dtype, int64_t n, uint8_t* codes, float* amax,
                          void* stream) {
  if (!x || !codes || !amax || n < 0) return NC_ERR_INVALID_ARG;
  if (src_dtype != NC_F32 && src_dtype != NC_BF16 && src_dtype != NC_F16) return NC_ERR_INVALID_ARG;
  if (n % 16 != 0) return NC_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(codes)) return NC_ERR_ALIGNMENT;
  if (nc_status s = device_ok()) return s;
  cudaStream_t st = S(stream);
  if (cudaMemsetAsync(amax, 0, sizeof(float), st) != cudaSuccess) return NC_ERR_CUDA;
  const Fp8Seg seg{x, codes, n, 0};
  const int kind = src_dtype == NC_F32 ? FP8_SRC_F32 : src_dtype == NC_F16 ? FP8_SRC_F16 : FP8_SRC_BF16;
  return fp8_quantize_launch(&seg, 1, kind, amax, true, st);
}

nc_status nc_linear_fp8(const uint8_t* a, const float* amax_a, const uint8_t* w, const float* amax_w,
                        void* out, int M, int N, int K, int64_t ldo, nc_epilogue epilogue, float cap,
                        nc_dtype dtype, uint32_t* dev_status, void* stream) {
  if (!a || !w || !amax_a || !amax_w || !out || M < 0 || N < 32 || K < 16 || !dtype_ok(dtype))
    return NC_ERR_INVALID_ARG;
  if ((int)epilogue < 0 || (int)epilogue > (int)NC_EPI_SOFTCAP_F32) return NC_ERR_INVALID_ARG;
  if (N % 32 != 0 || K % 16 != 0 || ldo < N || ldo % 8 != 0) return NC_ERR_SHAPE;
  if (epilogue == NC_EPI_SOFTCAP_F32 && !(cap > 0.0f)) return NC_ERR_INVALID_ARG;
  if (!aligned16(a) || !aligned16(w) || !aligned16(out)) return NC_ERR_ALIGNMENT;
  if (nc_status s = device_ok()) return s;
  if (M == 0) return NC_OK;
  EpiParams ep{};
  ep.out = out;
  ep.ldo = ldo;
  ep.cap = cap;
  ep.amax_a = amax_a;
  ep.amax_b = amax_w;
  return gemm_launch_e4m3(a, K, w, K, M, N, K, (int)epilogue, dtype == NC_F16, ep, dev_status, S(stream));
}

nc_status nc_qkv_rope(const uint16_t* a, const uint16_t* w, uint16_t* out, const float* table,
                      int M, int T, int C, int H, int Hkv, int D, float eps, nc_dtype dtype,
                      uint32_t* dev_status, void* stream) {
  if (!a || !w || !out || !table || M < 0 || T < 1 || C < 8 || H < 1 || Hkv < 1 ||
      !(eps >= 0.0f) || !dtype_ok(dtype))
    return NC_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return NC_ERR_SHAPE;
  if (C % 8 != 0) return NC_ERR_SHAPE;
  if (!aligned16(a) || !aligned16(w) || !aligned16(out) || !aligned16(table)) return NC_ERR_ALIGNMENT;
  if (nc_status s = device_ok()) return s;
  if (M == 0) return NC_OK;
  const int N = (H + 2 * Hkv) * D;
  EpiParams ep{};
  ep.out = out;
  ep.ldo = N;
  ep.rope = table;
  ep.T = T;
  ep.H = H;
  ep.Hkv = Hkv;
  ep.D = D;
  ep.eps = eps;
  return gemm_launch(a, C, w, C, M, N, C, EPI_QKV_ROPE, dtype == NC_F16, ep, dev_status, S(stream));
}

nc_status nc_softcap_ce(const float* z, const int32_t* targets, float* capped_out,
                        float* token_loss, int M, int V, float cap, uint32_t* dev_status,
                        void* stream) {
  if (!z || !targets || !token_loss || M < 0 || V < 4 || V % 4 != 0 || !(cap > 0.0f))
    return NC_ERR_INVALID_ARG;
  if (!aligned16(z) || (capped_out && !aligned16(capped_out))) return NC_ERR_ALIGNMENT;
  if (nc_status s = device_ok()) return s;
  return softcap_ce_launch(z, targets, capped_out, token_loss, M, V, cap, dev_status, S(stream));
}

nc_status nc_loss_mean(const float* token_loss, const int32_t* targets, int M, int V, float* loss,
                       void* stream) {
  if (!token_loss || !targets || !loss || M < 0 || V < 1) return NC_ERR_INVALID_ARG;
  if (nc_status s = device_ok()) return s;
  return loss_mean_launch(token_loss, targets, M, V, loss, S(stream));
}

// The one weight-cast launch: every fp32 matmul weight -> its bf16 value (held
// in fp16 when f16); c_q, c_k, c_v of a layer packed into one matrix, with the
// rows of c_q and c_k reordered so each RoPE pair is adjacent.
//
// With cfg->fp8 the weights of the chosen products are quantised to e4m3
// instead (same packing and row order, one byte per element): one amax launch
// and one quantise launch over all of them, each weight tensor with its own
// slot in `amax` (zeroed by the caller).
static nc_status launch_weight_cast(const nc_config* cfg, const nc_weights* w, uint16_t* wqkv, uint16_t* wo,
                                    uint16_t* wfc, uint16_t* wmp, uint16_t* wlm, size_t e_qkv, size_t e_wo,
                                    size_t e_fc, size_t e_mp, bool f16, cudaStream_t st, float* amax = nullptr) {
  const int C = cfg->d_model, D = cfg->head_dim, H = cfg->n_head, Hkv = cfg->n_kv_head, V = cfg->vocab;
  const size_t nq = (size_t)H * D * C, nk = (size_t)Hkv * D * C;
  const bool q_block = (cfg->fp8 & NC_FP8_BLOCK) != 0, q_head = (cfg->fp8 & NC_FP8_LM_HEAD) != 0;
  if (q_block || q_head) {
    std::vector<Fp8Seg> qs;
    qs.reserve(cfg->n_layer * 6 + 1);
    if (q_block) {
      for (int l = 0; l < cfg->n_layer; ++l) {
        uint8_t* dq = reinterpret_cast<uint8_t*>(wqkv) + l * e_qkv;
        qs.push_back({w->c_q[l], dq, (int64_t)nq, amax_w_slot(l, 0), true});
        qs.push_back({w->c_k[l], dq + nq, (int64_t)nk, amax_w_slot(l, 1), true});
        qs.push_back({w->c_v[l], dq + nq + nk, (int64_t)nk, amax_w_slot(l, 2)});
        qs.push_back({w->attn_proj[l], reinterpret_cast<uint8_t*>(wo) + l * e_wo, (int64_t)e_wo, amax_w_slot(l, 3)});
        qs.push_back({w->c_fc[l], reinterpret_cast<uint8_t*>(wfc) + l * e_fc, (int64_t)e_fc, amax_w_slot(l, 4)});
        qs.push_back({w->mlp_proj[l], reinterpret_cast<uint8_t*>(wmp) + l * e_mp, (int64_t)e_mp, amax_w_slot(l, 5)});
      }
    }
    if (q_head)
      qs.push_back({w->lm_head, reinterpret_cast<uint8_t*>(wlm), (int64_t)V * C, amax_wlm_slot(cfg->n_layer)});
    if (nc_status s = fp8_quantize_launch(qs.data(), (int)qs.size(), FP8_SRC_F32, amax, true, st, C, D)) return s;
  }
  std::vector<CastSeg> segs;
  segs.reserve(cfg->n_layer * 6 + 1);
  for (int l = 0; l < cfg->n_layer && !q_block; ++l) {
    uint16_t* dq = wqkv + l * e_qkv;
    segs.push_back({w->c_q[l], dq, (int64_t)nq, true});  // RoPE pairs made adjacent
    segs.push_back({w->c_k[l], dq + nq, (int64_t)nk, true});
    segs.push_back({w->c_v[l], dq + nq + nk, (int64_t)nk});
    segs.push_back({w->attn_proj[l], wo + l * e_wo, (int64_t)e_wo});
    segs.push_back({w->c_fc[l], wfc + l * e_fc, (int64_t)e_fc});
    segs.push_back({w->mlp_proj[l], wmp + l * e_mp, (int64_t)e_mp});
  }
  if (!q_head) segs.push_back({w->lm_head, wlm, (int64_t)V * C});
  if (segs.empty()) return NC_OK;
  return cast_launch(segs.data(), (int)segs.size(), f16, st, C, D);
}

// Checks the fp32 weight pointers of the plain block stack.
static nc_status check_weights(const nc_config* cfg, const nc_weights* w) {
  if (!w->wte || !w->lm_head || !w->c_q || !w->c_k || !w->c_v || !w->attn_proj || !w->c_fc || !w->mlp_proj)
    return NC_ERR_INVALID_ARG;
  if (!aligned16(w->wte) || !aligned16(w->lm_head)) return NC_ERR_ALIGNMENT;
  for (int l = 0; l < cfg->n_layer; ++l) {
    const float* ps[6] = {w->c_q[l], w->c_k[l], w->c_v[l], w->attn_proj[l], w->c_fc[l], w->mlp_proj[l]};
    for (const float* p : ps) {
      if (!p) return NC_ERR_INVALID_ARG;
      if (!aligned16(p)) return NC_ERR_ALIGNMENT;
    }
  }
  return NC_OK;
}

// The parameters of the further forward terms that cfg->extras switches on.
static nc_status check_extras(const nc_config* cfg, const nc_weights* w) {
  const uint32_t ex = cfg->extras;
  if (ex & NC_EXTRA_SMEAR) {
    if (!w->smear_gate) return NC_ERR_INVALID_ARG;
    if (!aligned16(w->smear_gate)) return NC_ERR_ALIGNMENT;
  }
  if (ex & NC_EXTRA_VALUE_EMBED) {
    if (!w->value_embeds || !w->ve_gates) return NC_ERR_INVALID_ARG;
    for (int l = 0; l < cfg->n_layer; ++l) {
      if (nc_layer_value_embed(cfg, l) != 1) continue;
      if (!w->value_embeds[l] || !w->ve_gates[l]) return NC_ERR_INVALID_ARG;
      if (!aligned16(w->value_embeds[l])) return NC_ERR_ALIGNMENT;
    }
  }
  if ((ex & NC_EXTRA_RESID_LAMBDAS) && (!w->resid_lambdas || !w->x0_lambdas)) return NC_ERR_INVALID_ARG;
  if ((ex & NC_EXTRA_BACKOUT) && !w->backout_lambda) return NC_ERR_INVALID_ARG;
  return NC_OK;
}

static nc_status forward_impl(const nc_config* cfg, const nc_weights* w, const int32_t* tokens,
                              const int32_t* targets, int B, int T, float* logits, float* token_loss,
                              float* loss, void* workspace, size_t ws_bytes, void* stream, nc_trace* trace,
                              const SessionRef* sess) {
  if (!cfg || !w || !tokens || !workspace) return NC_ERR_INVALID_ARG;
  if (!config_ok(cfg)) return NC_ERR_CONFIG;
  if (B < 1 || T < 1 || T > cfg->seq_len) return NC_ERR_SHAPE;
  if ((token_loss || loss) && !targets) return NC_ERR_INVALID_ARG;
  if ((int64_t)B * T > (int64_t)1 << 30) return NC_ERR_SHAPE;
  const WsLayout L = ws_layout(cfg, B, T, sess == nullptr);
  if (ws_bytes < L.total) return NC_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return NC_ERR_ALIGNMENT;
  if (logits && !aligned16(logits)) return NC_ERR_ALIGNMENT;
  if (nc_status s = check_weights(cfg, w)) return s;
  if (nc_status s = check_extras(cfg, w)) return s;
  const uint32_t ex = cfg->extras;
  if (trace) {
    const int need = forward_launch_count(cfg, targets != nullptr, loss != nullptr, logits != nullptr);
    trace->count = need;
    if (!trace->events || trace->capacity < need) return NC_ERR_INVALID_ARG;
    for (int i = 0; i < 2 * need; ++i)
      if (!trace->events[i]) return NC_ERR_INVALID_ARG;
  }
  if (nc_status s = device_ok()) return s;

  cudaStream_t st = S(stream);
  Tracer tr{trace, st, 0, false};
#define NC_RUN(kind, call)                          \
  do {                                              \
    if (!tr.begin(kind)) return NC_ERR_CUDA;        \
    nc_status s_ = (call);                          \
    if (s_ != NC_OK) return s_;                     \
    if (!tr.end()) return NC_ERR_CUDA;              \
  } while (0)
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  // 16-bit weights and RoPE table: in the workspace, or in the session (prefill)
  SessionLayout SL{};
  uint8_t* wbase = ws;
  size_t o_st = L.status, o_rope = L.rope, o_wqkv = L.wqkv, o_wo = L.wo, o_wfc = L.wfc, o_wmp = L.wmp,
         o_wlm = L.wlm;
  int T_rope = T;
  if (sess) {
    SL = session_layout(cfg, B, sess->T_max);
    wbase = sess->base;
    o_st = SL.status;
    o_rope = SL.rope;
    o_wqkv = SL.wqkv;
    o_wo = SL.wo;
    o_wfc = SL.wfc;
    o_wmp = SL.wmp;
    o_wlm = SL.wlm;
    T_rope = sess->T_max;
  }
  uint32_t* status = reinterpret_cast<uint32_t*>(wbase + o_st);
  float* rope = reinterpret_cast<float*>(wbase + o_rope);
  uint16_t* wqkv = reinterpret_cast<uint16_t*>(wbase + o_wqkv);
  uint16_t* wo = reinterpret_cast<uint16_t*>(wbase + o_wo);
  uint16_t* wfc = reinterpret_cast<uint16_t*>(wbase + o_wfc);
  uint16_t* wmp = reinterpret_cast<uint16_t*>(wbase + o_wmp);
  uint16_t* wlm = reinterpret_cast<uint16_t*>(wbase + o_wlm);
  float* x = reinterpret_cast<float*>(ws + L.x);
  uint16_t* a = reinterpret_cast<uint16_t*>(ws + L.a);
  uint16_t* qkv = reinterpret_cast<uint16_t*>(ws + L.qkv);
  uint16_t* o = reinterpret_cast<uint16_t*>(ws + L.o);
  uint16_t* h = reinterpret_cast<uint16_t*>(ws + L.h);
  float* part = reinterpret_cast<float*>(ws + L.part);
  float* tgt = reinterpret_cast<float*>(ws + L.tgt);
  float* tl = token_loss ? token_loss : reinterpret_cast<float*>(ws + L.tl);
  float* x0 = (ex & NC_EXTRA_RESID_LAMBDAS) ? reinterpret_cast<float*>(ws + L.x0) : nullptr;
  float* xmid = (ex & NC_EXTRA_BACKOUT) ? reinterpret_cast<float*>(ws + L.xmid) : nullptr;
  const bool q_block = (cfg->fp8 & NC_FP8_BLOCK) != 0, q_head = (cfg->fp8 & NC_FP8_LM_HEAD) != 0;
  uint8_t* a8 = cfg->fp8 ? ws + L.a8 : nullptr;
  float* amax = cfg->fp8 ? reinterpret_cast<float*>(ws + L.amax) : nullptr;
  const int mid = cfg->n_layer / 2;  // backout: the stream after the first n_layer / 2 blocks

  const int M = B * T;
  const int C = cfg->d_model, D = cfg->head_dim, H = cfg->n_head, Hkv = cfg->n_kv_head,
            V = cfg->vocab;
  const int NQKV = (H + 2 * Hkv) * D;
  const bool f16 = cfg->act_dtype == NC_F16;

  if (cudaMemsetAsync(status, 0, 256, st) != cudaSuccess) return NC_ERR_CUDA;
  if (amax && cudaMemsetAsync(amax, 0, (size_t)amax_slots(cfg->n_layer) * 4, st) != cudaSuccess)
    return NC_ERR_CUDA;
  NC_RUN(NC_K_ROPE_TABLE, rope_table_launch(rope, T_rope, D, cfg->rope_base, st, rope_pairs_of(rope, T_rope, D)));

  // fp32 -> bf16 weight cast (e4m3 for the fp8 products); c_q|c_k|c_v rows
  // packed into one matrix per layer.
  NC_RUN(NC_K_CAST, launch_weight_cast(cfg, w, wqkv, wo, wfc, wmp, wlm, L.wqkv_elems, L.wo_elems, L.wfc_elems,
                                       L.wmp_elems, f16, st, amax));
  const int src16 = f16 ? FP8_SRC_F16 : FP8_SRC_BF16;
  // e4m3 codes of the activation `src` ([M, K] 16-bit) into a8, amax into its slot
  // (the producers of the plain path fold the amax in themselves: fused = true)
  auto quant_act = [&](const uint16_t* src, int K, int slot, bool fused) -> nc_status {
    const Fp8Seg seg{src, a8, (int64_t)M * K, slot};
    return fp8_quantize_launch(&seg, 1, src16, amax, !fused, st);
  };
  auto slot_ptr = [&](int slot) { return amax ? amax + slot : nullptr; };

  if (ex & (NC_EXTRA_SMEAR | NC_EXTRA_RESID_LAMBDAS))
    NC_RUN(NC_K_EMBEDDING, embedding_extra_launch(tokens, w->wte, (ex & NC_EXTRA_SMEAR) ? w->smear_gate : nullptr,
                                                  x, x0, M, C, V, T, status, st));
  else
    NC_RUN(NC_K_EMBEDDING, embedding_launch(tokens, w->wte, x, M, C, V, status, st));

  for (int l = 0; l < cfg->n_layer; ++l) {
    const int W = nc_layer_window(cfg, l);
    float* keep = (xmid && l == mid) ? xmid : nullptr;
    const bool mixed = x0 || keep;
    if (mixed)  // x_mid = the stream entering block `mid`; then x = a_l x + b_l x0
      NC_RUN(NC_K_RMSNORM, rmsnorm_mix_launch(x, x0, x0 ? w->resid_lambdas + l : nullptr,
                                              x0 ? w->x0_lambdas + l : nullptr, keep, nullptr, nullptr,
                                              x0 != nullptr, a, M, C, cfg->norm_eps, f16, st));
    else
      NC_RUN(NC_K_RMSNORM, rmsnorm_launch(x, a, M, C, cfg->norm_eps, f16, st,
                                          q_block ? slot_ptr(amax_a_slot(cfg->n_layer, l, 0)) : nullptr));
    EpiParams eq{};  // QKV projection with RoPE + QK-norm in the epilogue
    eq.out = qkv;
    eq.ldo = NQKV;
    eq.rope = rope;
    eq.T = T;
    eq.H = H;
    eq.Hkv = Hkv;
    eq.D = D;
    eq.eps = cfg->norm_eps;
    eq.rope_T = T_rope;
    eq.rope_pairs = rope_pairs_of(rope, T_rope, D);
    if ((ex & NC_EXTRA_VALUE_EMBED) && nc_layer_value_embed(cfg, l) == 1) {
      eq.tokens = tokens;
      eq.ve = w->value_embeds[l];
      eq.ve_gate = w->ve_gates[l];
      eq.V = V;
    }
    if (q_block) {
      NC_RUN(NC_K_FP8_QUANT, quant_act(a, C, amax_a_slot(cfg->n_layer, l, 0), !mixed));
      eq.amax_a = amax + amax_a_slot(cfg->n_layer, l, 0);
      eq.amax_b = amax + amax_w_slot(l, 0);  // q, k, v
      NC_RUN(NC_K_GEMM_QKV, gemm_launch_e4m3(a8, C, reinterpret_cast<uint8_t*>(wqkv) + l * L.wqkv_elems, C, M,
                                             NQKV, C, EPI_QKV_ROPE_IL, f16, eq, status, st));
    } else {
      NC_RUN(NC_K_GEMM_QKV, gemm_launch(a, C, wqkv + l * L.wqkv_elems, C, M, NQKV, C, EPI_QKV_ROPE_IL, f16,
                                        eq, status, st));
    }
    if (sess) {  // keep this layer's k and v for decoding
      uint16_t* cache = reinterpret_cast<uint16_t*>(sess->base + SL.cache) + l * SL.cache_layer_elems;
      nc_status s_ = kv_append_launch(qkv, NQKV, H * D, 2 * Hkv * D, cache, M, T, sess->T_max, 0, st);
      if (s_ != NC_OK) return s_;
    }
    NC_RUN(NC_K_ATTENTION, attention_launch(qkv, qkv + H * D, qkv + (H + Hkv) * D, o, B, T, H, Hkv,
                                            D, W, NQKV, NQKV, f16, status, st,
                                            q_block ? slot_ptr(amax_a_slot(cfg->n_layer, l, 1)) : nullptr));
    EpiParams ep{};
    ep.out = x;
    ep.ldo = C;
    if (q_block) {  // the three remaining products in e4m3, each input quantised first
      const int Lc = cfg->n_layer;
      uint8_t* w8o = reinterpret_cast<uint8_t*>(wo) + l * L.wo_elems;
      uint8_t* w8fc = reinterpret_cast<uint8_t*>(wfc) + l * L.wfc_elems;
      uint8_t* w8mp = reinterpret_cast<uint8_t*>(wmp) + l * L.wmp_elems;
      NC_RUN(NC_K_FP8_QUANT, quant_act(o, H * D, amax_a_slot(Lc, l, 1), true));
      ep.amax_a = amax + amax_a_slot(Lc, l, 1);
      ep.amax_b = amax + amax_w_slot(l, 3);
      NC_RUN(NC_K_GEMM_ATTN_PROJ,
             gemm_launch_e4m3(a8, H * D, w8o, H * D, M, C, H * D, EPI_RESID_F32, f16, ep, status, st));
      NC_RUN(NC_K_RMSNORM, rmsnorm_launch(x, a, M, C, cfg->norm_eps, f16, st, amax + amax_a_slot(Lc, l, 2)));
      NC_RUN(NC_K_FP8_QUANT, quant_act(a, C, amax_a_slot(Lc, l, 2), true));
      ep.out = h;
      ep.ldo = 4 * C;
      ep.amax_a = amax + amax_a_slot(Lc, l, 2);
      ep.amax_b = amax + amax_w_slot(l, 4);
      ep.amax_out = amax + amax_a_slot(Lc, l, 3);
      NC_RUN(NC_K_GEMM_FC, gemm_launch_e4m3(a8, C, w8fc, C, M, 4 * C, C, EPI_RELU2_16, f16, ep, status, st));
      NC_RUN(NC_K_FP8_QUANT, quant_act(h, 4 * C, amax_a_slot(Lc, l, 3), true));
      ep.amax_out = nullptr;
      ep.out = x;
      ep.ldo = C;
      ep.amax_a = amax + amax_a_slot(Lc, l, 3);
      ep.amax_b = amax + amax_w_slot(l, 5);
      NC_RUN(NC_K_GEMM_MLP_PROJ,
             gemm_launch_e4m3(a8, 4 * C, w8mp, 4 * C, M, C, 4 * C, EPI_RESID_F32, f16, ep, status, st));
      continue;
    }
    NC_RUN(NC_K_GEMM_ATTN_PROJ, gemm_launch(o, H * D, wo + l * L.wo_elems, H * D, M, C, H * D,
                                            EPI_RESID_F32, f16, ep, status, st));
    NC_RUN(NC_K_RMSNORM, rmsnorm_launch(x, a, M, C, cfg->norm_eps, f16, st));
    ep.out = h;
    ep.ldo = 4 * C;
    NC_RUN(NC_K_GEMM_FC,
           gemm_launch(a, C, wfc + l * L.wfc_elems, C, M, 4 * C, C, EPI_RELU2_16, f16, ep, status, st));
    ep.out = x;
    ep.ldo = C;
    NC_RUN(NC_K_GEMM_MLP_PROJ, gemm_launch(h, 4 * C, wmp + l * L.wmp_elems, 4 * C, M, C, 4 * C,
                                           EPI_RESID_F32, f16, ep, status, st));
  }

  if (xmid)  // backout: x - lambda * x_mid, then the final norm
    NC_RUN(NC_K_RMSNORM, rmsnorm_mix_launch(x, nullptr, nullptr, nullptr, nullptr, xmid, w->backout_lambda, false,
                                            a, M, C, cfg->norm_eps, f16, st));
  else
    NC_RUN(NC_K_RMSNORM, rmsnorm_launch(x, a, M, C, cfg->norm_eps, f16, st,
                                        q_head ? slot_ptr(amax_alm_slot(cfg->n_layer)) : nullptr));
  // LM head: 16-bit, or e4m3 codes of the final normalised stream
  const int alm = amax_alm_slot(cfg->n_layer);
  if (q_head && (targets || logits)) NC_RUN(NC_K_FP8_QUANT, quant_act(a, C, alm, xmid == nullptr));
  auto lm_head = [&](int epi, const EpiParams& ep0) -> nc_status {
    if (!q_head) return gemm_launch(a, C, wlm, C, M, V, C, epi, f16, ep0, status, st);
    EpiParams e8 = ep0;
    e8.amax_a = amax + alm;
    e8.amax_b = amax + amax_wlm_slot(cfg->n_layer);
    return gemm_launch_e4m3(a8, C, reinterpret_cast<uint8_t*>(wlm), C, M, V, C, epi, f16, e8, status, st);
  };
  if (targets) {
    EpiParams ep{};
    ep.out = logits;
    ep.ldo = V;
    ep.cap = cfg->softcap;
    ep.store_logits = logits != nullptr;
    ep.ce_partial = part;
    ep.ce_target = tgt;
    ep.targets = targets;
    NC_RUN(NC_K_GEMM_LM_HEAD, lm_head(EPI_CE_PARTIAL, ep));
    NC_RUN(NC_K_CE_FINALIZE, ce_finalize_launch(part, gemm_ce_partials_per_row(V), tgt, targets, tl, M, V,
                                                cfg->softcap, status, st));
    if (loss) NC_RUN(NC_K_LOSS_MEAN, loss_mean_launch(tl, targets, M, V, loss, st));
  } else if (logits) {
    EpiParams ep{};
    ep.out = logits;
    ep.ldo = V;
    ep.cap = cfg->softcap;
    NC_RUN(NC_K_GEMM_LM_HEAD, lm_head(EPI_SOFTCAP_F32, ep));
  }
#undef NC_RUN
  return NC_OK;
}

nc_status nc_forward_traced(const nc_config* cfg, const nc_weights* w, const int32_t* tokens,
                            const int32_t* targets, int B, int T, float* logits,
                            float* token_loss, float* loss, void* workspace, size_t ws_bytes,
                            void* stream, nc_trace* trace) {
  return forward_impl(cfg, w, tokens, targets, B, T, logits, token_loss, loss, workspace, ws_bytes, stream,
                      trace, nullptr);
}

nc_status nc_forward(const nc_config* cfg, const nc_weights* w, const int32_t* tokens,
                     const int32_t* targets, int B, int T, float* logits, float* token_loss,
                     float* loss, void* workspace, size_t ws_bytes, void* stream) {
  return nc_forward_traced(cfg, w, tokens, targets, B, T, logits, token_loss, loss, workspace,
                           ws_bytes, stream, nullptr);
}

size_t nc_session_bytes(const nc_config* cfg, int B, int T_max) {
  if (!config_ok(cfg) || B < 1 || T_max < 1 || T_max > cfg->seq_len) return 0;
  return session_layout(cfg, B, T_max).total;
}

size_t nc_prefill_workspace_bytes(const nc_config* cfg, int B, int T) {
  if (!config_ok(cfg) || B < 1 || T < 1 || T > cfg->seq_len) return 0;
  return ws_layout(cfg, B, T, false).total;
}

nc_status nc_prefill(const nc_config* cfg, const nc_weights* w, const int32_t* tokens, int B, int T,
                     float* logits, void* session, size_t session_bytes, int T_max, void* workspace,
                     size_t ws_bytes, void* stream) {
  if (!cfg || !w || !session) return NC_ERR_INVALID_ARG;
  if (!config_ok(cfg) || cfg->fp8 != 0) return NC_ERR_CONFIG;
  if (T_max < 1 || T_max > cfg->seq_len || T < 0 || T > T_max || B < 1) return NC_ERR_SHAPE;
  const SessionLayout SL = session_layout(cfg, B, T_max);
  if (session_bytes < SL.total) return NC_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(session) & 255u) != 0) return NC_ERR_ALIGNMENT;
  if (T == 0) {  // no prompt: only the weight cast and the RoPE table
    if (nc_status s = check_weights(cfg, w)) return s;
    if (nc_status s = device_ok()) return s;
    uint8_t* base = static_cast<uint8_t*>(session);
    cudaStream_t st = S(stream);
    if (cudaMemsetAsync(base + SL.status, 0, 256, st) != cudaSuccess) return NC_ERR_CUDA;
    float* rope = reinterpret_cast<float*>(base + SL.rope);
    if (nc_status s = rope_table_launch(rope, T_max, cfg->head_dim, cfg->rope_base, st,
                                        rope_pairs_of(rope, T_max, cfg->head_dim)))
      return s;
    return launch_weight_cast(cfg, w, reinterpret_cast<uint16_t*>(base + SL.wqkv),
                              reinterpret_cast<uint16_t*>(base + SL.wo), reinterpret_cast<uint16_t*>(base + SL.wfc),
                              reinterpret_cast<uint16_t*>(base + SL.wmp), reinterpret_cast<uint16_t*>(base + SL.wlm),
                              SL.wqkv_elems, SL.wo_elems, SL.wfc_elems, SL.wmp_elems, cfg->act_dtype == NC_F16, st);
  }
  const SessionRef sess{static_cast<uint8_t*>(session), T_max};
  if (nc_status s = forward_impl(cfg, w, tokens, nullptr, B, T, logits, nullptr, nullptr, workspace, ws_bytes,
                                 stream, nullptr, &sess))
    return s;
  if (cfg->extras & NC_EXTRA_SMEAR)  // the prompt's tokens, for the smear of the first decode step
    if (cudaMemcpy2DAsync(static_cast<uint8_t*>(session) + SL.hist, (size_t)T_max * 4, tokens, (size_t)T * 4,
                          (size_t)T * 4, B, cudaMemcpyDeviceToDevice, S(stream)) != cudaSuccess)
      return NC_ERR_CUDA;
  return NC_OK;
}

// K slices for a residual-add GEMM with few output tiles: about one tile per SM.
static int resid_ksplit(int M, int N, int K) {
  const int tiles = ((M + 127) / 128) * ((N + 255) / 256);
  const int kb = (K + 63) / 64;
  int s = (device_sm_count() + tiles - 1) / tiles;
  return s < 1 ? 1 : (s > kb ? kb : s);
}

}  // extern "C"

// One decode step at host position `pos`, or at the position *pos_dev holds on
// the device (then advanced by one at the end of the step).
static nc_status decode_impl(const nc_config* cfg, const nc_weights* w, const int32_t* tokens, int B, int pos,
                             int32_t* pos_dev, float* logits, void* session, size_t session_bytes, int T_max,
                             void* stream) {
  if (!cfg || !w || !w->wte || !tokens || !logits || !session) return NC_ERR_INVALID_ARG;
  if (!config_ok(cfg) || cfg->fp8 != 0) return NC_ERR_CONFIG;
  if (T_max < 1 || T_max > cfg->seq_len || B < 1 || (!pos_dev && (pos < 0 || pos >= T_max))) return NC_ERR_SHAPE;
  if (pos_dev && T_max > decode_attention_max_splits() * 64) return NC_ERR_SHAPE;
  if (pos_dev && !aligned16(pos_dev)) return NC_ERR_ALIGNMENT;
  const SessionLayout SL = session_layout(cfg, B, T_max);
  if (session_bytes < SL.total) return NC_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(session) & 255u) != 0) return NC_ERR_ALIGNMENT;
  if (!aligned16(w->wte) || !aligned16(logits)) return NC_ERR_ALIGNMENT;
  if (cfg->n_head / cfg->n_kv_head > 8 || (cfg->n_head / cfg->n_kv_head) & (cfg->n_head / cfg->n_kv_head - 1))
    return NC_ERR_SHAPE;  // decode attention groups of 1, 2, 4 or 8 query heads
  if (nc_status s = check_extras(cfg, w)) return s;
  if (nc_status s = device_ok()) return s;

  cudaStream_t st = S(stream);
  uint8_t* base = static_cast<uint8_t*>(session);
  uint32_t* status = reinterpret_cast<uint32_t*>(base + SL.status);
  const float* rope = reinterpret_cast<const float*>(base + SL.rope);
  const uint16_t* wqkv = reinterpret_cast<const uint16_t*>(base + SL.wqkv);
  const uint16_t* wo = reinterpret_cast<const uint16_t*>(base + SL.wo);
  const uint16_t* wfc = reinterpret_cast<const uint16_t*>(base + SL.wfc);
  const uint16_t* wmp = reinterpret_cast<const uint16_t*>(base + SL.wmp);
  const uint16_t* wlm = reinterpret_cast<const uint16_t*>(base + SL.wlm);
  uint16_t* cache = reinterpret_cast<uint16_t*>(base + SL.cache);
  float* x = reinterpret_cast<float*>(base + SL.x);
  uint16_t* a = reinterpret_cast<uint16_t*>(base + SL.a);
  uint16_t* qkv = reinterpret_cast<uint16_t*>(base + SL.qkv);
  uint16_t* o = reinterpret_cast<uint16_t*>(base + SL.o);
  uint16_t* h = reinterpret_cast<uint16_t*>(base + SL.h);
  float* part = reinterpret_cast<float*>(base + SL.part);
  float* acc = reinterpret_cast<float*>(base + SL.acc);
  const uint32_t ex = cfg->extras;
  int32_t* hist = (ex & NC_EXTRA_SMEAR) ? reinterpret_cast<int32_t*>(base + SL.hist) : nullptr;
  float* x0 = (ex & NC_EXTRA_RESID_LAMBDAS) ? reinterpret_cast<float*>(base + SL.x0) : nullptr;
  float* xmid = (ex & NC_EXTRA_BACKOUT) ? reinterpret_cast<float*>(base + SL.xmid) : nullptr;
  const int mid = cfg->n_layer / 2;  // backout: the stream after the first n_layer / 2 blocks
  const int C = cfg->d_model, D = cfg->head_dim, H = cfg->n_head, Hkv = cfg->n_kv_head, V = cfg->vocab;
  const int NQKV = (H + 2 * Hkv) * D;
  const bool f16 = cfg->act_dtype == NC_F16;
  const float eps = cfg->norm_eps;
  nc_status s;
#define NC_TRY(call)    \
  do {                  \
    s = (call);         \
    if (s != NC_OK) return s; \
  } while (0)
  if (cudaMemsetAsync(status, 0, 256, st) != cudaSuccess) return NC_ERR_CUDA;
  if (ex & (NC_EXTRA_SMEAR | NC_EXTRA_RESID_LAMBDAS))
    NC_TRY(decode_embedding_launch(tokens, hist, w->wte, hist ? w->smear_gate : nullptr, x, x0, B, C, V, T_max, pos,
                                   pos_dev, status, st));
  else
    NC_TRY(embedding_launch(tokens, w->wte, x, B, C, V, status, st));
  // Few rows (B): every projection splits K.  The residual adds land in x
  // directly; QKV and c_fc sum into an fp32 scratch that a small kernel finishes
  // (RoPE + QK-norm + cache write, or ReLU^2).  Up to 32 rows the projections
  // run on the skinny GEMM (all rows per CTA, weights streamed once); beyond,
  // on the tcgen05 GEMM with split K.
  const bool skinny = B <= 32;
  const int ks_qkv = resid_ksplit(B, NQKV, C), ks_fc = resid_ksplit(B, 4 * C, C);
  // out (+)= in . w^T over the step's B rows
  auto proj = [&](const uint16_t* in, int K, const uint16_t* wt, int N, float* out, int ks) -> nc_status {
    if (skinny) return skinny_gemm_launch(in, K, wt, K, out, N, B, N, K, 0, 0.0f, f16, st);
    EpiParams e{};
    e.out = out;
    e.ldo = N;
    e.ksplit = ks;
    return gemm_launch(in, K, wt, K, B, N, K, EPI_RESID_F32, f16, e, status, st);
  };
  for (int l = 0; l < cfg->n_layer; ++l) {
    float* keep = (xmid && l == mid) ? xmid : nullptr;
    if (x0 || keep)  // x_mid = the stream entering block `mid`; then x = a_l x + b_l x0
      NC_TRY(rmsnorm_mix_launch(x, x0, x0 ? w->resid_lambdas + l : nullptr, x0 ? w->x0_lambdas + l : nullptr, keep,
                                nullptr, nullptr, x0 != nullptr, a, B, C, eps, f16, st));
    else
      NC_TRY(rmsnorm_launch(x, a, B, C, eps, f16, st));
    uint16_t* cl = cache + l * SL.cache_layer_elems;
    if (cudaMemsetAsync(acc, 0, (size_t)B * NQKV * 4, st) != cudaSuccess) return NC_ERR_CUDA;
    NC_TRY(proj(a, C, wqkv + l * SL.wqkv_elems, NQKV, acc, ks_qkv));
    DecodeVe ve{};
    if ((ex & NC_EXTRA_VALUE_EMBED) && nc_layer_value_embed(cfg, l) == 1)
      ve = DecodeVe{tokens, w->value_embeds[l], w->ve_gates[l], V};
    NC_TRY(qkv_finish_launch(acc, qkv, cl, rope, T_max, pos, B, H, Hkv, D, T_max, eps, f16, st, pos_dev, status,
                             ve));
    NC_TRY(decode_attention_launch(qkv, NQKV, cl, part, o, B, H, Hkv, D, T_max, pos, nc_layer_window(cfg, l),
                                   f16, st, pos_dev));
    // the residual adds: partial products over K land in x (atomic or TMA
    // reduce-add, in no fixed order)
    NC_TRY(proj(o, H * D, wo + l * SL.wo_elems, C, x, resid_ksplit(B, C, H * D)));
    NC_TRY(rmsnorm_launch(x, a, B, C, eps, f16, st));
    if (cudaMemsetAsync(acc, 0, (size_t)B * 4 * C * 4, st) != cudaSuccess) return NC_ERR_CUDA;
    NC_TRY(proj(a, C, wfc + l * SL.wfc_elems, 4 * C, acc, ks_fc));
    NC_TRY(relu2_finish_launch(acc, h, (int64_t)B * 4 * C, f16, st, status));
    NC_TRY(proj(h, 4 * C, wmp + l * SL.wmp_elems, C, x, resid_ksplit(B, C, 4 * C)));
  }
  if (xmid)  // backout: x - lambda * x_mid, then the final norm
    NC_TRY(rmsnorm_mix_launch(x, nullptr, nullptr, nullptr, nullptr, xmid, w->backout_lambda, false, a, B, C, eps, f16,
                              st));
  else
    NC_TRY(rmsnorm_launch(x, a, B, C, eps, f16, st));
  if (skinny) {
    NC_TRY(skinny_gemm_launch(a, C, wlm, C, logits, V, B, V, C, 2, cfg->softcap, f16, st));
  } else {
    EpiParams ep{};
    ep.out = logits;
    ep.ldo = V;
    ep.cap = cfg->softcap;
    NC_TRY(gemm_launch(a, C, wlm, C, B, V, C, EPI_SOFTCAP_F32, f16, ep, status, st));
  }
  if (pos_dev) NC_TRY(pos_advance_launch(pos_dev, st));
#undef NC_TRY
  return NC_OK;
}

extern "C" {

nc_status nc_decode_step(const nc_config* cfg, const nc_weights* w, const int32_t* tokens, int B, int pos,
                         float* logits, void* session, size_t session_bytes, int T_max, void* stream) {
  return decode_impl(cfg, w, tokens, B, pos, nullptr, logits, session, session_bytes, T_max, stream);
}

nc_status nc_decode_step_dev(const nc_config* cfg, const nc_weights* w, const int32_t* tokens, int B,
                             int32_t* pos_dev, float* logits, void* session, size_t session_bytes, int T_max,
                             void* stream) {
  if (!pos_dev) return NC_ERR_INVALID_ARG;
  return decode_impl(cfg, w, tokens, B, 0, pos_dev, logits, session, session_bytes, T_max, stream);
}

}  // extern "C"

namespace {

// Workspace of nc_forward_backward.  Per layer l: the residual stream entering
// the block (xs[2l]) and after attention (xs[2l+1]); xs[2L] is the final
// stream.  Offsets are 256-byte aligned.
struct TrainLayout {
  size_t status, rope, wqkv, wo, wfc, wmp, wlm, xs, qkv, rstd, o, lse, h, af, a, part, tgt, tl, scal, dz, dx, dx16,
      dy, du, dO, dqkv, delta, dwqkv, x0, xpre, dx0, dxf, sdz, total;
  size_t wqkv_elems, wo_elems, wfc_elems, wmp_elems;
};

TrainLayout train_layout(const nc_config* c, int B, int T) {
  TrainLayout L;
  const size_t M = (size_t)B * T, C = c->d_model, D = c->head_dim, H = c->n_head, Hkv = c->n_kv_head,
               V = c->vocab, NL = c->n_layer;
  const size_t nqkv = (H + 2 * Hkv) * D, HD = H * D;
  L.wqkv_elems = nqkv * C;
  L.wo_elems = C * HD;
  L.wfc_elems = 4 * C * C;
  L.wmp_elems = C * 4 * C;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  L.status = take(256);
  L.rope = take((size_t)T * D * 4 * 2);  // [2][T][D/2] and the pair-major copy
  L.wqkv = take(NL * L.wqkv_elems * 2);
  L.wo = take(NL * L.wo_elems * 2);
  L.wfc = take(NL * L.wfc_elems * 2);
  L.wmp = take(NL * L.wmp_elems * 2);
  L.wlm = take(V * C * 2);
  L.xs = take((2 * NL + 1) * M * C * 4);
  L.qkv = take(NL * M * nqkv * 2);
  L.rstd = take(NL * M * (H + Hkv) * 4);
  L.o = take(NL * M * HD * 2);
  L.lse = take(NL * M * H * 4);
  L.h = take(NL * M * 4 * C * 2);
  L.af = take(M * C * 2);
  L.a = take(M * C * 2);
  L.part = take(M * (size_t)gemm_ce_partials_per_row((int)V) * 4);
  L.tgt = take(M * 4);
  L.tl = take(M * 4);
  L.scal = take(256);  // 1 / (counted targets)
  L.dz = take(M * V * 2);
  L.dx = take(M * C * 4);
  L.dx16 = take(M * C * 2);
  L.dy = take(M * C * 4);
  L.du = take(M * 4 * C * 2);
  L.dO = take(M * HD * 2);
  L.dqkv = take(M * nqkv * 2);
  L.delta = take(M * H * 4);
  L.dwqkv = take(nqkv * C * 4);
  // further forward terms: x0, each block's stream before the lambda mix and
  // the gradient collected for x0 (resid lambdas); the final-norm gradient
  // (backout); the smear gates' gradient per token
  const bool lam = c->extras & NC_EXTRA_RESID_LAMBDAS;
  L.x0 = lam ? take(M * C * 4) : 0;
  L.xpre = lam ? take(NL * M * C * 4) : 0;
  L.dx0 = lam ? take(M * C * 4) : 0;
  L.dxf = (c->extras & NC_EXTRA_BACKOUT) ? take(M * C * 4) : 0;
  L.sdz = (c->extras & NC_EXTRA_SMEAR) ? take(M * 4) : 0;
  L.total = off;
  return L;
}

}  // namespace

extern "C" {

size_t nc_train_workspace_bytes(const nc_config* cfg, int B, int T) {
  if (!config_ok(cfg) || cfg->fp8 != 0 || B < 1 || T < 1 || T > cfg->seq_len) return 0;
  return train_layout(cfg, B, T).total;
}

nc_status nc_forward_backward(const nc_config* cfg, const nc_weights* w, const int32_t* tokens,
                              const int32_t* targets, int B, int T, float* loss, const nc_grads* g,
                              void* workspace, size_t ws_bytes, void* stream) {
  return nc_forward_backward_traced(cfg, w, tokens, targets, B, T, loss, g, workspace, ws_bytes, stream, nullptr);
}

nc_status nc_forward_backward_traced(const nc_config* cfg, const nc_weights* w, const int32_t* tokens,
                                     const int32_t* targets, int B, int T, float* loss, const nc_grads* g,
                                     void* workspace, size_t ws_bytes, void* stream, nc_trace* trace) {
  if (!cfg || !w || !tokens || !targets || !loss || !g || !workspace) return NC_ERR_INVALID_ARG;
  if (!config_ok(cfg) || cfg->fp8 != 0) return NC_ERR_CONFIG;
  if (B < 1 || T < 1 || T > cfg->seq_len || (int64_t)B * T > ((int64_t)1 << 30)) return NC_ERR_SHAPE;
  const TrainLayout L = train_layout(cfg, B, T);
  if (ws_bytes < L.total) return NC_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return NC_ERR_ALIGNMENT;
  if (nc_status s = check_weights(cfg, w)) return s;
  if (nc_status s = check_extras(cfg, w)) return s;
  if (!g->wte || !g->lm_head || !g->c_q || !g->c_k || !g->c_v || !g->attn_proj || !g->c_fc || !g->mlp_proj)
    return NC_ERR_INVALID_ARG;
  {  // gradients of the further terms
    const uint32_t ex = cfg->extras;
    if ((ex & NC_EXTRA_SMEAR) && !g->smear_gate) return NC_ERR_INVALID_ARG;
    if ((ex & NC_EXTRA_RESID_LAMBDAS) && (!g->resid_lambdas || !g->x0_lambdas)) return NC_ERR_INVALID_ARG;
    if ((ex & NC_EXTRA_BACKOUT) && !g->backout_lambda) return NC_ERR_INVALID_ARG;
    if (ex & NC_EXTRA_VALUE_EMBED) {
      if (!g->value_embeds || !g->ve_gates) return NC_ERR_INVALID_ARG;
      for (int l = 0; l < cfg->n_layer; ++l)
        if (nc_layer_value_embed(cfg, l) == 1 && (!g->value_embeds[l] || !g->ve_gates[l])) return NC_ERR_INVALID_ARG;
    }
  }
  if (!aligned16(g->wte) || !aligned16(g->lm_head) || !aligned16(loss)) return NC_ERR_ALIGNMENT;
  for (int l = 0; l < cfg->n_layer; ++l) {
    const float* ps[6] = {g->c_q[l], g->c_k[l], g->c_v[l], g->attn_proj[l], g->c_fc[l], g->mlp_proj[l]};
    for (const float* p : ps) {
      if (!p) return NC_ERR_INVALID_ARG;
      if (!aligned16(p)) return NC_ERR_ALIGNMENT;
    }
  }
  if (trace) {
    const int need = 12 + 24 * cfg->n_layer;
    trace->count = need;
    if (!trace->events || trace->capacity < need) return NC_ERR_INVALID_ARG;
    for (int i = 0; i < 2 * need; ++i)
      if (!trace->events[i]) return NC_ERR_INVALID_ARG;
  }
  if (nc_status s = device_ok()) return s;

  cudaStream_t st = S(stream);
  Tracer tr{trace, st, 0, false};
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int M = B * T, NL = cfg->n_layer;
  const int C = cfg->d_model, D = cfg->head_dim, H = cfg->n_head, Hkv = cfg->n_kv_head, V = cfg->vocab;
  const int NQKV = (H + 2 * Hkv) * D, HD = H * D;
  const bool f16 = cfg->act_dtype == NC_F16;
  const float eps = cfg->norm_eps;
  const size_t MC = (size_t)M * C;
  uint32_t* status = reinterpret_cast<uint32_t*>(ws + L.status);
  float* rope = reinterpret_cast<float*>(ws + L.rope);
  uint16_t* wqkv = reinterpret_cast<uint16_t*>(ws + L.wqkv);
  uint16_t* wo = reinterpret_cast<uint16_t*>(ws + L.wo);
  uint16_t* wfc = reinterpret_cast<uint16_t*>(ws + L.wfc);
  uint16_t* wmp = reinterpret_cast<uint16_t*>(ws + L.wmp);
  uint16_t* wlm = reinterpret_cast<uint16_t*>(ws + L.wlm);
  float* xs = reinterpret_cast<float*>(ws + L.xs);
  auto qkv_l = [&](int l) { return reinterpret_cast<uint16_t*>(ws + L.qkv) + (size_t)l * M * NQKV; };
  auto rstd_l = [&](int l) { return reinterpret_cast<float*>(ws + L.rstd) + (size_t)l * M * (H + Hkv); };
  auto o_l = [&](int l) { return reinterpret_cast<uint16_t*>(ws + L.o) + (size_t)l * M * HD; };
  auto lse_l = [&](int l) { return reinterpret_cast<float*>(ws + L.lse) + (size_t)l * M * H; };
  auto h_l = [&](int l) { return reinterpret_cast<uint16_t*>(ws + L.h) + (size_t)l * M * 4 * C; };
  uint16_t* af = reinterpret_cast<uint16_t*>(ws + L.af);
  uint16_t* a = reinterpret_cast<uint16_t*>(ws + L.a);
  float* part = reinterpret_cast<float*>(ws + L.part);
  float* tgt = reinterpret_cast<float*>(ws + L.tgt);
  float* tl = reinterpret_cast<float*>(ws + L.tl);
  float* inv = reinterpret_cast<float*>(ws + L.scal);
  uint16_t* dz = reinterpret_cast<uint16_t*>(ws + L.dz);
  float* dx = reinterpret_cast<float*>(ws + L.dx);
  uint16_t* dx16 = reinterpret_cast<uint16_t*>(ws + L.dx16);
  float* dy = reinterpret_cast<float*>(ws + L.dy);
  uint16_t* du = reinterpret_cast<uint16_t*>(ws + L.du);
  uint16_t* dO = reinterpret_cast<uint16_t*>(ws + L.dO);
  uint16_t* dqkv = reinterpret_cast<uint16_t*>(ws + L.dqkv);
  float* delta = reinterpret_cast<float*>(ws + L.delta);
  float* dwqkv = reinterpret_cast<float*>(ws + L.dwqkv);
  const uint32_t ex = cfg->extras;
  float* x0 = (ex & NC_EXTRA_RESID_LAMBDAS) ? reinterpret_cast<float*>(ws + L.x0) : nullptr;
  auto xpre_l = [&](int l) { return reinterpret_cast<float*>(ws + L.xpre) + (size_t)l * MC; };
  float* dx0 = x0 ? reinterpret_cast<float*>(ws + L.dx0) : nullptr;
  float* dxf = (ex & NC_EXTRA_BACKOUT) ? reinterpret_cast<float*>(ws + L.dxf) : nullptr;
  const int mid = NL / 2;  // backout: the stream entering block `mid`, before its lambda mix
  const float* x_back = dxf ? (x0 ? xpre_l(mid) : xs + (size_t)(2 * mid) * MC) : nullptr;

  nc_status s = NC_OK;
#define NC_RUN(kind, call)                   \
  do {                                       \
    if (!tr.begin(kind)) return NC_ERR_CUDA; \
    s = (call);                              \
    if (s != NC_OK) return s;                \
    if (!tr.end()) return NC_ERR_CUDA;       \
  } while (0)
  auto copy = [&](float* dst, const float* src) -> nc_status {
    return cudaMemcpyAsync(dst, src, MC * 4, cudaMemcpyDeviceToDevice, st) == cudaSuccess ? NC_OK : NC_ERR_CUDA;
  };
  // ---------------- forward, keeping what the backward reads
  if (cudaMemsetAsync(status, 0, 256, st) != cudaSuccess) return NC_ERR_CUDA;
  NC_RUN(NC_K_ROPE_TABLE, rope_table_launch(rope, T, D, cfg->rope_base, st, rope_pairs_of(rope, T, D)));
  NC_RUN(NC_K_CAST, launch_weight_cast(cfg, w, wqkv, wo, wfc, wmp, wlm, L.wqkv_elems, L.wo_elems, L.wfc_elems, L.wmp_elems,
                            f16, st));
  if (ex & (NC_EXTRA_SMEAR | NC_EXTRA_RESID_LAMBDAS))
    NC_RUN(NC_K_EMBEDDING, embedding_extra_launch(tokens, w->wte, (ex & NC_EXTRA_SMEAR) ? w->smear_gate : nullptr,
                                                  xs, x0, M, C, V, T, status, st));
  else
    NC_RUN(NC_K_EMBEDDING, embedding_launch(tokens, w->wte, xs, M, C, V, status, st));
  for (int l = 0; l < NL; ++l) {
    float* xin = xs + (size_t)(2 * l) * MC;
    float* xmid = xin + MC;
    float* xnext = xmid + MC;
    if (x0)  // x = resid_lambda x + x0_lambda x0 in place, the stream before it kept
      NC_RUN(NC_K_RMSNORM, rmsnorm_mix_launch(xin, x0, w->resid_lambdas + l, w->x0_lambdas + l, xpre_l(l), nullptr,
                                              nullptr, true, a, M, C, eps, f16, st));
    else
      NC_RUN(NC_K_RMSNORM, rmsnorm_launch(xin, a, M, C, eps, f16, st));
    EpiParams eq{};
    eq.out = qkv_l(l);
    eq.ldo = NQKV;
    eq.rope = rope;
    eq.T = T;
    eq.H = H;
    eq.Hkv = Hkv;
    eq.D = D;
    eq.eps = eps;
    eq.rope_T = T;
    eq.rope_pairs = rope_pairs_of(rope, T, D);
    eq.rstd_out = rstd_l(l);
    const bool ve_on = (ex & NC_EXTRA_VALUE_EMBED) && nc_layer_value_embed(cfg, l) == 1;
    if (ve_on) {  // v + gate * ve[token] in the epilogue
      eq.tokens = tokens;
      eq.ve = w->value_embeds[l];
      eq.ve_gate = w->ve_gates[l];
      eq.V = V;
    }
    NC_RUN(NC_K_GEMM_QKV, gemm_launch(a, C, wqkv + l * L.wqkv_elems, C, M, NQKV, C, EPI_QKV_ROPE_IL, f16, eq, status, st));
    uint16_t* q = qkv_l(l);
    NC_RUN(NC_K_ATTENTION, attention_launch(q, q + HD, q + (H + Hkv) * D, o_l(l), B, T, H, Hkv, D, nc_layer_window(cfg, l), NQKV,
                            NQKV, f16, status, st, nullptr, lse_l(l)));
    NC_RUN(NC_K_COPY, copy(xmid, xin));
    EpiParams ep{};
    ep.out = xmid;
    ep.ldo = C;
    NC_RUN(NC_K_GEMM_ATTN_PROJ, gemm_launch(o_l(l), HD, wo + l * L.wo_elems, HD, M, C, HD, EPI_RESID_F32, f16, ep, status, st));
    NC_RUN(NC_K_RMSNORM, rmsnorm_launch(xmid, a, M, C, eps, f16, st));
    ep.out = h_l(l);
    ep.ldo = 4 * C;
    NC_RUN(NC_K_GEMM_FC, gemm_launch(a, C, wfc + l * L.wfc_elems, C, M, 4 * C, C, EPI_RELU2_16, f16, ep, status, st));
    NC_RUN(NC_K_COPY, copy(xnext, xmid));
    ep.out = xnext;
    ep.ldo = C;
    NC_RUN(NC_K_GEMM_MLP_PROJ, gemm_launch(h_l(l), 4 * C, wmp + l * L.wmp_elems, 4 * C, M, C, 4 * C, EPI_RESID_F32, f16, ep, status,
                       st));
  }
  float* xf = xs + (size_t)(2 * NL) * MC;
  if (x_back)  // x -= backout_lambda x_back in place
    NC_RUN(NC_K_RMSNORM, rmsnorm_mix_launch(xf, nullptr, nullptr, nullptr, nullptr, x_back, w->backout_lambda, true,
                                            af, M, C, eps, f16, st));
  else
    NC_RUN(NC_K_RMSNORM, rmsnorm_launch(xf, af, M, C, eps, f16, st));
  {
    EpiParams ep{};
    ep.ldo = V;
    ep.cap = cfg->softcap;
    ep.ce_partial = part;
    ep.ce_target = tgt;
    ep.targets = targets;
    NC_RUN(NC_K_GEMM_LM_HEAD, gemm_launch(af, C, wlm, C, M, V, C, EPI_CE_PARTIAL, f16, ep, status, st));
    NC_RUN(NC_K_CE_FINALIZE, ce_finalize_launch(part, gemm_ce_partials_per_row(V), tgt, targets, tl, M, V, cfg->softcap, status, st));
    NC_RUN(NC_K_LOSS_MEAN, loss_mean_launch(tl, targets, M, V, loss, st, inv));
  }

  // ---------------- backward (gradients of the summed token loss; weight
  // gradients take the factor 1 / count from `inv`)
  auto wgrad = [&](const uint16_t* dyt, int64_t ld_dy, const uint16_t* xt, int64_t ld_x, int No, int Ko, float* out,
                   int64_t ldo) -> nc_status {  // out [No, Ko] += inv * dyt^T xt, over the M tokens
    EpiParams e{};
    e.out = out;
    e.ldo = ldo;
    e.alpha_ptr = inv;
    const int tiles = ((No + 127) / 128) * ((Ko + 255) / 256);
    const int nkb = (M + 63) / 64;
    int ks = (8 * device_sm_count() + tiles - 1) / tiles;
    ks = std::min(ks, std::max(1, nkb / 16));
    e.ksplit = std::max(ks, 1);
    return gemm_launch_layout(dyt, ld_dy, xt, ld_x, No, Ko, M, EPI_RESID_F32, f16, GEMM_TN, e, status, st);
  };
  auto dgrad = [&](const uint16_t* dyt, int K, const uint16_t* wt, int N, int epi, void* out,
                   const uint16_t* aux = nullptr) -> nc_status {  // out [M, N] = dyt [M, K] . wt [K, N]
    EpiParams e{};
    e.out = out;
    e.ldo = N;
    e.aux = aux;
    e.ld_aux = N;
    return gemm_launch_layout(dyt, K, wt, N, M, N, K, epi, f16, GEMM_NN, e, status, st);
  };
  {
    EpiParams ep{};
    ep.out = dz;
    ep.ldo = V;
    ep.cap = cfg->softcap;
    ep.targets = targets;
    ep.row_lse = tl;
    ep.ce_target = tgt;
    NC_RUN(NC_K_CE_BWD, gemm_launch(af, C, wlm, C, M, V, C, EPI_CE_BWD_16, f16, ep, status, st));
  }
  NC_RUN(NC_K_GEMM_WGRAD, wgrad(dz, V, af, C, V, C, g->lm_head, C));
  NC_RUN(NC_K_GEMM_DGRAD, dgrad(dz, V, wlm, C, EPI_STORE_F32, dy));
  NC_RUN(NC_K_NORM_BWD, rmsnorm_bwd_launch(xf, dy, dx, dx16, M, C, eps, false, f16, st));
  // The further terms' backward launches are not recorded in the trace.
#define NC_TRY_EX(call)                     \
  do {                                      \
    s = (call);                             \
    if (s != NC_OK) return s;               \
  } while (0)
  if (x_back) {  // x_final = x_L - lambda x_back: dlambda = -sum dx . x_back; keep dx_final
    NC_TRY_EX(dots_launch(dx, x_back, nullptr, (int64_t)MC, inv, -1.0f, g->backout_lambda, nullptr, st));
    NC_TRY_EX(cudaMemcpyAsync(dxf, dx, MC * 4, cudaMemcpyDeviceToDevice, st) == cudaSuccess ? NC_OK : NC_ERR_CUDA);
  }
  if (dx0) NC_TRY_EX(cudaMemsetAsync(dx0, 0, MC * 4, st) == cudaSuccess ? NC_OK : NC_ERR_CUDA);
  for (int l = NL - 1; l >= 0; --l) {
    float* xin = xs + (size_t)(2 * l) * MC;
    float* xmid = xin + MC;
    // MLP
    NC_RUN(NC_K_GEMM_WGRAD, wgrad(dx16, C, h_l(l), 4 * C, C, 4 * C, g->mlp_proj[l], 4 * C));
    NC_RUN(NC_K_GEMM_DGRAD, dgrad(dx16, C, wmp + l * L.wmp_elems, 4 * C, EPI_RELU2_BWD_16, du, h_l(l)));
    NC_RUN(NC_K_RMSNORM, rmsnorm_launch(xmid, a, M, C, eps, f16, st));
    NC_RUN(NC_K_GEMM_WGRAD, wgrad(du, 4 * C, a, C, 4 * C, C, g->c_fc[l], C));
    NC_RUN(NC_K_GEMM_DGRAD, dgrad(du, 4 * C, wfc + l * L.wfc_elems, C, EPI_STORE_F32, dy));
    NC_RUN(NC_K_NORM_BWD, rmsnorm_bwd_launch(xmid, dy, dx, dx16, M, C, eps, true, f16, st));
    // attention block
    NC_RUN(NC_K_GEMM_WGRAD, wgrad(dx16, C, o_l(l), HD, C, HD, g->attn_proj[l], HD));
    NC_RUN(NC_K_GEMM_DGRAD, dgrad(dx16, C, wo + l * L.wo_elems, HD, EPI_STORE_16, dO));
    NC_RUN(NC_K_ATTN_BWD, attn_bwd_launch(qkv_l(l), NQKV, o_l(l), dO, lse_l(l), delta, dqkv, B, T, H, Hkv, D,
                           nc_layer_window(cfg, l), f16, st, status));
    NC_RUN(NC_K_QK_BWD, qk_bwd_launch(dqkv, qkv_l(l), NQKV, rstd_l(l), rope, T, M, T, H, Hkv, D, f16, st));
    if ((ex & NC_EXTRA_VALUE_EMBED) && nc_layer_value_embed(cfg, l) == 1)  // v + gate ve[token]
      NC_TRY_EX(ve_bwd_launch(dqkv, NQKV, tokens, w->value_embeds[l], w->ve_gates[l], g->value_embeds[l],
                              g->ve_gates[l], M, H, Hkv, D, V, inv, f16, st));
    NC_RUN(NC_K_RMSNORM, rmsnorm_launch(xin, a, M, C, eps, f16, st));
    NC_RUN(NC_K_GEMM_WGRAD, cudaMemsetAsync(dwqkv, 0, (size_t)NQKV * C * 4, st) == cudaSuccess
                                ? wgrad(dqkv, NQKV, a, C, NQKV, C, dwqkv, C)
                                : NC_ERR_CUDA);
    NC_RUN(NC_K_EMB_BWD, qkv_grad_scatter_launch(dwqkv, g->c_q[l], g->c_k[l], g->c_v[l], H, Hkv, D, C, 1.0f, st));
    NC_RUN(NC_K_GEMM_DGRAD, dgrad(dqkv, NQKV, wqkv + l * L.wqkv_elems, C, EPI_STORE_F32, dy));
    NC_RUN(NC_K_NORM_BWD, rmsnorm_bwd_launch(xin, dy, dx, dx16, M, C, eps, true, f16, st));
    // dx: of the block's (mixed) input
    if (x0)  // x_in = resid_lambda x_pre + x0_lambda x0
      NC_TRY_EX(dots_launch(dx, xpre_l(l), x0, (int64_t)MC, inv, 1.0f, g->resid_lambdas + l, g->x0_lambdas + l, st));
    const bool back_here = x_back && l == mid;  // x_pre of block `mid` also enters the final norm
    if (x0 || back_here)
      NC_TRY_EX(mix_bwd_launch(dx, dx0, back_here ? dxf : nullptr, nullptr, x0 ? w->resid_lambdas + l : nullptr,
                               x0 ? w->x0_lambdas + l : nullptr, back_here ? w->backout_lambda : nullptr, dx16,
                               (int64_t)MC, f16, st));
  }
  if (dx0) NC_TRY_EX(mix_bwd_launch(dx, nullptr, nullptr, dx0, nullptr, nullptr, nullptr, nullptr, (int64_t)MC, f16, st));
  const float* demb = dx;
  if (ex & NC_EXTRA_SMEAR) {  // x_t = e_t + sigmoid(e_t . w) e_{t-1}
    NC_TRY_EX(smear_bwd_launch(tokens, w->wte, w->smear_gate, dx, dy, reinterpret_cast<float*>(ws + L.sdz),
                               g->smear_gate, M, T, C, V, inv, st));
    demb = dy;
  }
  NC_RUN(NC_K_EMB_BWD, embedding_bwd_launch(tokens, demb, g->wte, M, C, V, inv, st));
#undef NC_TRY_EX
#undef NC_RUN
  return NC_OK;
}

nc_status nc_selftest_bounded_wait(uint32_t* dev_status, uint32_t limit_us, void* stream) {
  if (!dev_status || limit_us < 1 || limit_us > 2000000u) return NC_ERR_INVALID_ARG;
  if (nc_status s = device_ok()) return s;
  return selftest_wait_launch(dev_status, (uint64_t)limit_us * 1000ull, S(stream));
}

nc_status nc_event_create(void** event) {
  if (!event) return NC_ERR_INVALID_ARG;
  cudaEvent_t e;
  if (cudaEventCreate(&e) != cudaSuccess) return NC_ERR_CUDA;
  *event = e;
  return NC_OK;
}

nc_status nc_event_destroy(void* event) {
  if (!event) return NC_ERR_INVALID_ARG;
  return cudaEventDestroy(static_cast<cudaEvent_t>(event)) == cudaSuccess ? NC_OK : NC_ERR_CUDA;
}

nc_status nc_stream_wait_event(void* stream, void* event) {
  if (!event) return NC_ERR_INVALID_ARG;
  return cudaStreamWaitEvent(S(stream), static_cast<cudaEvent_t>(event), 0) == cudaSuccess ? NC_OK : NC_ERR_CUDA;
}

nc_status nc_event_elapsed_ms(void* start, void* end, float* ms) {
  if (!start || !end || !ms) return NC_ERR_INVALID_ARG;
  if (cudaEventSynchronize(static_cast<cudaEvent_t>(end)) != cudaSuccess) return NC_ERR_CUDA;
  return cudaEventElapsedTime(ms, static_cast<cudaEvent_t>(start), static_cast<cudaEvent_t>(end)) ==
                 cudaSuccess
             ? NC_OK
             : NC_ERR_CUDA;
}

}  // extern "C"
