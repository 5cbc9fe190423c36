/*
 * nc.h -- C ABI of the B200 (sm_100a) forward pass + loss of the nanochat GPT
 * block stack.
 *
 * What is computed (page title, section):
 *   "从文本到聊天模型" (onehacker.top) §5: token embedding (§5.2), blocks
 *   x = x + attn(norm(x)); x = x + mlp(norm(x)) (§5.3), separate c_q/c_k/c_v
 *   projections with Q (B,T,H,D) and K/V (B,T,Hkv,D) (§5.4), causal attention
 *   (§5.5), RoPE (§5.6), ReLU^2 MLP C -> 4C -> C (§5.7), LM head and token
 *   cross-entropy with ignore_index = -1 (§5.8);
 *   "Nanochat与nanoGPT对比：关键升级" (lzwjava.github.io) §1: parameter-free
 *   RMSNorm, QK-norm after RoPE, GQA, no biases, untied lm_head, tanh logit
 *   soft-cap at +-15, SSSL sliding window (last layer full), final norm before
 *   the logit projection;
 *   nanochat README mirror (dev.wehub.plus), "精度 / dtype": weights are kept
 *   in fp32 and cast to bf16 at matmul time.
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers of the current CUDA device unless
 *     a parameter says "host".  The caller owns every buffer; the library
 *     allocates no device memory and frees nothing.
 *   - 16-bit tensors are uint16_t* holding bfloat16 or IEEE fp16 bit patterns, as
 *     the call's nc_dtype argument says.
 *   - Matrices are row-major.  Weights use the [out_features, in_features]
 *     layout of a bias-free linear layer, so y = x W^T.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Work is
 *     enqueued asynchronously; results are valid once the stream has synchronised.
 *   - Arguments are checked on the host before anything is enqueued; a failed
 *     check returns an error code and enqueues nothing.  Nothing aborts, traps
 *     or prints.
 *   - Device-detected conditions (a token id outside [0, V), a target outside
 *     {-1} U [0, V), a bounded wait inside a kernel that ran out) are OR-ed into
 *     a caller-provided 32-bit device status word as NC_DEV_* bits; kernels
 *     clamp indices so that no out-of-bounds access happens.  Pass NULL to
 *     ignore them.  nc_get_status() turns a status word into an nc_status.
 *   - Pointers must be 16-byte aligned (NC_ERR_ALIGNMENT otherwise).
 *   - Every entry point requires an sm_100 device (NC_ERR_UNSUPPORTED_DEVICE).
 */
#ifndef NC_H_
#define NC_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  NC_OK = 0,
  NC_ERR_INVALID_ARG = 1,        /* NULL pointer, negative size, bad enum */
  NC_ERR_CONFIG = 2,             /* inconsistent nc_config                   */
  NC_ERR_SHAPE = 3,              /* sizes the kernels do not support         */
  NC_ERR_ALIGNMENT = 4,          /* a pointer is not 16-byte aligned         */
  NC_ERR_WORKSPACE = 5,          /* workspace smaller than nc_workspace_bytes */
  NC_ERR_TOKEN_RANGE = 6,        /* device: token or target id out of range  */
  NC_ERR_TIMEOUT = 7,            /* device: a bounded wait in a kernel ran out */
  NC_ERR_UNSUPPORTED_DEVICE = 8, /* current device is not sm_100             */
  NC_ERR_CUDA = 9,               /* a CUDA runtime call failed               */
  NC_ERR_F16_RANGE = 10          /* device: a value stored as fp16 exceeded
                                    +-65504 and was saturated               */
} nc_status;

/* 16-bit storage formats. */
typedef enum {
  NC_BF16 = 0, /* bfloat16: 8 significant bits, fp32 range                     */
  NC_F16 = 1,  /* IEEE binary16: 11 significant bits, |x| <= 65504 (saturating) */
  NC_F32 = 2   /* fp32: accepted only as the source of nc_fp8_quantize          */
} nc_dtype;

/* Bits of the device status word. */
#define NC_DEV_TOKEN_RANGE 0x1u  /* a token id was outside [0, V): row 0 used  */
#define NC_DEV_TARGET_RANGE 0x2u /* a target was outside {-1} U [0, V): ignored */
#define NC_DEV_TIMEOUT 0x4u      /* a pipeline wait gave up; outputs invalid   */
#define NC_DEV_SMEM_ALIGN 0x8u   /* a kernel's shared-memory window was not 1024-byte
                                    aligned; it did nothing (reported as NC_ERR_CUDA) */
#define NC_DEV_F16_RANGE 0x20u   /* a projection output stored in fp16 (act_dtype
                                    NC_F16) exceeded +-65504 and was saturated to it
                                    (reported as NC_ERR_F16_RANGE) */
#define NC_DEV_POSITION 0x10u    /* nc_decode_step_dev read a position outside
                                    [0, T_max): nothing was written to the cache and
                                    the step's logits are invalid (reported as
                                    NC_ERR_SHAPE) */

/* Further terms of the full nanochat forward ("Nanochat与nanoGPT对比" §1,
 * architecture table and notes); bits of nc_config.extras.  Each reads its
 * weights from nc_weights.  The pages give one line per term; the readings
 * taken are stated here. */
#define NC_EXTRA_SMEAR 0x1u         /* after the embedding lookup:
                                       x_t = e_t + sigmoid(gate . e_t) e_{t-1}, position 0 of each
                                       row unchanged; gate is a bias-free linear map C -> 1 whose
                                       fp32 weight enters as bf16 like every linear weight       */
#define NC_EXTRA_VALUE_EMBED 0x2u   /* on every other layer counted back from the last (which
                                       always has one): v += gate[g] * table[token][g*D .. g*D+D)
                                       for kv head g, added to the v projection                   */
#define NC_EXTRA_RESID_LAMBDAS 0x4u /* before block l: x = resid_lambdas[l] x + x0_lambdas[l] x0,
                                       x0 the (smeared) embedding output                          */
#define NC_EXTRA_BACKOUT 0x8u       /* before the final norm: x -= backout_lambda * x_mid, x_mid
                                       the stream after the first n_layer / 2 blocks (before block
                                       n_layer / 2 mixes in x0)                                   */
#define NC_EXTRA_ALL 0xFu

/* nc_config.fp8: dynamic tensorwise FP8 ("Nanochat与nanoGPT对比：关键升级" §1,
 * architecture table, FP8-training row).  Each operand of a chosen matrix
 * product -- the activation entering it and the fp32 master weight -- is
 * quantised as a whole tensor: amax = max |x|, s = 448 / max(amax, 1e-12) in
 * fp32, codes = e4m3(x * s) rounded to nearest even and saturated at +-448; the
 * fp32 product of the codes is multiplied by 1 / (s_a s_w). */
#define NC_FP8_BLOCK 0x1u   /* the six block projections c_q, c_k, c_v, attention
                               c_proj, c_fc, MLP c_proj                          */
#define NC_FP8_LM_HEAD 0x2u /* the LM head                                       */
#define NC_FP8_ALL 0x3u

/* Model configuration.  "从文本到聊天模型" §5.1: d_model = depth * aspect_ratio,
 * n_head = d_model / head_dim.  window_pattern: one char per layer, cycled;
 * 'S' = short window (short_window keys), 'L' = full context; the last layer is
 * always 'L' ("Nanochat与nanoGPT对比" §1, sliding-window note). */
typedef struct {
  int32_t n_layer;
  int32_t d_model;
  int32_t n_head;
  int32_t n_kv_head;         /* n_head % n_kv_head == 0 (GQA groups)          */
  int32_t head_dim;          /* 64 or 128                                     */
  int32_t vocab;             /* multiple of 64                                */
  int32_t seq_len;           /* maximum T                                     */
  int32_t short_window;      /* keys visible in 'S' layers (seq_len / 4)      */
  char window_pattern[8];    /* NUL-terminated, e.g. "SSSL"                   */
  float softcap;             /* logits = softcap * tanh(z / softcap), 15      */
  float norm_eps;            /* RMSNorm epsilon, 1e-6                         */
  float rope_base;           /* RoPE base, 10000                              */
  int32_t act_dtype;         /* nc_dtype of activations and matmul operands:
                                NC_F16 (default) or NC_BF16.  Weights always
                                enter the matmuls as their bf16 (round to
                                nearest even) values; with NC_F16 those values
                                are held in fp16 (exact for |w| >= 2^-14) so
                                both tensor-core operands share one format. */
  uint32_t extras;           /* NC_EXTRA_* bits (0: the plain block stack)    */
  uint32_t fp8;              /* NC_FP8_* bits (0: every product in 16-bit)    */
} nc_config;

/* fp32 master weights (device pointers; the per-layer members are HOST arrays
 * of n_layer device pointers).  Read only. */
typedef struct {
  const float* wte;                  /* [V, C]                                */
  const float* const* c_q;           /* n_layer x [H*D, C]                    */
  const float* const* c_k;           /* n_layer x [Hkv*D, C]                  */
  const float* const* c_v;           /* n_layer x [Hkv*D, C]                  */
  const float* const* attn_proj;     /* n_layer x [C, H*D]                    */
  const float* const* c_fc;          /* n_layer x [4C, C]                     */
  const float* const* mlp_proj;      /* n_layer x [C, 4C]                     */
  const float* lm_head;              /* [V, C]                                */
  /* Read only for the terms enabled in nc_config.extras (may be NULL otherwise). */
  const float* smear_gate;           /* [C]                NC_EXTRA_SMEAR      */
  const float* const* value_embeds;  /* n_layer x [V, Hkv*D] fp32, and        */
  const float* const* ve_gates;      /* n_layer x [Hkv]: NC_EXTRA_VALUE_EMBED;
                                        entries of layers without a value
                                        embedding are not read (may be NULL)   */
  const float* resid_lambdas;        /* [n_layer]          NC_EXTRA_RESID_LAMBDAS */
  const float* x0_lambdas;           /* [n_layer]          NC_EXTRA_RESID_LAMBDAS */
  const float* backout_lambda;       /* [1]                NC_EXTRA_BACKOUT    */
} nc_weights;

/* ---------------------------------------------------------------- host-only */

/* Fills *out from the depth knob ("从文本到聊天模型" §5.1): d_model =
 * depth*aspect_ratio, n_head = d_model/head_dim, n_kv_head = n_kv_head or
 * n_head when 0, pattern "SSSL", short_window = seq_len/4, softcap 15,
 * norm_eps 1e-6, rope_base 10000, act_dtype NC_F16, extras 0, fp8 0.  Host only; touches no
 * device. */
nc_status nc_init_config(nc_config* out, int depth, int aspect_ratio, int head_dim,
                         int n_kv_head, int seq_len, int vocab);

/* Checks a configuration (NC_OK or NC_ERR_CONFIG).  Host only. */
nc_status nc_check_config(const nc_config* cfg);

/* Number of keys layer `layer` lets each query see (short_window or seq_len),
 * or -1 for a bad argument.  Host only. */
int nc_layer_window(const nc_config* cfg, int layer);

/* 1 if layer `layer` carries a value embedding under NC_EXTRA_VALUE_EMBED
 * (every other layer counted back from the last), 0 if not, -1 for a bad
 * argument.  Host only. */
int nc_layer_value_embed(const nc_config* cfg, int layer);

/* Bytes of workspace nc_forward needs for a [B, T] batch (0 on bad input); the
 * extras NC_EXTRA_RESID_LAMBDAS and NC_EXTRA_BACKOUT each add one fp32 [B*T, C]
 * stream.  Host only. */
size_t nc_workspace_bytes(const nc_config* cfg, int B, int T);

/* Algorithmic FLOPs of one forward over [B, T] tokens: 2 per multiply-add of
 * every projection and of attention counted only over visible keys.  Host only. */
double nc_forward_flops(const nc_config* cfg, int B, int T);

/* Human-readable name of a status code (static string). */
const char* nc_status_string(nc_status s);

/* Library ABI version (major*100 + minor). */
int nc_version(void);

/* ---------------------------------------------------------------- forward */

/* Whole forward + loss.
 *   tokens   [B, T] int32 (device), ids in [0, V).
 *   targets  [B, T] int32 (device) or NULL; -1 = ignored position.
 *   logits   [B, T, V] fp32 (device) or NULL: soft-capped logits.
 *   token_loss [B, T] fp32 (device) or NULL: NLL per position, 0 where ignored.
 *   loss     1 fp32 (device) or NULL: mean NLL over non-ignored targets (NaN if
 *            none).  token_loss/loss need targets.
 *   workspace/ws_bytes: device scratch of at least nc_workspace_bytes(cfg,B,T)
 *            bytes, 256-byte aligned.  Its first 4 bytes are the device status
 *            word of this call (cleared at the start of the call).
 * T <= seq_len.  Asynchronous on `stream`; poll errors with nc_get_status. */
nc_status nc_forward(const nc_config* cfg, const nc_weights* w, const int32_t* tokens,
                     const int32_t* targets, int B, int T, float* logits, float* token_loss,
                     float* loss, void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------- KV-cache inference */

/* "从文本到聊天模型" §10.1-10.4: the prompt runs once (prefill) and its keys
 * and values are kept per layer; each further token then runs the stack on one
 * position per row (decode) and attends over the kept keys instead of the
 * whole prefix.  The state between calls is one caller-owned device buffer,
 * the session:
 *   the 16-bit weights (cast once by nc_prefill from the fp32 weights),
 *   the RoPE table for T_max positions,
 *   the cache of every layer, [B][T_max][2][Hkv][D] 16-bit -- per row and
 *     position the k heads after RoPE and QK-norm (in the library's internal
 *     head-dimension order) then the v heads,
 *   with NC_EXTRA_SMEAR, the token id of every position [B][T_max] int32 (a
 *     step's smear mixes in the embedding of the previous position's token),
 *   the scratch of one decode step (with NC_EXTRA_RESID_LAMBDAS / _BACKOUT
 *     also the step's x0 and x_mid rows), and the device status word (first
 *     4 bytes, cleared by every call).
 * The KV-cache path computes in 16-bit: cfg->fp8 must be 0 (NC_ERR_CONFIG
 * otherwise).  Every term of cfg->extras is supported; its parameters in `w`
 * follow nc_forward's rules (NC_ERR_INVALID_ARG / NC_ERR_ALIGNMENT).  Decode
 * attention needs n_head / n_kv_head in {1, 2, 4, 8} (NC_ERR_SHAPE otherwise).
 * T_max <= cfg->seq_len. */

/* Session bytes for B rows of up to T_max positions (0 on bad input).  Host only. */
size_t nc_session_bytes(const nc_config* cfg, int B, int T_max);

/* Scratch bytes nc_prefill needs for a [B, T] prompt (the forward's workspace
 * without the weight copy, which lives in the session).  Host only. */
size_t nc_prefill_workspace_bytes(const nc_config* cfg, int B, int T);

/* Runs the forward over tokens [B, T] (device int32), casts the weights into
 * the session and stores positions [0, T) of every layer's cache.  logits
 * [B, T, V] fp32 (device) or NULL: the soft-capped logits of every position.
 * session: nc_session_bytes(cfg, B, T_max) bytes, 256-byte aligned;
 * workspace: nc_prefill_workspace_bytes(cfg, B, T) bytes, 256-byte aligned.
 * Asynchronous on `stream`. */
nc_status nc_prefill(const nc_config* cfg, const nc_weights* w, const int32_t* tokens, int B, int T,
                     float* logits, void* session, size_t session_bytes, int T_max, void* workspace,
                     size_t ws_bytes, void* stream);

/* One decode step: tokens [B] (device int32) are the tokens at position `pos`
 * of every row (0 <= pos < T_max); the session must hold positions [0, pos) of
 * the same rows (nc_prefill of T = pos tokens, then one step per further
 * position) and the weights cast from the same `w`, whose fp32 wte this step
 * reads.  Stores position pos of every layer's cache and writes logits [B, V]
 * fp32 (device, 16-byte aligned): the soft-capped logits at position pos,
 * equal to those of nc_forward over the whole prefix.  Asynchronous on
 * `stream`. */
nc_status nc_decode_step(const nc_config* cfg, const nc_weights* w, const int32_t* tokens, int B, int pos,
                         float* logits, void* session, size_t session_bytes, int T_max, void* stream);

/* nc_decode_step with the position in device memory: *pos_dev (one int32,
 * 16-byte aligned) is read by the step's kernels and advanced by one at the
 * end of the step, so the whole step can be captured
 * once in a CUDA graph and replayed for every further position.  The
 * attention then runs on a fixed grid of 32 chunks of 64 keys, which needs
 * T_max <= 2048 (NC_ERR_SHAPE otherwise); pos_dev misaligned: NC_ERR_ALIGNMENT.
 * A position outside [0, T_max) (the cache is full) is caught on the device:
 * the step writes nothing to the cache, its logits are invalid, and the
 * session's status word gets NC_DEV_POSITION (nc_get_status on the session
 * then returns NC_ERR_SHAPE).
 * The other rules are nc_decode_step's. */
nc_status nc_decode_step_dev(const nc_config* cfg, const nc_weights* w, const int32_t* tokens, int B,
                             int32_t* pos_dev, float* logits, void* session, size_t session_bytes, int T_max,
                             void* stream);

/* Kinds of kernel launch reported by nc_forward_traced. */
typedef enum {
  NC_K_ROPE_TABLE = 0,
  NC_K_CAST = 1,
  NC_K_EMBEDDING = 2,
  NC_K_RMSNORM = 3,
  NC_K_GEMM_QKV = 4,
  NC_K_ROPE_QKNORM = 5,
  NC_K_ATTENTION = 6,
  NC_K_GEMM_ATTN_PROJ = 7,
  NC_K_GEMM_FC = 8,
  NC_K_GEMM_MLP_PROJ = 9,
  NC_K_GEMM_LM_HEAD = 10,
  NC_K_CE_FINALIZE = 11,
  NC_K_LOSS_MEAN = 12,
  NC_K_FP8_QUANT = 13,  /* e4m3 quantisation of one activation (+ its amax when no producer folded it) */
  NC_K_COPY = 14,       /* residual-stream snapshot of the training forward (device copy) */
  NC_K_CE_BWD = 15,     /* logit gradient: lm_head recomputed, soft-cap + CE backward epilogue */
  NC_K_GEMM_DGRAD = 16, /* dX = dY W (tcgen05, W as the MN-major operand) */
  NC_K_GEMM_WGRAD = 17, /* dW += dY^T X over the tokens (tcgen05, both operands MN-major) */
  NC_K_NORM_BWD = 18,   /* RMSNorm backward into the residual gradient */
  NC_K_ATTN_BWD = 19,   /* attention backward: Delta, dQ, dK/dV (3 launches) */
  NC_K_QK_BWD = 20,     /* QK-norm + RoPE backward */
  NC_K_EMB_BWD = 21,    /* embedding backward, and the QKV weight-gradient scatter */
  NC_K_COUNT = 22
} nc_kernel_kind;

/* Per-launch timing hook.  `events` holds 2*capacity cudaEvent_t handles
 * created by nc_event_create; launch i is bracketed by events[2i] and
 * events[2i+1] recorded on the forward's stream, and kinds[i] names it.
 * On return `count` holds the number of launches (NC_ERR_INVALID_ARG, with
 * nothing enqueued, if capacity is too small: count then says how many are
 * needed). */
typedef struct {
  void* const* events;
  int32_t capacity;
  int32_t count;
  int32_t* kinds; /* host array of capacity entries */
} nc_trace;

/* nc_forward with a timing hook (trace may be NULL). */
nc_status nc_forward_traced(const nc_config* cfg, const nc_weights* w, const int32_t* tokens,
                            const int32_t* targets, int B, int T, float* logits,
                            float* token_loss, float* loss, void* workspace, size_t ws_bytes,
                            void* stream, nc_trace* trace);

/* Timing events (thin wrappers of the CUDA runtime; no device memory). */
nc_status nc_event_create(void** event);
nc_status nc_event_destroy(void* event);
/* Milliseconds between two recorded events (waits for `end`). */
nc_status nc_event_elapsed_ms(void* start, void* end, float* ms);
/* Work enqueued on `stream` after this call waits for `event` (one of a
 * trace's events: e.g. a side stream that starts a collective on a layer's
 * gradients once the launch that last writes them has finished).  Host only;
 * NULL stream: the legacy default stream. */
nc_status nc_stream_wait_event(void* stream, void* event);

/* Synchronises `stream` and returns the status recorded in the device status
 * word at `dev_status` (e.g. the workspace of nc_forward): NC_OK,
 * NC_ERR_TOKEN_RANGE, NC_ERR_TIMEOUT, or NC_ERR_CUDA for a sticky CUDA error. */
nc_status nc_get_status(const void* dev_status, void* stream);

/* ---------------------------------------------------------------- single steps */

/* Weight cast ("约100美元训出对话模型": fp32 weights converted to bf16 for the
 * matmul): each of n fp32 values is rounded to bf16 (nearest, ties to even).
 * container NC_BF16 stores the bf16 bits; NC_F16 stores that bf16 value as fp16
 * (exact for |w| >= 2^-14, nearest fp16 subnormal below).  n % 8 == 0. */
nc_status nc_cast_weights(const float* src, uint16_t* dst, int64_t n, nc_dtype container,
                          void* stream);

/* x[m, :] = wte[tokens[m], :] for m < M ("从文本到聊天模型" §5.2).
 * x [M, C] fp32; wte [V, C] fp32.  Bad ids set NC_DEV_TOKEN_RANGE and read row 0. */
nc_status nc_embedding(const int32_t* tokens, const float* wte, float* x, int M, int C, int V,
                       uint32_t* dev_status, void* stream);

/* out[m, :] = x[m, :] / sqrt(mean(x[m, :]^2) + eps), parameter-free RMSNorm
 * ("Nanochat与nanoGPT对比" §1).  x [M, C] fp32, out [M, C] 16-bit (dtype);
 * C % 8 == 0. */
nc_status nc_rmsnorm(const float* x, uint16_t* out, int M, int C, float eps, nc_dtype dtype,
                     void* stream);

/* RoPE angle table: table[0][t][i] = cos(t * base^(-2i/D)),
 * table[1][t][i] = sin(...), fp32, t < T, i < D/2 (angles in fp64). */
nc_status nc_rope_table(float* table, int T, int D, float base, void* stream);

/* In place: q <- rmsnorm(rope(q)), k <- rmsnorm(rope(k)) per head over D
 * ("从文本到聊天模型" §5.6; "Nanochat与nanoGPT对比" §1: QK-norm after RoPE).
 * q [B, T, H, D] 16-bit (dtype) with q_row_stride elements between
 * consecutive tokens (H*D when contiguous); k [B, T, Hkv, D] with
 * k_row_stride.  Pair (u_i, u_{i+D/2}) of the token at position t is rotated by
 * t * theta_i, table from nc_rope_table.  D in {64, 128}. */
nc_status nc_rope_qknorm(uint16_t* q, uint16_t* k, const float* table, int B, int T, int H,
                         int Hkv, int D, int64_t q_row_stride, int64_t k_row_stride, float eps,
                         nc_dtype dtype, void* stream);

/* Causal sliding-window attention with GQA ("从文本到聊天模型" §5.4-5.5):
 * out[b,i,h,:] = sum_j softmax_j(q[b,i,h,:].k[b,j,g,:] / sqrt(D)) v[b,j,g,:],
 * g = h / (H/Hkv), over keys j <= i with i - j < window (window <= 0 or
 * >= T: full causal).  q/out [B,T,H,D], k/v [B,T,Hkv,D], contiguous 16-bit
 * (dtype; the probabilities enter P.V in the same format).  D in {64, 128}. */
nc_status nc_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v, uint16_t* out,
                       int B, int T, int H, int Hkv, int D, int window, nc_dtype dtype,
                       void* stream);

/* Same with explicit token strides (elements between consecutive tokens) for
 * q, k, v (e.g. the three column blocks of one fused [M, (H+2Hkv)D] buffer);
 * out is contiguous [B, T, H, D]. */
nc_status nc_attention_strided(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                               uint16_t* out, int B, int T, int H, int Hkv, int D, int window,
                               int64_t q_row_stride, int64_t kv_row_stride, nc_dtype dtype,
                               void* stream);

/* Epilogues of nc_linear. */
typedef enum {
  NC_EPI_STORE_16 = 0,     /* out 16-bit (dtype) [M, ldo]: acc                   */
  NC_EPI_RELU2_16 = 1,     /* out 16-bit: relu(acc)^2 ("从文本到聊天模型" §5.7)  */
  NC_EPI_RESID_F32 = 2,    /* out fp32: out += acc (residual add, §5.3)          */
  NC_EPI_STORE_F32 = 3,    /* out fp32: acc                                      */
  NC_EPI_SOFTCAP_F32 = 4   /* out fp32: cap * tanh(acc / cap)                    */
} nc_epilogue;

/* out = epilogue(a @ w^T): a [M, K] and w [N, K] row-major 16-bit, both in
 * format dtype; 16-bit outputs use the same format.  out row stride ldo
 * elements (>= N).  tcgen05 tensor cores, fp32 accumulation in tensor memory.
 * K % 8 == 0, N % 32 == 0.  dev_status gets NC_DEV_TIMEOUT if a pipeline wait
 * ran out. */
nc_status nc_linear(const uint16_t* a, const uint16_t* w, void* out, int M, int N, int K,
                    int64_t ldo, nc_epilogue epilogue, float cap, nc_dtype dtype,
                    uint32_t* dev_status, void* stream);

/* ---------------------------------------------------------------- backward
 * The training micro-step's loss.backward() ("从文本到聊天模型" §6.5): the
 * mean loss of the plain block stack and its gradient with respect to every
 * fp32 master weight.  The fp32 -> 16-bit cast of a weight is taken as
 * straight-through (dW = dY^T X).  Targets of -1 contribute nothing; the mean
 * is over the others.  */

/* fp32 gradients, device pointers; the per-layer members are HOST arrays of
 * n_layer device pointers, each the shape of its weight in nc_weights.  The
 * backward ADDS into them (zero them for a fresh step, keep them to accumulate
 * micro-steps).  16-byte aligned. */
typedef struct {
  float* wte;                 /* [V, C]        */
  float* const* c_q;          /* n_layer x [H*D, C]   */
  float* const* c_k;          /* n_layer x [Hkv*D, C] */
  float* const* c_v;          /* n_layer x [Hkv*D, C] */
  float* const* attn_proj;    /* n_layer x [C, H*D]   */
  float* const* c_fc;         /* n_layer x [4C, C]    */
  float* const* mlp_proj;     /* n_layer x [C, 4C]    */
  float* lm_head;             /* [V, C]        */
  /* Written only for the terms enabled in nc_config.extras (may be NULL
   * otherwise), shapes as in nc_weights; summed over tokens with atomics (not
   * bitwise reproducible run to run). */
  float* smear_gate;          /* [C]                NC_EXTRA_SMEAR         */
  float* const* value_embeds; /* n_layer x [V, Hkv*D] NC_EXTRA_VALUE_EMBED;  */
  float* const* ve_gates;     /* n_layer x [Hkv]: entries of layers without a
                                 value embedding are not written (may be NULL) */
  float* resid_lambdas;       /* [n_layer]          NC_EXTRA_RESID_LAMBDAS */
  float* x0_lambdas;          /* [n_layer]          NC_EXTRA_RESID_LAMBDAS */
  float* backout_lambda;      /* [1]                NC_EXTRA_BACKOUT       */
} nc_grads;

/* Workspace bytes of nc_forward_backward for a [B, T] batch (0 on bad input):
 * the 16-bit weights, per layer the activations the backward reads (residual
 * stream at the block's input and after attention, q|k|v, the QK-norm factors,
 * the attention output and its log-sum-exp, the MLP hidden activations), the
 * 16-bit gradient of the logits [B*T, V] and the backward's scratch; with
 * NC_EXTRA_RESID_LAMBDAS also x0, each block's stream before the mix and a
 * gradient accumulator for x0 (n_layer + 2 fp32 [B*T, C] arrays), with
 * NC_EXTRA_BACKOUT one more such array.  Host only. */
size_t nc_train_workspace_bytes(const nc_config* cfg, int B, int T);

/* Forward with the activations kept, then the backward: writes *loss (device
 * float, the mean over counted targets) and adds the gradients into *g.
 * cfg->fp8 must be 0 (NC_ERR_CONFIG); the further terms of cfg->extras are
 * supported, their parameters' gradients going to the matching members of *g
 * ("Nanochat与nanoGPT对比" §1).  tokens, targets [B, T]
 * int32 device.  The attention backward and the projections' products run on
 * tcgen05 tensor cores.  Split-K weight gradients are summed in no fixed order
 * (not bitwise reproducible run to run).
 * Asynchronous on `stream`. */
nc_status nc_forward_backward(const nc_config* cfg, const nc_weights* w, const int32_t* tokens,
                              const int32_t* targets, int B, int T, float* loss, const nc_grads* g,
                              void* workspace, size_t ws_bytes, void* stream);

/* The same, recording each step's pair of events into *trace (as
 * nc_forward_traced: trace->count = the number of steps, 12 + 24 n_layer). */
nc_status nc_forward_backward_traced(const nc_config* cfg, const nc_weights* w, const int32_t* tokens,
                                     const int32_t* targets, int B, int T, float* loss, const nc_grads* g,
                                     void* workspace, size_t ws_bytes, void* stream, nc_trace* trace);

/* nc_attention_strided that also writes lse [B*T, H] (fp32, device): the
 * natural log-sum-exp of each query row's scaled, visible scores, which the
 * backward uses to recompute the attention weights. */
nc_status nc_attention_lse(const uint16_t* q, const uint16_t* k, const uint16_t* v, uint16_t* out, float* lse,
                           int B, int T, int H, int Hkv, int D, int window, int64_t q_row_stride,
                           int64_t kv_row_stride, nc_dtype dtype, void* stream);

/* Attention backward: qkv [B*T, (H + 2 Hkv) D] packed q | k | v heads (the
 * fused projection's layout), o and dO [B*T, H*D], lse as nc_attention_lse
 * writes it; dqkv gets dq | dk | dv in qkv's layout (dk, dv summed over the
 * query heads of each kv group).  delta (B*T*H fp32) is scratch.  tcgen05
 * tensor cores with the scores in tensor memory (one kernel per 128 keys for
 * dK, dV; one per 128 queries for dQ), fp32 accumulation; no atomics, so the
 * result is the same run to run. */
nc_status nc_attention_backward(const uint16_t* qkv, const uint16_t* o, const uint16_t* dO, const float* lse,
                                float* delta, uint16_t* dqkv, int B, int T, int H, int Hkv, int D, int window,
                                nc_dtype dtype, void* stream);

/* The two products of a linear layer's backward, on the tcgen05 GEMM with
 * 16-bit operands in format dtype (device, 16-byte aligned, row-major):
 * dgrad  dx [M, K] = dy [M, N] . w [N, K]  (w as stored for the forward);
 *        epilogue NC_EPI_STORE_16 (dx in dtype) or NC_EPI_STORE_F32 (fp32);
 * wgrad  dw [N, K] += alpha dy[M, N]^T . x [M, K]  (fp32, summed over the M
 *        rows; split over M in no fixed order).
 * N % 8 == 0 and K % 8 == 0; M >= 1. */
nc_status nc_linear_dgrad(const uint16_t* dy, const uint16_t* w, void* dx, int M, int N, int K,
                          nc_epilogue epilogue, nc_dtype dtype, uint32_t* dev_status, void* stream);
nc_status nc_linear_wgrad(const uint16_t* dy, const uint16_t* x, float* dw, int M, int N, int K, float alpha,
                          nc_dtype dtype, uint32_t* dev_status, void* stream);

/* Dynamic tensorwise e4m3 quantisation of one tensor (the NC_FP8_* rule
 * above): x [n] in src_dtype (NC_F32, NC_BF16 or NC_F16; device, 16-byte
 * aligned), n % 16 == 0.  Writes *amax (one device float; the call zeroes it
 * first) and then codes [n] (device, 16-byte aligned), in stream order.  Two
 * launches. */
nc_status nc_fp8_quantize(const void* x, nc_dtype src_dtype, int64_t n, uint8_t* codes, float* amax,
                          void* stream);

/* out = epilogue((a @ w^T) / (s_a s_w)) with e4m3 codes a [M, K] and w [N, K]
 * (row-major, device, 16-byte aligned) and their tensors' amax values amax_a,
 * amax_w (one device float each, as nc_fp8_quantize writes them; s = 448 /
 * max(amax, 1e-12)).  tcgen05.mma kind::f8f6f4, fp32 accumulation in tensor
 * memory.  16-bit outputs are in format dtype (NC_BF16 or NC_F16).  K % 16 ==
 * 0, N % 32 == 0, ldo as for nc_linear. */
nc_status nc_linear_fp8(const uint8_t* a, const float* amax_a, const uint8_t* w, const float* amax_w,
                        void* out, int M, int N, int K, int64_t ldo, nc_epilogue epilogue, float cap,
                        nc_dtype dtype, uint32_t* dev_status, void* stream);

/* Fused Q/K/V projection ("从文本到聊天模型" §5.4) + RoPE + QK-norm
 * ("Nanochat与nanoGPT对比" §1) in one GEMM: qkv = a @ w^T with w the
 * [(H+2Hkv)*D, C] stack of c_q, c_k, c_v; in each token row the first H heads
 * (q) and the next Hkv heads (k) are rotated (pair (u_i, u_{i+D/2}) of row m by
 * (m % T) * theta_i, table from nc_rope_table) and RMS-normalised over D; the
 * last Hkv heads (v) are stored as computed.  a [M, C], w, out [M, (H+2Hkv)*D]
 * 16-bit in format dtype.  D in {64, 128}, C % 8 == 0. */
nc_status nc_qkv_rope(const uint16_t* a, const uint16_t* w, uint16_t* out, const float* table,
                      int M, int T, int C, int H, int Hkv, int D, float eps, nc_dtype dtype,
                      uint32_t* dev_status, void* stream);

/* Fused soft-cap + log-softmax + NLL over the vocabulary ("Nanochat与nanoGPT对比"
 * §1 soft-cap; "从文本到聊天模型" §5.8 cross-entropy, ignore_index -1):
 *   l = cap * tanh(z / cap);  token_loss[m] = logsumexp(l[m, :]) - l[m, y_m]
 *   (0 where y_m == -1).  z [M, V] raw fp32 logits; capped_out [M, V] fp32 or
 *   NULL (may equal z); token_loss [M] fp32.  Bad targets set
 *   NC_DEV_TARGET_RANGE and count as ignored. */
nc_status nc_softcap_ce(const float* z, const int32_t* targets, float* capped_out,
                        float* token_loss, int M, int V, float cap, uint32_t* dev_status,
                        void* stream);

/* loss[0] = sum(token_loss[m] over targets[m] != -1 and in range) / count,
 * NaN if the count is 0; fixed-order (run-to-run deterministic) reduction. */
nc_status nc_loss_mean(const float* token_loss, const int32_t* targets, int M, int V,
                       float* loss, void* stream);

/* Loss head without any scratch allocation.  The pages have no counterpart
 * to this entry point; it exists for callers that cannot provide scratch
 * memory: code embedded in a host application whose memory manager owns the
 * whole device budget, and code on a latency-critical path where cudaMalloc's
 * implicit device-wide synchronisation is not acceptable.
 *
 * Computes what the last step of nc_forward computes, from the final-norm
 * activations: l = cap * tanh((a @ w_lm^T) / cap), token_loss[m] =
 * logsumexp(l[m, :]) - l[m, y_m] (0 where y_m == -1), loss = mean over valid
 * targets.  a [M, C] and w_lm [V, C] are 16-bit in format dtype (w_lm holding
 * the bf16-rounded weights, e.g. from nc_cast_weights); targets [M] int32;
 * token_loss [M] fp32 (required); loss 1 fp32 or NULL.
 *
 * Instead of a workspace it uses one fixed device array of this library
 * (about 8.4 MB, held on every GPU that loads the library until the process
 * exits), so it allocates nothing and calls no allocating routine.  Limits:
 * M <= 8192 rows and V <= 32768 (NC_ERR_SHAPE beyond them).  The first call
 * on a device looks up the array's device address (cudaGetSymbolAddress, with
 * that device current) and keeps it for the life of the process; make that
 * first call before any stream capture, and do not call this entry point on a
 * device after cudaDeviceReset (the kept address belonged to the destroyed
 * context).  All
 * calls share the array and it keeps the previous call's contents (nothing in
 * it needs clearing), so calls whose work overlaps on the GPU race with each
 * other: order them on one stream. */
nc_status nc_lm_head_loss_static(const uint16_t* a, const uint16_t* w_lm, const int32_t* targets,
                                 int M, int C, int V, float cap, nc_dtype dtype,
                                 float* token_loss, float* loss, uint32_t* dev_status,
                                 void* stream);

/* Self-test of the failure path of in-kernel waits: one CTA waits on an
 * mbarrier that nothing arrives on, through the same bounded wait the GEMM
 * pipeline uses, for at most limit_us microseconds, then sets NC_DEV_TIMEOUT in
 * *dev_status and exits normally (the context stays usable).  Expect
 * nc_get_status(dev_status) == NC_ERR_TIMEOUT afterwards.  limit_us in
 * [1, 2000000]. */
nc_status nc_selftest_bounded_wait(uint32_t* dev_status, uint32_t limit_us, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* NC_H_ */
