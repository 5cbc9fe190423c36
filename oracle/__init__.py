"""fp64 CPU oracle of the nanochat GPT forward pass + token cross-entropy.

TEST INFRASTRUCTURE ONLY.  This package is the plain, slow, obviously correct
statement of what the CUDA library computes.  Only the test-suite, the package's
``smoke()`` check and the CPU-baseline leg of the bench may import it; the
product path (the CUDA library and its Python binding) never does, and the
oracle imports nothing from the product path.  It shares no code, table or
constant generator with the CUDA side; both receive their inputs from the
separate ``workloads`` module, which holds no arithmetic of the method.

Sources (page title, section):

* "从文本到聊天模型" (onehacker.top) -- §4.1 input/target shift, §5.1 model
  configuration, §5.2 token embedding, §5.3 pre-norm residual block, §5.4
  separate Q/K/V projections and their (B,T,H,D) / (B,T,Hkv,D) shapes, §5.5 causal
  attention, §5.6 RoPE, §5.7 ReLU^2 MLP, §5.8 untied LM head and cross-entropy
  with ``ignore_index=-1``.
* "Nanochat与nanoGPT对比：关键升级" (lzwjava.github.io) -- §1 architecture table
  and its notes: RoPE without learned positions, parameter-free RMSNorm, ReLU^2,
  split c_q/c_k/c_v/c_proj, GQA, QK-norm applied after RoPE, no biases, untied
  embedding, no dropout, tanh logit soft-cap at +-15, SSSL sliding window (three
  quarter-context layers then one full layer, the last layer always full), the
  final normalisation before the logit projection (Backout note).
* "约100美元训出对话模型，nanochat源码全链路拆解" (ikfou.com) -- the example
  config (sequence_len 2048, vocab 32768, SSSL) and fp32 weights cast to bf16 at
  matmul time; nanochat README mirror (dev.wehub.plus), "精度 / dtype".

Readings where the pages are silent (each is a config field or a single
function here, and the CUDA library takes the same reading independently):

* RMSNorm eps = 1e-6; QK-norm is per head over the head dimension D.
* RoPE: theta_i = base^(-2i/D), base 10000, positions 0..T-1 in each row, pairs
  (u_i, u_{i+D/2}) rotated by +t*theta_i.
* softmax scale 1/sqrt(D), applied after QK-norm.
* window predicate: key j is visible from query i iff j <= i and i - j < W
  (exactly W keys including the query itself).
* layer l uses pattern[l % len(pattern)], and the last layer is forced full.
* GQA: query head h reads kv head h // (H / Hkv).
* weights enter every matrix product as their bf16 (round-to-nearest-even)
  values -- the pages fix that cast -- and the products and everything else are
  fp64; the embedding table is read as given (fp32, no cast).
* no norm after the embedding; one parameter-free RMSNorm before lm_head.
* soft-cap 15*tanh(z/15) is applied before the loss and the returned logits are
  the capped ones; loss = mean natural-log NLL over targets != -1 (NaN if none).

Further terms of the full nanochat forward ("Nanochat与nanoGPT对比" §1 table and
notes), each optional (``forward(..., extras=...)``), with these readings of the
one-line descriptions there:

* smear: gate is a bias-free linear map C -> 1 applied to the current token's
  embedding (its weight enters as bf16 like every linear layer);
  x_t = e_t + sigmoid(gate(e_t)) e_{t-1}, position 0 of each row unchanged;
* residual lambdas + x0: before block l, x = resid_lambdas[l] x +
  x0_lambdas[l] x0, x0 being the (smeared) embedding output;
* value embeddings: a table [V, Hkv*D] per layer on every other layer counted
  back from the last (which always has one); v = v + gate * table[idx] with one
  plain learnable gate per kv head, added to v after its projection;
* backout: x_mid is the stream after the first L // 2 blocks (before block
  L // 2 mixes in x0); before the final norm x = x - lambda * x_mid.

Those pins live in ``tests/test_oracle_extras.py``.

Backward ("从文本到聊天模型" §6.5: the training step's loss.backward()):
``oracle.grad.forward_backward`` gives the mean loss of the plain stack and its
gradient with respect to every fp32 master weight, the bf16 cast taken as
straight-through; pinned in ``tests/test_oracle_grad.py`` by finite
differences and torch float64 autograd.  With ``extras`` it also
differentiates the further terms (smear, residual lambdas with x0, value
embeddings, backout) and returns their parameters' gradients; pinned in
``tests/test_oracle_grad_extras.py`` by finite differences, by its loss
against the separately pinned ``forward(..., extras=...)``, and by neutral
terms leaving the plain gradients unchanged.

FP8 ("Nanochat与nanoGPT对比" §1 table, FP8-training row: dynamic tensor-level
e4m3/e5m2): ``forward(..., fp8="block" | "all")`` runs the block projections
(and with "all" the LM head) through dynamic tensorwise e4m3; the readings are
in ``oracle/fp8.py`` and its pins in ``tests/test_oracle_fp8.py``.  With
tensorwise scales the scale of an activation depends on every row and
position of the batch, so the fp8 forward is causal and row-independent only
up to that shared scale.

Parity pins live in ``tests/test_oracle_pins.py``.  Every function below is
pinned there by closed forms, invariants, brute force or an independent library
routine.  The composition of the full forward at random weights is pinned only
structurally (zero-projection closed form, causality, row independence): no page
prints logits or losses for any input, so the absolute values of a random-weight
forward are "parity unpinned" beyond those structural pins.
"""
from .model import (  # noqa: F401
    OracleConfig,
    derive_config,
    layer_windows,
    window_visible,
    rms_norm,
    rope_tables,
    rope,
    rope_qknorm,
    attention,
    relu2_mlp,
    to_bf16,
    linear,
    softcap,
    cross_entropy,
    embed,
    forward,
    smear,
    value_embed_layers,
    backout_layer,
)
from .fp8 import round_e4m3, quantize_e4m3, linear_e4m3, tensor_scale  # noqa: F401,E402
