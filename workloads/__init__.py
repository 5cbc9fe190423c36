"""Seeded synthetic workloads shared by the tests, the oracle checks and the bench.

This module holds shapes and random numbers only: no step of the forward pass is
computed here.  Both the CUDA path and the fp64 oracle receive the arrays built
below, so the two never share any arithmetic of the method.

Recipe (all draws are numpy ``Generator(PCG64(seed))``):

* weights, seed 1234, drawn in the fixed order ``wte``, then for each layer
  ``c_q, c_k, c_v, attn_proj, c_fc, mlp_proj``, then ``lm_head``; every tensor is
  float32 ``standard_normal * 0.02`` (N(0, 0.02), no zero-init), stored in the
  ``[out_features, in_features]`` layout of a bias-free linear layer;
* tokens, seed 5678, a ``[B, T+1]`` int32 array uniform in ``[0, V)``; the model
  reads ``[:, :-1]`` and is scored against ``[:, 1:]`` (the one-token shift of the
  pretraining dataloader);
* attention-sweep q/k/v, seed 91011, float32 ``standard_normal``;
* the further weights of the full nanochat forward (``make_extras``), seed 4321,
  in the order smear gate [C] (``standard_normal``), resid lambdas [L]
  (``1 + 0.1 * standard_normal``), x0 lambdas [L] (``0.1 * standard_normal``),
  backout lambda (``0.5 + 0.1 * standard_normal``); then, from the sub-stream
  ``PCG64([4321, l + 1])`` of layer l, a value embedding table [V, Hkv*D]
  (``0.5 * standard_normal``) and per-kv-head gates [Hkv] (``standard_normal``).  Tables are drawn for every layer; which layers
  use one is the model's rule, not the generator's.

The shapes are those of the five benchmark configurations of the nanochat
GPT forward: a tiny 2-layer model, d12, d20, d26 and a d26-depth GQA variant.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

WEIGHT_SEED = 1234
TOKEN_SEED = 5678
ATTN_SEED = 91011
EXTRAS_SEED = 4321
INIT_STD = 0.02


@dataclass(frozen=True)
class ModelShape:
    """Explicit sizes of one workload (no derivation happens here)."""

    name: str
    n_layer: int
    d_model: int
    n_head: int
    n_kv_head: int
    head_dim: int
    seq_len: int
    vocab: int
    batch: int
    short_window: int

    @property
    def tokens(self) -> int:
        return self.batch * self.seq_len


# The five model workloads.  Window sizes are a quarter of the context for the
# short layers (the SSSL pattern), written out explicitly.
SHAPES = {
    "tiny": ModelShape("tiny", 2, 128, 2, 2, 64, 256, 512, 2, 64),
    "d12": ModelShape("d12", 12, 768, 6, 6, 128, 2048, 32768, 8, 512),
    "d20": ModelShape("d20", 20, 1280, 10, 10, 128, 2048, 32768, 32, 512),
    "d26": ModelShape("d26", 26, 1664, 13, 13, 128, 2048, 32768, 16, 512),
    "d26_gqa": ModelShape("d26_gqa", 26, 2048, 16, 4, 128, 2048, 32768, 16, 512),
}

# Attention-only sweep: B=4, H=16 (kv heads 16 or 4), D=128.
ATTN_SWEEP = [
    dict(B=4, H=16, Hkv=hkv, D=128, T=T) for T in (2048, 4096, 8192) for hkv in (16, 4)
]

LAYER_WEIGHT_NAMES = ("c_q", "c_k", "c_v", "attn_proj", "c_fc", "mlp_proj")


def weight_shapes(s: ModelShape) -> dict:
    """[out, in] shape of every weight tensor of one layer, plus wte / lm_head."""
    C, H, Hkv, D = s.d_model, s.n_head, s.n_kv_head, s.head_dim
    return {
        "wte": (s.vocab, C),
        "c_q": (H * D, C),
        "c_k": (Hkv * D, C),
        "c_v": (Hkv * D, C),
        "attn_proj": (C, H * D),
        "c_fc": (4 * C, C),
        "mlp_proj": (C, 4 * C),
        "lm_head": (s.vocab, C),
    }


def make_weights(s: ModelShape, seed: int = WEIGHT_SEED) -> dict:
    """All weights as float32 numpy arrays.

    Returns ``{"wte": [V,C], "layers": [ {c_q, c_k, c_v, attn_proj, c_fc, mlp_proj}, ... ],
    "lm_head": [V,C]}``.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    shp = weight_shapes(s)

    def draw(name):
        a = rng.standard_normal(shp[name], dtype=np.float32)
        a *= np.float32(INIT_STD)
        return a

    out = {"wte": draw("wte"), "layers": []}
    for _ in range(s.n_layer):
        out["layers"].append({n: draw(n) for n in LAYER_WEIGHT_NAMES})
    out["lm_head"] = draw("lm_head")
    return out


def make_extras(s: ModelShape, seed: int = EXTRAS_SEED, layers=None) -> dict:
    """Seeded weights of the full nanochat forward's further terms (float32).

    ``layers`` (optional iterable of layer indices) limits which layers get a
    value-embedding table and gates drawn (the others are None); the draws of
    the drawn layers do not depend on that choice.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    L, C, V = s.n_layer, s.d_model, s.vocab
    kvw = s.n_kv_head * s.head_dim
    out = {
        "smear_gate": rng.standard_normal(C, dtype=np.float32),
        "resid_lambdas": (1.0 + 0.1 * rng.standard_normal(L)).astype(np.float32),
        "x0_lambdas": (0.1 * rng.standard_normal(L)).astype(np.float32),
        "backout_lambda": np.float32(0.5 + 0.1 * rng.standard_normal()),
        "value_embeds": [],
        "ve_gates": [],
    }
    keep = set(range(L)) if layers is None else set(layers)
    for l in range(L):
        # one sub-stream per layer, so skipping a layer leaves the others intact
        sub = np.random.Generator(np.random.PCG64([seed, l + 1]))
        if l in keep:
            t = sub.standard_normal((V, kvw), dtype=np.float32)
            t *= np.float32(0.5)
            out["value_embeds"].append(t)
            out["ve_gates"].append(sub.standard_normal(s.n_kv_head, dtype=np.float32))
        else:
            out["value_embeds"].append(None)
            out["ve_gates"].append(None)
    return out


def make_tokens(s: ModelShape, seed: int = TOKEN_SEED, batch: int | None = None,
                seq_len: int | None = None):
    """(inputs [B,T] int32, targets [B,T] int32) from one [B, T+1] uniform draw."""
    B = s.batch if batch is None else batch
    T = s.seq_len if seq_len is None else seq_len
    rng = np.random.Generator(np.random.PCG64(seed))
    row = rng.integers(0, s.vocab, size=(B, T + 1), dtype=np.int32)
    return np.ascontiguousarray(row[:, :-1]), np.ascontiguousarray(row[:, 1:])


def make_qkv(B: int, T: int, H: int, Hkv: int, D: int, seed: int = ATTN_SEED):
    """float32 N(0,1) q [B,T,H,D], k and v [B,T,Hkv,D] for the attention sweep."""
    rng = np.random.Generator(np.random.PCG64(seed))
    q = rng.standard_normal((B, T, H, D), dtype=np.float32)
    k = rng.standard_normal((B, T, Hkv, D), dtype=np.float32)
    v = rng.standard_normal((B, T, Hkv, D), dtype=np.float32)
    return q, k, v


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even), returned as float32.

    A storage-format conversion used to hand both sides identical bf16 inputs.
    """
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16) << 16
    nan = np.isnan(a)
    out = (r & 0xFFFFFFFF).astype(np.uint32).view(np.float32)
    out = np.where(nan, a, out)
    return out.reshape(a.shape)


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """uint16 bit patterns of ``round_to_bf16(a)`` (for uploading bf16 tensors)."""
    r = round_to_bf16(a)
    return (r.view(np.uint32) >> 16).astype(np.uint16)
