"""fp64 oracle of the nanochat GPT block-stack forward + cross-entropy.

TEST INFRASTRUCTURE ONLY -- see the package docstring for who may import this
module, the sources and the readings taken where the pages are silent.

Everything is numpy float64.  fp32 inputs (weights) are upcast exactly.  The
matrix products use numpy's matmul as a library primitive; nothing is blocked,
fused or reordered beyond the definitions written here.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

from .fp8 import linear_e4m3

F64 = np.float64


@dataclass(frozen=True)
class OracleConfig:
    n_layer: int
    d_model: int
    n_head: int
    n_kv_head: int
    head_dim: int
    seq_len: int
    vocab: int
    window_pattern: str = "SSSL"
    short_window: int = 0  # 0 -> seq_len // 4
    softcap: float = 15.0
    norm_eps: float = 1e-6
    rope_base: float = 10000.0

    @property
    def short(self) -> int:
        return self.short_window if self.short_window > 0 else self.seq_len // 4


def derive_config(depth: int, aspect_ratio: int = 64, head_dim: int = 128,
                  n_kv_head: int = 0, seq_len: int = 2048, vocab: int = 32768,
                  **kw) -> OracleConfig:
    """Depth-derived sizes.

    "从文本到聊天模型" §5.1: model_dim = depth * aspect_ratio and
    num_heads = model_dim // head_dim (d24: 1536 wide, 12 heads).
    n_kv_head = 0 means "as many kv heads as query heads" (plain MHA).
    """
    d_model = depth * aspect_ratio
    n_head = d_model // head_dim
    return OracleConfig(n_layer=depth, d_model=d_model, n_head=n_head,
                        n_kv_head=n_kv_head if n_kv_head > 0 else n_head,
                        head_dim=head_dim, seq_len=seq_len, vocab=vocab, **kw)


def layer_windows(cfg: OracleConfig) -> list:
    """Attention window (number of visible keys) of every layer.

    "Nanochat与nanoGPT对比：关键升级" §1, sliding-window note: in the SSSL
    pattern three layers use a short window of a quarter of the context and one
    layer the full context, cycling over the layers; the last layer is always
    full.  'S' -> short window, 'L' -> seq_len.
    """
    pat = cfg.window_pattern
    out = []
    for l in range(cfg.n_layer):
        ch = pat[l % len(pat)]
        if l == cfg.n_layer - 1:
            ch = "L"
        out.append(cfg.seq_len if ch == "L" else cfg.short)
    return out


def window_visible(i: int, j: int, W: int) -> bool:
    """Key j is visible from query i: causal ("从文本到聊天模型" §5.5) and inside
    a window of W keys that ends at the query itself."""
    return j <= i and (i - j) < W


def rms_norm(u: np.ndarray, eps: float) -> np.ndarray:
    """Parameter-free RMSNorm over the last axis ("Nanochat与nanoGPT对比" §1:
    RMSNorm without learnable parameters): u / sqrt(mean(u^2) + eps)."""
    u = np.asarray(u, dtype=F64)
    ms = np.mean(u * u, axis=-1, keepdims=True)
    return u / np.sqrt(ms + eps)


def rope_tables(T: int, D: int, base: float):
    """cos/sin of t * theta_i, theta_i = base^(-2i/D), shapes [T, D/2] (fp64)."""
    half = D // 2
    i = np.arange(half, dtype=F64)
    theta = base ** (-2.0 * i / D)
    t = np.arange(T, dtype=F64)
    ang = t[:, None] * theta[None, :]
    return np.cos(ang), np.sin(ang)


def rope(u: np.ndarray, cos: np.ndarray, sin: np.ndarray, pos0: int = 0) -> np.ndarray:
    """Rotary position embedding ("从文本到聊天模型" §5.6; "Nanochat与nanoGPT对比"
    §1: rotation in complex space, no learned position table).

    u: [..., T, heads, D] with the sequence axis third from the end.  Pair
    (u_i, u_{i+D/2}) at position t is rotated by the angle t * theta_i.
    """
    u = np.asarray(u, dtype=F64)
    T, D = u.shape[-3], u.shape[-1]
    half = D // 2
    c = cos[pos0:pos0 + T][:, None, :]  # [T, 1, D/2]
    s = sin[pos0:pos0 + T][:, None, :]
    a, b = u[..., :half], u[..., half:]
    return np.concatenate([a * c - b * s, a * s + b * c], axis=-1)


def rope_qknorm(q: np.ndarray, k: np.ndarray, cfg: OracleConfig):
    """RoPE, then per-head RMSNorm of q and k ("Nanochat与nanoGPT对比" §1: q and
    k are normalised after RoPE)."""
    T, D = q.shape[-3], q.shape[-1]
    cos, sin = rope_tables(T, D, cfg.rope_base)
    return (rms_norm(rope(q, cos, sin), cfg.norm_eps),
            rms_norm(rope(k, cos, sin), cfg.norm_eps))


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, W: int,
              query_positions=None) -> np.ndarray:
    """Causal sliding-window attention with GQA.

    q [B,T,H,D], k and v [B,T,Hkv,D] ("从文本到聊天模型" §5.4).  Query head h
    reads kv head h // (H/Hkv) (several query heads share one kv head).  For query
    i: s_j = q_i . k_j / sqrt(D) over the visible keys j, o_i = sum_j softmax(s)_j v_j.
    ``query_positions`` (optional) restricts the output to those rows; the
    result then has shape [B, len(query_positions), H, D].
    """
    q = np.asarray(q, dtype=F64)
    k = np.asarray(k, dtype=F64)
    v = np.asarray(v, dtype=F64)
    B, T, H, D = q.shape
    Hkv = k.shape[2]
    assert H % Hkv == 0
    group = H // Hkv
    rows = np.arange(T) if query_positions is None else np.asarray(query_positions)
    scale = 1.0 / math.sqrt(D)
    i = rows[:, None]
    j = np.arange(T)[None, :]
    visible = (j <= i) & ((i - j) < W)  # [R, T]
    out = np.zeros((B, len(rows), H, D), dtype=F64)
    for b in range(B):
        for h in range(H):
            g = h // group
            s = (q[b, rows, h, :] @ k[b, :, g, :].T) * scale  # [R, T]
            s = np.where(visible, s, -np.inf)
            s = s - s.max(axis=1, keepdims=True)
            p = np.exp(s)
            p = p / p.sum(axis=1, keepdims=True)
            out[b, :, h, :] = p @ v[b, :, g, :]
    return out


def relu2_mlp(a: np.ndarray, w_fc: np.ndarray, w_proj: np.ndarray, lin=None) -> np.ndarray:
    """"从文本到聊天模型" §5.7: c_fc (C -> 4C), relu(x)^2, c_proj (4C -> C).
    ``lin`` is the linear map to use (``linear`` unless given)."""
    lin = lin or linear
    h = lin(a, w_fc)
    h = np.maximum(h, 0.0) ** 2
    return lin(h, w_proj)


def softcap(z: np.ndarray, cap: float) -> np.ndarray:
    """"Nanochat与nanoGPT对比" §1: tanh logit soft-cap at +-cap."""
    return cap * np.tanh(np.asarray(z, dtype=F64) / cap)


def cross_entropy(logits: np.ndarray, targets: np.ndarray):
    """Token-level cross-entropy with ignore_index = -1 ("从文本到聊天模型" §5.8).

    logits [..., V], targets [...] int.  Returns (per-token NLL with 0 at ignored
    positions, mean NLL over the non-ignored positions; NaN if there are none).
    """
    l = np.asarray(logits, dtype=F64)
    y = np.asarray(targets).astype(np.int64)
    m = l.max(axis=-1, keepdims=True)
    lse = (m + np.log(np.exp(l - m).sum(axis=-1, keepdims=True)))[..., 0]
    valid = y != -1
    ysafe = np.where(valid, y, 0)
    picked = np.take_along_axis(l, ysafe[..., None], axis=-1)[..., 0]
    nll = np.where(valid, lse - picked, 0.0)
    n = int(valid.sum())
    loss = float(nll.sum() / n) if n > 0 else float("nan")
    return nll, loss


def to_bf16(w: np.ndarray) -> np.ndarray:
    """Round to the nearest bfloat16 value, ties to even, returned as float64.

    The method keeps its weights in fp32 and converts them to the compute dtype
    (bf16) when they enter a matrix product (nanochat README mirror, "精度 /
    dtype"; "约100美元训出对话模型" on the custom Linear layer).  bfloat16 keeps
    the top 16 bits of the fp32 pattern; the dropped low half is rounded half to
    even on the kept least-significant bit.  NaN stays NaN.
    """
    a = np.ascontiguousarray(w, dtype=np.float32)
    bits = a.view(np.uint32).astype(np.uint64)
    keep_lsb = (bits >> np.uint64(16)) & np.uint64(1)
    rounded = (bits + np.uint64(0x7FFF) + keep_lsb) >> np.uint64(16)
    out = (rounded << np.uint64(16)).astype(np.uint32).view(np.float32)
    out = np.where(np.isnan(a), a, out)
    return out.astype(F64)


def linear(x: np.ndarray, w: np.ndarray) -> np.ndarray:
    """Bias-free linear layer y = x W^T with W in [out, in] layout ("Nanochat与
    nanoGPT对比" §1: no biases).  The fp32 weight is cast to bf16 first (see
    ``to_bf16``); the product itself is exact fp64."""
    return np.asarray(x, dtype=F64) @ to_bf16(w).T


def embed(wte: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """"从文本到聊天模型" §5.2: x = wte(idx), (B,T) -> (B,T,C)."""
    return np.asarray(wte, dtype=F64)[np.asarray(idx)]


def value_embed_layers(n_layer: int) -> list:
    """Layers that carry a value embedding: every other layer, counted back from
    the last one, which always has one ("Nanochat与nanoGPT对比" §1, value
    residual note)."""
    return [(n_layer - 1 - l) % 2 == 0 for l in range(n_layer)]


def backout_layer(n_layer: int) -> int:
    """The block whose input is cached for backout: the middle of the stack,
    i.e. the residual stream after the first n_layer // 2 blocks (reading of the
    backout note in "Nanochat与nanoGPT对比" §1, which only says "a middle
    layer")."""
    return n_layer // 2


def smear(x: np.ndarray, gate_w: np.ndarray) -> np.ndarray:
    """"Nanochat与nanoGPT对比" §1, smear note: mix the previous token's embedding
    into the current one through a learnable gate, x_t + sigmoid(gate(x_t)) x_{t-1}.

    gate is a bias-free linear map C -> 1 (its fp32 weight enters as bf16, like
    every linear layer, see ``linear``); the first position of each row has no
    previous token and is left unchanged.  x: [B, T, C].
    """
    x = np.asarray(x, dtype=F64)
    z = linear(x, np.asarray(gate_w).reshape(1, -1))[..., 0]  # [B, T]
    g = 1.0 / (1.0 + np.exp(-z))
    prev = np.zeros_like(x)
    prev[:, 1:] = x[:, :-1]
    return x + g[..., None] * prev


def forward(cfg: OracleConfig, weights: dict, idx: np.ndarray, targets=None,
            want_logits: bool = True, extras: dict = None, fp8: str = None):
    """The whole forward for the rows of ``idx`` ([B, T] int).

    Steps in the order of "从文本到聊天模型" §5 (embedding, blocks of
    ``x = x + attn(norm(x)); x = x + mlp(norm(x))``, LM head, cross-entropy) with
    the block internals of "Nanochat与nanoGPT对比" §1 (split c_q/c_k/c_v,
    RoPE then QK-norm, SSSL windows, GQA, ReLU^2, final norm, soft-cap).

    ``extras`` (optional) adds the further terms of the full nanochat forward
    listed in "Nanochat与nanoGPT对比" §1; each key switches one on:

    * ``smear_gate`` [C]: x = smear(wte[idx]) (see ``smear``);
    * ``resid_lambdas`` / ``x0_lambdas`` [L]: before block l the stream becomes
      resid_lambdas[l] * x + x0_lambdas[l] * x0, x0 being the (smeared)
      embedding output;
    * ``value_embeds`` (list of L entries, [V, Hkv*D] or None) and ``ve_gates``
      (list of L entries, [Hkv] or None): on the layers of
      ``value_embed_layers``, v = v + gate * ve with ve = value_embeds[l][idx]
      and one gate per kv head;
    * ``backout_lambda`` (scalar): x_mid = the stream after the first
      ``backout_layer`` blocks; before the final norm x = x - lambda * x_mid.

    ``fp8`` (optional, "Nanochat与nanoGPT对比" §1, FP8-training row): "block"
    sends the six block projections through ``fp8.linear_e4m3`` (dynamic
    tensorwise e4m3 of both operands), "all" the LM head as well.

    Returns a dict with ``logits`` ([B,T,V] capped, fp64, if ``want_logits``),
    ``token_loss`` ([B,T]) and ``loss`` (scalar) when targets are given.
    """
    ex = extras or {}
    if fp8 not in (None, "block", "all"):
        raise ValueError(f"fp8 must be None, 'block' or 'all', not {fp8!r}")
    blin = linear_e4m3 if fp8 else linear
    hlin = linear_e4m3 if fp8 == "all" else linear
    idx = np.asarray(idx)
    B, T = idx.shape
    C, H, Hkv, D = cfg.d_model, cfg.n_head, cfg.n_kv_head, cfg.head_dim
    eps = cfg.norm_eps
    windows = layer_windows(cfg)
    cos, sin = rope_tables(T, D, cfg.rope_base)
    x = embed(weights["wte"], idx)  # [B,T,C]
    if "smear_gate" in ex:
        x = smear(x, ex["smear_gate"])
    x0 = x
    L = len(weights["layers"])
    x_mid = None
    for l, lw in enumerate(weights["layers"]):
        if "backout_lambda" in ex and l == backout_layer(L):
            x_mid = x
        if "resid_lambdas" in ex:
            x = F64(ex["resid_lambdas"][l]) * x + F64(ex["x0_lambdas"][l]) * x0
        a = rms_norm(x, eps)
        q = blin(a, lw["c_q"]).reshape(B, T, H, D)
        k = blin(a, lw["c_k"]).reshape(B, T, Hkv, D)
        v = blin(a, lw["c_v"]).reshape(B, T, Hkv, D)
        if "value_embeds" in ex and value_embed_layers(L)[l]:
            ve = embed(ex["value_embeds"][l], idx).reshape(B, T, Hkv, D)
            v = v + np.asarray(ex["ve_gates"][l], dtype=F64)[None, None, :, None] * ve
        q = rms_norm(rope(q, cos, sin), eps)
        k = rms_norm(rope(k, cos, sin), eps)
        o = attention(q, k, v, windows[l])
        x = x + blin(o.reshape(B, T, H * D), lw["attn_proj"])
        a = rms_norm(x, eps)
        x = x + relu2_mlp(a, lw["c_fc"], lw["mlp_proj"], lin=blin)
    if x_mid is not None:
        x = x - F64(ex["backout_lambda"]) * x_mid
    a = rms_norm(x, eps)
    logits = softcap(hlin(a, weights["lm_head"]), cfg.softcap)  # [B,T,V]
    res = {}
    if want_logits:
        res["logits"] = logits
    if targets is not None:
        nll, loss = cross_entropy(logits, np.asarray(targets))
        res["token_loss"] = nll
        res["loss"] = loss
    return res
