"""Pins of the oracle's further terms of the full nanochat forward.

"Nanochat与nanoGPT对比：关键升级" §1 lists them in its architecture table and
notes: value embeddings injected into V through a gate on alternating layers
(the last layer always has one), smear (the previous token's embedding mixed in
through a sigmoid gate), backout (a middle-layer stream subtracted before the
final norm) and per-layer residual lambdas with x0.  As in
``test_oracle_pins.py`` nothing here retypes an oracle formula: each pin is a
hand-computed value, a closed form reached by another route (scalar recurrences,
torch's own bf16 conversion), an exact reduction to the plain forward, or an
invariant.
"""
import math

import numpy as np
import torch

import oracle
from oracle import OracleConfig
from oracle.model import backout_layer, smear, value_embed_layers
from workloads import SHAPES, make_extras


def bf16_t(a):
    """fp32 weights as their bf16 values, through torch's own conversion."""
    return torch.from_numpy(np.asarray(a, dtype=np.float32)).to(torch.bfloat16).to(torch.float64).numpy()


def _cfg(**kw):
    base = dict(n_layer=4, d_model=32, n_head=2, n_kv_head=1, head_dim=16,
                seq_len=12, vocab=40, short_window=4)
    base.update(kw)
    return OracleConfig(**base)


def _weights(c, seed=5, std=0.3):
    rng = np.random.default_rng(seed)
    C, H, Hkv, D, V = c.d_model, c.n_head, c.n_kv_head, c.head_dim, c.vocab
    g = lambda *s: (rng.standard_normal(s) * std).astype(np.float32)
    return {"wte": g(V, C), "lm_head": g(V, C),
            "layers": [{"c_q": g(H * D, C), "c_k": g(Hkv * D, C), "c_v": g(Hkv * D, C),
                        "attn_proj": g(C, H * D), "c_fc": g(4 * C, C), "mlp_proj": g(C, 4 * C)}
                       for _ in range(c.n_layer)]}


def _extras(c, seed=9):
    rng = np.random.default_rng(seed)
    L, kvw = c.n_layer, c.n_kv_head * c.head_dim
    return {"smear_gate": rng.standard_normal(c.d_model).astype(np.float32),
            "resid_lambdas": (1 + 0.2 * rng.standard_normal(L)).astype(np.float32),
            "x0_lambdas": (0.2 * rng.standard_normal(L)).astype(np.float32),
            "backout_lambda": np.float32(0.4),
            "value_embeds": [rng.standard_normal((c.vocab, kvw)).astype(np.float32) for _ in range(L)],
            "ve_gates": [rng.standard_normal(c.n_kv_head).astype(np.float32) for _ in range(L)]}


def _rms(u, eps):
    return u / np.sqrt(np.mean(u * u, -1, keepdims=True) + eps)


def test_layer_choices_follow_the_page_words():
    # value embeddings: every other layer, the last one always included
    assert value_embed_layers(1) == [True]
    assert value_embed_layers(2) == [False, True]
    assert value_embed_layers(4) == [False, True, False, True]
    assert value_embed_layers(5) == [True, False, True, False, True]
    assert sum(value_embed_layers(20)) == 10 and value_embed_layers(20)[19]
    # backout: the middle of the stack
    assert [backout_layer(L) for L in (1, 2, 3, 12, 20, 26)] == [0, 1, 1, 6, 10, 13]


def test_smear_hand_values():
    # gate weights 0.5 and 0.25 are exact in bf16; x_t + sigmoid(w . x_t) x_{t-1}
    e = np.array([[[1.0, -1.0], [2.0, 0.0], [0.0, 4.0]]])
    w = np.array([0.5, 0.25], dtype=np.float32)
    s1 = 1.0 / (1.0 + math.exp(-1.0))  # w . e_1 = 1
    s2 = 1.0 / (1.0 + math.exp(-1.0))  # w . e_2 = 1
    want = np.array([[[1.0, -1.0], [2.0 + s1, -s1], [2.0 * s2, 4.0]]])
    np.testing.assert_allclose(smear(e, w), want, rtol=0, atol=1e-15)
    # first position unchanged; a strongly closed gate leaves every row alone
    big = np.array([-200.0, -200.0], dtype=np.float32)
    pos = np.abs(np.random.default_rng(1).standard_normal((2, 5, 2))) + 0.1
    np.testing.assert_allclose(smear(pos, big), pos, rtol=0, atol=1e-30)
    # the gate weight enters as its bf16 value (0.1 -> 0.10009765625)
    z = smear(np.array([[[0.0, 0.0], [1.0, 0.0]]]), np.array([0.1, 0.0], dtype=np.float32))
    assert abs(z[0, 1, 0] - 1.0) < 1e-15 and abs(z[0, 1, 1] - 0.0) < 1e-15
    z = smear(np.array([[[3.0, 0.0], [1.0, 0.0]]]), np.array([0.1, 0.0], dtype=np.float32))
    assert abs(z[0, 1, 0] - (1.0 + 3.0 / (1.0 + math.exp(-0.10009765625)))) < 1e-15


def test_neutral_extras_reduce_to_the_plain_forward_exactly():
    c = _cfg()
    w = _weights(c)
    ex = _extras(c)
    ex["resid_lambdas"][:] = 1
    ex["x0_lambdas"][:] = 0
    ex["backout_lambda"] = np.float32(0)
    for g in ex["ve_gates"]:
        g[:] = 0
    del ex["smear_gate"]
    rng = np.random.default_rng(2)
    idx = rng.integers(0, c.vocab, (2, c.seq_len))
    base = oracle.forward(c, w, idx)["logits"]
    got = oracle.forward(c, w, idx, extras=ex)["logits"]
    assert np.array_equal(base, got)
    # and a non-neutral term does change the result
    ex["backout_lambda"] = np.float32(0.5)
    assert not np.allclose(oracle.forward(c, w, idx, extras=ex)["logits"], base)


def test_zero_projections_closed_form_with_all_extras():
    # attn_proj = mlp_proj = 0: the blocks only mix the stream, so the final
    # stream is kappa * x0 with a scalar kappa from the lambda recurrence, and
    # x0 = smear(wte[idx]) computed here by hand.
    c = _cfg(n_layer=5)
    w = _weights(c)
    for lw in w["layers"]:
        lw["attn_proj"][:] = 0
        lw["mlp_proj"][:] = 0
    ex = _extras(c)
    rng = np.random.default_rng(4)
    idx = rng.integers(0, c.vocab, (2, c.seq_len))
    res = oracle.forward(c, w, idx, extras=ex)["logits"]

    e = w["wte"][idx].astype(np.float64)
    gw = bf16_t(ex["smear_gate"])
    x0 = e.copy()
    for t in range(1, c.seq_len):
        sig = 1.0 / (1.0 + np.exp(-(e[:, t] @ gw)))
        x0[:, t] = e[:, t] + sig[:, None] * e[:, t - 1]
    coef, coef_mid = 1.0, None
    for l in range(c.n_layer):
        if l == c.n_layer // 2:
            coef_mid = coef
        coef = float(ex["resid_lambdas"][l]) * coef + float(ex["x0_lambdas"][l])
    kappa = coef - float(ex["backout_lambda"]) * coef_mid
    a = _rms(kappa * x0, c.norm_eps)
    want = 15.0 * np.tanh((a @ bf16_t(w["lm_head"]).T) / 15.0)
    np.testing.assert_allclose(res, want, rtol=1e-12, atol=1e-12)


def test_value_embedding_single_token_closed_form():
    # T = 1: the only key of the single query is itself, so each head's output is
    # its kv head's v.  With c_v = 0, v = gate * ve, and with GQA both query heads
    # read kv head 0: o = [g ve, g ve].  mlp_proj = 0.
    c = _cfg(n_layer=1, seq_len=1, n_head=2, n_kv_head=1)
    w = _weights(c)
    lw = w["layers"][0]
    lw["c_v"][:] = 0
    lw["mlp_proj"][:] = 0
    ex = {"value_embeds": [np.random.default_rng(7).standard_normal((c.vocab, c.head_dim)).astype(np.float32)],
          "ve_gates": [np.array([0.75], dtype=np.float32)]}
    idx = np.array([[5], [11]])
    res = oracle.forward(c, w, idx, extras=ex)["logits"]
    e = w["wte"][idx].astype(np.float64)
    gv = 0.75 * ex["value_embeds"][0][idx].astype(np.float64)  # [B,1,D]
    o = np.concatenate([gv, gv], axis=-1)  # both query heads read kv head 0
    x = e + o @ bf16_t(lw["attn_proj"]).T
    want = 15.0 * np.tanh((_rms(x, c.norm_eps) @ bf16_t(w["lm_head"]).T) / 15.0)
    np.testing.assert_allclose(res, want, rtol=1e-12, atol=1e-12)
    # a layer without a value embedding (layer 0 of 2) ignores its table and
    # gate; layer 1's gate is zero, so nothing may change at all
    c2 = _cfg(n_layer=2, seq_len=1, n_head=2, n_kv_head=1)
    w2 = _weights(c2)
    tab = np.random.default_rng(8).standard_normal((c2.vocab, c2.head_dim)).astype(np.float32)
    a = oracle.forward(c2, w2, idx, extras={"value_embeds": [tab, tab],
                                            "ve_gates": [np.ones(1, np.float32),
                                                         np.zeros(1, np.float32)]})["logits"]
    b = oracle.forward(c2, w2, idx)["logits"]
    assert np.array_equal(a, b)


def test_backout_subtracts_the_middle_stream():
    # L = 2, block 0 zero: the stream after one block is wte[idx] = x_mid.  Block
    # 1 at T = 1 adds rms(e) Wv^T Wp^T (its attention output is its own v).
    c = _cfg(n_layer=2, seq_len=1, n_head=1, n_kv_head=1)
    w = _weights(c)
    w["layers"][0]["attn_proj"][:] = 0
    w["layers"][0]["mlp_proj"][:] = 0
    w["layers"][1]["mlp_proj"][:] = 0
    lam = 0.3
    idx = np.array([[3], [17]])
    res = oracle.forward(c, w, idx, extras={"backout_lambda": np.float32(lam)})["logits"]
    e = w["wte"][idx].astype(np.float64)
    v = _rms(e, c.norm_eps) @ bf16_t(w["layers"][1]["c_v"]).T
    x = e + v @ bf16_t(w["layers"][1]["attn_proj"]).T - float(np.float32(lam)) * e
    want = 15.0 * np.tanh((_rms(x, c.norm_eps) @ bf16_t(w["lm_head"]).T) / 15.0)
    np.testing.assert_allclose(res, want, rtol=1e-12, atol=1e-12)


def test_extras_keep_causality_and_row_independence():
    c = _cfg()
    w = _weights(c)
    ex = _extras(c)
    rng = np.random.default_rng(6)
    idx = rng.integers(0, c.vocab, (2, c.seq_len))
    full = oracle.forward(c, w, idx, extras=ex)["logits"]
    t = 7
    idx2 = idx.copy()
    idx2[:, t] = (idx2[:, t] + 1) % c.vocab
    alt = oracle.forward(c, w, idx2, extras=ex)["logits"]
    np.testing.assert_array_equal(full[:, :t], alt[:, :t])
    assert not np.allclose(full[:, t:], alt[:, t:])
    one = oracle.forward(c, w, idx[1:], extras=ex)["logits"]
    np.testing.assert_allclose(one[0], full[1], rtol=0, atol=1e-13)


def test_extras_generator_is_seeded_and_shaped():
    s = SHAPES["tiny"]
    a, b = make_extras(s), make_extras(s)
    assert np.array_equal(a["smear_gate"], b["smear_gate"])
    assert a["smear_gate"].shape == (s.d_model,)
    assert a["resid_lambdas"].shape == (s.n_layer,) and a["x0_lambdas"].shape == (s.n_layer,)
    assert all(t.shape == (s.vocab, s.n_kv_head * s.head_dim) for t in a["value_embeds"])
    assert all(g.shape == (s.n_kv_head,) for g in a["ve_gates"])
    only = make_extras(s, layers=[1])
    assert only["value_embeds"][0] is None and np.array_equal(only["value_embeds"][1], a["value_embeds"][1])
