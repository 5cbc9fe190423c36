"""Pins of the oracle's backward through the further terms of the full nanochat
forward ("Nanochat与nanoGPT对比" §1: smear, residual lambdas with x0, value
embeddings, backout), ``oracle.grad.forward_backward(..., extras=...)``.

Nothing here retypes the backward:

* the loss it returns equals ``oracle.forward``'s with the same extras (the
  separately written and separately pinned forward of ``oracle/model.py``);
* central finite differences of the loss (weight cast set to the identity) against
  the analytic directional derivative, for every extras parameter, each
  embedding table, and every block weight of one layer;
* the per-element term magnitudes bound the gradients;
* extras that leave the forward unchanged (zero value-embedding gates, unit
  resid lambdas, zero x0 lambdas, zero backout) leave every block gradient
  equal to the plain backward's.
"""
import numpy as np
import pytest

import oracle
from oracle import OracleConfig
from oracle.grad import forward_backward, loss_only

NAMES = ("c_q", "c_k", "c_v", "attn_proj", "c_fc", "mlp_proj")


def _cfg(**kw):
    base = dict(n_layer=4, d_model=32, n_head=2, n_kv_head=1, head_dim=16, seq_len=12, vocab=40,
                short_window=4)
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
    return {"smear_gate": (0.3 * rng.standard_normal(c.d_model)).astype(np.float32),
            "resid_lambdas": (1 + 0.2 * rng.standard_normal(L)).astype(np.float32),
            "x0_lambdas": (0.2 * rng.standard_normal(L)).astype(np.float32),
            "backout_lambda": np.float32(0.4),
            "value_embeds": [(0.5 * rng.standard_normal((c.vocab, kvw))).astype(np.float32) for _ in range(L)],
            "ve_gates": [rng.standard_normal(c.n_kv_head).astype(np.float32) for _ in range(L)]}


def _ident(a):
    return np.asarray(a, dtype=np.float64)


def _batch(c, seed):
    rng = np.random.default_rng(seed)
    idx = rng.integers(0, c.vocab, (2, c.seq_len))
    tgt = rng.integers(0, c.vocab, (2, c.seq_len))
    tgt[1, ::4] = -1
    return idx, tgt


def test_loss_equals_the_pinned_forward_with_extras():
    c = _cfg()
    w, ex = _weights(c), _extras(c)
    idx, tgt = _batch(c, 1)
    loss, _ = forward_backward(c, w, idx, tgt, extras=ex)
    assert loss == pytest.approx(oracle.forward(c, w, idx, tgt, extras=ex)["loss"], rel=1e-13)


def _ex_paths(c, ex):
    from oracle.model import value_embed_layers
    on = value_embed_layers(c.n_layer)
    paths = [("smear_gate",), ("resid_lambdas",), ("x0_lambdas",), ("backout_lambda",)]
    paths += [("value_embeds", l) for l in range(c.n_layer) if on[l]]
    paths += [("ve_gates", l) for l in range(c.n_layer) if on[l]]
    return paths


def _ex_get(d, p):
    return d[p[0]] if len(p) == 1 else d[p[0]][p[1]]


def _ex_with(ex, p, value):
    out = {k: (list(v) if isinstance(v, list) else v) for k, v in ex.items()}
    if len(p) == 1:
        out[p[0]] = value
    else:
        out[p[0]][p[1]] = value
    return out


def test_finite_differences_every_extras_parameter():
    c = _cfg()
    w, ex = _weights(c), _extras(c)
    idx, tgt = _batch(c, 2)
    _, g = forward_backward(c, w, idx, tgt, cast=_ident, extras=ex)
    rng = np.random.default_rng(3)
    eps = 1e-6
    for p in _ex_paths(c, ex):
        base = np.asarray(_ex_get(ex, p), dtype=np.float64)
        E = rng.standard_normal(base.shape)
        up = loss_only(c, w, idx, tgt, cast=_ident, extras=_ex_with(ex, p, base + eps * E))
        dn = loss_only(c, w, idx, tgt, cast=_ident, extras=_ex_with(ex, p, base - eps * E))
        num = (up - dn) / (2 * eps)
        ana = float(np.sum(np.asarray(_ex_get(g, p)) * E))
        assert abs(num - ana) <= 1e-6 * max(1.0, abs(ana)), (p, num, ana)


@pytest.mark.parametrize("layer", [0, 3])
def test_finite_differences_weights_through_the_extras(layer):
    c = _cfg()
    w, ex = _weights(c), _extras(c)
    idx, tgt = _batch(c, 4)
    _, g = forward_backward(c, w, idx, tgt, cast=_ident, extras=ex)
    rng = np.random.default_rng(5 + layer)
    eps = 1e-6
    targets = [("wte", None), ("lm_head", None)] + [(n, layer) for n in NAMES]
    for name, l in targets:
        base = (w[name] if l is None else w["layers"][l][name]).astype(np.float64)
        E = rng.standard_normal(base.shape)

        def with_w(v):
            out = {"wte": w["wte"], "lm_head": w["lm_head"], "layers": [dict(lw) for lw in w["layers"]]}
            if l is None:
                out[name] = v
            else:
                out["layers"][l][name] = v
            return out

        num = (loss_only(c, with_w(base + eps * E), idx, tgt, cast=_ident, extras=ex)
               - loss_only(c, with_w(base - eps * E), idx, tgt, cast=_ident, extras=ex)) / (2 * eps)
        gg = g[name] if l is None else g["layers"][l][name]
        ana = float(np.sum(gg * E))
        assert abs(num - ana) <= 1e-6 * max(1.0, abs(ana)), (name, l, num, ana)


def test_term_magnitudes_bound_the_extras_gradients():
    c = _cfg()
    w, ex = _weights(c), _extras(c)
    idx, tgt = _batch(c, 6)
    _, g, m = forward_backward(c, w, idx, tgt, extras=ex, magnitudes=True)
    for p in _ex_paths(c, ex):
        gv, mv = np.asarray(_ex_get(g, p)), np.asarray(_ex_get(m, p))
        assert np.all(np.abs(gv) <= mv * (1 + 1e-12) + 1e-300), p
        assert np.any(mv > 0), p


def test_neutral_extras_give_the_plain_gradients():
    c = _cfg()
    w = _weights(c)
    ex = _extras(c)
    L = c.n_layer
    # (a smear with a zero weight is not neutral: its gate is 1/2)
    ex = {"resid_lambdas": np.ones(L, dtype=np.float32), "x0_lambdas": np.zeros(L, dtype=np.float32),
          "backout_lambda": np.float32(0.0),
          "value_embeds": ex["value_embeds"], "ve_gates": [np.zeros(c.n_kv_head, dtype=np.float32)] * L}
    idx, tgt = _batch(c, 7)
    l0, g0 = forward_backward(c, w, idx, tgt)
    l1, g1 = forward_backward(c, w, idx, tgt, extras=ex)
    assert l1 == pytest.approx(l0, rel=1e-14)
    for l in range(L):
        for n in NAMES:
            np.testing.assert_allclose(g1["layers"][l][n], g0["layers"][l][n], rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(g1["wte"], g0["wte"], rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(g1["lm_head"], g0["lm_head"], rtol=1e-12, atol=1e-15)
