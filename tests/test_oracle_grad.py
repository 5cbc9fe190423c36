"""Pins of the oracle's backward (``oracle/grad.py``).

"从文本到聊天模型" §6.5 puts ``loss.backward()`` right after the forward's loss.
Nothing here retypes the oracle's backward:

* central finite differences of the loss (with the weight cast set to the
  identity, so the loss is smooth in the weights) against the analytic
  directional derivative, for every weight tensor;
* torch float64 autograd through an independently written composition of the
  forward (``F.rms_norm``, complex-number RoPE, ``F.scaled_dot_product_attention``
  with an explicit window mask, ``F.cross_entropy(ignore_index=-1)``), with the
  bf16 cast made straight-through -- the oracle's reading -- for every weight;
* ignored targets: a position whose target is -1 contributes no gradient.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from oracle import OracleConfig
from oracle.grad import forward_backward, loss_only

NAMES = ("c_q", "c_k", "c_v", "attn_proj", "c_fc", "mlp_proj")


def _cfg(**kw):
    base = dict(n_layer=2, d_model=32, n_head=4, n_kv_head=2, head_dim=16, seq_len=12, vocab=40,
                short_window=5)
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


def _ident(a):
    return np.asarray(a, dtype=np.float64)


def _with(w, path, value):
    out = {"wte": w["wte"], "lm_head": w["lm_head"], "layers": [dict(lw) for lw in w["layers"]]}
    if len(path) == 1:
        out[path[0]] = value
    else:
        out["layers"][path[0]][path[1]] = value
    return out


def _get(tree, path):
    return tree[path[0]] if len(path) == 1 else tree["layers"][path[0]][path[1]]


def test_loss_matches_the_forward():
    c = _cfg()
    w = _weights(c)
    rng = np.random.default_rng(1)
    idx = rng.integers(0, c.vocab, (2, c.seq_len))
    tgt = rng.integers(0, c.vocab, (2, c.seq_len))
    tgt[1, ::3] = -1
    loss, _ = forward_backward(c, w, idx, tgt)
    assert loss == pytest.approx(oracle.forward(c, w, idx, tgt)["loss"], rel=1e-13)


def test_finite_differences_every_weight():
    c = _cfg()
    w = _weights(c)
    rng = np.random.default_rng(2)
    idx = rng.integers(0, c.vocab, (2, c.seq_len))
    tgt = rng.integers(0, c.vocab, (2, c.seq_len))
    tgt[0, 4] = -1
    _, g = forward_backward(c, w, idx, tgt, cast=_ident)
    paths = [("wte",), ("lm_head",)] + [(l, n) for l in range(c.n_layer) for n in NAMES]
    eps = 1e-6
    for p in paths:
        base = _get(w, p).astype(np.float64)
        E = rng.standard_normal(base.shape)
        up = loss_only(c, _with(w, p, base + eps * E), idx, tgt, cast=_ident)
        dn = loss_only(c, _with(w, p, base - eps * E), idx, tgt, cast=_ident)
        num = (up - dn) / (2 * eps)
        ana = float(np.sum(_get(g, p) * E))
        assert abs(num - ana) <= 1e-6 * max(1.0, abs(ana)), (p, num, ana)


def _torch_loss(c, w, idx, tgt):
    """Independent torch composition of the forward, weights straight-through bf16."""
    f64 = torch.float64
    leaves = {}

    def leaf(name, a):
        t = torch.tensor(np.asarray(a, dtype=np.float64), dtype=f64, requires_grad=True)
        leaves[name] = t
        return t

    def st_bf16(t):  # value of the bf16 cast, gradient of the identity
        return t + (t.to(torch.bfloat16).to(f64) - t).detach()

    B, T = idx.shape
    C, H, Hkv, D, V = c.d_model, c.n_head, c.n_kv_head, c.head_dim, c.vocab
    wte = leaf("wte", w["wte"])
    lm = leaf("lm_head", w["lm_head"])
    x = wte[torch.as_tensor(idx)]
    pos = torch.arange(T, dtype=f64)
    inv = c.rope_base ** (-torch.arange(0, D, 2, dtype=f64) / D)
    rot = torch.polar(torch.ones(T, D // 2, dtype=f64), pos[:, None] * inv[None, :])  # e^{i t theta}

    def rope(u):  # [B, T, h, D]; pair (u_i, u_{i+D/2}) as the complex number u_i + i u_{i+D/2}
        z = torch.complex(u[..., : D // 2], u[..., D // 2:]) * rot[None, :, None, :]
        return torch.cat([z.real, z.imag], dim=-1)

    windows = oracle.layer_windows(c)
    for l, lw in enumerate(w["layers"]):
        W = {n: st_bf16(leaf(f"{l}.{n}", lw[n])) for n in NAMES}
        a = F.rms_norm(x, (C,), eps=c.norm_eps)
        q = F.rms_norm(rope((a @ W["c_q"].T).view(B, T, H, D)), (D,), eps=c.norm_eps)
        k = F.rms_norm(rope((a @ W["c_k"].T).view(B, T, Hkv, D)), (D,), eps=c.norm_eps)
        v = (a @ W["c_v"].T).view(B, T, Hkv, D)
        rep = H // Hkv
        kk = k.repeat_interleave(rep, dim=2).transpose(1, 2)
        vv = v.repeat_interleave(rep, dim=2).transpose(1, 2)
        i = torch.arange(T)[:, None]
        j = torch.arange(T)[None, :]
        mask = (j <= i) & (i - j < windows[l])
        o = F.scaled_dot_product_attention(q.transpose(1, 2), kk, vv, attn_mask=mask)
        x = x + o.transpose(1, 2).reshape(B, T, H * D) @ W["attn_proj"].T
        a2 = F.rms_norm(x, (C,), eps=c.norm_eps)
        x = x + torch.relu(a2 @ W["c_fc"].T).square() @ W["mlp_proj"].T
    z = F.rms_norm(x, (C,), eps=c.norm_eps) @ st_bf16(lm).T
    logits = c.softcap * torch.tanh(z / c.softcap)
    loss = F.cross_entropy(logits.view(-1, V), torch.as_tensor(tgt).view(-1), ignore_index=-1)
    loss.backward()
    return loss.item(), leaves


@pytest.mark.parametrize("kw", [dict(), dict(n_kv_head=4), dict(n_layer=3, short_window=3)])
def test_matches_torch_autograd(kw):
    c = _cfg(**kw)
    w = _weights(c, seed=7)
    rng = np.random.default_rng(3)
    idx = rng.integers(0, c.vocab, (2, c.seq_len))
    tgt = rng.integers(0, c.vocab, (2, c.seq_len))
    tgt[1, 2] = -1
    loss, g = forward_backward(c, w, idx, tgt)
    tloss, leaves = _torch_loss(c, w, idx, tgt)
    assert loss == pytest.approx(tloss, rel=1e-12)
    np.testing.assert_allclose(g["wte"], leaves["wte"].grad.numpy(), rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(g["lm_head"], leaves["lm_head"].grad.numpy(), rtol=1e-9, atol=1e-12)
    for l in range(c.n_layer):
        for n in NAMES:
            np.testing.assert_allclose(g["layers"][l][n], leaves[f"{l}.{n}"].grad.numpy(), rtol=1e-9,
                                       atol=1e-12, err_msg=f"layer {l} {n}")


def test_ignored_positions_get_no_gradient():
    c = _cfg(n_layer=1)
    w = _weights(c)
    rng = np.random.default_rng(4)
    idx = rng.integers(0, c.vocab, (1, c.seq_len))
    tgt = np.full((1, c.seq_len), -1)
    tgt[0, 3] = 7  # one counted position: only positions <= 3 can influence it
    _, g = forward_backward(c, w, idx, tgt)
    later = set(idx[0, 4:]) - set(idx[0, :4])
    for tok in later:  # tokens seen only after the counted position
        assert not g["wte"][tok].any()
    assert g["lm_head"].any()


def test_term_magnitudes_bound_the_gradient_and_are_exact_for_one_term():
    """The per-element term magnitudes (the scale the GPU gradients are compared
    against): by the triangle inequality they bound |gradient| element by
    element; with one token and one target every gradient element is a single
    term, so they equal |gradient| (wte: a single gathered row); the gradient
    values themselves do not change when magnitudes are asked for."""
    c = _cfg()
    w = _weights(c)
    rng = np.random.default_rng(8)
    idx = rng.integers(0, c.vocab, (2, c.seq_len))
    tgt = rng.integers(0, c.vocab, (2, c.seq_len))
    loss0, g0 = forward_backward(c, w, idx, tgt)
    loss, g, m = forward_backward(c, w, idx, tgt, magnitudes=True)
    assert loss == loss0
    leaves = [("wte",), ("lm_head",)] + [(l, n) for l in range(c.n_layer) for n in NAMES]
    for path in leaves:
        assert np.array_equal(_get(g, path), _get(g0, path))
        assert np.all(_get(m, path) >= np.abs(_get(g, path)) * (1 - 1e-12)), path
    c1 = _cfg(seq_len=1)
    _, g1, m1 = forward_backward(c1, w, idx[:1, :1], tgt[:1, :1], magnitudes=True)
    for path in leaves:
        np.testing.assert_allclose(_get(m1, path), np.abs(_get(g1, path)), rtol=1e-12, atol=1e-300,
                                   err_msg=str(path))
