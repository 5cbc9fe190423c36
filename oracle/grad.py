"""fp64 backward of the nanochat block stack: the training micro-step's
``loss.backward()``.

TEST INFRASTRUCTURE ONLY (see the package docstring for who may import it).

"从文本到聊天模型" §6.5 (training loop: forward, loss, backward, optimizer
step) puts the backward right after the loss the forward computes.  This
module gives, for the block stack of ``model.forward`` (without fp8), the mean
loss and its gradient with respect to every fp32 master weight: wte, lm_head
and, per layer, c_q, c_k, c_v, attn_proj, c_fc, mlp_proj; with ``extras`` (the
same dict ``model.forward`` takes: smear, residual lambdas with x0, value
embeddings, backout; "Nanochat与nanoGPT对比" §1) also the gradients of those
parameters.

Readings where the pages are silent:

* The fp32 -> bf16 cast of a weight at matmul time passes the gradient
  through unchanged to the fp32 master weight (a straight-through cast, as
  autocast does): dW = dY^T X, and the backward products use the same bf16
  weight values as the forward.
* The loss is the mean over targets != -1; ignored positions get no gradient.
* Embedding rows collect the gradient of every position holding their token.

The backward is derived step by step from the forward's definitions, in the
forward's notation, the steps in reverse order.  ``cast`` lets a test swap the
bf16 cast for the identity (finite differences need a loss that is smooth in
the weights).  The pins are in ``tests/test_oracle_grad.py``.
"""
from __future__ import annotations

import numpy as np

from .model import F64, OracleConfig, backout_layer, embed, layer_windows, rope_tables, to_bf16, value_embed_layers


def _rms_rstd(u, eps):
    return 1.0 / np.sqrt(np.mean(u * u, axis=-1, keepdims=True) + eps)


def rmsnorm_backward(y, r, dy):
    """y = u r with r = (mean(u^2) + eps)^(-1/2) per row: du = r (dy - y mean(dy y))."""
    return r * (dy - y * np.mean(dy * y, axis=-1, keepdims=True))


def _rope_apply(u, cos, sin, sign):
    """Rotate pairs (u_i, u_{i+D/2}) by sign * t * theta_i (u: [B, T, heads, D])."""
    D = u.shape[-1]
    h = D // 2
    c = cos[None, :, None, :]
    s = sign * sin[None, :, None, :]
    a, b = u[..., :h], u[..., h:]
    return np.concatenate([a * c - b * s, a * s + b * c], axis=-1)


def _mask(T, W):
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    return (j <= i) & ((i - j) < W)


def attention_backward(q, k, v, do, W):
    """Gradients of o = softmax(q k^T / sqrt(D), window W, causal) v for one
    layer, with query head h reading kv head h // (H / Hkv).

    q [B, T, H, D], k and v [B, T, Hkv, D], do = dL/do [B, T, H, D].  With
    P the attention weights: dV = P^T dO, dP = dO V^T, dS = P o (dP - rowsum(dP o P)),
    dQ = dS K / sqrt(D), dK = dS^T Q / sqrt(D) (summed over the heads of a group).
    Returns (dq, dk, dv) and P [B, H, T, T].
    """
    B, T, H, D = q.shape
    Hkv = k.shape[2]
    G = H // Hkv
    scale = 1.0 / np.sqrt(D)
    m = _mask(T, W)
    dq = np.zeros((B, T, H, D))
    dk = np.zeros((B, T, Hkv, D))
    dv = np.zeros((B, T, Hkv, D))
    P = np.empty((B, H, T, T))
    for h in range(H):
        g = h // G
        sc = np.einsum("bid,bjd->bij", q[:, :, h], k[:, :, g]) * scale
        sc = np.where(m[None], sc, -np.inf)
        sc = sc - sc.max(axis=-1, keepdims=True)
        e = np.exp(sc)
        Ph = e / e.sum(axis=-1, keepdims=True)
        P[:, h] = Ph
        dv[:, :, g] += np.einsum("bij,bid->bjd", Ph, do[:, :, h])
        dP = np.einsum("bid,bjd->bij", do[:, :, h], v[:, :, g])
        dS = Ph * (dP - np.sum(dP * Ph, axis=-1, keepdims=True)) * scale
        dq[:, :, h] = np.einsum("bij,bjd->bid", dS, k[:, :, g])
        dk[:, :, g] += np.einsum("bij,bid->bjd", dS, q[:, :, h])
    return dq, dk, dv, P


def _forward(cfg: OracleConfig, weights: dict, idx: np.ndarray, targets: np.ndarray, cast, extras=None):
    """The forward of ``model.forward`` keeping what the backward reads."""
    ex = extras or {}
    idx = np.asarray(idx)
    targets = np.asarray(targets)
    B, T = idx.shape
    H, Hkv, D = cfg.n_head, cfg.n_kv_head, cfg.head_dim
    G = H // Hkv
    eps, cap = cfg.norm_eps, cfg.softcap
    windows = layer_windows(cfg)
    cos, sin = rope_tables(T, D, cfg.rope_base)
    scale = 1.0 / np.sqrt(D)
    Wb = [{k: cast(v) for k, v in lw.items()} for lw in weights["layers"]]
    Wlm = cast(weights["lm_head"])

    # ---------------- forward, keeping what the backward reads
    x = embed(weights["wte"], idx)
    sm = None
    if "smear_gate" in ex:  # x_t + sigmoid(x_t . w_g) x_{t-1}
        wg = cast(np.asarray(ex["smear_gate"]).reshape(-1))
        e = x
        g = 1.0 / (1.0 + np.exp(-(e @ wg)))
        prev = np.zeros_like(e)
        prev[:, 1:] = e[:, :-1]
        x = e + g[..., None] * prev
        sm = dict(e=e, g=g, prev=prev, wg=wg)
    x0 = x
    L = len(Wb)
    ve_on = value_embed_layers(L) if "value_embeds" in ex else [False] * L
    mid = backout_layer(L) if "backout_lambda" in ex else -1
    x_back = None
    saved = []
    for l, lw in enumerate(Wb):
        s = {}
        if l == mid:
            x_back = x
        if "resid_lambdas" in ex:
            s["x_pre"] = x
            x = F64(ex["resid_lambdas"][l]) * x + F64(ex["x0_lambdas"][l]) * x0
        s["x_in"] = x
        r1 = _rms_rstd(x, eps)
        a = x * r1
        uq = (a @ lw["c_q"].T).reshape(B, T, H, D)
        uk = (a @ lw["c_k"].T).reshape(B, T, Hkv, D)
        v = (a @ lw["c_v"].T).reshape(B, T, Hkv, D)
        if ve_on[l]:  # v + gate * ve[idx], one gate per kv head
            ve = embed(ex["value_embeds"][l], idx).reshape(B, T, Hkv, D)
            v = v + np.asarray(ex["ve_gates"][l], dtype=F64)[None, None, :, None] * ve
            s["ve"] = ve
        pq = _rope_apply(uq, cos, sin, 1.0)
        pk = _rope_apply(uk, cos, sin, 1.0)
        rq, rk = _rms_rstd(pq, eps), _rms_rstd(pk, eps)
        q, k = pq * rq, pk * rk
        m = _mask(T, windows[l])
        P = np.empty((B, H, T, T))
        o = np.empty((B, T, H, D))
        for h in range(H):
            g = h // G
            sc = np.einsum("bid,bjd->bij", q[:, :, h], k[:, :, g]) * scale
            sc = np.where(m[None], sc, -np.inf)
            sc = sc - sc.max(axis=-1, keepdims=True)
            e = np.exp(sc)
            P[:, h] = e / e.sum(axis=-1, keepdims=True)
            o[:, :, h] = np.einsum("bij,bjd->bid", P[:, h], v[:, :, g])
        of = o.reshape(B, T, H * D)
        x_mid = x + of @ lw["attn_proj"].T
        r2 = _rms_rstd(x_mid, eps)
        a2 = x_mid * r2
        u = a2 @ lw["c_fc"].T
        hh = np.maximum(u, 0.0) ** 2
        x = x_mid + hh @ lw["mlp_proj"].T
        s.update(r1=r1, a=a, q=q, k=k, v=v, rq=rq, rk=rk, P=P, of=of, x_mid=x_mid, r2=r2, a2=a2, u=u, h=hh,
                 W=windows[l])
        saved.append(s)
    if x_back is not None:
        x = x - F64(ex["backout_lambda"]) * x_back
    rf = _rms_rstd(x, eps)
    af = x * rf
    z = af @ Wlm.T
    lg = cap * np.tanh(z / cap)
    mx = lg.max(axis=-1, keepdims=True)
    lse = mx[..., 0] + np.log(np.exp(lg - mx).sum(axis=-1))
    valid = targets != -1
    n = int(valid.sum())
    tl = np.where(valid, lse - np.take_along_axis(lg, np.where(valid, targets, 0)[..., None], -1)[..., 0], 0.0)
    loss = float(tl.sum() / n) if n else float("nan")
    return loss, dict(saved=saved, Wb=Wb, Wlm=Wlm, lg=lg, lse=lse, valid=valid, n=n, af=af, rf=rf, cos=cos,
                      sin=sin, idx=idx, targets=targets, ex=ex, sm=sm, x0=x0, ve_on=ve_on, mid=mid,
                      x_back=x_back)


def _term_magnitude(dy, x):
    """sum over tokens of |dy_m|^T |x_m|: the size of the terms whose sum is the
    weight gradient dy^T x (a scale for comparing a rounded computation of it)."""
    return np.abs(dy.reshape(-1, dy.shape[-1])).T @ np.abs(x.reshape(-1, x.shape[-1]))


def forward_backward(cfg: OracleConfig, weights: dict, idx: np.ndarray, targets: np.ndarray, cast=to_bf16,
                     magnitudes: bool = False, extras: dict = None):
    """Returns (loss, grads) with grads = {"wte", "lm_head", "layers": [{...}]},
    each the same shape as its weight, float64.  With magnitudes=True, returns
    (loss, grads, mags): mags has the same structure and holds, per gradient
    element, the sum of the absolute values of the per-token terms it adds up
    (for wte, of the rows it gathers).

    With ``extras`` (keys as in ``model.forward``) grads and mags also hold
    "smear_gate" [C], "resid_lambdas" and "x0_lambdas" [L], "value_embeds" and
    "ve_gates" (lists of L entries, None on layers without a value embedding)
    and "backout_lambda" (scalar), for the keys present.  The gates, lambdas
    and embedding tables enter the forward unrounded; the smear gate's weight is
    cast like every linear layer's (straight through)."""
    loss, c = _forward(cfg, weights, idx, targets, cast, extras)
    saved, Wb, Wlm, lg, lse, valid, n = c["saved"], c["Wb"], c["Wlm"], c["lg"], c["lse"], c["valid"], c["n"]
    af, rf, cos, sin, idx, targets = c["af"], c["rf"], c["cos"], c["sin"], c["idx"], c["targets"]
    B, T = idx.shape
    C, H, Hkv, D = cfg.d_model, cfg.n_head, cfg.n_kv_head, cfg.head_dim
    cap = cfg.softcap

    # ---------------- backward
    grads = {"layers": [dict() for _ in Wb]}
    p = np.exp(lg - lse[..., None])
    onehot = np.zeros_like(lg)
    bi, ti = np.nonzero(valid)
    onehot[bi, ti, targets[bi, ti]] = 1.0
    dlg = np.where(valid[..., None], (p - onehot) / max(n, 1), 0.0)
    dz = dlg * (1.0 - (lg / cap) ** 2)  # d/dz cap tanh(z / cap)
    grads["lm_head"] = np.einsum("btv,btc->vc", dz, af)
    mags = {"layers": [dict() for _ in Wb]}
    if magnitudes:
        mags["lm_head"] = _term_magnitude(dz, af)
    daf = dz @ Wlm
    dx = rmsnorm_backward(af, rf, daf)
    ex, x0, ve_on, mid, x_back = c["ex"], c["x0"], c["ve_on"], c["mid"], c["x_back"]
    L = len(Wb)
    lambdas = "resid_lambdas" in ex
    dx_final = dx  # gradient of the stream entering the final norm
    if x_back is not None:  # x_final = x_L - lambda x_back
        grads["backout_lambda"] = -float(np.sum(dx_final * x_back))
        mags["backout_lambda"] = float(np.sum(np.abs(dx_final * x_back)))
    if lambdas:
        for key in ("resid_lambdas", "x0_lambdas"):
            grads[key] = np.zeros(L)
            mags[key] = np.zeros(L)
        dx0 = np.zeros_like(dx)
    if "value_embeds" in ex:
        for key in ("value_embeds", "ve_gates"):
            grads[key] = [None] * L
            mags[key] = [None] * L
    for l in range(len(Wb) - 1, -1, -1):
        lw, s, gl = Wb[l], saved[l], grads["layers"][l]
        # MLP: x = x_mid + relu(u)^2 W_mp^T with u = norm(x_mid) W_fc^T
        gl["mlp_proj"] = np.einsum("btc,btf->cf", dx, s["h"])
        dh = dx @ lw["mlp_proj"]
        du = dh * 2.0 * np.maximum(s["u"], 0.0)
        gl["c_fc"] = np.einsum("btf,btc->fc", du, s["a2"])
        da2 = du @ lw["c_fc"]
        dx_mid = dx + rmsnorm_backward(s["a2"], s["r2"], da2)
        # attention block: x_mid = x_in + o W_p^T
        gl["attn_proj"] = np.einsum("btc,bte->ce", dx_mid, s["of"])
        do = (dx_mid @ lw["attn_proj"]).reshape(B, T, H, D)
        dq, dk, dv, _ = attention_backward(s["q"], s["k"], s["v"], do, s["W"])
        # QK-norm after RoPE, then the inverse rotation
        duq = _rope_apply(rmsnorm_backward(s["q"], s["rq"], dq), cos, sin, -1.0).reshape(B, T, H * D)
        duk = _rope_apply(rmsnorm_backward(s["k"], s["rk"], dk), cos, sin, -1.0).reshape(B, T, Hkv * D)
        dvf = dv.reshape(B, T, Hkv * D)
        if ve_on[l]:  # v = a W_v^T + gate * ve[idx]
            gate = np.asarray(ex["ve_gates"][l], dtype=F64)
            rows = (gate[None, None, :, None] * dv).reshape(-1, Hkv * D)
            gve = np.zeros(np.asarray(ex["value_embeds"][l]).shape, dtype=F64)
            np.add.at(gve, idx.reshape(-1), rows)
            grads["value_embeds"][l] = gve
            grads["ve_gates"][l] = np.einsum("btgd,btgd->g", dv, s["ve"])
            mve = np.zeros_like(gve)
            np.add.at(mve, idx.reshape(-1), np.abs(rows))
            mags["value_embeds"][l] = mve
            mags["ve_gates"][l] = np.einsum("btgd,btgd->g", np.abs(dv), np.abs(s["ve"]))
        gl["c_q"] = np.einsum("bte,btc->ec", duq, s["a"])
        gl["c_k"] = np.einsum("bte,btc->ec", duk, s["a"])
        gl["c_v"] = np.einsum("bte,btc->ec", dvf, s["a"])
        if magnitudes:
            ml = mags["layers"][l]
            ml["mlp_proj"] = _term_magnitude(dx, s["h"])
            ml["c_fc"] = _term_magnitude(du, s["a2"])
            ml["attn_proj"] = _term_magnitude(dx_mid, s["of"])
            ml["c_q"] = _term_magnitude(duq, s["a"])
            ml["c_k"] = _term_magnitude(duk, s["a"])
            ml["c_v"] = _term_magnitude(dvf, s["a"])
        da = duq @ lw["c_q"] + duk @ lw["c_k"] + dvf @ lw["c_v"]
        dx = dx_mid + rmsnorm_backward(s["a"], s["r1"], da)  # of the block's (mixed) input
        if lambdas:  # x_in = resid_lambda x_pre + x0_lambda x0
            grads["resid_lambdas"][l] = np.sum(dx * s["x_pre"])
            grads["x0_lambdas"][l] = np.sum(dx * x0)
            mags["resid_lambdas"][l] = np.sum(np.abs(dx * s["x_pre"]))
            mags["x0_lambdas"][l] = np.sum(np.abs(dx * x0))
            dx0 = dx0 + F64(ex["x0_lambdas"][l]) * dx
            dx = F64(ex["resid_lambdas"][l]) * dx
        if l == mid:  # the stream entering block `mid` is also subtracted before the final norm
            dx = dx - F64(ex["backout_lambda"]) * dx_final
    if lambdas:
        dx = dx + dx0
    sm = c["sm"]
    if sm is not None:  # x = e + g prev with g = sigmoid(e . w_g), prev_t = e_{t-1}
        e, g, prev, wg = sm["e"], sm["g"], sm["prev"], sm["wg"]
        dzg = np.sum(dx * prev, axis=-1) * g * (1.0 - g)
        grads["smear_gate"] = np.einsum("bt,btc->c", dzg, e)
        mags["smear_gate"] = np.einsum("bt,btc->c", np.abs(dzg), np.abs(e))
        de = dx + dzg[..., None] * wg[None, None, :]
        de[:, :-1] += g[:, 1:, None] * dx[:, 1:]
        dx = de
    dwte = np.zeros(np.asarray(weights["wte"]).shape, dtype=F64)
    np.add.at(dwte, idx.reshape(-1), dx.reshape(-1, C))
    grads["wte"] = dwte
    if not magnitudes:
        return loss, grads
    mwte = np.zeros_like(dwte)
    np.add.at(mwte, idx.reshape(-1), np.abs(dx.reshape(-1, C)))
    mags["wte"] = mwte
    return loss, grads, mags


def loss_only(cfg: OracleConfig, weights: dict, idx, targets, cast=to_bf16, extras: dict = None) -> float:
    """The same loss without the backward (for finite differences)."""
    return _forward(cfg, weights, idx, targets, cast, extras)[0]
