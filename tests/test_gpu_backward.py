"""GPU parity of the backward (nc_forward_backward and the two backward
products) against the oracle's ``oracle.grad.forward_backward``.

"从文本到聊天模型" §6.5: the training step's loss.backward().  Bars:

* dgrad / wgrad products on identical 16-bit inputs: the oracle forms them
  exactly in fp64; the kernel accumulates exact 16-bit products in fp32, so
  |err| <= 1e-5 |dy| |w| (or |dy|^T |x|) elementwise.
* whole-step gradients, element by element: a weight gradient element is a
  sum over tokens of products dy_m x_m, and the kernel forms each factor after
  a chain of 16-bit roundings (activations in the forward; the logit
  gradient, dx, dh, dO, P, dS, dq/dk/dv in the backward), each moving a value
  by at most u = 2^-11 (fp16) or 2^-8 (bf16) relative.  Along the longest chain
  there are at most 4 + 8 L of them for L layers, which bounds the error of
  every element by (4 + 8 L) u sum_m |dy_m| |x_m|, the magnitude the oracle
  reports beside each gradient (``magnitudes=True``).  Two effects escape a
  purely relative bound and get an absolute term of 4 u max|gradient| per
  tensor: factors that underflow into the 16-bit subnormal range (softmax
  probabilities of rarely chosen tokens in the logit gradient), and dx at a
  layer's input, which is a difference of much larger path contributions
  (the wte rows).  Also per tensor: relative Frobenius error <= 2e-2 (fp16) or
  5e-2 (bf16) and cosine >= 0.999; the loss within 5e-3 relative.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle.grad import forward_backward as oracle_fb
from workloads import SHAPES, ModelShape, make_tokens, make_weights

pytestmark = pytest.mark.gpu

DEV = "cuda"
NAMES = ("c_q", "c_k", "c_v", "attn_proj", "c_fc", "mlp_proj")


@pytest.mark.parametrize("M,N,K", [(300, 768, 1280), (1000, 128, 256), (5000, 768, 1280), (64, 1280, 5120)])
def test_linear_dgrad_wgrad(gpu, M, N, K):
    rng = np.random.default_rng(M + N + K)
    dy = rng.standard_normal((M, N)).astype(np.float16)
    w = (rng.standard_normal((N, K)) * 0.05).astype(np.float16)
    x = rng.standard_normal((M, K)).astype(np.float16)
    tdy, tw, tx = (torch.from_numpy(a).to(DEV) for a in (dy, w, x))
    dx = torch.empty((M, K), dtype=torch.float32, device=DEV)
    gpu.linear_dgrad(tdy, tw, dx)
    dx16 = torch.empty((M, K), dtype=torch.float16, device=DEV)
    gpu.linear_dgrad(tdy, tw, dx16)
    dw0 = rng.standard_normal((N, K)).astype(np.float32)
    dw = torch.from_numpy(dw0).to(DEV)
    gpu.linear_wgrad(tdy, tx, dw, alpha=0.5)
    torch.cuda.synchronize()
    dy64, w64, x64 = (a.astype(np.float64) for a in (dy, w, x))
    want = dy64 @ w64
    mag = np.abs(dy64) @ np.abs(w64)
    err = np.abs(dx.cpu().numpy() - want)
    assert (err <= 1e-5 * mag + 1e-6).all(), f"dgrad max err/mag {np.max(err / (mag + 1e-9)):.3e}"
    np.testing.assert_allclose(dx16.float().cpu().numpy(), want, rtol=2e-3, atol=2e-3 * np.abs(want).max())
    want_w = dw0 + 0.5 * (dy64.T @ x64)
    mag_w = 0.5 * (np.abs(dy64).T @ np.abs(x64))
    err_w = np.abs(dw.cpu().numpy() - want_w)
    assert (err_w <= 1e-5 * mag_w + 1e-5).all(), f"wgrad max err/mag {np.max(err_w / (mag_w + 1e-9)):.3e}"


def _oracle_cfg(s):
    return oracle.OracleConfig(s.n_layer, s.d_model, s.n_head, s.n_kv_head, s.head_dim, s.seq_len, s.vocab,
                               short_window=s.short_window)


def _compare(gpu_grads, want, bar, mags=None, c=None, n_chain=20):
    """Per tensor: relative Frobenius error <= bar and cosine >= 0.999; with the
    oracle's term magnitudes, every element within c * magnitude."""
    rows, bad = [], []

    def one(name, a, b, m):
        a = a.detach().double().cpu().numpy()
        rel = np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30)
        cos = float(np.sum(a * b) / max(np.linalg.norm(a) * np.linalg.norm(b), 1e-30))
        line = f"{name}: rel {rel:.3e} cos {cos:.6f}"
        ok = rel <= bar and cos >= 0.999
        if m is not None:
            err = np.abs(a - b)
            top = float(np.abs(b).max())
            kappa = 4.0 * c / n_chain  # 4 u
            ratio = float(np.max(err / np.maximum(m, 1e-30)))
            need = float(np.max((err - c * m) / max(top, 1e-30)))
            line += f" max err/magnitude {ratio:.3e} (c {c:.3e}); max excess/max|g| {need:.3e} (bar {kappa:.3e})"
            ok = ok and bool(np.all(err <= c * m + kappa * top + 1e-12))
        rows.append(line)
        if not ok:
            bad.append(name)

    mg = mags if mags is not None else {"wte": None, "lm_head": None, "layers": [dict() for _ in want["layers"]]}
    one("wte", gpu_grads["wte"], want["wte"], mg["wte"])
    one("lm_head", gpu_grads["lm_head"], want["lm_head"], mg["lm_head"])
    for l, lw in enumerate(want["layers"]):
        for n in NAMES:
            one(f"{l}.{n}", gpu_grads["layers"][l][n], lw[n], mg["layers"][l].get(n))
    print("\n".join(rows))
    assert not bad, "gradients off: " + ", ".join(bad) + "\n" + "\n".join(rows)
    return rows


def _chain_bar(n_layer, bf16=False):
    """(4 + 8 L) 16-bit roundings of u each along the longest chain."""
    return (4 + 8 * n_layer) * (2.0 ** -8 if bf16 else 2.0 ** -11)
# (the absolute term's 4 u is recovered in _compare as 4 c / (4 + 8 L); every case here has L = 2)


def _run(gpu, s, act_dtype=None, seed=None, ignore_every=0):
    w = make_weights(s)
    x, y = make_tokens(s) if seed is None else make_tokens(s, seed=seed)
    y = y.copy()
    if ignore_every:
        y[0, ::ignore_every] = -1
    kw = {} if act_dtype is None else {"act_dtype": act_dtype}
    cfg = gpu.make_config(s.n_layer, s.d_model, s.n_head, s.n_kv_head, s.head_dim, s.seq_len, s.vocab,
                          s.short_window, **kw)
    model = gpu.Model.from_numpy(cfg, w)
    loss, grads, ws = gpu.forward_backward(model, torch.from_numpy(x).to(DEV), torch.from_numpy(y).to(DEV))
    torch.cuda.synchronize()
    assert gpu.get_status(ws) == 0
    want_loss, want, mags = oracle_fb(_oracle_cfg(s), w, x, y, magnitudes=True)
    assert abs(loss.item() - want_loss) / abs(want_loss) <= 5e-3, (loss.item(), want_loss)
    return grads, want, mags


def test_forward_backward_tiny(gpu):
    """D = 64, two layers, both windows (T = 256 > the 64-key short window)."""
    grads, want, mags = _run(gpu, SHAPES["tiny"], ignore_every=7)
    _compare(grads, want, 2e-2, mags, _chain_bar(2))


def test_forward_backward_gqa_d128_ragged(gpu):
    """D = 128, 2 query heads per kv head, T = 200 (ragged tiles), window 48."""
    s = ModelShape("gqa", n_layer=2, d_model=256, n_head=4, n_kv_head=2, head_dim=128, vocab=512, seq_len=200,
                   batch=2, short_window=48)
    grads, want, mags = _run(gpu, s, seed=3)
    _compare(grads, want, 2e-2, mags, _chain_bar(2))


def test_forward_backward_bf16_activations(gpu):
    grads, want, mags = _run(gpu, SHAPES["tiny"], act_dtype=gpu.BF16, seed=11)
    _compare(grads, want, 5e-2, mags, _chain_bar(2, bf16=True))


def test_forward_backward_d20_width(gpu):
    """d20 widths (C = 1280, 10 heads, V = 32768) over two layers, one row."""
    f = SHAPES["d20"]
    s = ModelShape("d20_2l", n_layer=2, d_model=f.d_model, n_head=f.n_head, n_kv_head=f.n_kv_head,
                   head_dim=f.head_dim, vocab=f.vocab, seq_len=256, batch=1, short_window=64)
    grads, want, mags = _run(gpu, s, seed=5)
    _compare(grads, want, 2e-2, mags, _chain_bar(2))


def test_forward_backward_d20_width_full_context(gpu):
    """d20 widths over the full sequence: T = 2048 with the 512-key short window
    (layer 0) and a full-context layer (layer 1, the last), one row."""
    f = SHAPES["d20"]
    s = ModelShape("d20_2l_T2048", n_layer=2, d_model=f.d_model, n_head=f.n_head, n_kv_head=f.n_kv_head,
                   head_dim=f.head_dim, vocab=f.vocab, seq_len=2048, batch=1, short_window=512)
    grads, want, mags = _run(gpu, s, seed=9)
    _compare(grads, want, 2e-2, mags, _chain_bar(2))


def test_forward_backward_full_size_properties(gpu):
    """d20, B = 32, T = 2048: clean status, the forward's loss, finite
    gradients, run-to-run agreement and accumulation (a second call adds the
    same gradients again), both up to the summation order of the embedding
    atomics and the split-K partial sums of the weight gradients (bar 1e-5
    relative): everything else, the attention's log-sum-exp included, is
    bit-reproducible."""
    s = SHAPES["d20"]
    w = make_weights(s)
    x, y = make_tokens(s)
    cfg = gpu.make_config(s.n_layer, s.d_model, s.n_head, s.n_kv_head, s.head_dim, s.seq_len, s.vocab,
                          s.short_window)
    model = gpu.Model.from_numpy(cfg, w)
    tx, ty = torch.from_numpy(x).to(DEV), torch.from_numpy(y).to(DEV)
    loss, grads, ws = gpu.forward_backward(model, tx, ty)
    torch.cuda.synchronize()
    assert gpu.get_status(ws) == 0
    l0 = gpu.forward(model, tx, ty)["loss"].item()
    assert abs(loss.item() - l0) <= 1e-6 * abs(l0)
    snap = {"wte": grads["wte"].clone(), "c_fc0": grads["layers"][0]["c_fc"].clone(),
            "lm_head": grads["lm_head"].clone()}
    for t in [grads["wte"], grads["lm_head"]] + [v for lw in grads["layers"] for v in lw.values()]:
        assert torch.isfinite(t).all()
    _, fresh, _ = gpu.forward_backward(model, tx, ty, workspace=ws)  # run to run, from zeros
    gpu.forward_backward(model, tx, ty, grads=grads, workspace=ws)
    torch.cuda.synchronize()
    info = []
    for name, t, f in (("wte", grads["wte"], fresh["wte"]), ("c_fc0", grads["layers"][0]["c_fc"],
                                                             fresh["layers"][0]["c_fc"]),
                       ("lm_head", grads["lm_head"], fresh["lm_head"])):
        rel = ((t - 2 * snap[name]).norm() / (2 * snap[name]).norm()).item()
        rr = ((f - snap[name]).norm() / snap[name].norm()).item()
        info.append((name, rel, rr))
    print("accumulated vs 2x first, fresh vs first:", info)
    # summation order only: atomics (embedding rows) and split-K partial sums
    assert all(rel < 1e-5 and rr < 1e-5 for _, rel, rr in info), info


@pytest.mark.parametrize("B,T,H,Hkv,D,W", [(2, 300, 4, 2, 128, 100), (1, 256, 2, 2, 64, 256), (1, 1, 2, 1, 128, 1),
                                           (2, 130, 6, 2, 64, 40)])
def test_attention_backward_matches_oracle(gpu, B, T, H, Hkv, D, W):
    """The attention backward alone (nc_attention_lse + nc_attention_backward)
    against ``oracle.grad.attention_backward`` on the kernel's own 16-bit
    inputs; q and k normalised per head as QK-norm leaves them.  Bars: lse
    within 1e-3, dq/dk/dv relative Frobenius error <= 1e-2 (the kernel rounds P
    and dS to 16-bit for its second products and Delta uses the 16-bit o), and
    two runs bit-identical."""
    from oracle.grad import attention_backward
    rng = np.random.default_rng(T * 7 + H)
    q = rng.standard_normal((B, T, H, D))
    k = rng.standard_normal((B, T, Hkv, D))
    q *= np.sqrt(D) / np.linalg.norm(q, axis=-1, keepdims=True)
    k *= np.sqrt(D) / np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, Hkv, D))
    do = rng.standard_normal((B, T, H, D))
    packed = np.concatenate([q.reshape(B, T, H * D), k.reshape(B, T, Hkv * D), v.reshape(B, T, Hkv * D)], -1)
    qkv = torch.from_numpy(packed.astype(np.float16)).to(DEV)
    tdo = torch.from_numpy(do.reshape(B, T, H * D).astype(np.float16)).to(DEV)
    o = torch.empty((B, T, H * D), dtype=torch.float16, device=DEV)
    lse = torch.empty((B, T, H), dtype=torch.float32, device=DEV)
    gpu.attention_lse(qkv, o, lse, H, Hkv, D, W)
    d1 = torch.empty_like(qkv)
    d2 = torch.empty_like(qkv)
    gpu.attention_backward(qkv, o, tdo, lse, d1, H, Hkv, D, W)
    gpu.attention_backward(qkv, o, tdo, lse, d2, H, Hkv, D, W)
    torch.cuda.synchronize()
    assert torch.equal(d1, d2), "attention backward is not run-to-run identical"
    q16 = packed.astype(np.float16).astype(np.float64)
    qq = q16[..., :H * D].reshape(B, T, H, D)
    kk = q16[..., H * D:(H + Hkv) * D].reshape(B, T, Hkv, D)
    vv = q16[..., (H + Hkv) * D:].reshape(B, T, Hkv, D)
    dd = do.astype(np.float16).astype(np.float64)
    dq, dk, dv, P = attention_backward(qq, kk, vv, dd, W)
    # lse of the scaled visible scores
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    vis = (j <= i) & (i - j < W)
    G = H // Hkv
    want_lse = np.empty((B, T, H))
    for h in range(H):
        sc = np.einsum("bid,bjd->bij", qq[:, :, h], kk[:, :, h // G]) / np.sqrt(D)
        sc = np.where(vis[None], sc, -np.inf)
        mx = sc.max(-1, keepdims=True)
        want_lse[:, :, h] = (mx + np.log(np.exp(sc - mx).sum(-1, keepdims=True)))[..., 0]
    np.testing.assert_allclose(lse.cpu().numpy(), want_lse, rtol=0, atol=1e-3)
    got = d1.double().cpu().numpy()
    for name, a, b in (("dq", got[..., :H * D], dq.reshape(B, T, H * D)),
                       ("dk", got[..., H * D:(H + Hkv) * D], dk.reshape(B, T, Hkv * D)),
                       ("dv", got[..., (H + Hkv) * D:], dv.reshape(B, T, Hkv * D))):
        # (a floor of 1e-4 per element: with one visible key dS, and so dq and
        # dk, are exactly zero, and the kernel leaves rounding-level values)
        rel = np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-4 * np.sqrt(b.size))
        assert rel <= 1e-2, f"{name}: rel {rel:.3e}"
