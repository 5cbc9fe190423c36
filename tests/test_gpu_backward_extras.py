"""GPU parity of the training step with the further terms of the full nanochat
forward ("Nanochat与nanoGPT对比" §1: smear, value embeddings, residual lambdas
with x0, backout) against the fp64 oracle, ``oracle.grad.forward_backward(...,
extras=...)`` (pinned by ``tests/test_oracle_grad_extras.py``).

Every gradient -- of the block weights, wte, lm_head and each extras parameter
-- is compared element by element with the bound of ``tests/test_gpu_backward``:
|err| <= c * (sum of the absolute values of the terms it adds up) + 4 u max|g|,
with c the 16-bit rounding chain of the configuration.  The loss is within 5e-3
relative.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle.grad import forward_backward as oracle_fb
from test_gpu_backward import NAMES, _chain_bar, _compare
from workloads import SHAPES, ModelShape, make_extras, make_tokens, make_weights

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _oracle_cfg(s):
    return oracle.OracleConfig(s.n_layer, s.d_model, s.n_head, s.n_kv_head, s.head_dim, s.seq_len,
                               s.vocab, short_window=s.short_window)


def _run(gpu, s, seed):
    w = make_weights(s)
    L = s.n_layer
    ve_layers = [l for l in range(L) if oracle.value_embed_layers(L)[l]]
    ex = make_extras(s, layers=ve_layers)
    ex["smear_gate"] = ex["smear_gate"] * np.float32(0.2)  # gates away from saturation
    x, y = make_tokens(s, seed=seed)
    y = y.copy()
    y[0, ::5] = -1
    cfg = gpu.make_config(s.n_layer, s.d_model, s.n_head, s.n_kv_head, s.head_dim, s.seq_len, s.vocab,
                          s.short_window, extras=gpu.EXTRA_ALL)
    model = gpu.Model.from_numpy(cfg, w, extras=ex)
    loss, grads, ws = gpu.forward_backward(model, torch.from_numpy(x).to(DEV), torch.from_numpy(y).to(DEV))
    torch.cuda.synchronize()
    assert gpu.get_status(ws) == 0
    want_loss, want, mags = oracle_fb(_oracle_cfg(s), w, x, y, magnitudes=True, extras=ex)
    assert abs(loss.item() - want_loss) / abs(want_loss) <= 5e-3, (loss.item(), want_loss)
    return grads, want, mags, ve_layers


def _compare_extras(got, want, mags, c, ve_layers, n_layer):
    """Each extras gradient element within c * magnitude + 4 u max|g|."""
    kappa = 4.0 * c / (4 + 8 * n_layer)
    rows, bad = [], []
    items = [("smear_gate", got["smear_gate"], want["smear_gate"], mags["smear_gate"]),
             ("resid_lambdas", got["resid_lambdas"], want["resid_lambdas"], mags["resid_lambdas"]),
             ("x0_lambdas", got["x0_lambdas"], want["x0_lambdas"], mags["x0_lambdas"]),
             ("backout_lambda", got["backout_lambda"], np.array([want["backout_lambda"]]),
              np.array([mags["backout_lambda"]]))]
    for l in ve_layers:
        items.append((f"value_embeds[{l}]", got["value_embeds"][l], want["value_embeds"][l], mags["value_embeds"][l]))
        items.append((f"ve_gates[{l}]", got["ve_gates"][l], want["ve_gates"][l], mags["ve_gates"][l]))
    for name, a, b, m in items:
        a = a.detach().double().cpu().numpy().reshape(np.shape(b))
        b, m = np.asarray(b, dtype=np.float64), np.asarray(m, dtype=np.float64)
        err = np.abs(a - b)
        top = float(np.abs(b).max())
        ok = bool(np.all(err <= c * m + kappa * top + 1e-12))
        rows.append(f"{name}: max err {err.max():.3e}, max err/magnitude {float(np.max(err / np.maximum(m, 1e-30))):.3e}"
                    f" (c {c:.3e}), max|g| {top:.3e}")
        if not ok:
            bad.append(name)
    print("\n".join(rows))
    assert not bad, "extras gradients off: " + ", ".join(bad) + "\n" + "\n".join(rows)


def test_forward_backward_all_extras_tiny(gpu):
    """D = 64, two layers (value embedding on layer 1, backout at block 1), T = 256."""
    s = SHAPES["tiny"]
    grads, want, mags, ve_layers = _run(gpu, s, seed=21)
    _compare(grads, want, 2e-2, mags, _chain_bar(s.n_layer), n_chain=4 + 8 * s.n_layer)
    _compare_extras(grads["extras"], want, mags, _chain_bar(s.n_layer), ve_layers, s.n_layer)


def test_forward_backward_all_extras_gqa_d128_ragged(gpu):
    """D = 128, GQA 4/2, four layers (value embeddings on layers 1 and 3, backout
    at block 2), T = 200 with a 48-key window."""
    s = ModelShape("gqa4", n_layer=4, d_model=256, n_head=4, n_kv_head=2, head_dim=128, vocab=512, seq_len=200,
                   batch=2, short_window=48)
    grads, want, mags, ve_layers = _run(gpu, s, seed=22)
    _compare(grads, want, 2e-2, mags, _chain_bar(s.n_layer), n_chain=4 + 8 * s.n_layer)
    _compare_extras(grads["extras"], want, mags, _chain_bar(s.n_layer), ve_layers, s.n_layer)
