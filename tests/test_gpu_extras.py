"""GPU parity of the full nanochat forward's further terms against the oracle.

The terms ("Nanochat与nanoGPT对比：关键升级" §1: smear, value embeddings,
per-layer residual lambdas with x0, backout) are switched on through
``nc_config.extras``; their weights come from ``workloads.make_extras``.  The
bars are those of the plain forward: logits max-abs <= 3e-2, loss relative
error <= 5e-3.
"""
import numpy as np
import pytest
import torch

import oracle
from workloads import SHAPES, make_extras, make_tokens, make_weights

pytestmark = pytest.mark.gpu

DEV = "cuda"
PREFIX = 640  # > the 512-key short window


def _oracle_cfg(s):
    return oracle.OracleConfig(s.n_layer, s.d_model, s.n_head, s.n_kv_head, s.head_dim, s.seq_len,
                               s.vocab, short_window=s.short_window)


def _oracle_extras(ex, bits, nc):
    """The subset of ``ex`` the bits switch on, in the oracle's dict form."""
    out = {}
    if bits & nc.EXTRA_SMEAR:
        out["smear_gate"] = ex["smear_gate"]
    if bits & nc.EXTRA_RESID_LAMBDAS:
        out["resid_lambdas"] = ex["resid_lambdas"]
        out["x0_lambdas"] = ex["x0_lambdas"]
    if bits & nc.EXTRA_VALUE_EMBED:
        out["value_embeds"] = ex["value_embeds"]
        out["ve_gates"] = ex["ve_gates"]
    if bits & nc.EXTRA_BACKOUT:
        out["backout_lambda"] = ex["backout_lambda"]
    return out


def _setup(nc, name, bits, act_dtype=None, extras=None):
    s = SHAPES[name]
    w = make_weights(s)
    L = s.n_layer
    ve_layers = [l for l in range(L) if oracle.value_embed_layers(L)[l]]
    ex = make_extras(s, layers=ve_layers) if extras is None else extras
    kw = {} if act_dtype is None else {"act_dtype": act_dtype}
    cfg = nc.make_config(s.n_layer, s.d_model, s.n_head, s.n_kv_head, s.head_dim, s.seq_len, s.vocab,
                         s.short_window, extras=bits, **kw)
    model = nc.Model.from_numpy(cfg, w, extras=ex)
    return s, w, ex, model


def _check(res, want, what):
    err = np.abs(res["logits"] - want["logits"]).max()
    assert err <= 3e-2, f"{what} logits max-abs {err:.3e}"
    rel = abs(res["loss"] - want["loss"]) / abs(want["loss"])
    assert rel <= 5e-3, f"{what} loss rel {rel:.3e}"


@pytest.mark.parametrize("term", ["smear", "value_embed", "resid_lambdas", "backout", "all"])
def test_forward_extras_tiny(gpu, term):
    bits = {"smear": gpu.EXTRA_SMEAR, "value_embed": gpu.EXTRA_VALUE_EMBED,
            "resid_lambdas": gpu.EXTRA_RESID_LAMBDAS, "backout": gpu.EXTRA_BACKOUT,
            "all": gpu.EXTRA_ALL}[term]
    s, w, ex, model = _setup(gpu, "tiny", bits)
    x, y = make_tokens(s)
    y = y.copy()
    y[1, ::7] = -1
    r = gpu.forward(model, torch.from_numpy(x).to(DEV), torch.from_numpy(y).to(DEV), want_logits=True,
                    want_token_loss=True)
    assert gpu.get_status(r["workspace"]) == 0
    got = {"logits": r["logits"].cpu().numpy(), "loss": r["loss"].item()}
    want = oracle.forward(_oracle_cfg(s), w, x, y, extras=_oracle_extras(ex, bits, gpu))
    _check(got, want, f"tiny+{term}")
    np.testing.assert_allclose(r["token_loss"].cpu().numpy(), want["token_loss"], rtol=5e-3, atol=1e-3)
    # each term really changes the result
    plain = oracle.forward(_oracle_cfg(s), w, x, y)
    assert np.abs(plain["logits"] - want["logits"]).max() > 1e-2


def test_forward_extras_tiny_bf16_activations(gpu):
    s, w, ex, model = _setup(gpu, "tiny", gpu.EXTRA_ALL, act_dtype=gpu.BF16)
    x, y = make_tokens(s)
    r = gpu.forward(model, torch.from_numpy(x).to(DEV), torch.from_numpy(y).to(DEV), want_logits=True)
    assert gpu.get_status(r["workspace"]) == 0
    want = oracle.forward(_oracle_cfg(s), w, x, y, extras=_oracle_extras(ex, gpu.EXTRA_ALL, gpu))
    _check({"logits": r["logits"].cpu().numpy(), "loss": r["loss"].item()}, want, "tiny+all bf16")


@pytest.mark.parametrize("B,T", [(1, 1), (3, 100), (2, 65), (1, 256)])
def test_forward_extras_ragged(gpu, B, T):
    """Smear's first position, partial tiles and one-token rows with every term on."""
    s, w, ex, model = _setup(gpu, "tiny", gpu.EXTRA_ALL)
    x, y = make_tokens(s, seed=B * 100 + T, batch=B, seq_len=T)
    r = gpu.forward(model, torch.from_numpy(x).to(DEV), torch.from_numpy(y).to(DEV), want_logits=True)
    assert gpu.get_status(r["workspace"]) == 0
    want = oracle.forward(_oracle_cfg(s), w, x, y, extras=_oracle_extras(ex, gpu.EXTRA_ALL, gpu))
    _check({"logits": r["logits"].cpu().numpy(), "loss": r["loss"].item()}, want, f"ragged {B}x{T}")


def test_forward_neutral_extras_match_the_plain_forward(gpu):
    """resid lambdas 1 / x0 lambdas 0, zero value-embedding gates and backout 0
    route the stream through the fused kernels without changing it."""
    s = SHAPES["tiny"]
    L = s.n_layer
    ex = make_extras(s)
    ex["resid_lambdas"][:] = 1
    ex["x0_lambdas"][:] = 0
    ex["backout_lambda"] = np.float32(0)
    for g in ex["ve_gates"]:
        g[:] = 0
    bits = gpu.EXTRA_VALUE_EMBED | gpu.EXTRA_RESID_LAMBDAS | gpu.EXTRA_BACKOUT
    _, w, _, model = _setup(gpu, "tiny", bits, extras=ex)
    cfg0 = gpu.make_config(s.n_layer, s.d_model, s.n_head, s.n_kv_head, s.head_dim, s.seq_len, s.vocab,
                           s.short_window)
    plain = gpu.Model.from_numpy(cfg0, w)
    x, y = make_tokens(s)
    tx, ty = torch.from_numpy(x).to(DEV), torch.from_numpy(y).to(DEV)
    a = gpu.forward(model, tx, ty, want_logits=True)
    b = gpu.forward(plain, tx, ty, want_logits=True)
    torch.cuda.synchronize()
    assert L == 2 and (a["logits"] - b["logits"]).abs().max().item() <= 2e-3


@pytest.mark.parametrize("name", ["d20", "d26_gqa"])
def test_forward_extras_full_size_sampled_rows(gpu, name):
    """Every term on at full size; the oracle recomputes rows 0 and B-1 over
    their first PREFIX positions."""
    s, w, ex, model = _setup(gpu, name, gpu.EXTRA_ALL)
    x, y = make_tokens(s)
    tx, ty = torch.from_numpy(x).to(DEV), torch.from_numpy(y).to(DEV)
    r = gpu.forward(model, tx, ty, want_logits=True, want_token_loss=True)
    assert gpu.get_status(r["workspace"]) == 0
    rows = [0, s.batch - 1]
    got_logits = r["logits"][rows, :PREFIX].cpu().numpy()
    got_tl = r["token_loss"][rows, :PREFIX].cpu().numpy()
    fast = gpu.forward(model, tx, ty, want_token_loss=True)
    torch.cuda.synchronize()
    assert torch.equal(fast["token_loss"], r["token_loss"])
    del r, fast, model
    torch.cuda.empty_cache()
    want = oracle.forward(_oracle_cfg(s), w, x[rows, :PREFIX], y[rows, :PREFIX],
                          extras=_oracle_extras(ex, gpu.EXTRA_ALL, gpu))
    err = np.abs(got_logits - want["logits"]).max()
    assert err <= 3e-2, f"{name}+all logits max-abs {err:.3e}"
    rel_rows = np.abs(got_tl - want["token_loss"]) / np.abs(want["token_loss"])
    assert rel_rows.max() <= 5e-3, f"{name}+all per-token loss rel {rel_rows.max():.3e}"


def test_forward_extras_wide_rows(gpu):
    """d_model 2560 > 2048: the two-pass path of the fused norm kernels."""
    from workloads import ModelShape
    s = ModelShape("wide", n_layer=2, d_model=2560, n_head=20, n_kv_head=4, head_dim=128, vocab=512,
                   seq_len=64, batch=2, short_window=16)
    w = make_weights(s)
    ex = make_extras(s)
    bits = gpu.EXTRA_ALL
    cfg = gpu.make_config(s.n_layer, s.d_model, s.n_head, s.n_kv_head, s.head_dim, s.seq_len, s.vocab,
                          s.short_window, extras=bits)
    model = gpu.Model.from_numpy(cfg, w, extras=ex)
    x, y = make_tokens(s)
    r = gpu.forward(model, torch.from_numpy(x).to(DEV), torch.from_numpy(y).to(DEV), want_logits=True)
    assert gpu.get_status(r["workspace"]) == 0
    want = oracle.forward(_oracle_cfg(s), w, x, y, extras=_oracle_extras(ex, bits, gpu))
    _check({"logits": r["logits"].cpu().numpy(), "loss": r["loss"].item()}, want, "wide+all")
