"""KV-cache inference (nc_prefill / nc_decode_step / nc_decode_step_dev) with the
further terms of the full nanochat forward ("Nanochat与nanoGPT对比" §1: smear,
value embeddings, residual lambdas with x0, backout) against the fp64 oracle.

"从文本到聊天模型" §10.1-10.4: a decode step at position t gives the logits the
whole forward gives at t.  With the terms switched on, the oracle's reference
is ``oracle.forward(..., extras=...)`` over the prefix (pinned by
``tests/test_oracle_extras.py``).  The step's smear reads the previous
position's token from the session, so a step at position 0 has no smear and
the first step after a prompt mixes in the prompt's last token.  Bars as for
the forward: logits max-abs <= 3e-2.
"""
import numpy as np
import pytest
import torch

import oracle
from workloads import SHAPES, ModelShape, make_extras, make_tokens, make_weights

pytestmark = pytest.mark.gpu

DEV = "cuda"
BAR = 3e-2


def _oracle_cfg(s):
    return oracle.OracleConfig(s.n_layer, s.d_model, s.n_head, s.n_kv_head, s.head_dim, s.seq_len,
                               s.vocab, short_window=s.short_window)


def _model(nc, s):
    w = make_weights(s)
    L = s.n_layer
    ve_layers = [l for l in range(L) if oracle.value_embed_layers(L)[l]]
    ex = make_extras(s, layers=ve_layers)
    cfg = nc.make_config(s.n_layer, s.d_model, s.n_head, s.n_kv_head, s.head_dim, s.seq_len, s.vocab,
                         s.short_window, extras=nc.EXTRA_ALL)
    return w, ex, nc.Model.from_numpy(cfg, w, extras=ex)


def _want(s, w, ex, x):
    return oracle.forward(_oracle_cfg(s), w, x, extras=ex)["logits"]


def _decode_err(dec, want, T0):
    steps = dec.shape[0]
    return np.abs(dec.cpu().numpy() - np.transpose(want[:, T0:T0 + steps], (1, 0, 2))).max()


def _prefill_decode(nc, model, x, T0, steps, T_max, graph=False):
    B = x.shape[0]
    sess = nc.Session(model, B, T_max)
    tx = torch.from_numpy(x).to(DEV)
    pre = sess.prefill(tx[:, :T0].contiguous(), want_logits=T0 > 0)
    outs = []
    for k in range(steps):
        tok = tx[:, T0 + k].contiguous()
        outs.append((sess.decode_graph(tok) if graph else sess.decode(tok)).clone())
    torch.cuda.synchronize()
    assert sess.status() == 0
    return pre, torch.stack(outs)


def test_decode_all_extras_matches_forward_tiny(gpu):
    """D = 64, two layers; the prompt passes the 64-key short window."""
    s = SHAPES["tiny"]
    w, ex, model = _model(gpu, s)
    x, _ = make_tokens(s, batch=2, seed=31)
    T0, steps = 100, 12
    pre, dec = _prefill_decode(gpu, model, x, T0, steps, s.seq_len)
    fwd = gpu.forward(model, torch.from_numpy(x[:, :T0].copy()).to(DEV), None, want_logits=True)
    torch.cuda.synchronize()
    assert torch.equal(pre, fwd["logits"])  # prefill is the forward
    want = _want(s, w, ex, x[:, :T0 + steps])
    err = _decode_err(dec, want, T0)
    assert err <= BAR, f"tiny decode logits with extras max-abs {err:.3e}"
    assert np.abs(pre.cpu().numpy() - want[:, :T0]).max() <= BAR


def test_decode_all_extras_from_position_zero_and_graph(gpu):
    """Position 0 (no previous token: no smear), then the graph-replayed step
    (position and token record in device memory) after a one-token prompt."""
    s = SHAPES["tiny"]
    w, ex, model = _model(gpu, s)
    x, _ = make_tokens(s, batch=3, seed=32)
    want = _want(s, w, ex, x[:, :9])
    _, dec = _prefill_decode(gpu, model, x, 0, 6, 32)
    err = _decode_err(dec, want, 0)
    assert err <= BAR, f"decode from position 0 max-abs {err:.3e}"
    _, dec_g = _prefill_decode(gpu, model, x, 1, 8, 32, graph=True)
    err = _decode_err(dec_g, want, 1)
    assert err <= BAR, f"graph decode max-abs {err:.3e}"


def test_decode_all_extras_gqa_d128(gpu):
    """D = 128, GQA 4/2, four layers (value embeddings on layers 1 and 3,
    backout at block 2), a 48-key window; 40 rows, so the projections take
    the tcgen05 GEMM with split K rather than the skinny one."""
    s = ModelShape("gqa4", n_layer=4, d_model=256, n_head=4, n_kv_head=2, head_dim=128, vocab=512, seq_len=200,
                   batch=40, short_window=48)
    w, ex, model = _model(gpu, s)
    x, _ = make_tokens(s, batch=40, seed=33)
    T0, steps = 70, 5
    _, dec = _prefill_decode(gpu, model, x, T0, steps, 96)
    want = _want(s, w, ex, x[:, :T0 + steps])
    err = _decode_err(dec, want, T0)
    assert err <= BAR, f"gqa D128 decode with extras max-abs {err:.3e}"
