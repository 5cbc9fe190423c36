"""Pins of the oracle's dynamic tensorwise e4m3 path (``oracle/fp8.py``).

"Nanochat与nanoGPT对比：关键升级" §1 names dynamic tensor-level FP8 with
e4m3/e5m2 and nothing more; the readings are in the module docstring.  The
pins do not retype the oracle's formulas: the rounding is checked against
torch's own float8_e4m3fn conversion (an independent library routine) and hand
values from the format's definition; the quantiser and the product against
closed forms (exactly representable inputs, power-of-two rescaling, zero
tensors), an error bound of the format, and the scale's coupling of rows.
"""
import math

import numpy as np
import torch

import oracle
from oracle import OracleConfig
from oracle.fp8 import linear_e4m3, quantize_e4m3, round_e4m3, tensor_scale


def torch_e4m3(y):
    """torch's fp32 -> float8_e4m3fn -> fp32 round trip (NaN above 464: torch
    does not saturate, so callers stay within +-464)."""
    return torch.from_numpy(np.asarray(y, dtype=np.float32)).to(torch.float8_e4m3fn).to(torch.float64).numpy()


def all_e4m3_values():
    codes = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    return np.unique(codes[~np.isnan(codes)])


def test_e4m3_value_set_from_the_format_definition():
    vals = all_e4m3_values()
    pos = vals[vals > 0]
    # 15 normal binades x 8 mantissas, minus the NaN pattern, plus 7 subnormals
    assert len(pos) == 15 * 8 - 1 + 7
    assert pos.max() == 448.0 and pos.min() == 2.0 ** -9
    # every value is a fixed point of the oracle's rounding
    np.testing.assert_array_equal(round_e4m3(vals), vals)


def test_round_e4m3_hand_values():
    cases = {
        448.0: 448.0, 1000.0: 448.0, 464.0: 448.0,   # saturation; 464 ties to 448 (even)
        -1e30: -448.0,
        2.0 ** -9: 2.0 ** -9,                          # smallest subnormal
        2.0 ** -10: 0.0,                               # tie between 0 and 2^-9 -> 0 (even)
        3 * 2.0 ** -10: 2.0 ** -8,                     # tie 2^-9 (odd) / 2^-8 (even)
        1.0625: 1.0, 1.1875: 1.25,                     # ties inside [1, 2): spacing 1/8
        17.0: 16.0, 18.0: 18.0, 19.0: 20.0,            # spacing 2 in [16, 32); 19 ties to 20
        -0.3: -0.3125, 0.0: 0.0,
        1.9375: 2.0,                                   # tie at the top of a binade
    }
    for x, want in cases.items():
        assert round_e4m3(np.array([x]))[0] == want, x
    assert np.isnan(round_e4m3(np.array([np.nan]))[0])


def test_round_e4m3_matches_torch_conversion():
    rng = np.random.default_rng(11)
    vals = all_e4m3_values()
    mids = (vals[1:] + vals[:-1]) / 2  # every tie
    near = np.concatenate([np.nextafter(mids.astype(np.float32), np.float32(np.inf)),
                           np.nextafter(mids.astype(np.float32), np.float32(-np.inf))])
    rnd = np.concatenate([rng.standard_normal(200000) * s for s in (1e-3, 0.05, 1.0, 30.0, 150.0)])
    y = np.concatenate([vals, mids, near, rnd]).astype(np.float32)
    y = y[np.abs(y) <= 464.0]
    np.testing.assert_array_equal(round_e4m3(y.astype(np.float64)), torch_e4m3(y))


def test_quantize_amax_hits_the_format_maximum_and_codes_lie_in_the_set():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((37, 53)) * 0.01
    q, s = quantize_e4m3(x)
    assert s.dtype == np.float32
    i = np.unravel_index(np.argmax(np.abs(x)), x.shape)
    assert abs(q[i]) == 448.0
    assert np.abs(q).max() == 448.0
    assert np.isin(np.abs(q), all_e4m3_values()).all()
    # scale: fp32 division of 448 by the fp32 amax
    amax32 = np.float32(np.abs(x.astype(np.float32)).max())
    assert s == np.float32(448.0) / amax32


def test_quantize_is_invariant_under_power_of_two_rescaling():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((16, 40)).astype(np.float32)
    q1, s1 = quantize_e4m3(x)
    q2, s2 = quantize_e4m3(x * np.float32(8.0))
    np.testing.assert_array_equal(q1, q2)
    assert s1 == s2 * 8


def test_quantize_zero_tensor_and_floor():
    q, s = quantize_e4m3(np.zeros((3, 4)))
    assert s == np.float32(448.0) / np.float32(1e-12) and not q.any()
    # a tensor below the amax floor keeps its relative sizes only through the floor
    q, _ = quantize_e4m3(np.array([1e-14, -2e-14]))
    np.testing.assert_array_equal(q, round_e4m3(np.array([np.float32(1e-14) * np.float32(4.48e14),
                                                          np.float32(-2e-14) * np.float32(4.48e14)])))


def test_linear_e4m3_exact_on_representable_inputs():
    # operands built from e4m3 values whose amax is 448 (scale 1) or 224
    # (scale 2, exact): the product equals the plain product x W^T exactly
    rng = np.random.default_rng(5)
    vals = all_e4m3_values()
    vals = np.concatenate([vals, -vals])
    x = rng.choice(vals, (9, 48))
    w = rng.choice(vals, (7, 48))
    x[0, 0], w[0, 0] = 448.0, -448.0
    np.testing.assert_array_equal(linear_e4m3(x, w), x @ w.T)
    xh, wh = x / 2, w / 2  # amax 224, every element still an e4m3 value or a subnormal half
    ok = np.isin(np.abs(xh), vals).all() and np.isin(np.abs(wh), vals).all()
    if ok:
        np.testing.assert_array_equal(linear_e4m3(xh, wh), xh @ wh.T)


def test_linear_e4m3_within_the_format_error_bound():
    # |q/s - x| <= 2^-4 |x| for normals (half the 2^-3 relative spacing) and
    # <= 2^-10 / s in the subnormal range: bound the product error by those
    rng = np.random.default_rng(6)
    x = rng.standard_normal((20, 96))
    w = rng.standard_normal((30, 96)).astype(np.float32)
    got = linear_e4m3(x, w)
    exact = x @ w.astype(np.float64).T
    sx, sw = float(tensor_scale(x.astype(np.float32))), float(tensor_scale(w))
    ex = 2.0 ** -4 * np.abs(x) + 2.0 ** -10 / sx + 1e-7 * np.abs(x)
    ew = 2.0 ** -4 * np.abs(w) + 2.0 ** -10 / sw
    bound = ex @ np.abs(w).T + np.abs(x) @ ew.T + ex @ ew.T
    assert (np.abs(got - exact) <= bound).all()
    # and the quantisation really does something at this size
    assert np.abs(got - exact).max() > 1e-3


def _cfg(**kw):
    base = dict(n_layer=2, d_model=32, n_head=2, n_kv_head=1, head_dim=16, seq_len=12, vocab=40,
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


def test_forward_fp8_zero_projections_closed_form():
    # attn_proj = mlp_proj = 0 quantise to zero codes (amax floor), so the
    # blocks add nothing.  Embedding rows +-c (all entries equal magnitude)
    # normalise to +-1: amax 1, scale 448, codes +-448.  An LM head of e4m3
    # values with amax 448 has scale 1 and codes equal to itself, so the "all"
    # logits are softcap(sum of +-W), formed here by hand.
    c = _cfg()
    w = _weights(c)
    for lw in w["layers"]:
        lw["attn_proj"][:] = 0
        lw["mlp_proj"][:] = 0
    rng = np.random.default_rng(8)
    sign = rng.choice([-1.0, 1.0], (c.vocab, c.d_model)).astype(np.float32)
    w["wte"] = (sign * np.float32(0.37)).astype(np.float32)
    vals = all_e4m3_values()
    head = rng.choice(np.concatenate([vals[vals > 0.5], -vals[vals > 0.5]]), (c.vocab, c.d_model))
    head[0, 0] = 448.0
    w["lm_head"] = head.astype(np.float32)
    idx = rng.integers(0, c.vocab, (2, c.seq_len))
    got = oracle.forward(c, w, idx, fp8="all")["logits"]
    e = sign[idx].astype(np.float64)  # rms-normalised embedding (up to eps)
    rms = 0.37 / math.sqrt(0.37 ** 2 + c.norm_eps)
    # the normalised entries are +-rms; scale 448/rms (fp32), codes +-448 exactly
    want = 15.0 * np.tanh((e @ head.T) * rms / 15.0)
    np.testing.assert_allclose(got, want, rtol=1e-6, atol=1e-6)
    # "block" keeps the head in bf16 and changes nothing else here
    blk = oracle.forward(c, w, idx, fp8="block")["logits"]
    np.testing.assert_allclose(blk, oracle.forward(c, w, idx)["logits"], rtol=0, atol=1e-13)


def test_forward_fp8_scale_couples_rows():
    # tensorwise scales: a large activation in row 1 changes row 0's codes
    c = _cfg()
    w = _weights(c)
    rng = np.random.default_rng(9)
    idx = rng.integers(0, c.vocab, (2, c.seq_len))
    a = oracle.forward(c, w, idx, fp8="block")["logits"]
    one = oracle.forward(c, w, idx[:1], fp8="block")["logits"]
    plain_a = oracle.forward(c, w, idx)["logits"]
    plain_one = oracle.forward(c, w, idx[:1])["logits"]
    np.testing.assert_allclose(plain_one[0], plain_a[0], rtol=0, atol=1e-13)
    assert not np.array_equal(one[0], a[0])
    # but the difference is of the size of the quantisation itself
    assert np.abs(one[0] - a[0]).max() < 4 * np.abs(a - plain_a).max()


def test_forward_fp8_close_to_the_plain_forward():
    c = _cfg(n_layer=3)
    w = _weights(c, std=0.2)
    idx = np.random.default_rng(10).integers(0, c.vocab, (2, c.seq_len))
    tgt = np.roll(idx, -1, axis=1)
    p = oracle.forward(c, w, idx, tgt)
    f = oracle.forward(c, w, idx, tgt, fp8="all")
    d = np.abs(p["logits"] - f["logits"]).max()
    assert 1e-3 < d < 0.5
    assert abs(p["loss"] - f["loss"]) < 0.05 * p["loss"]


def test_forward_fp8_with_neutral_extras_is_the_plain_fp8_forward():
    # residual lambdas 1, x0 lambdas 0, value-embedding gates 0, backout 0:
    # every extra term adds exact zeros, so the e4m3 decisions are the same
    c = _cfg(n_layer=3)
    w = _weights(c)
    rng = np.random.default_rng(12)
    idx = rng.integers(0, c.vocab, (2, c.seq_len))
    L, kvw = c.n_layer, c.n_kv_head * c.head_dim
    ex = {"resid_lambdas": np.ones(L, np.float32), "x0_lambdas": np.zeros(L, np.float32),
          "value_embeds": [rng.standard_normal((c.vocab, kvw)).astype(np.float32) for _ in range(L)],
          "ve_gates": [np.zeros(c.n_kv_head, np.float32) for _ in range(L)],
          "backout_lambda": np.float32(0.0)}
    for mode in ("block", "all"):
        a = oracle.forward(c, w, idx, fp8=mode)["logits"]
        b = oracle.forward(c, w, idx, fp8=mode, extras=ex)["logits"]
        assert np.array_equal(a, b), mode
    ex["backout_lambda"] = np.float32(0.25)
    assert not np.array_equal(oracle.forward(c, w, idx, fp8="all", extras=ex)["logits"],
                              oracle.forward(c, w, idx, fp8="all")["logits"])
