"""Pins of the fp64 oracle against facts fixed by the pages and by mathematics.

No test here retypes an oracle formula to compare it with itself.  Each pin is
one of: a value printed on the pages (``tests/golden``), a closed form, an
invariant, brute-force enumeration on tiny inputs, or an independent library
routine (torch float64 on the CPU) that reaches the same definition by another
route.  Together they are chosen so that a dropped term, a wrong sign, a wrong
index or a transposed operand in the oracle fails at least one of them.
"""
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from oracle import OracleConfig
from workloads import SHAPES, make_tokens, make_weights, round_to_bf16

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf16_weights_torch(a):
    """fp32 weights as their bf16 values, through torch's own conversion."""
    return torch.from_numpy(np.asarray(a, dtype=np.float32)).to(torch.bfloat16).to(torch.float64)


def _golden_lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [l.split() for l in f if l.strip() and not l.startswith("#")]


def _cfg(**kw):
    base = dict(n_layer=2, d_model=64, n_head=4, n_kv_head=2, head_dim=16,
                seq_len=24, vocab=96, short_window=6)
    base.update(kw)
    return OracleConfig(**base)


# ---------------------------------------------------------------- config / windows

def test_derive_config_matches_page_examples():
    for parts in _golden_lines("config_examples.txt"):
        if parts[0] == "derive":
            depth, aspect, hd, model_dim, heads = map(int, parts[1:])
            c = oracle.derive_config(depth, aspect, hd)
            assert c.d_model == model_dim and c.n_head == heads
            assert c.n_kv_head == heads
            assert c.d_model // c.n_head == hd


def test_embedding_shape_matches_page_example():
    (_, B, T, C), = [p for p in _golden_lines("config_examples.txt") if p[0] == "embed_shape"]
    B, T, C = int(B), int(T), int(C)
    wte = np.zeros((8, C), dtype=np.float32)
    idx = np.zeros((B, T), dtype=np.int64)
    assert oracle.embed(wte, idx).shape == (B, T, C)


def test_sssl_windows_match_hand_written_rule():
    for n_layer, T, kinds in _golden_lines("sssl_windows.txt"):
        n_layer, T = int(n_layer), int(T)
        c = _cfg(n_layer=n_layer, seq_len=T, short_window=0)
        w = oracle.layer_windows(c)
        assert w == [T // 4 if ch == "S" else T for ch in kinds]


def test_benchmark_shapes_windows():
    # tiny: window 64/256; the big ones 512/2048, counts of full layers.
    s = SHAPES["tiny"]
    c = OracleConfig(s.n_layer, s.d_model, s.n_head, s.n_kv_head, s.head_dim, s.seq_len, s.vocab,
                     short_window=s.short_window)
    assert oracle.layer_windows(c) == [64, 256]
    for name, n_full in (("d12", 3), ("d20", 5), ("d26", 7), ("d26_gqa", 7)):
        s = SHAPES[name]
        c = OracleConfig(s.n_layer, s.d_model, s.n_head, s.n_kv_head, s.head_dim, s.seq_len,
                         s.vocab, short_window=s.short_window)
        w = oracle.layer_windows(c)
        assert w.count(2048) == n_full and w.count(512) == s.n_layer - n_full
        assert w[-1] == 2048


def test_window_predicate_brute_force():
    # W keys ending at the query: {max(0, i-W+1), ..., i}; enumerate every (i, j).
    for T in range(1, 17):
        for W in range(1, T + 1):
            for i in range(T):
                want = set(range(max(0, i - W + 1), i + 1))
                got = {j for j in range(T) if oracle.window_visible(i, j, W)}
                assert got == want
                assert len(got) == min(i + 1, W)


# ---------------------------------------------------------------- RMSNorm

def test_rmsnorm_closed_form():
    rng = np.random.default_rng(0)
    u = rng.standard_normal((5, 7, 33)) * 3.0
    for eps in (0.0, 1e-6, 0.5):
        out = oracle.rms_norm(u, eps)
        ms = np.mean(u * u, axis=-1)
        rms_out = np.sqrt(np.mean(out * out, axis=-1))
        np.testing.assert_allclose(rms_out, np.sqrt(ms / (ms + eps)), rtol=1e-13)
    # hand example: [3, 4] has mean square 12.5
    np.testing.assert_allclose(oracle.rms_norm(np.array([3.0, 4.0]), 0.0),
                               np.array([3.0, 4.0]) / math.sqrt(12.5), rtol=1e-15)
    # scale invariance with eps -> 0, and against torch's library rms_norm
    np.testing.assert_allclose(oracle.rms_norm(7.5 * u, 0.0), oracle.rms_norm(u, 0.0), rtol=1e-13)
    t = F.rms_norm(torch.from_numpy(u), (33,), eps=1e-6).numpy()
    np.testing.assert_allclose(oracle.rms_norm(u, 1e-6), t, rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------- RoPE

def test_rope_hand_rotation_and_pairing():
    # D = 2: theta_0 = 1, so (1, 0) at position t becomes (cos t, sin t).
    T = 9
    cos, sin = oracle.rope_tables(T, 2, 10000.0)
    u = np.zeros((1, T, 1, 2))
    u[..., 0] = 1.0
    r = oracle.rope(u, cos, sin)
    t = np.arange(T, dtype=np.float64)
    np.testing.assert_allclose(r[0, :, 0, 0], np.cos(t), atol=1e-15)
    np.testing.assert_allclose(r[0, :, 0, 1], np.sin(t), atol=1e-15)
    # D = 4, base 100: pair (u_1, u_3) rotates by t * 100^(-1/2) = t / 10.
    cos, sin = oracle.rope_tables(T, 4, 100.0)
    u = np.zeros((1, T, 1, 4))
    u[..., 1] = 1.0
    r = oracle.rope(u, cos, sin)
    np.testing.assert_allclose(r[0, :, 0, 1], np.cos(t / 10), atol=1e-15)
    np.testing.assert_allclose(r[0, :, 0, 3], np.sin(t / 10), atol=1e-15)
    np.testing.assert_allclose(r[0, :, 0, 0], 0.0, atol=1e-15)
    np.testing.assert_allclose(r[0, :, 0, 2], 0.0, atol=1e-15)


def test_rope_as_complex_multiplication():
    # "rotation in complex space": (a + i b) * exp(i t theta) with torch complex128.
    T, H, D = 11, 3, 16
    rng = np.random.default_rng(1)
    u = rng.standard_normal((2, T, H, D))
    cos, sin = oracle.rope_tables(T, D, 10000.0)
    r = oracle.rope(u, cos, sin)
    ut = torch.from_numpy(u)
    z = torch.complex(ut[..., :D // 2], ut[..., D // 2:])
    theta = 10000.0 ** (-torch.arange(D // 2, dtype=torch.float64) * 2 / D)
    ang = torch.arange(T, dtype=torch.float64)[:, None] * theta[None, :]
    zr = z * torch.polar(torch.ones_like(ang), ang)[None, :, None, :]
    want = torch.cat([zr.real, zr.imag], dim=-1).numpy()
    np.testing.assert_allclose(r, want, rtol=1e-12, atol=1e-12)


def test_rope_invariants():
    T, H, D = 13, 2, 32
    rng = np.random.default_rng(2)
    q = rng.standard_normal((1, T, H, D))
    k = rng.standard_normal((1, T, H, D))
    cos, sin = oracle.rope_tables(T + 5, D, 10000.0)
    rq, rk = oracle.rope(q, cos, sin), oracle.rope(k, cos, sin)
    # norm preservation
    np.testing.assert_allclose(np.linalg.norm(rq, axis=-1), np.linalg.norm(q, axis=-1), rtol=1e-13)
    # t = 0 is the identity
    np.testing.assert_allclose(rq[:, 0], q[:, 0], atol=1e-15)
    # relative-position law: <rope(q,m), rope(k,n)> depends only on m - n
    qv, kv = q[0, 0, 0], k[0, 0, 0]
    def at(vec, pos):
        x = np.zeros((1, 1, 1, D)); x[0, 0, 0] = vec
        return oracle.rope(x, cos, sin, pos0=pos)[0, 0, 0]
    for m, n, s in ((5, 2, 3), (7, 7, 4), (1, 6, 5)):
        np.testing.assert_allclose(at(qv, m) @ at(kv, n), at(qv, m + s) @ at(kv, n + s), rtol=1e-12)
    # QK-norm after RoPE equals QK-norm before RoPE when eps = 0 (norms preserved)
    np.testing.assert_allclose(oracle.rms_norm(rq, 0.0), oracle.rope(oracle.rms_norm(q, 0.0), cos, sin),
                               rtol=1e-12, atol=1e-13)


def test_rope_qknorm_unit_rms_and_scale_invariance():
    c = _cfg(head_dim=32, norm_eps=1e-6)
    rng = np.random.default_rng(3)
    q = rng.standard_normal((2, 10, 4, 32)) * 5
    k = rng.standard_normal((2, 10, 2, 32)) * 0.1
    qn, kn = oracle.rope_qknorm(q, k, c)
    for a, src in ((qn, q), (kn, k)):
        ms = np.mean(src * src, axis=-1)
        np.testing.assert_allclose(np.sqrt(np.mean(a * a, axis=-1)), np.sqrt(ms / (ms + 1e-6)), rtol=1e-12)
    q2, k2 = oracle.rope_qknorm(q * 1000.0, k * 1000.0, c)
    np.testing.assert_allclose(q2, qn, rtol=1e-6, atol=1e-9)
    np.testing.assert_allclose(k2, kn, rtol=1e-4, atol=1e-7)


# ---------------------------------------------------------------- attention

def _torch_attention(q, k, v, W):
    """Library routine: torch SDPA in float64, explicit window mask, GQA by repeat."""
    B, T, H, D = q.shape
    Hkv = k.shape[2]
    qt = torch.from_numpy(q).permute(0, 2, 1, 3)
    kt = torch.from_numpy(k).permute(0, 2, 1, 3).repeat_interleave(H // Hkv, dim=1)
    vt = torch.from_numpy(v).permute(0, 2, 1, 3).repeat_interleave(H // Hkv, dim=1)
    i = torch.arange(T)[:, None]
    j = torch.arange(T)[None, :]
    mask = (j <= i) & (j > i - W)
    o = F.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask)
    return o.permute(0, 2, 1, 3).numpy()


@pytest.mark.parametrize("H,Hkv,W", [(4, 4, 3), (4, 2, 5), (6, 2, 40), (4, 1, 1), (2, 2, 17)])
def test_attention_matches_library_sdpa(H, Hkv, W):
    rng = np.random.default_rng(H * 100 + Hkv * 10 + W)
    B, T, D = 2, 17, 8
    q = rng.standard_normal((B, T, H, D))
    k = rng.standard_normal((B, T, Hkv, D))
    v = rng.standard_normal((B, T, Hkv, D))
    np.testing.assert_allclose(oracle.attention(q, k, v, W), _torch_attention(q, k, v, W),
                               rtol=1e-12, atol=1e-12)


def test_attention_special_cases():
    rng = np.random.default_rng(7)
    B, T, H, Hkv, D = 2, 12, 4, 2, 8
    q = rng.standard_normal((B, T, H, D))
    k = rng.standard_normal((B, T, Hkv, D))
    v = rng.standard_normal((B, T, Hkv, D))
    vrep = np.repeat(v, H // Hkv, axis=2)
    # W = 1: every query sees only itself
    np.testing.assert_allclose(oracle.attention(q, k, v, 1), vrep, atol=1e-14)
    # row 0 sees only key 0, for every window
    for W in (1, 3, T):
        np.testing.assert_allclose(oracle.attention(q, k, v, W)[:, 0], vrep[:, 0], atol=1e-14)
    # W >= T is plain causal attention
    np.testing.assert_allclose(oracle.attention(q, k, v, T), oracle.attention(q, k, v, 10 * T), atol=0)
    # constant value rows give that value back
    vc = np.broadcast_to(rng.standard_normal((1, 1, Hkv, D)), v.shape).copy()
    np.testing.assert_allclose(oracle.attention(q, k, vc, 5), np.repeat(vc, H // Hkv, axis=2), atol=1e-13)
    # GQA equals MHA on contiguous-group repeated k, v
    krep = np.repeat(k, H // Hkv, axis=2)
    np.testing.assert_allclose(oracle.attention(q, k, v, 5), oracle.attention(q, krep, vrep, 5), atol=1e-14)
    # query-row sampling returns the same rows
    rows = [0, 5, 11]
    np.testing.assert_allclose(oracle.attention(q, k, v, 5, rows), oracle.attention(q, k, v, 5)[:, rows], atol=0)


# ---------------------------------------------------------------- bf16 weight cast

def test_to_bf16_hand_values():
    # bf16 keeps 8 significant bits: the spacing just above 1 is 2^-7.
    cases = [(1.0, 1.0), (1.0 + 2.0 ** -9, 1.0), (1.0 + 3 * 2.0 ** -9, 1.0 + 2.0 ** -7),
             (1.0 + 2.0 ** -8, 1.0),                         # tie -> even significand (1.0)
             (1.0 + 3 * 2.0 ** -8, 1.0 + 2.0 ** -6),          # tie -> even (1 + 2^-6)
             (-2.0 - 2.0 ** -7, -2.0), (0.0, 0.0), (3.0e38, 226 * 2.0 ** 120)]  # spacing 2^120 there
    got = oracle.to_bf16(np.array([c[0] for c in cases], dtype=np.float32))
    np.testing.assert_array_equal(got, np.array([c[1] for c in cases], dtype=np.float32).astype(np.float64))
    assert np.isnan(oracle.to_bf16(np.array([np.nan], dtype=np.float32)))[0]


def test_to_bf16_matches_torch_conversion():
    rng = np.random.default_rng(13)
    a = (rng.standard_normal(200_000) * 10.0 ** rng.uniform(-20, 20, 200_000)).astype(np.float32)
    bits = rng.integers(0, 2 ** 32, 20_000, dtype=np.uint64).astype(np.uint32)
    b = bits.view(np.float32)
    b = b[np.isfinite(b)]
    for x in (a, b):
        np.testing.assert_array_equal(oracle.to_bf16(x), bf16_weights_torch(x).numpy())


def test_linear_uses_cast_weights():
    # a weight that bf16 cannot hold changes the product: 1 + 2^-9 acts as 1
    x = np.array([[2.0, -1.0]])
    w = np.array([[1.0 + 2.0 ** -9, 0.5]], dtype=np.float32)
    np.testing.assert_array_equal(oracle.linear(x, w), [[2.0 - 0.5]])
    assert oracle.linear(np.eye(3), np.full((4, 3), 0.1, dtype=np.float32)).dtype == np.float64


# ---------------------------------------------------------------- MLP / soft-cap / CE

def test_relu2_mlp_hand_values():
    a = np.array([[1.0, -2.0, 3.0]])
    w_fc = np.eye(3)
    w_proj = np.array([[1.0, 1.0, 1.0], [0.0, 0.0, 2.0]])  # 3 -> 2
    # relu(.)^2 = [1, 0, 9]; proj -> [10, 18]
    np.testing.assert_allclose(oracle.relu2_mlp(a, w_fc, w_proj), [[10.0, 18.0]])
    assert np.all(oracle.relu2_mlp(a, w_fc, np.zeros((2, 3))) == 0)


def test_softcap_properties():
    z = np.linspace(-400, 400, 20001)
    l = oracle.softcap(z, 15.0)
    assert np.all(np.abs(l) <= 15.0) and np.all(np.abs(l[np.abs(z) < 100]) < 15.0)
    np.testing.assert_allclose(oracle.softcap(-z, 15.0), -l, atol=0)
    np.testing.assert_allclose(oracle.softcap(np.array([15.0]), 15.0), [15.0 * 0.7615941559557649], rtol=1e-15)
    small = np.array([1e-3, -0.02, 0.3])
    np.testing.assert_allclose(oracle.softcap(small, 15.0), small - small ** 3 / 675.0, rtol=1e-6)
    assert np.all(np.diff(l) >= 0)


def test_cross_entropy_closed_forms():
    V = 512
    # uniform logits: loss = ln V
    nll, loss = oracle.cross_entropy(np.zeros((3, V)), np.array([0, 7, 511]))
    np.testing.assert_allclose(nll, math.log(V), rtol=1e-15)
    assert abs(loss - math.log(V)) < 1e-15
    # capped one-hot: 15 at the target, 0 elsewhere
    l = np.zeros((2, V)); l[0, 3] = 15.0; l[1, 9] = 15.0
    nll, loss = oracle.cross_entropy(l, np.array([3, 9]))
    np.testing.assert_allclose(nll, math.log(math.exp(15) + V - 1) - 15, rtol=1e-13)
    # ignored targets drop out of the mean; all ignored -> NaN
    rng = np.random.default_rng(5)
    l = rng.standard_normal((6, V)) * 4
    y = np.array([1, -1, 5, -1, 500, 2])
    nll, loss = oracle.cross_entropy(l, y)
    assert nll[1] == 0 and nll[3] == 0
    lt = torch.from_numpy(l)
    want = F.cross_entropy(lt, torch.from_numpy(y), ignore_index=-1).item()
    want_rows = F.cross_entropy(lt, torch.from_numpy(y), ignore_index=-1, reduction="none").numpy()
    np.testing.assert_allclose(nll, want_rows, rtol=1e-13)
    assert abs(loss - want) < 1e-13
    _, loss = oracle.cross_entropy(l, np.full(6, -1))
    assert math.isnan(loss)


# ---------------------------------------------------------------- whole forward

def _small_weights(c, seed=11, std=0.02):
    rng = np.random.default_rng(seed)
    C, H, Hkv, D, V = c.d_model, c.n_head, c.n_kv_head, c.head_dim, c.vocab
    g = lambda *s: rng.standard_normal(s) * std
    return {"wte": g(V, C), "lm_head": g(V, C),
            "layers": [{"c_q": g(H * D, C), "c_k": g(Hkv * D, C), "c_v": g(Hkv * D, C),
                        "attn_proj": g(C, H * D), "c_fc": g(4 * C, C), "mlp_proj": g(C, 4 * C)}
                       for _ in range(c.n_layer)]}


def test_forward_zero_projections_closed_form():
    # With attn_proj = mlp_proj = 0 every block is the identity, so the logits are
    # 15 tanh(rms(wte[idx]) lm_head^T / 15).
    c = _cfg()
    w = _small_weights(c, std=0.5)
    for lw in w["layers"]:
        lw["attn_proj"][:] = 0
        lw["mlp_proj"][:] = 0
    rng = np.random.default_rng(3)
    idx = rng.integers(0, c.vocab, (2, c.seq_len))
    y = rng.integers(0, c.vocab, (2, c.seq_len))
    res = oracle.forward(c, w, idx, y)
    a = w["wte"][idx]
    a = a / np.sqrt(np.mean(a * a, -1, keepdims=True) + c.norm_eps)
    want = 15.0 * np.tanh((a @ bf16_weights_torch(w["lm_head"]).numpy().T) / 15.0)
    np.testing.assert_allclose(res["logits"], want, rtol=1e-12, atol=1e-12)
    want_nll = F.cross_entropy(torch.from_numpy(want).reshape(-1, c.vocab), torch.from_numpy(y).reshape(-1),
                               reduction="none").numpy().reshape(2, -1)
    np.testing.assert_allclose(res["token_loss"], want_nll, rtol=1e-12)


def test_forward_zero_lm_head_gives_ln_vocab():
    c = _cfg()
    w = _small_weights(c, std=0.3)
    w["lm_head"][:] = 0
    idx = np.arange(2 * c.seq_len).reshape(2, -1) % c.vocab
    y = idx.copy()
    y[0, 3] = -1
    res = oracle.forward(c, w, idx, y)
    assert abs(res["loss"] - math.log(c.vocab)) < 1e-13
    assert res["token_loss"][0, 3] == 0


def test_forward_causality_and_row_independence():
    c = _cfg(n_layer=3, seq_len=20, short_window=5)
    w = _small_weights(c, std=0.3)
    rng = np.random.default_rng(4)
    idx = rng.integers(0, c.vocab, (3, c.seq_len))
    base = oracle.forward(c, w, idx)["logits"]
    t = 11
    idx2 = idx.copy()
    idx2[:, t] = (idx2[:, t] + 1) % c.vocab
    pert = oracle.forward(c, w, idx2)["logits"]
    np.testing.assert_array_equal(pert[:, :t], base[:, :t])
    assert np.all(np.abs(pert[:, t:] - base[:, t:]).max(axis=-1) > 0)
    alone = oracle.forward(c, w, idx[1:2])["logits"]
    np.testing.assert_array_equal(alone[0], base[1])


def test_forward_qk_norm_makes_attention_scale_free():
    # QK-norm after RoPE: scaling c_q and c_k leaves the forward unchanged.
    c = _cfg(norm_eps=1e-12)
    w = _small_weights(c, std=0.3)
    rng = np.random.default_rng(8)
    idx = rng.integers(0, c.vocab, (1, c.seq_len))
    base = oracle.forward(c, w, idx)["logits"]
    for lw in w["layers"]:  # powers of two commute with the bf16 weight cast
        lw["c_q"] *= 32.0
        lw["c_k"] *= 0.0625
    np.testing.assert_allclose(oracle.forward(c, w, idx)["logits"], base, rtol=1e-7, atol=1e-8)


def test_forward_matches_independent_torch_composition():
    """Cross-check with a torch float64 forward built from library routines:
    F.embedding, F.rms_norm, complex-number RoPE, SDPA with a window mask and GQA,
    relu().square(), tanh and F.cross_entropy.  H*D != C so a transposed
    projection would not even type-check."""
    c = _cfg(n_layer=3, d_model=48, n_head=4, n_kv_head=2, head_dim=16, seq_len=21, short_window=7)
    w = _small_weights(c, std=0.2)
    rng = np.random.default_rng(9)
    idx = rng.integers(0, c.vocab, (2, c.seq_len))
    y = rng.integers(-1, c.vocab, (2, c.seq_len))
    res = oracle.forward(c, w, idx, y)

    T = bf16_weights_torch  # every weight enters its product as its bf16 value
    B, S = idx.shape
    H, Hkv, D, C = c.n_head, c.n_kv_head, c.head_dim, c.d_model
    theta = c.rope_base ** (-torch.arange(D // 2, dtype=torch.float64) * 2 / D)
    rot = torch.polar(torch.ones(S, D // 2, dtype=torch.float64),
                      torch.arange(S, dtype=torch.float64)[:, None] * theta[None])

    def rope_c(u):  # [B,S,h,D]
        z = torch.complex(u[..., :D // 2], u[..., D // 2:]) * rot[None, :, None, :]
        return torch.cat([z.real, z.imag], -1)

    nrm = lambda u: F.rms_norm(u, (u.shape[-1],), eps=c.norm_eps)
    x = F.embedding(torch.from_numpy(idx), torch.from_numpy(np.asarray(w["wte"], dtype=np.float64)))
    windows = [7, 7, 21]  # S S L (last layer forced full)
    for l, lw in enumerate(w["layers"]):
        a = nrm(x)
        q = rope_c((a @ T(lw["c_q"]).T).view(B, S, H, D))
        k = rope_c((a @ T(lw["c_k"]).T).view(B, S, Hkv, D))
        v = (a @ T(lw["c_v"]).T).view(B, S, Hkv, D)
        q, k = nrm(q), nrm(k)
        i = torch.arange(S)[:, None]; j = torch.arange(S)[None]
        mask = (j <= i) & (j > i - windows[l])
        o = F.scaled_dot_product_attention(q.transpose(1, 2), k.transpose(1, 2), v.transpose(1, 2),
                                           attn_mask=mask, enable_gqa=True).transpose(1, 2)
        x = x + o.reshape(B, S, H * D) @ T(lw["attn_proj"]).T
        x = x + F.relu(nrm(x) @ T(lw["c_fc"]).T).square() @ T(lw["mlp_proj"]).T
    logits = 15 * torch.tanh((nrm(x) @ T(w["lm_head"]).T) / 15)
    loss = F.cross_entropy(logits.view(-1, c.vocab), torch.from_numpy(y).view(-1), ignore_index=-1)
    np.testing.assert_allclose(res["logits"], logits.numpy(), rtol=1e-11, atol=1e-12)
    assert abs(res["loss"] - loss.item()) < 1e-12


# ---------------------------------------------------------------- seeded inputs

def test_token_shift_matches_page_example():
    rows = {p[0]: list(map(int, p[1:])) for p in _golden_lines("shift_example.txt")}
    row = np.array([rows["row"]])
    assert row[:, :-1].tolist() == [rows["inputs"]] and row[:, 1:].tolist() == [rows["targets"]]
    s = SHAPES["tiny"]
    x, y = make_tokens(s)
    assert x.shape == (s.batch, s.seq_len) and y.shape == x.shape
    np.testing.assert_array_equal(y[:, :-1], x[:, 1:])
    assert x.dtype == np.int32 and x.min() >= 0 and x.max() < s.vocab


def test_weights_are_seeded_and_shaped():
    s = SHAPES["tiny"]
    w1, w2 = make_weights(s), make_weights(s)
    assert w1["wte"].dtype == np.float32
    np.testing.assert_array_equal(w1["layers"][1]["c_fc"], w2["layers"][1]["c_fc"])
    assert w1["layers"][0]["c_q"].shape == (s.n_head * s.head_dim, s.d_model)
    assert abs(float(w1["lm_head"].std()) - 0.02) < 1e-3


def test_round_to_bf16_matches_torch():
    rng = np.random.default_rng(12)
    a = (rng.standard_normal(10000) * 10 ** rng.uniform(-5, 5, 10000)).astype(np.float32)
    want = torch.from_numpy(a).to(torch.bfloat16).to(torch.float32).numpy()
    np.testing.assert_array_equal(round_to_bf16(a), want)
