"""GPU parity: every step of the CUDA path against the fp64 oracle, through the C ABI.

Both sides receive the same seeded inputs from ``workloads``.  Where the CUDA
step consumes bf16, both sides get the same bf16-rounded values.  Tolerances:

* whole forward (the published bar): max-abs logit error <= 3e-2 and relative
  loss error <= 5e-3; attention output max-abs <= 2e-2;
* single steps, derived from the arithmetic: a 16-bit output carries at most
  half an ulp of rounding (2^-9 relative for bf16, 2^-12 for fp16) on top of
  fp32 arithmetic, so it must sit within twice that (2^-8, 2^-11) times |x|, plus
  a small absolute term for fp32 table/accumulation error; fp32 outputs of fp32
  arithmetic within 1e-5 relative.  Every single-step test runs in both formats.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from workloads import SHAPES, make_qkv, make_tokens, make_weights, round_to_bf16

pytestmark = pytest.mark.gpu

DEV = "cuda"
BF16_REL = 2.0 ** -8
REL = {"bf16": 2.0 ** -8, "f16": 2.0 ** -11}
TDT = {"bf16": torch.bfloat16, "f16": torch.float16}
DTYPES = ["f16", "bf16"]


def bf16_dev(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(DEV).to(torch.bfloat16)


def round16(a, dt):
    """float32 values rounded to the 16-bit format (nearest even), as float32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    return round_to_bf16(a) if dt == "bf16" else a.astype(np.float16).astype(np.float32)


def dev16(a, dt):
    return torch.from_numpy(round16(a, dt)).to(DEV).to(TDT[dt])


def host(t):
    return t.float().cpu().numpy().astype(np.float64)


def status_word():
    return torch.zeros(64, dtype=torch.int32, device=DEV)


def assert_close_bf16(got, want, atol, what, rel=BF16_REL):
    err = np.abs(got - want) - (rel * np.abs(want) + atol)
    worst = float(err.max()) if err.size else -1.0
    assert worst <= 0.0, f"{what}: exceeds the 16-bit bound by {worst:.3e} (max abs err {np.abs(got - want).max():.3e})"


# ---------------------------------------------------------------- single steps

def test_cast_weights_bit_exact(gpu):
    rng = np.random.default_rng(1)
    a = (rng.standard_normal(100_000) * 10.0 ** rng.uniform(-30, 30, 100_000)).astype(np.float32)
    a[:8] = [0.0, -0.0, 1.0, -1.5, 3.0e38, -3.0e38, 1e-40, 65504.0]
    src = torch.from_numpy(a).to(DEV)
    dst = torch.empty(a.size, dtype=torch.bfloat16, device=DEV)
    gpu.cast_weights(src, dst)
    torch.cuda.synchronize()
    want = torch.from_numpy(a).to(torch.bfloat16)
    assert torch.equal(dst.cpu().view(torch.int16), want.view(torch.int16))
    np.testing.assert_array_equal(dst.float().cpu().numpy(), oracle.to_bf16(a).astype(np.float32))
    # fp16 container: the bf16 value, held exactly where fp16 can (|w| >= 2^-14)
    w = (rng.standard_normal(100_000) * 0.02).astype(np.float32)
    w[:4] = [1e-6, -3e-5, 7e-5, 0.0]
    d16 = torch.empty(w.size, dtype=torch.float16, device=DEV)
    gpu.cast_weights(torch.from_numpy(w).to(DEV), d16)
    torch.cuda.synchronize()
    want = oracle.to_bf16(w)
    got = d16.cpu().numpy().astype(np.float64)
    normal = np.abs(want) >= 2.0 ** -14
    np.testing.assert_array_equal(got[normal], want[normal])
    assert np.abs(got[~normal] - want[~normal]).max() <= 2.0 ** -25


def test_embedding_exact_and_token_range(gpu):
    rng = np.random.default_rng(2)
    V, C, M = 512, 128, 333
    wte = rng.standard_normal((V, C)).astype(np.float32)
    tok = rng.integers(0, V, M).astype(np.int32)
    x = torch.empty((M, C), dtype=torch.float32, device=DEV)
    st = status_word()
    gpu.embedding(torch.from_numpy(tok).to(DEV), torch.from_numpy(wte).to(DEV), x, st)
    assert gpu.get_status(st) == 0
    np.testing.assert_array_equal(x.cpu().numpy(), oracle.embed(wte, tok).astype(np.float32))
    tok[5] = V + 3
    tok[9] = -2
    gpu.embedding(torch.from_numpy(tok).to(DEV), torch.from_numpy(wte).to(DEV), x, st)
    assert gpu.get_status(st) == 6
    np.testing.assert_array_equal(x[5].cpu().numpy(), wte[0])


@pytest.mark.parametrize("dt", DTYPES)
@pytest.mark.parametrize("C", [128, 768, 1280, 1664, 2048, 4096])
def test_rmsnorm_parity(gpu, C, dt):
    rng = np.random.default_rng(C)
    M = 1001
    x = (rng.standard_normal((M, C)) * rng.uniform(0.01, 30, (M, 1))).astype(np.float32)
    out = torch.empty((M, C), dtype=TDT[dt], device=DEV)
    gpu.rmsnorm(torch.from_numpy(x).to(DEV), out, eps=1e-6)
    torch.cuda.synchronize()
    assert_close_bf16(host(out), oracle.rms_norm(x, 1e-6), 1e-6, f"rmsnorm C={C}", rel=2 * REL[dt])


@pytest.mark.parametrize("T,D", [(300, 64), (2048, 128), (8192, 128)])
def test_rope_table(gpu, T, D):
    tab = torch.empty((2, T, D // 2), dtype=torch.float32, device=DEV)
    gpu.rope_table(tab, T, D, 10000.0)
    torch.cuda.synchronize()
    cos, sin = oracle.rope_tables(T, D, 10000.0)
    np.testing.assert_allclose(tab[0].cpu().numpy(), cos, atol=6e-8, rtol=0)
    np.testing.assert_allclose(tab[1].cpu().numpy(), sin, atol=6e-8, rtol=0)


@pytest.mark.parametrize("dt", DTYPES)
@pytest.mark.parametrize("D,H,Hkv,fused", [(64, 4, 2, False), (128, 4, 4, False), (128, 6, 2, True),
                                           (128, 10, 10, True)])
def test_rope_qknorm_parity(gpu, D, H, Hkv, fused, dt):
    rng = np.random.default_rng(D + H + Hkv)
    B, T = 2, 301
    q = round16((rng.standard_normal((B, T, H, D)) * 3).astype(np.float32), dt)
    k = round16((rng.standard_normal((B, T, Hkv, D)) * 0.2).astype(np.float32), dt)
    cfg = oracle.OracleConfig(1, 64, H, Hkv, D, T, 512)
    wq, wk = oracle.rope_qknorm(q, k, cfg)
    tab = torch.empty((2, T, D // 2), dtype=torch.float32, device=DEV)
    gpu.rope_table(tab, T, D, 10000.0)
    if fused:  # q and k as column blocks of one [B*T, (H+2Hkv)*D] buffer
        n = (H + 2 * Hkv) * D
        buf = torch.zeros((B * T, n), dtype=TDT[dt], device=DEV)
        buf[:, :H * D] = dev16(q.reshape(B * T, H * D), dt)
        buf[:, H * D:(H + Hkv) * D] = dev16(k.reshape(B * T, Hkv * D), dt)
        qv, kv = buf[:, :H * D], buf[:, H * D:(H + Hkv) * D]
        gpu.rope_qknorm(buf, buf[:, H * D:], tab, B, T, H, Hkv, D, q_row_stride=n, k_row_stride=n)
        torch.cuda.synchronize()
        gq, gk = host(qv).reshape(B, T, H, D), host(kv).reshape(B, T, Hkv, D)
        assert torch.all(buf[:, (H + Hkv) * D:] == 0)  # v block untouched
    else:
        tq, tk = dev16(q, dt), dev16(k, dt)
        gpu.rope_qknorm(tq, tk, tab, B, T, H, Hkv, D)
        torch.cuda.synchronize()
        gq, gk = host(tq), host(tk)
    assert_close_bf16(gq, wq, 1e-4, "rope_qknorm q", rel=2 * REL[dt])
    assert_close_bf16(gk, wk, 1e-4, "rope_qknorm k", rel=2 * REL[dt])


@pytest.mark.parametrize("T,H,Hkv,W,D", [(1, 2, 2, 0, 128), (17, 4, 4, 5, 128), (128, 4, 2, 64, 128),
                                         (300, 4, 1, 0, 128), (300, 4, 4, 1, 128), (1000, 4, 2, 200, 128),
                                         (1000, 2, 2, 1000, 128), (777, 8, 2, 256, 128), (256, 2, 2, 64, 64),
                                         (300, 4, 2, 0, 64), (129, 2, 1, 7, 64)])
@pytest.mark.parametrize("dt", DTYPES)
def test_attention_parity(gpu, T, H, Hkv, W, D, dt):
    B = 2
    q, k, v = make_qkv(B, T, H, Hkv, D, seed=T * 7 + W)
    q, k, v = round16(q, dt), round16(k, dt), round16(v, dt)
    out = torch.empty((B, T, H, D), dtype=TDT[dt], device=DEV)
    gpu.attention(dev16(q, dt), dev16(k, dt), dev16(v, dt), out, W)
    torch.cuda.synchronize()
    want = oracle.attention(q, k, v, W if W > 0 else T)
    err = np.abs(host(out) - want).max()
    assert err <= 2e-2, f"attention max-abs {err:.3e}"


@pytest.mark.parametrize("T", [2048, 4096, 8192])
@pytest.mark.parametrize("Hkv", [16, 4])
@pytest.mark.parametrize("full", [False, True])
@pytest.mark.parametrize("dt", DTYPES)
def test_attention_sweep_parity(gpu, T, Hkv, full, dt):
    """The attention-only workload: B=4, H=16, D=128, N(0,1) bf16 q/k/v, RoPE +
    QK-norm first (GPU kernel vs fp64 oracle from the same bf16 values), window
    T/4 or full; oracle evaluated on sampled query rows."""
    B, H, D = 4, 16, 128
    W = T if full else T // 4
    q, k, v = make_qkv(B, T, H, Hkv, D)
    q, k, v = round16(q, dt), round16(k, dt), round16(v, dt)
    tq, tk, tv = dev16(q, dt), dev16(k, dt), dev16(v, dt)
    tab = torch.empty((2, T, D // 2), dtype=torch.float32, device=DEV)
    gpu.rope_table(tab, T, D, 10000.0)
    gpu.rope_qknorm(tq, tk, tab, B, T, H, Hkv, D)
    out = torch.empty((B, T, H, D), dtype=TDT[dt], device=DEV)
    gpu.attention(tq, tk, tv, out, W)
    torch.cuda.synchronize()
    cfg = oracle.OracleConfig(1, 64, H, Hkv, D, T, 512)
    oq, ok = oracle.rope_qknorm(q, k, cfg)
    rng = np.random.default_rng(T + Hkv)
    rows = sorted(set([0, 1, 2, 63, 64, 127, 128, W - 1, W, W + 1, T // 2, T - 2, T - 1] +
                      list(rng.integers(0, T, 16))))
    rows = [r for r in rows if 0 <= r < T]
    want = oracle.attention(oq, ok, v, W, query_positions=rows)
    err = np.abs(host(out)[:, rows] - want).max()
    assert err <= 2e-2, f"attention sweep T={T} Hkv={Hkv} W={W}: max-abs {err:.3e}"


@pytest.mark.parametrize("W", [1024, 0])
def test_attention_lse_run_to_run_identical(gpu, W):
    """The forward attention with its log-sum-exp output (the backward reads it),
    twice on the same inputs with many work items per CTA (B=4, H=16, T=4096,
    four query heads per kv head; a 1024-key window and full causal): output
    and log-sum-exp are bit-identical -- no state crosses work items and every
    sum runs in a fixed order."""
    B, T, H, Hkv, D = 4, 4096, 16, 4, 128
    g = torch.Generator().manual_seed(5)
    qkv = torch.randn((B, T, H + 2 * Hkv, D), generator=g)
    qk = qkv[:, :, :H + Hkv]
    qkv[:, :, :H + Hkv] = qk / qk.pow(2).mean(-1, keepdim=True).sqrt()
    qkv = qkv.to(torch.float16).reshape(B, T, -1).contiguous().to(DEV)
    runs = []
    for _ in range(2):
        out = torch.full((B, T, H * D), float("nan"), dtype=torch.float16, device=DEV)
        lse = torch.full((B, T, H), float("nan"), dtype=torch.float32, device=DEV)
        gpu.attention_lse(qkv, out, lse, H, Hkv, D, W)
        runs.append((out, lse))
    torch.cuda.synchronize()
    assert torch.isfinite(runs[0][1]).all() and not torch.isnan(runs[0][0]).any()
    assert torch.equal(runs[0][0], runs[1][0]) and torch.equal(runs[0][1], runs[1][1])


GEMM_SHAPES = [(128, 256, 64), (1, 256, 128), (300, 352, 200), (1000, 800, 520), (64, 32, 8),
               (2048, 3840, 1280), (520, 5120, 1280), (256, 1280, 5120)]


@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
@pytest.mark.parametrize("epi", ["store_16", "relu2_16", "resid_f32", "store_f32", "softcap_f32"])
@pytest.mark.parametrize("dt", DTYPES)
def test_linear_parity(gpu, M, N, K, epi, dt):
    rng = np.random.default_rng(M * 31 + N * 7 + K)
    a = round16(rng.standard_normal((M, K)).astype(np.float32), dt)
    w = round16((rng.standard_normal((N, K)) / math.sqrt(K) * 3).astype(np.float32), dt)
    acc = a.astype(np.float64) @ w.astype(np.float64).T
    st = status_word()
    if epi in ("store_16", "relu2_16"):
        out = torch.full((M, N), float("nan"), dtype=TDT[dt], device=DEV)
        code = gpu.EPI_STORE_16 if epi == "store_16" else gpu.EPI_RELU2_16
        gpu.linear(dev16(a, dt), dev16(w, dt), out, code, status=st)
        want = acc if epi == "store_16" else np.maximum(acc, 0.0) ** 2
        assert gpu.get_status(st) == 0
        assert_close_bf16(host(out), want, 1e-5 * math.sqrt(K), f"linear {epi}", rel=2 * REL[dt])
    else:
        x0 = rng.standard_normal((M, N)).astype(np.float32)
        out = torch.from_numpy(x0).to(DEV) if epi == "resid_f32" else \
            torch.full((M, N), float("nan"), dtype=torch.float32, device=DEV)
        code = {"resid_f32": gpu.EPI_RESID_F32, "store_f32": gpu.EPI_STORE_F32,
                "softcap_f32": gpu.EPI_SOFTCAP_F32}[epi]
        gpu.linear(dev16(a, dt), dev16(w, dt), out, code, cap=15.0, status=st)
        want = {"resid_f32": x0 + acc, "store_f32": acc, "softcap_f32": oracle.softcap(acc, 15.0)}[epi]
        assert gpu.get_status(st) == 0
        got = out.cpu().numpy().astype(np.float64)
        np.testing.assert_allclose(got, want, rtol=1e-5, atol=2e-6 * math.sqrt(K), err_msg=f"linear {epi}")


@pytest.mark.parametrize("epi", ["store_16", "relu2_16"])
def test_linear_f16_saturation_flagged(gpu, epi):
    """fp16 activations saturate at +-65504: a ReLU^2 pre-activation above 256
    (or a stored product above 65504) sets NC_DEV_F16_RANGE, reported as
    NC_ERR_F16_RANGE; the same product just inside the range, and in bf16, does
    not.  Host-made inputs, no fault."""
    M, N, K = 300, 256, 64
    code = gpu.EPI_STORE_16 if epi == "store_16" else gpu.EPI_RELU2_16
    limit = 65504.0 if epi == "store_16" else 256.0  # largest pre-activation that fits
    for scale, dt, flagged in ((1.05, "f16", True), (0.95, "f16", False), (1.05, "bf16", False)):
        a = np.zeros((M, K), dtype=np.float32)
        a[:, :2] = 1.0
        w = np.zeros((N, K), dtype=np.float32)
        w[7, :2] = limit * scale / 2  # column 7 of every row: a pre-activation of limit * scale
        w[9, 0] = 1.0
        st = status_word()
        out = torch.empty((M, N), dtype=TDT[dt], device=DEV)
        gpu.linear(dev16(a, dt), dev16(w, dt), out, code, status=st)
        assert gpu.get_status(st) == (10 if flagged else 0), (epi, scale, dt)
        if flagged:
            assert host(out)[:, 7].max() == 65504.0  # saturated, not inf


def test_forward_f16_saturation_flagged(gpu):
    """The tiny forward with c_fc weights scaled so its pre-activations pass 256:
    the fp16 forward reports NC_ERR_F16_RANGE, the bf16 forward does not."""
    s = SHAPES["tiny"]
    w = make_weights(s)
    w = {**w, "layers": [dict(L) for L in w["layers"]]}
    w["layers"][0]["c_fc"] = w["layers"][0]["c_fc"] * 4000.0
    x, y = make_tokens(s)
    for act, want in ((gpu.F16, 10), (gpu.BF16, 0)):
        cfg = gpu.make_config(s.n_layer, s.d_model, s.n_head, s.n_kv_head, s.head_dim, s.seq_len, s.vocab,
                              s.short_window, act_dtype=act)
        model = gpu.Model.from_numpy(cfg, w)
        res = gpu.forward(model, torch.from_numpy(x).to(DEV), torch.from_numpy(y).to(DEV))
        assert gpu.get_status(res["workspace"]) == want


@pytest.mark.parametrize("dt", DTYPES)
@pytest.mark.parametrize("M,C,H,Hkv,D,T", [(2 * 300, 256, 2, 1, 64, 300), (1024, 768, 6, 6, 128, 512),
                                          (384, 512, 4, 2, 128, 128), (4096, 1280, 10, 10, 128, 2048)])
def test_qkv_rope_parity(gpu, M, C, H, Hkv, D, T, dt):
    """Fused QKV projection + RoPE + QK-norm against the oracle's projection, RoPE
    and per-head RMSNorm (positions restart every T rows)."""
    rng = np.random.default_rng(M + C + D)
    N = (H + 2 * Hkv) * D
    a = round16(rng.standard_normal((M, C)).astype(np.float32), dt)
    w = round16((rng.standard_normal((N, C)) * 0.02).astype(np.float32), dt)
    tab = torch.empty((2, T, D // 2), dtype=torch.float32, device=DEV)
    gpu.rope_table(tab, T, D, 10000.0)
    out = torch.full((M, N), float("nan"), dtype=TDT[dt], device=DEV)
    st = status_word()
    gpu.qkv_rope(dev16(a, dt), dev16(w, dt), out, tab, T, H, Hkv, D, eps=1e-6, status=st)
    assert gpu.get_status(st) == 0
    acc = a.astype(np.float64) @ w.astype(np.float64).T
    B = M // T
    q = acc[:, :H * D].reshape(B, T, H, D)
    k = acc[:, H * D:(H + Hkv) * D].reshape(B, T, Hkv, D)
    wq, wk = oracle.rope_qknorm(q, k, oracle.OracleConfig(1, C, H, Hkv, D, T, 512))
    got = host(out)
    assert_close_bf16(got[:, :H * D], wq.reshape(M, H * D), 2e-4, "qkv_rope q", rel=2 * REL[dt])
    assert_close_bf16(got[:, H * D:(H + Hkv) * D], wk.reshape(M, Hkv * D), 2e-4, "qkv_rope k", rel=2 * REL[dt])
    assert_close_bf16(got[:, (H + Hkv) * D:], acc[:, (H + Hkv) * D:], 2e-4, "qkv_rope v", rel=2 * REL[dt])


def test_linear_row_stride(gpu):
    """Output written into a column block of a wider buffer (ldo > N)."""
    rng = np.random.default_rng(5)
    M, N, K, ldo = 200, 256, 128, 640
    a = round_to_bf16(rng.standard_normal((M, K)).astype(np.float32))
    w = round_to_bf16(rng.standard_normal((N, K)).astype(np.float32))
    big = torch.zeros((M, ldo), dtype=torch.float32, device=DEV)
    gpu.linear(bf16_dev(a), bf16_dev(w), big[:, 128:128 + N], gpu.EPI_STORE_F32)
    torch.cuda.synchronize()
    got = big.cpu().numpy()
    np.testing.assert_allclose(got[:, 128:128 + N], a.astype(np.float64) @ w.T.astype(np.float64), rtol=1e-5, atol=1e-4)
    assert np.all(got[:, :128] == 0) and np.all(got[:, 128 + N:] == 0)


@pytest.mark.parametrize("V", [512, 32768])
def test_softcap_ce_parity(gpu, V):
    rng = np.random.default_rng(V)
    M = 300
    z = (rng.standard_normal((M, V)) * 6).astype(np.float32)
    y = rng.integers(0, V, M).astype(np.int32)
    y[::7] = -1
    tl = torch.empty(M, dtype=torch.float32, device=DEV)
    capped = torch.empty((M, V), dtype=torch.float32, device=DEV)
    st = status_word()
    gpu.softcap_ce(torch.from_numpy(z).to(DEV), torch.from_numpy(y).to(DEV), tl, capped, 15.0, st)
    assert gpu.get_status(st) == 0
    lc = oracle.softcap(z, 15.0)
    nll, loss = oracle.cross_entropy(lc, y)
    np.testing.assert_allclose(capped.cpu().numpy(), lc, rtol=0, atol=2e-5)
    np.testing.assert_allclose(tl.cpu().numpy(), nll, rtol=2e-5, atol=2e-5)
    lm = torch.empty((), dtype=torch.float32, device=DEV)
    gpu.loss_mean(tl, torch.from_numpy(y).to(DEV), V, lm)
    assert abs(lm.item() - loss) <= 2e-5 * abs(loss)
    # a target outside the vocabulary is flagged and ignored
    y[3] = V + 1
    gpu.softcap_ce(torch.from_numpy(z).to(DEV), torch.from_numpy(y).to(DEV), tl, None, 15.0, st)
    assert gpu.get_status(st) == 6
    assert tl[3].item() == 0.0


def test_loss_mean_empty_is_nan(gpu):
    tl = torch.ones(100, dtype=torch.float32, device=DEV)
    y = torch.full((100,), -1, dtype=torch.int32, device=DEV)
    lm = torch.empty((), dtype=torch.float32, device=DEV)
    gpu.loss_mean(tl, y, 512, lm)
    assert math.isnan(lm.item())


def test_bounded_wait_times_out_and_context_survives(gpu):
    st = status_word()
    gpu.selftest_bounded_wait(st, limit_us=20000)
    assert gpu.get_status(st) == 7
    # the context is still usable afterwards
    x = torch.ones(1024, device=DEV)
    assert x.sum().item() == 1024.0


# ---------------------------------------------------------------- whole forward

def _oracle_cfg(s):
    return oracle.OracleConfig(s.n_layer, s.d_model, s.n_head, s.n_kv_head, s.head_dim, s.seq_len,
                               s.vocab, short_window=s.short_window)


def _nc_cfg(nc, s):
    return nc.make_config(s.n_layer, s.d_model, s.n_head, s.n_kv_head, s.head_dim, s.seq_len, s.vocab,
                          s.short_window)


_MODELS = {}


def _model(nc, name):
    if name not in _MODELS:
        _MODELS.clear()
        torch.cuda.empty_cache()
        s = SHAPES[name]
        w = make_weights(s)
        _MODELS[name] = (w, nc.Model.from_numpy(_nc_cfg(nc, s), w))
    return _MODELS[name]


def test_forward_tiny_full_batch(gpu):
    s = SHAPES["tiny"]
    w, model = _model(gpu, "tiny")
    x, y = make_tokens(s)
    y = y.copy()
    y[0, ::5] = -1
    tx, ty = torch.from_numpy(x).to(DEV), torch.from_numpy(y).to(DEV)
    res = gpu.forward(model, tx, ty, want_logits=True, want_token_loss=True)
    assert gpu.get_status(res["workspace"]) == 0
    want = oracle.forward(_oracle_cfg(s), w, x, y)
    err = np.abs(res["logits"].cpu().numpy() - want["logits"]).max()
    assert err <= 3e-2, f"tiny logits max-abs {err:.3e}"
    rel = abs(res["loss"].item() - want["loss"]) / abs(want["loss"])
    assert rel <= 5e-3, f"tiny loss rel {rel:.3e}"
    np.testing.assert_allclose(res["token_loss"].cpu().numpy(), want["token_loss"], rtol=5e-3, atol=1e-3)
    # logits-only path (no targets) gives the same soft-capped logits
    res2 = gpu.forward(model, tx, None, want_logits=True)
    torch.cuda.synchronize()
    assert torch.equal(res2["logits"], res["logits"])


def test_forward_tiny_bf16_activations(gpu):
    """The all-bf16 activation mode (act_dtype NC_BF16) on the tiny workload."""
    s = SHAPES["tiny"]
    w = make_weights(s)
    cfg = gpu.make_config(s.n_layer, s.d_model, s.n_head, s.n_kv_head, s.head_dim, s.seq_len, s.vocab,
                          s.short_window, act_dtype=gpu.BF16)
    model = gpu.Model.from_numpy(cfg, w)
    x, y = make_tokens(s)
    res = gpu.forward(model, torch.from_numpy(x).to(DEV), torch.from_numpy(y).to(DEV), want_logits=True)
    assert gpu.get_status(res["workspace"]) == 0
    want = oracle.forward(_oracle_cfg(s), w, x, y)
    assert np.abs(res["logits"].cpu().numpy() - want["logits"]).max() <= 3e-2
    assert abs(res["loss"].item() - want["loss"]) <= 5e-3 * abs(want["loss"])


@pytest.mark.parametrize("B,T", [(1, 1), (3, 100), (1, 256), (2, 65)])
def test_forward_tiny_ragged(gpu, B, T):
    s = SHAPES["tiny"]
    w, model = _model(gpu, "tiny")
    x, y = make_tokens(s, seed=B * 1000 + T, batch=B, seq_len=T)
    res = gpu.forward(model, torch.from_numpy(x).to(DEV), torch.from_numpy(y).to(DEV), want_logits=True)
    assert gpu.get_status(res["workspace"]) == 0
    want = oracle.forward(_oracle_cfg(s), w, x, y)
    assert np.abs(res["logits"].cpu().numpy() - want["logits"]).max() <= 3e-2
    assert abs(res["loss"].item() - want["loss"]) <= 5e-3 * abs(want["loss"])


def test_forward_bad_tokens_flagged(gpu):
    s = SHAPES["tiny"]
    _, model = _model(gpu, "tiny")
    x, y = make_tokens(s)
    x, y = x.copy(), y.copy()
    x[1, 7] = s.vocab + 9
    res = gpu.forward(model, torch.from_numpy(x).to(DEV), torch.from_numpy(y).to(DEV))
    assert gpu.get_status(res["workspace"]) == 6
    x[1, 7] = 0
    y[0, 3] = -7
    res = gpu.forward(model, torch.from_numpy(x).to(DEV), torch.from_numpy(y).to(DEV))
    assert gpu.get_status(res["workspace"]) == 6


PREFIX = 640  # > the 512-key short window, so windowed rows are compared too


@pytest.mark.parametrize("name", ["d12", "d20", "d26", "d26_gqa"])
def test_forward_full_size_sampled_rows(gpu, name):
    """Full-size batch in the bench's launch configuration; the oracle recomputes
    the whole of row B-1 (all T positions: the full-context layers' attention
    over every prefix length, the short-window layers at every window offset)
    and row 0 over its first PREFIX positions (causality makes those outputs
    depend on nothing later).  Bars: logits max-abs <= 3e-2, per-token and
    mean loss relative <= 5e-3."""
    s = SHAPES[name]
    w, model = _model(gpu, name)
    x, y = make_tokens(s)
    tx, ty = torch.from_numpy(x).to(DEV), torch.from_numpy(y).to(DEV)
    res = gpu.forward(model, tx, ty, want_logits=True, want_token_loss=True)
    assert gpu.get_status(res["workspace"]) == 0
    full_row, pre_row = s.batch - 1, 0
    got = {"full": (res["logits"][full_row].cpu().numpy(), res["token_loss"][full_row].cpu().numpy()),
           "prefix": (res["logits"][pre_row, :PREFIX].cpu().numpy(),
                      res["token_loss"][pre_row, :PREFIX].cpu().numpy())}
    # the timed configuration (no logits requested) gives bit-identical losses
    res_fast = gpu.forward(model, tx, ty, want_token_loss=True)
    torch.cuda.synchronize()
    assert torch.equal(res_fast["token_loss"], res["token_loss"])
    assert res_fast["loss"].item() == res["loss"].item()
    tl_all = res["token_loss"].double()
    assert abs(tl_all.mean().item() - res["loss"].item()) <= 1e-5 * abs(res["loss"].item())
    del res, res_fast
    inputs = {"full": (x[[full_row]], y[[full_row]]), "prefix": (x[[pre_row], :PREFIX], y[[pre_row], :PREFIX])}
    for part, (xi, yi) in inputs.items():
        want = oracle.forward(_oracle_cfg(s), w, xi, yi)
        got_logits, got_tl = got[part]
        err = np.abs(got_logits - want["logits"][0]).max()
        assert err <= 3e-2, f"{name} {part} row logits max-abs {err:.3e}"
        rel_rows = np.abs(got_tl - want["token_loss"][0]) / np.abs(want["token_loss"][0])
        assert rel_rows.max() <= 5e-3, f"{name} {part} row per-token loss rel {rel_rows.max():.3e}"
        rel = abs(got_tl.mean() - want["loss"]) / abs(want["loss"])
        assert rel <= 5e-3, f"{name} {part} row loss rel {rel:.3e}"


def test_forward_deterministic_and_causal(gpu):
    s = SHAPES["d12"]
    _, model = _model(gpu, "d12")
    x, y = make_tokens(s, batch=2)
    tx, ty = torch.from_numpy(x).to(DEV), torch.from_numpy(y).to(DEV)
    a = gpu.forward(model, tx, ty, want_logits=True, want_token_loss=True)
    b = gpu.forward(model, tx, ty, want_logits=True, want_token_loss=True)
    torch.cuda.synchronize()
    assert torch.equal(a["logits"], b["logits"]) and torch.equal(a["token_loss"], b["token_loss"])
    t = 1500
    x2 = x.copy()
    x2[:, t] = (x2[:, t] + 1) % s.vocab
    c = gpu.forward(model, torch.from_numpy(x2).to(DEV), ty, want_logits=True)
    torch.cuda.synchronize()
    assert torch.equal(c["logits"][:, :t], a["logits"][:, :t])
    assert not torch.equal(c["logits"][:, t], a["logits"][:, t])
