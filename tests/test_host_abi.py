"""CPU-only checks of the C ABI: the library loads, exports every entry point the
header declares, derives configurations as the pages do, and rejects bad
arguments on the host before touching a device."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
from workloads import SHAPES

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
GOLDEN = os.path.join(ROOT, "tests", "golden")


def _declared_symbols():
    with open(os.path.join(ROOT, "include", "nc.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(nc_[a-z0-9_]+)\s*\(", text)))


def test_header_symbols_exported(nclib):
    names = _declared_symbols()
    assert len(names) >= 20
    L = nclib.lib()
    for n in names:
        assert hasattr(L, n), f"{n} declared in include/nc.h but not exported"
    assert L.nc_version() >= 100


def test_init_config_matches_pages_and_oracle(nclib):
    rows = [l.split() for l in open(os.path.join(GOLDEN, "config_examples.txt"))
            if l.strip() and not l.startswith("#") and l.startswith("derive")]
    for _, depth, aspect, hd, model_dim, heads in rows:
        c = nclib.init_config(int(depth), int(aspect), int(hd))
        assert (c.d_model, c.n_head, c.n_kv_head, c.head_dim) == (int(model_dim), int(heads), int(heads), int(hd))
        assert c.short_window == 512 and c.window_pattern == b"SSSL" and c.softcap == 15.0


@pytest.mark.parametrize("name", list(SHAPES))
def test_layer_windows_agree_with_oracle(nclib, name):
    s = SHAPES[name]
    c = nclib.make_config(s.n_layer, s.d_model, s.n_head, s.n_kv_head, s.head_dim, s.seq_len, s.vocab,
                          s.short_window)
    oc = oracle.OracleConfig(s.n_layer, s.d_model, s.n_head, s.n_kv_head, s.head_dim, s.seq_len, s.vocab,
                             short_window=s.short_window)
    assert [nclib.layer_window(c, l) for l in range(s.n_layer)] == oracle.layer_windows(oc)
    assert nclib.layer_window(c, s.n_layer) == -1


def test_forward_flops_counts(nclib):
    # published totals of the FLOP model (attention counted inside the window only)
    want = {"d12": 3.965, "d20": 61.011, "d26": 63.611, "d26_gqa": 83.650}
    for name, tf in want.items():
        s = SHAPES[name]
        c = nclib.make_config(s.n_layer, s.d_model, s.n_head, s.n_kv_head, s.head_dim, s.seq_len,
                              s.vocab, s.short_window)
        assert abs(nclib.forward_flops(c, s.batch, s.seq_len) / 1e12 - tf) < 5e-4
    # brute-force count of visible (query, key) pairs on a tiny case
    c = nclib.make_config(2, 128, 2, 1, 64, 16, 512, 5)
    T, B = 16, 3
    pairs = 0
    for W in (5, 16):
        pairs += sum(oracle.window_visible(i, j, W) for i in range(T) for j in range(T))
    M, C, D, H, Hkv, V = B * T, 128, 64, 2, 1, 512
    proj = 2 * (2 * M * C * (H + 2 * Hkv) * D + 2 * M * H * D * C + 16 * M * C * C) + 2 * M * C * V
    assert nclib.forward_flops(c, B, T) == pytest.approx(proj + 4 * D * H * B * pairs, rel=1e-12)


def test_workspace_bytes(nclib):
    c = nclib.init_config(20)
    ws = nclib.workspace_bytes(c, 32, 2048)
    assert 2.5e9 < ws < 3.5e9
    assert nclib.workspace_bytes(c, 32, 4096) == 0  # T > seq_len
    assert nclib.workspace_bytes(c, 0, 2048) == 0


def test_bad_configs_rejected(nclib):
    L = nclib.lib()
    c = nclib.NcConfig()
    assert L.nc_init_config(None, 20, 64, 128, 0, 2048, 32768) == 1
    assert L.nc_init_config(ctypes.byref(c), 20, 64, 128, 3, 2048, 32768) == 2  # 10 % 3 != 0
    assert L.nc_init_config(ctypes.byref(c), 20, 64, 96, 0, 2048, 32768) == 2  # head_dim
    assert L.nc_init_config(ctypes.byref(c), 20, 64, 128, 0, 2048, 1000) == 2  # vocab % 64
    good = nclib.init_config(2, 64, 64, 0, 256, 512)
    bad = nclib.NcConfig.from_buffer_copy(good)
    bad.window_pattern = b"SSXL"
    assert nclib.check_config(bad) == 2
    assert nclib.check_config(good) == 0


class _FakeWeights:
    """nc_weights whose device pointers are aligned integers never dereferenced."""

    def __init__(self, nclib, n_layer, base=1 << 40, misalign=False):
        mk = lambda: (ctypes.c_void_p * n_layer)(*[base + 4096 * i for i in range(n_layer)])
        self.arrs = [mk() for _ in range(6)]
        if misalign:
            self.arrs[4][0] = base + 8
        FPP = ctypes.POINTER(ctypes.c_void_p)
        self.w = nclib.NcWeights(base, *[ctypes.cast(a, FPP) for a in self.arrs], base + 64)


def _fwd(nclib, cfg, fw, B, T, tokens=1 << 41, targets=1 << 41, ws=1 << 42, ws_bytes=None, loss=None):
    L = nclib.lib()
    if ws_bytes is None:
        ws_bytes = max(nclib.workspace_bytes(cfg, B, T), 1)
    return L.nc_forward(ctypes.byref(cfg), ctypes.byref(fw.w), tokens, targets, B, T, None, None, loss,
                        ws, ws_bytes, None)


def test_forward_host_validation(nclib):
    cfg = nclib.init_config(2, 64, 64, 0, 256, 512)
    fw = _FakeWeights(nclib, 2)
    assert _fwd(nclib, cfg, fw, 2, 512) == 3                      # T > seq_len
    assert _fwd(nclib, cfg, fw, 0, 16) == 3                       # B < 1
    assert _fwd(nclib, cfg, fw, 2, 16, tokens=None) == 1          # NULL tokens
    assert _fwd(nclib, cfg, fw, 2, 16, targets=None, loss=1 << 43) == 1  # loss without targets
    assert _fwd(nclib, cfg, fw, 2, 16, ws_bytes=1024) == 5        # workspace too small
    assert _fwd(nclib, cfg, fw, 2, 16, ws=(1 << 42) + 16) == 4    # workspace not 256-aligned
    assert _fwd(nclib, cfg, _FakeWeights(nclib, 2, misalign=True), 2, 16) == 4
    bad = nclib.NcConfig.from_buffer_copy(cfg)
    bad.n_kv_head = 3
    assert _fwd(nclib, bad, fw, 2, 16) == 2


def test_no_device_fails_loudly(nclib):
    """With valid arguments and no sm_100 device every compute entry point refuses."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present; the device check passes there")
    cfg = nclib.init_config(2, 64, 64, 0, 256, 512)
    fw = _FakeWeights(nclib, 2)
    assert _fwd(nclib, cfg, fw, 2, 16) == 8
    L = nclib.lib()
    assert L.nc_rmsnorm(1 << 40, 1 << 41, 8, 128, 1e-6, 1, None) == 8
    assert L.nc_attention(1 << 40, 1 << 40, 1 << 40, 1 << 41, 1, 16, 2, 2, 128, 0, 1, None) == 8
    assert L.nc_linear(1 << 40, 1 << 40, 1 << 41, 128, 256, 64, 256, 0, 15.0, 1, None, None) == 8
    assert L.nc_selftest_bounded_wait(1 << 40, 100, None) == 8


def test_single_step_argument_checks(nclib):
    L = nclib.lib()
    A, B_ = 1 << 40, 1 << 41
    assert L.nc_linear(A, A, B_, 128, 250, 64, 256, 0, 15.0, 1, None, None) == 3  # N % 32
    assert L.nc_linear(A, A, B_, 128, 256, 60, 256, 0, 15.0, 1, None, None) == 3  # K % 8
    assert L.nc_linear(A + 2, A, B_, 128, 256, 64, 256, 0, 15.0, 1, None, None) == 4
    assert L.nc_linear(A, A, B_, 128, 256, 64, 256, 9, 15.0, 1, None, None) == 1  # epilogue
    assert L.nc_linear(A, A, B_, 128, 256, 64, 256, 0, 15.0, 7, None, None) == 1  # dtype
    assert L.nc_attention(A, A, A, B_, 1, 16, 4, 3, 128, 0, 1, None) == 1  # H % Hkv
    assert L.nc_attention(A, A, A, B_, 1, 16, 4, 4, 96, 0, 1, None) == 3
    assert L.nc_rope_qknorm(A, A, A, 1, 16, 2, 2, 96, 192, 192, 1e-6, 1, None) == 3
    assert L.nc_qkv_rope(A, A, B_, A, 128, 16, 128, 2, 2, 96, 1e-6, 1, None, None) == 3
    assert L.nc_cast_weights(A, B_, 12, 1, None) == 1
    assert L.nc_cast_weights(A, B_, 16, 5, None) == 1
    assert L.nc_softcap_ce(A, A, None, B_, 4, 512, -1.0, None, None) == 1
    assert L.nc_selftest_bounded_wait(None, 100, None) == 1
    assert L.nc_stream_wait_event(None, None) == 1  # no event
    assert L.nc_status_string(7) == b"bounded device wait ran out"
    c = nclib.init_config(2, 64, 64, 0, 256, 512)
    assert c.act_dtype == nclib.F16
    c.act_dtype = 3
    assert nclib.check_config(c) == 2


def test_extras_host_rules(nclib):
    """Full-nanochat terms: layer rule, config bits, workspace growth and host checks."""
    c4 = nclib.init_config(4, 64, 64, 0, 256, 512)
    c5 = nclib.init_config(5, 64, 64, 0, 256, 512)
    # every other layer counted back from the last (which always has one)
    assert [nclib.layer_value_embed(c4, l) for l in range(4)] == [0, 1, 0, 1]
    assert [nclib.layer_value_embed(c5, l) for l in range(5)] == [1, 0, 1, 0, 1]
    assert [bool(nclib.layer_value_embed(c5, l)) for l in range(5)] == oracle.value_embed_layers(5)
    assert nclib.layer_value_embed(c4, 4) == -1 and nclib.layer_value_embed(c4, -1) == -1
    bad = nclib.NcConfig.from_buffer_copy(c4)
    bad.extras = 16
    assert nclib.check_config(bad) == 2
    # x0 (resid lambdas) and x_mid (backout) streams are fp32 [B*T, C] each
    base = nclib.workspace_bytes(c4, 2, 256)
    stream = 2 * 256 * c4.d_model * 4
    for bits, n in ((nclib.EXTRA_SMEAR, 0), (nclib.EXTRA_VALUE_EMBED, 0), (nclib.EXTRA_RESID_LAMBDAS, 1),
                    (nclib.EXTRA_BACKOUT, 1), (nclib.EXTRA_ALL, 2)):
        cx = nclib.NcConfig.from_buffer_copy(c4)
        cx.extras = bits
        assert nclib.workspace_bytes(cx, 2, 256) == base + n * stream
    # enabled terms need their weights (checked before any device work)
    cfg = nclib.init_config(2, 64, 64, 0, 256, 512)
    fw = _FakeWeights(nclib, 2)
    for bits in (nclib.EXTRA_SMEAR, nclib.EXTRA_VALUE_EMBED, nclib.EXTRA_RESID_LAMBDAS, nclib.EXTRA_BACKOUT):
        cx = nclib.NcConfig.from_buffer_copy(cfg)
        cx.extras = bits
        assert _fwd(nclib, cx, fw, 2, 16) == 1
    # a value-embedding table is required only on the layers that use one
    cx = nclib.NcConfig.from_buffer_copy(cfg)
    cx.extras = nclib.EXTRA_VALUE_EMBED
    FPP = ctypes.POINTER(ctypes.c_void_p)
    tabs = (ctypes.c_void_p * 2)(None, 1 << 44)
    gates = (ctypes.c_void_p * 2)(None, (1 << 44) + 4096)
    fw.w.value_embeds, fw.w.ve_gates = ctypes.cast(tabs, FPP), ctypes.cast(gates, FPP)
    import torch
    want = 0 if torch.cuda.is_available() else 8  # passes the host checks
    if want == 8:
        assert _fwd(nclib, cx, fw, 2, 16) == 8
    tabs[1] = (1 << 44) + 8  # misaligned table
    assert _fwd(nclib, cx, fw, 2, 16) == 4


def test_kv_cache_host_rules(nclib):
    """Session sizing and the host-side refusals of nc_prefill / nc_decode_step."""
    L = nclib.lib()
    cfg = nclib.init_config(2, 64, 64, 0, 256, 512)
    n = L.nc_session_bytes(ctypes.byref(cfg), 2, 256)
    # at least the cache: layers x B x T_max x (k, v) x Hkv x D x 2 bytes
    assert n >= 2 * 2 * 256 * 2 * cfg.n_kv_head * cfg.head_dim * 2
    assert L.nc_session_bytes(ctypes.byref(cfg), 2, 257) == 0  # T_max > seq_len
    assert L.nc_prefill_workspace_bytes(ctypes.byref(cfg), 2, 100) < nclib.workspace_bytes(cfg, 2, 100)
    fw = _FakeWeights(nclib, 2)
    sess, tok, out = 1 << 43, 1 << 41, 1 << 44
    dec = lambda c, pos, nbytes=n, T_max=256: L.nc_decode_step(ctypes.byref(c), ctypes.byref(fw.w), tok, 2, pos,
                                                               out, sess, nbytes, T_max, None)
    assert dec(cfg, 256) == 3           # pos >= T_max
    assert dec(cfg, -1) == 3
    assert dec(cfg, 5, nbytes=n - 1) == 5  # session too small
    # the further terms: the session grows by the token record (smear) and the
    # x0 / x_mid rows; their parameters are checked as nc_forward checks them
    cx = nclib.NcConfig.from_buffer_copy(cfg)
    cx.extras = nclib.EXTRA_SMEAR
    nx = L.nc_session_bytes(ctypes.byref(cx), 2, 256)
    assert nx >= n + 2 * 256 * 4
    assert dec(cx, 5) == 5               # the plain stack's session is too small
    assert dec(cx, 5, nbytes=nx) == 1    # no smear gate
    call = nclib.NcConfig.from_buffer_copy(cfg)
    call.extras = nclib.EXTRA_ALL
    assert L.nc_session_bytes(ctypes.byref(call), 2, 256) >= nx + 2 * 2 * cfg.d_model * 4
    pre = lambda T, T_max=256: L.nc_prefill(ctypes.byref(cfg), ctypes.byref(fw.w), tok, 2, T, None, sess, n, T_max,
                                             1 << 42, 1 << 30, None)
    assert pre(300) == 3                 # T > T_max
    import torch
    if not torch.cuda.is_available():
        assert dec(cfg, 5) == 8          # valid arguments, no sm_100 device
        assert pre(100) == 8
        fw.w.smear_gate = (1 << 44) + 256
        assert dec(cx, 5, nbytes=nx) == 8
        fw.w.smear_gate = (1 << 44) + 8  # misaligned
        assert dec(cx, 5, nbytes=nx) == 4


def test_fp8_host_rules(nclib):
    """nc_config.fp8: accepted bits, workspace sizing, and the host-side
    refusals of the standalone e4m3 entry points and of the KV-cache path."""
    L = nclib.lib()
    cfg = nclib.init_config(2, 64, 64, 0, 256, 512)
    assert cfg.fp8 == 0
    base = nclib.workspace_bytes(cfg, 2, 100)
    for bits in (nclib.FP8_BLOCK, nclib.FP8_LM_HEAD, nclib.FP8_ALL):
        c = nclib.NcConfig.from_buffer_copy(cfg)
        c.fp8 = bits
        assert nclib.check_config(c) == 0
        assert nclib.workspace_bytes(c, 2, 100) > 0
    c = nclib.NcConfig.from_buffer_copy(cfg)
    c.fp8 = 4
    assert nclib.check_config(c) == 2
    assert nclib.workspace_bytes(c, 2, 100) == 0
    # e4m3 block weights take one byte instead of two; the a8 / amax scratch is M x 4C bytes + slots
    c.fp8 = nclib.FP8_BLOCK
    C, L_ = cfg.d_model, cfg.n_layer
    wblock = L_ * ((cfg.n_head + 2 * cfg.n_kv_head) * cfg.head_dim * C + C * cfg.n_head * cfg.head_dim + 8 * C * C)
    M = 200
    assert nclib.workspace_bytes(c, 2, 100) - base >= M * 4 * C - wblock - 4096
    # the KV-cache path is 16-bit only
    n = L.nc_session_bytes(ctypes.byref(cfg), 2, 256)
    fw = _FakeWeights(nclib, 2)
    assert L.nc_decode_step(ctypes.byref(c), ctypes.byref(fw.w), 1 << 41, 2, 5, 1 << 44, 1 << 43, n, 256, None) == 2
    assert L.nc_prefill(ctypes.byref(c), ctypes.byref(fw.w), 1 << 41, 2, 10, None, 1 << 43, n, 256,
                        1 << 42, 1 << 30, None) == 2
    # standalone entry points: argument checks before any device work
    q = lambda x, dt, n, codes, amax: L.nc_fp8_quantize(x, dt, n, codes, amax, None)
    assert q(None, nclib.F32, 16, 1 << 40, 1 << 41) == 1
    assert q(1 << 40, 7, 16, 1 << 40, 1 << 41) == 1      # bad source dtype
    assert q(1 << 40, nclib.F32, 24, 1 << 40, 1 << 41) == 3  # n % 16
    assert q((1 << 40) + 8, nclib.BF16, 16, 1 << 40, 1 << 41) == 4
    lin = lambda M, N, K, ldo, epi=0, dt=nclib.F16: L.nc_linear_fp8(1 << 40, 1 << 41, 1 << 42, 1 << 43, 1 << 44,
                                                                   M, N, K, ldo, epi, 15.0, dt, None, None)
    assert lin(128, 64, 8, 64) == 1      # K < 16
    assert lin(128, 64, 40, 64) == 3     # K % 16
    assert lin(128, 48, 64, 64) == 3     # N % 32
    assert lin(128, 64, 64, 32) == 3     # ldo < N
    assert lin(128, 64, 64, 64, epi=9) == 1
    assert lin(128, 64, 64, 64, dt=nclib.F32) == 1  # 16-bit outputs only
    import torch
    if not torch.cuda.is_available():
        assert lin(128, 64, 64, 64) == 8
        assert q(1 << 40, nclib.F32, 16, 1 << 40, 1 << 41) == 8


def test_backward_host_rules(nclib):
    """Sizing and host-side refusals of nc_forward_backward and the backward products."""
    L = nclib.lib()
    cfg = nclib.init_config(2, 64, 64, 0, 256, 512)
    n = nclib.train_workspace_bytes(cfg, 2, 100)
    M, C, V = 200, cfg.d_model, cfg.vocab
    # at least the saved residual streams (2L + 1 fp32 [M, C]) and the logit gradient [M, V] (16-bit)
    assert n >= (2 * cfg.n_layer + 1) * M * C * 4 + M * V * 2
    assert nclib.train_workspace_bytes(cfg, 2, 300) == 0  # T > seq_len
    c = nclib.NcConfig.from_buffer_copy(cfg)
    c.fp8 = nclib.FP8_BLOCK
    assert nclib.train_workspace_bytes(c, 2, 100) == 0  # e4m3 training is not supported
    # the further terms add x0, the pre-mix streams and the x0 gradient
    # (lambdas: n_layer + 2 fp32 [M, C]), the final-norm gradient (backout) and
    # the smear gates' per-token gradient
    for bits, extra in ((nclib.EXTRA_SMEAR, M * 4), (nclib.EXTRA_VALUE_EMBED, 0),
                        (nclib.EXTRA_RESID_LAMBDAS, (cfg.n_layer + 2) * M * C * 4),
                        (nclib.EXTRA_BACKOUT, M * C * 4)):
        c = nclib.NcConfig.from_buffer_copy(cfg)
        c.extras = bits
        got = nclib.train_workspace_bytes(c, 2, 100)
        assert extra <= got - n <= extra + 3 * 256, (bits, got - n, extra)
    fw = _FakeWeights(nclib, 2)
    arr = (ctypes.c_void_p * 2)(1 << 40, (1 << 40) + 4096)
    FPP = ctypes.POINTER(ctypes.c_void_p)
    g = nclib.NcGrads(1 << 41, *[ctypes.cast(arr, FPP)] * 6, 1 << 42)
    fb = lambda c, T=100, ws_bytes=n, loss=1 << 43, grads=g: L.nc_forward_backward(
        ctypes.byref(c), ctypes.byref(fw.w), 1 << 41, 1 << 41, 2, T, loss, ctypes.byref(grads), 1 << 44, ws_bytes,
        None)
    assert fb(cfg, T=300) == 3
    assert fb(cfg, ws_bytes=n - 1) == 5
    assert fb(cfg, loss=None) == 1
    c = nclib.NcConfig.from_buffer_copy(cfg)
    c.fp8 = nclib.FP8_BLOCK
    assert fb(c) == 2
    g_bad = nclib.NcGrads(1 << 41, *[ctypes.cast(arr, FPP)] * 6, (1 << 42) + 4)
    assert fb(cfg, grads=g_bad) == 4
    A = 1 << 40
    assert L.nc_linear_dgrad(A, A, A, 128, 60, 64, 3, 1, None, None) == 3     # N % 8
    assert L.nc_linear_dgrad(A, A, A, 128, 64, 64, 4, 1, None, None) == 1     # epilogue
    assert L.nc_linear_wgrad(A, A, A, 0, 64, 64, 1.0, 1, None, None) == 1     # M < 1
    assert L.nc_linear_wgrad(A + 2, A, A, 8, 64, 64, 1.0, 1, None, None) == 4
    import torch
    if not torch.cuda.is_available():
        assert fb(cfg) == 8
        assert L.nc_linear_dgrad(A, A, A, 128, 64, 64, 3, 1, None, None) == 8


def test_device_position_and_attention_backward_host_rules(nclib):
    """Host-side refusals of nc_decode_step_dev, nc_attention_lse and
    nc_attention_backward (before any device work)."""
    L = nclib.lib()
    cfg = nclib.init_config(2, 64, 64, 0, 4096, 512)
    fw = _FakeWeights(nclib, 2)
    n = L.nc_session_bytes(ctypes.byref(cfg), 2, 4096)
    dev = lambda pos_dev, T_max=4096, nbytes=n: L.nc_decode_step_dev(
        ctypes.byref(cfg), ctypes.byref(fw.w), 1 << 41, 2, pos_dev, 1 << 44, 1 << 43, nbytes, T_max, None)
    assert dev(None) == 1                       # no device position
    assert dev(1 << 42) == 3                    # the fixed attention grid covers T_max <= 2048
    assert dev((1 << 42) + 4, T_max=2048, nbytes=L.nc_session_bytes(ctypes.byref(cfg), 2, 2048)) == 4  # alignment
    c = nclib.NcConfig.from_buffer_copy(cfg)
    c.fp8 = nclib.FP8_BLOCK
    assert L.nc_decode_step_dev(ctypes.byref(c), ctypes.byref(fw.w), 1 << 41, 2, 1 << 42, 1 << 44, 1 << 43, n,
                                4096, None) == 2
    A = 1 << 40
    lse = lambda **kw: L.nc_attention_lse(kw.get("q", A), A, A, A, kw.get("lse", A), 1, 16, kw.get("H", 4),
                                          kw.get("Hkv", 2), kw.get("D", 128), 0, kw.get("qs", 512), 256, 1, None)
    assert lse(lse=None) == 1
    assert lse(H=3) == 1                         # H % Hkv
    assert lse(D=96) == 3
    assert lse(qs=100) == 1                      # row stride below H * D
    bwd = lambda **kw: L.nc_attention_backward(kw.get("qkv", A), A, A, A, kw.get("delta", A), A, 1, 16, 4, 2,
                                               kw.get("D", 128), 0, kw.get("dt", 1), None)
    assert bwd(delta=None) == 1
    assert bwd(D=80) == 3
    assert bwd(dt=5) == 1
    assert bwd(qkv=A + 8) == 4
    import torch
    if not torch.cuda.is_available():
        assert lse() == 8 and bwd() == 8
