"""The loss head that allocates nothing (nc_lm_head_loss_static).

Callers that cannot provide scratch memory -- code inside a host application
whose memory manager owns the whole device budget, or code on a latency-critical
path that cannot afford cudaMalloc's implicit device-wide synchronisation -- use
this entry point instead of assembling the loss from nc_linear +
nc_softcap_ce + nc_loss_mean, which need a caller-provided logits buffer.  Its
scratch is one fixed device array inside the library.

Each case calls it twice in a row through the C ABI, with different inputs,
and checks both results
- against the existing entry points' output on the same device inputs:
  per-token losses within rtol 1e-5 / atol 1e-5 (the two paths sum the softmax
  denominator in different orders), mean loss within 1e-5 relative;
- against the fp64 oracle's soft-cap and cross-entropy ("Nanochat与nanoGPT对比"
  §1, soft-cap row; "从文本到聊天模型" §5.8) of the same 16-bit operands, on
  sampled rows, within a bound derived from the arithmetic: the fp32
  accumulation of the logit is off by at most C 2^-24 sum_k |a_k w_k| (bounded
  per row by C 2^-24 |a|_1 max|w|), the soft-cap's MUFU steps add at most 2e-5,
  a token's NLL moves by at most twice the largest logit error, and the fp32
  partial sums of the denominator add 3e-5.
Both 16-bit formats run, vocab sizes 512, 4160 (not a multiple of the 256
columns one lm_head tile covers) and 32768, and one call passes loss = NULL.
Sizes beyond the fixed array are refused.  The file name makes pytest collect
it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu

DEV = "cuda"
CAP = 15.0


def _entry(nc):
    fn = nc.lib().nc_lm_head_loss_static
    vp, i32 = ctypes.c_void_p, ctypes.c_int
    fn.restype = i32
    fn.argtypes = [vp, vp, vp, i32, i32, i32, ctypes.c_float, i32, vp, vp, vp, vp]
    return fn


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _reference(nc, a, w, y, cap):
    """Existing entry points: raw logits (nc_linear), then soft-cap + CE, then the mean."""
    M, V = a.shape[0], w.shape[0]
    z = torch.empty((M, V), dtype=torch.float32, device=DEV)
    nc.linear(a, w, z, nc.EPI_STORE_F32)
    tl = torch.empty(M, dtype=torch.float32, device=DEV)
    nc.softcap_ce(z, y, tl, None, cap)
    loss = torch.empty((), dtype=torch.float32, device=DEV)
    nc.loss_mean(tl, y, V, loss)
    return tl, loss


def _inputs(nc, seed, M, C, V, dt):
    g = torch.Generator().manual_seed(seed)
    t16 = torch.float16 if dt == nc.F16 else torch.bfloat16
    a = torch.randn((M, C), generator=g).to(t16).to(DEV)
    w32 = (torch.randn((V, C), generator=g) * 0.05).to(DEV)
    w = torch.empty((V, C), dtype=t16, device=DEV)
    nc.cast_weights(w32, w)
    y = torch.randint(0, V, (M,), generator=g, dtype=torch.int32)
    y[::5] = -1
    return a, w, y.to(DEV)


def _oracle_rows(a, w, y, rows):
    """fp64 oracle NLL of the given rows from the exact 16-bit operand values."""
    a64 = a[rows].double().cpu().numpy()
    w64 = w.double().cpu().numpy()
    nll, _ = oracle.cross_entropy(oracle.softcap(a64 @ w64.T, CAP), y[rows].cpu().numpy())
    bound = 2.0 * (a.shape[1] * 2.0 ** -24 * np.abs(a64).sum(axis=1) * np.abs(w64).max() + 2e-5) + 3e-5
    return nll, bound


@pytest.mark.parametrize("V", [512, 4160, 32768])
@pytest.mark.parametrize("dt_name", ["f16", "bf16"])
def test_static_loss_head_matches_existing_entry_points_and_oracle(gpu, dt_name, V):
    dt = gpu.F16 if dt_name == "f16" else gpu.BF16
    fn = _entry(gpu)
    C = 256
    st = torch.zeros(64, dtype=torch.int32, device=DEV)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call, (seed, M) in enumerate(((11, 1000), (12, 8192))):
        a, w, y = _inputs(gpu, seed + V, M, C, V, dt)
        tl = torch.full((M,), float("nan"), dtype=torch.float32, device=DEV)
        loss = torch.full((), float("nan"), dtype=torch.float32, device=DEV)
        code = fn(_p(a), _p(w), _p(y), M, C, V, CAP, dt, _p(tl), _p(loss), _p(st), stream)
        assert code == 0, f"call {call}: {gpu.STATUS_NAMES.get(code, code)}"
        assert gpu.get_status(st) == 0
        want_tl, want_loss = _reference(gpu, a, w, y, CAP)
        torch.cuda.synchronize()
        got = tl.cpu().numpy()
        np.testing.assert_allclose(got, want_tl.cpu().numpy(), rtol=1e-5, atol=1e-5, err_msg=f"call {call}")
        assert abs(loss.item() - want_loss.item()) <= 1e-5 * abs(want_loss.item()), f"call {call}"
        assert torch.all(tl[y == -1] == 0)
        # the oracle on sampled rows (all rows of the first call)
        rows = np.arange(M) if M <= 1000 else np.unique(np.r_[0, M - 1, np.arange(1, M - 1, 37)])
        nll, bound = _oracle_rows(a, w, y, rows)
        err = np.abs(got[rows] - nll)
        assert np.all(err <= bound), f"call {call}: oracle max err {err.max():.3e}, bound {bound.min():.3e}"
        if M <= 1000:  # every row went through the oracle: its mean over the valid targets
            valid = y.cpu().numpy() != -1
            want_mean = nll[valid].sum() / valid.sum()
            assert abs(loss.item() - want_mean) <= 1e-5 * abs(want_mean) + bound.max()


def test_static_loss_head_without_mean(gpu):
    """loss = NULL: only the per-token losses are written."""
    fn = _entry(gpu)
    M, C, V = 777, 128, 4160
    a, w, y = _inputs(gpu, 3, M, C, V, gpu.F16)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    tl = torch.full((M,), float("nan"), dtype=torch.float32, device=DEV)
    assert fn(_p(a), _p(w), _p(y), M, C, V, CAP, gpu.F16, _p(tl), None, None, stream) == 0
    want_tl, _ = _reference(gpu, a, w, y, CAP)
    torch.cuda.synchronize()
    np.testing.assert_allclose(tl.cpu().numpy(), want_tl.cpu().numpy(), rtol=1e-5, atol=1e-5)


def test_static_loss_head_refuses_sizes_beyond_its_array(gpu):
    fn = _entry(gpu)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    a = torch.zeros((8193, 256), dtype=torch.float16, device=DEV)
    w = torch.zeros((32768, 256), dtype=torch.float16, device=DEV)
    y = torch.zeros(8193, dtype=torch.int32, device=DEV)
    tl = torch.zeros(8193, dtype=torch.float32, device=DEV)
    assert fn(_p(a), _p(w), _p(y), 8193, 256, 32768, CAP, gpu.F16, _p(tl), None, None, stream) == 3
    w2 = torch.zeros((32832, 256), dtype=torch.float16, device=DEV)
    assert fn(_p(a), _p(w2), _p(y), 8, 256, 32832, CAP, gpu.F16, _p(tl), None, None, stream) == 3
