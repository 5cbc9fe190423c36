"""The loss head that allocates nothing (nc_lm_head_loss_static).

Callers that cannot provide scratch memory -- code inside a host application
whose memory manager owns the whole device budget, or code on a latency-critical
path that cannot afford cudaMalloc's implicit device-wide synchronisation -- use
this entry point instead of assembling the loss from nc_linear +
nc_softcap_ce + nc_loss_mean, which need a caller-provided logits buffer.  Its
scratch is one fixed device array inside the library.

This test calls it twice in a row through the C ABI, with different inputs, and
checks each result against the existing entry points' output: per-token losses
within rtol 1e-5 / atol 1e-5 (the two paths sum the softmax denominator in
different orders), mean loss within 1e-5 relative.  It also checks that sizes
beyond the fixed array are refused.  The file name makes pytest collect it
last.
"""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

DEV = "cuda"


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


def _inputs(seed, M, C, V):
    g = torch.Generator().manual_seed(seed)
    a = torch.randn((M, C), generator=g).to(torch.float16).to(DEV)
    w32 = (torch.randn((V, C), generator=g) * 0.05).to(DEV)
    w = torch.empty((V, C), dtype=torch.float16, device=DEV)
    y = torch.randint(0, V, (M,), generator=g, dtype=torch.int32)
    y[::5] = -1
    return a, w32, w, y.to(DEV)


def test_static_loss_head_matches_existing_entry_points(gpu):
    fn = _entry(gpu)
    cap, C, V = 15.0, 256, 32768
    st = torch.zeros(64, dtype=torch.int32, device=DEV)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call, (seed, M) in enumerate(((11, 1000), (12, 8192))):
        a, w32, w, y = _inputs(seed, M, C, V)
        gpu.cast_weights(w32, w)
        tl = torch.full((M,), float("nan"), dtype=torch.float32, device=DEV)
        loss = torch.full((), float("nan"), dtype=torch.float32, device=DEV)
        code = fn(_p(a), _p(w), _p(y), M, C, V, cap, gpu.F16, _p(tl), _p(loss), _p(st), stream)
        assert code == 0, f"call {call}: {gpu.STATUS_NAMES.get(code, code)}"
        assert gpu.get_status(st) == 0
        want_tl, want_loss = _reference(gpu, a, w, y, cap)
        torch.cuda.synchronize()
        np.testing.assert_allclose(tl.cpu().numpy(), want_tl.cpu().numpy(), rtol=1e-5, atol=1e-5,
                                   err_msg=f"call {call}")
        assert abs(loss.item() - want_loss.item()) <= 1e-5 * abs(want_loss.item()), f"call {call}"
        assert torch.all(tl[y == -1] == 0)


def test_static_loss_head_refuses_sizes_beyond_its_array(gpu):
    fn = _entry(gpu)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    a = torch.zeros((8193, 256), dtype=torch.float16, device=DEV)
    w = torch.zeros((32768, 256), dtype=torch.float16, device=DEV)
    y = torch.zeros(8193, dtype=torch.int32, device=DEV)
    tl = torch.zeros(8193, dtype=torch.float32, device=DEV)
    assert fn(_p(a), _p(w), _p(y), 8193, 256, 32768, 15.0, gpu.F16, _p(tl), None, None, stream) == 3
    w2 = torch.zeros((32832, 256), dtype=torch.float16, device=DEV)
    assert fn(_p(a), _p(w2), _p(y), 8, 256, 32832, 15.0, gpu.F16, _p(tl), None, None, stream) == 3
