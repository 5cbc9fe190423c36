"""Dynamic tensorwise FP8 (e4m3) matrix products of the nanochat forward.

TEST INFRASTRUCTURE ONLY (see the package docstring for who may import it).

"Nanochat与nanoGPT对比：关键升级" §1, architecture table, FP8-training row:
nanochat trains with dynamic, tensor-level FP8 in the e4m3 / e5m2 formats.  The
row is all the pages say; the readings taken here (each one function below):

* e4m3 is the format of both operands of a forward matrix product (e5m2 is the
  format of gradients, which a forward does not form).
* e4m3 (OCP "E4M3FN"): 1 sign, 4 exponent bits with bias 7, 3 mantissa bits,
  subnormals, no infinities; the largest finite value is 1.75 * 2^8 = 448.
  Conversion rounds to the nearest value, ties to even, and saturates at +-448.
* "dynamic, tensor-level": one scale per tensor, from the tensor's current
  values: amax = max |x| over the whole tensor, s = 448 / max(amax, 1e-12)
  (the clamp keeps an all-zero tensor finite), codes q = e4m3(x * s).
* The quantised code is an integer decided by floating point, so the scale and
  the scaled value are formed in fp32, as a kernel forms them:
  x32 = fp32(x), s = fp32(448) / fp32(amax) rounded to fp32, y = fp32(x32 * s).
* the product of two quantised tensors is (q_a q_b^T) / (s_a s_b), formed here
  exactly (fp64 holds every partial sum of e4m3 products exactly for the inner
  sizes used).
* which products: the six block projections (c_q, c_k, c_v, attention c_proj,
  c_fc, MLP c_proj) take the activation entering them and their fp32 master
  weight through this path; the LM head optionally too.  The small gate maps
  (smear, value-embedding gates) stay as they are.

The pins are in ``tests/test_oracle_fp8.py``.
"""
from __future__ import annotations

import numpy as np

F64 = np.float64
E4M3_MAX = 448.0
AMAX_FLOOR = np.float32(1e-12)


def round_e4m3(y: np.ndarray) -> np.ndarray:
    """Nearest e4m3 value of each element of ``y`` (ties to even), saturated to
    +-448; NaN stays NaN.  Input and output are float64 (every e4m3 value is
    exact in float64).

    In the binade [2^e, 2^(e+1)) the three mantissa bits give a spacing of
    2^(e-3); below the smallest normal 2^-6 the subnormals keep the spacing
    2^-9 of that binade.  Rounding to that spacing with round-half-even on the
    integer count is rounding to even on the last mantissa bit.
    """
    y = np.asarray(y, dtype=F64)
    a = np.abs(y)
    _, ex = np.frexp(np.where(a > 0, a, 1.0))  # a = m * 2^ex, m in [0.5, 1)
    e = np.maximum(ex - 1, -6)
    quantum = np.ldexp(1.0, e - 3)
    r = np.rint(a / quantum) * quantum
    r = np.minimum(r, E4M3_MAX)
    out = np.copysign(r, y)
    return np.where(np.isnan(y), np.nan, out)


def tensor_scale(x32: np.ndarray) -> np.float32:
    """Scale of a tensor (fp32 values): 448 / max(amax, 1e-12), in fp32."""
    amax = np.float32(np.max(np.abs(x32))) if x32.size else np.float32(0.0)
    return np.float32(np.float32(E4M3_MAX) / np.maximum(amax, AMAX_FLOOR))


def quantize_e4m3(x: np.ndarray):
    """Dynamic tensorwise quantisation of the whole of ``x``.

    Returns (codes as float64 values, scale as float32) with
    codes = e4m3(fp32(fp32(x) * s)).
    """
    x32 = np.asarray(x, dtype=np.float32)
    s = tensor_scale(x32)
    y = (x32 * s).astype(np.float32)
    return round_e4m3(y.astype(F64)), s


def linear_e4m3(x: np.ndarray, w: np.ndarray) -> np.ndarray:
    """y = x W^T with both operands quantised tensorwise to e4m3 and the
    product rescaled by 1 / (s_x s_w).  x: [..., K] (quantised as one tensor),
    w: [N, K] fp32 master weight."""
    qx, sx = quantize_e4m3(x)
    qw, sw = quantize_e4m3(w)
    return (qx @ qw.T) / (F64(sx) * F64(sw))
