"""Pins of the oracle's SwiGLU epilogue (gate/up pair of a gated FFN layer).

The pages give no formula for the gated FFN of their Fig. 12 FFN layers; the
oracle takes the common reading: silu(gate) * up, each projection through the
W4A8 epilogue in fp32, silu(g) = g / (1 + exp(-g)), one bf16 rounding.  The
pins: a float64 evaluation of the same closed form (independent arithmetic),
exact special cases, and the gate/up interleave (row 2n gate, 2n + 1 up)
through a float64 product of the dequantized weights.
"""
import numpy as np
import pytest

import oracle
from w4a8_bit_weight_b200 import synth


def _bf16_of_f64(v: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even bf16 bit patterns of float64 values (through their
    fp32 value: exact for the sizes here, ties are counted in the 1-ulp bound)."""
    f = np.asarray(v, np.float64).astype(np.float32)
    b = f.view(np.uint32).astype(np.uint64)
    rounded = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def _ulps(a, b):
    def ordv(x):
        x = np.asarray(x).astype(np.int64) & 0xFFFF
        return np.where(x & 0x8000, -(x & 0x7FFF), x)
    return np.abs(ordv(a) - ordv(b))


def _silu64(g):
    return g / (1.0 + np.exp(-g))


def test_swiglu_epilogue_against_float64_closed_form():
    rng = np.random.default_rng(5)
    M, N = 64, 96
    acc = rng.integers(-2_000_000, 2_000_000, size=(M, 2 * N)).astype(np.int32)
    s_x = (rng.random(M) * 1e-3 + 1e-5).astype(np.float32)
    s_c = (rng.random(2 * N) * 1e-3 + 1e-5).astype(np.float32)
    out = oracle.swiglu_epilogue(acc, s_x, s_c)
    yg = acc[:, 0::2].astype(np.float64) * s_x[:, None].astype(np.float64) * s_c[None, 0::2].astype(np.float64)
    yu = acc[:, 1::2].astype(np.float64) * s_x[:, None].astype(np.float64) * s_c[None, 1::2].astype(np.float64)
    ref = _bf16_of_f64(_silu64(yg) * yu)
    u = _ulps(out, ref)
    assert u.max() <= 1
    assert (u == 0).mean() > 0.97  # fp32 steps against float64: a last-bit difference is rare
    # the gate goes through silu, the up projection does not: swapping them is caught
    swapped = _bf16_of_f64(_silu64(yu) * yg)
    assert (_ulps(out, swapped) > 1).mean() > 0.5


def test_swiglu_epilogue_special_cases():
    s_x = np.array([0.25], np.float32)
    s_c = np.ones(8, np.float32)
    acc = np.array([[0, 12345,       # silu(0) = 0
                     400, 0,         # up = 0
                     200, -8,        # gate = 50: exp(-50) is below fp32's half ulp of 1, silu(g) = g
                     -1000, 9]], np.int32)  # gate = -250: exp(250) overflows fp32, silu(g) = -0
    out = oracle.swiglu_epilogue(acc, s_x, s_c)[0]
    assert int(out[0]) & 0x7FFF == 0 and int(out[1]) & 0x7FFF == 0
    assert int(out[2]) == int(_bf16_of_f64(np.array([50.0 * -2.0]))[0])
    assert int(out[3]) & 0x7FFF == 0


def test_swiglu_interleave_against_float64_product():
    """Row 2n of the stacked weights is gate channel n, row 2n + 1 up channel n."""
    M, N, K = 7, 48, 256
    X, W = synth.make_problem(M, 2 * N, K, seed=33, n_outliers=2)
    qw, s_u8, a_u8, s_c, _ = oracle.quantize_weights(synth.bf16_bits(W))
    x_q, s_x = oracle.quantize_act(synth.bf16_bits(X))
    out, acc = oracle.w4a8_swiglu(x_q, s_x, qw, s_u8, a_u8, s_c)
    w_hat = oracle.dequant(qw, s_u8, a_u8).astype(np.float64)
    full = x_q.astype(np.float64) @ w_hat.T                     # exact integer sums
    np.testing.assert_array_equal(acc.astype(np.float64), full)
    yg = full[:, 0::2] * s_x[:, None].astype(np.float64) * s_c[None, 0::2].astype(np.float64)
    yu = full[:, 1::2] * s_x[:, None].astype(np.float64) * s_c[None, 1::2].astype(np.float64)
    assert _ulps(out, _bf16_of_f64(_silu64(yg) * yu)).max() <= 1
    # and the quantized layer approximates the float layer it came from (4-bit
    # weights: the GEMM pins use 0.25 of the spread for one projection; the
    # product of two such projections gets a looser bound)
    Xf = synth.bf16_bits(X).astype(np.uint32) << 16
    Wf = synth.bf16_bits(W).astype(np.uint32) << 16
    xf, wf = Xf.view(np.float32).astype(np.float64), Wf.view(np.float32).astype(np.float64)
    gf, uf = xf @ wf[0::2].T, xf @ wf[1::2].T
    ref = _silu64(gf) * uf
    got = (out.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert np.sqrt(np.mean((got - ref) ** 2)) < 0.3 * np.std(ref)


def test_swiglu_sampled_equals_full():
    M, N, K = 5, 40, 128
    X, W = synth.make_problem(M, 2 * N, K, seed=8, n_outliers=1)
    qw, s_u8, a_u8, s_c, _ = oracle.quantize_weights(synth.bf16_bits(W))
    x_q, s_x = oracle.quantize_act(synth.bf16_bits(X))
    out, acc = oracle.w4a8_swiglu(x_q, s_x, qw, s_u8, a_u8, s_c)
    mi, ni = np.meshgrid(np.arange(M), np.arange(N), indexing="ij")
    so, sa = oracle.w4a8_swiglu_sampled(x_q, s_x, qw, s_u8, a_u8, s_c, mi.ravel(), ni.ravel())
    np.testing.assert_array_equal(so, out.ravel())
    np.testing.assert_array_equal(sa, acc.reshape(M, N, 2).reshape(-1, 2))
