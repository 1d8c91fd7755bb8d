"""The W4 x FP8 variant against the oracle (needs a B200).

Quantizers: bit-exact (the same IEEE operations, round to nearest even and
saturation for e4m3).  GEMM: every product of an e4m3 activation and an INT4
weight is exact, but the tensor core sums them in fp32 in its own order, so
the output is compared with the oracle's exact sum within a bound derived
from that: |y - acc * s| <= 2^-8 |acc * s| (bf16 rounding) plus
K * 2^-22 * sum_k |x_k q_k| * s (fp32 accumulation, a rounding error of at
most 2^-23 of the partial sum's magnitude per addition, doubled).
"""
import numpy as np
import pytest
import torch

import oracle
import w4a8_bit_weight_b200 as lq
from w4a8_bit_weight_b200 import synth

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _u16(t):
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


# the schedule forms: 16-token tiles with 1, 2, 4 and 8 CTAs per cluster (two
# expansion groups, two MMA issuers, the overflow block at M = 1..16,
# N = K = 4096), 64- and 128-token tiles, ragged N, K and M tails
@pytest.mark.parametrize("M,N,K", [(16, 256, 512), (5, 384, 1024), (130, 256, 768), (16, 4096, 4096),
                                   (1, 4096, 4096), (200, 4096, 1024), (16, 1024, 4096), (40, 1024, 2048),
                                   (3, 400, 640), (300, 512, 1024), (64, 2048, 128)])
def test_w4f8_matches_oracle(M, N, K):
    torch.cuda.set_device(0)
    X, W = synth.make_problem(M, N, K, seed=M + N + K + 5, n_outliers=3)
    qw4, s_w = lq.lq_quantize_weights_w4(W.to(DEV))
    x_f8, s_x = lq.lq_quantize_act_f8(X.to(DEV))
    out = lq.lq_w4f8_gemm(x_f8, s_x, qw4, s_w)
    torch.cuda.synchronize()
    assert lq.lq_get_device_error() == 0
    o_qw4, o_sw = oracle.quantize_weights_w4(synth.bf16_bits(W))
    o_xf8, o_sx = oracle.quantize_act_f8(synth.bf16_bits(X))
    np.testing.assert_array_equal(qw4.cpu().numpy(), o_qw4)
    np.testing.assert_array_equal(s_w.cpu().numpy().view(np.uint32), o_sw.view(np.uint32))
    np.testing.assert_array_equal(x_f8.cpu().numpy(), o_xf8)
    assert float(s_x.cpu()[0]) == float(o_sx)
    o_out, o_acc = oracle.w4f8_gemm(o_xf8, o_sx, o_qw4, o_sw)
    scale = (np.float32(o_sx) * o_sw).astype(np.float64)[None, :]          # s_x * s_w[n] in fp32
    ref = o_acc * scale
    xd = torch.from_numpy(o_xf8.copy()).view(torch.float8_e4m3fn).double().numpy()
    u = np.stack([(o_qw4 >> (4 * h)) & 15 for h in (0, 1)], -1)
    q = (u.reshape(N, -1, 4, 2).transpose(0, 1, 3, 2).reshape(N, -1)).astype(np.float64) - 8
    absum = np.abs(xd) @ np.abs(q).T
    tol = np.abs(ref) * 2.0 ** -8 + scale * absum * (K * 2.0 ** -22) + 1e-30
    y = torch.from_numpy(_u16(out).view(np.int16)).view(torch.bfloat16).double().numpy()
    assert np.all(np.abs(y - ref) <= tol), float(np.max(np.abs(y - ref) / tol))
    # in practice the fp32 sums round to the same bf16 as the exact sums almost everywhere
    assert np.mean(_u16(out) == o_out) > 0.95


def test_w4f8_zero_activations():
    torch.cuda.set_device(0)
    _, W = synth.make_problem(1, 128, 256, seed=3)
    qw4, s_w = lq.lq_quantize_weights_w4(W.to(DEV))
    x_f8, s_x = lq.lq_quantize_act_f8(torch.zeros(4, 256, dtype=torch.bfloat16, device=DEV))
    out = lq.lq_w4f8_gemm(x_f8, s_x, qw4, s_w)
    torch.cuda.synchronize()
    assert float(s_x.cpu()[0]) == 1.0 and not x_f8.any() and not (out != 0).any()


def test_w4f8_repeatable():
    """Split-K partial sums are added in a fixed order: two calls give the same bits."""
    torch.cuda.set_device(0)
    X, W = synth.make_problem(16, 4096, 4096, seed=11, n_outliers=3)
    qw4, s_w = lq.lq_quantize_weights_w4(W.to(DEV))
    x_f8, s_x = lq.lq_quantize_act_f8(X.to(DEV))
    a = lq.lq_w4f8_gemm(x_f8, s_x, qw4, s_w)
    b = lq.lq_w4f8_gemm(x_f8, s_x, qw4, s_w)
    torch.cuda.synchronize()
    assert lq.lq_get_device_error() == 0
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_w4f8_all_codes():
    """Every INT4 code, -8 included, against exact sums: weights whose codes cycle
    through 0..15 (u = q + 8) and activations of +-1 in e4m3, so that acc is an
    exactly representable integer and the output is bf16(acc * s_x * s_w[n])."""
    torch.cuda.set_device(0)
    M, N, K = 16, 256, 1024
    rng = np.random.default_rng(7)
    u = rng.integers(0, 16, size=(N, K), dtype=np.uint8)
    # the LiquidQuant nibble layout: byte b of word j = u[8j + b] | u[8j + 4 + b] << 4
    g = u.reshape(N, K // 8, 2, 4)
    qw4 = (g[:, :, 0, :] | (g[:, :, 1, :] << 4)).reshape(N, K // 2).astype(np.uint8)
    xs = rng.choice(np.array([0x38, 0xB8, 0x00], dtype=np.uint8), size=(M, K))  # +1, -1, 0 in e4m3
    s_w = rng.uniform(0.5, 2.0, size=N).astype(np.float32)
    s_x = np.array([0.25], dtype=np.float32)
    out = lq.lq_w4f8_gemm(torch.from_numpy(xs).to(DEV), torch.from_numpy(s_x).to(DEV),
                          torch.from_numpy(qw4).to(DEV), torch.from_numpy(s_w).to(DEV))
    torch.cuda.synchronize()
    assert lq.lq_get_device_error() == 0
    xv = np.where(xs == 0x38, 1.0, np.where(xs == 0xB8, -1.0, 0.0))
    acc = xv @ (u.astype(np.float64) - 8).T
    ref = torch.from_numpy((acc * (np.float32(s_x[0]) * s_w).astype(np.float64)[None, :]).astype(np.float32))
    want = ref.to(torch.bfloat16).view(torch.int16).numpy()
    np.testing.assert_array_equal(_u16(out).view(np.int16), want)
