"""Zero-copy I/O (needs a B200): activations read from and outputs written to
pinned host memory directly by the kernels (include/lq.h, conventions).

Every case compares with the oracle, from the same bf16 inputs.  Pageable host
memory is refused before any launch: the tests first check, without launching
anything, that the library classifies such memory as not addressable, and only
then make the call that must be refused.
"""
import ctypes

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


def _ulps(a, b):
    def ordv(x):
        x = x.astype(np.int64)
        return np.where(x & 0x8000, -(x & 0x7FFF), x)
    return np.abs(ordv(a) - ordv(b))


def test_device_addressable_classification():
    torch.cuda.set_device(0)
    assert lq.lq_device_addressable(torch.empty(64, dtype=torch.uint8, device=DEV))
    assert lq.lq_device_addressable(torch.empty(64, dtype=torch.uint8).pin_memory())
    assert not lq.lq_device_addressable(torch.empty(64, dtype=torch.uint8))  # pageable


@pytest.mark.parametrize("M,N,K", [(16, 256, 512), (5, 4096, 4096), (40, 384, 1024)])
def test_quantize_and_gemm_through_pinned_host_memory(M, N, K):
    torch.cuda.set_device(0)
    X, W = synth.make_problem(M, N, K, seed=300 + M, n_outliers=3)
    qw, s, a, sc = lq.lq_quantize_weights(W.to(DEV))
    X_host = X.contiguous().pin_memory()
    xq, sx = lq.lq_quantize_act(X_host)  # read over the host link
    out_host = torch.full((M, N), float("nan"), dtype=torch.bfloat16).pin_memory()
    lq.lq_w4a8_gemm(xq, sx, qw, s, a, sc, out=out_host)  # written over the host link
    torch.cuda.synchronize()
    assert lq.lq_get_device_error() == 0
    o_qw, o_s, o_a, o_sc, _ = oracle.quantize_weights(synth.bf16_bits(W))
    o_xq, o_sx = oracle.quantize_act(synth.bf16_bits(X))
    np.testing.assert_array_equal(xq.cpu().numpy(), o_xq)
    np.testing.assert_array_equal(sx.cpu().numpy().view(np.uint32), o_sx.view(np.uint32))
    o_out, _ = oracle.w4a8_gemm(o_xq, o_sx, o_qw, o_s, o_a, o_sc)
    assert int(_ulps(_u16(out_host), o_out).max()) <= 1


@pytest.mark.parametrize("M", [1, 16])
def test_linear_pinned_in_and_out(M):
    torch.cuda.set_device(0)
    N, K = 4096, 4096
    X, W = synth.make_problem(M, N, K, seed=310 + M, n_outliers=3)
    qw, s, a, sc = lq.lq_quantize_weights(W.to(DEV))
    X_host = X.contiguous().pin_memory()
    o_qw, o_s, o_a, o_sc, _ = oracle.quantize_weights(synth.bf16_bits(W))
    o_xq, o_sx = oracle.quantize_act(synth.bf16_bits(X))
    o_out, _ = oracle.w4a8_gemm(o_xq, o_sx, o_qw, o_s, o_a, o_sc)
    for path in (lq.LINEAR_FUSED, lq.LINEAR_TWO_LAUNCHES):
        out_host = torch.full((M, N), float("nan"), dtype=torch.bfloat16).pin_memory()
        lq.lq_w4a8_linear(X_host, qw, s, a, sc, out=out_host, path=path)
        torch.cuda.synchronize()
        assert lq.lq_get_device_error() == 0
        assert int(_ulps(_u16(out_host), o_out).max()) <= 1


def test_w4f8_out_pinned_exact_sums():
    """W4 x FP8 written to pinned host memory; +-1 activations make the sums exact."""
    torch.cuda.set_device(0)
    M, N, K = 16, 256, 1024
    rng = np.random.default_rng(17)
    u = rng.integers(1, 16, size=(N, K), dtype=np.uint8)
    g = u.reshape(N, K // 8, 2, 4)
    qw4 = (g[:, :, 0, :] | (g[:, :, 1, :] << 4)).reshape(N, K // 2).astype(np.uint8)
    xs = rng.choice(np.array([0x38, 0xB8], dtype=np.uint8), size=(M, K))  # +1, -1 in e4m3
    s_w = rng.uniform(0.5, 2.0, size=N).astype(np.float32)
    s_x = np.array([0.5], dtype=np.float32)
    out_host = torch.full((M, N), float("nan"), dtype=torch.bfloat16).pin_memory()
    lq.lq_w4f8_gemm(torch.from_numpy(xs).to(DEV), torch.from_numpy(s_x).to(DEV), torch.from_numpy(qw4).to(DEV),
                    torch.from_numpy(s_w).to(DEV), out=out_host)
    torch.cuda.synchronize()
    assert lq.lq_get_device_error() == 0
    acc = np.where(xs == 0x38, 1.0, -1.0) @ (u.astype(np.float64) - 8).T
    ref = torch.from_numpy((acc * (np.float32(s_x[0]) * s_w).astype(np.float64)[None, :]).astype(np.float32))
    np.testing.assert_array_equal(_u16(out_host).view(np.int16), ref.to(torch.bfloat16).view(torch.int16).numpy())


def test_pageable_host_memory_refused_before_launch():
    torch.cuda.set_device(0)
    M, N, K = 16, 256, 512
    X, W = synth.make_problem(M, N, K, seed=320)
    qw, s, a, sc = lq.lq_quantize_weights(W.to(DEV))
    xq, sx = lq.lq_quantize_act(X.to(DEV))
    pageable_x = np.zeros((M, K), dtype=np.uint16)
    pageable_out = np.zeros((M, N), dtype=np.uint16)
    lib = lq.load_library()
    px = ctypes.c_void_p(pageable_x.ctypes.data)
    po = ctypes.c_void_p(pageable_out.ctypes.data)
    assert pageable_x.ctypes.data % 16 == 0 and pageable_out.ctypes.data % 16 == 0
    # the classification first (launches nothing); the calls below rely on it
    assert lib.lq_device_addressable(px) == 0 and lib.lq_device_addressable(po) == 0
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    xq2 = torch.empty_like(xq)
    sx2 = torch.empty_like(sx)
    assert lib.lq_quantize_act(px, M, K, ctypes.c_void_p(xq2.data_ptr()), ctypes.c_void_p(sx2.data_ptr()),
                               stream) == 1  # LQ_ERR_INVALID_ARG
    ws = torch.zeros(16, dtype=torch.uint8, device=DEV)
    P = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    assert lib.lq_w4a8_gemm(P(xq), P(sx), P(qw), P(s), P(a), P(sc), po, M, N, K, 64, P(ws), 16, stream) == 1
    torch.cuda.synchronize()
    assert lq.lq_get_device_error() == 0
    assert not pageable_out.any()
    # the binding refuses a host tensor that is not pinned
    with pytest.raises(ValueError):
        lq.lq_quantize_act(X)
