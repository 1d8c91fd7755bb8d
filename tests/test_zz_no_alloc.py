"""The allocation-free GEMM entry point (needs a B200).

lq_w4a8_gemm_noalloc exists for callers that must not allocate device memory
where they launch the GEMM (a serving framework's enqueue hook that owns all
device memory, a latency-critical loop that cannot block on the allocator).
It keeps its partial sums in a fixed scratch array inside the library instead
of a workspace.  These tests call it through the C ABI and check, on two calls
in a row, that it gives what lq_w4a8_gemm gives and what the CPU oracle's own
chain gives from the same bf16 inputs (bf16 within 1 ulp, the tolerance of the
other parity tests).  The file runs last so that a run that
stops at the first failure has already run every other test; it also passes
on its own in a fresh process.
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
LQ_ERR_WORKSPACE = 4


def _bits(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        return t.contiguous().view(torch.int16).cpu().numpy().astype(np.int64) & 0xFFFF
    return np.asarray(t).astype(np.int64) & 0xFFFF


def _ulps(a, b) -> int:
    """Largest |ord(a) - ord(b)| over bf16 bit patterns (a monotone order, +0 == -0)."""
    def ordv(x):
        x = _bits(x)
        return np.where(x & 0x8000, -(x & 0x7FFF), x)
    return int(np.abs(ordv(a) - ordv(b)).max()) if np.size(_bits(a)) else 0


def _call_noalloc(lib, xq, sx, qw, s, a, sc, out):
    M, K = xq.shape
    N = qw.shape[0]
    P = ctypes.c_void_p
    return lib.lq_w4a8_gemm_noalloc(P(xq.data_ptr()), P(sx.data_ptr()), P(qw.data_ptr()), P(s.data_ptr()),
                                    P(a.data_ptr()), P(sc.data_ptr()), P(out.data_ptr()), M, N, K, 64,
                                    P(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("M,N,K", [(16, 4096, 4096), (5, 272, 384), (64, 1024, 2048)])
def test_noalloc_matches_workspace_entry(M, N, K):
    lib = lq.load_library()
    torch.cuda.set_device(0)
    X, W = synth.make_problem(M, N, K, seed=17 + M, n_outliers=3)
    qw, s, a, sc = lq.lq_quantize_weights(W.to(DEV))
    xq, sx = lq.lq_quantize_act(X.to(DEV))
    ref = lq.lq_w4a8_gemm(xq, sx, qw, s, a, sc)
    # the oracle's own chain from the same bf16 inputs
    o_qw, o_s, o_a, o_sc, _ = oracle.quantize_weights(synth.bf16_bits(W))
    o_xq, o_sx = oracle.quantize_act(synth.bf16_bits(X))
    o_out, _ = oracle.w4a8_gemm(o_xq, o_sx, o_qw, o_s, o_a, o_sc)
    for _ in range(2):  # the shared scratch must give the same answer on repeated calls
        out = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
        assert _call_noalloc(lib, xq, sx, qw, s, a, sc, out) == 0
        torch.cuda.synchronize()
        assert lq.lq_get_device_error() == 0
        assert _ulps(out, o_out) <= 1
        assert _ulps(out, ref) <= 1


@pytest.mark.parametrize("M,N,K", [
    (256, 8192, 1024),   # stream-K partial sums would need 8 MiB, the array holds 4 MiB
    (16, 65536, 4096),   # 512 tiles: exactly 4 MiB of partial sums, plus the tile tickets
])
def test_noalloc_rejects_shapes_beyond_its_scratch(M, N, K):
    lib = lq.load_library()
    torch.cuda.set_device(0)
    xq = torch.zeros(M, K, dtype=torch.int8, device=DEV)
    sx = torch.ones(M, dtype=torch.float32, device=DEV)
    qw = torch.zeros(N, K // 2, dtype=torch.uint8, device=DEV)
    s = torch.ones(K // 64, N, dtype=torch.uint8, device=DEV)
    a = torch.full((K // 64, N), 128, dtype=torch.uint8, device=DEV)
    sc = torch.ones(N, dtype=torch.float32, device=DEV)
    out = torch.zeros(M, N, dtype=torch.bfloat16, device=DEV)
    assert _call_noalloc(lib, xq, sx, qw, s, a, sc, out) == LQ_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert not out.any()  # nothing was launched
