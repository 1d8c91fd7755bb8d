"""The fused SwiGLU epilogue of a gate/up pair (needs a B200).

lq_w4a8_gemm_swiglu multiplies the activations by one interleaved [2F, K]
weight matrix (row 2j gate channel j, row 2j+1 up channel j) and writes
bf16(silu(y_gate) * y_up) [M, F].  Against the oracle's chain from the same
bf16 inputs: within 1 bf16 ulp (CUDA's expf is within 2 fp32 ulp, the oracle's
libm expf correctly rounded or nearly; after one fp32 multiply the values
differ in the last fp32 bits at most, which moves a bf16 rounding by at most
one step), and the gate/up int32 accumulators bit-exact through lq_w4a8_gemm_i32.
Every schedule that has the epilogue: one CTA per tile, split-K clusters
(token slices sent from registers, and staged for wide tiles), CTA pairs.
"""
import numpy as np
import pytest
import torch

import oracle
import w4a8_bit_weight_b200 as lq
from w4a8_bit_weight_b200 import synth

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
T, PR = lq.SCHED_TILES, lq.SCHED_PAIR


def _u16(t):
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _ulps(a, b):
    def ordv(x):
        x = x.astype(np.int64)
        return np.where(x & 0x8000, -(x & 0x7FFF), x)
    return np.abs(ordv(a) - ordv(b))


CASES = [
    # M, 2F, K, block_t, schedule, split_k
    (16, 512, 512, 0, None, 0),      # automatic
    (1, 4096, 4096, 0, None, 0),     # decode: 16-token tiles in 4-CTA clusters, two expansion groups
    (5, 4096, 4096, 0, None, 0),
    (16, 2048, 4096, 0, None, 0),    # 8-CTA clusters: two tokens per slice
    (3, 272, 384, 16, T, 1),         # one CTA per tile, a partial last tile
    (40, 384, 1024, 64, T, 4),       # 64-token tiles, slices sent from registers
    (100, 256, 1152, 128, T, 4),     # 128-token tiles: slices staged and bulk-copied
    (300, 512, 1024, 0, PR, 0),      # CTA pairs, ragged M
    (512, 1024, 2048, 0, PR, 0),     # CTA pairs, several tiles per pair
]


@pytest.mark.parametrize("M,N,K,bt,sched,split", CASES)
def test_swiglu_against_oracle(M, N, K, bt, sched, split):
    torch.cuda.set_device(0)
    X, W = synth.make_problem(M, N, K, seed=500 + M + N, n_outliers=2)
    if M >= 3:
        X[2] = 0
    qw, s, a, sc = lq.lq_quantize_weights(W.to(DEV))
    xq, sx = lq.lq_quantize_act(X.to(DEV))
    out = torch.full((M, N // 2), float("nan"), dtype=torch.bfloat16, device=DEV)
    lq.lq_w4a8_gemm_swiglu(xq, sx, qw, s, a, sc, out=out, block_t=bt, schedule=sched, split_k=split)
    torch.cuda.synchronize()
    assert lq.lq_get_device_error() == 0
    o_qw, o_s, o_a, o_sc, _ = oracle.quantize_weights(synth.bf16_bits(W))
    o_xq, o_sx = oracle.quantize_act(synth.bf16_bits(X))
    o_out, o_acc = oracle.w4a8_swiglu(o_xq, o_sx, o_qw, o_s, o_a, o_sc)
    acc = lq.lq_w4a8_gemm_i32(xq, qw, s, a)
    np.testing.assert_array_equal(acc.cpu().numpy(), o_acc)
    u = _ulps(_u16(out), o_out)
    assert u.max() <= 1
    assert (u == 0).mean() > 0.95
    if M >= 3:
        assert not (_u16(out)[2] & 0x7FFF).any()  # a zero row gives zero


@pytest.mark.parametrize("M", [16, 256, 4096])
def test_swiglu_mlp_layer(M):
    """The MLP up/gate workload: F = 14336 gate and 14336 up channels, K = 4096
    (sampled outputs where the whole oracle would take too long)."""
    torch.cuda.set_device(0)
    w = synth.WORKLOADS["mlp_up"]
    X, W = synth.make_problem(max(w.Ms), 2 * w.N, w.K, seed=31, n_outliers=41)
    qw, s, a, sc = lq.lq_quantize_weights(W.to(DEV))
    Xm = X[:M].contiguous()
    xq, sx = lq.lq_quantize_act(Xm.to(DEV))
    out = lq.lq_w4a8_gemm_swiglu(xq, sx, qw, s, a, sc)
    torch.cuda.synchronize()
    assert lq.lq_get_device_error() == 0
    o_qw, o_s, o_a, o_sc, _ = oracle.quantize_weights(synth.bf16_bits(W))
    o_xq, o_sx = oracle.quantize_act(synth.bf16_bits(Xm))
    rng = np.random.default_rng(M)
    F = w.N
    edges_m = sorted({0, M - 1} | {m for m in (15, 16, 127, 128, 255, 256) if m < M})
    edges_n = sorted({0, F - 1, 63, 64, 127, 128})
    mi = [m for m in edges_m for _ in edges_n] + rng.integers(0, M, 20000).tolist()
    ni = [n for _ in edges_m for n in edges_n] + rng.integers(0, F, 20000).tolist()
    mi, ni = np.array(mi, np.int64), np.array(ni, np.int64)
    o_out, _ = oracle.w4a8_swiglu_sampled(o_xq, o_sx, o_qw, o_s, o_a, o_sc, mi, ni)
    u = _ulps(_u16(out)[mi, ni], o_out)
    assert u.max() <= 1
    assert (u == 0).mean() > 0.95


def test_swiglu_refuses_streamk_and_persistent():
    torch.cuda.set_device(0)
    M, N, K = 256, 256, 512
    X, W = synth.make_problem(M, N, K, seed=2)
    qw, s, a, sc = lq.lq_quantize_weights(W.to(DEV))
    xq, sx = lq.lq_quantize_act(X.to(DEV))
    for sch in (lq.SCHED_STREAMK, lq.SCHED_PERSISTENT):
        with pytest.raises(lq.LQError) as e:
            lq.lq_w4a8_gemm_swiglu(xq, sx, qw, s, a, sc, schedule=sch)
        assert e.value.status == 2
