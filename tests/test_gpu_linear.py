"""lq_w4a8_linear: activation quantization and the GEMM in one call (needs a B200).

For decode-sized batches the call is one fused launch (each CTA of a split-K
cluster quantizes its K-slice of X, the cluster combines the row maxima
through distributed shared memory); elsewhere it is the two launches.  Either
way the output must be bit-identical to lq_quantize_act followed by
lq_w4a8_gemm, and within 1 bf16 ulp of the oracle's chain.
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


def _ulps(a, b):
    def ordv(x):
        x = x.astype(np.int64)
        return np.where(x & 0x8000, -(x & 0x7FFF), x)
    return np.abs(ordv(a) - ordv(b))


# (M, N, K, fusable): the fused launch applies when M <= 16 and the automatic
# schedule is a split-K cluster (2, 4 or 8 CTAs) whose CTAs each hold at most
# 8 K-blocks of 128; the automatic path takes it for M <= 8
CASES = [
    (1, 4096, 4096, True),     # decode, 4-CTA clusters
    (4, 4096, 4096, True),
    (16, 4096, 4096, True),
    (5, 4096, 4096, True),     # tokens not a multiple of the 4 per quantizing warp
    (16, 2048, 4096, True),    # 8-CTA clusters
    (7, 4096, 1024, True),     # 2-CTA clusters
    (16, 1024, 2048, True),    # 4-CTA clusters, 4 K-blocks each
    (16, 256, 512, False),     # one CTA per tile: two launches
    (3, 14336, 4096, False),   # too many tiles for clusters
    (16, 4096, 14336, False),  # K-slices longer than the preloaded stages
    (24, 4096, 4096, False),   # M > 16
]


@pytest.mark.parametrize("M,N,K,fusable", CASES)
def test_linear_matches_two_step_and_oracle(M, N, K, fusable):
    torch.cuda.set_device(0)
    X, W = synth.make_problem(M, N, K, seed=100 + M + K // 128, n_outliers=3)
    if M >= 3:
        X[2] = 0  # a zero row: s_x = 1, codes 0, output row 0
    assert (lq.lq_w4a8_linear_workspace_size(M, N, K, lq.LINEAR_FUSED) == 0) == fusable
    assert (lq.lq_w4a8_linear_workspace_size(M, N, K) == 0) == (fusable and M <= 8)
    assert lq.lq_w4a8_linear_workspace_size(M, N, K, lq.LINEAR_TWO_LAUNCHES) > 0
    qw, s, a, sc = lq.lq_quantize_weights(W.to(DEV))
    Xd = X.to(DEV)
    xq, sx = lq.lq_quantize_act(Xd)
    ref = lq.lq_w4a8_gemm(xq, sx, qw, s, a, sc)
    paths = [lq.LINEAR_AUTO, lq.LINEAR_TWO_LAUNCHES] + ([lq.LINEAR_FUSED] if fusable else [])
    for path in paths:
        for _ in range(2):  # repeated calls give the same bits
            out = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
            lq.lq_w4a8_linear(Xd, qw, s, a, sc, out=out, path=path)
            torch.cuda.synchronize()
            assert lq.lq_get_device_error() == 0
            np.testing.assert_array_equal(_u16(out), _u16(ref))
    if not fusable:
        with pytest.raises(lq.LQError) as e:
            lq.lq_w4a8_linear(Xd, qw, s, a, sc, path=lq.LINEAR_FUSED)
        assert e.value.status == 2  # LQ_ERR_UNSUPPORTED_SHAPE
    # the oracle's own chain (its quantizers, its GEMM) from the same bf16 inputs
    o_qw, o_s, o_a, o_sc, _ = oracle.quantize_weights(synth.bf16_bits(W))
    o_xq, o_sx = oracle.quantize_act(synth.bf16_bits(X))
    if M * N * K <= 16 * 4096 * 4096:
        o_out, _ = oracle.w4a8_gemm(o_xq, o_sx, o_qw, o_s, o_a, o_sc)
        assert int(_ulps(_u16(out), o_out).max()) <= 1
    else:
        # larger layers: every tile corner and ragged edge plus 20000 random outputs,
        # each computed by the oracle on its own
        rng = np.random.default_rng(M + N + K)
        edge_m = sorted({0, M - 1} | {m for m in (15, 16) if m < M})
        edge_n = sorted({0, N - 1} | {n for n in range(127, N, 128)} | {n for n in range(128, N, 128)})
        mi = [m for m in edge_m for _ in edge_n] + rng.integers(0, M, 20000).tolist()
        ni = [n for _ in edge_m for n in edge_n] + rng.integers(0, N, 20000).tolist()
        mi, ni = np.array(mi, np.int64), np.array(ni, np.int64)
        o_out, _ = oracle.w4a8_gemm_sampled(o_xq, o_sx, o_qw, o_s, o_a, o_sc, mi, ni)
        assert int(_ulps(_u16(out)[mi, ni], o_out).max()) <= 1
    if M >= 3:
        assert not (_u16(out)[2] & 0x7FFF).any()


def test_linear_decode_workload_sampled_rows():
    """The decode workload (8 outlier channels x20) through the fused path, all three M."""
    torch.cuda.set_device(0)
    w = synth.WORKLOADS["decode"]
    X, W = synth.make_workload(w)
    qw, s, a, sc = lq.lq_quantize_weights(W.to(DEV))
    o_qw, o_s, o_a, o_sc, _ = oracle.quantize_weights(synth.bf16_bits(W))
    for M in w.Ms:
        out = lq.lq_w4a8_linear(X[:M].to(DEV), qw, s, a, sc, path=lq.LINEAR_FUSED)
        torch.cuda.synchronize()
        o_xq, o_sx = oracle.quantize_act(synth.bf16_bits(X[:M]))
        o_out, _ = oracle.w4a8_gemm(o_xq, o_sx, o_qw, o_s, o_a, o_sc)
        assert int(_ulps(_u16(out), o_out).max()) <= 1


def test_linear_fallback_workspace_rules():
    torch.cuda.set_device(0)
    M, N, K = 24, 256, 512
    need = lq.lq_w4a8_linear_workspace_size(M, N, K)
    assert need >= M * K + 4 * M
    X, W = synth.make_problem(M, N, K, seed=7)
    qw, s, a, sc = lq.lq_quantize_weights(W.to(DEV))
    Xd = X.to(DEV)
    small = torch.zeros(need - 16, dtype=torch.uint8, device=DEV)
    with pytest.raises(lq.LQError) as e:
        lq.lq_w4a8_linear(Xd, qw, s, a, sc, workspace_buf=small)
    assert e.value.status == 4  # LQ_ERR_WORKSPACE
    ws = torch.zeros(need, dtype=torch.uint8, device=DEV)
    out = lq.lq_w4a8_linear(Xd, qw, s, a, sc, workspace_buf=ws)
    xq, sx = lq.lq_quantize_act(Xd)
    np.testing.assert_array_equal(_u16(out), _u16(lq.lq_w4a8_gemm(xq, sx, qw, s, a, sc)))
