"""Parity of the CUDA path with the CPU oracle (needs a B200).

Both sides start from the same seeded bf16 tensors (w4a8_bit_weight_b200.synth)
and run their own chain: quantize weights, quantize activations, GEMM.  Codes,
scales, the INT8 expansion and the int32 accumulators must match bit for bit;
bf16 outputs within 1 bf16 ulp (the same operation order makes them equal in
practice, which the tests also report).
"""
import numpy as np
import pytest
import torch

import oracle
import w4a8_bit_weight_b200 as lq
from w4a8_bit_weight_b200 import synth

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _np(t):
    return t.detach().cpu().numpy()


def _bf16_ulps(a_u16: np.ndarray, b_u16: np.ndarray) -> np.ndarray:
    """|ord(a) - ord(b)| where ord maps bf16 bit patterns to a monotone integer (+0 == -0)."""
    def ordv(x):
        x = x.astype(np.int64)
        return np.where(x & 0x8000, -(x & 0x7FFF), x)
    return np.abs(ordv(a_u16) - ordv(b_u16))


def _u16(t):
    return _np(t.contiguous().view(torch.int16)).view(np.uint16)


def quantize_both(X, W):
    """GPU chain and oracle chain from the same bf16 inputs."""
    g_qw, g_s, g_a, g_sc = lq.lq_quantize_weights(W.to(DEV))
    g_xq, g_sx = lq.lq_quantize_act(X.to(DEV))
    o_qw, o_s, o_a, o_sc, _ = oracle.quantize_weights(synth.bf16_bits(W))
    o_xq, o_sx = oracle.quantize_act(synth.bf16_bits(X))
    return (g_qw, g_s, g_a, g_sc, g_xq, g_sx), (o_qw, o_s, o_a, o_sc, o_xq, o_sx)


def assert_quant_equal(g, o):
    g_qw, g_s, g_a, g_sc, g_xq, g_sx = g
    o_qw, o_s, o_a, o_sc, o_xq, o_sx = o
    np.testing.assert_array_equal(_np(g_qw), o_qw)
    np.testing.assert_array_equal(_np(g_s), o_s)
    np.testing.assert_array_equal(_np(g_a), o_a)
    np.testing.assert_array_equal(_np(g_sc).view(np.uint32), o_sc.view(np.uint32))
    np.testing.assert_array_equal(_np(g_xq), o_xq)
    np.testing.assert_array_equal(_np(g_sx).view(np.uint32), o_sx.view(np.uint32))


# ----------------------------------------------------------------------------
# quantizers and the expansion
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("M,N,K,outl", [(16, 256, 512, 0), (3, 48, 192, 2), (33, 4096, 4096, 8)])
def test_quantizers_bitexact(M, N, K, outl):
    X, W = synth.make_problem(M, N, K, seed=100 + M, n_outliers=outl)
    X[1] = 0           # zero activation row
    W[5] = 0           # zero weight row
    W[7, :64] = 0.25   # a constant group
    g, o = quantize_both(X, W)
    assert_quant_equal(g, o)


def test_dequant_bitexact():
    _, W = synth.make_problem(1, 512, 1024, seed=7)
    qw, s, a, sc = lq.lq_quantize_weights(W.to(DEV))
    w_gpu = _np(lq.lq_dequant_weights_i8(qw, s, a))
    w_ref = oracle.dequant(_np(qw), _np(s), _np(a))
    np.testing.assert_array_equal(w_gpu, w_ref)


def test_dequant_identity_all_codes_on_gpu():
    """Every (q, s, a) with q*s + a <= 255 through the device routine (same cases as the oracle pin)."""
    rows, ss, aa = [], [], []
    for s in range(1, 17):
        for a in range(256):
            qmax = min(15, (255 - a) // s)
            rows.append(np.arange(64) % (qmax + 1))
            ss.append(s)
            aa.append(a)
    codes = np.array(rows, np.uint8)
    N = codes.shape[0]
    N_pad = (N + 15) // 16 * 16
    codes = np.concatenate([codes, np.zeros((N_pad - N, 64), np.uint8)])
    c = codes.reshape(N_pad, 8, 8)
    qw = (c[:, :, 0:4] | (c[:, :, 4:8] << 4)).reshape(N_pad, 32).copy()
    s_u8 = np.array(ss + [1] * (N_pad - N), np.uint8).reshape(1, N_pad)
    a_u8 = np.array(aa + [0] * (N_pad - N), np.uint8).reshape(1, N_pad)
    w_gpu = _np(lq.lq_dequant_weights_i8(torch.from_numpy(qw).to(DEV), torch.from_numpy(s_u8).to(DEV),
                                         torch.from_numpy(a_u8).to(DEV)))
    w_ref = oracle.dequant(qw, s_u8, a_u8)
    np.testing.assert_array_equal(w_gpu, w_ref)


# ----------------------------------------------------------------------------
# GEMM: int32 bit-exact and bf16 within 1 ulp, across schedules
# ----------------------------------------------------------------------------

T, P, SK, PR = lq.SCHED_TILES, lq.SCHED_PERSISTENT, lq.SCHED_STREAMK, lq.SCHED_PAIR
SHAPES = [
    # M, N, K, block_t, schedule, split_k, grid   (0 / None = automatic)
    (16, 256, 512, 0, None, 0, 0),        # the tiny workload
    (1, 256, 512, 0, None, 0, 0),
    (1, 16, 128, 0, None, 0, 0),          # one K-block, N smaller than a tile
    (8, 4096, 14336, 0, None, 0, 0),      # automatic: 8-CTA clusters with streaming K-slices, 32-token tiles
    (512, 4096, 1024, 0, None, 0, 0),     # automatic: 128 tiles of 128 x 128 that cannot split K, persistent
    (16, 4352, 14336, 0, None, 0, 0),     # automatic: 34 tiles, more 8-CTA clusters than B200 places at once
    (1, 4608, 14336, 0, None, 0, 0),      # automatic: the same with 36 tiles at one token
    (3, 272, 384, 16, T, 0, 0),           # ragged N (one full + one 16-row tile)
    (17, 384, 1024, 32, T, 0, 0),         # ragged M
    (16, 256, 1024, 16, T, 1, 0),         # one CTA per tile: direct epilogue
    (16, 256, 1024, 16, T, 2, 0),         # cluster split-K, DSMEM reduction
    (5, 256, 1024, 16, T, 4, 0),
    (16, 512, 2048, 16, T, 8, 0),
    (32, 256, 1152, 32, T, 8, 0),         # 9 K-blocks over 8 CTAs: uneven slices
    (40, 384, 1024, 64, T, 4, 0),
    (100, 256, 640, 128, T, 2, 0),
    (100, 384, 1152, 128, T, 4, 0),       # 128-token tiles, 4-CTA clusters: 9 K-blocks unevenly
    (128, 384, 256, 128, T, 0, 0),
    (300, 256, 512, 256, T, 0, 0),        # ragged M with 256-token tiles
    (128, 128, 128, 0, P, 0, 0),          # persistent: one tile
    (300, 256, 512, 0, P, 0, 0),          # persistent: ragged M, one tile per CTA
    (256, 384, 1024, 0, P, 0, 2),         # persistent: 3 tiles per CTA, both accumulators reused
    (1000, 512, 640, 0, P, 0, 3),         # persistent: 32 tiles over 3 CTAs, ragged M
    (256, 256, 512, 0, PR, 0, 0),         # CTA pair: one 256 x 256 tile
    (300, 272, 1024, 0, PR, 0, 0),        # CTA pairs: ragged M and N
    (512, 512, 2048, 0, PR, 0, 2),        # one pair, four tiles: accumulator handed back and forth
    (1000, 768, 768, 0, PR, 0, 4),        # two pairs, 12 tiles, ragged M
    (512, 512, 1024, 0, PR, 0, 6),        # 4 tiles over 3 pairs: the last tile in token halves
    (700, 512, 512, 0, PR, 0, 10),        # 6 tiles over 5 pairs: ragged M in the split last tile
    (16, 256, 1024, 16, SK, 0, 2),        # stream-K, one CTA per tile
    (16, 256, 1024, 16, SK, 0, 3),        # stream-K: split tiles through the workspace
    (16, 256, 1024, 16, SK, 0, 16),       # one K-block per CTA
    (64, 512, 512, 64, SK, 0, 7),
    (100, 256, 640, 128, SK, 0, 5),
    (300, 256, 512, 256, SK, 0, 4),
    (256, 128, 2048, 256, SK, 0, 9),
]


@pytest.mark.parametrize("M,N,K,bt,sched,split,grid", SHAPES)
def test_gemm_parity(M, N, K, bt, sched, split, grid):
    X, W = synth.make_problem(M, N, K, seed=M * 7 + N + K, n_outliers=2)
    g, o = quantize_both(X, W)
    assert_quant_equal(g, o)
    g_qw, g_s, g_a, g_sc, g_xq, g_sx = g
    o_out, o_acc = oracle.w4a8_gemm(*[o[i] for i in (4, 5, 0, 1, 2, 3)])
    kw = dict(block_t=bt, schedule=sched, split_k=split, grid=grid)
    acc = lq.lq_w4a8_gemm_i32(g_xq, g_qw, g_s, g_a, **kw)
    out = lq.lq_w4a8_gemm(g_xq, g_sx, g_qw, g_s, g_a, g_sc, **kw)
    assert lq.lq_get_device_error() == 0
    np.testing.assert_array_equal(_np(acc), o_acc)
    ulps = _bf16_ulps(_u16(out), o_out)
    assert ulps.max() <= 1
    # a second call on the same (restored) workspace gives the same result
    out2 = lq.lq_w4a8_gemm(g_xq, g_sx, g_qw, g_s, g_a, g_sc, **kw)
    acc2 = lq.lq_w4a8_gemm_i32(g_xq, g_qw, g_s, g_a, **kw)
    torch.cuda.synchronize()
    assert torch.equal(out, out2) and torch.equal(acc, acc2)


def test_workspace_left_zero():
    M, N, K = 16, 256, 1024
    X, W = synth.make_problem(M, N, K, seed=3)
    qw, s, a, sc = lq.lq_quantize_weights(W.to(DEV))
    xq, sx = lq.lq_quantize_act(X.to(DEV))
    need = lq.lq_w4a8_gemm_workspace_size(M, N, K, 16, 0, 5, lq.SCHED_STREAMK)
    assert need > 0
    ws = torch.zeros(need, dtype=torch.uint8, device=DEV)
    for _ in range(3):
        lq.lq_w4a8_gemm(xq, sx, qw, s, a, sc, block_t=16, grid=5, workspace_buf=ws)
    torch.cuda.synchronize()
    assert int(ws.count_nonzero()) == 0


def test_degenerate_inputs():
    M, N, K = 20, 256, 512
    X, W = synth.make_problem(M, N, K, seed=5)
    X[0] = 0
    X[3, :] = 1.0       # constant row
    W[0] = 0
    W[9, :] = -0.5      # constant row: every group constant
    W[10, ::2] = 0.0
    g, o = quantize_both(X, W)
    assert_quant_equal(g, o)
    g_qw, g_s, g_a, g_sc, g_xq, g_sx = g
    o_out, o_acc = oracle.w4a8_gemm(*[o[i] for i in (4, 5, 0, 1, 2, 3)])
    out = lq.lq_w4a8_gemm(g_xq, g_sx, g_qw, g_s, g_a, g_sc)
    assert _bf16_ulps(_u16(out), o_out).max() <= 1
    assert not out[0].any() and not out[:, 0].any()


def test_extreme_accumulators():
    """All-max activations against all-max weights: |acc| near K*127*119 without overflow."""
    M, N, K = 16, 128, 8192
    X = torch.ones(M, K, dtype=torch.bfloat16)
    X[1::2] = -1.0
    W = torch.ones(N, K, dtype=torch.bfloat16)
    W[::3] = -1.0
    g, o = quantize_both(X, W)
    assert_quant_equal(g, o)
    g_qw, g_s, g_a, g_sc, g_xq, g_sx = g
    acc = lq.lq_w4a8_gemm_i32(g_xq, g_qw, g_s, g_a)
    o_out, o_acc = oracle.w4a8_gemm(*[o[i] for i in (4, 5, 0, 1, 2, 3)])
    np.testing.assert_array_equal(_np(acc), o_acc)
    assert abs(int(o_acc[0, 0])) == 127 * 119 * K


def test_empty_batch():
    _, W = synth.make_problem(1, 256, 512, seed=1)
    qw, s, a, sc = lq.lq_quantize_weights(W.to(DEV))
    xq = torch.empty(0, 512, dtype=torch.int8, device=DEV)
    sx = torch.empty(0, dtype=torch.float32, device=DEV)
    out = lq.lq_w4a8_gemm(xq, sx, qw, s, a, sc)
    assert out.shape == (0, 256)


# ----------------------------------------------------------------------------
# the workloads at full size: whole output where the oracle is quick, else a
# sample of outputs (tile corners, ragged edges and random points)
# ----------------------------------------------------------------------------

def _sample_points(M, N, n_rand, seed):
    rng = np.random.default_rng(seed)
    ms = set([0, M - 1] + [m for m in (15, 16, 127, 128, 255, 256) if m < M])
    ns = set([0, N - 1] + [n for n in (127, 128, 255, 256) if n < N])
    pts = [(m, n) for m in ms for n in ns]
    pts += list(zip(rng.integers(0, M, n_rand).tolist(), rng.integers(0, N, n_rand).tolist()))
    mi, ni = zip(*pts)
    return np.array(mi, np.int64), np.array(ni, np.int64)


def _workload_check(name, Ms, full_limit=4 * 10 ** 8, n_rand=20000):
    w = synth.WORKLOADS[name]
    X, W = synth.make_workload(w)
    Wd = W.to(DEV)
    g_qw, g_s, g_a, g_sc = lq.lq_quantize_weights(Wd)
    o_qw, o_s, o_a, o_sc, _ = oracle.quantize_weights(synth.bf16_bits(W))
    np.testing.assert_array_equal(_np(g_qw), o_qw)
    np.testing.assert_array_equal(_np(g_s), o_s)
    np.testing.assert_array_equal(_np(g_a), o_a)
    np.testing.assert_array_equal(_np(g_sc).view(np.uint32), o_sc.view(np.uint32))
    for M in Ms:
        Xm = X[:M].contiguous()
        g_xq, g_sx = lq.lq_quantize_act(Xm.to(DEV))
        o_xq, o_sx = oracle.quantize_act(synth.bf16_bits(Xm))
        np.testing.assert_array_equal(_np(g_xq), o_xq)
        np.testing.assert_array_equal(_np(g_sx).view(np.uint32), o_sx.view(np.uint32))
        out = lq.lq_w4a8_gemm(g_xq, g_sx, g_qw, g_s, g_a, g_sc)
        acc = lq.lq_w4a8_gemm_i32(g_xq, g_qw, g_s, g_a)
        assert lq.lq_get_device_error() == 0
        if M * w.N * w.K <= full_limit:
            o_out, o_acc = oracle.w4a8_gemm(o_xq, o_sx, o_qw, o_s, o_a, o_sc)
            np.testing.assert_array_equal(_np(acc), o_acc)
            assert _bf16_ulps(_u16(out), o_out).max() <= 1
        else:
            mi, ni = _sample_points(M, w.N, n_rand, seed=M)
            o_out, o_acc = oracle.w4a8_gemm_sampled(o_xq, o_sx, o_qw, o_s, o_a, o_sc, mi, ni)
            np.testing.assert_array_equal(_np(acc)[mi, ni], o_acc)
            assert _bf16_ulps(_u16(out)[mi, ni], o_out).max() <= 1


def test_workload_tiny():
    _workload_check("tiny", (16,))


def test_workload_decode():
    _workload_check("decode", (1, 4, 16))


def test_workload_prefill():
    _workload_check("prefill", (4096,))


def test_workload_mlp_up():
    _workload_check("mlp_up", (16, 256, 4096))


def test_workload_down_sweep():
    _workload_check("down_sweep", synth.WORKLOADS["down_sweep"].Ms)


def test_device_cluster_table_and_the_schedule_it_gives():
    """The device's cluster placement (lq_device_cluster_ctas) and the automatic
    schedule's use of it: a split's CTAs fit one wave of the clusters it needs."""
    import ctypes
    torch.cuda.set_device(0)
    lib = lq.load_library()
    cl = (ctypes.c_int * 3)()
    assert lib.lq_device_cluster_ctas(cl) == 0
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    for i, c in enumerate((2, 4, 8)):
        assert 0 < cl[i] <= 2 * sms and cl[i] % c == 0, tuple(cl)
    plan = (ctypes.c_int * 4)()
    for (M, N, K) in ((16, 4352, 14336), (1, 4608, 14336), (16, 4096, 14336), (16, 14336, 4096)):
        assert lib.lq_plan_gemm_ex(M, N, K, 0, 0, 0, 0, sms, cl, plan) == 0
        kind, bt, cs, grid = tuple(plan)
        if kind == 1 and cs in (2, 4, 8) and grid > sms:  # two CTAs per SM: the clusters must all fit
            assert grid <= cl[(2, 4, 8).index(cs)], (M, N, K, tuple(plan), tuple(cl))
