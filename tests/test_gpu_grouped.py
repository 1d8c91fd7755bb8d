"""Grouped W4A8 GEMM (one weight matrix per group, as for mixture-of-experts
layers) against the oracle (needs a B200).

Both sides quantize the same seeded bf16 tensors; the group row offsets live
on the device.  int32 accumulators must match bit for bit and bf16 outputs
within 1 bf16 ulp, for every token-tile width and cluster split, with empty
groups and groups whose rows end inside a token tile.
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


def _problem(sizes, N, K, seed, outliers=2):
    E = len(sizes)
    m_off = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    M = int(m_off[-1])
    X, W = synth.make_problem(max(M, 1), E * N, K, seed=seed, n_outliers=outliers)
    X = X[:M]
    g_qw, g_s, g_a, g_sc = lq.lq_quantize_weights(W.to(DEV))
    g_xq, g_sx = lq.lq_quantize_act(X.to(DEV))
    o_qw, o_s, o_a, o_sc, _ = oracle.quantize_weights(synth.bf16_bits(W))
    o_xq, o_sx = oracle.quantize_act(synth.bf16_bits(X))
    np.testing.assert_array_equal(g_qw.cpu().numpy(), o_qw)
    np.testing.assert_array_equal(g_xq.cpu().numpy(), o_xq)
    g = (g_xq, g_sx, g_qw, g_s, g_a, g_sc, torch.from_numpy(m_off).to(DEV))
    o = (o_xq, o_sx, o_qw, o_s, o_a, o_sc, m_off)
    return g, o


# (group sizes, N, K, block_t, split_k); 0 = automatic
CASES = [
    ([3, 0, 7, 20], 256, 512, 0, 0),            # an empty group; 16-token tiles
    ([3, 0, 7, 20], 256, 512, 16, 1),
    ([3, 0, 7, 20], 256, 512, 16, 2),
    ([3, 0, 7, 20], 256, 1024, 16, 4),
    ([3, 0, 7, 20], 256, 2048, 16, 8),
    ([17, 40, 1, 0, 33, 9, 64, 2], 128, 1024, 32, 0),
    ([17, 40, 1, 0, 33, 9, 64, 2], 128, 1024, 64, 4),
    ([130, 60], 256, 768, 128, 1),              # a group crossing token tiles, ragged ends
    ([130, 60], 256, 768, 128, 2),
    ([130, 60], 256, 1024, 128, 4),
    ([0, 0, 5], 128, 256, 0, 0),                # leading empty groups
    ([1], 384, 512, 0, 0),                      # one group: the plain GEMM
    ([300, 0, 520, 190], 256, 1024, 0, 0),      # > 128 rows per group: CTA pairs, ragged groups
    ([3, 700, 40], 512, 512, 256, 0),           # CTA pairs forced, a small group among large ones
    ([257], 256, 768, 256, 0),
]


@pytest.mark.parametrize("sizes,N,K,bt,split", CASES)
def test_grouped_matches_oracle(sizes, N, K, bt, split):
    torch.cuda.set_device(0)
    g, o = _problem(sizes, N, K, seed=sum(sizes) + N + K + bt + split)
    o_out, o_acc = oracle.w4a8_grouped_gemm(*o, N)
    acc = lq.lq_w4a8_grouped_gemm(*g, N, block_t=bt, split_k=split, out_i32=True)
    out = lq.lq_w4a8_grouped_gemm(*g, N, block_t=bt, split_k=split)
    torch.cuda.synchronize()
    assert lq.lq_get_device_error() == 0
    np.testing.assert_array_equal(acc.cpu().numpy(), o_acc)
    assert int(_ulps(_u16(out), o_out).max(initial=0)) <= 1
    # every row belongs to one group: the plain GEMM of that group gives the same bits
    m_off = o[6]
    for e in range(len(sizes)):
        r0, r1 = int(m_off[e]), int(m_off[e + 1])
        if r1 > r0:
            ref = lq.lq_w4a8_gemm(g[0][r0:r1], g[1][r0:r1], g[2][e * N:(e + 1) * N],
                                  g[3][:, e * N:(e + 1) * N].contiguous(), g[4][:, e * N:(e + 1) * N].contiguous(),
                                  g[5][e * N:(e + 1) * N])
            np.testing.assert_array_equal(_u16(out[r0:r1]), _u16(ref))


def test_grouped_moe_decode_and_prefill_shapes():
    """Mixtral-like expert layers (8 experts, N = 4096, K = 4096 to keep the oracle quick):
    a decode batch (16 tokens, top-2 routing: 32 rows) and a prefill-sized one (1024 rows)."""
    torch.cuda.set_device(0)
    rng = np.random.default_rng(5)
    for rows, N, K in ((32, 4096, 4096), (1024, 512, 2048)):
        sizes = np.bincount(rng.integers(0, 8, size=rows), minlength=8).tolist()
        g, o = _problem(sizes, N, K, seed=rows, outliers=8)
        out = lq.lq_w4a8_grouped_gemm(*g, N)
        torch.cuda.synchronize()
        assert lq.lq_get_device_error() == 0
        o_out, _ = oracle.w4a8_grouped_gemm(*o, N)
        assert int(_ulps(_u16(out), o_out).max()) <= 1


def test_grouped_offsets_written_by_a_preceding_kernel():
    """The offsets are read after the grid dependency wait: a kernel that writes them just
    before the GEMM on the same stream is seen."""
    torch.cuda.set_device(0)
    sizes, N, K = [5, 11, 0, 16], 256, 512
    g, o = _problem(sizes, N, K, seed=77)
    m_off = torch.zeros_like(g[6])
    for _ in range(3):
        m_off.zero_()
        m_off.copy_(g[6])          # device-side write, then the GEMM on the same stream
        out = lq.lq_w4a8_grouped_gemm(*g[:6], m_off, N)
    torch.cuda.synchronize()
    o_out, _ = oracle.w4a8_grouped_gemm(*o, N)
    assert int(_ulps(_u16(out), o_out).max()) <= 1
