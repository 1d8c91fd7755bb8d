"""The dequantization-pipeline ablation kernels against the oracle (needs a B200).

Per-element vs SWAR expansion, tensor-memory vs shared-memory A operand: every
variant must give the oracle's int32 accumulators bit for bit and bf16 outputs
within 1 ulp (bit-identical to the product kernel), across ragged sizes and
several K-blocks per CTA.
"""
import numpy as np
import pytest
import torch

import oracle
import w4a8_bit_weight_b200 as lq
from w4a8_bit_weight_b200 import synth

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
VARIANTS = [lq.ABL_IMPLICIT, lq.ABL_NAIVE, lq.ABL_EXPLICIT, lq.ABL_NAIVE_EXPLICIT]


def _u16(t):
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _ulps(a, b):
    def ordv(x):
        x = x.astype(np.int64)
        return np.where(x & 0x8000, -(x & 0x7FFF), x)
    return np.abs(ordv(a) - ordv(b))


@pytest.mark.parametrize("M,N,K,bt", [
    (16, 256, 512, 16),      # one K-block per CTA
    (5, 384, 4096, 16),      # 8 K-blocks per CTA (the overflow-block shape of the product kernel)
    (13, 272, 6144, 16),     # refills, ragged N
    (40, 256, 1024, 64),
    (64, 512, 4096, 64),     # several stages and refills
])
def test_ablation_variants_match_oracle(M, N, K, bt):
    torch.cuda.set_device(0)
    X, W = synth.make_problem(M, N, K, seed=M + N + K, n_outliers=3)
    qw, s, a, sc = lq.lq_quantize_weights(W.to(DEV))
    xq, sx = lq.lq_quantize_act(X.to(DEV))
    o_qw, o_s, o_a, o_sc, _ = oracle.quantize_weights(synth.bf16_bits(W))
    o_xq, o_sx = oracle.quantize_act(synth.bf16_bits(X))
    o_out, o_acc = oracle.w4a8_gemm(o_xq, o_sx, o_qw, o_s, o_a, o_sc)
    ref = lq.lq_w4a8_gemm(xq, sx, qw, s, a, sc, block_t=bt, split_k=4)
    for v in VARIANTS:
        acc = lq.lq_w4a8_gemm_ablation(xq, sx, qw, s, a, sc, v, bt, out_i32=True)
        out = lq.lq_w4a8_gemm_ablation(xq, sx, qw, s, a, sc, v, bt)
        torch.cuda.synchronize()
        assert lq.lq_get_device_error() == 0
        np.testing.assert_array_equal(acc.cpu().numpy(), o_acc, err_msg=f"variant {v}")
        assert int(_ulps(_u16(out), o_out).max()) <= 1
        np.testing.assert_array_equal(_u16(out), _u16(ref))
