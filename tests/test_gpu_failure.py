"""Failure detection without a fault (needs a B200): a bounded wait that runs
out is reported through the device error word, the other waits of the CTA
leave on the abort flag, and the context stays usable."""
import time

import numpy as np
import pytest
import torch

import oracle
import w4a8_bit_weight_b200 as lq
from w4a8_bit_weight_b200 import synth

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def test_bounded_wait_times_out_and_the_context_survives():
    torch.cuda.set_device(0)
    assert lq.lq_get_device_error() == 0
    t0 = time.time()
    lq.lq_test_wait_timeout()
    st = lq.lq_get_device_error()
    elapsed = time.time() - t0
    assert st == 6  # LQ_ERR_TIMEOUT
    # one 2 s limit: the second warp left on the abort flag instead of waiting out its own
    assert 1.5 < elapsed < 3.5, elapsed
    assert lq.lq_get_device_error() == 0  # read and cleared
    # the context still runs the GEMM correctly
    w = synth.WORKLOADS["tiny"]
    X, W = synth.make_workload(w)
    qw, s, a, sc = lq.lq_quantize_weights(W.to(DEV))
    xq, sx = lq.lq_quantize_act(X.to(DEV))
    acc = lq.lq_w4a8_gemm_i32(xq, qw, s, a)
    assert lq.lq_get_device_error() == 0
    o_qw, o_s, o_a, o_sc, _ = oracle.quantize_weights(synth.bf16_bits(W))
    o_xq, o_sx = oracle.quantize_act(synth.bf16_bits(X))
    _, o_acc = oracle.w4a8_gemm(o_xq, o_sx, o_qw, o_s, o_a, o_sc)
    np.testing.assert_array_equal(acc.cpu().numpy(), o_acc)
