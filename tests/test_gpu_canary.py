"""Canary guards around the outputs (needs a B200): every kernel writes its
output inside a buffer whose guard regions before and after hold a pattern;
the pattern must be untouched after the call, for ragged shapes of every
schedule (the sanitizer is not available on this machine, so out-of-bounds
writes are looked for this way)."""
import numpy as np
import pytest
import torch

import w4a8_bit_weight_b200 as lq
from w4a8_bit_weight_b200 import synth

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
GUARD = 4096  # elements on each side (a multiple of 8: the output stays 16-byte aligned)


def _guarded(shape, dtype, fill):
    n = int(np.prod(shape))
    buf = torch.full((n + 2 * GUARD,), fill, dtype=dtype, device=DEV)
    return buf, buf[GUARD:GUARD + n].view(*shape)


def _check_guards(buf, fill):
    torch.cuda.synchronize()
    head, tail = buf[:GUARD], buf[-GUARD:]
    ref = torch.full_like(head, fill)
    assert torch.equal(head, ref) and torch.equal(tail, ref)


@pytest.mark.parametrize("M,N,K,kw", [
    (3, 272, 384, dict(block_t=16, schedule=lq.SCHED_TILES)),
    (17, 384, 1024, dict(block_t=32, schedule=lq.SCHED_TILES)),
    (5, 256, 1024, dict(block_t=16, split_k=4)),
    (100, 384, 1152, dict(block_t=128, split_k=4)),
    (300, 256, 512, dict(block_t=256, schedule=lq.SCHED_TILES)),
    (300, 272, 1024, dict(schedule=lq.SCHED_PAIR)),
    (700, 512, 512, dict(schedule=lq.SCHED_PAIR, grid=10)),
    (300, 256, 512, dict(schedule=lq.SCHED_PERSISTENT)),
    (16, 256, 1024, dict(block_t=16, schedule=lq.SCHED_STREAMK, grid=3)),
])
def test_gemm_writes_stay_inside_the_output(M, N, K, kw):
    torch.cuda.set_device(0)
    X, W = synth.make_problem(M, N, K, seed=M + N + K, n_outliers=2)
    qw, s, a, sc = lq.lq_quantize_weights(W.to(DEV))
    xq, sx = lq.lq_quantize_act(X.to(DEV))
    buf, out = _guarded((M, N), torch.bfloat16, -3.0)
    lq.lq_w4a8_gemm(xq, sx, qw, s, a, sc, out=out, **kw)
    _check_guards(buf, -3.0)
    ibuf, iout = _guarded((M, N), torch.int32, 0x5A5A5A5A)
    lq.lq_w4a8_gemm_i32(xq, qw, s, a, out=iout, **kw)
    _check_guards(ibuf, 0x5A5A5A5A)
    assert lq.lq_get_device_error() == 0


def test_other_entry_points_write_inside_their_outputs():
    torch.cuda.set_device(0)
    M, N, K = 13, 384, 1024
    X, W = synth.make_problem(M, N, K, seed=5, n_outliers=2)
    Xd, Wd = X.to(DEV), W.to(DEV)
    # quantizers
    qbuf, qw = _guarded((N, K // 2), torch.uint8, 0xA5)
    sbuf, s = _guarded((K // 64, N), torch.uint8, 0xA5)
    abuf, a = _guarded((K // 64, N), torch.uint8, 0xA5)
    cbuf, sc = _guarded((N,), torch.float32, -7.0)
    lq.lq_quantize_weights(Wd, out=(qw, s, a, sc))
    for b, f in ((qbuf, 0xA5), (sbuf, 0xA5), (abuf, 0xA5), (cbuf, -7.0)):
        _check_guards(b, f)
    xbuf, xq = _guarded((M, K), torch.int8, -77)
    xsbuf, sx = _guarded((M,), torch.float32, -7.0)
    lq.lq_quantize_act(Xd, out=(xq, sx))
    _check_guards(xbuf, -77)
    _check_guards(xsbuf, -7.0)
    # fused linear path and grouped GEMM
    lbuf, lout = _guarded((M, N), torch.bfloat16, -3.0)
    lq.lq_w4a8_linear(Xd[:5].contiguous(), qw, s, a, sc, out=lout[:5])
    _check_guards(lbuf, -3.0)
    m_off = torch.tensor([0, 4, 4, 13], dtype=torch.int32, device=DEV)
    Xg, Wg = synth.make_problem(M, 3 * 256, 512, seed=6)
    gq, gs, ga, gc = lq.lq_quantize_weights(Wg.to(DEV))
    gxq, gsx = lq.lq_quantize_act(Xg.to(DEV))
    gbuf, gout = _guarded((M, 256), torch.bfloat16, -3.0)
    lq.lq_w4a8_grouped_gemm(gxq, gsx, gq, gs, ga, gc, m_off, 256, out=gout)
    _check_guards(gbuf, -3.0)
    # W4 x FP8
    q4, sw = lq.lq_quantize_weights_w4(Wd)
    x8, s8 = lq.lq_quantize_act_f8(Xd)
    fbuf, fout = _guarded((M, N), torch.bfloat16, -3.0)
    lq.lq_w4f8_gemm(x8, s8, q4, sw, out=fout)
    _check_guards(fbuf, -3.0)
    assert lq.lq_get_device_error() == 0
