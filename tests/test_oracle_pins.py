"""Pins of the CPU oracle to facts outside itself (CPU only).

Each test checks the oracle against something it does not compute itself:
exhaustive brute force over the method's code space, closed forms from two's
complement arithmetic, hand-worked examples (tests/golden/), invariants the
paper proves, library routines (numpy int64/float64 matmul, torch's bf16
rounding), and the quantization error bound.  The method's source is the
pith.science review of "LiquidGEMM" (arXiv 2509.01229); each test names the
passage it pins.
"""
import os

import numpy as np
import pytest
import torch

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _rows(fname):
    out = []
    with open(os.path.join(GOLD, fname)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            out.append([c.strip() for c in line.split("|")])
    return out


def _pack_rows(codes: np.ndarray) -> np.ndarray:
    """Packed layout of the format spec (tests/golden/pack_layout.txt), from codes [N, K]."""
    N, K = codes.shape
    c = codes.reshape(N, K // 8, 8).astype(np.uint8)
    b = c[:, :, 0:4] | (c[:, :, 4:8] << 4)
    return b.reshape(N, K // 2).copy()


# ---------------------------------------------------------------------------
# Dequantization identity (review: "What carries the argument", Eq. 12)
# ---------------------------------------------------------------------------

def test_dequant_identity_exhaustive():
    """All 16 codes x s in [1,16] x a in [0,255] with q*s + a <= 255: int8 result
    equals q*s + a - 128 (two's-complement congruence mod 2^8, the circularity
    rationale's 'standard math' axiom)."""
    G, K = 64, 64
    rows_codes, rows_s, rows_a = [], [], []
    for s in range(1, 17):
        for a in range(256):
            qmax = min(15, (255 - a) // s)
            if qmax < 0:
                continue
            rows_codes.append(np.arange(K) % (qmax + 1))
            rows_s.append(s)
            rows_a.append(a)
    codes = np.array(rows_codes, dtype=np.int64)
    N = codes.shape[0]
    qw = _pack_rows(codes)
    s_u8 = np.array(rows_s, np.uint8).reshape(1, N)
    a_u8 = np.array(rows_a, np.uint8).reshape(1, N)
    w = oracle.dequant(qw, s_u8, a_u8, G)
    expect = codes * np.array(rows_s)[:, None] + np.array(rows_a)[:, None] - 128
    assert expect.min() >= -128 and expect.max() <= 127
    np.testing.assert_array_equal(w.astype(np.int64), expect)
    # every (q, s, a) triple with q*s + a <= 255 was covered
    covered = {(int(q), s, a) for row, s, a in zip(codes, rows_s, rows_a) for q in set(row.tolist())}
    total = sum(1 for q in range(16) for s in range(1, 17) for a in range(256) if q * s + a <= 255)
    assert len(covered) == total


def test_dequant_rejects_uint8_overflow():
    """Outside the proven range the oracle reports an error instead of wrapping."""
    codes = np.full((1, 64), 15)
    with pytest.raises(oracle.OracleError):
        oracle.dequant(_pack_rows(codes), np.array([[16]], np.uint8), np.array([[20]], np.uint8))


# ---------------------------------------------------------------------------
# UINT8 range proof over every reachable group (review: major comment 3;
# circularity rationale, Eq. 11 with Q_i8 in [-119,119] and s_u8 <= 16)
# ---------------------------------------------------------------------------

def _reachable_groups():
    """Every (R, mn) with mn in [-119, 119-R], and every Q value in [mn, mn+R],
    spread over groups of 64 that each contain both mn and mn+R."""
    groups = []
    meta = []
    for R in range(0, 239):
        vals_all = np.arange(R + 1)
        per = 62
        chunks = [vals_all[i:i + per] for i in range(0, R + 1, per)]
        for mn in range(-119, 120 - R):
            for ch in chunks:
                g = np.empty(64, np.int64)
                g[0], g[1] = mn, mn + R
                g[2:2 + len(ch)] = mn + ch
                g[2 + len(ch):] = mn
                groups.append(g)
                meta.append((R, mn))
    return np.array(groups), np.array(meta)


@pytest.fixture(scope="module")
def reachable():
    groups, meta = _reachable_groups()
    q_i8 = groups.astype(np.int8).reshape(-1, 64)
    qw, s_u8, a_u8 = oracle.quantize_groups(q_i8, 64)
    return groups, meta, q_i8, qw, s_u8, a_u8


def test_uint8_range_all_reachable_groups(reachable):
    groups, meta, q_i8, qw, s_u8, a_u8 = reachable
    # every distinct (R, mn, value) case is present: sum_R (R+1)(239-R)
    distinct = {(R, mn, int(v)) for g, (R, mn) in zip(groups, meta) for v in np.unique(g)}
    assert len(distinct) == sum((R + 1) * (239 - R) for R in range(239)) == 2303960
    s = s_u8[0].astype(np.int64)
    a = a_u8[0].astype(np.int64)
    codes = np.stack([qw[:, 0::1] & 0x0F, qw >> 4], axis=-1)  # not in k order; only the range matters
    pre = codes.reshape(qw.shape[0], -1).astype(np.int64) * s[:, None] + a[:, None]
    assert pre.min() >= 0 and pre.max() <= 255
    assert pre.max() == 254  # round-to-nearest scale never reaches 255
    # the dequant runs without a range error on all of them
    w = oracle.dequant(qw, s_u8, a_u8, 64)
    assert w.shape == q_i8.shape


def test_scale_bounds(reachable):
    """s_u8 = round(R/15) with s >= 1; at most 16, the value major comment 3 derives for R = 238."""
    groups, meta, q_i8, qw, s_u8, a_u8 = reachable
    R = meta[:, 0]
    s = s_u8[0].astype(np.int64)
    assert s.min() >= 1 and s.max() == 16
    # round(R/15) = 16 exactly for R in [233, 238]
    assert set(R[s == 16].tolist()) == set(range(233, 239))
    # |s - R/15| <= 1/2 whenever R >= 8 (nearest integer); s = 1 for R <= 7
    big = R >= 8
    assert np.all(np.abs(s[big] - R[big] / 15.0) <= 0.5)
    assert np.all(s[~big] == 1)
    # offset a = 2^7 + min
    assert np.array_equal(a_u8[0].astype(np.int64), 128 + meta[:, 1])


def test_reconstruction_error_bound(reachable):
    """Q_hat - Q_i8 = s*round(u/s) - u: within s/2 when the code is not clamped, and the
    clamped codes reconstruct to 15*s + mn exactly."""
    groups, meta, q_i8, qw, s_u8, a_u8 = reachable
    w = oracle.dequant(qw, s_u8, a_u8, 64).astype(np.int64)
    s = s_u8[0].astype(np.int64)[:, None]
    mn = meta[:, 1][:, None]
    u = groups - mn
    err = w - groups
    unclamped = (2 * u + s) // (2 * s) <= 15
    assert np.all(2 * np.abs(err[unclamped]) <= s.repeat(64, 1)[unclamped])
    assert np.array_equal(w[~unclamped], (15 * s + mn).repeat(64, 1)[~unclamped])


# ---------------------------------------------------------------------------
# Hand-worked golden examples (tests/golden/lqq_groups.txt)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("row", _rows("lqq_groups.txt"), ids=lambda r: r[0])
def test_golden_groups(row):
    name, vals, s, a, q, pre, qhat = row
    vals = [int(v) for v in vals.split()]
    g = np.full(64, vals[0], np.int64)
    g[:len(vals)] = vals
    qw, s_u8, a_u8 = oracle.quantize_groups(g.astype(np.int8).reshape(1, 64))
    assert int(s_u8[0, 0]) == int(s) and int(a_u8[0, 0]) == int(a)
    codes = np.empty(64, np.int64)
    codes[0::8], codes[1::8], codes[2::8], codes[3::8] = [qw[0, b::4] & 15 for b in range(4)]
    codes[4::8], codes[5::8], codes[6::8], codes[7::8] = [qw[0, b::4] >> 4 for b in range(4)]
    n = len(vals)
    assert codes[:n].tolist() == [int(x) for x in q.split()]
    assert (codes[:n] * int(s) + int(a)).tolist() == [int(x) for x in pre.split()]
    w = oracle.dequant(qw, s_u8, a_u8)
    assert w[0, :n].tolist() == [int(x) for x in qhat.split()]


def test_golden_pack_layout():
    rows = {r[0]: r[1] for r in _rows("pack_layout.txt")}
    codes = np.array([int(x) for x in rows["codes"].split()], np.int64)
    want = [int(x) for x in rows["bytes"].split()]
    # the oracle packs exactly this: build a 64-wide group whose first 16 codes are these
    s = 1
    q_i8 = np.zeros((1, 64), np.int8)
    q_i8[0, :16] = codes  # mn = 0, R = 15 -> s = 1, a = 128, code = value
    q_i8[0, 16:] = 0
    qw, s_u8, a_u8 = oracle.quantize_groups(q_i8)
    assert int(s_u8[0, 0]) == s and int(a_u8[0, 0]) == 128
    assert qw[0, :8].tolist() == want


# ---------------------------------------------------------------------------
# Level 1 and activation casts (review: protective range [-119,119]; 8-bit
# per-token activations)
# ---------------------------------------------------------------------------

def _bf16_bits(vals):
    return torch.tensor(vals, dtype=torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("row", _rows("rounding.txt"), ids=lambda r: f"{r[0]}-{r[2][:12]}")
def test_golden_rounding(row):
    kind, bound, vals, codes, scale = row
    vals = [float(v) for v in vals.split()]
    bits = _bf16_bits(vals).reshape(1, -1)
    # the fixture values are exact in bf16
    assert np.array_equal(torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy()[0],
                          np.array(vals, np.float32))
    if kind == "weight":
        q, s = oracle.quantize_channels(bits)
    else:
        q, s = oracle.quantize_act(bits)
    assert q[0].tolist() == [int(c) for c in codes.split()]
    assert float(s[0]) == float(scale)


@pytest.mark.parametrize("which,bound", [("weight", 119), ("act", 127)])
def test_cast_invariants(which, bound):
    g = torch.Generator().manual_seed(11)
    x = torch.randn(64, 640, generator=g) * torch.logspace(-3, 2, 64).unsqueeze(1)
    x[5] = 0.0
    x[7, 3] = 1e4  # a lone outlier
    bits = x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    xf = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    q, s = oracle.quantize_channels(bits) if which == "weight" else oracle.quantize_act(bits)
    q = q.astype(np.int64)
    s = s.astype(np.float64)
    assert np.abs(q).max() <= bound
    amax = np.abs(xf).max(axis=1)
    nz = amax > 0
    # the largest magnitude of each row maps to +-bound, with its sign
    arg = np.abs(xf).argmax(axis=1)
    top = q[np.arange(64), arg]
    assert np.all(np.abs(top[nz]) == bound)
    assert np.all(np.sign(top[nz]) == np.sign(xf[np.arange(64), arg][nz]))
    # scale is amax / bound (to fp32 rounding), zero rows get scale 1 and codes 0
    np.testing.assert_allclose(s[nz], amax[nz] / bound, rtol=2 ** -23)
    assert s[5] == 1.0 and not q[5].any()
    # reconstruction within half a step (plus fp32 rounding of the scaled value)
    err = np.abs(q * s[:, None] - xf)
    assert np.all(err[nz] <= (0.5 + 1e-4) * s[nz, None])
    # codes keep the sign and order of the inputs
    assert np.all(np.sign(q) * np.sign(xf) >= 0)


# ---------------------------------------------------------------------------
# Contraction and epilogue (GEMM loop nest of Figure 2; scale epilogue)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("M,N,K", [(1, 1, 64), (3, 5, 128), (7, 9, 192), (16, 24, 512)])
def test_gemm_i32_matches_float64_matmul(M, N, K):
    rng = np.random.default_rng(M * 100 + N)
    x = rng.integers(-127, 128, (M, K)).astype(np.int8)
    w = rng.integers(-128, 128, (N, K)).astype(np.int8)
    acc = oracle.gemm_i32(x, w)
    ref = x.astype(np.float64) @ w.astype(np.float64).T  # exact: |sum| < 2^53
    np.testing.assert_array_equal(acc.astype(np.float64), ref)


def test_gemm_i32_extremes_and_range_check():
    K = 14336
    x = np.full((2, K), 127, np.int8)
    x[1] = -127
    w = np.full((2, K), -128, np.int8)
    w[1] = 127
    acc = oracle.gemm_i32(x, w)
    assert acc.tolist() == [[-127 * 128 * K, 127 * 127 * K], [127 * 128 * K, -127 * 127 * K]]
    big = np.full((1, 140000), 127, np.int8)
    with pytest.raises(oracle.OracleError):
        oracle.gemm_i32(big, big)


def test_bf16_rounding_matches_torch():
    g = torch.Generator().manual_seed(3)
    f = torch.cat([torch.randn(20000, generator=g) * 10.0 ** torch.randint(-30, 30, (20000,), generator=g),
                   torch.tensor([0.0, -0.0, 1.0, 1.00390625, 1.01171875, -1.00390625, 3.0e38,
                                 float("inf"), float("-inf"), 1e-40, -1e-42])])
    want = f.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.f32_to_bf16(float(v)) for v in f.numpy()], np.uint16)
    np.testing.assert_array_equal(got, want)


def test_epilogue_against_float64():
    rng = np.random.default_rng(5)
    M, N = 9, 13
    acc = rng.integers(-2 ** 27, 2 ** 27, (M, N)).astype(np.int32)
    sx = (rng.random(M) * 0.1 + 1e-3).astype(np.float32)
    sc = (rng.random(N) * 1e-3 + 1e-5).astype(np.float32)
    out = oracle.epilogue(acc, sx, sc)
    y = torch.from_numpy(out.view(np.int16)).view(torch.bfloat16).double().numpy()
    exact = acc.astype(np.float64) * sx[:, None].astype(np.float64) * sc[None, :].astype(np.float64)
    # bf16 keeps 8 significant bits: half an ulp is at most 2^-8 relative; fp32 steps add < 2^-22
    assert np.all(np.abs(y - exact) <= np.abs(exact) * (2 ** -8 + 2 ** -21))
    # row/column scales are not transposed: scaling one row changes only that row
    sx2 = sx.copy()
    sx2[4] *= 2
    out2 = oracle.epilogue(acc, sx2, sc)
    diff = out2 != out
    assert diff[4].all() and not np.delete(diff, 4, axis=0).any()


# ---------------------------------------------------------------------------
# Whole method against the unquantized product (quantization error bound)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("M,N,K,outliers", [(16, 256, 512, 0), (5, 48, 256, 4), (1, 16, 64, 0)])
def test_whole_path_within_quantization_bound(M, N, K, outliers):
    from w4a8_bit_weight_b200 import synth
    X, W = synth.make_problem(M, N, K, seed=M + N + K, n_outliers=outliers)
    xb, wb = synth.bf16_bits(X), synth.bf16_bits(W)
    qw, s_u8, a_u8, s_c, q_i8 = oracle.quantize_weights(wb)
    x_q, s_x = oracle.quantize_act(xb)
    out, acc = oracle.w4a8_gemm(x_q, s_x, qw, s_u8, a_u8, s_c)
    y = torch.from_numpy(out.view(np.int16)).view(torch.bfloat16).double().numpy()
    Xd, Wd = X.double().numpy(), W.double().numpy()
    ref = Xd @ Wd.T
    # error bound from the per-step guarantees:
    #  |x - x_q s_x| <= s_x/2;  |w - Q_i8 s_c| <= s_c/2;
    #  |Q_hat - Q_i8| <= E_g = max(s_u8/2, R_g - 15 s_u8)  (pinned above)
    Q = q_i8.astype(np.int64).reshape(N, K // 64, 64)
    R = Q.max(-1) - Q.min(-1)
    s = s_u8.T.astype(np.int64)
    Eg = np.maximum(s / 2.0, R - 15 * s)
    dw = (s_c[:, None].astype(np.float64) * (0.5 + np.repeat(Eg, 64, axis=1)))  # [N, K]
    dx = np.repeat(s_x[:, None].astype(np.float64) / 2.0, K, axis=1)            # [M, K]
    bound = dx @ np.abs(Wd).T + np.abs(Xd) @ dw.T + dx @ dw.T
    bound += np.abs(ref) * 2 ** -8 + 1e-6
    assert np.all(np.abs(y - ref) <= bound)
    # and it is a real check: 4-bit weights with 15 levels per group leave an rms error of
    # roughly a tenth of the output spread; a wrong index or operand gives ~100% or more
    assert np.sqrt(np.mean((y - ref) ** 2)) < 0.25 * np.std(ref)
    # int32 accumulators are the exact product of the dequantized operands
    w_hat = oracle.dequant(qw, s_u8, a_u8)
    np.testing.assert_array_equal(acc.astype(np.float64),
                                  x_q.astype(np.float64) @ w_hat.astype(np.float64).T)


def test_sampled_equals_full():
    from w4a8_bit_weight_b200 import synth
    X, W = synth.make_problem(7, 80, 256, seed=9, n_outliers=3)
    qw, s_u8, a_u8, s_c, _ = oracle.quantize_weights(synth.bf16_bits(W))
    x_q, s_x = oracle.quantize_act(synth.bf16_bits(X))
    out, acc = oracle.w4a8_gemm(x_q, s_x, qw, s_u8, a_u8, s_c)
    mi, ni = np.meshgrid(np.arange(7), np.arange(80), indexing="ij")
    so, sa = oracle.w4a8_gemm_sampled(x_q, s_x, qw, s_u8, a_u8, s_c, mi.ravel(), ni.ravel())
    np.testing.assert_array_equal(so, out.ravel())
    np.testing.assert_array_equal(sa, acc.ravel())


# ---------------------------------------------------------------------------
# Grouped GEMM (one weight matrix per group): against a float64 product of the
# dequantized stacked weights, each row taking the columns of its own group
# ---------------------------------------------------------------------------

def test_grouped_gemm_against_float64_rows():
    from w4a8_bit_weight_b200 import synth
    E, N, K = 4, 32, 256
    m_off = [0, 3, 3, 10, 13]          # group 1 is empty
    M = m_off[-1]
    X, W = synth.make_problem(M, E * N, K, seed=41, n_outliers=2)
    qw, s_u8, a_u8, s_c, _ = oracle.quantize_weights(synth.bf16_bits(W))
    x_q, s_x = oracle.quantize_act(synth.bf16_bits(X))
    out, acc = oracle.w4a8_grouped_gemm(x_q, s_x, qw, s_u8, a_u8, s_c, m_off, N)
    w_hat = oracle.dequant(qw, s_u8, a_u8).astype(np.float64)          # [E*N, K]
    full = x_q.astype(np.float64) @ w_hat.T                               # [M, E*N]
    for e in range(E):
        for m in range(m_off[e], m_off[e + 1]):
            np.testing.assert_array_equal(acc[m].astype(np.float64), full[m, e * N:(e + 1) * N])
            ref = oracle.epilogue(acc[m:m + 1], s_x[m:m + 1], s_c[e * N:(e + 1) * N])
            np.testing.assert_array_equal(out[m], ref[0])
    # one group is the plain GEMM
    o1, a1 = oracle.w4a8_grouped_gemm(x_q, s_x, qw[:N], s_u8[:, :N], a_u8[:, :N], s_c[:N], [0, M], N)
    o2, a2 = oracle.w4a8_gemm(x_q, s_x, qw[:N], s_u8[:, :N], a_u8[:, :N], s_c[:N])
    np.testing.assert_array_equal(a1, a2)
    np.testing.assert_array_equal(o1, o2)


# ---------------------------------------------------------------------------
# W4 x FP8 variant: e4m3 against torch's float8_e4m3fn (a library routine),
# the INT4 and FP8 quantizers against their closed forms, the GEMM against a
# float64 product of the decoded operands
# ---------------------------------------------------------------------------

def _torch_e4m3_code(x: float) -> int:
    return int(torch.tensor([x], dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8)[0])


def test_e4m3_decode_all_codes_match_torch():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).float().numpy()
    got = np.array([oracle.e4m3_to_f32(c) for c in range(256)], np.float32)
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(got[ok].view(np.uint32), ref[ok].view(np.uint32))
    assert oracle.e4m3_to_f32(0x7E) == 448.0 and oracle.e4m3_to_f32(0x01) == 2.0 ** -9


def test_e4m3_encode_matches_torch_rounding_and_saturates():
    # every bf16 value: round to nearest even wherever torch's conversion is finite
    bits = np.arange(65536, dtype=np.uint32) << 16
    vals = bits.view(np.float32)
    fin = np.isfinite(vals) & (np.abs(vals) <= 464.0)
    ref = torch.from_numpy(vals[fin].copy()).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.f32_to_e4m3(v) for v in vals[fin]], np.uint8)
    np.testing.assert_array_equal(got, ref)
    # ties between neighbouring codes go to the even code, as in torch
    for c in range(0x7E):
        lo, hi = oracle.e4m3_to_f32(c), oracle.e4m3_to_f32(c + 1)
        mid = np.float32((lo + hi) / 2)
        assert oracle.f32_to_e4m3(mid) == _torch_e4m3_code(float(mid)) == (c if c % 2 == 0 else c + 1)
        assert oracle.f32_to_e4m3(-mid) == 0x80 | (c if c % 2 == 0 else c + 1)
    # finite values beyond the largest code saturate to +-448 (torch gives NaN there)
    for x in (465.0, 500.0, 1e6, 3.4e38):
        assert oracle.f32_to_e4m3(x) == 0x7E and oracle.f32_to_e4m3(-x) == 0xFE
    assert oracle.f32_to_e4m3(float("nan")) == 0x7F


def test_w4_weight_quantizer_closed_form():
    from w4a8_bit_weight_b200 import synth
    _, W = synth.make_problem(1, 48, 256, seed=12, n_outliers=0)
    W[5] = 0
    wb = synth.bf16_bits(W)
    qw4, s_w = oracle.quantize_weights_w4(wb)
    w = W.float().numpy()
    u = np.empty(w.shape, np.int64)
    u[:, 0::8], u[:, 4::8] = (qw4[:, 0::4] & 15), (qw4[:, 0::4] >> 4)
    u[:, 1::8], u[:, 5::8] = (qw4[:, 1::4] & 15), (qw4[:, 1::4] >> 4)
    u[:, 2::8], u[:, 6::8] = (qw4[:, 2::4] & 15), (qw4[:, 2::4] >> 4)
    u[:, 3::8], u[:, 7::8] = (qw4[:, 3::4] & 15), (qw4[:, 3::4] >> 4)
    q = u - 8
    assert q.min() >= -7 and q.max() <= 7
    amax = np.abs(w).max(axis=1)
    for n in range(w.shape[0]):
        if amax[n] == 0:
            assert s_w[n] == 1.0 and (q[n] == 0).all()
            continue
        assert s_w[n] == np.float32(amax[n]) / np.float32(7.0)
        inv = np.float32(7.0) / np.float32(amax[n])
        np.testing.assert_array_equal(q[n], np.clip(np.rint((w[n] * inv).astype(np.float32)), -7, 7))
        assert np.abs(q[n][np.argmax(np.abs(w[n]))]) == 7
        assert np.all(np.abs(w[n] - q[n] * s_w[n]) <= s_w[n] * 0.5 * (1 + 1e-5))


def test_f8_activation_quantizer_closed_form():
    from w4a8_bit_weight_b200 import synth
    X, _ = synth.make_problem(6, 16, 128, seed=13, n_outliers=2)
    xb = synth.bf16_bits(X)
    x_f8, s_x = oracle.quantize_act_f8(xb)
    x = X.float().numpy()
    amax = np.float32(np.abs(x).max())
    assert s_x == amax / np.float32(448.0)
    inv = np.float32(448.0) / amax
    ref = torch.from_numpy((x * inv).astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(x_f8, ref)
    assert (x_f8 & 0x7F).max() == 0x7E       # the largest |x| maps to 448
    z, sz = oracle.quantize_act_f8(np.zeros((2, 64), np.uint16))
    assert sz == 1.0 and not z.any()


def test_w4f8_gemm_exact_against_float64():
    from w4a8_bit_weight_b200 import synth
    X, W = synth.make_problem(9, 40, 512, seed=14, n_outliers=3)
    qw4, s_w = oracle.quantize_weights_w4(synth.bf16_bits(W))
    x_f8, s_x = oracle.quantize_act_f8(synth.bf16_bits(X))
    out, acc = oracle.w4f8_gemm(x_f8, s_x, qw4, s_w)
    xv = torch.from_numpy(x_f8.copy()).view(torch.float8_e4m3fn).double().numpy()
    u = np.stack([(qw4 >> (4 * h)) & 15 for h in (0, 1)], -1)            # [N, K/2, 2]: low, high nibble
    u = u.reshape(qw4.shape[0], -1, 4, 2).transpose(0, 1, 3, 2).reshape(qw4.shape[0], -1)
    q = u.astype(np.float64) - 8
    np.testing.assert_array_equal(acc, xv @ q.T)
    y = torch.from_numpy(acc.astype(np.float32)) * (torch.tensor(s_x) * torch.from_numpy(s_w))
    np.testing.assert_array_equal(out, y.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16))
    # a real approximation of the bf16 product: 7 levels per sign per channel, FP8 activations
    ref = X.double().numpy() @ W.double().numpy().T
    got = torch.from_numpy(out.view(np.int16)).view(torch.bfloat16).double().numpy()
    assert np.sqrt(np.mean((got - ref) ** 2)) < 0.35 * np.std(ref)
