"""The C ABI on the CPU: the library loads, exports every entry point declared in
include/lq.h, and rejects bad arguments before touching a device (no GPU needed)."""
import ctypes

import pytest
import torch

import w4a8_bit_weight_b200 as lq
from w4a8_bit_weight_b200 import build as lqbuild


@pytest.fixture(scope="module")
def lib():
    lqbuild.build()
    return lq.load_library()


def test_exports_every_header_symbol(lib):
    names = lq.header_symbols()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n
    assert "lq_quantize_weights" in names and "lq_quantize_act" in names and "lq_w4a8_gemm" in names


def test_version_and_status_strings(lib):
    assert lq.lq_version() >= 100
    for code in range(8):
        s = lq.lq_status_string(code)
        assert s.startswith(lq.STATUS[code])


P = ctypes.c_void_p
GOOD = P(1 << 20)      # a 16-byte aligned fake address; never dereferenced on these paths
ODD = P((1 << 20) + 8)


def gemm(lib, M=16, N=256, K=512, group=64, x=GOOD, sx=GOOD, qw=GOOD, s=GOOD, a=GOOD, sc=GOOD, out=GOOD,
         bt=0, sched=0, split=0, grid=0):
    return lib.lq_w4a8_gemm_ex(x, sx, qw, s, a, sc, out, M, N, K, group, None, 0, bt, sched, split, grid, 0,
                               None)


@pytest.mark.parametrize("kw,code", [
    (dict(group=32), 2), (dict(K=192), 2), (dict(K=64), 2), (dict(K=0), 2), (dict(K=262144), 2),
    (dict(N=8), 2), (dict(N=200), 2), (dict(N=0), 2),
    (dict(M=-1), 1), (dict(N=-16), 1),
    (dict(x=P(0)), 1), (dict(qw=P(0)), 1), (dict(s=P(0)), 1), (dict(a=P(0)), 1), (dict(out=P(0)), 1),
    (dict(sx=P(0)), 1), (dict(sc=P(0)), 1),
    (dict(x=ODD), 3), (dict(qw=ODD), 3), (dict(s=ODD), 3), (dict(a=ODD), 3), (dict(out=ODD), 3),
    (dict(sx=P((1 << 20) + 2)), 3),
    (dict(bt=48), 1), (dict(sched=6), 1), (dict(sched=-1), 1),
    (dict(sched=3, grid=-1), 1), (dict(sched=1, split=-1), 1), (dict(sched=1, split=3), 1),
    (dict(split=2), 1), (dict(grid=4), 1),        # the automatic schedule takes no split or grid
    (dict(sched=1, split=2, grid=4), 1),          # a cluster split has no grid
    (dict(sched=3, split=2, grid=4), 1),          # stream-K has no cluster split
    (dict(sched=1, bt=64, split=8), 1),           # split 8 only for tiles of <= 32 tokens
    (dict(sched=1, bt=128, split=8), 1),
    (dict(sched=1, bt=256, split=2), 1),          # 256-token tiles are never split
    (dict(sched=2, bt=64), 1),                    # the persistent schedule uses 128-token tiles
    (dict(sched=4, bt=128), 1),                   # CTA pairs use 256-token tiles
    (dict(sched=4, split=2), 1),
    (dict(sched=5), 1),
])
def test_gemm_rejects_before_launch(lib, kw, code):
    assert gemm(lib, **kw) == code


def test_gemm_empty_batch_is_a_noop(lib):
    # M == 0: nothing to do and no device touched, even with NULL buffers
    assert lib.lq_w4a8_gemm(None, None, None, None, None, None, None, 0, 256, 512, 64, None, 0, None) == 0


def test_quantize_rejects_before_launch(lib):
    q = lib.lq_quantize_weights
    assert q(GOOD, 16, 96, 64, GOOD, GOOD, GOOD, GOOD, None) == 2      # K % 64
    assert q(GOOD, 16, 128, 32, GOOD, GOOD, GOOD, GOOD, None) == 2     # group
    assert q(GOOD, 0, 128, 64, GOOD, GOOD, GOOD, GOOD, None) == 2      # N >= 1
    assert q(None, 16, 128, 64, GOOD, GOOD, GOOD, GOOD, None) == 1
    assert q(ODD, 16, 128, 64, GOOD, GOOD, GOOD, GOOD, None) == 3
    a = lib.lq_quantize_act
    assert a(GOOD, 4, 24, GOOD, GOOD, None) == 2                        # K % 16
    assert a(GOOD, -1, 64, GOOD, GOOD, None) == 1
    assert a(None, 0, 64, None, None, None) == 0                        # empty batch
    assert a(ODD, 4, 64, GOOD, GOOD, None) == 3
    d = lib.lq_dequant_weights_i8
    assert d(GOOD, GOOD, GOOD, 16, 100, 64, GOOD, None) == 2
    assert d(GOOD, GOOD, GOOD, 16, 128, 64, ODD, None) == 3


def test_workspace_size_rules(lib):
    # invalid shapes need no workspace; the query never touches a device
    assert lib.lq_w4a8_gemm_workspace_size(16, 200, 512) == 0
    assert lib.lq_w4a8_gemm_workspace_size(0, 256, 512) == 0
    # the automatic schedule and cluster splits never need a workspace
    assert lib.lq_w4a8_gemm_workspace_size(16, 4096, 4096) == 0
    assert lib.lq_w4a8_gemm_workspace_size_ex(16, 256, 512, 16, 1, 4, 0) == 0
    assert lib.lq_w4a8_gemm_workspace_size_ex(4096, 4096, 4096, 0, 2, 0, 0) == 0
    # stream-K with one CTA per tile (grid = tiles): no tile is shared, no workspace
    assert lib.lq_w4a8_gemm_workspace_size_ex(16, 256, 512, 16, 3, 0, 2) == 0
    # 3 CTAs over 2 tiles x 4 K-blocks: split tiles need [tiles][16][128] int32 + tickets
    assert lib.lq_w4a8_gemm_workspace_size_ex(16, 256, 512, 16, 3, 0, 3) == 2 * 16 * 128 * 4 + 16


def test_linear_rejects_before_launch(lib):
    f = lib.lq_w4a8_linear

    def call(M=16, N=256, K=512, group=64, X=GOOD, qw=GOOD, s=GOOD, a=GOOD, sc=GOOD, out=GOOD):
        return f(X, qw, s, a, sc, out, M, N, K, group, None, 0, None)

    assert call(group=32) == 2
    assert call(K=192) == 2
    assert call(N=200) == 2
    assert call(M=-1) == 1
    assert call(X=P(0)) == 1
    assert call(sc=P(0)) == 1
    assert call(out=P(0)) == 1
    assert call(X=ODD) == 3
    assert call(out=ODD) == 3
    assert call(sc=P((1 << 20) + 2)) == 3
    assert f(None, None, None, None, None, None, 0, 256, 512, 64, None, 0, None) == 0  # empty batch
    fx = lib.lq_w4a8_linear_ex
    assert fx(GOOD, GOOD, GOOD, GOOD, GOOD, GOOD, 16, 256, 512, 64, None, 0, 3, None) == 1   # unknown path
    assert fx(GOOD, GOOD, GOOD, GOOD, GOOD, GOOD, 16, 256, 512, 64, None, 0, -1, None) == 1


def test_linear_workspace_size_rules(lib):
    w = lib.lq_w4a8_linear_workspace_size
    wx = lib.lq_w4a8_linear_workspace_size_ex
    # small batches in split-K clusters whose CTAs preload their K-slice: one fused launch
    assert w(1, 4096, 4096) == 0
    assert w(8, 4096, 4096) == 0
    assert w(8, 2048, 4096) == 0
    # 9..16 tokens may take it too, but the automatic path uses two launches there
    assert wx(16, 4096, 4096, 2) == 0
    assert w(16, 4096, 4096) == 16 * 4096 + 64
    assert wx(4, 4096, 4096, 1) == 4 * 4096 + 16
    # otherwise two launches: x_q and s_x (16-byte aligned) carved from the workspace
    assert w(24, 4096, 4096) == 24 * 4096 + 96
    assert w(16, 256, 512) == 16 * 512 + 64
    assert w(16, 4096, 14336) == 16 * 14336 + 64
    assert w(16, 200, 512) == 0   # invalid shape
    assert wx(16, 4096, 4096, 5) == 0  # invalid path


def test_grouped_rejects_before_launch(lib):
    f = lib.lq_w4a8_grouped_gemm_ex

    def call(M=32, N=256, K=512, group=64, groups=4, x=GOOD, sx=GOOD, qw=GOOD, s=GOOD, a=GOOD, sc=GOOD,
             off=GOOD, out=GOOD, bt=0, split=0, i32=0):
        return f(x, sx, qw, s, a, sc, off, groups, out, M, N, K, group, bt, split, i32, None)

    assert call(N=192) == 2                  # a weight tile would span two groups
    assert call(N=200) == 2 and call(K=192) == 2 and call(group=32) == 2
    assert call(groups=0) == 1 and call(groups=lq.MAX_GROUPS + 1) == 1
    assert call(bt=48) == 1 and call(split=-1) == 1 and call(bt=256, split=2) == 1
    assert call(bt=256, N=128) == 2 and call(bt=256, K=384) == 2   # pairs: N % 256, K % 256
    assert call(bt=64, split=8) == 1         # split 8 only for tiles of <= 32 tokens
    assert call(off=P(0)) == 1 and call(x=P(0)) == 1 and call(sc=P(0)) == 1
    assert call(i32=1, sc=P(0), sx=P(0)) != 1  # the int32 form takes no scales (then needs a device)
    assert call(x=ODD) == 3 and call(out=ODD) == 3 and call(off=P((1 << 20) + 2)) == 3
    assert call(M=0) == 0                    # empty batch: nothing to launch
    assert call(M=-1) == 1


def test_ablation_rejects_before_launch(lib):
    f = lib.lq_w4a8_gemm_ablation

    def call(variant=0, bt=16, split=4, M=16, N=256, K=512, x=GOOD, out=GOOD):
        return f(x, GOOD, GOOD, GOOD, GOOD, GOOD, out, M, N, K, 64, variant, bt, split, 0, None)

    assert call(variant=4) == 1 and call(variant=-1) == 1
    assert call(bt=32) == 2 and call(bt=128) == 2 and call(split=2) == 2
    assert call(K=192) == 2 and call(x=ODD) == 3 and call(out=P(0)) == 1
    assert call(M=0) == 0


def _plan(lib, M, N, K, sms=148, bt=0, sched=0, split=0, grid=0):
    out = (ctypes.c_int * 4)()
    st = lib.lq_plan_gemm(M, N, K, bt, sched, split, grid, sms, out)
    return st, tuple(out)


@pytest.mark.parametrize("M,N,K,plan", [
    # (kind, token tile, CTAs per cluster, grid) on 148 SMs; kinds: 1 tiles, 2 persistent, 4 CTA pairs
    (16, 4096, 4096, (1, 16, 4, 128)),       # decode: 4-CTA clusters, one wave
    (1, 4096, 14336, (1, 32, 8, 256)),       # long K-slices: 8-CTA clusters, two CTAs per SM, as 32-token tiles
    (16, 4096, 14336, (1, 32, 8, 256)),      # the same at 16 tokens
    (32, 4096, 14336, (1, 32, 8, 256)),      # 32-token tiles in 8-CTA clusters fit two per SM (7 stages)
    (64, 4096, 14336, (1, 64, 4, 128)),      # 64-token tiles: 4-CTA clusters, one per SM
    (128, 4096, 14336, (1, 128, 4, 128)),    # 128-token tiles in 4-CTA clusters
    (256, 4096, 14336, (1, 128, 2, 128)),    # 16 pair tiles: too few for pairs; 64 tiles, 2-CTA clusters
    (16, 14336, 4096, (1, 16, 2, 224)),      # 112 tiles: 2-CTA clusters, two per SM
    (128, 14336, 4096, (2, 128, 1, 112)),    # at most 128 tokens: never pairs; 112 tiles: persistent
    (512, 4096, 14336, (2, 128, 1, 128)),    # 16 pair tiles: too few; 128 tiles cannot split K: persistent
    (256, 14336, 4096, (4, 256, 2, 112)),    # 56 pair tiles >= 148 / 4: CTA pairs
    (1024, 4096, 14336, (4, 256, 2, 128)),   # 64 pair tiles: 64 pairs
    (4096, 4096, 4096, (4, 256, 2, 148)),    # prefill: 74 persistent pairs
    (4096, 4096, 384, (2, 128, 1, 148)),     # K not a multiple of 256: persistent 128-token tiles
])
def test_automatic_schedule(lib, M, N, K, plan):
    st, got = _plan(lib, M, N, K)
    assert st == 0 and got == plan, got


B200_CLUSTER_CTAS = (296, 284, 264)  # 2-, 4-, 8-CTA clusters, two CTAs per SM, on a 148-SM B200


def _plan_ex(lib, M, N, K, cl, sms=148):
    out = (ctypes.c_int * 4)()
    arr = None if cl is None else (ctypes.c_int * 3)(*cl)
    st = lib.lq_plan_gemm_ex(M, N, K, 0, 0, 0, 0, sms, arr, out)
    return st, tuple(out)


@pytest.mark.parametrize("M,N,K,flat,placed", [
    # 34 and 36 weight tiles: 8-CTA clusters would take 272 / 288 CTAs, more than the 264
    # that B200 places at once, so the placed plan keeps 16-token tiles in 4-CTA clusters
    (16, 4352, 14336, (1, 32, 8, 272), (1, 16, 4, 136)),
    (1, 4608, 14336, (1, 32, 8, 288), (1, 16, 4, 144)),
    # 32 tiles x 8 = 256 CTAs fit one wave either way
    (16, 4096, 14336, (1, 32, 8, 256), (1, 32, 8, 256)),
    (16, 3584, 14336, (1, 32, 8, 224), (1, 32, 8, 224)),
    # 2-CTA clusters reach every SM; 4-CTA decode clusters are one CTA per SM anyway
    (16, 14336, 4096, (1, 16, 2, 224), (1, 16, 2, 224)),
    (16, 4096, 4096, (1, 16, 4, 128), (1, 16, 4, 128)),
])
def test_schedule_counts_cluster_placement(lib, M, N, K, flat, placed):
    assert _plan_ex(lib, M, N, K, None) == (0, flat)
    assert _plan(lib, M, N, K) == (0, flat)  # lq_plan_gemm: every SM reachable
    assert _plan_ex(lib, M, N, K, B200_CLUSTER_CTAS) == (0, placed)


def test_plan_ex_rejects_bad_cluster_table(lib):
    assert _plan_ex(lib, 16, 4096, 4096, (296, 0, 264))[0] == 1
    assert _plan_ex(lib, 16, 4096, 4096, (296, 284, -1))[0] == 1
    assert lib.lq_device_cluster_ctas(None) == 1


def test_cluster_table_never_exceeds_two_per_sm(lib):
    # a table larger than two CTAs per SM counts as two per SM
    for M, N, K in ((16, 4352, 14336), (16, 14336, 4096), (16, 4096, 4096)):
        assert _plan_ex(lib, M, N, K, (10 ** 6,) * 3) == _plan_ex(lib, M, N, K, None)


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the answer without a device")
def test_device_cluster_table_needs_a_device(lib):
    out = (ctypes.c_int * 3)(-7, -7, -7)
    assert lib.lq_device_cluster_ctas(out) == 5  # LQ_ERR_CUDA
    assert tuple(out) == (-7, -7, -7)


def test_plan_follows_explicit_choices(lib):
    assert _plan(lib, 16, 256, 1024, bt=16, sched=1, split=2) == (0, (1, 16, 2, 4))
    assert _plan(lib, 16, 256, 1024, bt=16, sched=3, grid=3) == (0, (3, 16, 0, 3))
    assert _plan(lib, 512, 512, 2048, sched=4, grid=2) == (0, (4, 256, 2, 2))
    assert _plan(lib, 16, 256, 1024, bt=64, sched=1, split=8)[0] == 1     # split 8 needs <= 32 tokens
    assert _plan(lib, 300, 256, 384, sched=4)[0] == 2                     # pairs need K % 256 == 0
    assert _plan(lib, 16, 4096, 4096, sms=0)[0] == 1


def test_w4f8_entry_points_reject_before_launch(lib):
    qw = lib.lq_quantize_weights_w4
    assert qw(GOOD, 16, 192 + 8, GOOD, GOOD, None) == 2      # K % 16
    assert qw(GOOD, -1, 256, GOOD, GOOD, None) == 1
    assert qw(None, 16, 256, GOOD, GOOD, None) == 1
    assert qw(ODD, 16, 256, GOOD, GOOD, None) == 3
    assert qw(None, 0, 256, None, None, None) == 0           # no rows: nothing to do
    qa = lib.lq_quantize_act_f8
    assert qa(GOOD, 4, 100, GOOD, GOOD, None) == 2
    assert qa(GOOD, 4, 256, GOOD, None, None) == 1            # s_x always written
    assert qa(ODD, 4, 256, GOOD, GOOD, None) == 3
    assert qa(GOOD, 4, 256, GOOD, P((1 << 20) + 2), None) == 3
    g = lib.lq_w4f8_gemm
    assert g(GOOD, GOOD, GOOD, GOOD, GOOD, 16, 200, 512, None) == 2   # N % 16
    assert g(GOOD, GOOD, GOOD, GOOD, GOOD, 16, 256, 192, None) == 2   # K % 128
    assert g(GOOD, None, GOOD, GOOD, GOOD, 16, 256, 512, None) == 1
    assert g(GOOD, GOOD, GOOD, GOOD, ODD, 16, 256, 512, None) == 3
    assert g(None, None, None, None, None, 0, 256, 512, None) == 0    # empty batch


def test_header_is_plain_c_and_links_from_c(lib, tmp_path):
    """include/lq.h compiles as strict C99, and a C program linked against the library
    calls it without Python (the calls used touch no device)."""
    import os
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    src = tmp_path / "use_lq.c"
    src.write_text(
        '#include <stdio.h>\n#include "lq.h"\n'
        "int main(void) {\n"
        "  int plan[4];\n"
        "  if (lq_version() < 100) return 1;\n"
        "  if (lq_plan_gemm(16, 4096, 4096, 0, LQ_SCHED_AUTO, 0, 0, 148, plan) != LQ_OK) return 2;\n"
        "  if (plan[0] != LQ_SCHED_TILES || plan[1] != 16 || plan[2] != 4) return 3;\n"
        "  if (lq_w4a8_gemm_workspace_size(16, 4096, 4096) != 0) return 4;\n"
        '  printf("%s\\n", lq_status_string(LQ_ERR_WORKSPACE));\n'
        "  return 0;\n}\n")
    libdir = os.path.join(root, "w4a8_bit_weight_b200")
    exe = tmp_path / "use_lq"
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(root, "include"),
                    str(src), "-L", libdir, "-llq_b200", "-Wl,-rpath," + libdir, "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, (r.returncode, r.stderr)
    assert r.stdout.strip().startswith(lq.STATUS[4])


def test_timeout_status_clears_cached_workspaces():
    """After LQ_ERR_TIMEOUT a stream-K call may have left partial sums in its workspace:
    the binding zeroes every cached GEMM workspace (and only those)."""
    import torch
    import w4a8_bit_weight_b200 as lq
    saved = dict(lq._ws)
    try:
        lq._ws.clear()
        gemm_ws = torch.full((64,), 7, dtype=torch.uint8)
        lin_ws = torch.full((64,), 9, dtype=torch.uint8)
        lq._ws[("gemm", 0)] = gemm_ws
        lq._ws[("linear", 0)] = lin_ws
        lq._after_device_error(0)
        assert int(gemm_ws.min()) == 7
        lq._after_device_error(lq.LQ_ERR_TIMEOUT)
        assert not gemm_ws.any()
        assert int(lin_ws.min()) == 9  # lq_w4a8_linear's front holds x_q / s_x, not sums
    finally:
        lq._ws.clear()
        lq._ws.update(saved)
