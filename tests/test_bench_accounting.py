"""The bench's algorithmic byte and op counts (CPU): the closed forms for the
workloads' layers, cross-checked against an element-by-element count of the
tensors each pass reads and writes."""
import bench
from w4a8_bit_weight_b200 import synth


def _count(M, N, K, G=64, activations_bf16=False):
    # packed u4 weights + u8 scales and offsets + fp32 channel scales
    w = N * K // 2 + 2 * (K // G) * N + 4 * N
    if activations_bf16:
        x = 2 * M * K                      # bf16 activations in
    else:
        x = M * K + 4 * M                  # int8 codes + fp32 token scales
    return w + x + 2 * M * N               # bf16 out


def test_gemm_and_linear_bytes():
    for (M, N, K) in [(1, 4096, 4096), (16, 4096, 4096), (4096, 4096, 4096), (256, 14336, 4096),
                      (8192, 4096, 14336), (16, 256, 512)]:
        assert bench.gemm_bytes(M, N, K) == _count(M, N, K)
        assert bench.linear_bytes(M, N, K) == _count(M, N, K, activations_bf16=True)
    # the decode layer's GEMM bytes as the bench reports them (8.94 / 8.98 / 9.13 MB)
    assert [bench.gemm_bytes(M, 4096, 4096) for M in (1, 4, 16)] == [8941572, 8978448, 9125952]
    assert bench.gemm_bytes(4096, 4096, 4096) == 59277312


def test_step_accounting_sums_the_workload_batches():
    for name in ("decode", "prefill", "mlp_up", "tiny"):
        w = synth.WORKLOADS[name]
        gb, ab, ops = bench.step_accounting(w)
        assert ab == 0
        assert gb == sum(_count(M, w.N, w.K, activations_bf16=True) for M in w.Ms)
        assert ops == sum(2 * M * w.N * w.K for M in w.Ms)
