"""B200 (sm_100a) LiquidQuant W4A8 GEMM -- Python binding of the C ABI in include/lq.h.

Argument marshalling only: every step of the path runs in the CUDA library
``liblq_b200.so`` built in-tree (``python -m w4a8_bit_weight_b200.build``).
PyTorch supplies device memory and the current stream.  There is no CPU
fallback: calling any op without the built library, or on a device that is
not compute capability 10.0, raises.

Functions keep the C names:
    lq_quantize_weights(W)                       -> (qw, s_u8, a_u8, s_c)
    lq_quantize_act(X)                           -> (x_q, s_x)
    lq_w4a8_gemm(x_q, s_x, qw, s_u8, a_u8, s_c)  -> out bf16 [M, N]
    lq_w4a8_gemm_i32(x_q, qw, s_u8, a_u8)        -> acc int32 [M, N]
    lq_dequant_weights_i8(qw, s_u8, a_u8)        -> w_i8 int8 [N, K]
"""
from __future__ import annotations

import ctypes
import os
import re
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblq_b200.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "lq.h")
GROUP = 64
MAX_GROUPS = 1024  # LQ_MAX_GROUPS in lq.h
SCHED_AUTO, SCHED_TILES, SCHED_PERSISTENT, SCHED_STREAMK, SCHED_PAIR = 0, 1, 2, 3, 4

STATUS = {
    0: "LQ_OK", 1: "LQ_ERR_INVALID_ARG", 2: "LQ_ERR_UNSUPPORTED_SHAPE", 3: "LQ_ERR_MISALIGNED",
    4: "LQ_ERR_WORKSPACE", 5: "LQ_ERR_CUDA", 6: "LQ_ERR_TIMEOUT", 7: "LQ_ERR_ARCH",
}


class LQError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn}: {STATUS.get(status, status)}")


_lib = None
_lock = threading.Lock()


def load_library(path: str = LIB_PATH):
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(path):
            raise RuntimeError(f"CUDA library not built: {path} is missing "
                               "(run python -m w4a8_bit_weight_b200.build)")
        lib = ctypes.CDLL(path)
        P, I, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        sig = {
            "lq_version": ([], I),
            "lq_device_addressable": ([P], I),
            "lq_status_string": ([I], ctypes.c_char_p),
            "lq_quantize_weights": ([P, I, I, I, P, P, P, P, P], I),
            "lq_quantize_act": ([P, I, I, P, P, P], I),
            "lq_w4a8_gemm_workspace_size": ([I, I, I], Z),
            "lq_w4a8_gemm_workspace_size_ex": ([I, I, I, I, I, I, I], Z),
            "lq_w4a8_gemm": ([P, P, P, P, P, P, P, I, I, I, I, P, Z, P], I),
            "lq_w4a8_gemm_ex": ([P, P, P, P, P, P, P, I, I, I, I, P, Z, I, I, I, I, I, P], I),
            "lq_w4a8_gemm_i32": ([P, P, P, P, P, I, I, I, I, P, Z, P], I),
            "lq_w4a8_gemm_swiglu": ([P, P, P, P, P, P, P, I, I, I, I, P, Z, P], I),
            "lq_w4a8_gemm_swiglu_ex": ([P, P, P, P, P, P, P, I, I, I, I, P, Z, I, I, I, I, P], I),
            "lq_dequant_weights_i8": ([P, P, P, I, I, I, P, P], I),
            "lq_get_device_error": ([P], I),
            "lq_w4a8_gemm_noalloc": ([P, P, P, P, P, P, P, I, I, I, I, P], I),
            "lq_w4a8_linear_workspace_size": ([I, I, I], Z),
            "lq_w4a8_linear": ([P, P, P, P, P, P, I, I, I, I, P, Z, P], I),
            "lq_w4a8_linear_workspace_size_ex": ([I, I, I, I], Z),
            "lq_w4a8_linear_ex": ([P, P, P, P, P, P, I, I, I, I, P, Z, I, P], I),
            "lq_w4a8_grouped_gemm": ([P, P, P, P, P, P, P, I, P, I, I, I, I, P], I),
            "lq_w4a8_gemm_ablation": ([P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, P], I),
            "lq_test_wait_timeout": ([P], I),
            "lq_plan_gemm": ([I, I, I, I, I, I, I, I, P], I),
            "lq_plan_gemm_ex": ([I, I, I, I, I, I, I, I, P, P], I),
            "lq_device_cluster_ctas": ([P], I),
            "lq_quantize_weights_w4": ([P, I, I, P, P, P], I),
            "lq_quantize_act_f8": ([P, I, I, P, P, P], I),
            "lq_w4f8_gemm": ([P, P, P, P, P, I, I, I, P], I),
            "lq_w4a8_grouped_gemm_ex": ([P, P, P, P, P, P, P, I, P, I, I, I, I, I, I, I, P], I),
        }
        for name, (args, res) in sig.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = res
        _lib = lib
        return lib


def header_symbols(path: str = HEADER_PATH):
    """Names of the entry points declared in include/lq.h."""
    with open(path) as f:
        text = f.read()
    return sorted(set(re.findall(r"^LQ_API\s+[\w\s\*]+?\b(lq_\w+)\s*\(", text, re.M)))


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _check(fn: str, st: int):
    if st != 0:
        raise LQError(fn, st)


def _need(t: torch.Tensor, dtype, name: str, shape=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _need_io(t: torch.Tensor, dtype, name: str, shape=None):
    """_need, except that a pinned host tensor is accepted too: activations read and
    outputs written by the kernels directly over the host link (zero-copy I/O, lq.h)."""
    if isinstance(t, torch.Tensor) and not t.is_cuda and t.is_pinned():
        if t.dtype != dtype:
            raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        if shape is not None and tuple(t.shape) != tuple(shape):
            raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
        return
    _need(t, dtype, name, shape)


def _cuda_device(t: torch.Tensor) -> torch.device:
    """The device a call runs on: the tensor's, or the current one for a pinned host tensor."""
    return t.device if t.is_cuda else torch.device("cuda", torch.cuda.current_device())


def lq_device_addressable(t: torch.Tensor) -> bool:
    """Whether the current device reads and writes t's memory at its address (lq.h)."""
    return bool(load_library().lq_device_addressable(_ptr(t)))


# ----------------------------------------------------------------------------
# workspace: one zero-filled scratch buffer per device, grown on demand.  The
# kernels leave it zero-filled after every call, so it is cleared only once.
# ----------------------------------------------------------------------------
_ws = {}


def workspace(nbytes: int, device, kind: str = "gemm") -> torch.Tensor | None:
    """kind "gemm": the GEMM's zero-filled scratch; kind "linear": lq_w4a8_linear's,
    whose front holds x_q and s_x (so it is never zero there) -- kept apart."""
    if nbytes == 0:
        return None
    dev = torch.device(device)
    key = (kind, dev.index if dev.index is not None else torch.cuda.current_device())
    buf = _ws.get(key)
    if buf is None or buf.numel() < nbytes:
        buf = torch.zeros(max(nbytes, 1 << 20), dtype=torch.uint8, device=dev)
        _ws[key] = buf
    return buf


def lq_version() -> int:
    return load_library().lq_version()


def lq_status_string(status: int) -> str:
    return load_library().lq_status_string(status).decode()


def lq_quantize_weights(W: torch.Tensor, group: int = GROUP, out=None):
    """Offline LiquidQuant of W [N, K] bf16 -> (qw [N,K/2] u8, s_u8 [K/64,N] u8, a_u8 [K/64,N] u8, s_c [N] f32)."""
    lib = load_library()
    _need(W, torch.bfloat16, "W")
    N, K = W.shape
    dev = W.device
    if out is None:
        out = (torch.empty(N, K // 2, dtype=torch.uint8, device=dev),
               torch.empty(max(K // group, 0), N, dtype=torch.uint8, device=dev),
               torch.empty(max(K // group, 0), N, dtype=torch.uint8, device=dev),
               torch.empty(N, dtype=torch.float32, device=dev))
    qw, s, a, sc = out
    with torch.cuda.device(dev):
        _check("lq_quantize_weights", lib.lq_quantize_weights(
            _ptr(W), N, K, group, _ptr(qw), _ptr(s), _ptr(a), _ptr(sc), _stream(dev)))
    return qw, s, a, sc


def lq_quantize_act(X: torch.Tensor, out=None):
    """Per-token symmetric INT8 of X [M, K] bf16 -> (x_q [M,K] int8, s_x [M] f32).
    X may be a pinned host tensor (read over the host link)."""
    lib = load_library()
    _need_io(X, torch.bfloat16, "X")
    M, K = X.shape
    dev = _cuda_device(X)
    if out is None:
        out = (torch.empty(M, K, dtype=torch.int8, device=dev),
               torch.empty(M, dtype=torch.float32, device=dev))
    xq, sx = out
    with torch.cuda.device(dev):
        _check("lq_quantize_act", lib.lq_quantize_act(_ptr(X), M, K, _ptr(xq), _ptr(sx), _stream(dev)))
    return xq, sx


def _sched(schedule, split_k, grid):
    """Default the schedule from the other knobs (split_k -> tiles, grid -> stream-K)."""
    if schedule is not None:
        return schedule
    if grid:
        return SCHED_STREAMK
    if split_k:
        return SCHED_TILES
    return SCHED_AUTO


def lq_w4a8_gemm_workspace_size(M: int, N: int, K: int, block_t: int = 0, split_k: int = 0,
                                grid: int = 0, schedule: int | None = None) -> int:
    lib = load_library()
    sch = _sched(schedule, split_k, grid)
    if block_t == 0 and split_k == 0 and grid == 0 and sch == SCHED_AUTO:
        return int(lib.lq_w4a8_gemm_workspace_size(M, N, K))
    return int(lib.lq_w4a8_gemm_workspace_size_ex(M, N, K, block_t, sch, split_k, grid))


def _gemm(x_q, s_x, qw, s_u8, a_u8, s_c, out, group, block_t, split_k, grid, out_i32, ws, schedule=None):
    lib = load_library()
    _need(x_q, torch.int8, "x_q")
    M, K = x_q.shape
    N = qw.shape[0]
    _need(qw, torch.uint8, "qw", (N, K // 2))
    _need(s_u8, torch.uint8, "s_u8", (K // group, N))
    _need(a_u8, torch.uint8, "a_u8", (K // group, N))
    if not out_i32:
        _need(s_x, torch.float32, "s_x", (M,))
        _need(s_c, torch.float32, "s_c", (N,))
    odt = torch.int32 if out_i32 else torch.bfloat16
    if out is None:
        out = torch.empty(M, N, dtype=odt, device=x_q.device)
    _need_io(out, odt, "out", (M, N))
    with torch.cuda.device(x_q.device):
        sch = _sched(schedule, split_k, grid)
        need = lq_w4a8_gemm_workspace_size(M, N, K, block_t, split_k, grid, sch)
        if ws is None:
            ws = workspace(need, x_q.device)
        nbytes = ws.numel() * ws.element_size() if ws is not None else 0
        _check("lq_w4a8_gemm", lib.lq_w4a8_gemm_ex(
            _ptr(x_q), _ptr(s_x), _ptr(qw), _ptr(s_u8), _ptr(a_u8), _ptr(s_c), _ptr(out),
            M, N, K, group, _ptr(ws), nbytes, block_t, sch, split_k, grid, 1 if out_i32 else 0,
            _stream(x_q.device)))
    return out


def lq_w4a8_gemm(x_q, s_x, qw, s_u8, a_u8, s_c, out=None, group: int = GROUP,
                 block_t: int = 0, split_k: int = 0, grid: int = 0, workspace_buf=None,
                 schedule: int | None = None):
    """W4A8 GEMM: bf16(float(x_q @ dequant(qw)^T) * s_x[m] * s_c[n]) -> [M, N] bf16.

    block_t / schedule / split_k / grid override the automatic schedule (lq_w4a8_gemm_ex in lq.h)."""
    return _gemm(x_q, s_x, qw, s_u8, a_u8, s_c, out, group, block_t, split_k, grid, False, workspace_buf,
                 schedule)


def lq_w4a8_gemm_i32(x_q, qw, s_u8, a_u8, out=None, group: int = GROUP, block_t: int = 0,
                     split_k: int = 0, grid: int = 0, workspace_buf=None, schedule: int | None = None):
    """The int32 accumulators x_q @ dequant(qw)^T -> [M, N] int32."""
    return _gemm(x_q, None, qw, s_u8, a_u8, None, out, group, block_t, split_k, grid, True, workspace_buf,
                 schedule)


def lq_w4a8_gemm_swiglu(x_q, s_x, qw, s_u8, a_u8, s_c, out=None, group: int = GROUP, workspace_buf=None,
                        block_t: int = 0, split_k: int = 0, schedule: int | None = None):
    """Gate/up pair of a gated FFN layer in one GEMM: the weights are one interleaved
    [2F, K] matrix (row 2j gate channel j, row 2j+1 up channel j), the output
    bf16(silu(gate) * up) -> [M, F] bf16 (lq_w4a8_gemm_swiglu in lq.h)."""
    lib = load_library()
    _need(x_q, torch.int8, "x_q")
    M, K = x_q.shape
    N = qw.shape[0]
    _need(qw, torch.uint8, "qw", (N, K // 2))
    _need(s_u8, torch.uint8, "s_u8", (K // group, N))
    _need(a_u8, torch.uint8, "a_u8", (K // group, N))
    _need(s_x, torch.float32, "s_x", (M,))
    _need(s_c, torch.float32, "s_c", (N,))
    if N % 2:
        raise ValueError("the gate/up weights come in row pairs")
    if out is None:
        out = torch.empty(M, N // 2, dtype=torch.bfloat16, device=x_q.device)
    _need_io(out, torch.bfloat16, "out", (M, N // 2))
    with torch.cuda.device(x_q.device):
        ws = workspace_buf
        sch = _sched(schedule, split_k, 0)
        if ws is None:
            ws = workspace(lq_w4a8_gemm_workspace_size(M, N, K, block_t, split_k, 0, sch), x_q.device)
        nbytes = ws.numel() * ws.element_size() if ws is not None else 0
        _check("lq_w4a8_gemm_swiglu", lib.lq_w4a8_gemm_swiglu_ex(
            _ptr(x_q), _ptr(s_x), _ptr(qw), _ptr(s_u8), _ptr(a_u8), _ptr(s_c), _ptr(out), M, N, K, group,
            _ptr(ws), nbytes, block_t, sch, split_k, 0, _stream(x_q.device)))
    return out


# paths of lq_w4a8_linear (LQ_LINEAR_* in lq.h)
LINEAR_AUTO, LINEAR_TWO_LAUNCHES, LINEAR_FUSED = 0, 1, 2


def lq_w4a8_linear_workspace_size(M: int, N: int, K: int, path: int = LINEAR_AUTO) -> int:
    return int(load_library().lq_w4a8_linear_workspace_size_ex(M, N, K, path))


def lq_w4a8_linear(X, qw, s_u8, a_u8, s_c, out=None, group: int = GROUP, workspace_buf=None,
                   path: int = LINEAR_AUTO):
    """Activation quantization + W4A8 GEMM in one call: bf16 X [M, K] -> [M, N] bf16,
    bit-identical to lq_w4a8_gemm(*lq_quantize_act(X), ...).  One fused launch for
    small decode batches, two launches otherwise (lq_w4a8_linear in lq.h); `path`
    forces one of them (LINEAR_*)."""
    lib = load_library()
    _need_io(X, torch.bfloat16, "X")
    M, K = X.shape
    N = qw.shape[0]
    _need(qw, torch.uint8, "qw", (N, K // 2))
    _need(s_u8, torch.uint8, "s_u8", (K // group, N))
    _need(a_u8, torch.uint8, "a_u8", (K // group, N))
    _need(s_c, torch.float32, "s_c", (N,))
    dev = qw.device
    if out is None:
        out = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    _need_io(out, torch.bfloat16, "out", (M, N))
    with torch.cuda.device(dev):
        ws = workspace_buf
        if ws is None:
            ws = workspace(lq_w4a8_linear_workspace_size(M, N, K, path), dev, kind="linear")
        nbytes = ws.numel() * ws.element_size() if ws is not None else 0
        _check("lq_w4a8_linear", lib.lq_w4a8_linear_ex(
            _ptr(X), _ptr(qw), _ptr(s_u8), _ptr(a_u8), _ptr(s_c), _ptr(out), M, N, K, group,
            _ptr(ws), nbytes, path, _stream(dev)))
    return out


def lq_w4a8_gemm_noalloc(x_q, s_x, qw, s_u8, a_u8, s_c, out=None, group: int = GROUP):
    """lq_w4a8_gemm without a workspace, for callers that may not allocate device memory
    where they launch the GEMM; its scratch is a fixed 4 MiB array inside the library.
    Calls on one device share that array and must not overlap on the GPU."""
    lib = load_library()
    _need(x_q, torch.int8, "x_q")
    M, K = x_q.shape
    N = qw.shape[0]
    _need(qw, torch.uint8, "qw", (N, K // 2))
    _need(s_u8, torch.uint8, "s_u8", (K // group, N))
    _need(a_u8, torch.uint8, "a_u8", (K // group, N))
    _need(s_x, torch.float32, "s_x", (M,))
    _need(s_c, torch.float32, "s_c", (N,))
    if out is None:
        out = torch.empty(M, N, dtype=torch.bfloat16, device=x_q.device)
    _need_io(out, torch.bfloat16, "out", (M, N))
    with torch.cuda.device(x_q.device):
        _check("lq_w4a8_gemm_noalloc", lib.lq_w4a8_gemm_noalloc(
            _ptr(x_q), _ptr(s_x), _ptr(qw), _ptr(s_u8), _ptr(a_u8), _ptr(s_c), _ptr(out),
            M, N, K, group, _stream(x_q.device)))
    return out


def lq_w4a8_grouped_gemm(x_q, s_x, qw, s_u8, a_u8, s_c, m_off, N: int, out=None, group: int = GROUP,
                         block_t: int = 0, split_k: int = 0, out_i32: bool = False):
    """Grouped W4A8 GEMM (mixture-of-experts layer): rows [m_off[e], m_off[e+1]) of x_q times
    weight rows [e*N, (e+1)*N) of the stacked quantized weights -> [M, N] bf16 (int32 with out_i32).

    m_off is a device int32 tensor of groups + 1 non-decreasing row offsets (0 ... M)."""
    lib = load_library()
    _need(x_q, torch.int8, "x_q")
    M, K = x_q.shape
    _need(m_off, torch.int32, "m_off")
    if m_off.dim() != 1 or m_off.numel() < 2:
        raise ValueError("m_off must hold groups + 1 >= 2 offsets")
    G = m_off.numel() - 1
    _need(qw, torch.uint8, "qw", (G * N, K // 2))
    _need(s_u8, torch.uint8, "s_u8", (K // group, G * N))
    _need(a_u8, torch.uint8, "a_u8", (K // group, G * N))
    if not out_i32:
        _need(s_x, torch.float32, "s_x", (M,))
        _need(s_c, torch.float32, "s_c", (G * N,))
    odt = torch.int32 if out_i32 else torch.bfloat16
    if out is None:
        out = torch.empty(M, N, dtype=odt, device=x_q.device)
    _need_io(out, odt, "out", (M, N))
    with torch.cuda.device(x_q.device):
        _check("lq_w4a8_grouped_gemm", lib.lq_w4a8_grouped_gemm_ex(
            _ptr(x_q), _ptr(s_x), _ptr(qw), _ptr(s_u8), _ptr(a_u8), _ptr(s_c), _ptr(m_off), G, _ptr(out),
            M, N, K, group, block_t, split_k, 1 if out_i32 else 0, _stream(x_q.device)))
    return out


# variants of lq_w4a8_gemm_ablation (LQ_ABL_* in lq.h)
ABL_IMPLICIT, ABL_NAIVE, ABL_EXPLICIT, ABL_NAIVE_EXPLICIT = 0, 1, 2, 3


def lq_w4a8_gemm_ablation(x_q, s_x, qw, s_u8, a_u8, s_c, variant: int, block_t: int, split_k: int = 4,
                          out=None, group: int = GROUP, out_i32: bool = False):
    """Test and measurement only: the GEMM with the dequantization arithmetic and pipeline
    of one ablation variant (ABL_*), 16- or 64-token tiles in 4-CTA clusters."""
    lib = load_library()
    _need(x_q, torch.int8, "x_q")
    M, K = x_q.shape
    N = qw.shape[0]
    _need(qw, torch.uint8, "qw", (N, K // 2))
    if not out_i32:
        _need(s_x, torch.float32, "s_x", (M,))
        _need(s_c, torch.float32, "s_c", (N,))
    odt = torch.int32 if out_i32 else torch.bfloat16
    if out is None:
        out = torch.empty(M, N, dtype=odt, device=x_q.device)
    _need_io(out, odt, "out", (M, N))
    with torch.cuda.device(x_q.device):
        _check("lq_w4a8_gemm_ablation", lib.lq_w4a8_gemm_ablation(
            _ptr(x_q), _ptr(s_x), _ptr(qw), _ptr(s_u8), _ptr(a_u8), _ptr(s_c), _ptr(out), M, N, K, group,
            variant, block_t, split_k, 1 if out_i32 else 0, _stream(x_q.device)))
    return out


def lq_dequant_weights_i8(qw, s_u8, a_u8, group: int = GROUP, out=None):
    """LiquidQuant expansion written out: int8((q*s + a) XOR 0x80) -> [N, K] int8."""
    lib = load_library()
    N, K = qw.shape[0], qw.shape[1] * 2
    _need(qw, torch.uint8, "qw")
    _need(s_u8, torch.uint8, "s_u8", (K // group, N))
    _need(a_u8, torch.uint8, "a_u8", (K // group, N))
    if out is None:
        out = torch.empty(N, K, dtype=torch.int8, device=qw.device)
    with torch.cuda.device(qw.device):
        _check("lq_dequant_weights_i8", lib.lq_dequant_weights_i8(
            _ptr(qw), _ptr(s_u8), _ptr(a_u8), N, K, group, _ptr(out), _stream(qw.device)))
    return out


def lq_quantize_weights_w4(W: torch.Tensor, out=None):
    """W4 x FP8 variant: per-channel symmetric INT4 weights -> (qw4 [N, K/2] uint8, s_w [N] fp32)."""
    lib = load_library()
    _need(W, torch.bfloat16, "W")
    N, K = W.shape
    qw4, s_w = out if out is not None else (torch.empty(N, K // 2, dtype=torch.uint8, device=W.device),
                                            torch.empty(N, dtype=torch.float32, device=W.device))
    with torch.cuda.device(W.device):
        _check("lq_quantize_weights_w4", lib.lq_quantize_weights_w4(_ptr(W), N, K, _ptr(qw4), _ptr(s_w),
                                                                    _stream(W.device)))
    return qw4, s_w


def lq_quantize_act_f8(X: torch.Tensor, out=None):
    """W4 x FP8 variant: e4m3 codes with one scale for the tensor -> (x_f8 [M, K] uint8, s_x [1] fp32)."""
    lib = load_library()
    _need_io(X, torch.bfloat16, "X")
    M, K = X.shape
    dev = _cuda_device(X)
    x_f8, s_x = out if out is not None else (torch.empty(M, K, dtype=torch.uint8, device=dev),
                                             torch.empty(1, dtype=torch.float32, device=dev))
    with torch.cuda.device(dev):
        _check("lq_quantize_act_f8", lib.lq_quantize_act_f8(_ptr(X), M, K, _ptr(x_f8), _ptr(s_x),
                                                            _stream(dev)))
    return x_f8, s_x


def lq_w4f8_gemm(x_f8, s_x, qw4, s_w, out=None):
    """W4 x FP8 GEMM: bf16(fp32 sum_k e4m3(x) * q * s_x * s_w[n]) -> [M, N] bf16."""
    lib = load_library()
    _need(x_f8, torch.uint8, "x_f8")
    M, K = x_f8.shape
    N = qw4.shape[0]
    _need(qw4, torch.uint8, "qw4", (N, K // 2))
    _need(s_x, torch.float32, "s_x", (1,))
    _need(s_w, torch.float32, "s_w", (N,))
    if out is None:
        out = torch.empty(M, N, dtype=torch.bfloat16, device=x_f8.device)
    _need_io(out, torch.bfloat16, "out", (M, N))
    with torch.cuda.device(x_f8.device):
        _check("lq_w4f8_gemm", lib.lq_w4f8_gemm(_ptr(x_f8), _ptr(s_x), _ptr(qw4), _ptr(s_w), _ptr(out), M, N, K,
                                                _stream(x_f8.device)))
    return out


def lq_test_wait_timeout(device=None) -> None:
    """Test only: a kernel whose bounded waits run out (about 2 s); see lq.h."""
    lib = load_library()
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(dev):
        _check("lq_test_wait_timeout", lib.lq_test_wait_timeout(_stream(dev)))


LQ_ERR_TIMEOUT = 6


def _after_device_error(status: int) -> None:
    """A kernel that gave up a wait (LQ_ERR_TIMEOUT) may have left partial sums
    and tile tickets in a stream-K workspace, which the kernels otherwise restore
    to zero: clear every cached GEMM workspace so that later calls start clean."""
    if status == LQ_ERR_TIMEOUT:
        for (kind, _), buf in _ws.items():
            if kind == "gemm":
                buf.zero_()


def lq_get_device_error(device=None) -> int:
    """Synchronizes the current stream; returns and clears the library's device error status.
    After LQ_ERR_TIMEOUT the cached GEMM workspaces are cleared again (see _after_device_error)."""
    lib = load_library()
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    with torch.cuda.device(dev):
        status = int(lib.lq_get_device_error(_stream(dev)))
        _after_device_error(status)
        return status


class W4A8Linear:
    """A linear layer y = x W^T with LiquidQuant W4A8 weights, quantized once at construction."""

    def __init__(self, weight: torch.Tensor):
        self.N, self.K = weight.shape
        self.qw, self.s_u8, self.a_u8, self.s_c = lq_quantize_weights(weight.contiguous())

    def __call__(self, x: torch.Tensor) -> torch.Tensor:
        x_q, s_x = lq_quantize_act(x.contiguous())
        return lq_w4a8_gemm(x_q, s_x, self.qw, self.s_u8, self.a_u8, self.s_c)
