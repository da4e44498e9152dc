"""Python binding of libgptq_w4a16.so (ctypes; argument marshalling only).

Every step of the layer runs in the library's CUDA kernels.  PyTorch supplies
device memory and the current stream; this module checks tensor dtypes and
devices, passes raw pointers, and turns status codes into exceptions.  There is
no CPU path: if the library is missing or the device is not sm_100, calls
raise.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "_lib", "libgptq_w4a16.so")

KERNEL_AUTO, KERNEL_DECODE, KERNEL_PREFILL = 0, 1, 2
DECODE_MAX_M = 64
LORA_DECODE_MAX_M = 32
MAX_GROUPED = 8
MAX_LORA_RANK = 256
LORA_SCRATCH_BYTES = 8 << 20
GIDX_MAX_GROUPS = 640
GROUP_SIZES = (-1, 16, 32, 64, 128, 256, 512, 1024)

STATUS = {0: "GPTQ_OK", 1: "GPTQ_ERR_NULL", 2: "GPTQ_ERR_SHAPE", 3: "GPTQ_ERR_GROUP",
          4: "GPTQ_ERR_ALIGN", 5: "GPTQ_ERR_DEVICE", 6: "GPTQ_ERR_CUDA",
          7: "GPTQ_ERR_TIMEOUT", 8: "GPTQ_ERR_ALIAS", 9: "GPTQ_ERR_KERNEL",
          10: "GPTQ_ERR_INDEX"}

# Every entry point declared in include/gptq_w4a16.h.
EXPORTS = ("gptq_w4a16_gemm", "gptq_w4a16_gemm_kernel", "gptq_w4a16_gemm_decode_splits",
           "gptq_w4a16_gemm_grouped", "gptq_w4a16_gemm_asym", "gptq_w4a16_gemm_gidx",
           "gptq_w4a16_gemm_lora", "gptq_w4a16_gemm_lora_noalloc",
           "gptq_dequant",
           "gptq_w4a16_select", "gptq_status_string", "gptq_device_error", "gptq_version")


class GptqError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status


_lock = threading.Lock()
_lib = None

_p = ctypes.c_void_p
_i64 = ctypes.c_int64
_i32 = ctypes.c_int32


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the library once (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(path):
                raise RuntimeError(
                    f"CUDA library not built: {path} is missing "
                    "(run `python -m int4_weight_only_gptq_b200.build`)")
            lib = ctypes.CDLL(path)
            gemm_args = [_p, _p, _p, _i64, _i64, _i64, _i32, _p, _p]
            lib.gptq_w4a16_gemm.argtypes = gemm_args
            lib.gptq_w4a16_gemm_kernel.argtypes = gemm_args + [_i32]
            lib.gptq_w4a16_gemm_decode_splits.argtypes = gemm_args + [_i32]
            lib.gptq_w4a16_gemm_grouped.argtypes = [_p, _p, _p, _p, _i32, _i64, _i64, _i32,
                                                    _p, _p]
            lib.gptq_w4a16_gemm_lora.argtypes = [_p, _p, _p, _i64, _i64, _i64, _i32, _p, _p,
                                                 _i64, _p, _p, _p]
            lib.gptq_w4a16_gemm_asym.argtypes = [_p, _p, _p, _p, _i64, _i64, _i64, _i32, _p, _p]
            lib.gptq_w4a16_gemm_gidx.argtypes = [_p, _p, _p, _p, _i64, _i64, _i64, _i64, _p, _p]
            lib.gptq_w4a16_gemm_lora_noalloc.argtypes = [_p, _p, _p, _i64, _i64, _i64, _i32,
                                                         _p, _p, _i64, _p, _p]
            lib.gptq_dequant.argtypes = [_p, _p, _i64, _i64, _i32, _p, _p]
            lib.gptq_w4a16_select.argtypes = [_i64, _i64, _i64, _i32,
                                              ctypes.POINTER(_i32), ctypes.POINTER(_i32)]
            lib.gptq_status_string.restype = ctypes.c_char_p
            lib.gptq_status_string.argtypes = [ctypes.c_int]
            lib.gptq_device_error.argtypes = []
            lib.gptq_version.restype = ctypes.c_char_p
            for name in ("gptq_w4a16_gemm", "gptq_w4a16_gemm_kernel",
                         "gptq_w4a16_gemm_decode_splits", "gptq_w4a16_gemm_grouped",
                         "gptq_w4a16_gemm_asym", "gptq_w4a16_gemm_gidx", "gptq_w4a16_gemm_lora",
                         "gptq_w4a16_gemm_lora_noalloc",
                         "gptq_dequant",
                         "gptq_w4a16_select", "gptq_device_error"):
                getattr(lib, name).restype = ctypes.c_int
            _lib = lib
    return _lib


def status_string(status: int) -> str:
    return load().gptq_status_string(int(status)).decode()


def _check(status: int):
    if status != 0:
        raise GptqError(status, status_string(status))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream, device):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _as_bits16(t: torch.Tensor) -> torch.Tensor:
    if t.dtype == torch.float16:
        return t
    if t.dtype in (torch.int16, torch.uint16):
        return t
    raise TypeError(f"expected a float16 tensor, got {t.dtype}")


def _require(t: torch.Tensor, name: str, dtype_ok, device):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous (row-major)")
    if not dtype_ok(t.dtype):
        raise TypeError(f"{name} has dtype {t.dtype}")


def n_groups(K: int, group: int) -> int:
    """Scale rows of a layer: one for group -1 or a group of K or more, else
    ceil(K / group) (a ragged last group when group does not divide K)."""
    return 1 if group == -1 or group >= K else -(-K // group)


def layer_shapes(x, qweight, scales, group: int) -> tuple[int, int, int]:
    """(M, K, N) of a layer call, after checking that x [M, K], qweight
    [K/8, N] and scales [n_groups(K, group), N] agree.  The C ABI sees only
    pointers and the sizes it is given, and builds its tensor maps from them,
    so a tensor smaller than those sizes would be read past its end: the
    shapes are checked here, before the library is called.  An unsupported
    group is left to the library (GPTQ_ERR_GROUP)."""
    if x.dim() != 2 or qweight.dim() != 2 or scales.dim() != 2:
        raise ValueError("x, qweight and scales must be 2-D")
    M, K = (int(v) for v in x.shape)
    N = int(qweight.shape[1])
    if int(qweight.shape[0]) * 8 != K:
        raise ValueError(f"qweight rows {qweight.shape[0]} do not match K={K}")
    if group in GROUP_SIZES and K > 0:
        want = (n_groups(K, group), N)
        if tuple(scales.shape) != want:
            raise ValueError(f"scales has shape {tuple(scales.shape)}, expected {want} "
                             f"for K={K}, group={group}")
    return M, K, N


def adapter_shapes(lora_a, lora_b, K: int, N: int) -> int:
    """The adapter's rank, after checking lora_a [rank, K] and lora_b [N, rank]."""
    if lora_a.dim() != 2 or lora_b.dim() != 2:
        raise ValueError("lora_a and lora_b must be 2-D")
    rank = int(lora_a.shape[0])
    if int(lora_a.shape[1]) != K:
        raise ValueError(f"lora_a has shape {tuple(lora_a.shape)}, expected ({rank}, {K})")
    if tuple(lora_b.shape) != (N, rank):
        raise ValueError(f"lora_b has shape {tuple(lora_b.shape)}, expected {(N, rank)}")
    return rank


def _check_shape(t, name: str, shape: tuple):
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def gemm(x: torch.Tensor, qweight: torch.Tensor, scales: torch.Tensor, group: int,
         out: torch.Tensor | None = None, stream=None, kernel: int = KERNEL_AUTO,
         decode_splits: int = 0) -> torch.Tensor:
    """Y[M, N] = x[M, K] . dequant(qweight[K/8, N], scales[n_groups, N]) (FP16)."""
    lib = load()
    dev = qweight.device
    _require(qweight, "qweight", lambda d: d == torch.int32, None)
    _require(scales, "scales", lambda d: d == torch.float16, dev)
    _require(x, "x", lambda d: d == torch.float16, dev)
    M, K, N = layer_shapes(x, qweight, scales, group)
    if out is None:
        out = torch.empty((M, N), dtype=torch.float16, device=dev)
    else:
        _require(out, "out", lambda d: d == torch.float16, dev)
        _check_shape(out, "out", (M, N))
    s = _stream_handle(stream, dev)
    args = (_ptr(x), _ptr(qweight), _ptr(scales), M, K, N, group, _ptr(out), s)
    with torch.cuda.device(dev):  # the library works on the current device
        if decode_splits:
            _check(lib.gptq_w4a16_gemm_decode_splits(*args, decode_splits))
        elif kernel == KERNEL_AUTO:
            _check(lib.gptq_w4a16_gemm(*args))
        else:
            _check(lib.gptq_w4a16_gemm_kernel(*args, kernel))
    return out


def gemm_grouped(x: torch.Tensor, qweights, scales, group: int, outs=None,
                 stream=None) -> list:
    """Y_i = x . dequant(qweights[i], scales[i]) for linears sharing x (one
    decode launch for M <= DECODE_MAX_M)."""
    lib = load()
    if not 1 <= len(qweights) <= MAX_GROUPED or len(scales) != len(qweights):
        raise ValueError(f"need 1..{MAX_GROUPED} linears with one scales tensor each")
    dev = qweights[0].device
    _require(x, "x", lambda d: d == torch.float16, dev)
    if x.dim() != 2:
        raise ValueError("x must be 2-D")
    M, K = x.shape
    Ns = []
    for i, (qw, sc) in enumerate(zip(qweights, scales)):
        _require(qw, f"qweights[{i}]", lambda d: d == torch.int32, dev)
        _require(sc, f"scales[{i}]", lambda d: d == torch.float16, dev)
        if qw.dim() != 2 or qw.shape[0] * 8 != K:
            raise ValueError(f"qweights[{i}] does not match K={K}")
        layer_shapes(x, qw, sc, group)
        Ns.append(int(qw.shape[1]))
    if outs is None:
        outs = [torch.empty((M, n), dtype=torch.float16, device=dev) for n in Ns]
    else:
        if len(outs) != len(Ns):
            raise ValueError("one output per linear")
        for i, (o, n) in enumerate(zip(outs, Ns)):
            _require(o, f"outs[{i}]", lambda d: d == torch.float16, dev)
            if tuple(o.shape) != (M, n):
                raise ValueError(f"outs[{i}] has shape {tuple(o.shape)}, expected {(M, n)}")
    count = len(Ns)
    qa = (ctypes.c_void_p * count)(*[_ptr(q) for q in qweights])
    sa = (ctypes.c_void_p * count)(*[_ptr(t) for t in scales])
    na = (ctypes.c_int64 * count)(*Ns)
    ya = (ctypes.c_void_p * count)(*[_ptr(o) for o in outs])
    with torch.cuda.device(dev):
        _check(lib.gptq_w4a16_gemm_grouped(_ptr(x), qa, sa, na, count, M, K, group, ya,
                                           _stream_handle(stream, dev)))
    return outs


def gemm_asym(x: torch.Tensor, qweight: torch.Tensor, scales: torch.Tensor,
              qzeros: torch.Tensor, group: int, out: torch.Tensor | None = None,
              stream=None) -> torch.Tensor:
    """Y = x . W, W = fp16((q - z) * s) with zeros packed in qzeros
    [n_groups, N/8] int32 (eight per word along N); N % 32 == 0."""
    lib = load()
    dev = qweight.device
    _require(qweight, "qweight", lambda d: d == torch.int32, None)
    _require(scales, "scales", lambda d: d == torch.float16, dev)
    _require(qzeros, "qzeros", lambda d: d == torch.int32, dev)
    _require(x, "x", lambda d: d == torch.float16, dev)
    M, K, N = layer_shapes(x, qweight, scales, group)
    if qzeros.dim() != 2 or tuple(qzeros.shape) != (scales.shape[0], N // 8):
        raise ValueError(f"qzeros has shape {tuple(qzeros.shape)}, expected "
                         f"{(scales.shape[0], N // 8)}")
    if out is None:
        out = torch.empty((M, N), dtype=torch.float16, device=dev)
    else:
        _require(out, "out", lambda d: d == torch.float16, dev)
        _check_shape(out, "out", (M, N))
    with torch.cuda.device(dev):
        _check(lib.gptq_w4a16_gemm_asym(_ptr(x), _ptr(qweight), _ptr(scales), _ptr(qzeros), M,
                                        K, N, group, _ptr(out), _stream_handle(stream, dev)))
    return out


def gidx_shapes(x, qweight, scales, g_idx) -> tuple[int, int, int, int]:
    """(M, K, N, n_groups) of an act-order call, after checking x [M, K],
    qweight [K/8, N], scales [n_groups, N] and g_idx [K]."""
    M, K, N = layer_shapes(x, qweight, scales, 0)  # 0: scales checked below
    if int(scales.shape[1]) != N:
        raise ValueError(f"scales has shape {tuple(scales.shape)}, expected (n_groups, {N})")
    if g_idx.dim() != 1 or int(g_idx.shape[0]) != K:
        raise ValueError(f"g_idx has shape {tuple(g_idx.shape)}, expected ({K},)")
    return M, K, N, int(scales.shape[0])


def gemm_gidx(x: torch.Tensor, qweight: torch.Tensor, scales: torch.Tensor,
              g_idx: torch.Tensor, out: torch.Tensor | None = None,
              stream=None) -> torch.Tensor:
    """Y = x . W, W[k, n] = fp16((q[k, n] - 8) * scales[g_idx[k], n]) (act
    order): g_idx [K] int32 with entries in 0 .. n_groups - 1, scales
    [n_groups, N], n_groups <= GIDX_MAX_GROUPS.  An out-of-range index is
    reported by device_error() as GPTQ_ERR_INDEX."""
    lib = load()
    dev = qweight.device
    _require(qweight, "qweight", lambda d: d == torch.int32, None)
    _require(scales, "scales", lambda d: d == torch.float16, dev)
    _require(g_idx, "g_idx", lambda d: d == torch.int32, dev)
    _require(x, "x", lambda d: d == torch.float16, dev)
    M, K, N, ng = gidx_shapes(x, qweight, scales, g_idx)
    if out is None:
        out = torch.empty((M, N), dtype=torch.float16, device=dev)
    else:
        _require(out, "out", lambda d: d == torch.float16, dev)
        _check_shape(out, "out", (M, N))
    with torch.cuda.device(dev):
        _check(lib.gptq_w4a16_gemm_gidx(_ptr(x), _ptr(qweight), _ptr(scales), _ptr(g_idx), M, K,
                                        N, ng, _ptr(out), _stream_handle(stream, dev)))
    return out


def gemm_lora(x: torch.Tensor, qweight: torch.Tensor, scales: torch.Tensor, group: int,
              lora_a: torch.Tensor, lora_b: torch.Tensor, t_work: torch.Tensor | None = None,
              out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Y = x . dequant(qweight, scales) + fp16(x . lora_a^T) . lora_b^T (FP16),
    lora_a [rank, K], lora_b [N, rank] with the adapter's scaling applied;
    t_work [M, rank] receives fp16(x . lora_a^T)."""
    lib = load()
    dev = qweight.device
    _require(qweight, "qweight", lambda d: d == torch.int32, None)
    _require(scales, "scales", lambda d: d == torch.float16, dev)
    _require(x, "x", lambda d: d == torch.float16, dev)
    _require(lora_a, "lora_a", lambda d: d == torch.float16, dev)
    _require(lora_b, "lora_b", lambda d: d == torch.float16, dev)
    M, K, N = layer_shapes(x, qweight, scales, group)
    rank = adapter_shapes(lora_a, lora_b, K, N)
    if t_work is None:
        t_work = torch.empty((M, rank), dtype=torch.float16, device=dev)
    else:
        _require(t_work, "t_work", lambda d: d == torch.float16, dev)
        _check_shape(t_work, "t_work", (M, rank))
    if out is None:
        out = torch.empty((M, N), dtype=torch.float16, device=dev)
    else:
        _require(out, "out", lambda d: d == torch.float16, dev)
        _check_shape(out, "out", (M, N))
    with torch.cuda.device(dev):
        _check(lib.gptq_w4a16_gemm_lora(_ptr(x), _ptr(qweight), _ptr(scales), M, K, N, group,
                                        _ptr(lora_a), _ptr(lora_b), rank, _ptr(t_work),
                                        _ptr(out), _stream_handle(stream, dev)))
    return out


def gemm_lora_noalloc(x: torch.Tensor, qweight: torch.Tensor, scales: torch.Tensor,
                      group: int, lora_a: torch.Tensor, lora_b: torch.Tensor,
                      out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """gemm_lora with T kept in the library's static device buffer (no work
    tensor; M * rank * 2 <= LORA_SCRATCH_BYTES; calls that may overlap in time
    share the buffer and race)."""
    lib = load()
    dev = qweight.device
    _require(qweight, "qweight", lambda d: d == torch.int32, None)
    _require(scales, "scales", lambda d: d == torch.float16, dev)
    _require(x, "x", lambda d: d == torch.float16, dev)
    _require(lora_a, "lora_a", lambda d: d == torch.float16, dev)
    _require(lora_b, "lora_b", lambda d: d == torch.float16, dev)
    M, K, N = layer_shapes(x, qweight, scales, group)
    rank = adapter_shapes(lora_a, lora_b, K, N)
    if out is None:
        out = torch.empty((M, N), dtype=torch.float16, device=dev)
    else:
        _require(out, "out", lambda d: d == torch.float16, dev)
        _check_shape(out, "out", (M, N))
    with torch.cuda.device(dev):
        _check(lib.gptq_w4a16_gemm_lora_noalloc(_ptr(x), _ptr(qweight), _ptr(scales), M, K, N,
                                                group, _ptr(lora_a), _ptr(lora_b), rank,
                                                _ptr(out), _stream_handle(stream, dev)))
    return out


def dequant(qweight: torch.Tensor, scales: torch.Tensor, group: int,
            out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """W[K, N] = fp16((q - 8) * s): the debugging entry."""
    lib = load()
    dev = qweight.device
    _require(qweight, "qweight", lambda d: d == torch.int32, None)
    _require(scales, "scales", lambda d: d == torch.float16, dev)
    if qweight.dim() != 2 or scales.dim() != 2:
        raise ValueError("qweight and scales must be 2-D")
    K, N = int(qweight.shape[0]) * 8, int(qweight.shape[1])
    if group in GROUP_SIZES and tuple(scales.shape) != (n_groups(K, group), N):
        raise ValueError(f"scales has shape {tuple(scales.shape)}, expected "
                         f"{(n_groups(K, group), N)} for K={K}, group={group}")
    if out is None:
        out = torch.empty((K, N), dtype=torch.float16, device=dev)
    else:
        _require(out, "out", lambda d: d == torch.float16, dev)
        _check_shape(out, "out", (K, N))
    with torch.cuda.device(dev):
        _check(lib.gptq_dequant(_ptr(qweight), _ptr(scales), K, N, group, _ptr(out),
                                _stream_handle(stream, dev)))
    return out


def select(M: int, K: int, N: int, group: int) -> tuple[int, int]:
    """(kernel_id, split_k) the dispatcher picks for this shape."""
    lib = load()
    k, s = _i32(-1), _i32(-1)
    _check(lib.gptq_w4a16_select(M, K, N, group, ctypes.byref(k), ctypes.byref(s)))
    return k.value, s.value


def device_error() -> int:
    """Read and clear the device error word (synchronises the device)."""
    return int(load().gptq_device_error())


def version() -> str:
    return load().gptq_version().decode()
