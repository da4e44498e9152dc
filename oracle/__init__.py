"""CPU oracle for the symmetric INT4 GPTQ W4A16 linear layer.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU
baseline leg may import this package; the library and its Python binding never
do.  The arithmetic lives in ``gptq_oracle.c`` (plain C, binary64, one element
at a time); this module only compiles it with gcc and marshals numpy arrays.

Definition (GPTQ-Pro README, "Runtime contract"; GPTQModel wiki "Installation
and Quickstart", "Defaults and compatibility decisions"):
    q[k,n] = (uint32(qweight[k//8, n]) >> 4*(k%8)) & 0xF
    W[k,n] = fp16_RNE((q[k,n] - 8) * scales[k//G, n])
    Y[m,n] = sum_k x[m,k] * W[k,n]            (binary64, k ascending)

With a LoRA adapter (GPTQ-Pro README, "Runtime contract": adapters on the
linear path; GPTQModel README, "PEFT LoRA Training and Adapter Loading": the
adapter stays separate from the packed weights), read with PEFT's layouts and
the adapter's scaling already in lora_b:
    T[m,j] = fp16_RNE(sum_k x[m,k] * lora_a[j,k])          lora_a [r, K]
    Y[m,n] += sum_j T[m,j] * lora_b[n,j]                    lora_b [N, r]

With asymmetric zero points (GPTQModel wiki, "Defaults and compatibility
decisions": sym; GPTQ-Pro README: asymmetric weights outside that fork's
contract), read with GPTQ's packed qzeros [n_groups, N/8] (eight codes per
int32 along N, lowest nibble = lowest n), each zero taken as stored:
    z[g,n] = (uint32(qzeros[g, n//8]) >> 4*(n%8)) & 0xF
    W[k,n] = fp16_RNE((q[k,n] - z[k//G, n]) * scales[k//G, n])

With act order (GPTQ-Pro README, "Runtime contract": desc_act=False only there,
act-order checkpoints outside that fork's contract; GPTQModel wiki, "Defaults
and compatibility decisions": desc_act), read with GPTQ's group index per input
channel g_idx [K] int32, qweight keeping the channels in their own order:
    W[k,n] = fp16_RNE((q[k,n] - 8) * scales[g_idx[k], n])
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gptq_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "liboracle.so")
_lock = threading.Lock()
_lib = None

_i64 = ctypes.c_int64
_i32 = ctypes.c_int32
_p = ctypes.c_void_p


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, no fast-math) into oracle/_build."""
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_LIB_PATH) or \
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".{os.getpid()}.tmp"
        subprocess.run(["gcc", "-O2", "-fno-fast-math", "-std=c11", "-fopenmp", "-shared",
                        "-fPIC", "-o", tmp, _SRC, "-lm"], check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            lib.oracle_set_threads.argtypes = [ctypes.c_int]
            lib.oracle_get_threads.restype = ctypes.c_int
            lib.oracle_half_to_double.restype = ctypes.c_double
            lib.oracle_half_to_double.argtypes = [ctypes.c_uint16]
            lib.oracle_double_to_half.restype = ctypes.c_uint16
            lib.oracle_double_to_half.argtypes = [ctypes.c_double]
            lib.oracle_round_to_half.argtypes = [_p, _i64, _p]
            lib.oracle_unpack.argtypes = [_p, _i64, _i64, _p]
            lib.oracle_pack.argtypes = [_p, _i64, _i64, _p]
            lib.oracle_num_groups.restype = _i64
            lib.oracle_num_groups.argtypes = [_i64, _i32]
            lib.oracle_dequant.argtypes = [_p, _p, _i64, _i64, _i32, _p]
            lib.oracle_gemm.restype = ctypes.c_int
            lib.oracle_gemm.argtypes = [_p, _p, _p, _i64, _i64, _i64, _i32, _p]
            lib.oracle_gemm_entries.argtypes = [_p, _p, _p, _i64, _i64, _i64, _i32,
                                                _i64, _p, _p, _p]
            lib.oracle_gemm_rows.argtypes = [_p, _p, _p, _i64, _i64, _i64, _i32,
                                             _i64, _p, _p]
            lib.oracle_lora_down.argtypes = [_p, _p, _i64, _i64, _i64, _p]
            lib.oracle_dequant_asym.argtypes = [_p, _p, _p, _i64, _i64, _i32, _p]
            lib.oracle_gemm_asym_rows.argtypes = [_p, _p, _p, _p, _i64, _i64, _i64, _i32,
                                                  _i64, _p, _p]
            lib.oracle_lora_up_add.argtypes = [_p, _p, _i64, _i64, _i64, _p, _p]
            lib.oracle_dequant_gidx.argtypes = [_p, _p, _p, _i64, _i64, _i64, _p]
            lib.oracle_dequant_gidx.restype = ctypes.c_int
            lib.oracle_gemm_gidx_rows.argtypes = [_p, _p, _p, _p, _i64, _i64, _i64, _i64,
                                                  _i64, _p, _p]
            lib.oracle_gemm_gidx_rows.restype = ctypes.c_int
            _lib = lib
    return _lib


def _c(a, dtype):
    a = np.ascontiguousarray(a)
    if a.dtype != dtype:
        raise TypeError(f"expected {dtype}, got {a.dtype}")
    return a


def _ptr(a):
    return a.ctypes.data_as(_p)


def _bits16(a):
    a = np.ascontiguousarray(a)
    if a.dtype == np.float16:
        return a.view(np.uint16)
    return _c(a, np.uint16)


def set_threads(n: int) -> None:
    """Threads used to split independent outputs (results do not change)."""
    _load().oracle_set_threads(int(n))


def get_threads() -> int:
    return int(_load().oracle_get_threads())


def half_to_double(h: int) -> float:
    return _load().oracle_half_to_double(int(h))


def double_to_half_bits(v: float) -> int:
    return int(_load().oracle_double_to_half(float(v)))


def round_to_half(v: np.ndarray) -> np.ndarray:
    """binary64 -> binary16 (round to nearest, ties to even), as float16."""
    v = _c(np.asarray(v, dtype=np.float64), np.float64)
    out = np.empty(v.shape, dtype=np.uint16)
    _load().oracle_round_to_half(_ptr(v), v.size, _ptr(out))
    return out.view(np.float16)


def num_groups(K: int, group: int) -> int:
    return int(_load().oracle_num_groups(K, group))


def unpack(qweight: np.ndarray) -> np.ndarray:
    """int32 [K/8, N] -> uint8 codes [K, N]."""
    qw = _c(qweight, np.int32)
    K, N = qw.shape[0] * 8, qw.shape[1]
    codes = np.empty((K, N), dtype=np.uint8)
    _load().oracle_unpack(_ptr(qw), K, N, _ptr(codes))
    return codes


def pack(codes: np.ndarray) -> np.ndarray:
    """uint8 codes [K, N] (values 0..15) -> int32 [K/8, N]."""
    c = _c(codes, np.uint8)
    K, N = c.shape
    if K % 8:
        raise ValueError("K must be a multiple of 8")
    qw = np.empty((K // 8, N), dtype=np.int32)
    _load().oracle_pack(_ptr(c), K, N, _ptr(qw))
    return qw


def dequant(qweight: np.ndarray, scales: np.ndarray, group: int) -> np.ndarray:
    """W = fp16((q - 8) * s) as float16 [K, N]."""
    qw = _c(qweight, np.int32)
    s = _bits16(scales)
    K, N = qw.shape[0] * 8, qw.shape[1]
    if s.shape != (num_groups(K, group), N):
        raise ValueError(f"scales shape {s.shape} does not match K={K}, group={group}")
    w = np.empty((K, N), dtype=np.uint16)
    _load().oracle_dequant(_ptr(qw), _ptr(s), K, N, group, _ptr(w))
    return w.view(np.float16)


def gemm(x: np.ndarray, qweight: np.ndarray, scales: np.ndarray, group: int) -> np.ndarray:
    """Y = x . W in binary64, float64 [M, N]."""
    xb = _bits16(x)
    qw = _c(qweight, np.int32)
    s = _bits16(scales)
    M, K = xb.shape
    N = qw.shape[1]
    if qw.shape[0] * 8 != K:
        raise ValueError("x and qweight disagree on K")
    y = np.empty((M, N), dtype=np.float64)
    if _load().oracle_gemm(_ptr(xb), _ptr(qw), _ptr(s), M, K, N, group, _ptr(y)):
        raise MemoryError("oracle_gemm could not allocate its dequantised copy")
    return y


def gemm_entries(x, qweight, scales, group, ms, ns) -> np.ndarray:
    """Y[ms[i], ns[i]] in binary64, for sampled checks on large problems."""
    xb = _bits16(x)
    qw = _c(qweight, np.int32)
    s = _bits16(scales)
    M, K = xb.shape
    N = qw.shape[1]
    ms = _c(np.asarray(ms, dtype=np.int64), np.int64)
    ns = _c(np.asarray(ns, dtype=np.int64), np.int64)
    if ms.shape != ns.shape:
        raise ValueError("ms and ns must have the same length")
    if ms.size and (ms.min() < 0 or ms.max() >= M or ns.min() < 0 or ns.max() >= N):
        raise IndexError("sample index out of range")
    out = np.empty(ms.shape, dtype=np.float64)
    _load().oracle_gemm_entries(_ptr(xb), _ptr(qw), _ptr(s), M, K, N, group,
                                ms.size, _ptr(ms), _ptr(ns), _ptr(out))
    return out


def gemm_rows(x, qweight, scales, group, ms) -> np.ndarray:
    """Full rows Y[ms, :] in binary64, float64 [len(ms), N]."""
    xb = _bits16(x)
    qw = _c(qweight, np.int32)
    s = _bits16(scales)
    M, K = xb.shape
    N = qw.shape[1]
    ms = _c(np.asarray(ms, dtype=np.int64), np.int64)
    if ms.size and (ms.min() < 0 or ms.max() >= M):
        raise IndexError("row index out of range")
    out = np.empty((ms.size, N), dtype=np.float64)
    _load().oracle_gemm_rows(_ptr(xb), _ptr(qw), _ptr(s), M, K, N, group,
                             ms.size, _ptr(ms), _ptr(out))
    return out


def lora_down(x: np.ndarray, lora_a: np.ndarray) -> np.ndarray:
    """T = fp16(x . lora_a^T) as float16 [M, r] (binary64 sums)."""
    xb = _bits16(x)
    a = _bits16(lora_a)
    M, K = xb.shape
    r = a.shape[0]
    if a.shape[1] != K:
        raise ValueError("x and lora_a disagree on K")
    t = np.empty((M, r), dtype=np.uint16)
    _load().oracle_lora_down(_ptr(xb), _ptr(a), M, K, r, _ptr(t))
    return t.view(np.float16)


def lora_up_add(t: np.ndarray, lora_b: np.ndarray, y: np.ndarray, ms=None) -> np.ndarray:
    """y[i, :] += t[ms[i], :] . lora_b^T in binary64 (ms = all rows by default)."""
    tb = _bits16(t)
    b = _bits16(lora_b)
    M, r = tb.shape
    N = b.shape[0]
    if b.shape[1] != r:
        raise ValueError("t and lora_b disagree on the rank")
    ms = np.arange(M, dtype=np.int64) if ms is None else np.asarray(ms, dtype=np.int64)
    ms = _c(ms, np.int64)
    if ms.size and (ms.min() < 0 or ms.max() >= M):
        raise IndexError("row index out of range")
    out = _c(np.asarray(y, dtype=np.float64), np.float64)
    if out.shape != (ms.size, N):
        raise ValueError("y has the wrong shape")
    _load().oracle_lora_up_add(_ptr(tb), _ptr(b), r, N, ms.size, _ptr(ms), _ptr(out))
    return out


def gemm_lora(x, qweight, scales, group, lora_a, lora_b) -> np.ndarray:
    """Y = x . W + fp16(x . lora_a^T) . lora_b^T in binary64, float64 [M, N]."""
    return lora_up_add(lora_down(x, lora_a), lora_b, gemm(x, qweight, scales, group))


def gemm_lora_rows(x, qweight, scales, group, lora_a, lora_b, ms) -> np.ndarray:
    """Rows ms of gemm_lora, for problems too large to compute whole."""
    ms = np.asarray(ms, dtype=np.int64)
    xs = np.ascontiguousarray(np.asarray(x)[ms])
    return lora_up_add(lora_down(xs, lora_a), lora_b, gemm_rows(x, qweight, scales, group, ms))


def pack_zeros(zcodes: np.ndarray) -> np.ndarray:
    """Zero codes [n_groups, N] (0..15) -> qzeros int32 [n_groups, N/8], eight
    codes per word along N, lowest nibble = lowest n."""
    z = np.asarray(zcodes, dtype=np.uint32)
    G, N = z.shape
    if N % 8:
        raise ValueError("N must be a multiple of 8")
    words = np.zeros((G, N // 8), dtype=np.uint32)
    for j in range(8):
        words |= (z[:, j::8] & 0xF) << (4 * j)
    return words.view(np.int32)


def dequant_asym(qweight, scales, qzeros, group) -> np.ndarray:
    """W = fp16((q - z) * s) as float16 [K, N]."""
    qw = _c(qweight, np.int32)
    s = _bits16(scales)
    qz = _c(qzeros, np.int32)
    K, N = qw.shape[0] * 8, qw.shape[1]
    if s.shape != (num_groups(K, group), N) or qz.shape != (s.shape[0], N // 8):
        raise ValueError("scales or qzeros do not match K, N and the group")
    w = np.empty((K, N), dtype=np.uint16)
    _load().oracle_dequant_asym(_ptr(qw), _ptr(s), _ptr(qz), K, N, group, _ptr(w))
    return w.view(np.float16)


def gemm_asym_rows(x, qweight, scales, qzeros, group, ms) -> np.ndarray:
    """Rows ms of Y = x . W_asym in binary64, float64 [len(ms), N]."""
    xb = _bits16(x)
    qw = _c(qweight, np.int32)
    s = _bits16(scales)
    qz = _c(qzeros, np.int32)
    M, K = xb.shape
    N = qw.shape[1]
    if qz.shape != (s.shape[0], N // 8):
        raise ValueError("qzeros do not match the scales")
    ms = _c(np.asarray(ms, dtype=np.int64), np.int64)
    if ms.size and (ms.min() < 0 or ms.max() >= M):
        raise IndexError("row index out of range")
    out = np.empty((ms.size, N), dtype=np.float64)
    _load().oracle_gemm_asym_rows(_ptr(xb), _ptr(qw), _ptr(s), _ptr(qz), M, K, N, group,
                                  ms.size, _ptr(ms), _ptr(out))
    return out


def gemm_asym(x, qweight, scales, qzeros, group) -> np.ndarray:
    """Y = x . W_asym in binary64, float64 [M, N]."""
    return gemm_asym_rows(x, qweight, scales, qzeros, group, np.arange(np.asarray(x).shape[0]))


def _gidx(g_idx, K, n_groups):
    g = np.asarray(g_idx)
    if not np.issubdtype(g.dtype, np.integer):
        raise TypeError(f"g_idx must be integer, got {g.dtype}")
    if g.shape != (K,):
        raise ValueError(f"g_idx must have shape ({K},)")
    if g.size and (g.min() < 0 or g.max() >= n_groups):
        raise ValueError("g_idx entry outside 0 .. n_groups - 1")
    return np.ascontiguousarray(g, dtype=np.int32)


def dequant_gidx(qweight, scales, g_idx) -> np.ndarray:
    """W = fp16((q - 8) * scales[g_idx[k]]) as float16 [K, N] (act order)."""
    qw = _c(qweight, np.int32)
    s = _bits16(scales)
    K, N = qw.shape[0] * 8, qw.shape[1]
    if s.shape[1] != N:
        raise ValueError("scales do not match N")
    g = _gidx(g_idx, K, s.shape[0])
    w = np.empty((K, N), dtype=np.uint16)
    if _load().oracle_dequant_gidx(_ptr(qw), _ptr(s), _ptr(g), K, N, s.shape[0], _ptr(w)):
        raise ValueError("g_idx entry out of range")
    return w.view(np.float16)


def gemm_gidx_rows(x, qweight, scales, g_idx, ms) -> np.ndarray:
    """Rows ms of Y = x . W_act_order in binary64, float64 [len(ms), N]."""
    xb = _bits16(x)
    qw = _c(qweight, np.int32)
    s = _bits16(scales)
    M, K = xb.shape
    N = qw.shape[1]
    if qw.shape[0] * 8 != K or s.shape[1] != N:
        raise ValueError("qweight or scales do not match x")
    g = _gidx(g_idx, K, s.shape[0])
    ms = _c(np.asarray(ms, dtype=np.int64), np.int64)
    if ms.size and (ms.min() < 0 or ms.max() >= M):
        raise IndexError("row index out of range")
    out = np.empty((ms.size, N), dtype=np.float64)
    if _load().oracle_gemm_gidx_rows(_ptr(xb), _ptr(qw), _ptr(s), _ptr(g), M, K, N,
                                     s.shape[0], ms.size, _ptr(ms), _ptr(out)):
        raise ValueError("g_idx entry out of range")
    return out


def gemm_gidx(x, qweight, scales, g_idx) -> np.ndarray:
    """Y = x . W_act_order in binary64, float64 [M, N]."""
    return gemm_gidx_rows(x, qweight, scales, g_idx, np.arange(np.asarray(x).shape[0]))
