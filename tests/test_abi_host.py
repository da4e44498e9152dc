"""The C ABI on the host (no GPU needed): the library loads, exports every
entry point declared in include/*.h, and rejects bad arguments with the right
status before touching a device.  No call here launches a kernel."""
import ctypes
import glob
import os
import re

import pytest

from int4_weight_only_gptq_b200 import binding
from int4_weight_only_gptq_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build()
    return binding.load()


def declared_entry_points():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        names += re.findall(r"GPTQ_API\s+[\w\s\*]*?\b(gptq_\w+)\s*\(", text)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    names = declared_entry_points()
    assert len(names) >= 8
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(binding.EXPORTS)


def test_version_and_status_strings(lib):
    assert binding.version() == "0.1.0"
    for st in range(11):
        assert binding.status_string(st) != "unknown status"
    assert binding.status_string(12345) == "unknown status"


# fake, aligned device-looking addresses: never dereferenced because every
# call below fails a host-side check first (or returns early for M == 0)
X, QW, S, Y = 0x10000, 0x200000, 0x400000, 0x800000


def call(lib, x=X, qw=QW, s=S, M=4, K=512, N=256, g=128, y=Y, kernel=None):
    args = (ctypes.c_void_p(x), ctypes.c_void_p(qw), ctypes.c_void_p(s), M, K, N, g,
            ctypes.c_void_p(y), None)
    if kernel is None:
        return lib.gptq_w4a16_gemm(*args)
    return lib.gptq_w4a16_gemm_kernel(*args, kernel)


@pytest.mark.parametrize("kw,status", [
    (dict(M=-1), 2), (dict(K=0), 2), (dict(K=-16), 2), (dict(N=0), 2),
    (dict(K=520), 2), (dict(N=252), 2), (dict(K=65536 + 16), 2),
    (dict(N=(1 << 20) + 8), 2), (dict(M=(1 << 23) + 1), 2),
    (dict(g=0), 3), (dict(g=8), 3), (dict(g=100), 3), (dict(g=2048), 3), (dict(g=-2), 3),
    (dict(qw=0), 1), (dict(s=0), 1), (dict(x=0), 1), (dict(y=0), 1),
    (dict(x=X + 2), 4), (dict(qw=QW + 4), 4), (dict(s=S + 8), 4), (dict(y=Y + 2), 4),
    (dict(y=X), 8), (dict(y=QW + 16), 8), (dict(y=S), 8),
    (dict(kernel=3), 9), (dict(kernel=-1), 9), (dict(kernel=1, M=65), 9),
])
def test_gemm_argument_checks(lib, kw, status):
    assert call(lib, **kw) == status


def test_empty_m_is_a_no_op(lib):
    # M == 0: success without a device and without x / y
    assert call(lib, M=0, x=0, y=0) == 0
    assert call(lib, M=0, x=0, y=0, kernel=2) == 0


def test_no_device_is_reported(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    assert call(lib) == 5
    k, s = ctypes.c_int32(), ctypes.c_int32()
    assert lib.gptq_w4a16_select(1, 512, 256, 128, ctypes.byref(k), ctypes.byref(s)) == 5


def test_dequant_and_select_checks(lib):
    v = ctypes.c_void_p
    assert lib.gptq_dequant(v(QW), v(S), 520, 256, 128, v(Y), None) == 2
    assert lib.gptq_dequant(v(QW), v(S), 512, 256, 7, v(Y), None) == 3
    assert lib.gptq_dequant(None, v(S), 512, 256, 128, v(Y), None) == 1
    assert lib.gptq_dequant(v(QW), v(S), 512, 256, 128, None, None) == 1
    assert lib.gptq_dequant(v(QW), v(S), 512, 256, 128, v(Y + 2), None) == 4
    assert lib.gptq_dequant(v(QW), v(S), 512, 256, 128, v(QW), None) == 8
    assert lib.gptq_w4a16_select(1, 512, 250, 128, None, None) == 2
    assert lib.gptq_w4a16_select(1, 512, 256, 3, None, None) == 3
    assert lib.gptq_w4a16_gemm_decode_splits(v(X), v(QW), v(S), 1, 512, 256, 128, v(Y),
                                             None, 0) == 9
    assert lib.gptq_w4a16_gemm_decode_splits(v(X), v(QW), v(S), 1, 512, 256, 128, v(Y),
                                             None, 9) == 9


def test_binding_refuses_cpu_tensors(lib):
    import torch
    x = torch.zeros(1, 512, dtype=torch.float16)
    qw = torch.zeros(64, 256, dtype=torch.int32)
    s = torch.zeros(4, 256, dtype=torch.float16)
    with pytest.raises(ValueError):
        binding.gemm(x, qw, s, 128)


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(RuntimeError, match="not built"):
        binding.load.__wrapped__ if hasattr(binding.load, "__wrapped__") else None
        saved = binding._lib
        binding._lib = None
        try:
            binding.load(str(tmp_path / "nope.so"))
        finally:
            binding._lib = saved


# ---- gptq_w4a16_gemm_grouped: host-side checks ------------------------------

Y2, QW2, S2 = 0xC00000, 0x1000000, 0x1400000


def call_grouped(lib, count=2, x=X, qws=(QW, QW2), ss=(S, S2), ns=(256, 136), ys=(Y, Y2),
                 M=4, K=512, g=128, arrays=True):
    n = max(count, 1)
    qa = (ctypes.c_void_p * n)(*[ctypes.c_void_p(v) for v in (list(qws) + [QW] * n)[:n]])
    sa = (ctypes.c_void_p * n)(*[ctypes.c_void_p(v) for v in (list(ss) + [S] * n)[:n]])
    na = (ctypes.c_int64 * n)(*(list(ns) + [256] * n)[:n])
    ya = (ctypes.c_void_p * n)(*[ctypes.c_void_p(v) for v in (list(ys) + [Y] * n)[:n]])
    if not arrays:
        qa = sa = na = ya = None
    return lib.gptq_w4a16_gemm_grouped(ctypes.c_void_p(x), qa, sa, na, count, M, K, g, ya, None)


@pytest.mark.parametrize("kw,status", [
    (dict(count=0), 2), (dict(count=9), 2), (dict(arrays=False), 1),
    (dict(ns=(256, 252)), 2), (dict(ns=(256, 0)), 2), (dict(K=520), 2), (dict(g=100), 3),
    (dict(qws=(QW, 0)), 1), (dict(ss=(0, S2)), 1), (dict(x=0), 1), (dict(ys=(Y, 0)), 1),
    (dict(ys=(Y, Y2 + 2)), 4), (dict(qws=(QW + 4, QW2)), 4), (dict(x=X + 2), 4),
    (dict(ys=(Y, Y + 16)), 8),            # two outputs overlap
    (dict(ys=(Y, QW + 64)), 8),           # an output overlaps another linear's qweight
    (dict(ys=(S2, Y2)), 8),               # an output overlaps another linear's scales
    (dict(ys=(X, Y2)), 8),                # an output overlaps x
])
def test_grouped_argument_checks(lib, kw, status):
    assert call_grouped(lib, **kw) == status


def test_grouped_empty_m_and_no_device(lib):
    import torch
    assert call_grouped(lib, M=0, x=0, ys=(0, 0)) == 0
    if not torch.cuda.is_available():
        assert call_grouped(lib) == 5


# ---- gptq_w4a16_gemm_lora: host-side checks ----------------------------------
# Fake device addresses: lora_a [32, 512] (32 KB), lora_b [256, 32] (16 KB),
# t_work [4, 32] (256 B); disjoint from the ones above.

LA, LB, TW = 0x1800000, 0x1C00000, 0x2000000


def call_lora(lib, x=X, qw=QW, s=S, M=4, K=512, N=256, g=128, a=LA, b=LB, rank=32, t=TW,
              y=Y):
    v = ctypes.c_void_p
    return lib.gptq_w4a16_gemm_lora(v(x), v(qw), v(s), M, K, N, g, v(a), v(b), rank, v(t), v(y),
                                    None)


@pytest.mark.parametrize("kw,status", [
    (dict(rank=0), 2), (dict(rank=8), 2), (dict(rank=40), 2), (dict(rank=272), 2),
    (dict(K=520), 2), (dict(N=252), 2), (dict(g=100), 3),
    (dict(a=0), 1), (dict(b=0), 1), (dict(qw=0), 1), (dict(t=0), 1), (dict(x=0), 1),
    (dict(y=0), 1),
    (dict(a=LA + 2), 4), (dict(b=LB + 8), 4), (dict(t=TW + 2), 4), (dict(x=X + 2), 4),
    (dict(t=X), 8),            # T would overwrite x
    (dict(t=LA + 64), 8),      # T would overwrite lora_a
    (dict(t=LB), 8),           # T would overwrite lora_b
    (dict(y=TW), 8),           # Y would overwrite T
    (dict(y=LB), 8),           # Y would overwrite lora_b
    (dict(t=QW + 16), 8),
])
def test_lora_argument_checks(lib, kw, status):
    assert call_lora(lib, **kw) == status


def test_lora_empty_m_and_no_device(lib):
    import torch
    assert call_lora(lib, M=0, x=0, t=0, y=0) == 0
    # the adapter and rank are still checked when M == 0
    assert call_lora(lib, M=0, x=0, t=0, y=0, rank=24) == 2
    assert call_lora(lib, M=0, x=0, t=0, y=0, a=0) == 1
    if not torch.cuda.is_available():
        assert call_lora(lib) == 5


# ---- gptq_w4a16_gemm_asym: host-side checks ----------------------------------
# Fake qzeros [4, 32] (512 B) for K=512, N=256, group 128.

QZ = 0x2400000


def call_asym(lib, x=X, qw=QW, s=S, qz=QZ, M=4, K=512, N=256, g=128, y=Y):
    v = ctypes.c_void_p
    return lib.gptq_w4a16_gemm_asym(v(x), v(qw), v(s), v(qz), M, K, N, g, v(y), None)


@pytest.mark.parametrize("kw,status", [
    (dict(N=264), 2), (dict(N=8), 2), (dict(K=520), 2), (dict(g=100), 3),
    (dict(qz=0), 1), (dict(qw=0), 1), (dict(x=0), 1), (dict(y=0), 1),
    (dict(qz=QZ + 4), 4), (dict(y=Y + 2), 4),
    (dict(y=QZ), 8), (dict(y=X), 8), (dict(y=S + 32), 8),
])
def test_asym_argument_checks(lib, kw, status):
    assert call_asym(lib, **kw) == status


def test_asym_empty_m_and_no_device(lib):
    import torch
    assert call_asym(lib, M=0, x=0, y=0) == 0
    assert call_asym(lib, M=0, x=0, y=0, qz=0) == 1
    if not torch.cuda.is_available():
        assert call_asym(lib) == 5


# ---- gptq_w4a16_gemm_gidx: host-side checks ----------------------------------
# Fake g_idx [512] (2 KB) for K=512, N=256 and four groups.

GI = 0x2800000


def call_gidx(lib, x=X, qw=QW, s=S, gi=GI, M=4, K=512, N=256, ng=4, y=Y):
    v = ctypes.c_void_p
    return lib.gptq_w4a16_gemm_gidx(v(x), v(qw), v(s), v(gi), M, K, N, ng, v(y), None)


@pytest.mark.parametrize("kw,status", [
    (dict(M=-1), 2), (dict(K=520), 2), (dict(N=252), 2), (dict(K=65536 + 16), 2),
    (dict(ng=0), 2), (dict(ng=-1), 2), (dict(ng=641), 2),
    (dict(gi=0), 1), (dict(qw=0), 1), (dict(s=0), 1), (dict(x=0), 1), (dict(y=0), 1),
    (dict(gi=GI + 4), 4), (dict(x=X + 2), 4), (dict(y=Y + 2), 4),
    (dict(y=GI), 8), (dict(y=X), 8), (dict(y=S + 32), 8), (dict(y=QW), 8),
])
def test_gidx_argument_checks(lib, kw, status):
    assert call_gidx(lib, **kw) == status


def test_gidx_empty_m_and_no_device(lib):
    import torch
    assert call_gidx(lib, M=0, x=0, y=0) == 0
    assert call_gidx(lib, M=0, x=0, y=0, gi=0) == 1
    assert call_gidx(lib, M=0, x=0, y=0, ng=640) == 0
    if not torch.cuda.is_available():
        assert call_gidx(lib) == 5


# ---- binding: shape checks before the library is called ----------------------
# The C ABI sees pointers and the sizes it is given; a tensor smaller than those
# sizes would be read or written past its end, so the binding checks shapes.
# The checks are pure shape logic and run here on CPU tensors.

def _t(*shape, dtype=None):
    import torch
    return torch.zeros(shape, dtype=dtype or torch.float16)


def test_n_groups():
    assert binding.n_groups(512, 128) == 4
    assert binding.n_groups(528, 128) == 5       # ragged last group
    assert binding.n_groups(512, -1) == 1
    assert binding.n_groups(512, 1024) == 1      # a group of K or more is one group
    assert binding.n_groups(512, 512) == 1


def test_layer_shapes_accept_and_reject():
    import torch
    i32 = torch.int32
    assert binding.layer_shapes(_t(3, 512), _t(64, 256, dtype=i32), _t(4, 256), 128) == (3, 512, 256)
    assert binding.layer_shapes(_t(3, 528), _t(66, 256, dtype=i32), _t(5, 256), 128) == (3, 528, 256)
    assert binding.layer_shapes(_t(1, 512), _t(64, 256, dtype=i32), _t(1, 256), -1) == (1, 512, 256)
    bad = [
        (_t(3, 512), _t(63, 256, dtype=i32), _t(4, 256), 128),     # qweight rows != K/8
        (_t(3, 512), _t(64, 256, dtype=i32), _t(2, 256), 128),     # scales for group 256
        (_t(3, 512), _t(64, 256, dtype=i32), _t(4, 248), 128),     # scales narrower than N
        (_t(3, 512), _t(64, 256, dtype=i32), _t(4, 256), -1),      # group -1 has one row
        (_t(512), _t(64, 256, dtype=i32), _t(4, 256), 128),        # x not 2-D
        (_t(3, 512), _t(64, 256, dtype=i32), _t(1024), 128),       # scales not 2-D
    ]
    for args in bad:
        with pytest.raises(ValueError):
            binding.layer_shapes(*args)
    # an unsupported group is the library's to report (GPTQ_ERR_GROUP)
    assert binding.layer_shapes(_t(3, 512), _t(64, 256, dtype=i32), _t(7, 256), 100) == (3, 512, 256)


def test_adapter_shapes_accept_and_reject():
    assert binding.adapter_shapes(_t(32, 512), _t(256, 32), 512, 256) == 32
    for a, b in ((_t(32, 520), _t(256, 32)),     # lora_a does not match K
                 (_t(32, 512), _t(248, 32)),     # lora_b rows != N
                 (_t(32, 512), _t(256, 48)),     # lora_b rank != lora_a rank
                 (_t(32 * 512), _t(256, 32))):   # lora_a not 2-D
        with pytest.raises(ValueError):
            binding.adapter_shapes(a, b, 512, 256)


def test_gidx_shapes_accept_and_reject():
    import torch
    x, qw = _t(4, 512), _t(64, 256, dtype=torch.int32)
    gi = _t(512, dtype=torch.int32)
    assert binding.gidx_shapes(x, qw, _t(7, 256), gi) == (4, 512, 256, 7)
    for s, g in ((_t(7, 248), gi),                             # scales columns != N
                 (_t(7, 256), _t(520, dtype=torch.int32)),     # g_idx length != K
                 (_t(7, 256), _t(1, 512, dtype=torch.int32)),  # g_idx not 1-D
                 (_t(7 * 256), gi)):                           # scales not 2-D
        with pytest.raises(ValueError):
            binding.gidx_shapes(x, qw, s, g)
