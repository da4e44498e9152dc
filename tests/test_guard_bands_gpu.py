"""Bounds of every write, checked with guard bands (in place of a sanitizer).

Each output (Y, T, the dequantised W) is placed inside a larger device buffer
whose bytes are a seeded random pattern.  After the call, the bytes before and
after the output must still hold the pattern, and the inputs must be unchanged:
no kernel may write outside the output it was given, also on ragged shapes
(M, N and K that are not multiples of the tiles, a ragged last group) and in
every kernel path (decode 16- to 64-token tiles, K splits reduced over a
cluster, forced single-CTA prefill, pair prefill with 128- and 256-token tiles,
grouped linears, asymmetric zeros, the LoRA adapter in both kernels, the
dequantisation entry).  Fail-closed execution is part of the contract (GPTQ-Pro
README, "Why GPTQ-Pro"); the output is also checked against the oracle, so a
write that lands in the wrong place inside the output shows too.
"""
import numpy as np
import pytest
import torch

import oracle
from int4_weight_only_gptq_b200 import binding as B
from int4_weight_only_gptq_b200 import workloads as W

pytestmark = pytest.mark.gpu
TOL = 1e-2
GUARD = 8192  # bytes on each side; keeps the output 16-byte aligned


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from int4_weight_only_gptq_b200.build import build
    build()
    B.load()
    assert B.device_error() == 0
    yield
    assert B.device_error() == 0


class Guarded:
    """A [rows, cols] FP16 tensor inside a buffer of patterned bytes."""

    def __init__(self, rows, cols, seed):
        n = rows * cols * 2
        rng = np.random.default_rng(seed)
        self.pattern = rng.integers(0, 256, size=GUARD * 2 + n, dtype=np.uint8)
        self.buf = torch.from_numpy(self.pattern.copy()).cuda()
        self.n = n
        self.t = self.buf[GUARD:GUARD + n].view(torch.float16).view(rows, cols)

    def check(self, label):
        got = self.buf.cpu().numpy()
        assert np.array_equal(got[:GUARD], self.pattern[:GUARD]), f"{label}: write before the output"
        assert np.array_equal(got[GUARD + self.n:], self.pattern[GUARD + self.n:]), \
            f"{label}: write past the end of the output"

    def numpy(self):
        return self.t.cpu().numpy()


def f16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.float16).cuda()


def inputs(p):
    return f16(p.x), torch.from_numpy(p.qweight).cuda(), f16(p.scales)


def unchanged(label, *pairs):
    torch.cuda.synchronize()
    for dev_t, host in pairs:
        got = dev_t.cpu().numpy().view(np.uint8).ravel()
        assert np.array_equal(got, np.ascontiguousarray(host).view(np.uint8).ravel()), \
            f"{label}: an input was modified"


def rel_err(y, ref):
    y = y.astype(np.float64)
    return float(np.max(np.abs(y - ref) / (1.0 + np.abs(ref)))) if y.size else 0.0


LAYER_CASES = [  # (label, M, K, N, G, kernel, splits)
    ("decode 16-token tile", 5, 528, 136, 128, B.KERNEL_DECODE, 0),
    ("decode 32-token tile", 27, 1040, 264, 16, B.KERNEL_DECODE, 0),
    ("decode K split over a cluster", 3, 5120, 136, 128, B.KERNEL_AUTO, 4),
    ("decode K split, ragged K", 16, 2064, 72, 32, B.KERNEL_AUTO, 3),
    ("decode 48-token tile", 41, 1040, 136, 32, B.KERNEL_AUTO, 0),
    ("decode 64-token tile, K split", 63, 2064, 264, 128, B.KERNEL_AUTO, 2),
    ("decode persistent (more column blocks than SMs)", 7, 528, 20488, 64, B.KERNEL_AUTO, 0),
    ("forced single-CTA prefill", 20, 528, 136, 64, B.KERNEL_PREFILL, 0),
    ("pair prefill 128-token tile", 100, 528, 392, 128, B.KERNEL_AUTO, 0),
    ("pair prefill 256-token tile", 300, 1040, 264, -1, B.KERNEL_AUTO, 0),
    ("pair prefill several tiles", 777, 2064, 520, 1024, B.KERNEL_AUTO, 0),
]


@pytest.mark.parametrize("label,M,K,N,G,kernel,splits", LAYER_CASES)
def test_layer_writes_stay_inside_y(label, M, K, N, G, kernel, splits):
    p = W.make_problem(M, K, N, G, seed=M + K + N)
    x, qw, s = inputs(p)
    y = Guarded(M, N, seed=M * 31 + N)
    B.gemm(x, qw, s, G, out=y.t, kernel=kernel, decode_splits=splits)
    torch.cuda.synchronize()
    assert B.device_error() == 0
    y.check(label)
    unchanged(label, (x, p.x), (qw, p.qweight), (s, p.scales))
    err = rel_err(y.numpy(), oracle.gemm(p.x, p.qweight, p.scales, G))
    print(f"[parity] guard bands, {label} M={M} K={K} N={N} G={G}: {err:.3e}")
    assert err <= TOL


@pytest.mark.parametrize("M", [3, 24, 130])
def test_grouped_writes_stay_inside_each_y(M):
    K, G, Ns = 528, 128, (136, 264, 8)
    ps = [W.make_problem(M, K, n, G, seed=i + M) for i, n in enumerate(Ns)]
    x = f16(ps[0].x)
    qws = [torch.from_numpy(p.qweight).cuda() for p in ps]
    ss = [f16(p.scales) for p in ps]
    ys = [Guarded(M, n, seed=7 * i + M) for i, n in enumerate(Ns)]
    B.gemm_grouped(x, qws, ss, G, outs=[g.t for g in ys])
    torch.cuda.synchronize()
    assert B.device_error() == 0
    for i, (p, g) in enumerate(zip(ps, ys)):
        g.check(f"grouped linear {i}")
        ref = oracle.gemm(ps[0].x, p.qweight, p.scales, G)
        assert rel_err(g.numpy(), ref) <= TOL
    unchanged("grouped", (x, ps[0].x), *[(q, p.qweight) for q, p in zip(qws, ps)])


@pytest.mark.parametrize("M,N", [(7, 160), (27, 96), (130, 416)])
def test_asym_writes_stay_inside_y(M, N):
    K, G = 1040, 64
    p = W.make_problem(M, K, N, G, seed=M + 5)
    qz = W.make_qzeros(p.scales.shape[0], N, seed=M)
    x, qw, s = inputs(p)
    qzd = torch.from_numpy(qz).cuda()
    y = Guarded(M, N, seed=M + 1)
    B.gemm_asym(x, qw, s, qzd, G, out=y.t)
    torch.cuda.synchronize()
    assert B.device_error() == 0
    y.check("asym")
    unchanged("asym", (x, p.x), (qw, p.qweight), (s, p.scales), (qzd, qz))
    assert rel_err(y.numpy(), oracle.gemm_asym(p.x, p.qweight, p.scales, qz, G)) <= TOL


@pytest.mark.parametrize("M,r", [(1, 48), (5, 80), (20, 48), (32, 16), (100, 80), (300, 48)])
def test_lora_writes_stay_inside_t_and_y(M, r):
    K, N, G = 528, 136, 128
    p = W.make_problem(M, K, N, G, seed=M + r)
    ad = W.make_adapter(K, N, r, seed=M + r)
    x, qw, s = inputs(p)
    a, b = f16(ad.lora_a), f16(ad.lora_b)
    t = Guarded(M, r, seed=3 * M + r)
    y = Guarded(M, N, seed=5 * M + r)
    B.gemm_lora(x, qw, s, G, a, b, t_work=t.t, out=y.t)
    torch.cuda.synchronize()
    assert B.device_error() == 0
    t.check("lora T")
    y.check("lora Y")
    unchanged("lora", (x, p.x), (qw, p.qweight), (s, p.scales), (a, ad.lora_a), (b, ad.lora_b))
    ref = oracle.gemm_lora(p.x, p.qweight, p.scales, G, ad.lora_a, ad.lora_b)
    assert rel_err(y.numpy(), ref) <= TOL


@pytest.mark.parametrize("K,N,G", [(528, 136, 128), (64, 8, 16), (2064, 264, -1)])
def test_dequant_writes_stay_inside_w(K, N, G):
    p = W.make_problem(1, K, N, G, seed=K + N)
    _, qw, s = inputs(p)
    w = Guarded(K, N, seed=K)
    B.dequant(qw, s, G, out=w.t)
    torch.cuda.synchronize()
    w.check("dequant")
    unchanged("dequant", (qw, p.qweight), (s, p.scales))
    ref = oracle.dequant(p.qweight, p.scales, G)
    assert np.array_equal(w.numpy().view(np.uint16), ref.view(np.uint16))


def test_empty_m_writes_nothing():
    p = W.make_problem(1, 512, 256, 128, seed=3)
    _, qw, s = inputs(p)
    x = torch.empty((0, 512), dtype=torch.float16, device="cuda")
    y = Guarded(0, 256, seed=4)
    B.gemm(x, qw, s, 128, out=y.t)
    torch.cuda.synchronize()
    y.check("M = 0")
