"""Act-order weights (gptq_w4a16_gemm_gidx) against the oracle.

    W[k, n] = fp16((q[k, n] - 8) * scales[g_idx[k], n])

Read from the GPTQ-Pro README ("Runtime contract", act order outside its
contract) and the GPTQModel wiki (desc_act); the oracle's act-order functions
are pinned on the CPU.  Bars: Y within max |y - y_ref| / (1 + |y_ref|) <= 1e-2
of the binary64 oracle; bitwise where the definition leaves no freedom (one-hot
X reproduces a row of W; consecutive indices reproduce the plain layer, whose
kernel sums in the same order); a bad index is reported, never read outside
the scales.
"""
import numpy as np
import pytest
import torch

import oracle
from int4_weight_only_gptq_b200 import binding as B
from int4_weight_only_gptq_b200 import workloads as W

pytestmark = pytest.mark.gpu
TOL = 1e-2
GPTQ_ERR_INDEX = 10


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from int4_weight_only_gptq_b200.build import build
    build()
    B.load()
    assert B.device_error() == 0
    yield
    assert B.device_error() == 0


def f16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.float16).cuda()


def run_gidx(x, qweight, scales, g_idx, out=None):
    y = B.gemm_gidx(f16(x), torch.from_numpy(qweight).cuda(), f16(scales),
                    torch.from_numpy(np.ascontiguousarray(g_idx, dtype=np.int32)).cuda(), out=out)
    torch.cuda.synchronize()
    return y.cpu().numpy()


def rel_err(y, ref):
    y = y.astype(np.float64)
    return float(np.max(np.abs(y - ref) / (1.0 + np.abs(ref)))) if y.size else 0.0


CASES = [  # (M, K, N, G, kind)
    (1, 528, 136, 128, "perm"),      # ragged K and last group, 16-token tile, 512-k stages
    (5, 2064, 264, 32, "perm"),      # K split over a cluster (256-k stages)
    (16, 1040, 200, 16, "random"),   # groups of unequal size, ragged N
    (17, 5120, 72, 128, "perm"),     # 32-token tile
    (40, 2048, 136, 64, "random"),   # 48-token tile
    (64, 1536, 264, 512, "perm"),    # 64-token tile
    (65, 528, 136, 128, "perm"),     # two token tiles, the second with one token
    (130, 1040, 200, 32, "perm"),    # three token tiles
    (300, 96, 8, 16, "random"),      # a single k stage, one narrow column block
    (7, 17408, 136, 32, "perm"),     # 544 groups: the down-projection's scale tile
    (3, 8192, 72, 16, "perm"),       # 512 groups
    (2, 512, 256, -1, "perm"),       # one group
]


@pytest.mark.parametrize("M,K,N,G,kind", CASES)
def test_gidx_parity(M, K, N, G, kind):
    p = W.make_problem(M, K, N, G, seed=M + K + N)
    g = W.make_gidx(K, G, seed=M + K, kind=kind)
    y = run_gidx(p.x, p.qweight, p.scales, g)
    ref = oracle.gemm_gidx(p.x, p.qweight, p.scales, g)
    err = rel_err(y, ref)
    print(f"[parity] act order M={M} K={K} N={N} G={G} {kind}: {err:.3e}")
    assert np.all(np.isfinite(y))
    assert err <= TOL


@pytest.mark.parametrize("M,K,N,G", [
    (1, 528, 136, 128), (16, 5120, 264, 32), (9, 2064, 72, 16), (32, 1040, 200, -1),
    (48, 2048, 136, 64), (64, 1536, 264, 1024), (3, 17408, 136, 32), (1, 5120, 1024, 128),
])
def test_consecutive_indices_give_the_plain_layer_bitwise(M, K, N, G):
    p = W.make_problem(M, K, N, G, seed=M * 3 + K)
    g = W.make_gidx(K, G, kind="consecutive")
    y = run_gidx(p.x, p.qweight, p.scales, g)
    y_plain = B.gemm(f16(p.x), torch.from_numpy(p.qweight).cuda(), f16(p.scales), G)
    torch.cuda.synchronize()
    assert np.array_equal(y.view(np.uint16), y_plain.cpu().numpy().view(np.uint16))


@pytest.mark.parametrize("K,N,G,kind", [(528, 136, 128, "perm"), (2064, 264, 16, "random"),
                                        (17408, 72, 32, "perm")])
def test_one_hot_x_reproduces_rows_of_w_bitwise(K, N, G, kind):
    # row m of X is one-hot at k_m: Y[m, :] is W[k_m, :] (one exact product)
    p = W.make_problem(1, K, N, G, seed=K + N)
    g = W.make_gidx(K, G, seed=K, kind=kind)
    rng = np.random.default_rng(K)
    ks = np.concatenate([[0, K - 1], rng.choice(K, size=14, replace=False)])
    x = np.zeros((len(ks), K), dtype=np.float16)
    x[np.arange(len(ks)), ks] = 1.0
    y = run_gidx(x, p.qweight, p.scales, g)
    w = oracle.dequant_gidx(p.qweight, p.scales, g)
    assert np.array_equal(y.view(np.uint16), w[ks].view(np.uint16))


@pytest.mark.parametrize("M", [1, 16, 130])
def test_gidx_up_projection_full(M):
    # the 5120 -> 17408 linear with act order (40 groups of 128), sampled rows
    p = W.prefill(M)
    g = W.make_gidx(p.K, p.group, seed=M, kind="perm")
    y = run_gidx(p.x, p.qweight, p.scales, g)
    rows = sorted({0, M // 2, M - 1})
    ref = oracle.gemm_gidx_rows(p.x, p.qweight, p.scales, g, rows)
    err = rel_err(y[rows], ref)
    print(f"[parity] act order up-projection M={M}: {err:.3e} over rows {rows}")
    assert err <= TOL


def test_gidx_down_projection_full():
    # 17408 -> 5120 with groups of 32 (544 scale rows) and outlier channels
    p = W.decode_down(4)
    g = W.make_gidx(p.K, p.group, seed=4, kind="perm")
    y = run_gidx(p.x, p.qweight, p.scales, g)
    ref = oracle.gemm_gidx_rows(p.x, p.qweight, p.scales, g, [0, 3])
    err = rel_err(y[[0, 3]], ref)
    print(f"[parity] act order down-projection M=4: {err:.3e}")
    assert err <= TOL


def test_gidx_is_deterministic():
    p = W.make_problem(40, 5120, 264, 128, seed=11)
    g = W.make_gidx(5120, 128, seed=11, kind="perm")
    a = run_gidx(p.x, p.qweight, p.scales, g)
    b = run_gidx(p.x, p.qweight, p.scales, g)
    assert np.array_equal(a.view(np.uint16), b.view(np.uint16))


@pytest.mark.parametrize("bad", [5, -1, 1 << 30])
def test_out_of_range_index_is_reported(bad):
    p = W.make_problem(3, 528, 136, 128, seed=2)   # 5 groups
    g = W.make_gidx(528, 128, seed=2, kind="perm")
    g[77] = bad
    run_gidx(p.x, p.qweight, p.scales, g)
    assert B.device_error() == GPTQ_ERR_INDEX
    assert B.device_error() == 0   # read once, then cleared
    # the next call with valid indices is unaffected
    g[77] = 0
    y = run_gidx(p.x, p.qweight, p.scales, g)
    assert rel_err(y, oracle.gemm_gidx(p.x, p.qweight, p.scales, g)) <= TOL
    assert B.device_error() == 0


@pytest.mark.parametrize("M,K,N,G", [(65, 528, 264, 128), (130, 2064, 136, 32), (7, 1040, 8, 16)])
def test_gidx_writes_stay_inside_y(M, K, N, G):
    guard = 8192
    p = W.make_problem(M, K, N, G, seed=M + N)
    g = W.make_gidx(K, G, seed=M, kind="perm")
    pattern = np.random.default_rng(M).integers(0, 256, size=2 * guard + M * N * 2, dtype=np.uint8)
    buf = torch.from_numpy(pattern.copy()).cuda()
    out = buf[guard:guard + M * N * 2].view(torch.float16).view(M, N)
    y = run_gidx(p.x, p.qweight, p.scales, g, out=out)
    got = buf.cpu().numpy()
    assert np.array_equal(got[:guard], pattern[:guard])
    assert np.array_equal(got[guard + M * N * 2:], pattern[guard + M * N * 2:])
    assert rel_err(y, oracle.gemm_gidx(p.x, p.qweight, p.scales, g)) <= TOL


def test_mis_shaped_g_idx_is_refused_before_the_library_is_called():
    p = W.make_problem(2, 512, 256, 128, seed=1)
    with pytest.raises(ValueError):
        run_gidx(p.x, p.qweight, p.scales, np.zeros(500, dtype=np.int32))
