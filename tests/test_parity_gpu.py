"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Bars (written here):
  * dequantised weights: bit-exact;
  * Y: max |y_gpu - y_ref| / (1 + |y_ref|) <= 1e-2 against the binary64
    oracle, and every reported error is printed;
  * integer work that floating point cannot blur (one-hot X, all codes 8,
    integer-exact inputs): bitwise equal;
  * determinism: two runs give bitwise-identical Y.
Full-size problems are compared on sampled rows (every column of those rows).
"""
import numpy as np
import pytest
import torch

import oracle
from int4_weight_only_gptq_b200 import binding as B
from int4_weight_only_gptq_b200 import workloads as W

pytestmark = pytest.mark.gpu
TOL = 1e-2


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from int4_weight_only_gptq_b200.build import build
    build()
    B.load()
    assert B.device_error() == 0
    yield
    assert B.device_error() == 0


def dev(p):
    x = torch.from_numpy(p.x.view(np.int16)).view(torch.float16).cuda()
    qw = torch.from_numpy(p.qweight).cuda()
    s = torch.from_numpy(p.scales.view(np.int16)).view(torch.float16).cuda()
    return x, qw, s


def rel_err(y_gpu, y_ref):
    y = y_gpu.astype(np.float64)
    return float(np.max(np.abs(y - y_ref) / (1.0 + np.abs(y_ref)))) if y.size else 0.0


def run(p, kernel=B.KERNEL_AUTO, splits=0):
    x, qw, s = dev(p)
    y = B.gemm(x, qw, s, p.group, kernel=kernel, decode_splits=splits)
    torch.cuda.synchronize()
    return y.cpu().numpy()


def check_rows(p, y, rows, label):
    ref = oracle.gemm_rows(p.x, p.qweight, p.scales, p.group, rows)
    err = rel_err(y[rows], ref)
    print(f"[parity] {label}: max rel err {err:.3e} over {len(rows)} rows x {p.N} cols")
    assert np.all(np.isfinite(y[rows]))
    assert err <= TOL, f"{label}: {err}"
    return err


def sample_rows(M, n=4, seed=0):
    rng = np.random.default_rng(seed)
    rows = {0, M - 1}
    rows.update(int(r) for r in rng.integers(0, M, size=max(0, n - 2)))
    return sorted(rows)


# ---- dequantisation: bit-exact ----------------------------------------------

@pytest.mark.parametrize("K,N,G", [(512, 256, 128), (528, 24, 128), (64, 8, 16), (48, 40, 32),
                                   (5120, 5120, -1), (1024, 136, 1024), (160, 64, 64)])
def test_dequant_bit_exact(K, N, G):
    p = W.make_problem(1, K, N, G, seed=K + N)
    _, qw, s = dev(p)
    w = B.dequant(qw, s, G)
    torch.cuda.synchronize()
    ref = oracle.dequant(p.qweight, p.scales, G)
    assert np.array_equal(w.cpu().numpy().view(np.uint16), ref.view(np.uint16))


def test_dequant_bit_exact_full_size_up_projection():
    p = W.decode_up()
    _, qw, s = dev(p)
    w = B.dequant(qw, s, p.group).cpu().numpy()
    ref = oracle.dequant(p.qweight, p.scales, p.group)
    assert np.array_equal(w.view(np.uint16), ref.view(np.uint16))


def test_dequant_every_code_and_scale():
    """All 16 codes x every finite FP16 scale, bit-exact."""
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    bits = bits[(bits & 0x7C00) != 0x7C00]
    N = (bits.size // 8) * 8
    scales = bits[:N].view(np.float16).reshape(1, N)
    qw = np.empty((2, N), dtype=np.int32)
    qw[0] = np.int32(0x76543210)
    qw[1] = np.uint32(0xFEDCBA98).view(np.int32)
    w = B.dequant(torch.from_numpy(qw).cuda(),
                  torch.from_numpy(scales.view(np.int16)).view(torch.float16).cuda(), -1)
    ref = oracle.dequant(qw, scales, -1)
    assert np.array_equal(w.cpu().numpy().view(np.uint16), ref.view(np.uint16))


# ---- the GEMM on the tiny workload, both kernels ----------------------------

@pytest.mark.parametrize("M", [1, 4])
@pytest.mark.parametrize("kernel", [B.KERNEL_AUTO, B.KERNEL_DECODE, B.KERNEL_PREFILL])
def test_tiny(M, kernel):
    p = W.tiny(M)
    y = run(p, kernel)
    ref = oracle.gemm(p.x, p.qweight, p.scales, p.group)
    err = rel_err(y, ref)
    print(f"[parity] tiny M={M} kernel={kernel}: max rel err {err:.3e}")
    assert err <= TOL


# ---- ragged and edge shapes -----------------------------------------------

EDGE = [  # (M, K, N, G)
    (1, 16, 8, -1), (3, 48, 40, 16), (5, 528, 24, 128), (7, 96, 72, 32), (8, 160, 264, 64),
    (9, 64, 8, 16), (13, 1040, 136, 1024), (16, 272, 520, 16), (2, 5120, 8, 512),
    # K-stages that straddle group boundaries (stages of 512 k, or 256 k when
    # K is split), ragged last stages
    (4, 3072, 64, 1024), (3, 2304, 16, 512), (8, 6144, 24, 256), (1, 1600, 72, 512),
    (12, 2560, 40, 1024), (16, 1536, 200, 512),
    # the 32-token tile (17 <= M <= 32)
    (17, 528, 136, 128), (24, 2048, 72, 16), (32, 1040, 264, -1), (29, 6144, 40, 32),
    # the 48- and 64-token tiles (33 <= M <= 64, 256-k stages)
    (33, 528, 136, 128), (40, 2048, 72, 16), (48, 1040, 264, -1), (57, 6144, 40, 32),
    (64, 1536, 200, 512), (49, 3072, 64, 1024), (64, 96, 8, 64),
]


@pytest.mark.parametrize("M,K,N,G", EDGE)
@pytest.mark.parametrize("kernel", [B.KERNEL_DECODE, B.KERNEL_PREFILL])
def test_edge_shapes_small_m(M, K, N, G, kernel):
    p = W.make_problem(M, K, N, G, seed=M * 7 + K + N)
    y = run(p, kernel)
    ref = oracle.gemm(p.x, p.qweight, p.scales, G)
    err = rel_err(y, ref)
    print(f"[parity] edge M={M} K={K} N={N} G={G} kernel={kernel}: {err:.3e}")
    assert err <= TOL


@pytest.mark.parametrize("M,K,N,G", [(17, 64, 8, 16), (129, 528, 136, 128), (300, 96, 264, 32),
                                     (257, 1040, 128, -1), (513, 160, 392, 64),
                                     # token tiles of 64 (M <= 64) and 128 (M <= 128)
                                     (33, 96, 72, 32), (64, 160, 136, 64), (100, 528, 264, 128),
                                     (128, 1040, 128, -1), (65, 2048, 200, 16),
                                     # CTA-pair tiles (M > 128): the odd CTA's half partly
                                     # filled, empty, or with one row; padding CTAs (odd
                                     # number of 128-column tiles); a single k stage
                                     (200, 2048, 392, 128), (256, 528, 200, 16),
                                     (385, 96, 136, 32), (160, 64, 8, -1), (255, 1024, 24, 64)])
def test_edge_shapes_prefill(M, K, N, G):
    p = W.make_problem(M, K, N, G, seed=M + K + N)
    y = run(p, B.KERNEL_PREFILL)
    ref = oracle.gemm(p.x, p.qweight, p.scales, G)
    err = rel_err(y, ref)
    print(f"[parity] prefill M={M} K={K} N={N} G={G}: {err:.3e}")
    assert err <= TOL


@pytest.mark.parametrize("M", [6, 40, 64])
@pytest.mark.parametrize("splits", [1, 2, 3, 4, 5, 6, 7, 8])
def test_decode_every_split(M, splits):
    # M = 6: 512-k stages without a split, 256-k stages with one; M = 40 and
    # 64: 256-k stages of the 48- and 64-token tiles
    p = W.make_problem(M, 2048, 200, 32, seed=splits + M)
    y = run(p, splits=splits)
    ref = oracle.gemm(p.x, p.qweight, p.scales, 32)
    assert rel_err(y, ref) <= TOL


# ---- closed forms and exact cases -----------------------------------------

@pytest.mark.parametrize("kernel", [B.KERNEL_DECODE, B.KERNEL_PREFILL])
def test_all_codes_eight_gives_exact_zero(kernel):
    p = W.make_problem(16, 512, 256, 128, seed=3)
    p.qweight[:] = np.uint32(0x88888888).view(np.int32)
    y = run(p, kernel)
    assert np.all(y.astype(np.float64) == 0.0)


def test_one_hot_x_32_token_tile_bitwise():
    """Decode with 32 tokens: every row one-hot at a different k."""
    p = W.make_problem(32, 2048, 136, 64, seed=14)
    ks = [0, 1, 2, 3, 4, 5, 6, 7, 8, 63, 64, 65, 127, 128, 255, 256, 511, 512, 777, 1000,
          1023, 1024, 1500, 1535, 1536, 1600, 1800, 2000, 2040, 2045, 2046, 2047]
    p.x[:] = 0
    for m, k in enumerate(ks):
        p.x[m, k] = 1
    y = run(p, B.KERNEL_DECODE)
    w = oracle.dequant(p.qweight, p.scales, 64)
    for m, k in enumerate(ks):
        assert np.array_equal(y[m].view(np.uint16), w[k].view(np.uint16)), (m, k)


@pytest.mark.parametrize("kernel", [B.KERNEL_DECODE, B.KERNEL_PREFILL])
def test_one_hot_x_reproduces_dequantised_rows_bitwise(kernel):
    p = W.make_problem(16, 1024, 264, 32, seed=4)
    ks = [0, 1, 7, 8, 100, 511, 512, 777, 1000, 1023, 64, 65, 3, 300, 900, 31]
    p.x[:] = 0
    for m, k in enumerate(ks):
        p.x[m, k] = 1
    y = run(p, kernel)
    w = oracle.dequant(p.qweight, p.scales, 32)
    for m, k in enumerate(ks):
        assert np.array_equal(y[m].view(np.uint16), w[k].view(np.uint16)), (m, k)


@pytest.mark.parametrize("kernel", [B.KERNEL_DECODE, B.KERNEL_PREFILL])
@pytest.mark.parametrize("M", [1, 16])
def test_one_hot_x_every_scale_range_bitwise(kernel, M):
    """Scales from subnormal to 8, negative and zero, mixed within every group of
    columns: the decode kernel takes a six-operation form for 0 < s < 2^-4
    and the magic-number form otherwise; both must give the definition's
    rounded weight, so one-hot X reproduces the dequantised rows (bitwise
    where the weight is not zero; a zero weight must come out as a zero)."""
    K, N, G = 1024, 264, 128
    p = W.make_problem(M, K, N, G, seed=40 + M)
    rng = np.random.default_rng(40 + M)
    ranges = [(2.0 ** -24, 2.0 ** -14), (2.0 ** -14, 2.0 ** -4), (2.0 ** -4, 2.0 ** -4),
              (2.0 ** -4, 1.0), (1.0, 8.0)]
    pick = rng.integers(0, len(ranges), size=p.scales.shape)
    lo = np.array([r[0] for r in ranges])[pick]
    hi = np.array([r[1] for r in ranges])[pick]
    mag = np.exp(rng.uniform(np.log(lo), np.log(hi)))
    sign = np.where(rng.random(p.scales.shape) < 0.15, -1.0, 1.0)
    s = (sign * mag).astype(np.float16)
    s[rng.random(p.scales.shape) < 0.03] = 0
    p.scales[:] = s
    ks = rng.integers(0, K, size=M)
    p.x[:] = 0
    p.x[np.arange(M), ks] = 1
    y = run(p, kernel)
    w = oracle.dequant(p.qweight, p.scales, G)[ks]
    nz = w != 0
    assert np.array_equal(y[nz].view(np.uint16), w[nz].view(np.uint16))
    assert np.all(y[~nz] == 0)


def test_one_hot_x_pair_tile_bitwise():
    """256 tokens = both halves of a CTA-pair tile (rows 0..127 loaded by
    the even CTA, 128..255 by the odd one), 264 columns = two pairs, the
    second with a padding CTA: each output row is one dequantised weight
    row, bit for bit, so a token or column landing in the wrong place fails."""
    p = W.make_problem(256, 1024, 264, 32, seed=5)
    rng = np.random.default_rng(5)
    ks = rng.integers(0, 1024, size=256)
    p.x[:] = 0
    p.x[np.arange(256), ks] = 1
    y = run(p, B.KERNEL_PREFILL)
    w = oracle.dequant(p.qweight, p.scales, 32)
    for m in range(256):
        assert np.array_equal(y[m].view(np.uint16), w[ks[m]].view(np.uint16)), (m, ks[m])


@pytest.mark.parametrize("M", [129, 200, 256, 300])
def test_integer_exact_inputs_pair_tile_bitwise(M):
    rng = np.random.default_rng(M)
    p = W.make_problem(M, 2048, 392, 64, seed=M)
    p.x[:] = rng.integers(-4, 5, size=p.x.shape).astype(np.float16)
    p.scales[:] = np.float16(2.0 ** -6)
    y = run(p, B.KERNEL_PREFILL)
    ref = oracle.round_to_half(oracle.gemm(p.x, p.qweight, p.scales, 64))
    assert np.array_equal(y.view(np.uint16), ref.view(np.uint16))


@pytest.mark.parametrize("kernel", [B.KERNEL_DECODE, B.KERNEL_PREFILL])
@pytest.mark.parametrize("M", [1, 5, 16, 27, 32])
def test_integer_exact_inputs_match_bitwise(kernel, M):
    """x in {-4..4}, scales 2^-6: every product and partial sum is exact in
    FP32, so any summation order gives the oracle's value exactly."""
    rng = np.random.default_rng(M)
    p = W.make_problem(M, 2048, 136, 64, seed=M)
    p.x[:] = rng.integers(-4, 5, size=p.x.shape).astype(np.float16)
    p.scales[:] = np.float16(2.0 ** -6)
    y = run(p, kernel)
    ref = oracle.round_to_half(oracle.gemm(p.x, p.qweight, p.scales, 64))
    assert np.array_equal(y.view(np.uint16), ref.view(np.uint16))


@pytest.mark.parametrize("kernel,M", [(B.KERNEL_DECODE, 1), (B.KERNEL_DECODE, 16),
                                      (B.KERNEL_DECODE, 32), (B.KERNEL_PREFILL, 300)])
def test_deterministic(kernel, M):
    p = W.make_problem(M, 5120, 1024, 128, seed=9)
    a, b = run(p, kernel), run(p, kernel)
    assert np.array_equal(a.view(np.uint16), b.view(np.uint16))


def test_empty_m():
    p = W.make_problem(1, 512, 256, 128)
    _, qw, s = dev(p)
    x = torch.empty((0, 512), dtype=torch.float16, device="cuda")
    y = B.gemm(x, qw, s, 128)
    assert y.shape == (0, 256)


def test_maximum_k_and_n():
    p = W.make_problem(2, 1 << 16, 8, 1024, seed=11)
    y = run(p, B.KERNEL_DECODE)
    check_rows(p, y, [0, 1], "max K decode")
    y = run(p, B.KERNEL_PREFILL)
    check_rows(p, y, [0, 1], "max K prefill")
    q = W.make_problem(1, 16, 1 << 20, -1, seed=12)
    y = run(q)
    ref = oracle.gemm(q.x, q.qweight, q.scales, -1)
    assert rel_err(y, ref) <= TOL


# ---- the workloads at full size (sampled rows, every column) --------------------

def test_decode_up_projection_full():
    p = W.decode_up()
    assert B.select(1, 5120, 17408, 128)[0] == B.KERNEL_DECODE
    check_rows(p, run(p), [0], "decode up-projection M=1")


@pytest.mark.parametrize("M", [1, 2, 4, 8, 16, 32])
def test_decode_down_projection_sweep(M):
    p = W.decode_down(M)
    assert B.select(M, 17408, 5120, 32)[0] == B.KERNEL_DECODE
    check_rows(p, run(p), sample_rows(M, 3), f"decode down-projection M={M}")


@pytest.mark.parametrize("M", [33, 48, 64, 65])
def test_mid_m_full(M):
    # 48- and 64-token decode tiles up to M = 64, the pair prefill above
    p = W.prefill(M)
    kernel = B.select(M, 5120, 17408, 128)[0]
    assert kernel == (B.KERNEL_DECODE if M <= B.DECODE_MAX_M else B.KERNEL_PREFILL)
    check_rows(p, run(p), sample_rows(M, 3), f"mid-M up-projection M={M}")


@pytest.mark.parametrize("M", [512, 2048, 8192])
def test_prefill_full(M):
    p = W.prefill(M)
    assert B.select(M, 5120, 17408, 128)[0] == B.KERNEL_PREFILL
    check_rows(p, run(p), sample_rows(M, 3), f"prefill M={M}")


@pytest.mark.parametrize("G", W.GROUP_SIZES)
@pytest.mark.parametrize("M", [1, 16, 4096])
def test_group_sweep(G, M):
    p = W.group_sweep(G, M)
    check_rows(p, run(p), sample_rows(M, 2), f"square G={G} M={M}")


@pytest.mark.parametrize("which", [n for n, _, _, _ in W.LAYER_LINEARS])
@pytest.mark.parametrize("M", [1, 16, 4096])
def test_layer_linears(which, M):
    p = W.layer_linear(which, M)
    check_rows(p, run(p), sample_rows(M, 2), f"layer {which} M={M}")


# ---- several linears sharing X in one call ------------------------------------

def grouped_problem(M, K, Ns, G, seed):
    ps = [W.make_problem(M, K, n, G, seed=seed + i) for i, n in enumerate(Ns)]
    for q in ps[1:]:
        q.x[:] = ps[0].x  # one shared X
    return ps


def run_grouped(ps):
    x = torch.from_numpy(ps[0].x.view(np.int16)).view(torch.float16).cuda()
    qws = [torch.from_numpy(p.qweight).cuda() for p in ps]
    ss = [torch.from_numpy(p.scales.view(np.int16)).view(torch.float16).cuda() for p in ps]
    ys = B.gemm_grouped(x, qws, ss, ps[0].group)
    torch.cuda.synchronize()
    return [y.cpu().numpy() for y in ys]


# More column blocks than SMs at up to 16 tokens: one persistent wave, each CTA
# walking blocks c, c + 148, ... with two alternating accumulator sets.
PERSISTENT = [  # (M, K, Ns, G)
    (1, 512, (17408, 17408), 128),            # gate+up shape: 272 blocks, two per CTA
    (16, 528, (20480,), 32),                  # one wide linear, 160 blocks, ragged K
    (5, 1040, (40968,), 16),                  # 321 blocks (three for some CTAs), ragged N
    (3, 2048, (17408,) * 8, 64),              # 1088 blocks: seven or eight per CTA
    (9, 512, (8, 20480, 24, 136), -1),        # narrow and wide linears mixed, one group
]


@pytest.mark.parametrize("M,K,Ns,G", PERSISTENT)
def test_persistent_decode_parity(M, K, Ns, G):
    ps = grouped_problem(M, K, Ns, G, seed=M + K + len(Ns))
    ys = run_grouped(ps)
    for i, (p, y) in enumerate(zip(ps, ys)):
        ref = oracle.gemm(p.x, p.qweight, p.scales, G)
        err = rel_err(y, ref)
        print(f"[parity] persistent M={M} K={K} linear {i} N={p.N} G={G}: {err:.3e}")
        assert np.all(np.isfinite(y))
        assert err <= TOL
    assert B.device_error() == 0


@pytest.mark.parametrize("M", [1, 16])
def test_persistent_gate_up_equals_separate_calls_bitwise(M):
    # the same stages and accumulation order per column as one launch per linear
    ps = grouped_problem(M, 5120, (17408, 17408), 128, seed=M)
    ys = run_grouped(ps)
    for p, y in zip(ps, ys):
        assert np.array_equal(y.view(np.uint16), run(p).view(np.uint16))
    rows = sorted({0, M - 1})
    for p, y in zip(ps, ys):
        check_rows(p, y, rows, f"persistent gate+up M={M}")


@pytest.mark.parametrize("M,K,Ns,G", [
    (1, 2048, (264, 136, 8), 128), (5, 1040, (72, 200), 32), (16, 2560, (128, 128, 40, 8), 16),
    (32, 1536, (136, 264), -1), (33, 528, (64, 24), 128), (64, 2064, (136, 40, 8), 32),
    (65, 528, (64, 24), 128),                               # M = 65: one prefill launch each
    (3, 512, (8, 8, 8, 8, 8, 8, 8, 8), 64),                  # the most linears per call
])
def test_grouped_parity(M, K, Ns, G):
    ps = grouped_problem(M, K, Ns, G, seed=M + K)
    ys = run_grouped(ps)
    for i, (p, y) in enumerate(zip(ps, ys)):
        ref = oracle.gemm(p.x, p.qweight, p.scales, G)
        err = rel_err(y, ref)
        print(f"[parity] grouped M={M} K={K} linear {i} N={p.N} G={G}: {err:.3e}")
        assert err <= TOL


def test_grouped_one_hot_bitwise():
    ps = grouped_problem(16, 1024, (264, 136), 32, seed=21)
    ks = [0, 1, 7, 8, 100, 511, 512, 777, 1000, 1023, 64, 65, 3, 300, 900, 31]
    for p in ps:
        p.x[:] = 0
        for m, k in enumerate(ks):
            p.x[m, k] = 1
    ys = run_grouped(ps)
    for p, y in zip(ps, ys):
        w = oracle.dequant(p.qweight, p.scales, 32)
        for m, k in enumerate(ks):
            assert np.array_equal(y[m].view(np.uint16), w[k].view(np.uint16)), (m, k)


def test_grouped_single_linear_equals_plain_call_bitwise():
    p = W.make_problem(7, 4096, 392, 128, seed=22)
    (y,) = run_grouped([p])
    assert np.array_equal(y.view(np.uint16), run(p).view(np.uint16))


def test_grouped_qkv_full_size():
    ps = grouped_problem(1, 5120, (5120, 5120, 5120), 128, seed=23)
    ys = run_grouped(ps)
    for i, (p, y) in enumerate(zip(ps, ys)):
        check_rows(p, y, [0], f"grouped q/k/v linear {i}")


# ---- LoRA adapter on the linear path (gptq_w4a16_gemm_lora) --------------------

def run_lora(p, ad, t_out=False):
    x, qw, s = dev(p)
    a = torch.from_numpy(ad.lora_a.view(np.int16)).view(torch.float16).cuda()
    b = torch.from_numpy(ad.lora_b.view(np.int16)).view(torch.float16).cuda()
    t = torch.empty((p.M, ad.rank), dtype=torch.float16, device="cuda")
    y = B.gemm_lora(x, qw, s, p.group, a, b, t_work=t)
    torch.cuda.synchronize()
    assert B.device_error() == 0
    return (y.cpu().numpy(), t.cpu().numpy()) if t_out else y.cpu().numpy()


def check_t(t_gpu, x, lora_a):
    """T on the GPU is an FP32 sum rounded to FP16; the oracle's is a binary64
    sum rounded to FP16.  They may differ by the FP32 summation error bound
    (K-1) * 2^-24 * sum_k |x_k a_jk| plus one FP16 ulp of the result."""
    t_ref = oracle.lora_down(x, lora_a).astype(np.float64)
    K = x.shape[1]
    bound = (np.spacing(np.abs(t_ref).astype(np.float16)).astype(np.float64) +
             (K - 1) * 2.0 ** -24 *
             (np.abs(x.astype(np.float64)) @ np.abs(lora_a.astype(np.float64)).T))
    assert np.all(np.abs(t_gpu.astype(np.float64) - t_ref) <= bound), \
        "T differs from fp16(x . lora_a^T) by more than the FP32 summation bound"


@pytest.mark.parametrize("M,K,N,G,r", [
    (1, 512, 256, 128, 16), (5, 1024, 264, 32, 32), (16, 2048, 136, -1, 64),
    (33, 528, 136, 128, 48),            # 128-token pair tile, ragged K, rank not a multiple of 32
    (128, 1040, 392, 16, 128),          # odd number of column tiles (padding CTA)
    (200, 2048, 392, 64, 64),           # 256-token pair tile, odd CTA's half partly filled
    (300, 96, 264, 32, 256),            # largest rank, single k stage
    (2048, 5120, 512, 128, 32),         # several token tiles per cluster
])
def test_lora_parity(M, K, N, G, r):
    p = W.make_problem(M, K, N, G, seed=M + r)
    ad = W.make_adapter(K, N, r, seed=M + r)
    y, t = run_lora(p, ad, t_out=True)
    check_t(t, p.x, ad.lora_a)
    ref = oracle.gemm_lora(p.x, p.qweight, p.scales, G, ad.lora_a, ad.lora_b)
    err = rel_err(y, ref)
    print(f"[parity] lora M={M} K={K} N={N} G={G} r={r}: {err:.3e}")
    assert np.all(np.isfinite(y))
    assert err <= TOL


# K not a multiple of 256: the down-projection's last 256-k piece is short in
# both small-M forms (per-lane up to 8 tokens, staged rows from 9 to 32), and
# ranks 48 / 80 leave a ragged last 128-rank piece in the decode's adapter stage.
@pytest.mark.parametrize("M", [1, 5, 8, 9, 16, 32])
@pytest.mark.parametrize("K,r", [(528, 48), (1040, 80), (2064, 16)])
def test_lora_small_m_ragged_k(M, K, r):
    N, G = 264, 16 if K == 528 else 128
    p = W.make_problem(M, K, N, G, seed=M * 3 + K + r)
    ad = W.make_adapter(K, N, r, seed=M * 3 + K + r)
    y, t = run_lora(p, ad, t_out=True)
    check_t(t, p.x, ad.lora_a)
    ref = oracle.gemm_lora(p.x, p.qweight, p.scales, G, ad.lora_a, ad.lora_b)
    err = rel_err(y, ref)
    print(f"[parity] lora small M={M} K={K} N={N} G={G} r={r}: {err:.3e}")
    assert np.all(np.isfinite(y))
    assert err <= TOL


# Up to 32 tokens T is computed by CTAs of the layer's own launch on the SMs
# its column blocks leave free; with no SM free (148 column blocks or more) it
# comes from a launch of its own before the layer's.
@pytest.mark.parametrize("M,K,N,r", [(4, 512, 18944, 32), (20, 528, 19200, 16),
                                     (1, 1040, 20480, 128)])
def test_lora_without_free_sms_takes_the_separate_t_launch(M, K, N, r):
    p = W.make_problem(M, K, N, 64, seed=M + N)
    ad = W.make_adapter(K, N, r, seed=M + N)
    y, t = run_lora(p, ad, t_out=True)
    check_t(t, p.x, ad.lora_a)
    rows = sorted({0, M - 1})
    ref = oracle.gemm_lora_rows(p.x, p.qweight, p.scales, 64, ad.lora_a, ad.lora_b, rows)
    err = rel_err(y[rows], ref)
    print(f"[parity] lora, no free SM, M={M} K={K} N={N} r={r}: {err:.3e}")
    assert err <= TOL


@pytest.mark.parametrize("noalloc", [False, True])
def test_lora_fused_form_replayed_from_a_cuda_graph(noalloc):
    # the hand-over slot of T must start at zero on every replay
    M, K, N, G, r = 16, 2048, 1024, 128, 32
    p = W.make_problem(M, K, N, G, seed=5)
    ad = W.make_adapter(K, N, r, seed=5)
    x, qw, s = dev(p)
    a = torch.from_numpy(ad.lora_a.view(np.int16)).view(torch.float16).cuda()
    b = torch.from_numpy(ad.lora_b.view(np.int16)).view(torch.float16).cuda()
    t = torch.empty((M, r), dtype=torch.float16, device="cuda")
    ys = [torch.empty((M, N), dtype=torch.float16, device="cuda") for _ in range(3)]

    def call(y):
        if noalloc:
            B.gemm_lora_noalloc(x, qw, s, G, a, b, out=y)
        else:
            B.gemm_lora(x, qw, s, G, a, b, t_work=t, out=y)

    call(ys[0])
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for y in ys:
            call(y)
    for _ in range(4):
        for y in ys:
            y.zero_()
        graph.replay()
    torch.cuda.synchronize()
    assert B.device_error() == 0
    ref = oracle.gemm_lora(p.x, p.qweight, p.scales, G, ad.lora_a, ad.lora_b)
    for y in ys:
        assert rel_err(y.cpu().numpy(), ref) <= TOL


@pytest.mark.parametrize("M", [1, 40, 300])
def test_lora_integer_exact_inputs_bitwise(M):
    """Integer x and codes, power-of-two scales, sparse +-1 lora_a and lora_b
    in multiples of 2^-6: T and every product and partial sum are exact, so
    any summation order must reproduce the oracle's rounding bit for bit."""
    rng = np.random.default_rng(M)
    K, N, r = 1024, 264, 32
    p = W.make_problem(M, K, N, 64, seed=M)
    p.x[:] = rng.integers(-4, 5, size=p.x.shape).astype(np.float16)
    p.scales[:] = np.float16(2.0 ** -6)
    ad = W.make_adapter(K, N, r, seed=M)
    ad.lora_a[:] = (rng.integers(-1, 2, size=ad.lora_a.shape) *
                    (rng.random(ad.lora_a.shape) < 1 / 16)).astype(np.float16)
    ad.lora_b[:] = (rng.integers(-8, 9, size=ad.lora_b.shape) * 2.0 ** -6).astype(np.float16)
    y, t = run_lora(p, ad, t_out=True)
    t_ref = oracle.lora_down(p.x, ad.lora_a)
    assert np.array_equal(t.view(np.uint16), t_ref.view(np.uint16))
    ref = oracle.round_to_half(oracle.gemm_lora(p.x, p.qweight, p.scales, 64, ad.lora_a,
                                                ad.lora_b))
    assert np.array_equal(y.view(np.uint16), ref.view(np.uint16))


def test_lora_zero_adapter_equals_the_plain_layer_bitwise():
    """lora_b = 0 adds exact zeros to the same accumulator: above 32 tokens the
    plain call runs the same kernel, so Y must be identical."""
    p = W.make_problem(200, 2048, 392, 128, seed=21)
    ad = W.make_adapter(2048, 392, 32, seed=21)
    ad.lora_b[:] = 0
    assert np.array_equal(run_lora(p, ad).view(np.uint16), run(p).view(np.uint16))


def test_lora_one_hot_reproduces_weight_row_plus_t_column_bitwise():
    """x one-hot at k*, lora_a one-hot at k_j, lora_b one-hot at j_n: Y[m, n]
    is fp16(W[k*, n] + [k_{j_n} == k*]), with every step exact."""
    M, K, N, r = 64, 1024, 264, 32
    p = W.make_problem(M, K, N, 32, seed=8)
    rng = np.random.default_rng(8)
    ks = rng.integers(0, K, size=M)
    p.x[:] = 0
    p.x[np.arange(M), ks] = 1
    ad = W.make_adapter(K, N, r, seed=8)
    kj = rng.integers(0, K, size=r)
    kj[:8] = ks[:8]                     # some adapter rows hit the rows' own k
    ad.lora_a[:] = 0
    ad.lora_a[np.arange(r), kj] = 1
    jn = rng.integers(0, r, size=N)
    ad.lora_b[:] = 0
    ad.lora_b[np.arange(N), jn] = 1
    y = run_lora(p, ad)
    w = oracle.dequant(p.qweight, p.scales, 32).astype(np.float64)
    hit = (kj[jn][None, :] == ks[:, None]).astype(np.float64)
    ref = oracle.round_to_half(w[ks] + hit)
    assert np.array_equal(y.view(np.uint16), ref.view(np.uint16))


def test_lora_deterministic():
    p = W.make_problem(16, 5120, 1024, 128, seed=9)
    ad = W.make_adapter(5120, 1024, 64, seed=9)
    a, b = run_lora(p, ad), run_lora(p, ad)
    assert np.array_equal(a.view(np.uint16), b.view(np.uint16))


@pytest.mark.parametrize("M", [1, 16, 2048])
def test_lora_up_projection_full_size(M):
    p = W.prefill(M) if M > 16 else (W.decode_up() if M == 1 else W.make_problem(
        16, 5120, 17408, 128, seed=0))
    ad = W.make_adapter(p.K, p.N, 32, seed=M)
    y = run_lora(p, ad)
    rows = sorted({0, M // 2, M - 1})
    ref = oracle.gemm_lora_rows(p.x, p.qweight, p.scales, p.group, ad.lora_a, ad.lora_b, rows)
    err = rel_err(y[rows], ref)
    print(f"[parity] lora up-projection M={M}: {err:.3e} over rows {rows}")
    assert np.all(np.isfinite(y[rows]))
    assert err <= TOL


# ---- asymmetric zero points (gptq_w4a16_gemm_asym) ------------------------------

def run_asym(p, qzeros):
    x, qw, s = dev(p)
    qz = torch.from_numpy(qzeros).cuda()
    y = B.gemm_asym(x, qw, s, qz, p.group)
    torch.cuda.synchronize()
    assert B.device_error() == 0
    return y.cpu().numpy()


@pytest.mark.parametrize("M,K,N,G", [
    # decode kernel (M <= 64): 16- to 64-token tiles, groups of 16 and 32
    (1, 512, 256, 128), (5, 512, 256, 16), (7, 1024, 160, 32), (16, 2048, 288, -1),
    (24, 1040, 224, 128), (32, 6144, 96, 64), (33, 528, 128, 16), (64, 2064, 160, 32),
    (65, 528, 128, 16),                 # 128-token pair tile, ragged K and last group
    (130, 1040, 416, 64),               # 256-token pair tile, odd number of column tiles
    (300, 96, 224, 32),                 # a single k stage
    (2048, 5120, 512, 128),             # several token tiles per cluster
])
def test_asym_parity(M, K, N, G):
    p = W.make_problem(M, K, N, G, seed=M + K)
    qz = W.make_qzeros(p.scales.shape[0], N, seed=M + K)
    y = run_asym(p, qz)
    ref = oracle.gemm_asym(p.x, p.qweight, p.scales, qz, G)
    err = rel_err(y, ref)
    print(f"[parity] asym M={M} K={K} N={N} G={G}: {err:.3e}")
    assert np.all(np.isfinite(y))
    assert err <= TOL


@pytest.mark.parametrize("M,G", [(1, 128), (16, 32), (200, 128)])
def test_asym_with_every_zero_eight_equals_the_symmetric_layer_bitwise(M, G):
    """The symmetric call runs the same kernel (decode up to 32 tokens, the
    pair kernel above); with all zeros 8 the dequantised values are identical,
    hence Y too."""
    p = W.make_problem(M, 2048, 416, G, seed=31)
    qz = np.full((p.scales.shape[0], p.N // 8), 0x88888888, dtype=np.uint32).view(np.int32)
    assert np.array_equal(run_asym(p, qz).view(np.uint16), run(p).view(np.uint16))


@pytest.mark.parametrize("M", [1, 20, 40, 300])
def test_asym_integer_exact_inputs_bitwise(M):
    rng = np.random.default_rng(M)
    p = W.make_problem(M, 2048, 160, 64, seed=M)
    p.x[:] = rng.integers(-4, 5, size=p.x.shape).astype(np.float16)
    p.scales[:] = np.float16(2.0 ** -6)
    qz = W.make_qzeros(p.scales.shape[0], p.N, seed=M)
    y = run_asym(p, qz)
    ref = oracle.round_to_half(oracle.gemm_asym(p.x, p.qweight, p.scales, qz, 64))
    assert np.array_equal(y.view(np.uint16), ref.view(np.uint16))


def test_asym_one_hot_x_reproduces_dequantised_rows_bitwise():
    M, K, N, G = 64, 1024, 288, 32
    p = W.make_problem(M, K, N, G, seed=12)
    qz = W.make_qzeros(p.scales.shape[0], N, seed=12)
    ks = np.random.default_rng(12).integers(0, K, size=M)
    p.x[:] = 0
    p.x[np.arange(M), ks] = 1
    y = run_asym(p, qz)
    w = oracle.dequant_asym(p.qweight, p.scales, qz, G)
    assert np.array_equal(y.view(np.uint16), w[ks].view(np.uint16))


@pytest.mark.parametrize("M", [1, 2048])
def test_asym_up_projection_full_size(M):
    p = W.decode_up() if M == 1 else W.prefill(M)
    qz = W.make_qzeros(p.scales.shape[0], p.N, seed=M)
    y = run_asym(p, qz)
    rows = sorted({0, M // 2, M - 1})
    ref = oracle.gemm_asym_rows(p.x, p.qweight, p.scales, qz, p.group, rows)
    err = rel_err(y[rows], ref)
    print(f"[parity] asym up-projection M={M}: {err:.3e} over rows {rows}")
    assert err <= TOL
