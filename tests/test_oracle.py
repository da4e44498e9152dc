"""Pins for the CPU oracle (no GPU).

The oracle is checked against things other than itself: hand-derived binary16
encodings and worked examples (tests/golden/), numpy's independent binary16
conversion over every input, mathematical invariants of round-to-nearest-even,
closed forms of the layer, and numpy's einsum on tiny shapes.
"""
import numpy as np
import pytest

import oracle
from golden_io import binary16_cases, worked_examples

ALL_BITS = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
FINITE_BITS = ALL_BITS[(ALL_BITS & 0x7C00) != 0x7C00]


# ---- binary16 ------------------------------------------------------------

def test_half_to_double_matches_numpy_for_every_pattern():
    ours = np.array([oracle.half_to_double(int(b)) for b in ALL_BITS])
    ref = ALL_BITS.view(np.float16).astype(np.float64)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    # signed zeros are distinct patterns
    assert np.array_equal(np.signbit(ours[~nan]), np.signbit(ref[~nan]))


def test_round_trip_every_finite_half():
    vals = FINITE_BITS.view(np.float16).astype(np.float64)
    assert np.array_equal(oracle.round_to_half(vals).view(np.uint16), FINITE_BITS)


def test_golden_binary16_cases():
    for value, bits, note in binary16_cases():
        got = oracle.double_to_half_bits(value)
        assert got == bits, f"{value!r}: got {got:#06x}, want {bits:#06x} ({note})"


def test_ties_go_to_even_and_neighbours_to_nearest():
    # every pair of adjacent positive finite halves: the exact midpoint rounds
    # to the one with the even fraction; a hair either side rounds to the
    # nearer one.
    lo_bits = np.arange(0, 0x7BFF, dtype=np.uint16)
    lo = lo_bits.view(np.float16).astype(np.float64)
    hi = (lo_bits + 1).view(np.float16).astype(np.float64)
    mid = (lo + hi) / 2.0                      # exact in binary64
    even_is_lo = (lo_bits & 1) == 0
    want = np.where(even_is_lo, lo_bits, lo_bits + 1).astype(np.uint16)
    assert np.array_equal(oracle.round_to_half(mid).view(np.uint16), want)
    eps = (hi - lo) / 1024.0
    assert np.array_equal(oracle.round_to_half(mid - eps).view(np.uint16), lo_bits)
    assert np.array_equal(oracle.round_to_half(mid + eps).view(np.uint16), lo_bits + 1)
    # the same for negative values
    assert np.array_equal(oracle.round_to_half(-mid).view(np.uint16), want | 0x8000)


def test_overflow_threshold():
    assert oracle.double_to_half_bits(65519.999) == 0x7BFF
    assert oracle.double_to_half_bits(65520.0) == 0x7C00
    assert oracle.double_to_half_bits(1e300) == 0x7C00
    assert oracle.double_to_half_bits(-np.inf) == 0xFC00
    assert (oracle.double_to_half_bits(np.nan) & 0x7C00) == 0x7C00


# ---- packing ---------------------------------------------------------------

def test_pack_unpack_round_trip_all_bit_patterns():
    rng = np.random.default_rng(1)
    qw = rng.integers(-(2 ** 31), 2 ** 31, size=(6, 40), dtype=np.int64).astype(np.int32)
    qw[0, 0] = -1          # every nibble 15
    qw[0, 1] = -(2 ** 31)  # only the top nibble set (negative int32)
    qw[0, 2] = 0
    codes = oracle.unpack(qw)
    assert codes.shape == (48, 40) and codes.max() <= 15
    assert np.array_equal(oracle.pack(codes), qw)
    assert np.all(codes[0:8, 0] == 15)
    assert list(codes[0:8, 1]) == [0] * 7 + [8]


def test_single_nonzero_nibble_lands_on_one_weight():
    K, N = 32, 16
    for (k, n, c) in [(0, 0, 0), (7, 3, 15), (8, 15, 1), (31, 9, 12), (13, 2, 3)]:
        codes = np.full((K, N), 8, dtype=np.uint8)
        codes[k, n] = c
        qw = oracle.pack(codes)
        # the word holding it: row k // 8, nibble k % 8 (lowest nibble = lowest k)
        word = np.uint32(0x88888888) & ~np.uint32(0xF << (4 * (k % 8))) | np.uint32(c << (4 * (k % 8)))
        assert qw.view(np.uint32)[k // 8, n] == word
        scales = np.full((1, N), 0.5, dtype=np.float16)
        w = oracle.dequant(qw, scales, -1).astype(np.float64)
        expect = np.zeros((K, N))
        expect[k, n] = (c - 8) * 0.5
        assert np.array_equal(w, expect)


# ---- dequantisation ----------------------------------------------------------

def test_dequant_exhaustive_against_numpy_float16():
    """All 16 codes x every finite binary16 scale, against numpy's own rounding.

    (q - 8) * s is exact in float32 (a 4-bit integer times an 11-bit
    significand), so numpy's float32 -> float16 cast is the single rounding the
    definition asks for, implemented independently of the oracle."""
    scales = FINITE_BITS.view(np.float16).reshape(1, -1)
    N = scales.shape[1]
    qw = np.empty((2, N), dtype=np.int32)
    qw[0, :] = np.int32(0x76543210)           # codes 0..7 for k = 0..7
    qw[1, :] = np.uint32(0xFEDCBA98).view(np.int32)  # codes 8..15 for k = 8..15
    w = oracle.dequant(qw, scales, -1)
    with np.errstate(over="ignore"):  # -8 * 65504 overflows to -inf on both sides
        ref = ((np.arange(16, dtype=np.float32) - 8)[:, None]
               * scales.astype(np.float32)).astype(np.float16)
    assert np.array_equal(w.view(np.uint16), ref.view(np.uint16))


def test_dequant_group_indexing_and_ragged_tail():
    rng = np.random.default_rng(2)
    for K, G in [(64, 16), (64, 32), (528, 128), (40, 16), (48, 1024), (96, -1), (256, 256)]:
        N = 24
        codes = rng.integers(0, 16, size=(K, N)).astype(np.uint8)
        ng = oracle.num_groups(K, G)
        assert ng == (1 if G == -1 or G >= K else -(-K // G))
        scales = rng.uniform(1e-3, 2e-2, size=(ng, N)).astype(np.float16)
        w = oracle.dequant(oracle.pack(codes), scales, G).astype(np.float64)
        # independent group expansion: repeat each scale row over its rows
        step = K if G == -1 else G
        s_rows = np.repeat(scales.astype(np.float32), step, axis=0)[:K]
        ref = ((codes.astype(np.float32) - 8) * s_rows).astype(np.float16).astype(np.float64)
        assert np.array_equal(w, ref), (K, G)


def test_golden_worked_examples():
    for name, ex in worked_examples().items():
        qw, s, G = ex["qweight"], ex["scales"], ex["group"]
        if "codes" in ex:
            assert np.array_equal(oracle.unpack(qw).astype(np.int64), ex["codes"]), name
        if "W" in ex:
            assert np.array_equal(oracle.dequant(qw, s, G).astype(np.float64), ex["W"]), name
        for x, y in ex["xy"]:
            assert np.array_equal(oracle.gemm(x, qw, s, G), y), name


# ---- the layer -------------------------------------------------------------

def _rand_problem(rng, M, K, N, G):
    x = rng.standard_normal((M, K)).astype(np.float16)
    qw = rng.integers(0, 2 ** 32, size=(K // 8, N), dtype=np.uint64).astype(np.uint32).view(np.int32)
    s = rng.uniform(1e-3, 2e-2, size=(oracle.num_groups(K, G), N)).astype(np.float16)
    return x, qw, s


@pytest.mark.parametrize("M,K,N,G", [(1, 16, 8, -1), (2, 32, 16, 16), (3, 48, 24, 32),
                                     (4, 64, 8, 16), (1, 512, 256, 128), (4, 512, 256, 128),
                                     (5, 80, 40, 32)])
def test_gemm_against_numpy_einsum(M, K, N, G):
    rng = np.random.default_rng(M * 1000 + K + N)
    x, qw, s = _rand_problem(rng, M, K, N, G)
    y = oracle.gemm(x, qw, s, G)
    w = oracle.dequant(qw, s, G).astype(np.float64)
    ref = np.einsum("mk,kn->mn", x.astype(np.float64), w)
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)
    # brute force: the same sum written element by element
    m, n = M - 1, N // 2
    brute = sum(float(x[m, k]) * float(w[k, n]) for k in range(K))
    assert abs(brute - y[m, n]) <= 1e-12 * (1 + abs(brute))


@pytest.mark.parametrize("c", [0, 1, 7, 8, 9, 15])
def test_closed_form_all_codes_equal(c):
    """All codes c: Y = x . fp16((c-8) * s_expanded); c = 8 gives exactly 0."""
    rng = np.random.default_rng(c)
    M, K, N, G = 3, 96, 16, 32
    x = rng.standard_normal((M, K)).astype(np.float16)
    word = np.uint32(c * 0x11111111)
    qw = np.full((K // 8, N), word, dtype=np.uint32).view(np.int32)
    s = rng.uniform(1e-3, 2e-2, size=(K // G, N)).astype(np.float16)
    y = oracle.gemm(x, qw, s, G)
    w = ((c - 8) * np.repeat(s.astype(np.float32), G, axis=0)).astype(np.float16).astype(np.float64)
    ref = x.astype(np.float64) @ w
    assert np.allclose(y, ref, rtol=1e-12, atol=0)
    if c == 8:
        assert np.all(y == 0.0)
    # the same closed form with the scale factored out per group (exact when
    # (c-8)*s needs no rounding, true for c - 8 a power of two or zero)
    if c - 8 in (-8, 1, 0):
        per_group = sum((c - 8) * (x[:, g * G:(g + 1) * G].astype(np.float64).sum(axis=1)[:, None]
                                   * s[g].astype(np.float64)[None, :]) for g in range(K // G))
        assert np.allclose(y, per_group, rtol=1e-12, atol=1e-12)


def test_one_hot_x_reproduces_a_weight_row():
    rng = np.random.default_rng(3)
    x, qw, s = _rand_problem(rng, 4, 64, 32, 16)
    x[:] = 0
    for m, k in enumerate([0, 17, 40, 63]):
        x[m, k] = 1
    y = oracle.gemm(x, qw, s, 16)
    w = oracle.dequant(qw, s, 16).astype(np.float64)
    for m, k in enumerate([0, 17, 40, 63]):
        assert np.array_equal(y[m], w[k])


def test_group_minus_one_factors_out_the_scale():
    rng = np.random.default_rng(4)
    x, qw, _ = _rand_problem(rng, 2, 64, 16, -1)
    s = np.full((1, 16), 0.25, dtype=np.float16)  # power of two: (q-8)*s is exact
    y = oracle.gemm(x, qw, s, -1)
    q = oracle.unpack(qw).astype(np.float64) - 8
    assert np.allclose(y, 0.25 * (x.astype(np.float64) @ q), rtol=1e-12, atol=1e-12)
    # group >= K is the same single group
    assert np.array_equal(oracle.gemm(x, qw, s, 1024), y)


def test_entries_and_rows_match_full_gemm():
    rng = np.random.default_rng(5)
    x, qw, s = _rand_problem(rng, 6, 128, 40, 32)
    y = oracle.gemm(x, qw, s, 32)
    ms = [0, 5, 3, 3]
    ns = [0, 39, 17, 18]
    assert np.array_equal(oracle.gemm_entries(x, qw, s, 32, ms, ns), y[ms, ns])
    assert np.array_equal(oracle.gemm_rows(x, qw, s, 32, [5, 0]), y[[5, 0]])


def test_linearity_sanity():
    rng = np.random.default_rng(6)
    _, qw, s = _rand_problem(rng, 2, 64, 16, 16)
    # eighths in [-1/2, 1/2): 2*x1 + x2 is exact in binary16
    x1 = (rng.integers(-4, 4, size=(2, 64)) / 8).astype(np.float16)
    x2 = (rng.integers(-4, 4, size=(2, 64)) / 8).astype(np.float16)
    xs = (2 * x1.astype(np.float64) + x2.astype(np.float64)).astype(np.float16)
    y = oracle.gemm(xs, qw, s, 16)
    assert np.allclose(y, 2 * oracle.gemm(x1, qw, s, 16) + oracle.gemm(x2, qw, s, 16),
                       rtol=1e-12, atol=1e-12)


def test_validation_errors():
    qw = np.zeros((2, 8), dtype=np.int32)
    with pytest.raises(ValueError):
        oracle.dequant(qw, np.zeros((2, 8), dtype=np.float16), -1)
    with pytest.raises(IndexError):
        oracle.gemm_entries(np.zeros((1, 16), np.float16), qw, np.zeros((1, 8), np.float16),
                            -1, [1], [0])


# ---- LoRA adapter ----------------------------------------------------------

def _lora_problem(M, K, N, r, seed, G=32):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K)).astype(np.float16)
    qw = oracle.pack(rng.integers(0, 16, size=(K, N)).astype(np.uint8))
    s = rng.uniform(1e-3, 2e-2, size=(oracle.num_groups(K, G), N)).astype(np.float16)
    a = (rng.standard_normal((r, K)) * 0.05).astype(np.float16)
    b = (rng.standard_normal((N, r)) * 0.05).astype(np.float16)
    return x, qw, s, G, a, b


def test_lora_down_integer_inputs_match_numpy_bitwise():
    """Integer inputs: every product and sum is exact, so any summation order
    gives the same binary64 value and the FP16 rounding must agree."""
    rng = np.random.default_rng(1)
    x = rng.integers(-8, 9, size=(5, 64)).astype(np.float16)
    a = rng.integers(-8, 9, size=(16, 64)).astype(np.float16)
    ref = (x.astype(np.float64) @ a.astype(np.float64).T).astype(np.float16)
    assert np.array_equal(oracle.lora_down(x, a).view(np.uint16), ref.view(np.uint16))


def test_lora_down_random_within_one_ulp_of_numpy():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((7, 96)).astype(np.float16)
    a = rng.standard_normal((32, 96)).astype(np.float16)
    ours = oracle.lora_down(x, a).astype(np.float64)
    ref = (x.astype(np.float64) @ a.astype(np.float64).T)
    ulp = np.spacing(np.abs(ref).astype(np.float16)).astype(np.float64)
    assert np.all(np.abs(ours - ref) <= ulp)


@pytest.mark.parametrize("M,K,N,r", [(1, 16, 8, 16), (3, 48, 24, 16), (4, 64, 40, 32)])
def test_gemm_lora_against_numpy_einsum(M, K, N, r):
    x, qw, s, G, a, b = _lora_problem(M, K, N, r, seed=M + K)
    t = (x.astype(np.float64) @ a.astype(np.float64).T).astype(np.float16)
    w = oracle.dequant(qw, s, G).astype(np.float64)
    ref = np.einsum("mk,kn->mn", x.astype(np.float64), w) + \
        np.einsum("mj,nj->mn", t.astype(np.float64), b.astype(np.float64))
    ours = oracle.gemm_lora(x, qw, s, G, a, b)
    assert np.allclose(ours, ref, rtol=1e-12, atol=1e-12)


def test_lora_zero_up_projection_leaves_the_layer_unchanged():
    x, qw, s, G, a, b = _lora_problem(3, 64, 16, 16, seed=3)
    b[:] = 0
    assert np.array_equal(oracle.gemm_lora(x, qw, s, G, a, b), oracle.gemm(x, qw, s, G))


def test_lora_one_hot_down_copies_x_columns():
    """lora_a rows one-hot at k_j: T[:, j] is exactly x[:, k_j]."""
    x, qw, s, G, a, b = _lora_problem(4, 64, 16, 16, seed=4)
    ks = np.random.default_rng(4).integers(0, 64, size=16)
    a[:] = 0
    a[np.arange(16), ks] = 1
    t = oracle.lora_down(x, a)
    assert np.array_equal(t.view(np.uint16), x[:, ks].view(np.uint16))


def test_lora_one_hot_up_adds_one_t_column():
    """lora_b rows one-hot at j_n: Y_lora - Y is exactly T[:, j_n]."""
    x, qw, s, G, a, b = _lora_problem(4, 64, 24, 16, seed=5)
    js = np.random.default_rng(5).integers(0, 16, size=24)
    b[:] = 0
    b[np.arange(24), js] = 1
    t = oracle.lora_down(x, a).astype(np.float64)
    delta = oracle.gemm_lora(x, qw, s, G, a, b) - oracle.gemm(x, qw, s, G)
    assert np.array_equal(delta, t[:, js])


def test_lora_rank_one_is_an_outer_product():
    x, qw, s, G, a, b = _lora_problem(5, 32, 16, 1, seed=6)
    t = oracle.lora_down(x, a).astype(np.float64)
    delta = oracle.gemm_lora(x, qw, s, G, a, b) - oracle.gemm(x, qw, s, G)
    assert np.allclose(delta, np.outer(t[:, 0], b[:, 0].astype(np.float64)), rtol=0, atol=1e-12)


def test_gemm_lora_rows_match_the_whole_result():
    x, qw, s, G, a, b = _lora_problem(6, 64, 16, 16, seed=7)
    full = oracle.gemm_lora(x, qw, s, G, a, b)
    rows = oracle.gemm_lora_rows(x, qw, s, G, a, b, [5, 0, 3])
    assert np.array_equal(rows, full[[5, 0, 3]])


# ---- asymmetric zero points ----------------------------------------------------

def _asym_problem(M, K, N, G, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K)).astype(np.float16)
    qw = oracle.pack(rng.integers(0, 16, size=(K, N)).astype(np.uint8))
    ng = oracle.num_groups(K, G)
    s = rng.uniform(1e-3, 2e-2, size=(ng, N)).astype(np.float16)
    z = rng.integers(0, 16, size=(ng, N))
    return x, qw, s, oracle.pack_zeros(z), z


def test_asym_with_every_zero_eight_is_the_symmetric_layer():
    x, qw, s, _, _ = _asym_problem(4, 96, 24, 32, seed=1)
    qz = oracle.pack_zeros(np.full(s.shape, 8))
    assert np.array_equal(oracle.dequant_asym(qw, s, qz, 32).view(np.uint16),
                          oracle.dequant(qw, s, 32).view(np.uint16))
    assert np.array_equal(oracle.gemm_asym(x, qw, s, qz, 32), oracle.gemm(x, qw, s, 32))


def test_asym_dequant_every_code_and_zero_against_numpy():
    """All 16 x 16 (code, zero) pairs with many scales: (q - z) * s is exact in
    float32 (5-bit integer times an 11-bit significand), so numpy's float32
    product rounded by numpy to float16 is the independent reference."""
    rng = np.random.default_rng(2)
    svals = np.concatenate([rng.uniform(1e-4, 8.0, 62), [2.0 ** -14, 65504.0]]).astype(np.float16)
    K, N = 16 * 16, 64                       # row k: code k % 16; group k // 16: zero (k // 16)
    codes = np.tile((np.arange(K) % 16)[:, None], (1, N)).astype(np.uint8)
    qw = oracle.pack(codes)
    s = np.tile(svals[None, :], (16, 1))     # group g: the same 64 scales
    z = np.tile(np.arange(16)[:, None], (1, N))
    w = oracle.dequant_asym(qw, s, oracle.pack_zeros(z), 16)
    q = codes.astype(np.float32)
    zz = np.repeat(z, 16, axis=0).astype(np.float32)
    with np.errstate(over="ignore"):  # products beyond the FP16 range become inf, as defined
        ref = ((q - zz) * np.repeat(s, 16, axis=0).astype(np.float32)).astype(np.float16)
    assert np.array_equal(w.view(np.uint16), ref.view(np.uint16))


def test_asym_zero_nibble_lands_on_one_group_and_column():
    x, qw, s, _, _ = _asym_problem(2, 128, 32, 32, seed=3)
    base = np.zeros(s.shape, dtype=np.int64)
    w0 = oracle.dequant_asym(qw, s, oracle.pack_zeros(base), 32)
    z = base.copy()
    z[2, 13] = 5
    w1 = oracle.dequant_asym(qw, s, oracle.pack_zeros(z), 32)
    diff = np.argwhere(w0.view(np.uint16) != w1.view(np.uint16))
    assert diff.size and set(diff[:, 1]) == {13} and set(diff[:, 0] // 32) == {2}


def test_asym_code_equal_to_zero_gives_exact_zero():
    K, N, G = 64, 16, 16
    rng = np.random.default_rng(4)
    z = rng.integers(0, 16, size=(K // G, N))
    codes = np.repeat(z, G, axis=0).astype(np.uint8)
    s = rng.uniform(1e-3, 2e-2, size=z.shape).astype(np.float16)
    x = rng.standard_normal((3, K)).astype(np.float16)
    y = oracle.gemm_asym(x, oracle.pack(codes), s, oracle.pack_zeros(z), G)
    assert np.array_equal(y, np.zeros_like(y))


@pytest.mark.parametrize("M,K,N,G", [(1, 16, 8, -1), (3, 48, 24, 16), (2, 96, 40, 32)])
def test_gemm_asym_against_numpy_einsum(M, K, N, G):
    x, qw, s, qz, z = _asym_problem(M, K, N, G, seed=M + K)
    codes = oracle.unpack(qw).astype(np.float64)
    g = np.arange(K) // (K if G == -1 else G)
    w = ((codes - z[g]) * s[g].astype(np.float64)).astype(np.float16).astype(np.float64)
    ref = np.einsum("mk,kn->mn", x.astype(np.float64), w)
    assert np.allclose(oracle.gemm_asym(x, qw, s, qz, G), ref, rtol=1e-12, atol=1e-12)


# ---- act order (per-channel group index) --------------------------------------

def _np_codes(qw):
    """Codes [K, N] from qweight by numpy shifts (independent of the oracle)."""
    u = np.asarray(qw).view(np.uint32)
    K = u.shape[0] * 8
    k = np.arange(K)
    return ((u[k // 8] >> (4 * (k % 8))[:, None].astype(np.uint32)) & 0xF).astype(np.int64)


def _np_pack(codes):
    """Codes [K, N] -> qweight [K/8, N] by numpy (independent of the oracle)."""
    c = np.asarray(codes, dtype=np.uint32)
    words = np.zeros((c.shape[0] // 8, c.shape[1]), dtype=np.uint32)
    for j in range(8):
        words |= (c[j::8] & 0xF) << (4 * j)
    return words.view(np.int32)


def _np_dequant_gidx(qw, s, g_idx):
    """(q - 8) * s[g_idx[k]] is exact in float32; numpy rounds it to float16."""
    q = _np_codes(qw).astype(np.float32)
    with np.errstate(over="ignore"):  # products beyond the FP16 range become inf, as defined
        return ((q - 8.0) * np.asarray(s)[np.asarray(g_idx)].astype(np.float32)).astype(np.float16)


def _gidx_problem(M, K, N, ng, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K)).astype(np.float16)
    qw = _np_pack(rng.integers(0, 16, size=(K, N)))
    s = rng.uniform(1e-3, 2e-2, size=(ng, N)).astype(np.float16)
    g = rng.integers(0, ng, size=K).astype(np.int32)
    return x, qw, s, g


@pytest.mark.parametrize("K,G", [(128, 16), (512, 128), (528, 128), (96, -1)])
def test_gidx_with_consecutive_groups_is_the_plain_layer(K, G):
    rng = np.random.default_rng(K)
    N = 24
    qw = _np_pack(rng.integers(0, 16, size=(K, N)))
    ng = oracle.num_groups(K, G)
    s = rng.uniform(1e-3, 2e-2, size=(ng, N)).astype(np.float16)
    x = rng.standard_normal((3, K)).astype(np.float16)
    g = np.arange(K) // (K if G == -1 else G)
    assert np.array_equal(oracle.dequant_gidx(qw, s, g).view(np.uint16),
                          oracle.dequant(qw, s, G).view(np.uint16))
    assert np.array_equal(oracle.gemm_gidx(x, qw, s, g), oracle.gemm(x, qw, s, G))


def test_gidx_dequant_against_numpy_float16():
    """Every code, scattered group indices, ordinary and extreme scales."""
    rng = np.random.default_rng(5)
    K, N, ng = 256, 64, 7
    svals = np.concatenate([rng.uniform(1e-4, 8.0, (ng, N - 2)),
                            np.full((ng, 1), 2.0 ** -14), np.full((ng, 1), 65504.0)], axis=1)
    s = svals.astype(np.float16)
    qw = _np_pack(np.tile((np.arange(K) % 16)[:, None], (1, N)))
    g = rng.integers(0, ng, size=K)
    assert np.array_equal(oracle.dequant_gidx(qw, s, g).view(np.uint16),
                          _np_dequant_gidx(qw, s, g).view(np.uint16))


def test_gemm_gidx_against_numpy_einsum():
    for M, K, N, ng in ((1, 16, 8, 1), (3, 64, 24, 5), (2, 160, 40, 9)):
        x, qw, s, g = _gidx_problem(M, K, N, ng, seed=M + K)
        w = _np_dequant_gidx(qw, s, g).astype(np.float64)
        ref = np.einsum("mk,kn->mn", x.astype(np.float64), w)
        assert np.allclose(oracle.gemm_gidx(x, qw, s, g), ref, rtol=1e-12, atol=1e-12)


def test_gidx_channel_permutation_leaves_y_unchanged():
    """Permuting the input channels of x, the qweight rows and g_idx together
    is the same layer (only the order of the sum over k changes)."""
    x, qw, s, g = _gidx_problem(4, 128, 32, 6, seed=9)
    perm = np.random.default_rng(9).permutation(128)
    qw_p = _np_pack(_np_codes(qw)[perm])
    y = oracle.gemm_gidx(x, qw, s, g)
    y_p = oracle.gemm_gidx(np.ascontiguousarray(x[:, perm]), qw_p, s, g[perm])
    assert np.allclose(y_p, y, rtol=1e-12, atol=1e-12)
    w_p = oracle.dequant_gidx(qw_p, s, g[perm])
    assert np.array_equal(w_p.view(np.uint16), oracle.dequant_gidx(qw, s, g)[perm].view(np.uint16))


def test_gidx_one_entry_moves_one_weight_row():
    x, qw, s, g = _gidx_problem(2, 64, 16, 4, seed=11)
    w0 = oracle.dequant_gidx(qw, s, g)
    g1 = g.copy()
    g1[37] = (g[37] + 1) % 4
    w1 = oracle.dequant_gidx(qw, s, g1)
    rows = set(np.argwhere(w0.view(np.uint16) != w1.view(np.uint16))[:, 0])
    assert rows == {37}


def test_gidx_rejects_bad_indices():
    x, qw, s, g = _gidx_problem(1, 32, 8, 3, seed=12)
    for bad in (-1, 3):
        gb = g.copy()
        gb[5] = bad
        with pytest.raises(ValueError):
            oracle.dequant_gidx(qw, s, gb)
        with pytest.raises(ValueError):
            oracle.gemm_gidx(x, qw, s, gb)
    with pytest.raises(ValueError):
        oracle.dequant_gidx(qw, s, g[:-1])
    with pytest.raises(TypeError):
        oracle.dequant_gidx(qw, s, g.astype(np.float64))


# ---- thread-count independence ------------------------------------------------
# OpenMP threads only split independent outputs; each output's sum runs
# sequentially in k.  So the result must not depend on the thread count: one
# thread and every core give bitwise-identical outputs.

def test_results_do_not_depend_on_thread_count():
    import os
    rng = np.random.default_rng(7)
    M, K, N, G, r = 5, 528, 264, 128, 48
    x = rng.standard_normal((M, K)).astype(np.float16)
    qw = rng.integers(-2**31, 2**31, size=(K // 8, N), dtype=np.int64).astype(np.int32)
    sc = rng.uniform(1e-3, 2e-2, size=(oracle.num_groups(K, G), N)).astype(np.float16)
    la = (rng.standard_normal((r, K)) / np.sqrt(K)).astype(np.float16)
    lb = (rng.standard_normal((N, r)) * 0.05).astype(np.float16)
    zc = rng.integers(0, 16, size=(oracle.num_groups(K, G), N)).astype(np.uint8)
    qz = oracle.pack_zeros(zc)
    ms = np.array([0, 2, 4], dtype=np.int64)
    ns = rng.integers(0, N, size=40).astype(np.int64)
    mm = rng.integers(0, M, size=40).astype(np.int64)

    def run_all():
        return (oracle.gemm(x, qw, sc, G), oracle.gemm_rows(x, qw, sc, G, ms),
                oracle.gemm_entries(x, qw, sc, G, mm, ns), oracle.lora_down(x, la),
                oracle.gemm_lora(x, qw, sc, G, la, lb), oracle.gemm_asym(x, qw, sc, qz, G),
                oracle.dequant(qw, sc, G))

    saved = oracle.get_threads()
    many = max(4, os.cpu_count() or 4)
    try:
        oracle.set_threads(1)
        assert oracle.get_threads() == 1
        one = run_all()
        oracle.set_threads(many)
        assert oracle.get_threads() == many
        lots = run_all()
    finally:
        oracle.set_threads(saved)
    for a, b in zip(one, lots):
        assert a.dtype == b.dtype and a.shape == b.shape
        assert a.tobytes() == b.tobytes()
