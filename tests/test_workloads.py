"""The seeded input generator: shapes, determinism, distributions (no GPU)."""
import numpy as np

from int4_weight_only_gptq_b200 import workloads as W


def test_tiny_shapes_and_determinism():
    a, b = W.tiny(4), W.tiny(4)
    assert a.x.shape == (4, 512) and a.x.dtype == np.float16
    assert a.qweight.shape == (64, 256) and a.qweight.dtype == np.int32
    assert a.scales.shape == (4, 256) and a.scales.dtype == np.float16
    assert np.array_equal(a.x.view(np.uint16), b.x.view(np.uint16))
    assert np.array_equal(a.qweight, b.qweight)
    assert np.array_equal(a.scales.view(np.uint16), b.scales.view(np.uint16))
    c = W.make_problem(4, 512, 256, 128, seed=1)
    assert not np.array_equal(a.qweight, c.qweight)


def test_scale_ranges_and_code_uniformity():
    p = W.decode_down(1)
    s = p.scales.astype(np.float64)
    assert p.scales.shape == (544, 5120)
    assert s.min() >= 4.9e-4 and s.max() <= 5.01e-2
    # log-uniform: the median sits near the geometric mean 5e-3
    assert 3.5e-3 < np.median(s) < 7e-3
    nib = (p.qweight.view(np.uint32)[:64, :256, None] >> (4 * np.arange(8, dtype=np.uint32))) & 0xF
    counts = np.bincount(nib.ravel(), minlength=16)
    assert counts.min() > 0.8 * counts.mean()
    u = W.tiny(1).scales.astype(np.float64)
    assert u.min() >= 0.99e-3 and u.max() <= 2.01e-2


def test_outlier_channels():
    p = W.make_problem(4, 17408, 8, 32, outlier_frac=0.01, scale_dist="log_uniform",
                       scale_range=(5e-4, 5e-2))
    big = np.abs(p.x.astype(np.float64)).max(axis=0) > 6.0
    # 174 channels are scaled x20, the others are N(0,1): nearly all of the
    # scaled ones exceed 6 in at least one of 4 rows, almost none of the rest do
    assert 150 <= big.sum() <= 180
    assert int(np.floor(0.01 * 17408)) == 174


def test_group_counts():
    assert W.num_groups(5120, -1) == 1
    assert W.num_groups(5120, 16) == 320
    assert W.num_groups(528, 128) == 5
    assert W.num_groups(64, 1024) == 1
    for g in W.GROUP_SIZES:
        p = W.group_sweep(g, 1)
        assert p.scales.shape == (W.num_groups(5120, g), 5120)


def test_algorithmic_bytes():
    p = W.decode_up()
    assert p.algorithmic_bytes == 46_002_176
    assert W.prefill(512).flops == 2 * 512 * 5120 * 17408


def test_gidx_generator():
    # consecutive indices are the plain layer's groups
    assert np.array_equal(W.make_gidx(40, 16, kind="consecutive"), np.arange(40) // 16)
    # act order: every group holds exactly `group` channels (the last the rest)
    g = W.make_gidx(528, 128, seed=5, kind="perm")
    assert g.dtype == np.int32 and g.shape == (528,)
    assert np.bincount(g).tolist() == [128, 128, 128, 128, 16]
    assert not np.array_equal(g, np.arange(528) // 128)
    # random: indices in range, seeded
    r = W.make_gidx(1040, 32, seed=1, kind="random")
    assert r.min() >= 0 and r.max() < 33
    assert np.array_equal(r, W.make_gidx(1040, 32, seed=1, kind="random"))
    # one group (group -1): every index 0
    assert not W.make_gidx(64, -1, kind="perm").any()
