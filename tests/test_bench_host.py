"""Host logic of bench.py that needs no GPU: the kernel-code digest that keeps
recorded ncu traffic attached to the kernels it was measured on."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_code_only_drops_comments_keeps_literals():
    src = 'int a = 1; // one\n/* block\n comment */ const char* s = "x // y /* z */";\n'
    assert bench._code_only(src) == 'int a = 1; const char* s = "x // y /* z */";'


def test_code_only_collapses_blank_space_only():
    assert bench._code_only("a  +\n\n b") == bench._code_only("a + b")
    assert bench._code_only("a+b") != bench._code_only("a + b")


def _digest_of(tmp_path, files):
    csrc = tmp_path / "int4_weight_only_gptq_b200" / "csrc"
    csrc.mkdir(parents=True)
    for name, text in files.items():
        (csrc / name).write_text(text)
    old = bench.ROOT
    bench.ROOT = str(tmp_path)
    try:
        return bench.kernel_source_digest()
    finally:
        bench.ROOT = old


def test_digest_ignores_comment_edits_and_sees_code_edits(tmp_path):
    base = {"k.cu": "__global__ void k(int* p) { p[0] = 1; }  // store\n", "h.cuh": "#pragma once\n"}
    commented = {"k.cu": "// a kernel\n__global__ void k(int* p) { p[0] = 1; }\n",
                 "h.cuh": "#pragma once  /* header */\n"}
    changed = {"k.cu": "__global__ void k(int* p) { p[0] = 2; }\n", "h.cuh": "#pragma once\n"}
    d0 = _digest_of(tmp_path / "a", base)
    assert _digest_of(tmp_path / "b", commented) == d0
    assert _digest_of(tmp_path / "c", changed) != d0



def test_reference_arm_prints_the_contract_line():
    """`bench.py --impl reference` (the oracle on the host cores) prints one JSON
    line with the contract's keys, its e2e equal to its own value with no
    host-device traffic, and a cpu_baseline describing the run."""
    import json
    import subprocess
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"], capture_output=True, text=True,
                       timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["n_gpus"] == 1 and d["steps"] == 1
    assert d["warmup"] >= 3  # the contract's minimum is applied
    assert d["value"] > 0 and d["higher_is_better"] is True
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1
    assert "workload" in d["config"]


def test_parity_on_rows_measures_the_required_error():
    import numpy as np
    ref = np.array([[1.0, -3.0, 0.0], [10.0, 0.5, -0.25]])
    y = np.zeros((4, 3), dtype=np.float16)
    y[1] = ref[0]
    y[3] = ref[1]
    y[3, 0] = 10.5  # off by 0.5 where |y_ref| = 10: 0.5 / 11
    out = bench.parity_on_rows(y, ref, [1, 3])
    assert abs(out["max_rel_err"] - 0.5 / 11) < 1e-12
    assert out["within"] is False and out["rows"] == [1, 3] and out["bound"] == 1e-2
    y[3, 0] = 10.0
    out = bench.parity_on_rows(y, ref, [1, 3])
    assert out["max_rel_err"] == 0.0 and out["within"] is True


def test_parity_on_rows_flags_non_finite_and_shape_errors():
    import numpy as np
    import pytest
    ref = np.zeros((1, 2))
    y = np.array([[np.inf, 0.0]], dtype=np.float16)
    assert bench.parity_on_rows(y, ref, [0])["within"] is False
    with pytest.raises(ValueError):
        bench.parity_on_rows(np.zeros((2, 3)), ref, [0])


def test_cpu_baseline_reports_parity_of_a_given_output():
    """The CPU leg compares the output it is handed with its own oracle rows:
    the oracle's FP16-rounded result is within the bound, a perturbed one is
    caught."""
    import numpy as np
    import oracle
    from int4_weight_only_gptq_b200 import workloads as W
    p = W.tiny(4)
    y = oracle.gemm(p.x, p.qweight, p.scales, p.group).astype(np.float16)
    cb = bench.cpu_baseline(p, p.algorithmic_bytes, "hbm", budget_s=0.01, y_gpu=y)
    assert cb["parity"]["within"] and cb["parity"]["max_rel_err"] < 1e-3
    assert cb["parity"]["rows"] == [0, 1, 2, 3]
    y[2, 5] = np.float16(float(y[2, 5]) + 1.0)
    cb = bench.cpu_baseline(p, p.algorithmic_bytes, "hbm", budget_s=0.01, y_gpu=y)
    assert cb["parity"]["max_rel_err"] > 0.1 and not cb["parity"]["within"]
    assert "parity" not in bench.cpu_baseline(p, p.algorithmic_bytes, "hbm", budget_s=0.01)


def test_headline_keys_pick_the_metric_halves_from_the_sweep():
    sweep = {"prefill_M2048": {"ms": 0.25}, "prefill_M8192": {"ms": 0.95},
             "decode_down_M1": {"ms": 0.017}, "decode_down_M16": {"ms": 0.018},
             "midm_up_M64": {"ms": 0.02}, "square_g128_M1": {"ms": 0.01}}
    h = bench.headline_keys(sweep)
    assert set(h) == {"prefill", "decode_down", "midm"}
    assert h["prefill"] == {"M2048": {"ms": 0.25}, "M8192": {"ms": 0.95}}
    assert h["decode_down"]["M16"] == {"ms": 0.018}
    assert h["midm"] == {"M64": {"ms": 0.02}}


def test_roofline_entries():
    from int4_weight_only_gptq_b200 import workloads as W
    p = W.decode_up()
    e = bench.hbm_entry(p, p.algorithmic_bytes / 6523.3e9 * 1e3, 6523.3)
    assert abs(e["roofline"]["frac"] - 1.0) < 1e-3 and e["roofline"]["unit"] == "GB/s"
    q = W.make_problem(2048, 5120, 17408, 128, seed=0)
    t = bench.tensor_entry(q, q.flops / 1637.3e12 * 1e3, 1637.3)
    assert abs(t["roofline"]["frac"] - 1.0) < 1e-3 and t["roofline"]["unit"] == "TFLOP/s"


def test_cpu_model_is_named():
    assert isinstance(bench.cpu_model(), str) and bench.cpu_model()
