"""bench.py's reference arm (the oracle timed on the host's cores) runs without a GPU and prints
one JSON line with the keys the benchmark contract requires."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "0"], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, out.stdout
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "tokens/s" and d["steps"] == 1
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"] and d["cpu_baseline"]["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert "workload" in d["config"]


def test_bench_selection_report_helpers():
    """The bench's selection report: the CPU baseline's sampled descents compared with given rows
    (equal rows pass, a doctored row is counted as differing and not admissible), and the needle
    recall count."""
    import numpy as np
    import bench
    import workloads
    w = workloads.Workload("bench-needle", 1, 8, 2, 256 * 64, 256 * 64, 64, 64, 4, 16, 1, "needle", 18)
    cpu = bench.oracle_sample(w, budget_s=1.0)
    sample = cpu.pop("_sample")
    nqb = w.seq_q // w.block
    rows = np.full((nqb, w.topk), -1, dtype=np.int32)
    for i, sel in sample["sel"].items():
        rows[i, :len(sel)] = sel
    rep = bench.check_sampled_selection(w, sample, rows)
    assert rep["rows"] == len(sample["sel"]) and rep["differ"] == 0
    i = max(sample["sel"], key=lambda t: len(sample["sel"][t]))
    assert len(sample["sel"][i]) == w.topk
    rows[i, 0] = rows[i, 1]            # a repeated block
    rep = bench.check_sampled_selection(w, sample, rows)
    assert rep["differ"] == 1 and rep["differ_admissible"] == 0
    idx = np.full((1, w.heads_kv, nqb, w.topk), -1, dtype=np.int32)
    for kvh in range(w.heads_kv):
        for n, (qi, j) in enumerate(workloads.needles(w, 0, kvh)):
            if n % 2 == 0:
                idx[0, kvh, qi, 0] = j
    rec = bench.needle_recall(w, idx)
    assert rec["planted"] == 16 * w.heads_kv and rec["selected"] == 8 * w.heads_kv


def test_bench_names_the_attention_kernel_the_library_launches():
    """The roofline's kernel label follows the launcher's rule: two 128-row tiles per CTA for the
    GQA groups of 64-token blocks, two units per CTA for units of at most 128 rows."""
    import bench
    import workloads
    import block_sparse_long_pisa_b200 as pisa
    name = lambda n, per=0: bench.attention_kernel_name(pisa.Shape.of(workloads.WORKLOADS[n], select_per_qhead=per))
    assert name("gqa128k") == "attn_prefill_kernel<128,64,2>"
    assert name("gqa128k", 1) == "attn_prefill_dual_kernel<128,64>"
    assert name("causal32k") == "attn_prefill_dual_kernel<128,64>"
    assert name("long1m") == "attn_prefill_dual_kernel<128,128>"
    assert name("tiny") == "attn_prefill_dual_kernel<64,64>"
