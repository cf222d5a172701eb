"""bench.py's reference arm on the CPU: one JSON line with the keys of the
measurement contract (the oracle timed on the host, a bounded sample)."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_contract_line():
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "LOCAL_RANK", "WORLD_SIZE")}
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], env=env, capture_output=True, text=True, timeout=600)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [ln for ln in p.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1, lines
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["value"] > 0 and d["unit"] == "TOPS" and d["higher_is_better"] is True
    assert d["steps"] == 1 and d["warmup"] == 3 and d["n_gpus"] == 1
    assert d["config"]["workload"].startswith("flux")
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    e = d["e2e"]
    assert e["value"] == d["value"] and e["unit"] == d["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0


def test_softmax_roofline_takes_the_lower_ceiling():
    """The attention kernel against its softmax ceilings: the exponential unit
    (measured rate / exponentials per score) and the issue slots (four warp
    instructions per SM and clock over the kernel's warp instructions per
    score); achieved scores per second over the lower one."""
    sys.path.insert(0, ROOT)
    import bench
    from quantized_attention_qk_b200.inputs import WORKLOADS

    w = WORKLOADS["flux"]
    scores = w.B * w.H * w.N * w.N
    r = bench._softmax_roofline(w, attn_ms=0.2, kept=1.0, ex2_rate=4.0e12, sm_mhz=2000.0, sms=148,
                                instr_per_score=0.25)
    assert abs(r["achieved"] - scores / 0.2e-3 / 1e12) < 1e-4
    assert abs(r["ceilings"]["ex2"] - 4.0 / bench.EX2_PER_SCORE) < 1e-4
    assert abs(r["ceilings"]["issue"] - 4 * 148 * 2.0e9 / 0.25 / 1e12) < 1e-4
    assert r["peak"] == min(r["ceilings"].values())
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-3
    # without an instruction count only the exponential ceiling is stated
    r2 = bench._softmax_roofline(w, 0.2, 1.0, 4.0e12, 2000.0, 148, None)
    assert set(r2["ceilings"]) == {"ex2"} and r2["peak"] == r2["ceilings"]["ex2"]
    # a kept fraction (block-sparse) scales the scores the kernel computed
    r3 = bench._softmax_roofline(w, 0.2, 0.5, 4.0e12, 2000.0, 148, None)
    assert abs(r3["achieved"] - r2["achieved"] / 2) < 1e-4


def test_quantize_roofline_counts_the_algorithmic_bytes():
    """The quantize pass against HBM: 13 bytes per element of B*H*N*d (Q read
    and coded, K and V read twice and coded) per second, over the copy
    bandwidth."""
    sys.path.insert(0, ROOT)
    import bench
    from quantized_attention_qk_b200.inputs import WORKLOADS

    w = WORKLOADS["video"]
    r = bench._quant_roofline(w, 0.5, 6000.0, "measured", 123)
    nbytes = 13 * w.B * w.H * w.N * w.d
    assert r["algorithmic_bytes"] == nbytes and r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert abs(r["achieved"] - nbytes / 0.5e-3 / 1e9) < 0.1
    assert abs(r["frac"] - r["achieved"] / 6000.0) < 1e-4
    assert r["traffic"] == 123 and r["quant_ms"] == 0.5


def test_traffic_records_hold_only_for_the_source_they_were_taken_on():
    """A DRAM count is reported only while the kernel's source has the hash the
    record was taken on, and only for a workload it was taken on."""
    sys.path.insert(0, ROOT)
    import bench

    for rec, src in (("k_attn_traffic.txt", "sage_attn.cu"), ("k_qpass_traffic.txt", "sage_quant.cu")):
        assert bench._profile_traffic(rec, src, "no such workload") is None
        assert bench._profile_traffic(rec, "sage_api.cu", "flux") is None  # another file's hash
    assert bench._profile_traffic("no_such_record.txt", "sage_quant.cu", "flux") is None
