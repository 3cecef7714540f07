"""Host logic of bench.py: the reference arm (the CPU oracle timed on the host)
keeps the benchmark's one-line JSON contract, and under a multi-rank launch
only rank 0 does the work and prints; the roofline's DRAM traffic is taken
from a committed ncu summary only while the kernel source is unchanged."""
import json
import os
import subprocess
import sys

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(env_extra, steps=2):
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    env.update(env_extra)
    return subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", str(steps),
                           "--warmup", "0"], cwd=ROOT, env=env, capture_output=True, text=True,
                          timeout=600)


def test_reference_arm_prints_one_contract_line():
    r = _run({})
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1, lines
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["metric"] == bench.METRIC and d["unit"] == "tokens/s"
    assert d["value"] > 0 and d["higher_is_better"] is True
    assert d["n_gpus"] == 1 and d["steps"] == 2 and d["warmup"] == 0
    assert d["ms_per_step"] > 0 and d["dtype"] == "f64" and d["data"] == "synthetic"
    assert d["config"]["workload"] == bench.WORKLOAD
    assert d["vs_baseline"] is None
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    # tokens/s follows from the timed block applications: 10 per forward of 128 tokens
    assert abs(d["value"] - 128 / (d["ms_per_step"] / 1e3 * 10)) <= 0.01 * d["value"]


def test_reference_arm_other_ranks_exit_without_work():
    r = _run({"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""


def test_roofline_traffic_only_for_the_profiled_source(tmp_path, monkeypatch):
    """The per-launch DRAM bytes from a committed ncu summary are reported only
    while the kernel source hashes to the value the summary recorded."""
    (tmp_path / "profiles").mkdir()
    (tmp_path / "k.cu").write_text("kernel v1\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h = bench.source_hash("k.cu")
    (tmp_path / "profiles" / "k.md").write_text(
        f"# summary\n\nsource_sha256_16: {h}\ndram_bytes_per_launch: 17884160\n")
    assert bench.ncu_traffic("k.md", ["k.cu"]) == 17884160.0
    (tmp_path / "k.cu").write_text("kernel v2\n")          # the kernel changed since the capture
    assert bench.ncu_traffic("k.md", ["k.cu"]) is None
    assert bench.ncu_traffic("missing.md", ["k.cu"]) is None


def test_decode_roofline_accounting():
    """The decode roofline's byte counts: one 407M-shaped block is its packed
    codes plus fp16 scales for QKV, O, gate, up and down (INT4: 67.1 M weights
    at half a byte plus one 2-byte scale per 128; INT3: padded 10-codes-per-
    word rows), and t = HBM bytes / HBM bandwidth + L2 bytes / L2 bandwidth."""
    import weight_shared_looped_b200 as tl
    d, f = 2048, 8192
    n_w = 3 * d * d + d * d + 3 * f * d
    assert bench.block_bytes(tl, 4) == n_w // 2 + n_w // 128 * 2 == 34603008
    words3 = 4 * ((d // 10 + 1 + 3) // 4)            # K = 2048: 205 words, padded to 208
    words3_f = 4 * ((f // 10 + 1 + 3) // 4)          # K = 8192: 820 words (already whole vectors)
    rows_d, rows_f = 3 * d + d + 2 * f, d            # rows with K = d and with K = f
    assert bench.block_bytes(tl, 3) == (rows_d * words3 + rows_f * words3_f) * 4 + n_w // 128 * 2
    r = bench.decode_roofline(t_step=100e-6, hbm_bytes=6.4e8, l2_bytes=1.6e9, hbm_gbs=6400.0,
                              l2_gbs=16000.0)
    assert r["roofline_us"] == 200.0                 # 100 us of HBM + 100 us of L2
    assert r["frac_roofline"] == 2.0 and r["frac_hbm"] == 1.0
    assert r["hbm_bytes_per_step"] == 640000000 and r["l2_bytes_per_step"] == 1600000000
