"""Host-side arithmetic of bench.py, checked on the CPU: the algorithmic work each kernel is
credited with, the per-kernel roofline figures derived from a trace, the clock summary and the
DRAM traffic read from the committed ncu summaries."""
import re
from pathlib import Path
from types import SimpleNamespace

import numpy as np
import pytest

import bench

ROOT = Path(__file__).resolve().parents[1]


def _problem(B, T, Hq, Hkv, G):
    """Only the shapes and the group counts enter the work formulas."""
    q = np.broadcast_to(np.float32(0), (B, Hq, T, 64))
    k = np.broadcast_to(np.float32(0), (B, Hkv, T, 64))
    return SimpleNamespace(q=q, k=k, G=np.asarray(G, np.int32))


@pytest.mark.parametrize("B,T,Hq,Hkv", [(1, 4096, 14, 2), (2, 300, 8, 1), (1, 128, 4, 4)])
def test_kernel_work_splits_the_prefill_flops(B, T, Hq, Hkv):
    """Deltas plus readout equal eq. (4)-(5)'s work over the packed features, less the first
    chunk's readout, which has no prefix state to read (its rows are all intra-chunk)."""
    p = _problem(B, T, Hq, Hkv, [3] * Hq)
    w = bench.kernel_work(p, 128)
    first = 2.0 * B * Hq * min(T, 128) * bench.F * bench.W
    assert w["delta_tc"][0] + w["readout_tc"][0] + first == pytest.approx(
        bench.prefill_flops(B, T, Hq, Hkv), rel=1e-12)
    assert {k: v[1] for k, v in w.items()} == {"delta_tc": "flop", "readout_tc": "flop",
                                               "intra_tc": "flop", "scan": "byte"}


def test_kernel_work_intra_pairs_by_brute_force():
    """The intra-chunk kernel is credited per causal pair inside a chunk: count the pairs."""
    B, T, Hq, Hkv, chunk = 1, 300, 4, 2, 128
    G = [1, 2, 4, 8]
    pairs = sum(1 for i in range(T) for j in range(i + 1) if i // chunk == j // chunk)
    per_pair = sum(2 * 64 * (g + 1) + 2 * 65 for g in G)
    w = bench.kernel_work(_problem(B, T, Hq, Hkv, G), chunk)
    assert w["intra_tc"][0] == B * pairs * per_pair


def test_kernel_work_scan_bytes():
    """The scan reads every fp32 chunk delta once and writes the bf16 images of every prefix
    but the first (65 live rows of each 64-row slice) and the fp32 final state."""
    B, T, Hkv = 1, 4096, 2
    NC = T // 128
    w = bench.kernel_work(_problem(B, T, 14, Hkv, [3] * 14), 128)
    fp32_in = NC * 65 * 2176 * 4
    images = (NC - 1) * 34 * 65 * 64 * 2
    final = 2176 * 65 * 4
    assert w["scan"][0] == B * Hkv * (fp32_in + images + final)


def test_kernel_rooflines_from_a_trace():
    pk = {"bf16_tflops": 1590.0, "hbm_gbs": 6650.0, "sm_max_mhz": 1965.0}
    work = {"readout_tc": (2.0e10, "flop"), "scan": (3.0e7, "byte")}
    prof = {"readout_tc": (4, 0.4), "scan": (4, 0.1), "prep": (2, 0.1)}
    out = bench.kernel_rooflines(prof, work, pk, "fallback", 4)
    r = out["readout_tc"]
    assert r["avg_launch_ms"] == pytest.approx(0.1)
    assert r["achieved"] == pytest.approx(2.0e10 / 1e-4 / 1e12)        # 200 TFLOP/s
    assert r["frac"] == pytest.approx(200.0 / 1590.0)
    s = out["scan"]
    assert s["achieved"] == pytest.approx(3.0e7 / 2.5e-5 / 1e9)         # 1200 GB/s
    assert s["bound"] == "hbm" and s["unit"] == "GB/s"
    assert out["prep"]["bound"] == "alu"
    assert out["prep"]["peak"] == pytest.approx(148 * 128 * 2 * 1965.0e6 / 1e12)
    assert sum(v["share"] for v in out.values()) == pytest.approx(1.0, abs=1e-3)


def test_clock_summary():
    c = bench.ClockSampler(0)
    c.lines = [
        "0, 1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active",
        "0, 1800, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1900, 1965, 950.0, 0x0, Not Active, Not Active, Not Active, Not Active",
        "garbage",
        "0, [N/A], 1965, 1.0, 0x0, Not Active, Not Active, Not Active, Not Active",
    ]
    s = c.summary()
    assert s == {"sm_mhz": 1900.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"],
                 "samples": 3}
    c.lines = ["0, 1965, 1965, 1.0, 0x8, Active, Not Active, Not Active, Not Active"]
    assert c.summary()["reasons"] == ["hw_slowdown"]
    c.lines = []
    assert c.summary()["samples"] == 0 and c.summary()["sm_mhz"] is None


def _traced_kernel_names():
    """Names under which the library's tracer records its launches."""
    names = set()
    for f in (ROOT / "positive_quadratic_b200" / "csrc").glob("*.cu*"):
        names |= set(re.findall(r'LaunchScope\s+\w+\("([a-z_0-9]+)"', f.read_text()))
    return names


def test_profiled_traffic_names_traced_kernels():
    """The committed ncu summaries give DRAM bytes per launch for kernels the tracer knows by
    the same names, so the bench line can attach them to its roofline."""
    names = _traced_kernel_names()
    pre = bench.profiled_traffic("config1")
    assert set(pre) == {"delta_tc", "intra_tc", "scan", "readout_tc"}
    dec = bench.profiled_traffic("config1", "decode_batch64_sections.md")
    assert set(dec) == {"decode"}
    for k, v in {**pre, **dec}.items():
        assert k in names, k
        assert isinstance(v, int) and v > 0
    assert bench.profiled_traffic("config3_16k") == {}


def test_scan_traffic_is_close_to_its_algorithmic_bytes():
    """The scan's measured DRAM bytes per launch stay near what it must move (the fp32 deltas
    may still be partly in L2 when it runs, so it can read fewer)."""
    p = _problem(1, 4096, 14, 2, [3] * 14)
    alg = bench.kernel_work(p, 128)["scan"][0]
    got = bench.profiled_traffic("config1")["scan"]
    assert 0.5 * alg <= got <= 1.25 * alg


def _run_bench(env_extra, *argv):
    import json
    import os
    import subprocess
    import sys
    env = dict(os.environ, **env_extra)
    r = subprocess.run([sys.executable, str(ROOT / "bench.py"), *argv], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    return [json.loads(ln) for ln in lines]


def test_reference_arm_prints_one_contract_line():
    """bench.py --impl reference times the fp64 oracle on the host (no GPU needed) and prints
    one JSON line with the keys of the benchmark contract."""
    (out,) = _run_bench({"RANK": "0", "WORLD_SIZE": "1"}, "--impl", "reference", "--steps",
                        "2", "--warmup", "3")
    assert out["impl"] == "reference" and out["n_gpus"] == 1
    assert out["steps"] == 2 and out["warmup"] == 3
    assert out["value"] > 0 and out["unit"] == "tokens/s" and out["higher_is_better"] is True
    assert out["ms_per_step"] == pytest.approx(512 / out["value"] * 1e3, rel=1e-6)
    assert out["cpu_baseline"]["kind"] == "oracle" and out["cpu_baseline"]["cores"] >= 1
    assert out["cpu_baseline"]["value"] == out["value"]
    assert out["e2e"] == {"value": out["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                          "d2h_bytes_per_step": 0}
    assert "T=4096" in out["config"]["workload"]


def test_reference_arm_other_ranks_do_no_work():
    assert _run_bench({"RANK": "1", "WORLD_SIZE": "2"}, "--impl", "reference", "--gpus", "2",
                      "--steps", "2", "--warmup", "3") == []
