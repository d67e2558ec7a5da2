"""Host-side pieces of bench.py that need no GPU: the CPU-oracle sample behind `cpu_baseline`
and the reference arm, and the algorithmic units each sample is credited with."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_decode_sample_counts_the_pages_of_its_sequences():
    """The decode sample runs one decode step of the `seqs` shortest sequences; its units are
    the cache bytes of those sequences' pages (partial pages in full), per KV head: d/2 + d/16
    bytes of K codes and scales and d + d/32 of V per token."""
    dt, units, desc = bench.oracle_sample("paged_decode_s64", seqs=2)
    lay = bench._inputs("paged_decode_s64")
    d, hkv = lay.cfg["d"], lay.cfg["Hkv"]
    lens = sorted(int(n) for n in lay.lens.tolist())[:2]
    per_tok = d // 2 + d // 16 + d + d // 32
    assert units == sum((n + 63) // 64 * 64 for n in lens) * hkv * per_tok
    assert desc.startswith("2 sequence(s)") and dt > 0


def test_prefill_sample_counts_visible_pairs():
    """The prefill sample's units are 4·d FLOPs per visible (query, key) pair of its rows:
    under the causal mask, row i sees i + 1 keys."""
    dt, flops, desc = bench.oracle_sample("prefill_h16_n4096", rows=32, heads=2)
    d = bench.workloads.WORKLOADS["prefill_h16_n4096"]["d"]
    n = bench.workloads.WORKLOADS["prefill_h16_n4096"]["N"]
    import numpy as np
    rows = np.sort(np.random.default_rng(0).choice(n, size=32, replace=False))
    assert flops == 2 * 4.0 * d * float((rows + 1).sum())
    assert desc == "2 query head(s) x 32 seeded query rows (of 4096)" and dt > 0


def test_reference_arm_decode_line():
    """`--impl reference` on the decode workload: one JSON line in GB/s with the oracle as its
    baseline and no host-device copies."""
    cmd = [sys.executable, "bench.py", "--impl", "reference", "--workload", "paged_decode_s64",
           "--steps", "1", "--warmup", "0"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["unit"] == "GB/s" and line["value"] > 0
    assert line["config"] == bench.config_of("paged_decode_s64")
    assert line["cpu_baseline"]["value"] == line["value"] and line["e2e"]["d2h_bytes_per_step"] == 0
