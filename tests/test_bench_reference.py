"""The benchmark's reference arm (the oracle, timed on the host) and its
configuration text: host-only, no GPU."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_line_has_the_contract_keys():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "tiny", "--steps", "2", "--warmup", "1"],
                         capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference"
    assert line["steps"] == 2 and line["warmup"] == 1
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["cpu_baseline"]["value"] == line["value"] == line["e2e"]["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0
    # every step is a real timed sample: the claimed time fits in the run
    assert line["ms_per_step"] * (line["steps"] + line["warmup"]) < 300e3


def test_oracle_sample_is_the_steps_work_for_its_tokens():
    """A sample of the whole tiny batch computes what the full oracle step
    computes; samples run single-threaded and on a thread pool."""
    sys.path.insert(0, ROOT)
    import bench
    from mxfp4_moe_block_b200 import synth
    sh = synth.SHAPES["tiny"]
    full = bench.OracleSample(sh, sh.T)
    assert full.n_tok == sh.T and full.seqs == (0, sh.S)
    assert full.run() > 0
    pooled = bench.OracleSample(sh, sh.T, workers=4)
    assert pooled.run() > 0
    assert f"{sh.T} of the step's {sh.T} tokens" in full.text()
    big = synth.SHAPES["multilayer"]
    assert bench.sample_tokens(big, 1) == 1
    assert bench.sample_tokens(big, 64) == 8
    assert bench.sample_tokens(sh, 1) == sh.T


def test_l2_statement_follows_the_weight_bytes():
    sys.path.insert(0, ROOT)
    import bench
    from mxfp4_moe_block_b200 import synth
    assert bench.l2_statement(synth.SHAPES["batch1"]).startswith("inputs larger than L2")
    assert bench.l2_statement(synth.SHAPES["tiny"]).startswith("inputs smaller than L2")


def test_cpulist_parser():
    """bench.py places the e2e host buffers on the GPU's NUMA node from the
    device's sysfs cpulist."""
    sys.path.insert(0, ROOT)
    import bench
    assert bench.parse_cpulist("0-3,8,10-11\n") == {0, 1, 2, 3, 8, 10, 11}
    assert bench.parse_cpulist("5") == {5}
    assert bench.parse_cpulist("") == set()
