"""bench.py on the CPU: the algorithmic byte counts behind the roofline fields, and the
reference arm's JSON line (the oracle timed on the host cores)."""
import json
import os
import subprocess
import sys

import bench
from gated_delta_rule_122_b200.inputs import workload

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_prefill_algorithmic_bytes():
    # per head-token: q, k, v, alpha (bf16, 4 x 256 B) + beta (2 B) + o (fp32, 512 B) = 1538 B,
    # plus one fp32 128 x 128 final state per (sequence, head); an initial state adds another
    w = workload("prefill")
    heads_tokens = 2 * 8192 * 64
    states = 2 * 64 * 128 * 128 * 4
    assert bench.prefill_bytes(w, with_s0=False) == heads_tokens * 1538 + states
    assert bench.prefill_bytes(w, with_s0=True) == heads_tokens * 1538 + 2 * states


def test_decode_algorithmic_bytes():
    # per (sequence, head): the state read and written (2 x 64 KiB), q, k, v, alpha (bf16),
    # beta (2 B), o (fp32)
    w = workload("decode")
    per_head = 2 * 65536 + 4 * 256 + 2 + 512
    assert bench.decode_bytes(w) == 256 * 64 * per_head


def test_reference_arm_prints_one_json_line():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1")
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "0"], capture_output=True, text=True, cwd=ROOT,
                         env=env, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["unit"] == "Mtokens/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["higher_is_better"] is True
