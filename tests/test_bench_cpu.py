"""bench.py pieces that run without a GPU: the reference arm (the fp64 oracle
timed on host cores) prints one well-formed JSON line, and the algorithmic
byte / flop counts used for the roofline match the workload arithmetic."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def test_reference_arm_json_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "0"],
                       cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] == 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["config"]["workload"] == "prefill_h96_T8192_d128_bf16"


def test_algorithmic_counts():
    import bench
    from linear_attention_recurrence_11_b200.inputs import WORKLOADS
    w = WORKLOADS["prefill_h96_T8192_d128_bf16"]
    b, f = bench.prefill_algorithmic(w, 2)
    th = 8192 * 96
    # q, k, g, v, o at 128 x 2 bytes + beta, per token-head; S_T once per head
    assert b == th * (5 * 256 + 2) + 96 * 128 * 128 * 4
    # 6 d^2 + C (3 dk + 2 dv) + C^2 / 3 per token-head
    assert abs(f - th * (6 * 128 * 128 + 64 * 640 + 64 * 64 / 3)) < 1.0
    bd, _ = bench.decode_algorithmic(256, 96, 128, 128, 2)
    assert bd == 256 * 96 * (2 * 128 * 128 * 4 + 4 * 128 * 2 + 2 + 128 * 2)
    assert bench.weak_scaling_value(100, 10, 1000.0, 4) == 4000.0


def test_multi_decode_algorithmic_bytes():
    import bench
    state = 128 * 128 * 4
    per_tok = (3 * 128 + 128 + 1) * 2
    # nothing accepted: the verification alone (states read once, all inputs, all outputs)
    assert bench.multi_decode_algorithmic(2, 3, 4, 128, 128, [0, 0]) == \
        2 * 3 * state + 2 * 4 * 3 * per_tok + 2 * 4 * 3 * 128 * 2
    # one request commits 3 tokens: its states read and written, 3 more tokens' inputs
    assert bench.multi_decode_algorithmic(2, 3, 4, 128, 128, [3, 0]) - \
        bench.multi_decode_algorithmic(2, 3, 4, 128, 128, [0, 0]) == 2 * 3 * state + 3 * 3 * per_tok
