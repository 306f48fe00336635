"""bench.py host helpers on CPU: when a committed ncu traffic figure still describes the kernel."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

SRC = os.path.join(ROOT, "mxfp4_expert_gemm_b200", "csrc", "moe_mx.cu")


def test_code_sha_ignores_comments_and_layout_only():
    code = open(SRC, encoding="utf-8").read()
    base = bench.code_sha(code)
    assert bench.code_sha("// a new note\n" + code.replace("\n", "\n  ", 3)) == base
    assert bench.code_sha(code.replace("/*", "/* reworded", 1)) == base
    assert bench.code_sha(code.replace("kWaitLimitNs = 2000000000ull", "kWaitLimitNs = 1000000000ull", 1)) != base


def test_traffic_is_reported_only_for_the_kernel_it_was_taken_on():
    """bench.py returns a committed ncu DRAM figure while the kernel source (without comments)
    is the one it was captured on, and null otherwise."""
    t = json.load(open(os.path.join(ROOT, "profiles", "ncu_traffic.json")))
    assert t, "no committed ncu traffic"
    current = bench.file_sha(SRC)
    for key, ent in t.items():
        cfg, _, act = key.partition("/")
        got = bench.ncu_traffic("gate_up", cfg, act or "bf16")
        want = ent["gate_up"]["dram_bytes_per_launch"] if ent["gate_up"]["source_sha"] == current else None
        assert got == want, key
    assert bench.ncu_traffic("gate_up", "no_such_workload") is None
