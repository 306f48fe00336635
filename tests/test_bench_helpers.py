"""bench.py host helpers on CPU: when a committed ncu traffic figure still describes the kernel."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

SRC = os.path.join(ROOT, "mxfp4_expert_gemm_b200", "csrc", "moe_mx.cu")
TRAFFIC = os.path.join(ROOT, "profiles", "ncu_traffic.json")


def test_code_sha_ignores_comments_and_layout_only():
    code = open(SRC, encoding="utf-8").read()
    base = bench.code_sha(code)
    assert bench.code_sha("// a new note\n" + code.replace("\n", "\n  ", 3)) == base
    assert bench.code_sha(code.replace("/*", "/* reworded", 1)) == base
    assert bench.code_sha(code.replace("kWaitLimitNs = 2000000000ull", "kWaitLimitNs = 1000000000ull", 1)) != base


def test_capture_hash_covers_the_kernel_headers():
    """A change to a header the kernel includes makes its captures stale."""
    files = bench.KERNEL_SOURCES["gate_up"]
    assert {"moe_mx.cu", "moe_internal.cuh", "sm100_ptx.cuh"} <= set(files)
    text = "".join(open(os.path.join(bench.CSRC, f), encoding="utf-8").read() + "\n" for f in files)
    assert bench.sources_sha(files) == bench.code_sha(text)
    ptx = open(os.path.join(bench.CSRC, "sm100_ptx.cuh"), encoding="utf-8").read()
    changed = text.replace(ptx, ptx.replace("smem_u32", "smem_u32_", 1))
    assert bench.code_sha(changed) != bench.sources_sha(files)


def test_committed_traffic_entries_match_the_current_sources():
    """profiles/ncu_traffic.json holds only captures of the code as it is now: an entry whose
    kernel (or one of its headers) changed since its capture must be re-captured or removed."""
    t = json.load(open(TRAFFIC))
    for key, kernels in t.items():
        cfg, _, act = key.partition("/")
        for kernel, ent in kernels.items():
            assert ent["sources"] == bench.KERNEL_SOURCES[kernel], (key, kernel)
            assert ent["source_sha"] == bench.sources_sha(ent["sources"]), f"stale capture: {key} {kernel}"
            assert bench.ncu_traffic(kernel, cfg, act or "bf16") == ent["dram_bytes_per_launch"]
    assert bench.ncu_traffic("gate_up", "no_such_workload") is None
