"""Host-side logic of bench.py that needs no GPU: the recorded ncu traffic
is attached only to the exact capture it came from."""
import argparse
import hashlib
import os

import bench


def _args(**kw):
    a = dict(workload="qwen3_32b_128k", sel_fmt="bf16", batch=None)
    a.update(kw)
    return argparse.Namespace(**a)


def _source_hash(rec):
    h = hashlib.sha256()
    for name in rec["files"]:
        with open(os.path.join(bench.ROOT, "block_sparse_long_spot_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def test_traffic_only_for_the_captured_workload_format_and_batch():
    rec = bench.NCU_TRAFFIC["qwen3_32b_128k"]
    got = bench.measured_traffic(_args())
    # the recorded bytes while the kernel source matches the capture, else none
    assert got == (rec["bytes"] if _source_hash(rec) == rec["sha256"] else None)
    assert bench.measured_traffic(_args(sel_fmt="int4")) is None
    assert bench.measured_traffic(_args(batch=2)) is None
    assert bench.measured_traffic(_args(workload="qwen3_4b_32k")) is None

