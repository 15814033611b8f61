"""bench.py's traffic record: the DRAM bytes of a kernel are reported only while
the kernel's sources hash to the value recorded with the ncu capture."""
import hashlib
import json
import os

import bench


def _record(root, sources, sha, nbytes=123):
    os.makedirs(os.path.join(root, "profiles"), exist_ok=True)
    with open(os.path.join(root, "profiles", "traffic.json"), "w") as f:
        json.dump({"attn_prefill_kernel": {"dram_bytes_per_launch": nbytes, "sources": sources,
                                           "sources_sha256": sha}}, f)


def test_traffic_is_null_once_a_source_changes(tmp_path, monkeypatch):
    root = str(tmp_path)
    src = os.path.join(root, "k.cuh")
    with open(src, "w") as f:
        f.write("kernel v1")
    sha = hashlib.sha256(b"kernel v1").hexdigest()
    _record(root, ["k.cuh"], sha)
    monkeypatch.setattr(bench, "ROOT", root)
    assert bench.recorded_traffic("attn_prefill_kernel") == 123
    assert bench.recorded_traffic("attn_merge_kernel") is None        # no record for it
    with open(src, "w") as f:
        f.write("kernel v2")
    assert bench.recorded_traffic("attn_prefill_kernel") is None

