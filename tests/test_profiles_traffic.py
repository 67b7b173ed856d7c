"""The DRAM traffic the benchmark reports comes from committed ncu summaries
(profiles/traffic.json).  Every entry must still describe the kernel source
it was captured on (its hash), name an existing summary, and give byte counts
that add up; otherwise the benchmark would report stale counters."""
import hashlib
import json
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TABLE = os.path.join(ROOT, "profiles", "traffic.json")


def _entries():
    with open(TABLE) as f:
        table = json.load(f)
    for kernel, per_workload in table.items():
        for workload, ent in per_workload.items():
            yield kernel, workload, ent


def test_every_entry_matches_its_kernel_source():
    stale = []
    for kernel, workload, ent in _entries():
        h = hashlib.sha256()
        for rel in ent["sources"]:
            with open(os.path.join(ROOT, rel), "rb") as f:
                h.update(f.read())
        if h.hexdigest()[:16] != ent["source_hash"]:
            stale.append(f"{kernel}/{workload}")
    assert not stale, f"captures older than their kernel sources: {stale}"


def test_every_entry_names_its_summary_and_adds_up():
    for kernel, workload, ent in _entries():
        assert os.path.exists(os.path.join(ROOT, ent["capture"])), ent["capture"]
        total = ent.get("bytes_per_launch") or ent.get("bytes_per_call")
        assert total == ent["dram_read_bytes"] + ent["dram_write_bytes"], f"{kernel}/{workload}"
