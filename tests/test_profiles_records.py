"""The committed DRAM-traffic records (profiles/traffic.json) and how bench.py uses them.

bench.py reports an ncu-measured traffic figure beside a roofline only while the record was taken on
the kernel's current sources (a hash of them is stored with the record); once a source changes, the
figure is reported as null until the record is re-captured. These checks keep the records well
formed, check that lookup rule, and warn (rather than fail, since a re-capture needs a GPU) about
records a source change has made stale.
"""
import json
import os
import re
import warnings

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
RECORDS = os.path.join(ROOT, "profiles", "traffic.json")


def _records():
    with open(RECORDS) as f:
        return json.load(f)


def test_kernel_sources_exist():
    csrc = os.path.join(ROOT, "gated_linear_attention_dn_b200", "csrc")
    for kernel, files in bench.KERNEL_SOURCES.items():
        for fn in files:
            assert os.path.exists(os.path.join(csrc, fn)), f"{kernel}: {fn} missing"


def test_records_well_formed():
    recs = _records()
    assert recs, "no traffic records"
    for entry, r in recs.items():
        kernel = entry.split(":")[0]
        assert kernel in bench.KERNEL_SOURCES, f"{entry}: unknown kernel {kernel}"
        for key in ("kernel", "workload", "dram_read", "dram_write", "bytes_per_launch", "source_hash"):
            assert key in r, f"{entry}: no {key}"
        assert r["dram_read"] > 0 and r["dram_write"] > 0, entry
        assert r["bytes_per_launch"] == r["dram_read"] + r["dram_write"], entry
        assert re.fullmatch(r"[0-9a-f]{16}", r["source_hash"]), entry


def test_lookup_follows_the_source_hash():
    for entry, r in _records().items():
        kernel = entry.split(":")[0]
        current = bench.kernel_source_hash(kernel) == r["source_hash"]
        got = bench.recorded_traffic(kernel, entry)
        if current:
            assert got == r["bytes_per_launch"], entry
        else:
            assert got is None, f"{entry}: a stale record was returned"
            warnings.warn(f"{entry}: traffic recorded on other sources of {kernel}; bench.py reports null "
                          "until it is re-captured")


def test_hash_changes_with_any_source():
    # the hash covers every listed file and its name: two kernels with different file lists differ
    hashes = {k: bench.kernel_source_hash(k) for k in bench.KERNEL_SOURCES}
    assert len(set(hashes.values())) == len(hashes)
