"""Host-side helpers of bench.py that shape reported numbers: nearest-rank
percentiles of per-call times, the DRAM-traffic lookup keyed by kernel source,
and the run conditions.  CPU only."""
import hashlib
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_percentiles_nearest_rank():
    xs = [float(i) for i in range(1, 101)]  # 1 .. 100
    p = bench.percentiles(list(reversed(xs)))
    assert (p["p50"], p["p95"], p["p99"], p["calls"]) == (50.0, 95.0, 99.0, 100)
    ten = [5.0, 1.0, 9.0, 3.0, 7.0, 2.0, 8.0, 4.0, 6.0, 10.0]
    p = bench.percentiles(ten)
    # nearest rank: ceil(q * n) -> p50 is the 5th smallest, p95 and p99 the 10th
    assert (p["p50"], p["p95"], p["p99"]) == (5.0, 10.0, 10.0)
    assert bench.percentiles([]) is None
    assert bench.percentiles([2.5])["p99"] == 2.5


def test_traffic_lookup_follows_the_kernel_source():
    """A recorded traffic figure is reported only while the kernel's source
    still hashes to the recorded prefix."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    rows = [l.split() for l in open(path) if l.strip() and not l.startswith("#")]
    src = {"gdn_prefill_pool": "prefill_chain.cu", "gdn_decode": "decode.cu"}
    for key, fname in src.items():
        rec = [r for r in rows if r[0] == key]
        assert len(rec) == 1, key
        sha = hashlib.sha256(open(os.path.join(ROOT, "gated_deltanet_04_b200", "csrc", fname),
                                  "rb").read()).hexdigest()[:16]
        got = bench.traffic_for(key, fname)
        if rec[0][1] == sha:
            assert got == float(rec[0][2])
        else:
            assert got is None
    assert bench.traffic_for("no_such_kernel", "decode.cu") is None


def test_run_conditions_keys():
    c = bench.run_conditions()
    assert {"cpu_model", "nproc", "torch"} <= set(c)
    assert c["nproc"] >= 1
