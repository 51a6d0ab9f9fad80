"""Host-side pieces of bench.py that need no GPU."""

import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def test_traffic_figures_match_the_default_run():
    """The DRAM traffic quoted in the roofline was captured on the bench's default workload and
    schedule: every key of that configuration is a bench argument, the defaults equal it (so the
    default run quotes the figures), and another workload does not."""
    import bench
    args = bench.parse_args([])
    for k, v in bench.NCU_TRAFFIC_CONFIG.items():
        assert hasattr(args, k), k
        assert getattr(args, k) == v, (k, getattr(args, k), v)
    other = bench.parse_args(["--workload", "skew"])
    assert not all(getattr(other, k) == v for k, v in bench.NCU_TRAFFIC_CONFIG.items())


def test_traffic_figures_are_keyed_by_source_hashes():
    """Every quoted figure names the hash of the sources it was taken on (16 hex digits of a
    sha256 over the kernel's files), the form bench._src_hash computes, so a changed kernel
    source makes the bench report its traffic as null."""
    import bench
    for kernel, rec in bench.NCU_TRAFFIC.items():
        assert rec["bytes"] > 0
        assert len(rec["src"]) == 16 and int(rec["src"], 16) >= 0
        assert len(bench._src_hash(kernel)) == 16
