"""bench.py's argument checks, on the CPU: the main line times dot-product
workloads only (the learned-coordinate and decode workloads are timed under
"workloads"), and --extra names only known workloads.  Both are refused
before any device is touched."""
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench(*args):
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args],
                          capture_output=True, text=True, timeout=120)


def test_main_workload_is_a_dot_product_one():
    for name in ("dist_16k", "decode_16k"):
        r = _bench("--workload", name)
        assert r.returncode == 2 and "invalid choice" in r.stderr, r.stderr


def test_unknown_extra_workload_is_refused():
    r = _bench("--extra", "csr_1m,no_such_workload")
    assert r.returncode == 2 and "no_such_workload" in r.stderr, r.stderr
