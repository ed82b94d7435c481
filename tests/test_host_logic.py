"""Host-side logic that needs no GPU: the binding fails loudly without the
library (there is no CPU path to fall back to), and bench.py's traffic record is
used only for the kernel source and size it was captured on."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def test_missing_library_raises():
    """With the library path pointing nowhere every call raises LaplexError
    before touching a tensor."""
    code = (
        "import exact_laplace_b200.laplex as X\n"
        "X.LIB_PATH = '/nonexistent/liblaplex.so'\n"
        "X._lib = None\n"
        "try:\n"
        "    X.lib()\n"
        "except X.LaplexError as e:\n"
        "    assert e.status == X.ECUDA and 'missing' in str(e), e\n"
        "    print('raised')\n"
        "else:\n"
        "    raise SystemExit('no error')\n"
        "try:\n"
        "    X.workspace_size(X.OP_SYM, 10)\n"
        "except X.LaplexError:\n"
        "    print('raised')\n"
    )
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.split() == ["raised", "raised"]


def test_traffic_record_matches_source_and_size():
    import bench
    sha = bench.src_sha("sym_stream.cu", "scan_core.cuh", "common.cuh", "bulk.cuh")
    rec = None
    for line in open(os.path.join(ROOT, "profiles", "traffic.txt")):
        if line.startswith("key=k_tile_local_presorted_b1"):
            rec = dict(tok.split("=", 1) for tok in line.split())
    assert rec is not None
    n = int(rec["n"])
    got = bench.traffic_from_profile("k_tile_local_presorted_b1", rec["src_sha"], n)
    assert got == float(rec["bytes_per_launch"])
    # another size, another source or another kernel: no figure
    assert bench.traffic_from_profile("k_tile_local_presorted_b1", rec["src_sha"], n // 2) is None
    assert bench.traffic_from_profile("k_tile_local_presorted_b1", "0" * 16, n) is None
    assert bench.traffic_from_profile("k_other", rec["src_sha"], n) is None
    # the record is current for the headline kernel's sources as they stand
    assert rec["src_sha"] == sha
    # the traffic is within 2 % of the algorithmic 12 bytes per anchor
    assert abs(float(rec["bytes_per_launch"]) / (12 * n) - 1) < 0.02


def test_workload_config_names_the_workload():
    import bench
    cfg = bench.workload_config(1 << 30, 1)
    assert cfg["n"] == 1 << 30 and "workload" in cfg and cfg["B"] == 1
