"""The bench's reference (oracle) arm must not map the product library, and
both arms must print the same config (CPU)."""
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROBE = r"""
import sys
sys.argv = ["bench.py"]
sys.path.insert(0, {root!r})
import bench
case, N, step_bytes, _ = bench.decode_workload()
step = bench.oracle_decode_sample(case, 4096, [0, 1])
maps = open("/proc/self/maps").read()
print("MAPPED" if "libtbq4.so" in maps else "CLEAN")
print("PKG" if "long_context_attention_tbq4_b200" in sys.modules else "NOPKG")
"""


def test_reference_arm_does_not_map_the_product_library():
    out = subprocess.run([sys.executable, "-c", PROBE.format(root=ROOT)], cwd=ROOT,
                         capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = out.stdout.split()
    assert "CLEAN" in lines and "NOPKG" in lines, out.stdout


def test_both_arms_print_the_same_config():
    sys.path.insert(0, ROOT)
    import bench
    W = bench.load_workloads()
    case = W.decode_case("cfg", 0, 1, 24, 4, [64])
    assert bench.decode_config(case, 262144, 1) == bench.decode_config(case, 262144, 1)
    src = open(os.path.join(ROOT, "bench.py")).read()
    # the product line and the reference line both take their config from
    # decode_config and nowhere else
    assert src.count('"config": decode_config(') == 2
