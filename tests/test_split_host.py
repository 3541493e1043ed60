"""The attention work split and the merge's record enumeration, checked on
the CPU: tests/native/split_check.cu includes the kernels' own headers
(cta_of, merge_record), is compiled as host code by nvcc and compared there
against brute force (every kept tile in exactly one CTA, a record reported
written exactly when its warp pair owns a tile, no slot shared by two
units, every slot inside the partial buffers)."""
import os
import subprocess

from block_sparse_kv_spattn_b200 import build as B

HERE = os.path.dirname(os.path.abspath(__file__))


def test_split_and_merge_records_against_brute_force(tmp_path):
    exe = str(tmp_path / "split_check")
    subprocess.run([B._nvcc(), *B.ARCH, "-O2", "-std=c++17", "-I", B.CSRC, "-I", B.INCLUDE,
                    os.path.join(HERE, "native", "split_check.cu"), "-o", exe], check=True, timeout=300)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout[-2000:]
    assert r.stdout.startswith("ok ")
    assert int(r.stdout.split()[1]) > 1000
