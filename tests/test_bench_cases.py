"""The bench's single-kernel capture cases (`bench.py --case`), on the CPU:
every case names a kernel the built library contains, so the ncu commands
under profiles/ (`-k regex:<kernel>`) keep matching; and the algorithmic-byte
count of the expert FFN adds up the tensors it names."""
import os
import shutil
import subprocess

import pytest

import bench

LIB = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "precision_moe_numerics_quantize_b200", "libnvfp4moe.so")


@pytest.mark.skipif(not os.path.exists(LIB) or shutil.which("nm") is None,
                    reason="library not built or nm missing")
def test_case_kernels_exist_in_the_library():
    syms = subprocess.run(["nm", "-C", LIB], capture_output=True, text=True, check=True).stdout
    for case, kernel in bench.CASES.items():
        assert f"nvfp4moe::{kernel}" in syms or f"nvfp4moe{len(kernel)}{kernel}" in syms, (case, kernel)


def test_expert_fwd_bytes_adds_the_named_tensors():
    d, f, E, R = 4096, 2560, 384, 147968
    b = bench.expert_fwd_bytes(d, f, E, R)
    assert b["weights"] == 0.5625 * 3 * d * f * E  # W1 (2f x d) + W2 (d x f), codes + E4M3 scales
    assert b["xq"] == 0.5625 * R * d
    assert b["h_write"] == 2.0 * R * f
    assert b["hq_write_read"] == 2 * 0.5625 * R * f
    assert b["y_write"] == 2.0 * R * d
    # the full-size layer (147968 padded routed rows): 9.53 GB
    assert abs(sum(b.values()) / 1e9 - 9.53) < 0.01
