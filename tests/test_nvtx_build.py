"""The optional NVTX build (-DSD_NVTX) compiles: the entry-point files with the flag, on the CPU.

The default build defines the range macro away, so its library is what the other tests load;
this only guards the flagged path against rotting.  nvcc cross-compiles for sm_100a without a
GPU."""
import os
import shutil
import subprocess

import pytest

from speculative_decoding_attention_verify_b200 import build as B

NVCC = B.NVCC if os.path.exists(B.NVCC) else shutil.which("nvcc")


@pytest.mark.skipif(not NVCC, reason="nvcc not available")
@pytest.mark.parametrize("src", ["sd_api.cu", "sd_noalloc.cu", "draft_layer.cu"])
def test_entry_points_compile_with_nvtx_ranges(src, tmp_path):
    flags = [f for f in B.FLAGS if f != "-DSD_NVTX"] + ["-DSD_NVTX"]
    obj = tmp_path / (src[:-3] + ".o")
    r = subprocess.run([NVCC] + B.ARCH + flags + ["-c", os.path.join(B.CSRC, src), "-o", str(obj)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    assert obj.stat().st_size > 0
