"""Build options compile: the tracing build (-DDSA_NVTX=1, NVTX ranges per layer and
index window in the layer loop) is valid host code for sm_100a."""
import shutil
import subprocess

import pytest

from sparse_attention_17_b200 import build as B


@pytest.mark.skipif(shutil.which("nvcc") is None and not B.Path("/usr/local/cuda/bin/nvcc").exists(),
                    reason="needs nvcc")
def test_nvtx_build_of_the_c_abi_compiles(tmp_path):
    obj = tmp_path / "capi_nvtx.o"
    subprocess.run([B.nvcc(), *B.ARCH, "-std=c++17", "-O1", "-DDSA_NVTX=1", f"-I{B.INCLUDE}",
                    "-c", str(B.CSRC / "capi.cu"), "-o", str(obj)], check=True)
    assert obj.stat().st_size > 0
