"""Register and spill report of the tensor-core attention kernels (ptxas, on
the CPU): all three instantiations (16-bit scores, 8-bit scores, Q's RoPE in
the kernel) must compile without spills within the 168 registers per thread
that 384 threads per SM allow."""
import os
import re
import shutil
import subprocess

import pytest

from chunk_causal_attention_block_b200 import build as wfbuild


def test_attention_kernels_compile_without_spills(tmp_path):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("no nvcc")
    src = os.path.join(wfbuild.CSRC, "attn_sm100.cu")
    r = subprocess.run([nvcc] + wfbuild.NVCC_FLAGS + ["-Xptxas", "-v", "-c", src, "-o", str(tmp_path / "a.o")],
                       capture_output=True, text=True, check=True)
    report = r.stdout + r.stderr
    blocks = re.findall(r"Compiling entry function '([^']*attn_fwd_sm100[^']*)'.*?\n(.*?)\nptxas info\s+: Used (\d+) registers",
                        report, flags=re.S)
    assert len(blocks) == 3, report
    for name, props, regs in blocks:
        assert "0 bytes spill stores, 0 bytes spill loads" in props, (name, props)
        assert int(regs) <= 168, (name, regs)
