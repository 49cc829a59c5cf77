"""The C ABI from plain C: include/wf.h compiles as C99 and a C program that
links libwf.so builds a round plan byte-identical to the one the Python
binding gets.  Host-only calls: no device is needed."""
import os
import shutil
import subprocess

import numpy as np
import pytest

from chunk_causal_attention_block_b200 import wf

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _cc():
    cc = shutil.which("gcc") or shutil.which("cc")
    if not cc:
        pytest.skip("no C compiler")
    return cc


def test_headers_compile_as_c99(tmp_path):
    src = tmp_path / "h.c"
    src.write_text('#include "wf.h"\n#include "wf_synth.h"\nint main(void) { return WF_OK; }\n')
    subprocess.run([_cc(), "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                    "-c", str(src), "-o", str(tmp_path / "h.o")], check=True)


def test_c_program_plans_the_same_bytes_as_the_binding(tmp_path):
    libdir = os.path.dirname(wf.lib()._name)
    exe = tmp_path / "plan_from_c"
    subprocess.run([_cc(), "-std=c11", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c", "plan_from_c.c"), "-o", str(exe), "-L", libdir, "-lwf",
                    f"-Wl,-rpath,{libdir}"], check=True)
    out = tmp_path / "plan.bin"
    subprocess.run([str(exe), str(out)], check=True)
    got = np.fromfile(out, dtype=np.uint8)
    d = wf.make_desc(12, 128, 30, 52, 3, 7, 4, 16, [250, 500, 750, 1000], dtype=wf.WF_BF16, num_ctas=148)
    n = wf.wf_plan_bytes(d)
    buf = np.zeros(n + 64, dtype=np.uint8)
    off = (-buf.ctypes.data) % 16
    want = buf[off:off + n]
    wf.wf_plan_round(d, want)
    assert got.size == n and np.array_equal(got, want)
