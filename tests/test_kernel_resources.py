"""The tensor-core kernels compile for sm_100a without register spills.

A spill puts per-thread state in local memory: in the attention's softmax
loop, the backward's softmax pieces or a projection's epilogue it costs far
more than it saves, and nothing else in the CPU suite would notice it.  The
check compiles each kernel source once with ptxas' resource report (no
device needed) and reads the spill counts it prints for every entry
function.
"""
import os
import re
import shutil
import subprocess
import tempfile
from concurrent.futures import ThreadPoolExecutor

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(ROOT, "causal_attention_rtr_b200", "csrc")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
SOURCES = ["attn_tc.cu", "attn_bwd.cu", "gemm_tc.cu"]


def _report(src, out_dir):
    cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
           "-I" + os.path.join(ROOT, "include"), "-I" + CSRC, "--expt-relaxed-constexpr",
           "-Xptxas", "-v", "-c", os.path.join(CSRC, src), "-o", os.path.join(out_dir, src + ".o")]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr[-2000:]
    return res.stderr


@pytest.mark.skipif(not (os.path.exists(NVCC) or shutil.which("nvcc")), reason="nvcc not available")
def test_tensor_core_kernels_do_not_spill():
    with tempfile.TemporaryDirectory() as d:
        with ThreadPoolExecutor(len(SOURCES)) as ex:
            reports = dict(zip(SOURCES, ex.map(lambda s: _report(s, d), SOURCES)))
    for src, text in reports.items():
        entries = re.findall(r"Compiling entry function '([^']+)'", text)
        spills = re.findall(r"(\d+) bytes spill stores, (\d+) bytes spill loads", text)
        assert entries and len(spills) == len(entries), f"{src}: could not read the ptxas report"
        bad = [(name, s, l) for name, (s, l) in zip(entries, spills) if int(s) or int(l)]
        assert not bad, f"{src}: spills in {bad}"
