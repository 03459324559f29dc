"""Static resource checks of the CUDA kernels, without a GPU: every kernel is
compiled for sm_100a with ptxas's resource report, and no instantiation may
spill registers to local memory."""
import concurrent.futures as cf
import os
import re
import shutil
import subprocess

import pytest

from query_aware_sparse_tb_b200 import build

def _ptxas_report(src):
    cmd = [build.NVCC, *build.FLAGS, "-Xptxas", "-v", "-c", os.path.join(build.CSRC, src), "-o", os.devnull]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr
    return res.stderr


def _spills(report):
    """{mangled kernel name: spill-store bytes} from a ptxas -v report."""
    out, cur = {}, None
    for line in report.splitlines():
        m = re.search(r"Compiling entry function '([^']+)'", line)
        if m:
            cur = m.group(1)
        m = re.search(r"(\d+) bytes spill stores", line)
        if m and cur is not None:
            out[cur] = int(m.group(1))
    return out


def test_no_register_spills():
    if shutil.which(build.NVCC) is None:
        pytest.skip("nvcc not available")
    with cf.ThreadPoolExecutor(len(build.SOURCES)) as ex:
        reports = list(ex.map(_ptxas_report, build.SOURCES))
    spills = {}
    for r in reports:
        spills.update(_spills(r))
    assert any("attn_kernel" in k for k in spills) and any("score_hist_kernel" in k for k in spills)
    assert any("sel_cluster_kernel" in k for k in spills)
    bad = {k: v for k, v in spills.items() if v > 0}
    assert not bad, f"kernels that spill registers: {bad}"
