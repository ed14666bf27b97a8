"""Register pressure of the kernels, from what ptxas reports (CPU, no GPU).

Every kernel source is compiled for sm_100a with the library's flags and
`-Xptxas -v`; no entry function may spill registers beyond the allowance
below. The allowances are the spills measured today, all on paths that the
timed workloads do not take, except the block selection with fused coarse
scores at d_I = 128 (36 bytes), which is on the 16 x 128K decode path.
"""
from __future__ import annotations

import os
import re
import shutil
import subprocess

import pytest

from long_context_sparse_lsa_b200 import build

# mangled-name fragment -> spill-store bytes accepted
KNOWN_SPILLS = {
    "attend_kernelILi2E": 400,            # groups of 16 query heads (TMA bulk-copy K path)
    "fine_score_kernelILi128ELi8E": 400,  # 64 indexer heads, per-lane gathers
    "fine_score_tma_kernelILi8E": 128,    # 64 indexer heads
    "select_kernelImLb0ELi128ELi2E": 40,  # block selection with coarse scores, d_I 128, <= 16 heads
    "select_kernelImLb0ELi64ELi2E": 16,   # the same at d_I 64
    "select_kernelImLb0ELi64ELi1E": 8,    # d_I 64, <= 8 heads
}
HOT = ["attend_rk_kernelILb0E", "attend_rk_kernelILb1E", "attend_merge_kernel", "fine_score_tma_kernelILi2E",
       "select_kernelIjLb1ELi0ELi0E", "fine_score_tc_kernel", "append_kernelILi128E", "block_sums_kernelILi128E"]


def _spills(src: str) -> dict[str, int]:
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    out = os.path.join(build.BUILD_DIR, "ptxas_check.o")
    os.makedirs(build.BUILD_DIR, exist_ok=True)
    cmd = [nvcc, *build.ARCH, *build.NVCC_FLAGS, "-Xptxas", "-v", "-c", os.path.join(build.CSRC, src), "-o", out]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr[-2000:]
    found, cur = {}, None
    for line in r.stderr.splitlines():
        m = re.search(r"Function properties for (\S+)", line)
        if m:
            cur = m.group(1)
        m = re.search(r"(\d+) bytes spill stores", line)
        if m and cur is not None:
            found[cur] = int(m.group(1))
    return found


@pytest.mark.skipif(shutil.which("nvcc") is None and not os.path.exists("/usr/local/cuda/bin/nvcc"),
                    reason="nvcc not available")
def test_no_unexpected_register_spills():
    found = {}
    for src in ("attend.cu", "index_score.cu", "index_select.cu", "index_prefill_tc.cu", "block_sums.cu"):
        found.update(_spills(src))
    assert found, "ptxas reported no functions"
    for fn, spill in found.items():
        allow = max([v for k, v in KNOWN_SPILLS.items() if k in fn], default=0)
        assert spill <= allow, f"{fn}: {spill} bytes of spill stores (allowed {allow})"
    # the hot kernels are all there and spill nothing
    for frag in HOT:
        hits = [fn for fn in found if frag in fn]
        assert hits, f"no entry function matches {frag}"
        assert all(found[fn] == 0 for fn in hits), frag
