"""The hot kernels compile for sm_100a without register spills (ptxas -v, no GPU needed).

A spill puts per-thread state in local memory on the page loop's critical path; this
check runs the compiler the build uses on the attention and score units and reads the
resource report it prints for every kernel."""
import os
import re
import shutil
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "sparse_mixed_precision_kvq_b200", "csrc")


# Known: the fused score + select instance of score_kernel (MODE 2, kvq_score_select, not on
# the default four-call path) keeps 4 bytes of its selection state in local memory at
# D = 128 bf16.
ALLOWED = {"12score_kernelILi128ELb1ELi2E": 4}


@pytest.mark.parametrize("unit,kernel", [("attn.cu", "attn_kernel"), ("score.cu", "score_kernel"),
                                         ("select.cu", "select_kernel"), ("quad.cu", "quad_score_kernel"),
                                         ("append.cu", "requant_kernel")])
def test_no_spills(unit, kernel):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    with tempfile.TemporaryDirectory() as tmp:
        from sparse_mixed_precision_kvq_b200 import build as B   # the build's own flags
        r = subprocess.run([nvcc, *B.ARCH, *B.COMMON, *B.PER_FILE.get(unit, []), "-Xptxas", "-v", "-c",
                            os.path.join(CSRC, unit), "-o", os.path.join(tmp, "u.o")],
                           capture_output=True, text=True)
    assert r.returncode == 0, r.stderr[-2000:]
    report = r.stdout + r.stderr
    blocks = re.split(r"Compiling entry function", report)
    seen = 0
    for blk in blocks[1:]:
        name = blk.split("'")[1] if "'" in blk else ""
        if kernel not in name:
            continue
        seen += 1
        m = re.search(r"(\d+) bytes spill stores, (\d+) bytes spill loads", blk)
        assert m is not None, name
        allowed = max([v for k, v in ALLOWED.items() if k in name], default=0)
        assert int(m.group(1)) <= allowed and int(m.group(2)) <= allowed, f"{name}: {m.group(0)}"
    assert seen > 0
