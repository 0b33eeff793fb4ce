"""The packed-word decoder used by the re-quantiser inverts the writer's layout map
(host program compiled with nvcc; no GPU needed)."""
import os
import shutil
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_word_decoder_inverts_the_element_map():
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    with tempfile.TemporaryDirectory() as tmp:
        exe = os.path.join(tmp, "layout_inverse_check")
        subprocess.run([nvcc, "-std=c++17", "-x", "cu", "-Wno-deprecated-gpu-targets", "-diag-suppress", "20011",
                        "-I", os.path.join(ROOT, "include"),
                        "-I", os.path.join(ROOT, "sparse_mixed_precision_kvq_b200", "csrc"),
                        os.path.join(ROOT, "tests", "layout_inverse_check.cu"), "-o", exe],
                       check=True, capture_output=True)
        r = subprocess.run([exe], capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "mismatches: 0" in r.stdout
