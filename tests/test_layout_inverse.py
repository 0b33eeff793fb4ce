"""Host programs compiled with nvcc (no GPU needed): the packed-word decoder used by the
re-quantiser inverts the writer's layout map, and the library's element map equals the
oracle's independently written layout."""
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


def test_library_element_map_equals_the_oracle_layout():
    """The library's element -> (word, bit) map (host build of elem_pos) equals the
    oracle's independently written layout for every tier, kind and D."""
    import numpy as np
    from oracle.layout import _positions
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    with tempfile.TemporaryDirectory() as tmp:
        exe = os.path.join(tmp, "layout_dump")
        subprocess.run([nvcc, "-std=c++17", "-x", "cu", "-Wno-deprecated-gpu-targets",
                        "-I", os.path.join(ROOT, "include"),
                        "-I", os.path.join(ROOT, "sparse_mixed_precision_kvq_b200", "csrc"),
                        os.path.join(ROOT, "tests", "layout_dump.cu"), "-o", exe],
                       check=True, capture_output=True)
        out = subprocess.run([exe], capture_output=True, text=True, check=True).stdout
    rows = np.array([list(map(int, ln.split())) for ln in out.splitlines()])
    n = 0
    for tier in range(6):
        for kind in range(2):
            for D in (64, 128):
                sel = rows[(rows[:, 0] == tier) & (rows[:, 1] == kind) & (rows[:, 2] == D)]
                word, bit = _positions("kv"[kind], tier, D)
                assert np.array_equal(sel[:, 5], word[sel[:, 3], sel[:, 4]]), (tier, kind, D)
                assert np.array_equal(sel[:, 6], bit[sel[:, 3], sel[:, 4]]), (tier, kind, D)
                n += sel.shape[0]
    assert n == 6 * 2 * 16 * (64 + 128)
