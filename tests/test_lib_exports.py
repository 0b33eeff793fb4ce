"""The C-ABI library loads and exports every symbol include/kvq.h declares (no GPU needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kvq.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(kvq_[a-z_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from sparse_mixed_precision_kvq_b200 import build
    path = build.build()
    return ctypes.CDLL(path)


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert len(names) >= 9
    for n in names:
        assert hasattr(lib, n), n


def test_binding_mirrors_the_header():
    from sparse_mixed_precision_kvq_b200 import kvq
    assert sorted(kvq.EXPORTS) == _declared()
    for n in kvq.EXPORTS:
        assert callable(getattr(kvq, n))


def _param_counts():
    src = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    out = {}
    for name, params in re.findall(r"\b(kvq_[a-z_]+)\s*\(([^)]*)\)\s*;", src):
        params = params.strip()
        out[name] = 0 if params in ("", "void") else params.count(",") + 1
    return out


def test_every_binding_declares_its_argument_types():
    """Without argtypes ctypes passes a Python int as a C int, which would truncate a
    device pointer; every entry point must declare one ctypes type per header parameter,
    and a pointer-sized type wherever the header takes a pointer."""
    from sparse_mixed_precision_kvq_b200 import kvq
    counts = _param_counts()
    assert sorted(counts) == _declared()
    src = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    for n in kvq.EXPORTS:
        at = getattr(kvq._lib, n).argtypes
        assert at is not None and len(at) == counts[n], n
        params = re.search(n + r"\s*\(([^)]*)\)", src).group(1).strip()
        if params in ("", "void"):
            continue
        for decl, ty in zip(params.split(","), at):
            if "*" in decl or "stream" in decl:
                assert ctypes.sizeof(ty) == 8, (n, decl)


def test_host_helpers_without_gpu():
    from sparse_mixed_precision_kvq_b200 import kvq
    assert [2 * kvq.kvq_chunk_bytes(t, 128) for t in range(6)] == [8192, 4608, 2560, 1536, 768, 4352]
    assert kvq.kvq_chunk_bytes(6, 128) == 0 and kvq.kvq_chunk_bytes(0, 96) == 0
    assert kvq.kvq_status_string(0) == "ok" and "workspace" in kvq.kvq_status_string(3)


def _check_invalid_arguments_rejected_on_host():
    """Argument checks run before any CUDA call, so they work without a device."""
    from sparse_mixed_precision_kvq_b200 import kvq
    c = kvq.KvqCache()
    c.B, c.Hq, c.Hkv, c.D, c.page_size, c.max_pages, c.dtype = 1, 8, 2, 96, 16, 4, 0
    st = kvq._lib.kvq_page_scores(ctypes.byref(c), None, None, None)
    assert st == 2          # D = 96 unsupported
    c.D = 64
    st = kvq._lib.kvq_page_scores(ctypes.byref(c), None, None, None)
    assert st == 1          # null pointers
    c.Hq = 24               # G = 12 > 8
    assert kvq._lib.kvq_append(ctypes.byref(c), None, None, None, None) == 2


def _check_quad_arguments_rejected_on_host():
    """Every case fails its host-side check before anything is enqueued (no device needed)."""
    from sparse_mixed_precision_kvq_b200 import kvq
    c = kvq.KvqCache()
    c.B, c.Hq, c.Hkv, c.D, c.page_size, c.max_pages, c.dtype = 1, 8, 2, 64, 16, 4, 1
    c.block_table = c.seq_len = c.summary = c.open_ksum = c.err_word = 4096
    c.pool[0], c.pool_slots[0] = 4096, 4
    qd = kvq.KvqQuad()
    qd.rank, qd.basis, qd.lambda_, qd.open_sums = 12, 4096, 4096, 4096
    ref, qref = ctypes.byref(c), ctypes.byref(qd)
    assert kvq._lib.kvq_quad_page_scores(ref, qref, 4096, 0.1, 4096, None) == 2      # rank 12: unsupported
    qd.rank = 40
    assert kvq._lib.kvq_quad_append(ref, qref, 4096, 4096, None) == 2                # rank 40 > 32
    qd.rank = 16
    assert kvq._lib.kvq_quad_page_scores(ref, qref, 4096, 0.0, 4096, None) == 1      # sm_scale 0
    assert kvq._lib.kvq_quad_page_scores(ref, qref, 4100, 0.1, 4096, None) == 1      # q not 16-byte aligned
    assert kvq._lib.kvq_quad_page_scores(ref, None, 4096, 0.1, 4096, None) == 1      # no quad state
    qd.lambda_ = 4104
    assert kvq._lib.kvq_quad_build(ref, qref, 4096, 4096, 16, None) == 1             # lambda not 16-byte aligned
    qd.lambda_, qd.basis = 4096, None
    assert kvq._lib.kvq_quad_append(ref, qref, 4096, 4096, None) == 1                # no basis
    qd.basis, qd.rank = 4096, 12
    assert kvq._lib.kvq_quad_append_scores(ref, qref, 4096, 4096, 4096, 4096, 0.1, 4096, None) == 2  # rank 12
    qd.rank = 16
    assert kvq._lib.kvq_quad_append_scores(ref, qref, None, 4096, 4096, 4096, 0.1, 4096, None) == 1  # no pos
    assert kvq._lib.kvq_quad_append_scores(ref, qref, 4096, 4096, 4096, 4096, -1.0, 4096, None) == 1  # bad scale


def _check_host_tiers_mask_checked_on_host():
    """A host_tiers bit past the last tier is rejected before anything is enqueued."""
    from sparse_mixed_precision_kvq_b200 import kvq
    c = kvq.KvqCache()
    c.B, c.Hq, c.Hkv, c.D, c.page_size, c.max_pages, c.dtype = 1, 8, 2, 64, 16, 4, 1
    c.block_table = c.seq_len = c.summary = c.open_ksum = c.err_word = 4096
    c.pool[0], c.pool_slots[0] = 4096, 4
    c.host_tiers = 1 << 6
    assert kvq._lib.kvq_page_scores(ctypes.byref(c), 4096, 4096, None) == 1
    assert kvq._lib.kvq_append(ctypes.byref(c), 4096, 4096, 4096, None) == 1


def test_single_tier_workload_override():
    """bench --tier T: every prefilled page at tier T, the page opened by the append 16-bit."""
    import numpy as np
    import bench
    for tier in range(6):
        w = bench.rank_workload("c1", 0, batch=2, tier=tier)
        for b in range(w.B):
            t = w.tiers(b)
            P0 = w.pages_before(b)
            assert np.all(t[:P0] == tier) and np.all(t[P0:] == 0)


def test_algorithmic_bytes_by_hand():
    """The roofline numerator: selected K+V chunks per tier + q + out + page lists for the
    attention; every page summary + q + the fp32 scores for the page scores."""
    import numpy as np
    import bench
    from sparse_mixed_precision_kvq_b200 import workloads as W
    w = W.make("c0", lens=np.array([100]), tier_fracs={W.TIER_F16: 0.5, W.TIER_I4: 0.5})
    tier_tbl, _, _ = w.slot_map()
    sel = np.array([[[0, 3, 6], [1, 2, 0]]], dtype=np.int32)
    cnt = np.array([[3, 2]], dtype=np.int32)
    nb = bench.algorithmic_bytes(w, sel, cnt, tier_tbl)
    chunk = {0: 2 * 16 * 64 * 2, 2: 2 * (16 * 64 // 2 + 16 * 2 * 4)}   # K+V at D = 64
    pages = [int(tier_tbl[0, p]) for p in (0, 3, 6, 1, 2)]
    qo = 2 * (1 * 8 * 64 * 2)
    assert nb["attn"] == sum(chunk[t] for t in pages) + qo + 5 * 4
    P = (100 + 15) // 16
    assert nb["score"] == P * 2 * 64 * 2 + 8 * 64 * 2 + 2 * w.max_pages * 4
    assert nb["append"] == 0 and nb["select"] == 2 * w.max_pages * 4 + 5 * 4
    nq = bench.algorithmic_bytes(w, sel, cnt, tier_tbl, quad_rank=16)
    assert nq["score"] - nb["score"] == P * 2 * 16 * 2


def test_kernel_rooflines_cover_every_path():
    import bench
    nbytes = dict(attn=1000, score=300, select=20, append=40)
    paths = {"calls": ["append", "page_scores", "select_topk", "sparse_decode_attn"],
             "three": ["append_scores", "select_topk", "sparse_decode_attn"],
             "two": ["score_select", "sparse_decode_attn"], "fused": ["decode_step"]}
    for names in paths.values():
        r = bench.kernel_rooflines(names, [0.001] * len(names), nbytes, peak=1.0)
        assert sum(v["bytes"] for v in r.values()) == 1360
        for v in r.values():
            assert abs(v["gbs"] - v["bytes"] / 1e-6 / 1e9) < 1e-9 and v["frac"] == v["gbs"]


def test_plain_c_caller(lib):
    """The header compiles as C99 and a plain C program links libkvq and gets answers from
    its host-only entry points (no GPU)."""
    import shutil
    import subprocess
    import tempfile
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    libdir = os.path.join(ROOT, "sparse_mixed_precision_kvq_b200", "lib")
    with tempfile.TemporaryDirectory() as tmp:
        exe = os.path.join(tmp, "c_abi_check")
        subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
                        os.path.join(ROOT, "tests", "c_abi_check.c"), "-L", libdir, "-lkvq",
                        "-Wl,-rpath," + libdir, "-o", exe], check=True, capture_output=True)
        r = subprocess.run([exe], capture_output=True, text=True)
    assert r.returncode == 0 and "c abi ok" in r.stdout, (r.returncode, r.stdout, r.stderr)


def _check_requantize_arguments_checked_on_host():
    """n < 0 or missing items are rejected, n == 0 is a no-op, all before anything is enqueued."""
    from sparse_mixed_precision_kvq_b200 import kvq
    c = kvq.KvqCache()
    c.B, c.Hq, c.Hkv, c.D, c.page_size, c.max_pages, c.dtype = 1, 8, 2, 64, 16, 4, 1
    c.block_table = c.seq_len = c.summary = c.open_ksum = c.err_word = 4096
    c.pool[0], c.pool_slots[0] = 4096, 4
    ref = ctypes.byref(c)
    assert kvq._lib.kvq_requantize_pages(ref, 4096, -1, None) == 1
    assert kvq._lib.kvq_requantize_pages(ref, None, 3, None) == 1
    assert kvq._lib.kvq_requantize_pages(ref, None, 0, None) == 0


def _check_coverage_limits_on_host():
    """Coverage selection's limits are checked before anything is enqueued: at most 8192
    candidates, at most 41984 pages (the cut's scratch), coverage <= 1, sm_scale > 0."""
    from sparse_mixed_precision_kvq_b200 import kvq
    c = kvq.KvqCache()
    c.B, c.Hq, c.Hkv, c.D, c.page_size, c.dtype = 1, 8, 2, 64, 16, 1
    c.block_table = c.seq_len = c.summary = c.open_ksum = c.err_word = 4096
    c.pool[0], c.pool_slots[0] = 4096, 4
    ref = ctypes.byref(c)

    def sel(max_pages, ns, nr, ppm, scale):
        c.max_pages = max_pages
        prm = kvq.SelectParams(-1, 0, ns, nr, ppm, scale)
        return kvq._lib.kvq_select_topk(ref, 4096, ctypes.byref(prm), 4096, 4096, max_pages, None)

    assert sel(9000, 0, 0, 950000, 0.1) == 2            # 9000 candidates > 8192
    assert sel(42000, 1, 33999, 950000, 0.1) == 2       # 8000 candidates, but 42000 pages > 41984
    assert sel(4000, 1, 4, 1000001, 0.1) == 1           # coverage above 1
    assert sel(4000, 1, 4, 950000, 0.0) == 1            # sm_scale 0


def _run_without_gpu(check: str):
    """Run ``check`` (a function of this module) in a child process that sees no CUDA
    device.  These checks hand made-up device addresses to the entry points and rely on
    the host-side argument checks rejecting the call; if a check ever let one through,
    the launch would fail with "no device" in the child instead of touching memory."""
    import subprocess
    import sys
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    code = f"import sys; sys.path.insert(0, {ROOT!r}); import tests.test_lib_exports as t; t.{check}()"
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr


def test_invalid_arguments_rejected_on_host():
    _run_without_gpu('_check_invalid_arguments_rejected_on_host')


def test_quad_arguments_rejected_on_host():
    _run_without_gpu('_check_quad_arguments_rejected_on_host')


def test_host_tiers_mask_checked_on_host():
    _run_without_gpu('_check_host_tiers_mask_checked_on_host')


def test_requantize_arguments_checked_on_host():
    _run_without_gpu('_check_requantize_arguments_checked_on_host')


def test_coverage_limits_checked_on_host():
    _run_without_gpu('_check_coverage_limits_on_host')


def test_recorded_traffic_applies_only_to_its_workload_and_source():
    """bench reports the ncu DRAM bytes of profiles/traffic.json only for a plain run of the
    workload they were captured on, and only while the kernel's source (its file and the
    package headers it includes) is the one captured."""
    import json
    import bench
    rec = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))["attn.cu"]
    assert bench.kernel_traffic("attn.cu", None) is None
    other = "c2" if rec["workload"] != "c2" else "c1"
    assert bench.kernel_traffic("attn.cu", other) is None
    got = bench.kernel_traffic("attn.cu", rec["workload"])
    if rec["source_sha256_16"] == bench.kernel_source_hash("attn.cu"):
        assert got is not None and got["dram_bytes_per_launch"] == rec["dram_bytes_per_launch"]
    else:
        assert got is None
