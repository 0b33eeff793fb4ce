"""Pools in pinned host memory (AMASS "What is in the box", Stage B: a host-DRAM pool the
device reads in place), in both variants the page names: K and V of a tier in host memory
(kvq_cache.host_tiers, "mem-kv"), or only the V chunks, in a pool of their own, with the
K chunks resident on the device (kvq_cache.vpool + host_vtiers, "mem-v").  The attention
kernel fetches host chunks with per-lane asynchronous loads and device chunks with bulk
copies; every byte, selection and output must equal the all-device cache's, and the
step must still match the oracle.  A separate V pool on the device (layout only) is
checked the same way."""
import numpy as np
import pytest
import torch

from oracle.step import prepare
from sparse_mixed_precision_kvq_b200 import workloads as W
from tests.parity_helpers import check_output, oracle_step, out_to_f64, query_and_new

pytestmark = pytest.mark.gpu

ALL_TIERS = {W.TIER_F16: 0.16, W.TIER_I8: 0.17, W.TIER_I4: 0.17, W.TIER_I2: 0.17, W.TIER_I1: 0.17, W.TIER_F8: 0.16}
CASES = {
    "c1_16bit": lambda: W.small("c1"),
    "alltiers_f16_d64": lambda: W.make("c0", B=2, lens=np.array([1000, 333]), append=True, tier_fracs=ALL_TIERS),
    "alltiers_bf16_d128": lambda: W.make("c1", B=2, Hq=16, Hkv=4, lens=np.array([700, 1500]), tier_fracs=ALL_TIERS,
                                         k_frac_bp=2000),
}


@pytest.fixture(scope="module")
def kvq():
    from sparse_mixed_precision_kvq_b200 import kvq as k
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return k


def _run(kvq, w, host_tiers, v_tiers=0, host_v_tiers=0):
    cache = kvq.cache_from_workload(w, host_tiers=host_tiers, v_tiers=v_tiers, host_v_tiers=host_v_tiers)
    step = kvq.DecodeStep(w, cache)
    step.run()
    torch.cuda.synchronize()
    assert cache.err_bits() == 0, hex(cache.err_bits())
    if host_tiers:
        assert any(p is not None and not p.is_cuda for p in cache.pools)
    if host_v_tiers:
        assert any(v is not None and not v.is_cuda for v in cache.vpools)
    chunks = {}  # every chunk of every (b, page, g, kind), wherever the layout puts it
    for b in range(w.B):
        for p in range(w.pages_after(b)):
            for g in range(w.Hkv):
                for kind in (0, 1):
                    chunks[(b, p, g, kind)] = cache.chunk_view(b, p, g, kind)[1].cpu().numpy()
    return dict(out=step.out.cpu().view(torch.int16).numpy(), lse=step.lse.cpu().numpy(),
                sel=step.sel.cpu().numpy(), cnt=step.cnt.cpu().numpy(), chunks=chunks,
                pools=[None if p is None else p.cpu().numpy() for p in cache.pools])


@pytest.mark.parametrize("name,mask", [("c1_16bit", 0b000001), ("alltiers_f16_d64", 0b101010),
                                       ("alltiers_f16_d64", 0b111111), ("alltiers_bf16_d128", 0b010101)])
def test_host_pools_give_the_device_results(kvq, name, mask):
    w = CASES[name]()
    a, b = _run(kvq, w, 0), _run(kvq, w, mask)
    for key in ("out", "lse", "sel", "cnt"):
        assert np.array_equal(a[key], b[key]), key
    for pa, pb in zip(a["pools"], b["pools"]):
        assert (pa is None) == (pb is None) and (pa is None or np.array_equal(pa, pb))


@pytest.mark.parametrize("name,vmask,hvmask,hmask", [
    ("c1_16bit", 0b000001, 0b000001, 0),               # mem-v: 16-bit V in host memory, K on the device
    ("alltiers_f16_d64", 0b111111, 0b111111, 0),       # mem-v on every tier
    ("alltiers_bf16_d128", 0b111111, 0b010101, 0),     # mem-v on some tiers, device V pools on the others
    ("alltiers_bf16_d128", 0b101010, 0b001010, 0b100000),  # K and V in host memory for one tier too
    ("alltiers_bf16_d128", 0b111111, 0, 0),            # separate V pools, all on the device
])
def test_separate_v_pools_give_the_device_results(kvq, name, vmask, hvmask, hmask):
    w = CASES[name]()
    a, b = _run(kvq, w, 0), _run(kvq, w, hmask, v_tiers=vmask, host_v_tiers=hvmask)
    for key in ("out", "lse", "sel", "cnt"):
        assert np.array_equal(a[key], b[key]), key
    for k, ca in a["chunks"].items():
        assert np.array_equal(ca, b["chunks"][k]), k


def test_mem_v_matches_the_oracle(kvq):
    w = CASES["alltiers_bf16_d128"]()
    cache = kvq.cache_from_workload(w, host_v_tiers=0b111111)
    step = kvq.DecodeStep(w, cache)
    step.run()
    torch.cuda.synchronize()
    assert cache.err_bits() == 0
    q, kn, vn = query_and_new(w)
    out = out_to_f64(step.out, w.dtype)
    sel, cnt = step.sel.cpu().numpy(), step.cnt.cpu().numpy()
    for b in range(w.B):
        for g in range(w.Hkv):
            r = oracle_step(w, prepare(w, b, g), b, g, q, kn, vn, sel=sel[b, g, :cnt[b, g]])
            for i in range(w.G):
                check_output(out[b, g * w.G + i], r["out"][i], f"b={b} g={g} h={i}", w.dtype)


def test_demotion_into_and_out_of_a_host_v_pool(kvq):
    """kvq_requantize_pages reads and writes separate (host) V chunks like adjacent ones."""
    w = W.make("c1", B=2, Hq=8, Hkv=2, lens=np.array([300, 170]), append=False)
    _, _, counts = w.slot_map()
    items, nxt = [], list(counts)       # new slots follow the used ones of each pool
    for b in range(w.B):
        for p in range(1, w.pages_before(b) - 1):
            t = 2 if p % 2 else 4
            items.append((b, p, int(np.uint32((t << 29) | nxt[t]).view(np.int32))))
            nxt[t] += 1
    spare = [n - c for n, c in zip(nxt, counts)]
    res = []
    for vm in (0, 0b111111):
        cache = kvq.cache_from_workload(w, spare=spare, host_v_tiers=vm)
        kvq.kvq_requantize_pages(cache, torch.tensor(items, dtype=torch.int32, device="cuda"))
        torch.cuda.synchronize()
        assert cache.err_bits() == 0
        res.append({(b, p, g, k): cache.chunk_view(b, p, g, k)[1].cpu().numpy()
                    for b in range(w.B) for p in range(w.pages_before(b)) for g in range(w.Hkv) for k in (0, 1)})
    for key, ca in res[0].items():
        assert np.array_equal(ca, res[1][key]), key


def test_host_pools_match_the_oracle(kvq):
    w = CASES["alltiers_bf16_d128"]()
    cache = kvq.cache_from_workload(w, host_tiers=0b111111)
    step = kvq.DecodeStep(w, cache)
    step.run()
    torch.cuda.synchronize()
    assert cache.err_bits() == 0
    q, kn, vn = query_and_new(w)
    out = out_to_f64(step.out, w.dtype)
    sel, cnt = step.sel.cpu().numpy(), step.cnt.cpu().numpy()
    for b in range(w.B):
        for g in range(w.Hkv):
            r = oracle_step(w, prepare(w, b, g), b, g, q, kn, vn, sel=sel[b, g, :cnt[b, g]])
            for i in range(w.G):
                check_output(out[b, g * w.G + i], r["out"][i], f"b={b} g={g} h={i}", w.dtype)


@pytest.mark.parametrize("opts", [dict(host_tiers=0b1), dict(v_tiers=0b1), dict(host_v_tiers=0b1)])
def test_fused_step_rejects_host_and_separate_pools(kvq, opts):
    w = CASES["c1_16bit"]()
    cache = kvq.cache_from_workload(w, **opts)
    step = kvq.DecodeStep(w, cache)
    with pytest.raises(kvq.KvqError):
        step.run_fused()
