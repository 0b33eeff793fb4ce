"""Pools in pinned host memory (kvq_cache.host_tiers; AMASS "What is in the box", Stage B:
a host-DRAM pool the device reads in place).  The attention kernel fetches those pages
with per-lane asynchronous loads instead of bulk copies; every byte and every output must
equal the all-device cache's, and the step must still match the oracle."""
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


def _run(kvq, w, host_tiers):
    cache = kvq.cache_from_workload(w, host_tiers=host_tiers)
    step = kvq.DecodeStep(w, cache)
    step.run()
    torch.cuda.synchronize()
    assert cache.err_bits() == 0, hex(cache.err_bits())
    if host_tiers:
        assert any(p is not None and not p.is_cuda for p in cache.pools)
    return dict(out=step.out.cpu().view(torch.int16).numpy(), lse=step.lse.cpu().numpy(),
                sel=step.sel.cpu().numpy(), cnt=step.cnt.cpu().numpy(),
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


def test_fused_step_rejects_host_pools(kvq):
    w = CASES["c1_16bit"]()
    cache = kvq.cache_from_workload(w, host_tiers=0b1)
    step = kvq.DecodeStep(w, cache)
    with pytest.raises(kvq.KvqError):
        step.run_fused()
