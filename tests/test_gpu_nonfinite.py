"""Non-finite input in an FP8 page: flagged, stored as the oracle stores it, and read back
alike by the fp16 and the bf16 paths.

A key holding a NaN (or an infinity) lands in an FP8 page.  The library flags
KVQ_DERR_NONFINITE, stores the group with the fp16 NaN scale 0x7E00 and zero codes (the
oracle's bytes, bit for bit), reads the whole group back as NaN (kvq_dequant_page), and
the attention of that kv head over the page is NaN in both 16-bit types, while the other
kv head, which holds only finite values, still matches the oracle.
"""
import numpy as np
import pytest
import torch

from oracle.cache import build, page_bytes
from sparse_mixed_precision_kvq_b200 import workloads as W
from tests.parity_helpers import check_output, gpu_chunk, oracle_outputs_on, out_to_f64, pools_to_cpu, query_and_new

pytestmark = pytest.mark.gpu

BAD = {"f16": 0x7E00, "bf16": 0x7FC0}   # quiet NaN patterns


@pytest.mark.parametrize("bad_value", ["nan", "inf"])
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_fp8_group_with_nonfinite_key(dtype, bad_value):
    from sparse_mixed_precision_kvq_b200 import kvq
    w = W.make("c0", lens=np.array([64]), append=False, dtype=dtype, tier_fracs={W.TIER_F8: 1.0},
               k_abs=100, n_recent=0)
    tier_tbl, slot_tbl, counts = w.slot_map()
    cache = kvq.PagedCache(w.B, w.Hq, w.Hkv, w.D, w.max_pages, w.dtype, counts)
    cache.block_table.copy_(torch.from_numpy(kvq.encode_block_table(tier_tbl, slot_tbl)))
    cache.seq_len.copy_(torch.from_numpy(w.lens.astype(np.int32)))
    keys = [w.keys_bits(0, g).copy() for g in range(w.Hkv)]
    vals = [w.values_bits(0, g) for g in range(w.Hkv)]
    inf_bits = 0x7C00 if dtype == "f16" else 0x7F80
    keys[1][20, 37] = BAD[dtype] if bad_value == "nan" else inf_bits   # page 1, channel group 1 of kv head 1
    ksrc = torch.from_numpy(np.stack(keys).view(np.int16)).cuda()
    vsrc = torch.from_numpy(np.stack(vals).view(np.int16)).cuda()
    cu = torch.tensor([0, 64], dtype=torch.int64, device="cuda")
    kvq.kvq_build_pages(cache, ksrc, vsrc, cu)
    torch.cuda.synchronize()
    assert cache.err_bits() & kvq.DERR_NONFINITE

    pools, bt = pools_to_cpu(cache), cache.block_table.cpu().numpy()
    shs = [build(keys[g], vals[g], w.dtype, w.tiers(0), capacity_pages=w.max_pages) for g in range(w.Hkv)]
    for g in range(w.Hkv):
        for p in range(4):
            for kind, kk in ((0, "k"), (1, "v")):
                _, got = gpu_chunk(pools, bt, w.Hkv, w.D, 0, p, g, kind)
                assert np.array_equal(got, page_bytes(shs[g], p, kk)), (g, p, kk)
    # the group reads back as NaN, its neighbours as the oracle's values
    out = torch.empty((w.Hkv, 2, 16, w.D), dtype=torch.float32, device="cuda")
    kvq.kvq_dequant_page(cache, 0, 1, out)
    got = out.cpu().numpy().astype(np.float64)
    assert np.all(np.isnan(got[1, 0, 4, 32:64]))
    assert np.array_equal(got[1, 0, 4, :32], shs[1].khat[20, :32])
    assert np.array_equal(got[0, 0], shs[0].khat[16:32])

    # attention over all four pages: NaN for kv head 1's query heads, the oracle's for kv head 0
    q, _, _ = query_and_new(w)
    step = kvq.DecodeStep(w, cache)
    sel = torch.arange(4, dtype=torch.int32, device="cuda").repeat(w.B, w.Hkv, 1).contiguous()
    cnt = torch.full((w.B, w.Hkv), 4, dtype=torch.int32, device="cuda")
    kvq.kvq_sparse_decode_attn(cache, step.q, sel, cnt, 4, w.sm_scale, step.out, step.lse, step.ws)
    torch.cuda.synchronize()
    o = out_to_f64(step.out, w.dtype)
    G = w.G
    assert np.all(np.isnan(o[0, G:2 * G]))
    ref, _ = oracle_outputs_on(w, shs[0], 0, 0, q, np.arange(4))
    for i in range(G):
        check_output(o[0, i], ref[i], f"{dtype} head {i}", w.dtype)
