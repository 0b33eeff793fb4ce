"""kvq_sparse_decode_attn_noalloc: the attention entry point that allocates nothing.

Callers that cannot allocate device memory at decode time (an engine that gave its device
memory to its own KV page pool, a plugin without an allocation hook) use this variant; its
split-K scratch is a static device array inside the library.  This file is collected last
so that a run stopping at the first failure has run every other test first.

The check: through the C ABI, on two calls in a row (two different workloads, so stale
scratch from the first call cannot hide a bug in the second), the output and
log-sum-exp equal those of kvq_sparse_decode_attn with a caller workspace, within the
output tolerance the parity tests use.  Also: a batch beyond the static scratch is
rejected, and a batch with too many (sequence, kv head) segments gets the same status
from both entry points.
"""
import numpy as np
import pytest
import torch

from sparse_mixed_precision_kvq_b200 import workloads as W
from tests.parity_helpers import check_output, out_to_f64

pytestmark = pytest.mark.gpu


def _case(kvq, w):
    cache = kvq.cache_from_workload(w)
    step = kvq.DecodeStep(w, cache)
    step.run()                                   # reference: caller-provided workspace
    torch.cuda.synchronize()
    ref_out, ref_lse = out_to_f64(step.out, w.dtype), step.lse.cpu().numpy()
    out = torch.full_like(step.out, float("nan"))
    lse = torch.full_like(step.lse, float("nan"))
    kvq.kvq_sparse_decode_attn_noalloc(cache, step.q, step.sel, step.cnt, step.kmax, w.sm_scale, out, lse)
    torch.cuda.synchronize()
    assert cache.err_bits() == 0
    got_out, got_lse = out_to_f64(out, w.dtype), lse.cpu().numpy()
    for b in range(w.B):
        for h in range(w.Hq):
            check_output(got_out[b, h], ref_out[b, h], f"noalloc b={b} h={h}", w.dtype)
    fin = np.isfinite(ref_lse)
    assert np.array_equal(fin, np.isfinite(got_lse))
    assert np.allclose(got_lse[fin], ref_lse[fin], rtol=1e-6, atol=1e-6)


def test_noalloc_matches_workspace_entry_point_twice():
    from sparse_mixed_precision_kvq_b200 import kvq
    assert torch.cuda.is_available()
    assert kvq.kvq_noalloc_scratch_bytes() == 16 << 20
    _case(kvq, W.small("c4"))                   # first call: ragged batch, all four tiers, G = 8
    _case(kvq, W.small("c1"))                   # second call: other shapes, 16-bit pages, G = 4


def test_noalloc_rejects_a_batch_beyond_the_static_scratch():
    from sparse_mixed_precision_kvq_b200 import kvq
    w = W.make("c4", B=1200, Hq=16, Hkv=2, lens=np.full(1200, 16), append=False)
    cache = kvq.PagedCache(w.B, w.Hq, w.Hkv, w.D, 2, w.dtype, [w.B * 2, 0, 0, 0, 0])
    assert kvq.kvq_workspace_size(cache, 2) > kvq.kvq_noalloc_scratch_bytes()
    q = torch.zeros((w.B, w.Hq, w.D), dtype=torch.bfloat16, device="cuda")
    sel = torch.zeros((w.B, w.Hkv, 2), dtype=torch.int32, device="cuda")
    cnt = torch.zeros((w.B, w.Hkv), dtype=torch.int32, device="cuda")
    out = torch.empty_like(q)
    with pytest.raises(kvq.KvqError, match="workspace"):
        kvq.kvq_sparse_decode_attn_noalloc(cache, q, sel, cnt, 2, w.sm_scale, out, None)


def test_noalloc_status_matches_the_workspace_entry_point():
    """B*Hkv >= 5632 segments: both entry points answer "unsupported"."""
    from sparse_mixed_precision_kvq_b200 import kvq
    B, Hq, Hkv, D = 3100, 4, 2, 128
    cache = kvq.PagedCache(B, Hq, Hkv, D, 1, "bf16", [B, 0, 0, 0, 0])
    q = torch.zeros((B, Hq, D), dtype=torch.bfloat16, device="cuda")
    sel = torch.zeros((B, Hkv, 1), dtype=torch.int32, device="cuda")
    cnt = torch.zeros((B, Hkv), dtype=torch.int32, device="cuda")
    out = torch.empty_like(q)
    ws = torch.zeros(1 << 14, dtype=torch.float32, device="cuda")
    with pytest.raises(kvq.KvqError, match="unsupported"):
        kvq.kvq_sparse_decode_attn(cache, q, sel, cnt, 1, 0.1, out, None, ws)
    with pytest.raises(kvq.KvqError, match="unsupported"):
        kvq.kvq_sparse_decode_attn_noalloc(cache, q, sel, cnt, 1, 0.1, out, None)



@pytest.mark.parametrize("B, ok", [(2815, True), (3000, False)])
def test_segment_limit_boundary(B, ok):
    """The attention's shared memory grows by 6 bytes per (sequence, kv head) segment beside
    the 16-bit-only kernel's 24 KB-per-warp rings: 5630 segments launch (every one empty:
    zero outputs, -inf lse), 6000 would exceed a CTA's 227 KB and are refused on the host
    with "unsupported" by both entry points instead of failing the launch."""
    from sparse_mixed_precision_kvq_b200 import kvq
    Hq, Hkv, D = 4, 2, 128
    cache = kvq.PagedCache(B, Hq, Hkv, D, 1, "bf16", [B, 0, 0, 0, 0])
    q = torch.zeros((B, Hq, D), dtype=torch.bfloat16, device="cuda")
    sel = torch.zeros((B, Hkv, 1), dtype=torch.int32, device="cuda")
    cnt = torch.zeros((B, Hkv), dtype=torch.int32, device="cuda")
    out = torch.full_like(q, 7.0)
    lse = torch.zeros((B, Hq), dtype=torch.float32, device="cuda")
    if ok:
        ws = torch.zeros(kvq.kvq_workspace_size(cache, 1) // 4 + 4, dtype=torch.float32, device="cuda")
        kvq.kvq_workspace_init(ws)
        kvq.kvq_sparse_decode_attn(cache, q, sel, cnt, 1, 0.1, out, lse, ws)
        torch.cuda.synchronize()
        assert not out.float().abs().sum().item() and bool(torch.isneginf(lse).all())
        out.fill_(7.0)
        kvq.kvq_sparse_decode_attn_noalloc(cache, q, sel, cnt, 1, 0.1, out, lse)
        torch.cuda.synchronize()
        assert not out.float().abs().sum().item()
    else:
        ws = torch.zeros(1 << 14, dtype=torch.float32, device="cuda")
        with pytest.raises(kvq.KvqError, match="unsupported"):
            kvq.kvq_sparse_decode_attn(cache, q, sel, cnt, 1, 0.1, out, lse, ws)
        with pytest.raises(kvq.KvqError, match="unsupported"):
            kvq.kvq_sparse_decode_attn_noalloc(cache, q, sel, cnt, 1, 0.1, out, lse)
