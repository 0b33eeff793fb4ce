"""Python binding of libkvq (ctypes): the C ABI of ``include/kvq.h`` with the same names.

Every function here only marshals arguments (``torch.Tensor.data_ptr()``, the current
CUDA stream) and raises on a non-OK status; all work runs in the CUDA kernels of
``libkvq.so``.  There is no CPU fallback: importing this module fails when the library
has not been built, and calls fail when no CUDA device is present.

``PagedCache`` allocates the cache's device tensors with PyTorch (plumbing only) and
fills a ``kvq_cache`` struct that points at them.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_char_p, c_float, c_int32, c_int64, c_size_t, c_void_p

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "lib", "libkvq.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"libkvq.so not found at {LIB_PATH}: build it with "
        "`python -m sparse_mixed_precision_kvq_b200.build` (there is no CPU fallback)")
_lib = ctypes.CDLL(LIB_PATH)

TIER_16, TIER_I8, TIER_I4, TIER_I2, TIER_I1, TIER_F8 = 0, 1, 2, 3, 4, 5
DT_F16, DT_BF16 = 0, 1
STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported", 3: "workspace too small", 4: "CUDA error"}

DERR_BAD_PAGE, DERR_FP16_RANGE, DERR_NAN_SCORE, DERR_KMAX = 0x1, 0x2, 0x4, 0x8
DERR_NONFINITE, DERR_TIMEOUT, DERR_BAD_POS = 0x10, 0x20, 0x40
WS_WAIT_LIMIT_WORD = 16383  # workspace head word: bounded-wait limit in microseconds (0: 2 s)

EXPORTS = ["kvq_chunk_bytes", "kvq_status_string", "kvq_append", "kvq_build_pages", "kvq_page_scores",
           "kvq_select_topk", "kvq_workspace_size", "kvq_sparse_decode_attn", "kvq_dequant_page",
           "kvq_sparse_decode_attn_noalloc", "kvq_noalloc_scratch_bytes", "kvq_workspace_init",
           "kvq_step_workspace_size", "kvq_decode_step", "kvq_score_select", "kvq_append_scores",
           "kvq_requantize_pages", "kvq_quad_build", "kvq_quad_append", "kvq_quad_page_scores",
           "kvq_quad_append_scores", "kvq_set_grid_override"]


class KvqCache(ctypes.Structure):
    _fields_ = [("B", c_int32), ("Hq", c_int32), ("Hkv", c_int32), ("D", c_int32),
                ("page_size", c_int32), ("max_pages", c_int32), ("dtype", c_int32), ("host_tiers", c_int32),
                ("block_table", c_void_p), ("seq_len", c_void_p), ("pool", c_void_p * 6),
                ("pool_slots", c_int64 * 6), ("summary", c_void_p), ("open_ksum", c_void_p),
                ("err_word", c_void_p), ("vpool", c_void_p * 6), ("host_vtiers", c_int32), ("reserved0", c_int32)]


class SelectParams(ctypes.Structure):
    _fields_ = [("k_abs", c_int32), ("k_frac_bp", c_int32), ("n_sink", c_int32), ("n_recent", c_int32),
                ("coverage_ppm", c_int32), ("sm_scale", c_float)]


class KvqQuad(ctypes.Structure):
    _fields_ = [("rank", c_int32), ("reserved", c_int32), ("basis", c_void_p), ("lambda_", c_void_p),
                ("open_sums", c_void_p)]


_P = POINTER(KvqCache)
_PQ = POINTER(KvqQuad)
_lib.kvq_chunk_bytes.argtypes, _lib.kvq_chunk_bytes.restype = [c_int32, c_int32], c_size_t
_lib.kvq_status_string.argtypes, _lib.kvq_status_string.restype = [c_int32], c_char_p
_lib.kvq_append.argtypes = [_P, c_void_p, c_void_p, c_void_p, c_void_p]
_lib.kvq_build_pages.argtypes = [_P, c_void_p, c_void_p, c_void_p, c_int64, c_void_p]
_lib.kvq_page_scores.argtypes = [_P, c_void_p, c_void_p, c_void_p]
_lib.kvq_select_topk.argtypes = [_P, c_void_p, POINTER(SelectParams), c_void_p, c_void_p, c_int32, c_void_p]
_lib.kvq_workspace_size.argtypes = [_P, c_int32, POINTER(c_size_t)]
_lib.kvq_sparse_decode_attn.argtypes = [_P, c_void_p, c_void_p, c_void_p, c_int32, c_float, c_void_p,
                                        c_void_p, c_void_p, c_size_t, c_void_p]
_lib.kvq_dequant_page.argtypes = [_P, c_int32, c_int32, c_void_p, c_void_p]
_lib.kvq_sparse_decode_attn_noalloc.argtypes = [_P, c_void_p, c_void_p, c_void_p, c_int32, c_float, c_void_p,
                                                c_void_p, c_void_p]
_lib.kvq_noalloc_scratch_bytes.argtypes, _lib.kvq_noalloc_scratch_bytes.restype = [], c_size_t
_lib.kvq_workspace_init.argtypes = [c_void_p, c_size_t, c_void_p]
_lib.kvq_step_workspace_size.argtypes = [_P, c_int32, POINTER(c_size_t)]
_lib.kvq_decode_step.argtypes = [_P, c_void_p, c_void_p, c_void_p, c_void_p, POINTER(SelectParams), c_void_p,
                                 c_void_p, c_void_p, c_int32, c_float, c_void_p, c_void_p, c_void_p, c_size_t,
                                 c_void_p]
_lib.kvq_score_select.argtypes = [_P, c_void_p, c_void_p, c_void_p, c_void_p, POINTER(SelectParams), c_void_p,
                                  c_void_p, c_void_p, c_int32, c_void_p, c_size_t, c_void_p]
_lib.kvq_append_scores.argtypes = [_P, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p]
_lib.kvq_requantize_pages.argtypes = [_P, c_void_p, c_int32, c_void_p]
_lib.kvq_set_grid_override.argtypes = [c_int32]
_lib.kvq_quad_build.argtypes = [_P, _PQ, c_void_p, c_void_p, c_int64, c_void_p]
_lib.kvq_quad_append.argtypes = [_P, _PQ, c_void_p, c_void_p, c_void_p]
_lib.kvq_quad_page_scores.argtypes = [_P, _PQ, c_void_p, c_float, c_void_p, c_void_p]
_lib.kvq_quad_append_scores.argtypes = [_P, _PQ, c_void_p, c_void_p, c_void_p, c_void_p, c_float, c_void_p, c_void_p]
for _f in EXPORTS[2:9] + ["kvq_sparse_decode_attn_noalloc", "kvq_workspace_init", "kvq_step_workspace_size",
                          "kvq_decode_step", "kvq_score_select", "kvq_append_scores", "kvq_requantize_pages",
                          "kvq_quad_build", "kvq_quad_append", "kvq_quad_page_scores", "kvq_quad_append_scores",
                          "kvq_set_grid_override"]:
    getattr(_lib, _f).restype = c_int32


class KvqError(RuntimeError):
    pass


def _check(st: int, what: str):
    if st != 0:
        raise KvqError(f"{what}: {_lib.kvq_status_string(st).decode()} ({st})")


def _ptr(t) -> int:
    return 0 if t is None else int(t.data_ptr())


def _stream(stream) -> int:
    if stream is None:
        import torch
        return int(torch.cuda.current_stream().cuda_stream)
    return int(getattr(stream, "cuda_stream", stream))


def kvq_chunk_bytes(tier: int, D: int) -> int:
    return int(_lib.kvq_chunk_bytes(tier, D))


def kvq_status_string(st: int) -> str:
    return _lib.kvq_status_string(st).decode()


def kvq_append(cache, pos, k_new, v_new, stream=None):
    _check(_lib.kvq_append(cache.ref(), _ptr(pos), _ptr(k_new), _ptr(v_new), _stream(stream)), "kvq_append")


def kvq_build_pages(cache, k_src, v_src, cu_seqlens, stream=None):
    _check(_lib.kvq_build_pages(cache.ref(), _ptr(k_src), _ptr(v_src), _ptr(cu_seqlens), int(k_src.shape[1]),
                                _stream(stream)), "kvq_build_pages")


def kvq_page_scores(cache, q, scores, stream=None):
    _check(_lib.kvq_page_scores(cache.ref(), _ptr(q), _ptr(scores), _stream(stream)), "kvq_page_scores")


def kvq_select_topk(cache, scores, params: SelectParams, sel, cnt, kmax: int, stream=None):
    _check(_lib.kvq_select_topk(cache.ref(), _ptr(scores), ctypes.byref(params), _ptr(sel), _ptr(cnt), kmax,
                                _stream(stream)), "kvq_select_topk")


def kvq_workspace_size(cache, kmax: int) -> int:
    n = c_size_t(0)
    _check(_lib.kvq_workspace_size(cache.ref(), kmax, ctypes.byref(n)), "kvq_workspace_size")
    return int(n.value)


def kvq_set_grid_override(ctas: int):
    """Attention / fused-step grid of ``ctas`` CTAs for every later call (0: one per SM)."""
    _check(_lib.kvq_set_grid_override(int(ctas)), "kvq_set_grid_override")


def kvq_workspace_init(workspace, stream=None):
    _check(_lib.kvq_workspace_init(_ptr(workspace), int(workspace.numel() * workspace.element_size()),
                                   _stream(stream)), "kvq_workspace_init")


def kvq_sparse_decode_attn(cache, q, sel, cnt, kmax: int, sm_scale: float, out, lse, workspace, stream=None):
    _check(_lib.kvq_sparse_decode_attn(cache.ref(), _ptr(q), _ptr(sel), _ptr(cnt), kmax, sm_scale, _ptr(out),
                                       _ptr(lse), _ptr(workspace), int(workspace.numel() * workspace.element_size()),
                                       _stream(stream)), "kvq_sparse_decode_attn")


def kvq_step_workspace_size(cache, kmax: int) -> int:
    n = c_size_t(0)
    _check(_lib.kvq_step_workspace_size(cache.ref(), kmax, ctypes.byref(n)), "kvq_step_workspace_size")
    return int(n.value)


def kvq_decode_step(cache, pos, k_new, v_new, q, params: SelectParams, scores, sel, cnt, kmax: int,
                    sm_scale: float, out, lse, workspace, stream=None):
    """The whole decode step (append if ``pos`` is not None, scores, selection, attention) in one launch."""
    _check(_lib.kvq_decode_step(cache.ref(), _ptr(pos), _ptr(k_new), _ptr(v_new), _ptr(q), ctypes.byref(params),
                                _ptr(scores), _ptr(sel), _ptr(cnt), kmax, sm_scale, _ptr(out), _ptr(lse),
                                _ptr(workspace), int(workspace.numel() * workspace.element_size()),
                                _stream(stream)), "kvq_decode_step")


def kvq_append_scores(cache, pos, k_new, v_new, q, scores, stream=None):
    """kvq_append + kvq_page_scores as one call: two chained kernels, the score sweep beside the append."""
    _check(_lib.kvq_append_scores(cache.ref(), _ptr(pos), _ptr(k_new), _ptr(v_new), _ptr(q), _ptr(scores),
                                  _stream(stream)), "kvq_append_scores")


def kvq_score_select(cache, pos, k_new, v_new, q, params: SelectParams, scores, sel, cnt, kmax: int, workspace,
                     stream=None):
    """kvq_append (if ``pos`` is not None) + kvq_page_scores + kvq_select_topk in one launch."""
    _check(_lib.kvq_score_select(cache.ref(), _ptr(pos), _ptr(k_new), _ptr(v_new), _ptr(q), ctypes.byref(params),
                                 _ptr(scores), _ptr(sel), _ptr(cnt), kmax, _ptr(workspace),
                                 int(workspace.numel() * workspace.element_size()), _stream(stream)),
           "kvq_score_select")


def kvq_sparse_decode_attn_noalloc(cache, q, sel, cnt, kmax: int, sm_scale: float, out, lse, stream=None):
    """kvq_sparse_decode_attn with the library's static device scratch: allocates nothing."""
    _check(_lib.kvq_sparse_decode_attn_noalloc(cache.ref(), _ptr(q), _ptr(sel), _ptr(cnt), kmax, sm_scale,
                                               _ptr(out), _ptr(lse), _stream(stream)),
           "kvq_sparse_decode_attn_noalloc")


def kvq_noalloc_scratch_bytes() -> int:
    return int(_lib.kvq_noalloc_scratch_bytes())


def kvq_dequant_page(cache, b: int, page: int, out, stream=None):
    _check(_lib.kvq_dequant_page(cache.ref(), b, page, _ptr(out), _stream(stream)), "kvq_dequant_page")


def kvq_requantize_pages(cache, items, stream=None):
    """``items``: device int32 tensor [n, 3] of (b, page, new block-table entry)."""
    n = 0 if items is None else int(items.shape[0])
    _check(_lib.kvq_requantize_pages(cache.ref(), _ptr(items) if n else None, n, _stream(stream)),
           "kvq_requantize_pages")


def kvq_quad_build(cache, quad, k_src, cu_seqlens, stream=None):
    _check(_lib.kvq_quad_build(cache.ref(), quad.ref(), _ptr(k_src), _ptr(cu_seqlens), int(k_src.shape[1]),
                               _stream(stream)), "kvq_quad_build")


def kvq_quad_append(cache, quad, pos, k_new, stream=None):
    _check(_lib.kvq_quad_append(cache.ref(), quad.ref(), _ptr(pos), _ptr(k_new), _stream(stream)), "kvq_quad_append")


def kvq_quad_page_scores(cache, quad, q, sm_scale: float, scores, stream=None):
    _check(_lib.kvq_quad_page_scores(cache.ref(), quad.ref(), _ptr(q), float(sm_scale), _ptr(scores),
                                     _stream(stream)), "kvq_quad_page_scores")


def kvq_quad_append_scores(cache, quad, pos, k_new, v_new, q, sm_scale: float, scores, stream=None):
    _check(_lib.kvq_quad_append_scores(cache.ref(), quad.ref(), _ptr(pos), _ptr(k_new), _ptr(v_new), _ptr(q),
                                       float(sm_scale), _ptr(scores), _stream(stream)), "kvq_quad_append_scores")


# ------------------------------------------------------------------------- allocation
def encode_block_table(tier_tbl: np.ndarray, slot_tbl: np.ndarray) -> np.ndarray:
    """(tier << 29) | slot as int32; unused entries (tier < 0) get an invalid tier (7)."""
    t = np.where(tier_tbl < 0, 7, tier_tbl).astype(np.int64)
    s = np.where(slot_tbl < 0, 0, slot_tbl).astype(np.int64)
    return ((t << 29) | s).astype(np.uint32).view(np.int32)


class PagedCache:
    """Device tensors of a paged cache plus the ``kvq_cache`` struct pointing at them.

    ``host_tiers`` (bit t): pool t -- K and V chunks -- in pinned host memory.
    ``v_tiers`` (bit t): tier t keeps its V chunks in a pool of their own; ``host_v_tiers``
    (bit t, implies the v_tiers bit): that V pool in pinned host memory while the K pool
    stays on the device (the "mem-v" variant of a host-DRAM value tier)."""

    def __init__(self, B, Hq, Hkv, D, max_pages, dtype: str, pool_slots, device="cuda", host_tiers: int = 0,
                 v_tiers: int = 0, host_v_tiers: int = 0):
        import torch
        self.B, self.Hq, self.Hkv, self.D, self.max_pages = B, Hq, Hkv, D, max_pages
        self.dtype = dtype
        self.tdtype = torch.bfloat16 if dtype == "bf16" else torch.float16
        dev = torch.device(device)
        self.device = dev
        self.block_table = torch.full((B, max_pages), -1, dtype=torch.int32, device=dev)
        self.seq_len = torch.zeros(B, dtype=torch.int32, device=dev)
        self.pool_slots = [int(x) for x in pool_slots] + [0] * (6 - len(pool_slots))
        self.pools, self.vpools = [], []
        self.host_tiers = int(host_tiers)
        self.host_v_tiers = int(host_v_tiers)
        self.v_tiers = int(v_tiers) | self.host_v_tiers

        def alloc(nbytes, host):  # pinned host memory is read by the device in place
            if host:
                return torch.zeros(nbytes, dtype=torch.uint8, pin_memory=True)
            return torch.zeros(nbytes, dtype=torch.uint8, device=dev)

        for tier, n in enumerate(self.pool_slots):
            if n <= 0:
                self.pools.append(None)
                self.vpools.append(None)
                continue
            cb = n * Hkv * kvq_chunk_bytes(tier, D)
            if (self.v_tiers >> tier) & 1:
                self.pools.append(alloc(cb, (self.host_tiers >> tier) & 1))
                self.vpools.append(alloc(cb, (self.host_v_tiers >> tier) & 1))
            else:
                self.pools.append(alloc(2 * cb, (self.host_tiers >> tier) & 1))
                self.vpools.append(None)
        self.summary = torch.zeros((B, Hkv, max_pages, D), dtype=torch.float16, device=dev)
        self.open_ksum = torch.zeros((B, Hkv, D), dtype=torch.float64, device=dev)
        self.err = torch.zeros(1, dtype=torch.int32, device=dev)
        self.quad = None  # a QuadState when the quad page score is maintained
        self._s = KvqCache()
        s = self._s
        s.B, s.Hq, s.Hkv, s.D, s.page_size, s.max_pages = B, Hq, Hkv, D, 16, max_pages
        s.dtype = DT_BF16 if dtype == "bf16" else DT_F16
        s.host_tiers = self.host_tiers
        s.block_table, s.seq_len = _ptr(self.block_table), _ptr(self.seq_len)
        for i in range(6):
            s.pool[i] = _ptr(self.pools[i]) if self.pools[i] is not None else None
            s.vpool[i] = _ptr(self.vpools[i]) if self.vpools[i] is not None else None
            s.pool_slots[i] = self.pool_slots[i]
        s.host_vtiers = sum(1 << i for i in range(6) if (self.host_v_tiers >> i) & 1 and self.vpools[i] is not None)
        s.summary, s.open_ksum, s.err_word = _ptr(self.summary), _ptr(self.open_ksum), _ptr(self.err)

    def ref(self):
        return ctypes.byref(self._s)

    def err_bits(self) -> int:
        return int(self.err.item()) & 0xFFFFFFFF

    def pool_bytes(self) -> int:
        return sum(p.numel() for p in self.pools + self.vpools if p is not None)

    def chunk_view(self, b: int, page: int, g: int, kind: int):
        """Bytes (uint8 tensor view) of one chunk of logical page ``page`` (host-side lookup)."""
        e = int(self.block_table[b, page].item()) & 0xFFFFFFFF
        tier, slot = e >> 29, e & 0x1FFFFFFF
        cb = kvq_chunk_bytes(tier, self.D)
        if self.vpools[tier] is not None:
            o = (slot * self.Hkv + g) * cb
            return tier, (self.vpools[tier] if kind else self.pools[tier])[o:o + cb]
        o = ((slot * self.Hkv + g) * 2 + kind) * cb
        return tier, self.pools[tier][o:o + cb]


class QuadState:
    """Device buffers of the quad page-score state of a cache and its ``kvq_quad`` struct.

    ``basis``: fp32 ``[Hkv, rank, D]`` (host array or tensor), copied to the device."""

    def __init__(self, cache: PagedCache, basis):
        import torch
        b = torch.as_tensor(np.asarray(basis, dtype=np.float32)).to(cache.device).contiguous()
        self.rank = int(b.shape[1])
        self.basis = b
        self.lam = torch.zeros((cache.B, cache.Hkv, cache.max_pages, self.rank), dtype=torch.float16,
                               device=cache.device)
        self.open = torch.zeros((cache.B, cache.Hkv, 2, self.rank), dtype=torch.float64, device=cache.device)
        self._s = KvqQuad()
        self._s.rank = self.rank
        self._s.basis, self._s.lambda_, self._s.open_sums = _ptr(self.basis), _ptr(self.lam), _ptr(self.open)

    def ref(self):
        return ctypes.byref(self._s)


def cache_from_workload(w, device="cuda", threads: int = 8, spare=None, quad_basis=None, host_tiers: int = 0,
                        v_tiers: int = 0, host_v_tiers: int = 0):
    """Allocate a cache for workload ``w`` and store its prefilled context with kvq_build_pages.

    After the call ``seq_len`` holds the prefilled lengths (before the step's append).
    ``spare`` (optional, per tier) adds free slots after the used ones of each pool.
    ``quad_basis`` (optional, fp32 ``[Hkv, rank, D]``) also builds the quad page-score state
    (``cache.quad``) from the same keys with kvq_quad_build.  ``host_tiers`` (bit t) puts
    pool t in pinned host memory that the kernels read in place; ``v_tiers`` /
    ``host_v_tiers`` (bit t) give tier t a separate V pool, on the device or in pinned
    host memory.
    """
    import torch
    from concurrent.futures import ThreadPoolExecutor
    tier_tbl, slot_tbl, counts = w.slot_map()
    if spare is not None:
        counts = [int(c) + int(x) for c, x in zip(counts, spare)]
    cache = PagedCache(w.B, w.Hq, w.Hkv, w.D, w.max_pages, w.dtype, counts, device, host_tiers=host_tiers,
                       v_tiers=v_tiers, host_v_tiers=host_v_tiers)
    cache.block_table.copy_(torch.from_numpy(encode_block_table(tier_tbl, slot_tbl)))
    lens = np.asarray(w.lens, dtype=np.int64)
    cache.seq_len.copy_(torch.from_numpy(lens.astype(np.int32)))
    cu = np.zeros(w.B + 1, dtype=np.int64)
    cu[1:] = np.cumsum(lens)
    total = int(cu[-1])
    ksrc = torch.empty((w.Hkv, max(total, 1), w.D), dtype=torch.int16, device=device)
    vsrc = torch.empty_like(ksrc)
    pairs = [(b, g) for b in range(w.B) for g in range(w.Hkv) if lens[b] > 0]

    def draw(bg):
        b, g = bg
        return bg, w.keys_bits(b, g), w.values_bits(b, g)

    with ThreadPoolExecutor(max_workers=threads) as ex:
        for (b, g), kb, vb in ex.map(draw, pairs):
            s, e = int(cu[b]), int(cu[b + 1])
            ksrc[g, s:e].copy_(torch.from_numpy(kb.view(np.int16)))
            vsrc[g, s:e].copy_(torch.from_numpy(vb.view(np.int16)))
    cu_t = torch.from_numpy(cu).to(device)
    kvq_build_pages(cache, ksrc, vsrc, cu_t)
    cache.quad = None
    if quad_basis is not None:
        cache.quad = QuadState(cache, quad_basis)
        kvq_quad_build(cache, cache.quad, ksrc, cu_t)
    torch.cuda.synchronize(device)
    del ksrc, vsrc
    return cache


def select_params(w, coverage=None) -> SelectParams:
    """The workload's budget selection, or coverage selection at ``coverage`` (0..1)."""
    if coverage is None:
        return SelectParams(w.k_abs, w.k_frac_bp, w.n_sink, w.n_recent)
    return SelectParams(-1, 0, w.n_sink, w.n_recent, int(round(coverage * 1e6)), w.sm_scale)


def packed_buffer(specs, device):
    """One device buffer holding tensors of the given (shape, dtype) at 256-byte aligned
    offsets, so that one copy moves them all: returns the uint8 buffer and the typed views."""
    import torch
    sizes = [int(np.prod(shape)) * torch.empty((), dtype=dt).element_size() for shape, dt in specs]
    offs, n = [], 0
    for nb in sizes:
        n = (n + 255) // 256 * 256
        offs.append(n)
        n += nb
    buf = torch.empty(max(n, 1), dtype=torch.uint8, device=device)
    return buf, [buf[o:o + nb].view(dt).view(shape) for (shape, dt), o, nb in zip(specs, offs, sizes)]


class DecodeStep:
    """The buffers and calls of one decode step of workload ``w`` on ``cache``.

    The step's inputs (q, and k_new, v_new when it appends) are views into one device
    buffer ``io_in`` and its outputs (out, lse) into ``io_out``, so that a caller moves
    each direction with a single copy.

    ``run()`` enqueues: kvq_append (if the workload appends) -> kvq_page_scores ->
    kvq_select_topk -> kvq_sparse_decode_attn, all on the current stream.  With
    ``quad=True`` (the cache built with a quad basis) the page score is the quad score:
    kvq_append -> kvq_quad_append -> kvq_quad_page_scores -> select -> attention.
    """

    def __init__(self, w, cache: PagedCache, device="cuda", coverage=None, quad=False):
        import torch
        self.w, self.cache = w, cache
        dt = cache.tdtype
        bits = w.query_bits()
        ins = [(bits.shape, dt)]
        if w.append:
            kn, vn = w.new_kv_bits()
            ins += [(kn.shape, dt), (vn.shape, dt)]
        self.io_in, views = packed_buffer(ins, device)
        self.q = views[0]
        self.q.copy_(torch.from_numpy(bits.view(np.int16)).view(dt))
        if w.append:
            self.k_new, self.v_new = views[1], views[2]
            self.k_new.copy_(torch.from_numpy(kn.view(np.int16)).view(dt))
            self.v_new.copy_(torch.from_numpy(vn.view(np.int16)).view(dt))
            self.pos = torch.from_numpy(np.asarray(w.lens, dtype=np.int32)).to(device)
        self.kmax = w.kmax() if coverage is None else w.max_pages
        self.quad = cache.quad if quad else None
        if quad:
            assert self.quad is not None, "the cache has no quad state (cache_from_workload(quad_basis=...))"
        self.params = select_params(w, coverage)
        if quad and coverage is not None:
            self.params.sm_scale = 1.0  # the quad score already carries the softmax scale
        self.scores = torch.empty((w.B, w.Hkv, w.max_pages), dtype=torch.float32, device=device)
        self.sel = torch.zeros((w.B, w.Hkv, self.kmax), dtype=torch.int32, device=device)
        self.cnt = torch.zeros((w.B, w.Hkv), dtype=torch.int32, device=device)
        self.io_out, (self.out, self.lse) = packed_buffer([((w.B, w.Hq, w.D), dt), ((w.B, w.Hq), torch.float32)],
                                                          device)
        nws = max(kvq_workspace_size(cache, self.kmax), kvq_step_workspace_size(cache, self.kmax))
        self.ws = torch.empty((nws + 15) // 16 * 4, dtype=torch.float32, device=device)
        kvq_workspace_init(self.ws)
        cache.seq_len.copy_(torch.from_numpy(w.final_lens().astype(np.int32)))

    def append(self):
        if self.w.append:
            kvq_append(self.cache, self.pos, self.k_new, self.v_new)
            if self.quad is not None:
                kvq_quad_append(self.cache, self.quad, self.pos, self.k_new)

    def scores_(self):
        if self.quad is not None:
            kvq_quad_page_scores(self.cache, self.quad, self.q, self.w.sm_scale, self.scores)
        else:
            kvq_page_scores(self.cache, self.q, self.scores)

    def select(self):
        kvq_select_topk(self.cache, self.scores, self.params, self.sel, self.cnt, self.kmax)

    def attend(self):
        kvq_sparse_decode_attn(self.cache, self.q, self.sel, self.cnt, self.kmax, self.w.sm_scale, self.out,
                               self.lse, self.ws)

    def run(self):
        self.append()
        self.scores_()
        self.select()
        self.attend()

    def score_select(self):
        assert self.quad is None, "the fused launches score pages with the mean-key score"
        kvq_score_select(self.cache, self.pos if self.w.append else None, self.k_new if self.w.append else None,
                         self.v_new if self.w.append else None, self.q, self.params, self.scores, self.sel, self.cnt,
                         self.kmax, self.ws)

    def append_scores(self):
        if self.w.append and self.quad is not None:
            kvq_quad_append_scores(self.cache, self.quad, self.pos, self.k_new, self.v_new, self.q, self.w.sm_scale,
                                   self.scores)
        elif self.w.append:
            kvq_append_scores(self.cache, self.pos, self.k_new, self.v_new, self.q, self.scores)
        else:
            self.scores_()

    def run_three(self):
        """The same step as ``run()`` in three calls: kvq_append_scores, select, attention."""
        self.append_scores()
        self.select()
        self.attend()

    def run_two(self):
        """The same step as ``run()`` in two launches: kvq_score_select, kvq_sparse_decode_attn."""
        self.score_select()
        self.attend()

    def run_fused(self):
        """The same step as ``run()`` in one kvq_decode_step launch."""
        assert self.quad is None, "the fused launches score pages with the mean-key score"
        kvq_decode_step(self.cache, self.pos if self.w.append else None, self.k_new if self.w.append else None,
                        self.v_new if self.w.append else None, self.q, self.params, self.scores, self.sel, self.cnt,
                        self.kmax, self.w.sm_scale, self.out, self.lse, self.ws)
