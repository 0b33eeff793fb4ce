/*
 * kvq.h -- C ABI of libkvq: sparse mixed-precision paged decode attention on B200.
 *
 * One decode step of one attention layer over a paged KV cache:
 *
 *   kvq_append             write the step's new K/V token into its page (quantised to the
 *                          page's tier) and refresh the page's mean-key summary;
 *   kvq_page_scores        score every page from its summary;
 *   kvq_select_topk        pick the top pages plus forced sink/recent pages;
 *   kvq_sparse_decode_attn attend only the selected pages (split-K + log-sum-exp combine),
 *                          unpacking and dequantising cold pages in registers;
 *   kvq_append_scores      the first two as one call (two chained kernels; same results);
 *   kvq_score_select       the first three in one launch (same results);
 *   kvq_decode_step        the four above in one persistent launch (same results);
 *   kvq_quad_*             the quad (Gaussian-MGF) page score and its per-page state;
 *   kvq_requantize_pages   tier demotion: re-encode pages into a colder tier.
 *
 * Sources: AMASS "decode-time sparse KV-cache attention for vLLM" (amass-kv 0.1.1),
 * section "What is in the box" (per-page summary -> page score -> small selected working
 * set -> sparse paged kernel reading only those pages) and "Quickstart" (budget: fixed
 * selected fraction); ARGUS "Virtual Memory for Transformers" (argus_cache 0.1.7.1),
 * sections "The One-Minute Explanation" / "Visual Architecture" (fp16 hot pages; the
 * cascade FP8, INT8, INT4 2-way, INT2 4-way, 1-bit 8-way packed for cold pages;
 * reconstruction only when a query touches a page), "Why It Works" (dequantise, then
 * attend) and "Quickstart" (sink_tokens); AMASS Stage B (a pinned, device-mapped
 * host-DRAM pool: kvq_cache.host_tiers).
 *
 * Conventions (every call):
 *  - Pointers named "device" are device memory owned by the caller; the library never
 *    allocates, frees or synchronises.  All work is enqueued on the given stream; a call
 *    returns after enqueueing.  Host structs (kvq_cache, kvq_select_params) are read
 *    during the call only.
 *  - Return: KVQ_OK, or an argument error found on the host before anything is enqueued
 *    (KVQ_ERR_INVALID_ARG / KVQ_ERR_UNSUPPORTED / KVQ_ERR_WORKSPACE), or KVQ_ERR_CUDA when
 *    the launch itself failed (cudaGetLastError).
 *  - Data errors found on the device (bad block-table entry, page or position out of
 *    range, non-finite input, fp16 metadata overflow, NaN score, too many selected pages,
 *    a pipeline wait that ran out) set bits in *err_word (sticky; the caller clears it).
 *    The offending unit is skipped or clamped.  Kernels never trap.
 *  - Calls on different streams that write the same cache memory must not overlap.
 *  - Kernels are launched with programmatic dependent launch: a call's kernel may start
 *    while the previous kernel on the stream finishes, and reads some inputs of the call
 *    (seq_len, the block table, pos, q) before it waits for that kernel.  A kernel of the
 *    caller that lets its dependents launch early (griddepcontrol.launch_dependents) must
 *    therefore have written those inputs before it does; kernels that do not (the
 *    default) finish before the next call's kernels start.
 *
 * Cache layout (all device memory, T = 16 tokens per page, D in {64, 128}):
 *  - block_table [B][max_pages] int32: entry = (tier << 29) | slot, tier in kvq_tier.
 *    A logical page's tier is shared by all kv heads.
 *  - pool[tier]: pool_slots[tier] physical slots (device memory, or pinned host memory
 *    mapped into the device address space when bit tier of host_tiers is set); slot s
 *    holds, for kv head g and kind k (0 = K, 1 = V), one chunk of
 *    kvq_chunk_bytes(tier, D) bytes at byte offset
 *    ((s * Hkv + g) * 2 + k) * kvq_chunk_bytes(tier, D).  Base must be 16-byte aligned.
 *    Chunk = codes then meta.  Codes order: each element (t, d) belongs to lane
 *    lam, register pair R = 4*(d/16) + r and half h, with c = d % 16:
 *      K:  lam = 4*(t%8) + (c%8)/2,  r = 2*(c/8) + t/8,  h = c%2
 *      V:  lam = 4*(c%8) + (t%8)/2,  r = 2*(t/8) + c/8,  h = t%2
 *    16-bit tier: half h of uint32 word (d/16*32 + lam)*4 + r.
 *    b-bit tiers: lane word w = R/(16/b), slot j = R%(16/b); low code at bits b*j,
 *    high code at bits 16 + b*j; NW = D*b/64 words per lane, PW = min(4, NW); lane word
 *    w is uint32 ((w/PW)*32 + lam)*PW + w%PW of the codes area.  1-bit code 1 = +.
 *    FP8 codes use the 8-bit layout (e4m3 bytes).
 *    Meta: b = 8/4/2: uint32 [T][D/32] = scale_fp16 | zero_fp16 << 16;
 *          1-bit:     uint16 [T][D/32] = magnitude fp16;
 *          fp8:       uint16 [T][D/32] = scale fp16.  Empty slots are zero.
 *    Value read back: 16-bit: as stored; b-bit: fp32(c * scale + zero) (one rounding);
 *    1-bit: +m or -m; fp8: e4m3(c) * scale (exact in fp32).
 *  - summary [B][Hkv][max_pages][D] fp16: fp16(mean of the page's keys as they arrived).
 *  - open_ksum [B][Hkv][D] double: running fp64 sum of the keys of the page that holds
 *    position seq_len-1 when that page is not full.
 *  - seq_len [B] int32: tokens in each sequence (read by scores/select/attention; the
 *    caller advances it after kvq_append).
 */
#ifndef KVQ_H_
#define KVQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* kvq_stream_t; /* identical to cudaStream_t; NULL = legacy stream */

typedef enum {
  KVQ_OK = 0,
  KVQ_ERR_INVALID_ARG = 1,
  KVQ_ERR_UNSUPPORTED = 2,
  KVQ_ERR_WORKSPACE = 3,
  KVQ_ERR_CUDA = 4
} kvq_status;

typedef enum { KVQ_DT_F16 = 0, KVQ_DT_BF16 = 1 } kvq_dtype;

typedef enum {
  KVQ_TIER_16 = 0, /* cache dtype, unchanged */
  KVQ_TIER_I8 = 1, /* 8-bit codes, per-32-channel fp16 scale/zero */
  KVQ_TIER_I4 = 2, /* 4-bit codes, two per byte */
  KVQ_TIER_I2 = 3, /* 2-bit codes, four per byte */
  KVQ_TIER_I1 = 4, /* sign bits, eight per byte, per-32-channel fp16 magnitude */
  KVQ_TIER_F8 = 5  /* FP8 e4m3 codes, per-32-channel fp16 scale = fp16(amax/448),
                      code = e4m3(x/scale) round-half-even, saturating (ARGUS cascade FP16 -> FP8 -> INT8) */
} kvq_tier;

/* device error-word bits */
#define KVQ_DERR_BAD_PAGE 0x1u      /* block-table entry with bad tier/slot, or page out of range */
#define KVQ_DERR_FP16_RANGE 0x2u    /* fp16 scale/zero/magnitude/summary saturated at +-65504 */
#define KVQ_DERR_NAN_SCORE 0x4u     /* NaN page score (ranked lowest) */
#define KVQ_DERR_KMAX 0x8u          /* more selected pages than kmax (list truncated) */
#define KVQ_DERR_NONFINITE 0x10u    /* non-finite key/value quantised */
#define KVQ_DERR_TIMEOUT 0x20u      /* a bounded pipeline wait ran out (work skipped) */
#define KVQ_DERR_BAD_POS 0x40u      /* append position outside the block table */

typedef struct {
  int32_t B, Hq, Hkv, D;   /* batch, query heads, kv heads (Hq % Hkv == 0, Hq/Hkv <= 8), head dim */
  int32_t page_size;       /* must be 16 */
  int32_t max_pages;       /* block-table row length (logical pages per sequence) */
  int32_t dtype;           /* kvq_dtype of keys, values, queries and outputs */
  int32_t host_tiers;      /* bit t set: pool[t] is pinned host memory mapped into the device address
                              space (AMASS "What is in the box", Stage B: a host-DRAM pool read
                              by the device); the attention kernel reads those pages with per-thread
                              asynchronous loads instead of bulk copies; kvq_decode_step rejects it */
  int32_t* block_table;    /* device [B][max_pages] */
  int32_t* seq_len;        /* device [B] */
  void* pool[6];           /* device, per tier (NULL if unused) */
  int64_t pool_slots[6];   /* slots in each pool */
  uint16_t* summary;       /* device [B][Hkv][max_pages][D] fp16 bits, 16-byte aligned */
  double* open_ksum;       /* device [B][Hkv][D] */
  uint32_t* err_word;      /* device, 1 word */
  void* vpool[6];          /* optional, per tier: a separate pool of V chunks (NULL: V chunks sit
                              next to the K chunks in pool[t]).  When set, pool[t] holds the K
                              chunk of (slot, kv head g) at byte (slot*Hkv + g) * chunk and
                              vpool[t] its V chunk at the same offset; both have pool_slots[t]
                              slots.  16-byte aligned. */
  int32_t host_vtiers;     /* bit t set: vpool[t] is pinned host memory mapped into the device
                              address space (AMASS "What is in the box", Stage B, the "mem-v"
                              variant: values in host DRAM, keys resident on the device) */
  int32_t reserved0;       /* must be 0 */
} kvq_cache;

typedef struct {
  int32_t k_abs;      /* >= 0: select this many pages; < 0: use k_frac_bp */
  int32_t k_frac_bp;  /* fraction in basis points: k = ceil(P * k_frac_bp / 10000) per sequence */
  int32_t n_sink;     /* first n_sink pages always attended (in addition to k) */
  int32_t n_recent;   /* last n_recent pages always attended (in addition to k) */
  int32_t coverage_ppm; /* > 0: coverage selection instead of k (AMASS "Quickstart" coverage):
                           the fewest best pages whose estimated mass, with the forced pages',
                           reaches coverage_ppm / 1e6 of the total; mass of page p estimated
                           as n_p * exp(sm_scale * s_p), n_p its valid tokens; ties: lower page */
  float sm_scale;     /* softmax scale of the mass estimate (coverage only) */
} kvq_select_params;

/* Bytes of one chunk (one page, one kv head, K or V) of a tier; 0 for a bad tier/D. */
size_t kvq_chunk_bytes(int32_t tier, int32_t D);

/* Human-readable status. */
const char* kvq_status_string(kvq_status s);

/*
 * kvq_append -- write one new token per sequence into the cache.
 * (ARGUS "The One-Minute Explanation": new tokens are hot; cold tiers per "Visual
 *  Architecture".  AMASS "What is in the box": the per-page summary the score reads.)
 *  pos    device [B] int32: logical position written for each sequence (normally
 *         seq_len[b]); pos < 0 skips the sequence.  The page pos/16 must already have a
 *         block-table entry; when pos % 16 == 0 the page's chunks are cleared first.
 *  k_new, v_new  device [B][Hkv][D] in the cache dtype.
 *  Quantises the token into its page's tier (per 32-channel group: zero = fp16(min),
 *  scale = fp16((max-min)/(2^b-1)), code = clamp(rint((x-zero)/scale)); 1-bit: sign and
 *  fp16(mean|x|)), sets open_ksum = (pos%16 ? open_ksum : 0) + k (fp64) and
 *  summary[b][g][pos/16] = fp16(open_ksum / (pos%16 + 1)).  Does not change seq_len.
 *  A page written by append must not be shared with another sequence.
 */
kvq_status kvq_append(const kvq_cache* cache, const int32_t* pos, const void* k_new,
                      const void* v_new, kvq_stream_t stream);

/*
 * kvq_build_pages -- store a prefilled context (bulk form of kvq_append).
 *  k_src, v_src  device [Hkv][src_tokens][D] in the cache dtype; sequence b's token i is
 *                row cu_seqlens[b] + i.
 *  cu_seqlens    device [B+1] int64.
 *  Stores tokens [0, seq_len[b]) of every sequence into the pages named by the block
 *  table (same quantiser as kvq_append), writes every page's summary and the open page's
 *  open_ksum.  Token slots past seq_len are zero.
 */
kvq_status kvq_build_pages(const kvq_cache* cache, const void* k_src, const void* v_src,
                           const int64_t* cu_seqlens, int64_t src_tokens, kvq_stream_t stream);

/*
 * kvq_page_scores -- page score (AMASS "What is in the box": compact per-page score;
 * its "quad" form is not given, the mean-key form is used).
 *  q       device [B][Hq][D] in the cache dtype.
 *  scores  device [B][Hkv][max_pages] fp32 out:
 *          scores[b][g][p] = max over h in [g*G, g*G+G) of sum_d q[b][h][d] * summary[b][g][p][d]
 *          for p < ceil(seq_len[b]/16), and -inf for the remaining pages.
 */
kvq_status kvq_page_scores(const kvq_cache* cache, const void* q, float* scores,
                           kvq_stream_t stream);

/*
 * kvq_select_topk -- per (sequence, kv head) page selection (AMASS "Quickstart" budget;
 * ARGUS "Quickstart" sink_tokens).
 *  scores  device [B][Hkv][max_pages] fp32 (as written by kvq_page_scores).
 *  params  host: budget k and forced sink/recent page counts.
 *  sel     device [B][Hkv][kmax] int32 out: forced pages plus the k best other pages
 *          (score descending, lower page index first on ties, NaN lowest), ascending.
 *  cnt     device [B][Hkv] int32 out: entries written to sel (<= kmax).
 *  kmax    row length of sel; a longer selection is truncated and flagged.
 *  With params->coverage_ppm > 0 the k best are replaced by the coverage choice; the
 *  candidates of a sequence (pages minus forced ones) must number at most 8192 and
 *  cache->max_pages at most 41984 (else KVQ_ERR_UNSUPPORTED).  The running mass that
 *  decides the cut is summed in fixed point (2^-46 units, order-independent), so the
 *  choice is deterministic and is the exact-arithmetic one except where the covered mass
 *  lies within about 1e-10 of the total from the target; pages of zero mass (NaN or
 *  underflowed scores) are never chosen as candidates.
 */
kvq_status kvq_select_topk(const kvq_cache* cache, const float* scores,
                           const kvq_select_params* params, int32_t* sel, int32_t* cnt,
                           int32_t kmax, kvq_stream_t stream);

/* Workspace bytes kvq_sparse_decode_attn needs on the current device for this cache. */
kvq_status kvq_workspace_size(const kvq_cache* cache, int32_t kmax, size_t* bytes);

/*
 * kvq_workspace_init -- make a newly allocated workspace ready (zeroes its first 64 KiB,
 * the arrival counters of the split-K combine and of kvq_decode_step's work queue; a
 * workspace that is all zero is ready too).  Enqueued on stream.  Every
 * kvq_sparse_decode_attn and kvq_decode_step call leaves the counters zero again, so
 * this is needed once per workspace, not per call (and again after a call that flagged
 * KVQ_DERR_TIMEOUT).  One workspace may serve both calls.
 * Word KVQ_WS_WAIT_LIMIT_WORD (uint32) of that head is never a counter: it is the limit,
 * in microseconds, of every bounded wait of a kvq_sparse_decode_attn or kvq_decode_step
 * call on this workspace (a wait on a copy in flight, or on another CTA's result).  0 (as
 * kvq_workspace_init leaves it) means 2 s.  A wait that runs out sets KVQ_DERR_TIMEOUT,
 * skips the rest of the work and returns; the workspace is then re-initialised.
 */
#define KVQ_WS_WAIT_LIMIT_WORD 16383
kvq_status kvq_workspace_init(void* workspace, size_t ws_bytes, kvq_stream_t stream);

/*
 * kvq_set_grid_override -- testing and tuning aid (the source pages have no counterpart):
 * run the attention kernel and kvq_decode_step on `ctas` CTAs instead of one per SM, for
 * every later call in the process (0 restores the default).  Fewer CTAs give each warp
 * more pages, so small batches reach the deep-pipeline paths full-size batches take.
 * kvq_workspace_size depends on it: size workspaces after setting it.  Not thread-safe
 * with respect to calls running in other threads.  ctas in [0, 65535].
 */
kvq_status kvq_set_grid_override(int32_t ctas);

/*
 * kvq_sparse_decode_attn -- attention of each query head over the tokens of its kv
 * head's selected pages (AMASS "What is in the box"; ARGUS "Why It Works": low-bit
 * values are turned back into high precision before attention).
 *  q         device [B][Hq][D], cache dtype.
 *  sel, cnt  as written by kvq_select_topk (pages must be < ceil(seq_len/16)).
 *  sm_scale  softmax scale (1/sqrt(D) for standard attention).
 *  out       device [B][Hq][D] cache dtype out: softmax(sm_scale * q.k) v over the tokens
 *            of the selected pages; zeros when a kv head has no selected page; NaN (and a
 *            NaN lse) when a key or value read back is NaN (non-finite input, flagged).
 *  lse       device [B][Hq] fp32 out (may be NULL): natural-log log-sum-exp of the
 *            scaled logits (-inf when nothing is selected).
 *  workspace device scratch of at least kvq_workspace_size() bytes, prepared once with
 *            kvq_workspace_init (split-K partials; the last CTA of each (b, kv head) merges
 *            them, counted by arrival counters the call leaves at zero).  B*Hkv < 5632.
 */
kvq_status kvq_sparse_decode_attn(const kvq_cache* cache, const void* q, const int32_t* sel,
                                  const int32_t* cnt, int32_t kmax, float sm_scale, void* out,
                                  float* lse, void* workspace, size_t ws_bytes,
                                  kvq_stream_t stream);

/*
 * kvq_sparse_decode_attn_noalloc -- kvq_sparse_decode_attn without a caller workspace.
 * (The source pages have no counterpart: this is an interface for callers that cannot
 *  allocate device memory at decode time, e.g. an engine that gave all device memory to
 *  its own KV page pool, or a plugin with no allocation hook.)
 *  Same arguments and results as kvq_sparse_decode_attn minus the workspace.  The split-K
 *  scratch is a static device array of kvq_noalloc_scratch_bytes() (16 MiB) inside the
 *  library, held by every GPU that loads it until the process exits.  Allocates nothing
 *  (no cudaMalloc/cudaFree).  Returns KVQ_ERR_WORKSPACE when kvq_workspace_size() for
 *  this cache exceeds the static size, and KVQ_ERR_UNSUPPORTED for B*Hkv >= 5632 as
 *  kvq_sparse_decode_attn does.  Each call made outside a stream capture looks up the
 *  array's device address on the current device (cudaGetSymbolAddress; a re-created
 *  context gets its new address); a call made while the stream captures reuses the last
 *  lookup, so make the first call on each device before any stream capture.  Each call
 *  clears the array's B*Hkv arrival counters with an asynchronous memset on `stream`
 *  before the attention launch.  All calls share the array: calls whose work overlaps on
 *  the GPU race.
 */
kvq_status kvq_sparse_decode_attn_noalloc(const kvq_cache* cache, const void* q, const int32_t* sel,
                                          const int32_t* cnt, int32_t kmax, float sm_scale, void* out,
                                          float* lse, kvq_stream_t stream);

/* Size in bytes of the static scratch used by kvq_sparse_decode_attn_noalloc. */
size_t kvq_noalloc_scratch_bytes(void);

/*
 * kvq_append_scores -- kvq_append followed by kvq_page_scores, with the same results, as
 * two kernels chained by programmatic dependent launch: the score sweep starts while the
 * append runs and scores every 16-page tile except those holding a page pos[b] / 16; it
 * scores those after the append has completed.  Arguments as those two calls (pos, k_new,
 * v_new required).  pos, q and seq_len must not be written by the append's own kernel
 * (they are inputs of the call), and the sweep may read them before the append completes.
 */
kvq_status kvq_append_scores(const kvq_cache* cache, const int32_t* pos, const void* k_new,
                             const void* v_new, const void* q, float* scores, kvq_stream_t stream);

/*
 * kvq_score_select -- kvq_append (when pos is not NULL), kvq_page_scores and
 * kvq_select_topk in one launch, with the same results (AMASS "What is in the box":
 * score every page from its summary, keep the best).  The warp that scores the tile of a
 * sequence's appended token writes the token first; the CTA that finishes the last score
 * tile of a (b, kv head) selects its pages.  Arguments as those three calls; workspace:
 * any kvq workspace of at least 64 KiB prepared with kvq_workspace_init (per-(b, kv head)
 * tile counters at its head; the call leaves them zero).  B*Hkv <= 8191,
 * max_pages <= 51200.  Coverage selection is not supported here (KVQ_ERR_UNSUPPORTED).
 */
kvq_status kvq_score_select(const kvq_cache* cache, const int32_t* pos, const void* k_new,
                            const void* v_new, const void* q, const kvq_select_params* params,
                            float* scores, int32_t* sel, int32_t* cnt, int32_t kmax, void* workspace,
                            size_t ws_bytes, kvq_stream_t stream);

/* Workspace bytes kvq_decode_step needs for this cache and kmax. */
kvq_status kvq_step_workspace_size(const kvq_cache* cache, int32_t kmax, size_t* bytes);

/*
 * kvq_decode_step -- one whole decode step in one launch: kvq_append (when pos is not
 * NULL), kvq_page_scores, kvq_select_topk and kvq_sparse_decode_attn, with the same
 * arithmetic and the same results as those four calls made in that order (AMASS "What is
 * in the box": score every page from its summary, attend only the selected pages; ARGUS
 * "The One-Minute Explanation" / "Visual Architecture": the new token is written into its
 * page's tier).  A persistent kernel streams the summaries and then the selected pages,
 * choosing each (b, kv head)'s pages as soon as all its scores exist.
 *  pos, k_new, v_new  as kvq_append; pos may be NULL (no append).  seq_len must already
 *            count the appended token (pos[b] / 16 < ceil(seq_len[b] / 16), else the token
 *            is not written and KVQ_DERR_BAD_POS is set).
 *  q, params, sel, cnt, kmax, sm_scale, out, lse  as kvq_select_topk and
 *            kvq_sparse_decode_attn.
 *  scores    device [B][Hkv][max_pages] fp32 out: the page scores for p < ceil(seq_len/16)
 *            (entries past that are not written).
 *  workspace device scratch of at least kvq_step_workspace_size() bytes, prepared once
 *            with kvq_workspace_init.
 *  Returns KVQ_ERR_UNSUPPORTED for coverage selection, for pools in host memory
 *  (host_tiers != 0), when B*Hkv > 8183, or when the per-CTA tables and selection keys
 *  (4 * (3B + max_pages) bytes) leave too little shared memory for the page ring.
 */
kvq_status kvq_decode_step(const kvq_cache* cache, const int32_t* pos, const void* k_new,
                           const void* v_new, const void* q, const kvq_select_params* params,
                           float* scores, int32_t* sel, int32_t* cnt, int32_t kmax, float sm_scale,
                           void* out, float* lse, void* workspace, size_t ws_bytes,
                           kvq_stream_t stream);

/*
 * quad page score (AMASS "decode-time sparse KV-cache attention for vLLM", "What is in the
 * box", Stage A: a quadratic Gaussian-MGF page score from a tiny per-page summary holding
 * r' eigenvalues per page).  The pages give no formula, rank or basis; this library reads
 * it as follows.  Keys of page p ~ N(mu_p, Sigma_p); with the caller's orthonormal basis
 * rows u_1..u_r' of a kv head, page p keeps lambda[p][i] = u_i^T Sigma_p u_i (the (1/n)
 * variance of the page's keys, as they arrived, along u_i), and its score for query head h
 * is log E[exp(s q_h.k)] ~= s q_h.kbar_p + 1/2 s^2 sum_i lambda[p][i] (u_i.q_h)^2 (kbar_p
 * the fp16 mean-key summary), maximised over the kv head's query heads.
 * State arithmetic (fp64, no fused multiply-add, so built and appended pages agree bit for
 * bit): y_i = sum_d u[i][d] k[d] in channel order; per page S1_i = sum_t y_i, S2_i =
 * sum_t y_i^2 in token order; lambda = fp16(max(S2/n - (S1/n)^2, 0)), saturating (flagged).
 */
typedef struct {
  int32_t rank;        /* r', a multiple of 8 in [8, 32] */
  int32_t reserved;
  const float* basis;  /* device [Hkv][rank][D] fp32, the basis rows of each kv head (caller-owned) */
  uint16_t* lambda;    /* device [B][Hkv][max_pages][rank] fp16 bits */
  double* open_sums;   /* device [B][Hkv][2][rank]: S1 then S2 of each sequence's open page */
} kvq_quad;

/* kvq_quad_build -- quad state of a prefilled context (same inputs as kvq_build_pages):
 *  lambda of every page holding tokens, and the open page's sums (zero when the last page
 *  is full).  Pages past seq_len are not written. */
kvq_status kvq_quad_build(const kvq_cache* cache, const kvq_quad* quad, const void* k_src,
                          const int64_t* cu_seqlens, int64_t src_tokens, kvq_stream_t stream);

/* kvq_quad_append -- advance the quad state by one token per sequence (same pos and k_new
 *  as kvq_append; pos < 0 skips, pos >= max_pages*16 sets KVQ_DERR_BAD_POS): the open
 *  page's sums restart at a page boundary, and lambda[pos/16] is refreshed. */
kvq_status kvq_quad_append(const kvq_cache* cache, const kvq_quad* quad, const int32_t* pos,
                           const void* k_new, kvq_stream_t stream);

/* kvq_quad_page_scores -- scores[b][g][p] = max over h in the group of
 *  sm_scale * q_h.kbar_p + 0.5 * sm_scale^2 * sum_i lambda[b][g][p][i] * (u_i.q_h)^2,
 *  fp32, for p < ceil(seq_len[b]/16), -inf for the remaining pages (layouts as
 *  kvq_page_scores; q must be 16-byte aligned).  Feed the result to kvq_select_topk; for
 *  coverage selection pass sm_scale = 1 there (the score already carries the scale). */
kvq_status kvq_quad_page_scores(const kvq_cache* cache, const kvq_quad* quad, const void* q,
                                float sm_scale, float* scores, kvq_stream_t stream);

/* kvq_quad_append_scores -- kvq_append + kvq_quad_append + kvq_quad_page_scores in one
 *  launch, with the same results (the warp that scores the tile holding a sequence's new
 *  token writes the token and its quad state first).  pos, k_new, v_new as kvq_append. */
kvq_status kvq_quad_append_scores(const kvq_cache* cache, const kvq_quad* quad, const int32_t* pos,
                                  const void* k_new, const void* v_new, const void* q, float sm_scale,
                                  float* scores, kvq_stream_t stream);

/*
 * kvq_requantize_pages -- tier demotion: move pages to a lower-precision tier.
 * (ARGUS "Virtual Memory for Transformers", "Visual Architecture": pages cool down the
 *  cascade FP16 -> INT8 -> INT4 -> INT2 -> 1-bit.)
 *  items  device [n][3] int32: (b, page, new block-table entry (tier << 29) | slot).
 *  For every item, each kv head's K and V values of the page are read back from the
 *  current tier (the 16-bit value, fp32(c*scale+zero) or +-m, as kvq_dequant_page) and
 *  quantised again with kvq_append's quantiser into the new entry's tier and slot, token
 *  slots past seq_len zero; then block_table[b][page] = new entry.  The page summary and
 *  open_ksum are unchanged (they follow the keys as they arrived), so later appends to an
 *  open page continue in the new tier.
 *  The new tier must be a quantised one (1..5) and the new (tier, slot) must differ from
 *  the current one; an item that is out of range, names a page without tokens, has an
 *  invalid current or new entry, or aliases its own slot is skipped with
 *  KVQ_DERR_BAD_PAGE.  The caller owns slot allocation: new slots must not be referenced
 *  by any block-table entry, one item per (b, page), and the old slot may be reused once
 *  the call's work on the stream is complete.  Two kernel launches; n == 0 is a no-op.
 */
kvq_status kvq_requantize_pages(const kvq_cache* cache, const int32_t* items, int32_t n,
                                kvq_stream_t stream);

/*
 * kvq_dequant_page -- values read back from storage for one logical page (testing aid).
 *  out device [Hkv][2][16][D] fp32: for each kv head, K then V, every token slot: the
 *  16-bit value, fp32(c * scale + zero), +-m, or e4m3(c) * scale, per the page's tier.
 */
kvq_status kvq_dequant_page(const kvq_cache* cache, int32_t b, int32_t page, float* out,
                            kvq_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* KVQ_H_ */
