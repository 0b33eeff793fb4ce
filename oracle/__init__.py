"""CPU oracle for sparse mixed-precision paged decode attention.

TEST INFRASTRUCTURE ONLY.  This package is a plain, slow, fp64 numpy restatement of
what the decode path computes: per-group quantisation and bit packing of cold pages
(int8 / int4 / int2 / 1-bit and fp8 e4m3), tier demotion, the per-page mean-key
summary, the page score and the quad (Gaussian-MGF) page score with its per-page
eigenvalue state, the top-k and coverage page selections with forced sink/recent pages,
and attention over the selected pages with dequantisation on read.
Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference legs of
``bench.py`` may import it.  The CUDA library never calls it and shares no code with
it; the two meet only in the seeded input generators, which hold no arithmetic of
the method.

Sources (web pages about KV-cache compression; cited by title and section):

* AMASS -- "decode-time sparse KV-cache attention for vLLM" (amass-kv 0.1.1):
  "What is in the box" (per-page summary feeding a page score -- Stage A, the quad
  score over r' per-page eigenvalues --, a small selected working set, a sparse paged
  kernel that reads only those pages) and "Quickstart" (``budget``: a fixed
  selected-page fraction; ``coverage``: nucleus coverage of the page masses).
* ARGUS -- "Virtual Memory for Transformers" (argus_cache 0.1.7.1): "The One-Minute
  Explanation" and "Visual Architecture" (hot fp16 pages, cold pages down the cascade
  FP8, INT8, INT4 2-way, INT2 4-way and 1-bit 8-way packed as they cool; transient
  high-precision reconstruction only when a query touches a page), "Quickstart" (``sink_tokens``:
  leading tokens kept in fp16) and "Why It Works" (no low-bit matmul: dequantise,
  then attend).
* AdaptiveKV (0.1.0): "Architecture Overview" (2/4-bit uint8 bit-packing engine).

Where the pages leave a step open the plainest reading is taken; each reading is
stated in the docstring of the function that applies it.

Parity status: every function here is pinned by ``tests/test_oracle_*.py`` against
brute force, closed forms or a separately written textbook formula.
"""
