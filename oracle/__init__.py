"""CPU oracle for the paged decode step.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import anything from this package.  The
CUDA library never calls into it and this package never imports the CUDA
library or its Python binding: the two share no code.  Inputs for both come
from the seeded generators in ``workloads.py``.

What the oracle computes, in plain and slow form (fp64 unless a function says
otherwise):

* ``attention``   - decode attention over a sequence's *contiguous* K/V
                    history: out = softmax(scale * q K^T) V, two-pass softmax.
* ``allocator``   - a reference block manager: FIFO free queue, per-sequence
                    block tables with fill counts, refcounts, fork,
                    copy-on-write and free.
* ``numerics``    - exact decoding of fp16 / bf16 / FP8-E4M3 bit patterns and
                    FP8-E4M3 encoding (round to nearest even, saturating).
* ``engine``      - the decode round: allocator + contiguous histories; append
                    first, then attend (the new token sees itself).
* ``toy_transformer`` - the cached-vs-recompute check on a small multi-layer
                    model, with exact multiply-accumulate counts.
* ``closed_forms``    - per-token KV bytes, pool capacity, utilisation.
* ``simulator``   - the exhibit's allocation bench (arrivals, FCFS, block size
                    vs max-length reservation).

Every function cites the page passage it follows by page title and section.
Pages: "KV 缓存与分页注意力" (world.lapla.si, exhibit F55), the "KV 缓存" topic
page (aiinfact.com, levels 1-3), and "读懂PagedAttention：vLLM的KV缓存与GPU显存管理"
(iplexlaw.co.kr).

Parity status: every function here is pinned by a ``-m "not gpu"`` test
against closed forms, printed values from the pages, library routines or
brute force; none is "parity unpinned".
"""
