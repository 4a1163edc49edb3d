"""Float64 CPU oracle for compressed sparse KV decode attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import or call anything in this package.
The product path (the C-ABI library and its Python binding) never touches it,
and this package shares no code with the CUDA path: both sides only consume
the same input bytes from ``datagen``.

What it computes, and where each definition comes from (the pages are:
[P1] "How DeepSeek V4 Uses Less Memory: KV Cache Explained",
[P2] "DeepSeek V4 KV Cache" visual walkthrough,
[P3] "KV cache at 890 bytes per token: how DeepSeek squeezed attention memory"):

* ``compress``   c4a / c128a compressors: [P1] "c4a (the milder scheme)" and
                 "c128a (the aggressive scheme)"; [P2] Step 4 diagrams.
* ``rope``       rotary embedding on the last 64 channels and its inverse on
                 the output: [P1] "Shared key and value".
* ``formats``    fp8 E4M3 per-row, fp4 E2M1 with an E4M3 scale per 16
                 channels: [P1] quantisation paragraphs; [P3] "storing the
                 main KV in FP4".
* ``indexer``    one 128-dim indexer dot per compressed entry and the top-512
                 selection: [P1] "c4a" paragraph and indexer paragraph;
                 [P2] Step 5.
* ``attention``  shared K/V decode attention over selected (or all) compressed
                 entries plus the 128-token window: [P1] "The sliding window",
                 "Shared key and value"; [P2] Steps 3, 5, 6.
* ``footprint``  closed-form cache sizes: [P1] opening summary, "To judge the
                 saving", hybrid cache manager paragraph.

Parity status: every function here is pinned by tests in
``tests/test_oracle_*.py`` against values the pages print, closed forms,
textbook/library routines or brute force.  Whether the spec choices match
DeepSeek's production numerics cannot be pinned from the pages (no page prints
an attention output); that is a statement about the spec, not about this code.
"""
from . import formats, rope, compress, indexer, attention, footprint  # noqa: F401
