"""CPU oracle for the CSA2 compressed sparse-attention step.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The CUDA library never calls it and shares no code with it.

Plain NumPy, exact or float64 arithmetic, written for a reader to check by eye
against the definitions it cites:

* ``codecs``    - E2M1, E4M3 (OCP "FN"), UE8M0 scalar formats.
* ``quant``     - FP4 main-KV entry (E2M1 + one E4M3 scale per 16 channels,
                  288 B) and FP8 sliding-window entry (E4M3 + UE8M0 per 32
                  channels, 528 B); plain E4M3 cast of indexer keys/queries.
* ``indexer``   - lightning-indexer scores, Top-K, the hierarchical candidate
                  pool and re-indexing inside it.
* ``attention`` - sparse MLA attention over selected entries + window.
* ``layers``    - Full / Reindex / Reuse layer stacks.
* ``accounting``- cache bytes per entry / per token.

Parity unpinned (the pages give no code): the exact E4M3 scale rounding rule
(round-to-nearest-even of amax/6), the UE8M0 exponent rule (ceil(log2(amax/448)))
and the pool block score (max over 8 positions) are this project's readings of
the pages; they are pinned only to their own stated definitions.
"""
