"""Oracle: a plain, slow, obviously correct CPU statement of the hot path.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it. The
product (``trie_constrained_beam_b200``) never imports it and has no CPU
fallback; the oracle and the CUDA path share no code except the seeded input
generators in ``sidgen``.

Everything is numpy in float64. Sources (web pages, cited by title/section):

* flashrec 0.1.0 (PyPI page), introduction: a semantic ID is a short,
  fixed-depth token sequence; a request decodes 3-5 steps at beam widths of
  50-512 or more, every continuation restricted to the catalog.
* flashrec 0.1.0, Features > Decoding, "SID constraint": a dense or CSR trie
  restricts decoding to valid SIDs, lm_head is evaluated over the SID token
  range only, illegal SIDs are never candidates.
* flashrec 0.1.0, Features > Decoding, "Scheduling": beam rows of several
  requests share one step.
* flashrec 0.1.0, Features > Serving, "API": deterministic top-k at
  temperature 0; Gumbel top-k without replacement above it.
* flashrec 0.1.0, Quickstart: beams come back ranked best-first with a
  sequence score; without a catalog the engine decodes the full vocabulary.
* SPRINT (paper summary), inference paragraph: only valid SIDs of a prefix
  trie are scored, by a token log-probability sum, then top-K; one pass gives
  an L-by-M table and scoring a SID is a table lookup.

Readings where the pages are silent (each restated where it is used):
log-softmax over the full codebook of the level with invalid children at
-inf and no renormalisation; one live root row per request at step 0;
ties broken by (score desc, parent slot asc, code asc); fewer than n
candidates are padded with (-inf, -1, -1, -1).

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
(brute-force enumeration, library special cases, invariants, published
generator vectors); none is "parity unpinned".
"""
from .trie import OracleTrie  # noqa: F401
from .beam import (  # noqa: F401
    NEG_INF,
    beam_finalize,
    beam_search,
    beam_step,
    log_softmax_full,
)
from .catalog import catalog_score_topk  # noqa: F401
from .lmhead import lmhead_logits, fused_lmhead_step  # noqa: F401
from .gumbel import beam_step_gumbel, gumbel, philox4x32_10  # noqa: F401
