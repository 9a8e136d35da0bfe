"""CPU float64 oracle for iS-KV (basis-synchronized online low-rank KV compression).

TEST INFRASTRUCTURE ONLY.  This package is a plain, slow, obviously correct
restatement of what the method computes, used to check the CUDA library.  Only
``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` / reference
legs of ``bench.py`` may import it.  It shares no code with the CUDA path and
imports nothing from ``online_rank_kv_b200``; the product path never calls it.

Sources (web pages, cited by title and section):
  * "iS-KV -- Basis-synchronized online low-rank KV compression -- What does it
    mean?" (learnaivisually.com explainer): TL;DR, Jargon (Block-incremental
    SVD, Pre-RoPE keys, Persistent-KV compression) and the body paragraphs on
    the recent window, block folding, basis synchronization and drift, and the
    A40 memory test.
  * "KV-CoRE" technical summary (gist.science), section 2 Methodology: the
    covariance route to the batch SVD, used only by the tests as an independent
    cross-check.

Parity status per function is stated in each docstring ("pinned by ..." or
"parity unpinned").
"""

from .iskv_oracle import (  # noqa: F401
    bf16_round,
    ready_blocks,
    rope_inv_freq,
    rope_rotate,
    fold_block,
    HeadFactor,
    dense_decode,
    full_kv_bytes,
    persistent_kv_bytes,
    LatentQuant,
    joint_head_decode,
)
