"""fp64 CPU oracle for routed block-sparse attention with proxy residual.

TEST INFRASTRUCTURE ONLY.  The product path never imports this package: only
the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may call it.  It shares no code with the CUDA library.

The oracle is written step by step from the method as the pages state it,
plainly and slowly, in float64 from the exact bf16 inputs:

* block-mean pooling of queries and keys (PARK page, abstract and
  sections 4.1-4.2: blocks are represented by their averaged queries/keys);
* proxy logit Qbar_i . Kbar_j / sqrt(d) + ln n_j -- the centroid estimate
  that PARK page section D.2 shows to be a Jensen lower bound on the exact
  block log-mass -- and its softmax over key blocks;
* Top-p routing: blocks taken in descending estimated importance while the
  accumulated estimate is still below the threshold (PARK page section 3.2),
  with a dynamic, clamped budget (Sol-Attn abstract, thelatestinai page);
* one softmax per query token over the exact tokens of its kept blocks, plus
  (residual mode) one pseudo-key per dropped block that reuses the block's
  proxy score (Sol-Attn abstract: the skipped blocks are approximated from
  the scores the router already computed);
* as an alternative selection, a fixed threshold on each block's proxy
  probability (Sol-Attn abstract: on-the-fly block thresholding);
* optional token reordering before blocking and its inverse after
  (DFSAttn abstract: Hilbert curve-based token reordering);
* the probe-fitted residual correction (SparsePR page, section 2B): exact
  dense rows for a few probes (chosen by the seeded generator and passed in),
  a ridge-fitted affine map of their residuals, restricted to the residuals'
  leading right singular subspace (:mod:`oracle.probe_residual`).

Readings where the pages are silent are listed in the module docstrings of
:mod:`oracle.spattn_ref` and :mod:`oracle.hilbert`.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
and ``tests/test_oracle_probe_residual.py``
against closed forms, library routines (torch fp64 softmax attention),
brute-force enumeration or invariants; none is "parity unpinned".
"""
from .spattn_ref import (  # noqa: F401
    decode_bf16, block_sizes, gather_tokens, scatter_tokens, block_means,
    proxy_logits, block_softmax, route_rows, route_threshold, attend_block, attention,
    forward, exact_block_logmass, attention_flops, MASS_MARGIN, TIE_MARGIN,
)
from .hilbert import hilbert_index, hilbert_perm  # noqa: F401
from . import probe_residual  # noqa: F401
