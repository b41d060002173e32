"""CPU oracle for the DynamicRad block-sparse attention hot path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports, calls or links
this package: only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` use it.  It shares no code with the CUDA library.

It is a plain, slow, float64 restatement of what the path computes, written
from "DynamicRad: Content-Adaptive Sparse Attention for Long Video Diffusion"
(arXiv 2604.20470):

* ``geometry``  -- Sec. 3.1, Eqs. 1-7 and "Density control within blocks":
  the radial candidate block set and the always-kept near-frame set;
* ``selection`` -- Sec. 3.2 and Algorithm 1 in the block-pooled form: block
  mean pooling, block proxy scores, static-ratio (top rho, k from Eq. 8) and
  dynamic-threshold (smallest prefix reaching softmax block mass tau);
* ``attention`` -- Sec. 3.3, Eqs. 12-13 with epsilon -> 0: softmax attention
  restricted to the kept blocks, with its log-sum-exp;
* ``sampling``  -- the paper-exact static-ratio mode of Sec. 3.2 (Eq. 8):
  k = max(1, floor(|P| * rho)) token pairs per frame pair, drawn with a seeded
  SplitMix64 generator, aggregated to blocks as in Sec. 3.1;
* ``dynamic_tokens`` -- the paper-exact dynamic-threshold mode of Sec. 3.2
  (Eqs. 9-11, Eq. 19): fused-head proxy logits on the candidate token pairs,
  per-frame-pair z-scores, tau_1 / tau_2 thresholds with the top-pair
  fallback, aggregated to blocks;
* ``backward``  -- gradients dQ, dK, dV of the block-masked attention (for the
  mask-aware fine-tuning of Sec. 3.3);
* ``proxy``     -- the objective of the offline parameter search on the
  feature-drift proxy (Appendix C.2-C.4, Eq. 22).

Every function is pinned by ``-m "not gpu"`` tests to closed forms, library
routines for special cases, brute force on tiny inputs, or invariants the
paper states (for example the discarded-mass bound of Appendix C.3).  The
absolute values of masks and attention outputs on the synthetic workloads
have no printed counterpart in the paper: beyond those pins they are
"parity unpinned".
"""
