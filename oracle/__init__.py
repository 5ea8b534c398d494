"""Plain, slow, fp64 CPU oracle for block-sparse long-context prefill.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may use it.  It shares no code with
the CUDA library (no kernels, headers, helpers or constants); the two meet only
in the seeded input generator of ``workloads``.

Sources (page title and the part of it each function follows):

* AnchorAttention: Difference-Aware Sparse Attention with Stripe Granularity
  - Eq. (1): anchor = max score over the initial (sink) key block and the local
    key block;
  - Eq. (2): stripe mask I(avgpool(x_a) - avgpool(Q)K^T/sqrt(d) <= theta);
  - Eq. (3): the kept index set I of discrete key coordinates;
  - Sec. 3.4 / Appendix C, Algorithm 2: the anchor is the row-max buffer M
    (the review notes the listing's ``Acc`` is a mis-print for M).
* SALE: Low-bit Estimation for Efficient Sparse Attention in Long-context LLM
  Prefilling
  - Sec. 3.2: 4-bit quantised Q/K estimate of S (SageAttention2-style);
  - Sec. 3.3: Relative Attention Score P~ = exp(S~ - em_i) / el_i over the
    sink-local area;
  - Sec. 3.4, Eq. (4) as corrected by the review: S~ >= ln(tau * el_i) + em_i;
  - block skipping: a (bq x bk) block is skipped when every score is below tau.

Modules:

* ``selection`` -- anchor (stripe) selection and SALE (block) selection;
* ``attention`` -- masked softmax attention over a kept key set, and an
  independently written dense causal attention;
* ``calibration`` -- SALE's per-head tau calibration (Sec. 3.3, Appendix C);
* ``decode`` -- decode-shaped reuse of a prefill plan (SpotAttention Fig. 2,
  Sec. 3; KVpop Sec. 3, transposed attention);
* ``fp8`` -- E4M3 rounding and SageAttention-style quantisation for an FP8
  Computation Pass (SALE review, Summary).

Every function here is pinned by tests in ``tests/test_oracle_*.py`` against
closed forms, invariants, special cases and brute force; see the module
docstrings for which pin covers which function.
"""

from . import attention, calibration, decode, fp8, selection  # noqa: F401
