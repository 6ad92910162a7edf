"""Plain CPU oracle for the vocab-sliced logits projection and the per-row sampler.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The product path (``vocab_sharded_logits_b200``) never imports it and
shares no code with it: no kernels, helpers, tables or constants.

Every function here restates a plain definition, in float64 unless the
definition itself fixes another precision, with no blocking, fusion or
reordering beyond what the definition states:

* ``oracle.gemm``     - the vocab-slice projection with no gather
  ("Qwen4Exp batch-sharded sampling: inside vLLM PR #61018", orcarouter.ai
  blog, section "batch-sharded sampling in one paragraph" and section "why
  three lines were the whole job": each rank returns only its own vocab slice
  of ``lm_head(hidden)``).
* ``oracle.philox``   - Philox4x32-10 written from its published description
  (Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3",
  SC'11, section 3.2 and Table 2).
* ``oracle.sampler``  - temperature, top-k, top-p, Gumbel-max draw and top-n
  logprobs over the concatenated vocab slices of one row.  The pages name the
  sampler's top-k / top-p / logprob work and the batch x (spec+1) x vocab logits
  (same page, section "batch-sharded sampling in one paragraph"); the draw
  (Gumbel-max keyed by Philox4x32 on (seed, request, position, token)) and the
  exact tie / threshold readings are the plainest readings stated in each
  function's docstring.  ``processed_logprobs`` gives the log-probabilities of
  the distribution the draw samples from (after temperature, top-k, top-p).
* ``oracle.verify``   - speculative verification of deterministic drafts over
  a request's (spec + 1) rows (same page: the acceptance length of section
  "the 1.5 % estimate"; draft logits are left for later in section
  "batch-sharded sampling in one paragraph").
* ``oracle.tile_stats`` - per block of 128 ids of a vocab slice, the maxima of
  its four 32-id quarters, its sum of exp and its smallest finite logit: the
  statistics the projection can emit tile by tile so that the sampler reads
  only the tiles that can hold its candidates (a reading of the same section;
  the record is the library's, stated in the module).
* ``oracle.timing``   - the harness that times the sampler oracle on the
  host's cores for the CPU baseline (no arithmetic of the method).

Pins (see ``tests/test_oracle_*.py``): the Philox known-answer vectors of the
Random123 distribution, brute-force enumeration on tiny vocabularies, closed
forms (greedy == argmax, top_k=1, top_p -> 0, top_p=1 keeps all, sum of
probabilities == 1), exact integer GEMMs, and chi-square tests of the draw
frequencies; the processed logprobs against the library log-softmax (full
vocabulary), point masses, and the frequencies of the oracle's own draws; the
verification against an independent formulation and, by sampling, against
the rejection rule it implements for a point-mass draft.
No function here is "parity unpinned".
"""
