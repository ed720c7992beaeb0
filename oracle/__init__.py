"""CPU oracle for the Gemma-4-26B-A4B MoE feed-forward block.

TEST INFRASTRUCTURE ONLY. Only the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it. The
library's own path never calls into this package, and this package never
imports the library: the two share nothing but the seeded input generators.

Everything here is plain numpy in float64 (the NVFP4 quantiser takes its
rounding decisions in float32, the precision the format is defined in), written
to be read against the pages:

* ``moe_oracle`` - router, softmax, top-k, renormalisation, permutation,
  GeGLU experts, shared MLP, branch sum, inter-block RMSNorm;
* ``nvfp4``     - e2m1 / e4m3 codecs and the group-16 NVFP4 quantiser;
* ``wformats``  - the weight-only formats SFP8 and Q4_0 (readings stated in
  the module) and the block on weights in those formats;
* ``sandwich``  - the pre/post-FFN RMSNorm sandwich and residual;
* ``counts``    - parameter counts implied by the layer shapes.

Parity status: every function is pinned by a ``-m "not gpu"`` test to
something other than itself (page values, closed forms, library routines,
brute force). No worked numerical example of the block's output exists on the
pages, so actual output values are pinned only through those invariants and
through two independent CPU evaluations (grouped-by-expert and dense
per-token).
"""
