"""CPU oracle of the ZeRO partitioned mixed-precision Adam step.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline / reference leg of ``bench.py`` may import or run anything
in this directory.  The product (the CUDA library and its Python binding)
never imports it, and this package never imports the product.

Contents:
  plan.py       partition maps, per-stage memory and communication closed forms,
                HBM bytes of the step (plain Python integers / Fractions)
  zero_oracle.c the elementwise core: rank-order fp32 sum of bf16 gradients,
                fp32 Adam in a fixed operation order, bf16 round-to-nearest-even
  core.py       ctypes binding of the C core (built by build.py with gcc)
  step.py       stage-0 replicated step and stages 1-3 partitioned step drivers,
                stage-3 layer gather
  adam_fp64.py  textbook float64 Adam, to bound the fp32 core's rounding

Every function is pinned by a ``-m "not gpu"`` test against something other
than itself (values the pages print, closed forms, torch's own Adam and bf16
conversion, exact rational sums, brute force on tiny inputs).
"""
