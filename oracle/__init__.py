"""CPU oracle for the K2 routed-MoE layer forward pass (test infrastructure).

This package is test infrastructure only. The tests, the package's smoke
check and the benchmark's CPU-baseline leg may import it; the product path
(the C-ABI library and its Python binding) never does and shares no code with
it.

Modules:
  e4m3   -- OCP FP8 E4M3 ("e4m3fn") encode/decode written from the format's
            definition (sign, 4 exponent bits with bias 7, 3 mantissa bits,
            no infinities, S.1111.111 = NaN, largest finite 448).
  moe    -- the layer in float64 with numpy: router, biased top-k selection,
            normalisation and scaling, SwiGLU experts, weighted combine with
            the shared expert, and the FP8 block-scaled variant.
  brute  -- the same definition as explicit per-element Python loops, for
            tiny shapes only; it pins the vectorised oracle.

Parity status: every function is pinned by a test in tests/test_oracle_*.py
against brute force, closed forms, invariants, a library routine or values
printed on the pages. Nothing here is "parity unpinned".
"""
