"""Plain, slow, float64 CPU oracle of the FFN-service MoE layer -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference legs of
``bench.py`` may import anything in this package.  The product (``libafd_ffn.so`` and its
Python binding in ``ffn_side_expert_b200``) never imports, links or calls it, and the two
share no code: their only common dependency is the seeded input generator ``synth``.

Modules
- ``oracle.moe``   router, top-k, gate weights, dispatch order, SwiGLU experts, combine
- ``oracle.fp8``   e4m3 rounding and the per-row quantisation mirror of the W8A8 path
- ``oracle.comm``  the pages' per-token dispatch/combine byte account

Pins (every function is checked against something other than itself, in tests marked
``not gpu``): closed forms of silu; a hand-derived worked example of one SwiGLU expert
(tests/test_oracle_expert.py::test_swiglu_worked_example); the E=1, k=1 layer against a dense FFN; top-k
against a brute-force search over all k-subsets; the two gate-weight formulas against each
other and sum-to-one; the dispatch order against an O(T^2 k) recount; the combine against
a one-hot gather and linearity; every e4m3 code against ml_dtypes and torch; the per-row
quantisation against torch's fp32 path, including rows where only an fp32 scale gives the
right code; the W8A8 expert (hidden and SwiGLU rows quantised) against a hand-worked example
and a scalar-loop layer; and the communication account against the number printed on the
A/F 分离 page.  tests/test_oracle_mutations.py plants eleven plausible mistakes and checks that
each one fails its pins.
The pages print no numeric example of the MoE computation itself, so no pin of the expert
arithmetic comes from the pages: those pins are mathematical.
"""
from . import comm, fp8, moe  # noqa: F401
