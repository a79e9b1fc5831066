"""CPU oracle for the ARKV tri-state KV cache decode path -- TEST INFRASTRUCTURE ONLY.

A plain, slow, float64 restatement of what the method on the ARKV page computes
("ARKV: Adaptive and Resource-Efficient KV Cache Management under Limited
Memory Budget for Long-Context Inference in LLMs", gist.science), written from
the page's description; the CUDA library is checked against it.

Only `tests/`, `__graft_entry__.smoke()` and `bench.py`'s CPU-baseline and
reference legs may import or run anything in this package.  The product path
(the `mixed_precision_kv_arkv_b200` package and its CUDA library) never does,
and this package imports nothing from the product.

Parity unpinned: the per-layer Original:Quantized ratio map `oq_ratio` is a
reading (the page names its inputs -- attention entropy, variance, kurtosis --
and its direction, not a formula); it is pinned only by its own closed-form
cases.  Everything else is pinned by tests against closed forms, library
routines, exact rational arithmetic or brute force.
"""
