"""B200-native (sm_100a) Prism Attention decode hot path.

Quantized proposal scoring with a top-kappa_p candidate pool, exact
rescoring and top-kappa inside the pool, and sparse flash-decode over the
selected rows -- hand-written CUDA behind the C ABI of ``libprism.so``
(declared in ``include/prism.h``).  ``kv_cache_top_proposal_b200.prism``
is the thin ctypes binding; ``kv_cache_top_proposal_b200.workload`` builds
seeded synthetic caches.  Import the submodule you need.
"""
