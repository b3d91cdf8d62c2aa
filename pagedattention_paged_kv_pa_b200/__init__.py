"""PagedAttention decode over a paged KV pool, for B200 (sm_100a).

The kernels and the host block allocator live in ``libpa_b200.so`` behind the
C ABI of ``include/pa.h``; ``binding`` is its thin Python binding (import it to
use the library -- it raises if the library is not built).  ``workloads``
makes seeded synthetic inputs.
"""
__all__ = ["binding", "workloads", "build"]
