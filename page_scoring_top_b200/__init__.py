"""B200-native page indexer: score each request's candidate KV pages against
its query heads and keep the top-K page indices.

The compute runs in ``libidx.so`` (CUDA for sm_100a behind a C ABI declared in
``include/idx.h``).  ``page_scoring_top_b200.binding`` is the thin Python
binding over that ABI; ``page_scoring_top_b200.synth`` draws the seeded
synthetic inputs.  Importing this package loads nothing: the CUDA library is
opened on first use, and its absence is an error, never a fallback.
"""

__all__ = ["binding", "synth"]
