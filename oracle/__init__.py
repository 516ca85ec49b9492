"""CPU oracle for the paged KV-cache decode path — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import, call, link or execute anything in this package. The
product (``paged_kv_cache_320_b200``) never imports it and has no CPU fallback.

The oracle is plain, slow and written from the pages' description of the
method, not from the GPU code; it shares no code with the CUDA path:

* ``attention``     paged single-query decode attention, fp64 (the plain definition:
                    gather each sequence's blocks, then softmax attention).
* ``cache_ops``     the cache write through a slot mapping, the block copy, and the
                    swap of whole blocks out to and back from a host buffer.
* ``block_manager`` the host block manager: free list, refcounts, fork, copy-on-write,
                    prefix caching (its own splitmix64 hash chain), the free list's order.
* ``utilisation``   the memory-utilisation estimate.
* ``c/``            the same attention and cache write in plain C (fp64
                    accumulation, OpenMP over (sequence, head)); the timed baseline.

Pins (in ``tests/test_oracle_*.py``): brute force on tiny inputs, closed forms
(one-token context, constant keys), library routine (torch's scaled-dot-product
attention in float64 on contiguous K/V), invariance under block placement,
GQA reducing to MHA with repeated KV heads, the log-sum-exp merge identity,
hand-worked allocator traces and utilisation values (``tests/golden/``); for prefix
caching (``tests/test_prefix_cache.py``) the published splitmix64 outputs, a
hand-worked trace and a check that every slot holds the K/V of its sequence's own
token prefix.
"""
