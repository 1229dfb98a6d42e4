"""CPU oracle for the low-rank KV-cache decode path — TEST INFRASTRUCTURE ONLY.

A plain, slow, fp64 NumPy restatement of what the path computes, used to check
the CUDA library.  Only the tests, `__graft_entry__.smoke()` and the CPU
baseline leg of `bench.py` may import it; the product path never does.  It
shares no code with the CUDA library (`rank_kv_cache_lr_b200/`) and imports
nothing from it.

Sources (the pages describe the method, not an implementation):
  * TraceKV: Policy-Preserving Low-Rank KV Cache Compression for Reasoning
    Vision-Language Models — abstract: the cache stores low-dimensional latents
    of the KV states, optionally combined with quantization; "optimized
    low-rank attention kernels" run decode on them.
  * iS-KV: Online Low-Rank KV Cache Compression via Block-Incremental SVD —
    abstract and method section: an exact recent window, older states folded
    into bounded-rank latents, and historical coordinates synchronized when
    the basis is updated.

Modules:
  quant      int4 group quantiser (asymmetric, group 32, fp16 scale/zero),
             nibble packing, exact dequantisation, bf16 storage rounding.
  attention  reconstruction K = Z B, rotate-half RoPE, textbook softmax
             attention, the decode definition over a stored cache.
  iskv       step simulator for the windowed cache: append with fold, basis
             sync, decode.
  svd        truncated SVD bases and the Eckart-Young error.
  incsvd     block-incremental SVD update of the basis, with the sync rotation.

Every function is pinned by a `-m "not gpu"` test against closed forms,
invariants, special cases or brute force (tests/test_oracle_pins.py).
"""

from . import attention, incsvd, iskv, quant, svd  # noqa: F401
