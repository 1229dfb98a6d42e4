"""Failure paths that can be tested without faulting a GPU.

- Bounded waits: a cache whose wait limit is a few nanoseconds makes the tensor-core decode
  give up on its first wait that is not already satisfied.  The kernel must record
  LR_ERR_TIMEOUT, finish its own copies and MMAs, free its tensor memory and return; the next
  decode on the same cache (default limit) must match the oracle.  A kernel that kept its
  tensor memory would make that next decode stall in its allocation, so the check also
  covers the release.
- Host fault injection: the n-th device allocation of lr_cache_create fails (LR_ERR_OOM,
  nothing leaked), the n-th kernel launch of a decode fails (LR_ERR_CUDA, the cache stays
  usable), and a created-then-destroyed cache returns every byte.
"""
import numpy as np
import pytest

import synth
from tests import helpers as H

pytestmark = pytest.mark.gpu

CASES = [("qwen4k", {}), ("qwen16k", {}), ("qwen32k", {"layer": 11})]


def _problem(kind, kw):
    if kind == "qwen32k":
        return synth.small_variant("qwen32k", batch=2, length=300, **kw)
    return synth.small_variant(kind, length=700, batch=2, **kw)


@pytest.mark.parametrize("kind,kw", CASES, ids=[c[0] for c in CASES])
def test_wait_timeout_is_reported_and_the_cache_recovers(lib, kind, kw):
    p = _problem(kind, kw)
    c = H.fill_cache(lib, p)
    assert lib.lr_cache_plan(c).path == lib.LR_PATH_TC
    assert lib.lr_device_error(c) == 0
    lib.lr_cache_set_wait_limit(c, 4)                      # 4 ns: the first real wait gives up
    H.gpu_decode(lib, p, c)
    assert lib.lr_device_error(c) == lib.LR_ERR_TIMEOUT
    assert lib.lr_device_error(c) == 0                     # reading clears the word
    lib.lr_cache_set_wait_limit(c, 0)
    got, lse = H.gpu_decode(lib, p, c)
    assert lib.lr_device_error(c) == 0
    ref, ref_lse = H.oracle_decode(p)
    lse_tol = H.decode_lse_bound(p, p.q) if p.quant_bits == 4 else None
    H.compare(p, got, ref, lse, ref_lse, tag=f"after timeout {kind}", lse_tol=lse_tol)
    lib.lr_cache_destroy(c)


def _free_bytes():
    """Free device memory with torch's cached blocks returned (the test's own tensors
    would otherwise keep 2 MB blocks of the caching allocator)."""
    import torch
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return torch.cuda.mem_get_info()[0]


def test_allocation_faults_in_create_leak_nothing(lib):
    p = synth.small_variant("qwen16k", length=300, batch=2)
    args = [H.to_dev(p, x) for x in (p.A_k, p.B_k, p.A_v, p.B_v)]
    desc = H.desc_for(lib, p)
    base = _free_bytes()
    failures = 0
    for n in range(64):
        lib.lr_debug_inject_fault(lib.LR_FAULT_ALLOC, n)
        try:
            c = lib.lr_cache_create(desc, *args)
        except lib.LRError as e:
            assert e.status == lib.LR_ERR_OOM
            failures += 1
            assert _free_bytes() == base, f"allocation {n} failed and leaked"
            continue
        lib.lr_debug_inject_fault(lib.LR_FAULT_ALLOC, -1)
        # every allocation succeeded: the cache works and destroy returns everything
        assert failures == n and n > 5
        for s in range(0, p.hist_len, 128):
            import torch
            lib.lr_kv_append_latent(c, torch.from_numpy(np.ascontiguousarray(p.z_k[:, s:s + 128])).cuda(),
                                    torch.from_numpy(np.ascontiguousarray(p.z_v[:, s:s + 128])).cuda())
        got, lse = H.gpu_decode(lib, p, c)
        ref, ref_lse = H.oracle_decode(p)
        H.compare(p, got, ref, lse, ref_lse, tag="after allocation faults", lse_tol=H.decode_lse_bound(p, p.q))
        lib.lr_cache_destroy(c)
        assert _free_bytes() == base, "destroy did not return every byte"
        break
    else:
        pytest.fail("lr_cache_create never succeeded")
    lib.lr_debug_inject_fault(lib.LR_FAULT_ALLOC, -1)


@pytest.mark.parametrize("kind", ["qwen4k", "hybrid"])
def test_launch_faults_in_decode_report_and_recover(lib, kind):
    import torch
    p = synth.small_variant(kind, batch=2, length=500) if kind == "qwen4k" else synth.small_variant(kind, batch=2)
    c = H.fill_cache(lib, p)
    ref, ref_lse = H.oracle_decode(p)
    qd = H.to_dev(p, p.q)
    out = torch.empty_like(qd)
    seen = 0
    for n in range(16):
        lib.lr_debug_inject_fault(lib.LR_FAULT_LAUNCH, n)
        n0 = lib.lr_launch_count()
        try:
            lib.lr_attn_decode(c, qd, out)
        except lib.LRError as e:
            assert e.status == lib.LR_ERR_CUDA
            assert lib.lr_launch_count() - n0 == n          # the n launches before it went out
            seen += 1
            continue
        lib.lr_debug_inject_fault(lib.LR_FAULT_LAUNCH, -1)
        assert seen == n and n >= 2                         # a decode has at least 2 launches
        break
    torch.cuda.synchronize()
    lib.lr_debug_inject_fault(lib.LR_FAULT_LAUNCH, -1)
    got, lse = H.gpu_decode(lib, p, c)
    H.compare(p, got, ref, lse, ref_lse, tag=f"after launch faults {kind}")
    assert lib.lr_device_error(c) == 0
    lib.lr_cache_destroy(c)
