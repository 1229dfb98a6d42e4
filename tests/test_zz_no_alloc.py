"""The decode entry point that allocates nothing.  It serves callers that cannot call
cudaMalloc at decode time: engines that hold nearly all device memory in their own pools,
and decode loops that cannot pay for cudaMalloc's implicit device synchronisation.

Through the C ABI, its output must match the CPU oracle within the parity tolerance, on
two calls in a row that share the library's static working array.  The latents, bases and
query are buffers the caller owns, filled here straight from the generator (no cache).
"""
import numpy as np
import pytest

import synth
from tests import helpers as H

pytestmark = pytest.mark.gpu


def _caller_buffers(p):
    """Latents [B][T][r] and bases in the storage dtype, rounded by the generator."""
    zk = H.to_dev(p, p.store(np.asarray(p.z_k, np.float64)))
    zv = H.to_dev(p, p.store(np.asarray(p.z_v, np.float64)))
    return zk, zv, H.to_dev(p, p.B_k), H.to_dev(p, p.B_v)


def _decode(lib, p, zk, zv, bk, bv, q):
    import torch
    qd = H.to_dev(p, q)
    out = torch.empty_like(qd)
    lse = torch.empty((p.batch, p.n_q_heads), dtype=torch.float32, device="cuda")
    desc = H.desc_for(lib, p, capacity=p.hist_len)
    lib.lr_attn_decode_noalloc(desc, p.hist_len, zk, zv, bk, bv, qd, out, lse)
    torch.cuda.synchronize()
    return out.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("kind", ["tiny", "qwen4k"])
def test_noalloc_decode_matches_oracle(lib, kind):
    p = synth.small_variant(kind) if kind == "tiny" else synth.small_variant(kind, length=700, batch=2)
    zk, zv, bk, bv = _caller_buffers(p)
    queries = [p.q, p.store(H.stored_value(p, p.q) * H.sharp_factor(p))]
    for q in queries:                           # two calls in a row, different queries
        got, got_lse = _decode(lib, p, zk, zv, bk, bv, q)
        ref, ref_lse = H.oracle_decode(p, q)
        H.compare(p, got, ref, got_lse, ref_lse, tag=f"noalloc {kind}")


def test_noalloc_fewer_splits_when_the_array_is_too_small(lib):
    """Batch 16, 28 query heads, r = 256, 4096 tokens: the automatic split count (19)
    needs 9.2 MB of working memory, more than the array holds, so the call plans fewer
    splits.  Checked on two batch rows against the oracle, two calls in a row."""
    p = synth.small_variant("qwen4k", length=4096, batch=16)
    zk, zv, bk, bv = _caller_buffers(p)
    rows = [0, 15]
    for q in [p.q, p.store(H.stored_value(p, p.q) * H.sharp_factor(p))]:
        got, got_lse = _decode(lib, p, zk, zv, bk, bv, q)
        ref, ref_lse = H.oracle_decode(p, q, rows=rows)
        pairs = [(b, j) for b in rows for j in range(p.n_q_heads)]
        H.compare(p, got, ref, got_lse, ref_lse, pairs=pairs, tag="noalloc fewer splits")


def test_noalloc_sees_bases_written_just_before_the_call(lib):
    """The caller rewrites B_k and B_v on the stream right before the call; the decode
    must use the new bases."""
    import torch
    p = synth.small_variant("qwen4k", length=300, batch=2)
    zk, zv, bk, bv = _caller_buffers(p)
    p2 = synth.small_variant("qwen4k", length=300, batch=2, seed=7)     # other bases
    new_bk, new_bv = H.to_dev(p2, p2.B_k), H.to_dev(p2, p2.B_v)
    for _ in range(2):
        bk.zero_()
        bv.zero_()
        torch.cuda.synchronize()
        bk.copy_(new_bk)                         # same stream, immediately before
        bv.copy_(new_bv)
        got, got_lse = _decode(lib, p, zk, zv, bk, bv, p.q)
        pb = synth.dataclasses.replace(p, B_k=p2.B_k, B_v=p2.B_v)
        ref, ref_lse = H.oracle_decode(pb, p.q)
        H.compare(pb, got, ref, got_lse, ref_lse, tag="noalloc new bases")


def test_noalloc_rejects_oversized_work(lib):
    import torch
    p = synth.small_variant("qwen4k", length=64, batch=2)
    zk, zv, bk, bv = _caller_buffers(p)
    big = lib.make_desc(4096, 32, 8, 128, 256, 256, 128)     # 4 * 4096 * 32 * 514 B > 8 MiB
    q = torch.zeros((4096, 32, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(lib.LRError) as e:
        lib.lr_attn_decode_noalloc(big, 64, zk, zv, bk, bv, q, torch.empty_like(q))
    assert e.value.status == lib.LR_ERR_CAPACITY


def test_noalloc_rejects_unaligned_bases(lib):
    """Bases that do not start on a 16-byte boundary are refused before any launch."""
    import torch
    p = synth.small_variant("qwen4k", length=64, batch=2)
    zk, zv, bk, bv = _caller_buffers(p)
    desc = H.desc_for(lib, p, capacity=p.hist_len)
    qd = H.to_dev(p, p.q)
    flat = torch.empty(bk.numel() + 8, dtype=bk.dtype, device="cuda")
    shifted = flat[1:1 + bk.numel()].view_as(bk)             # 2 bytes past a 16-byte boundary
    launches = lib.lr_launch_count()
    for args in [(shifted, bv), (bk, shifted)]:
        with pytest.raises(lib.LRError) as e:
            lib.lr_attn_decode_noalloc(desc, p.hist_len, zk, zv, *args, qd, torch.empty_like(qd))
        assert e.value.status == lib.LR_ERR_INVALID_ARG
    assert lib.lr_launch_count() == launches
