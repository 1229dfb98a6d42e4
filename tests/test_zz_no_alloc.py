"""The decode entry point that allocates nothing (for callers that cannot call
cudaMalloc at decode time): through the C ABI, its output must match the regular
cache decode within the parity tolerance, on two calls in a row that share the
library's static working array."""
import numpy as np
import pytest

import synth
from tests import helpers as H

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("kind", ["tiny", "qwen4k"])
def test_noalloc_decode_matches_cache_decode(lib, kind):
    import torch
    p = synth.small_variant(kind) if kind == "tiny" else synth.small_variant(kind, length=700, batch=2)
    cache = H.fill_cache(lib, p)
    view = lib.lr_cache_view_get(cache)
    desc = H.desc_for(lib, p)
    queries = [p.q, p.store(H.stored_value(p, p.q) * H.sharp_factor(p))]
    for q in queries:                           # two calls in a row, different queries
        ref, ref_lse = H.gpu_decode(lib, p, cache, q)
        qd = H.to_dev(p, q)
        out = torch.empty_like(qd)
        lse = torch.empty((p.batch, p.n_q_heads), dtype=torch.float32, device="cuda")
        lib.lr_attn_decode_noalloc(desc, p.length, view.z_k, view.z_v, view.B_k, view.B_v, qd, out, lse)
        torch.cuda.synchronize()
        got = out.float().cpu().numpy().astype(np.float64)
        got_lse = lse.cpu().numpy().astype(np.float64)
        H.compare(p, got, ref, got_lse, ref_lse, tag=f"noalloc {kind}")


def test_noalloc_rejects_oversized_work(lib):
    import torch
    p = synth.small_variant("qwen4k", length=64, batch=2)
    cache = H.fill_cache(lib, p)
    view = lib.lr_cache_view_get(cache)
    big = lib.make_desc(4096, 32, 8, 128, 256, 256, 128)     # 4 * 4096 * 32 * 514 B > 8 MiB
    q = torch.zeros((4096, 32, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(lib.LRError) as e:
        lib.lr_attn_decode_noalloc(big, 64, view.z_k, view.z_v, view.B_k, view.B_v, q, torch.empty_like(q))
    assert e.value.status == lib.LR_ERR_CAPACITY
