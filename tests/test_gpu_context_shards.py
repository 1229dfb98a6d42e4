"""Context-sharded decode on one GPU: the context of every sequence is cut into consecutive
slices held by separate caches (one per GPU in a multi-GPU run); each cache's partial
(lr_attn_decode_partial) is stacked as an all-gather would deliver it and merged
(lr_merge_partials).  The result must match the oracle over the whole context, for bf16 and
int4 latents, uneven slices and one-token slices."""
import dataclasses

import numpy as np
import pytest

import synth
from tests import helpers as H

pytestmark = pytest.mark.gpu


def _slice(p, a, b):
    return dataclasses.replace(p, hist_len=b - a, z_k=p.z_k[:, a:b], z_v=p.z_v[:, a:b])


@pytest.mark.parametrize("kind,cuts", [("qwen4k", [0, 300, 700]), ("qwen16k", [0, 129, 130, 700]),
                                       ("tiny", [0, 1, 256]), ("qwen4k", [0, 128, 256, 384, 700])])
def test_sharded_partials_merge_to_the_whole_context(lib, kind, cuts):
    import torch
    p = synth.small_variant(kind, length=700, batch=2) if kind != "tiny" else synth.make_tiny()
    if kind == "tiny":
        cuts = [0, 1, p.hist_len]
    p = dataclasses.replace(p, q=p.store(H.stored_value(p, p.q) * H.sharp_factor(p)))
    caches = [H.fill_cache(lib, _slice(p, a, b), capacity=p.length + 8) for a, b in zip(cuts[:-1], cuts[1:])]
    qd = H.to_dev(p, p.q)
    rv = p.rank_v
    parts_o = torch.empty((len(caches), p.batch, p.n_q_heads, rv), dtype=torch.float32, device="cuda")
    parts_ml = torch.empty((len(caches), p.batch, p.n_q_heads, 2), dtype=torch.float32, device="cuda")
    for i, c in enumerate(caches):
        lib.lr_attn_decode_partial(c, qd, parts_o[i], parts_ml[i])
    out = torch.empty_like(qd)
    lse = torch.empty((p.batch, p.n_q_heads), dtype=torch.float32, device="cuda")
    lib.lr_merge_partials(caches[0], parts_o, parts_ml, out, lse)
    # shard order does not matter
    out2 = torch.empty_like(qd)
    lib.lr_merge_partials(caches[-1], parts_o.flip(0).contiguous(), parts_ml.flip(0).contiguous(), out2)
    torch.cuda.synchronize()
    ref, ref_lse = H.oracle_decode(p)
    got = out.float().cpu().numpy().astype(np.float64)
    tc_int4 = lib.lr_cache_plan(caches[0]).path == lib.LR_PATH_TC and p.quant_bits == 4
    H.compare(p, got, ref, lse.cpu().numpy().astype(np.float64), ref_lse, tag=f"shards {kind} {cuts}",
              lse_tol=H.decode_lse_bound(p, p.q) if tc_int4 else None)
    H.compare(p, out2.float().cpu().numpy().astype(np.float64), ref, tag=f"shards reversed {kind}")
    for c in caches:
        lib.lr_cache_destroy(c)


def test_sharding_refuses_windows_and_keys_before_rope(lib):
    import torch
    for p in (synth.small_variant("hybrid", batch=2, hist_len=200), synth.small_variant("qwen32k", batch=2, length=200)):
        c = H.fill_cache(lib, p)
        qd = H.to_dev(p, p.q)
        po = torch.empty((p.batch, p.n_q_heads, p.rank_v), dtype=torch.float32, device="cuda")
        pm = torch.empty((p.batch, p.n_q_heads, 2), dtype=torch.float32, device="cuda")
        with pytest.raises(lib.LRError) as e:
            lib.lr_attn_decode_partial(c, qd, po, pm)
        assert e.value.status == lib.LR_ERR_UNSUPPORTED
        lib.lr_cache_destroy(c)
