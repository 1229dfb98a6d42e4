"""Decode over a batch whose rows hold different numbers of tokens (lr_attn_decode_varlen):
row b attends to its first row_len[b] history tokens.  Checked against the oracle run on each
row truncated to its own length, on every decode path, with lengths at the tile edges (1,
127, 128, 129) and the full length, so that some sequence splits of the short rows are
empty."""
import dataclasses

import numpy as np
import pytest

import synth
from tests import helpers as H

pytestmark = pytest.mark.gpu

LENGTHS = [1, 127, 128, 129, None]        # None: the full history


def _row_problem(p, b, n):
    return dataclasses.replace(p, batch=1, hist_len=n, z_k=p.z_k[b:b + 1, :n], z_v=p.z_v[b:b + 1, :n],
                               q=p.q[b:b + 1])


def _check(lib, p, c, lens, tag):
    import torch
    qd = H.to_dev(p, p.q)
    out = torch.empty_like(qd)
    lse = torch.empty((p.batch, p.n_q_heads), dtype=torch.float32, device="cuda")
    rl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    lib.lr_attn_decode_varlen(c, qd, out, rl, lse)
    torch.cuda.synchronize()
    got = out.float().cpu().numpy().astype(np.float64)
    got_lse = lse.cpu().numpy().astype(np.float64)
    tc_int4 = lib.lr_cache_plan(c).path == lib.LR_PATH_TC and p.quant_bits == 4
    for b, n in enumerate(lens):
        pb = _row_problem(p, b, n)
        ref, ref_lse = H.oracle_decode(pb)
        lse_tol = H.decode_lse_bound(pb, pb.q) if tc_int4 else None
        H.compare(pb, got[b:b + 1], ref, got_lse[b:b + 1], ref_lse, tag=f"{tag} row {b} len {n}", lse_tol=lse_tol)


CASES = [("tiny", None, 0), ("qwen4k", None, 0), ("qwen4k", "simt", 0), ("qwen4k", None, 9),
         ("qwen16k", None, 0), ("qwen16k", None, 7), ("qwen32k", None, 0)]


@pytest.mark.parametrize("kind,path,splits", CASES)
def test_varlen_rows_match_oracle(lib, kind, path, splits):
    full = 256 if kind == "tiny" else 600
    nb = len(LENGTHS)
    if kind == "tiny":
        base = synth.make_tiny()
        p = dataclasses.replace(base, batch=nb, z_k=np.repeat(base.z_k, nb, 0), z_v=np.repeat(base.z_v, nb, 0),
                                q=np.repeat(base.q, nb, 0))
    elif kind == "qwen32k":
        p = synth.small_variant("qwen32k", layer=11, batch=nb, length=full)
    else:
        p = synth.small_variant(kind, batch=nb, length=full)
    # distinct rows: each row's query scaled so the softmax is sharp
    p = dataclasses.replace(p, q=p.store(H.stored_value(p, p.q) * H.sharp_factor(p)))
    c = H.fill_cache(lib, p)
    if path == "simt":
        lib.lr_cache_set_path(c, lib.LR_PATH_SIMT, splits)
    elif splits:
        lib.lr_cache_set_path(c, lib.LR_PATH_AUTO, splits)
    lens = [n if n is not None else p.hist_len for n in LENGTHS]
    _check(lib, p, c, lens, f"varlen {kind} {path or 'auto'} splits={splits}")
    lib.lr_cache_destroy(c)


def test_varlen_clamps_out_of_range_lengths(lib):
    import torch
    p = synth.small_variant("qwen4k", batch=3, length=300)
    c = H.fill_cache(lib, p)
    qd = H.to_dev(p, p.q)
    outs = []
    for lens in ([0, p.hist_len + 50, -3], [1, p.hist_len, 1]):
        out = torch.empty_like(qd)
        lib.lr_attn_decode_varlen(c, qd, out, torch.tensor(lens, dtype=torch.int32, device="cuda"))
        torch.cuda.synchronize()
        outs.append(out.float().cpu().numpy())
    assert np.array_equal(outs[0], outs[1])
    lib.lr_cache_destroy(c)


def test_varlen_rejects_windowed_caches(lib):
    import torch
    p = synth.small_variant("hybrid", batch=2, hist_len=200)
    c = H.fill_cache(lib, p)
    qd = H.to_dev(p, p.q)
    with pytest.raises(lib.LRError) as e:
        lib.lr_attn_decode_varlen(c, qd, torch.empty_like(qd), torch.ones(2, dtype=torch.int32, device="cuda"))
    assert e.value.status == lib.LR_ERR_UNSUPPORTED
    lib.lr_cache_destroy(c)
