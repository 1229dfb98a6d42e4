"""Context-sharded decode over several GPUs: one process per GPU, each holding a contiguous
slice of the same sequences' context in its own cache (same bases, same query).

Per step, every rank computes the rank-space partial of its slice (lr_attn_decode_partial),
the partials are exchanged with one all-gather over the process group (NCCL over NVLink /
NVSwitch; B x Hq x (r_v + 2) fp32 per rank: 462 KB at batch 16, 28 heads, r_v = 256), and
every rank merges them by the log-sum-exp rule and projects once (lr_merge_partials).  The
arithmetic runs in the library's kernels; this module only moves the partials.
"""
from __future__ import annotations

from . import lr_attn_decode_partial, lr_merge_partials


def gather_partials(part_o, part_ml, group=None):
    """All-gather of the per-rank partials: [B][Hq][r_v] and [B][Hq][2] -> [n][...] in rank
    order on every rank."""
    import torch
    import torch.distributed as dist
    n = dist.get_world_size(group)
    all_o = torch.empty((n, *part_o.shape), dtype=part_o.dtype, device=part_o.device)
    all_ml = torch.empty((n, *part_ml.shape), dtype=part_ml.dtype, device=part_ml.device)
    dist.all_gather_into_tensor(all_o, part_o.contiguous(), group=group)
    dist.all_gather_into_tensor(all_ml, part_ml.contiguous(), group=group)
    return all_o, all_ml


def decode_context_sharded(cache, q, out, lse=None, group=None):
    """Attention of q over the whole sharded context, written to `out` (and `lse`) on every
    rank.  `cache` holds this rank's slice; every rank passes the same q."""
    import torch
    d = cache.desc
    rv = (d.latent_groups if d.latent_groups > 1 else 1) * d.rank_v
    part_o = torch.empty((d.batch, d.n_q_heads, rv), dtype=torch.float32, device=q.device)
    part_ml = torch.empty((d.batch, d.n_q_heads, 2), dtype=torch.float32, device=q.device)
    lr_attn_decode_partial(cache, q, part_o, part_ml)
    all_o, all_ml = gather_partials(part_o, part_ml, group)
    lr_merge_partials(cache, all_o, all_ml, out, lse)
