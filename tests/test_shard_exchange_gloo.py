"""The exchange step of the context-sharded decode on the CPU, with two gloo ranks: the
all-gather delivers every rank's partials in rank order, and merging per-slice softmax
results by the log-sum-exp rule (the rule lr_merge_partials applies) reproduces the oracle's
attention over the whole context."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _gather(part_o, part_ml, group=None):
    """The exchange of rank_kv_cache_lr_b200.sharded, restated for CPU tensors (that module
    imports the CUDA library, which a CPU test cannot load)."""
    import torch
    import torch.distributed as dist
    n = dist.get_world_size(group)
    all_o = [torch.empty_like(part_o) for _ in range(n)]
    all_ml = [torch.empty_like(part_ml) for _ in range(n)]
    dist.all_gather(all_o, part_o, group=group)
    dist.all_gather(all_ml, part_ml, group=group)
    return torch.stack(all_o), torch.stack(all_ml)


def _rank_main(rank, world, port, q):
    import sys
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import synth
    from oracle import attention
    from tests import helpers as H
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        p = synth.small_variant("qwen4k", length=600, batch=2)
        cuts = [0, 250, 600]
        a, b = cuts[rank], cuts[rank + 1]
        qv = H.stored_value(p, p.q)
        Zk = H.oracle_latents(p, p.z_k.reshape(-1, p.rank_k)).reshape(p.z_k.shape)[:, a:b]
        Zv = H.oracle_latents(p, p.z_v.reshape(-1, p.rank_v)).reshape(p.z_v.shape)[:, a:b]
        o, lse = attention.decode(qv, Zk, Zv, H.stored_value(p, p.B_k), H.stored_value(p, p.B_v), p.n_kv_heads)
        all_o, all_l = _gather(torch.from_numpy(o), torch.from_numpy(lse))
        assert torch.equal(all_o[rank], torch.from_numpy(o))     # rank order kept
        lse_t = torch.logsumexp(all_l, dim=0)
        w = torch.exp(all_l - lse_t)                             # weight of each slice
        merged = (w[..., None] * all_o).sum(0).numpy()
        q.put((rank, merged, lse_t.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_two_rank_exchange_and_merge_rule():
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import synth
    from tests import helpers as H
    world = 2
    ctx = mp.get_context("spawn")
    qu = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, qu)) for r in range(world)]
    for pr in procs:
        pr.start()
    res = sorted(qu.get(timeout=150) for _ in range(world))
    for pr in procs:
        pr.join(60)
    assert all(pr.exitcode == 0 for pr in procs)
    p = synth.small_variant("qwen4k", length=600, batch=2)
    ref, ref_lse = H.oracle_decode(p)
    for _, merged, lse in res:
        assert np.max(np.abs(merged - ref)) <= 1e-12 * max(1.0, np.max(np.abs(ref)))
        assert np.max(np.abs(lse - ref_lse)) <= 1e-12
