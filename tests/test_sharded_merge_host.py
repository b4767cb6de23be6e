"""The exchange step of a context-sharded pool, with two gloo ranks on the CPU.

Each rank owns a contiguous slice of the context.  It scores its slice and
keeps its own top-P (the oracle stands in for the kernels here: this test is
about the exchange).  One all-gather of (score, global position) pairs gives
every rank the union of the local pools; the top-P of that union is the
global pool, exactly, because a slice can contribute at most P members to the
global top-P and each of them is in that slice's own top-P under the same tie
rule.  Both ranks must end with the pool and top-K that the oracle computes
on the whole context."""
import os
import socket
import sys

import numpy as np
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(seed=7, ctx=20000, H=8, D=64, near=2750):
    """Random keys, with rows 9800..10199 (across the slice boundary at
    10000) set to copies of the row ranked `near` by score: 400 equal scores
    at the pool's threshold, which only the lower-position rule splits."""
    import oracle as O
    rng = np.random.default_rng(seed)
    keys = rng.integers(-16, 17, size=(ctx, D)).astype(np.int8)
    q = rng.integers(-16, 17, size=(H, D)).astype(np.int8)
    w = rng.integers(1, 9, size=H).astype(np.int8)
    s = O.index_scores(q, w, keys)
    keys[9800:10200] = keys[np.argsort(-s, kind="stable")[near]]
    return keys, q, w


def _rank_main(rank, world, port, P, K, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    import oracle as O
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        keys, q, w = _inputs()
        ctx = len(keys)
        lo, hi = ctx * rank // world, ctx * (rank + 1) // world
        s = O.index_scores(q, w, keys[lo:hi])
        local = O.top_k_positions(s, np.arange(lo, hi), P)            # global positions, ascending
        payload = torch.from_numpy(np.stack([s[local - lo], local]).astype(np.int64))   # [2][P]
        parts = [torch.empty_like(payload) for _ in range(world)]
        dist.all_gather(parts, payload)
        allp = torch.cat(parts, dim=1).numpy()
        pool = O.top_k_positions(allp[0], allp[1], P)
        sel = O.top_k_positions(allp[0], allp[1], K)
        out.put((rank, pool.tolist(), sel.tolist()))
    finally:
        dist.destroy_process_group()


def test_union_of_local_pools_gives_the_global_pool():
    import oracle as O
    P, K = 3000, 512
    ctx_ = mp.get_context("spawn")
    out = ctx_.Queue()
    port = _free_port()
    procs = [ctx_.Process(target=_rank_main, args=(r, 2, port, P, K, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    assert codes == [0, 0], codes
    res = sorted(out.get(timeout=10) for _ in range(2))
    keys, q, w = _inputs()
    _, ref_pool, ref_sel = O.full_index(q, w, keys, len(keys) - 1, P, K)
    for rank, pool, sel in res:
        assert pool == ref_pool.tolist(), f"rank {rank} pool"
        assert sel == ref_sel.tolist(), f"rank {rank} selection"
