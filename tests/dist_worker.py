"""Body of one rank of the two-process gloo test (imported by the spawned children)."""
import os
from datetime import timedelta


def run(rank, world, port, queue):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import torch.distributed as dist

    import oracle
    from linear_attention_token_gdn_b200 import dist as gd
    from linear_attention_token_gdn_b200 import inputs

    dist.init_process_group("gloo", timeout=timedelta(seconds=60))
    try:
        r, w, local = gd.env_rank()
        local_time = 0.5 * (r + 1)                        # rank 1 is the slower one
        t = gd.max_over_ranks(local_time, w, device="cpu")
        gd.barrier(w, cuda=False)
        seed = gd.rank_seed(inputs.SEED_BASE, r)
        x = inputs.make_prefill(inputs.TINY, "cpu", seed=seed)      # this rank's own replica of the workload
        y, _ = oracle.recurrence(x["q"], x["k"], x["v"], x["g"], x["beta"], None, x["cu_seqlens"])
        queue.put({"rank": r, "world": w, "local": local, "t": t, "seed": seed, "y_sum": float(abs(y).sum()),
                   "value": gd.aggregate(64, w, t)})
    finally:
        dist.destroy_process_group()


def run_cp(rank, world, port, queue, segs):
    """One rank of a context-parallel prefill on CPU: its segment of each sequence, the maps
    formed by the oracle (fp64), the product's gather and fold over gloo, then the oracle run
    over the segment from the folded state."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import numpy as np
    import torch
    import torch.distributed as dist

    import oracle
    from linear_attention_token_gdn_b200 import cp
    from linear_attention_token_gdn_b200 import inputs

    dist.init_process_group("gloo", timeout=timedelta(seconds=60))
    try:
        x = inputs.make_prefill(inputs.TINY, "cpu", B=2, T=sum(segs), H=2, d=16, S0_std=0.05)
        T = sum(segs)
        a, b = sum(segs[:rank]), sum(segs[:rank + 1])
        idx = np.concatenate([np.arange(a, b), T + np.arange(a, b)])      # this rank's part of both sequences
        part = {n: x[n][idx] for n in ("q", "k", "v", "g", "beta")}
        cu = np.array([0, b - a, 2 * (b - a)], dtype=np.int32)
        eye = np.broadcast_to(np.eye(16), (2, 2, 16, 16)).copy()
        _, M = oracle.recurrence(part["q"], part["k"], np.zeros((len(idx), 2, 16)), part["g"], part["beta"], eye, cu)
        _, B = oracle.recurrence(part["q"], part["k"], part["v"], part["g"], part["beta"], None, cu)
        maps = cp.gather_maps(torch.from_numpy(M), torch.from_numpy(B))
        S0 = x["S0"].double()
        S = cp.fold_maps(maps, rank, S0, lambda M_, B_, S_: M_ @ S_ + B_)
        y, S_T = oracle.recurrence(part["q"], part["k"], part["v"], part["g"], part["beta"], S.numpy(), cu)
        queue.put({"rank": rank, "y": y, "S_T": S_T})
    finally:
        dist.destroy_process_group()
