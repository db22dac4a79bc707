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
