"""Worker of the two-rank host tests (started with the spawn method)."""
import json
import os


def rank_worker(rank: int, world: int, port: int, out_dir: str, rank_ms: list) -> None:
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch
    import torch.distributed as dist

    import bench
    bench.init_distributed(world, rank, backend="gloo")
    slowest = bench.max_over_ranks(rank_ms[rank], torch.device("cpu"))
    rate = bench.whole_job_rate(1000.0, 5, world, slowest)
    dist.barrier()
    dist.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump({"max_ms": slowest, "rate": rate}, f)
