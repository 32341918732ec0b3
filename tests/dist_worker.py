"""One rank of the two-rank CPU check of bench.py's replica plumbing (gloo).

Run under torch.distributed.run; writes rank_<r>.json into the directory given
as the only argument.  Checks, from inside each rank: the process group comes
up through bench.dist_init, max_over_ranks returns the largest value any rank
passed, every rank's replica batch differs while the layer weights agree.
"""
import hashlib
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import torch.distributed as dist  # noqa: E402

import bench  # noqa: E402
import synth  # noqa: E402


def digest(a) -> str:
    return hashlib.sha256(a.tobytes()).hexdigest()[:16]


def main(out_dir: str) -> int:
    rank, world = bench.dist_init("gloo")
    assert world == int(os.environ["WORLD_SIZE"]) and dist.is_initialized()
    bench.barrier()
    got = bench.max_over_ranks(10.0 + 3.5 * rank)
    prob = synth.make_problem(1, replica=rank)
    mine = {"x": digest(prob.x), "w": digest(prob.W_gate) + digest(prob.W_r)}
    every = [None] * world
    dist.all_gather_object(every, mine)
    bench.barrier()
    dist.destroy_process_group()
    with open(os.path.join(out_dir, "rank_%d.json" % rank), "w") as f:
        json.dump({"rank": rank, "world": world, "max": got, "all": every}, f)
    return 0


if __name__ == "__main__":
    sys.exit(main(sys.argv[1]))
