"""The multi-GPU benchmark path (independent replicas) as two gloo ranks on the CPU.

``bench.py --gpus N`` under torchrun runs N replicas of the stage, each on its
own batch, with no collective on the data path; timing is the maximum over
ranks, and the reference arm runs on rank 0 only. This exercises that logic
with world_size 2 over gloo: distinct per-rank batches, the max-over-ranks
reduction, and the rank-0-only reference line.
"""
import contextlib
import hashlib
import io
import json
import multiprocessing as mp
import os
import socket
import sys
from datetime import timedelta

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank: int, world: int, port: int, q):
    try:
        sys.path.insert(0, ROOT)
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                          WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
        import torch
        import torch.distributed as dist

        dist.init_process_group("gloo", rank=rank, world_size=world,
                                timeout=timedelta(seconds=60))
        import bench
        from dlrm_embedding_bag_b200 import synthetic as syn

        w = syn.CONFIGS["c2"].scaled(B=64, N=1000, name="c2_small")
        idx = syn.make_indices(w, replica=rank)
        digest = hashlib.sha256(idx.tobytes()).hexdigest()
        digests = [None] * world
        dist.all_gather_object(digests, digest)
        top = bench.max_over_ranks(1.5 + rank, world, torch.device("cpu"))
        args = bench.parse_args(["--gpus", str(world), "--steps", "2", "--warmup", "3",
                                 "--impl", "reference", "--config", "tiny"])
        out = io.StringIO()
        with contextlib.redirect_stdout(out):
            rc = bench.run_reference(args, syn.CONFIGS["tiny"])
        dist.barrier()
        dist.destroy_process_group()
        q.put((rank, digests, top, rc, out.getvalue()))
    except Exception as e:  # noqa: BLE001 - report to the parent
        q.put((rank, repr(e), None, None, None))


def test_two_gloo_replicas():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = {}
    for _ in procs:
        rank, digests, top, rc, text = q.get(timeout=240)
        results[rank] = (digests, top, rc, text)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank in (0, 1):
        digests, top, rc, text = results[rank]
        assert isinstance(digests, list), digests  # an exception string otherwise
        assert digests[0] != digests[1], "replicas must draw distinct batches"
        assert top == 2.5, "timing is the maximum over ranks"
        assert rc == 0
    assert results[1][3] == "", "only rank 0 runs and prints the reference arm"
    line = json.loads(results[0][3])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0
