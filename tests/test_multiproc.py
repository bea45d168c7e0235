"""The bench's multi-rank logic on CPU with the gloo backend (world size 2): every
rank gets its own independent batch (weak scaling, no data-path collective), the
reported time is the max over ranks, and the reference arm prints only on rank 0."""
import os
import socket
import subprocess
import sys

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    from long_context_attention_fwd_b200 import inputs as I
    w = bench.rank_workload(I.workload(0), rank)
    x = I.make_inputs(w)
    t = bench.max_over_ranks([1.0 + rank, 10.0 - rank], torch.device("cpu"))
    q.put((rank, w.seed, int(x["q"][0, 0, 0]), t))
    dist.barrier()
    dist.destroy_process_group()


def test_two_ranks_independent_batches_and_max_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, s0, q0, t0), (r1, s1, q1, t1) = res
    assert s0 != s1 and q0 != q1          # each rank draws its own batch
    assert t0 == t1 == [2.0, 10.0]        # element-wise max over ranks


def test_reference_arm_prints_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""
