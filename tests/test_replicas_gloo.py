"""The multi-GPU path of bench.py is replicas: every rank solves its own (b, h) problems and
the job's time is the slowest rank's.  Its host logic runs here as two gloo ranks on CPU."""
import datetime
import os
import socket
import subprocess
import sys

import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        sys.path.insert(0, ROOT)
        import bench
        from gated_delta_rule_107_b200.inputs import make_inputs
        step_ms = 2.0 + 3.0 * rank  # the second rank is the slow one
        slowest = bench.max_over_ranks(step_ms)
        x = make_inputs("gdn", "bf16", 1, 16, 2, 64, 64, seed=bench.replica_seed(1002, rank))
        q.put((rank, slowest, bench.weak_scaling_value(4096, world, slowest), float(x["q"].float().sum())))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_replicas_take_the_slowest_rank_and_draw_their_own_inputs():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(2))
    assert [g[1] for g in got] == [5.0, 5.0]                           # both ranks see the max
    assert all(abs(g[2] - 4096 * 2 / 5e-3) < 1e-6 for g in got)        # all units / slowest time
    assert got[0][3] != got[1][3]                                       # independent replicas


def test_max_over_ranks_without_a_process_group_is_the_value():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.25) == 3.25
    assert bench.weak_scaling_value(100, 1, 1000.0) == 100.0


def test_reference_arm_on_other_ranks_exits_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1"],
                       env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""
