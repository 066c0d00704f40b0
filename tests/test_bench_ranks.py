"""Host logic of bench.py's multi-GPU path (independent replicas, one process
per GPU): timings combine as the maximum over ranks and throughput as the units
of all ranks over that time.  Run as two gloo ranks on CPU (no GPU)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    import sys
    import torch.distributed as dist
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r is slow on a different entry: the maxima come from different ranks
        local = [1.0 + rank, 10.0 - rank, 0.5 * (rank + 1)]
        got = bench.max_over_ranks(local, "cpu")
        out[rank] = got + [bench.replicas_throughput(1000.0, got[0], world)]
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_max_timings_and_job_throughput():
    ctx = mp.get_context("spawn")
    port = _free_port()
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        res = dict(out)
    assert res[0] == res[1]
    t0, e2e, dec, value = res[0]
    assert (t0, e2e, dec) == (2.0, 10.0, 1.0)
    # 1000 units per rank per step, 2 ranks, slowest step 2 ms -> 1e6 units/s
    assert value == pytest.approx(1000.0 * 2 / 2e-3)


def test_single_replica_throughput():
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    assert bench.replicas_throughput(500.0, 4.0, 1) == pytest.approx(125000.0)


def test_reference_arm_runs_on_rank_zero_only():
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_reference_arm_times_the_rotating_oracle_in_reconstruct_mode():
    """bench.py --impl reference --decode reconstruct times the oracle's
    reconstruct-then-attend (with the rotary base) on a bounded sample."""
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    from workloads import get_config
    value, ms, cores, sample = bench.cpu_oracle_steps(get_config("llama"), 1, 0, budget_s=1.0, rope_theta=500000.0)
    assert value > 0 and ms > 0 and cores >= 1
    assert "rotary base 500000" in sample
