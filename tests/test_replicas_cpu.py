"""The multi-GPU form is replicas only: every rank runs its own layer and the
ranks exchange nothing but the timing, reduced to the slowest rank.  Here two
gloo ranks on the CPU run that reduction and the throughput formula."""
import json
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out_dir):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        my_ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        mx = bench.max_over_ranks(my_ms, world, "cpu")
        value = bench.job_throughput(world, 8, 20, mx)
        with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
            json.dump({"max": mx, "value": value}, f)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time(tmp_path):
    world, port = 2, _free_port()
    mp.spawn(_rank, args=(world, port, str(tmp_path)), nprocs=world, join=True)
    res = [json.load(open(tmp_path / f"r{r}.json")) for r in range(world)]
    for r in res:
        assert r["max"] == 15.0
        # 2 ranks x 8 tokens x 20 steps over 15 ms
        assert r["value"] == pytest.approx(2 * 8 * 20 / 0.015)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1, "cpu") == 3.5
    assert bench.job_throughput(1, 1, 50, 6.5) == pytest.approx(50 / 0.0065)


def _ref_run(env_extra):
    import subprocess
    env = dict(os.environ, **env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config",
                           "tiny", "--steps", "3", "--warmup", "3"], capture_output=True, text=True, env=env,
                          timeout=300)


def test_reference_arm_line():
    """The reference arm (the oracle on the host cores) prints the contract's
    line on rank 0: same metric and workload as the CUDA arm, K timed steps."""
    r = _ref_run({})
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["metric"] == "MoE-layer tokens/s"
    assert line["steps"] == 3 and line["warmup"] == 3 and line["higher_is_better"] is True
    assert line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
    assert line["config"]["workload"].startswith("tiny:")


def test_reference_arm_other_ranks_do_nothing():
    r = _ref_run({"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""
