"""Host-side logic of bench.py on CPU: the max-over-ranks aggregation with
two gloo ranks, and the oracle reference arm's JSON line."""
import json
import os
import socket
import subprocess
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    value, t_max = bench.aggregate(10, 100.0 * (rank + 1), world)
    q.put((rank, value, t_max))
    dist.barrier()
    dist.destroy_process_group()


def test_aggregate_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # 2 ranks x 10 steps over the slowest rank's 200 ms
    for _, value, t_max in got:
        assert t_max == 200.0
        assert abs(value - 100.0) < 1e-9


def _run_bench(args, env_extra=None):
    env = dict(os.environ)
    env.update(env_extra or {})
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True,
                       text=True, env=env, timeout=600)
    assert r.returncode == 0, r.stderr
    return r.stdout


def test_reference_arm_json_line():
    out = _run_bench(["--impl", "reference", "--steps", "3", "--warmup", "3", "--workload", "tiny_f32",
                      "--ref-budget", "1"])
    line = json.loads(out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "iter/s" and line["higher_is_better"]
    assert line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
    assert line["config"]["workload"] == "tiny_f32"


def test_reference_arm_out_of_core_uses_the_reduced_rows():
    out = _run_bench(["--impl", "reference", "--steps", "3", "--warmup", "3", "--workload", "ooc_f16",
                      "--ref-budget", "1", "--ooc-rows", str(1 << 20)])
    line = json.loads(out.strip().splitlines()[-1])
    cfg = line["config"]
    assert cfg["workload"] == "ooc_f16" and cfg["N"] == 1 << 20 and cfg["K"] == 8192 and cfg["D"] == 128
    assert line["impl"] == "reference" and line["value"] > 0


def test_reference_arm_only_rank0_prints():
    out = _run_bench(["--impl", "reference", "--steps", "3", "--warmup", "3", "--workload", "tiny_f32",
                      "--ref-budget", "1"], {"RANK": "1", "WORLD_SIZE": "2"})
    assert out.strip() == ""
