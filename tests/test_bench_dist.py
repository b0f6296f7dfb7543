"""Multi-rank host logic of bench.py on CPU (gloo, world size 2): the time used
for the job is the slowest rank's, and the value counts every rank's bytes."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        w, r, local = bench.dist_env()
        ms = 1.0 + rank                      # rank 1 is slower
        ms_max = bench.max_over_ranks(ms)
        value = bench.aggregate_gbs(1_000_000_000, w, ms_max / 1e3)
        q.put((r, w, local, ms_max, value))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_aggregate_two_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, (r, w, local, ms_max, value) in enumerate(res):
        assert (r, w, local) == (rank, 2, rank)
        assert ms_max == pytest.approx(2.0)              # slowest rank
        assert value == pytest.approx(2 * 1e9 / 2e-3 / 1e9)  # both ranks' bytes / slowest time


def test_single_process_identity():
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.aggregate_gbs(10**9, 1, 1.0) == pytest.approx(1.0)


def test_reference_arm_other_ranks_exit_without_work(monkeypatch, capsys):
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.main(["--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"]) == 0
    assert capsys.readouterr().out == ""


def test_reference_arm_json_line(capsys):
    """The reference arm (the fp64 oracle on the host cores) prints one JSON line
    with the bench keys, its own cpu_baseline and an e2e with no copies."""
    import json
    import bench
    assert bench.main(["--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "3"]) == 0
    lines = [l for l in capsys.readouterr().out.splitlines() if l.strip()]
    assert len(lines) == 1
    j = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in j, key
    assert j["impl"] == "reference" and j["n_gpus"] == 1 and j["steps"] == 1 and j["warmup"] == 3
    assert j["config"]["workload"] == "tiny" and j["dtype"] == "f64" and j["higher_is_better"] is True
    assert j["value"] > 0 and j["ms_per_step"] > 0
    cb = j["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == j["value"]
    e2e = j["e2e"]
    assert e2e["value"] == j["value"] and e2e["unit"] == j["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_strong_scaling_shards_partition_the_job():
    """--scaling strong: the ranks' (batch, head) ranges cover every (b, h) of
    the job exactly once, on whole head groups, for every supported GPU count."""
    import bench
    for B, H, G in [(2, 70, 4), (2, 36, 4), (1, 18, 2), (4, 9, 4), (1, 70, 4)]:
        groups = -(-H // G)
        for world in (1, 2, 4, 8):
            if not (B % world == 0 or (world % B == 0 and groups >= world // B)):
                with pytest.raises(ValueError):
                    bench.shard(world, 0, B, H, G)
                continue
            seen = {}
            for r in range(world):
                b0, b1, h0, h1 = bench.shard(world, r, B, H, G)
                assert 0 <= b0 < b1 <= B and 0 <= h0 < h1 <= H
                assert h0 % G == 0 and (h1 % G == 0 or h1 == H)
                for b in range(b0, b1):
                    for h in range(h0, h1):
                        assert (b, h) not in seen
                        seen[(b, h)] = r
            assert len(seen) == B * H
    # the 4096px job over 8 GPUs: a batch per four ranks, head groups 4 / 5 / 4 / 5
    assert [bench.shard(8, r, 2, 70, 4) for r in range(4)] == [
        (0, 1, 0, 16), (0, 1, 16, 36), (0, 1, 36, 52), (0, 1, 52, 70)]
    with pytest.raises(ValueError):
        bench.shard(3, 0, 2, 70, 4)


def test_strong_scaling_flag_parses():
    import bench
    assert bench.parse_args(["--scaling", "strong", "--gpus", "4"]).scaling == "strong"
    assert bench.parse_args([]).scaling == "weak"


def test_strong_scaling_rank_workloads_sum_to_the_job():
    import bench
    from linear_attention_diffusion_relu_b200.workloads import WORKLOADS
    job = WORKLOADS["4096px"]
    for world in (2, 4, 8):
        parts = [bench.rank_workload(job, world, r, "strong") for r in range(world)]
        assert sum(w.algorithmic_bytes(2) for w, _ in parts) == job.algorithmic_bytes(2)
        assert all(w.N == job.N and w.d == job.d and w.name != job.name for w, _ in parts)
    w, part = bench.rank_workload(job, 8, 1, "strong")
    assert (w.B, w.H, part) == (1, 20, (0, 1, 16, 36))
    assert bench.rank_workload(job, 8, 1, "weak") == (job, None)
    assert bench.rank_workload(job, 1, 0, "strong") == (job, None)
