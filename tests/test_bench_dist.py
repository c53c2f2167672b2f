"""Multi-process (gloo, CPU) checks of bench.py's replica plumbing: whole-job
throughput is the sum of tokens over ranks divided by the max time over ranks;
the reference arm runs on rank 0 only."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    dist = bench.init_dist("gloo")
    tokens = 1000.0 * (rank + 1)
    secs = 0.5 + rank          # rank 1 is the slowest
    value, tmax = bench.aggregate_throughput(dist, tokens, secs, "cpu")
    out[rank] = (value, tmax)
    dist.barrier()
    dist.destroy_process_group()


def test_aggregate_over_two_gloo_ranks():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
    for r in range(world):
        value, tmax = out[r]
        assert tmax == pytest.approx(1.5)
        assert value == pytest.approx((1000.0 + 2000.0) / 1.5)


def _worker_shared(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    dist = bench.init_dist("gloo")
    # vocabulary-parallel: both ranks work on the same 8192 tokens
    value, tmax = bench.aggregate_shared_batch(dist, 8192.0, 0.25 + 0.25 * rank, "cpu")
    shard = bench.vocab_shard(256000, world, rank)
    out[rank] = (value, tmax, shard)
    dist.barrier()
    dist.destroy_process_group()


def test_vocab_parallel_aggregate_over_two_gloo_ranks():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker_shared, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
    shards = []
    for r in range(world):
        value, tmax, shard = out[r]
        assert tmax == pytest.approx(0.5)
        assert value == pytest.approx(8192.0 / 0.5)     # the shared batch is counted once
        shards.append(shard)
    assert shards[0][0] == 0 and shards[0][0] + shards[0][1] == shards[1][0]
    assert shards[1][0] + shards[1][1] == 256000


@pytest.mark.parametrize("V,world", [(256000, 8), (151936, 3), (4096 + 77, 2), (513, 3), (128256, 5)])
def test_vocab_shards_cover_the_vocabulary_in_whole_tiles(V, world):
    sys.path.insert(0, ROOT)
    import bench
    shards = [bench.vocab_shard(V, world, r) for r in range(world)]
    pos = 0
    for v0, n in shards:
        assert v0 == pos and n >= 0
        assert v0 % 256 == 0
        pos += n
    assert pos == V
    sizes = [-(-n // 256) for _, n in shards]
    assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1


def test_vocab_shards_need_a_tile_per_rank():
    sys.path.insert(0, ROOT)
    import bench
    with pytest.raises(ValueError):
        bench.vocab_shard(300, 4, 0)


def test_single_process_aggregate_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    v, t = bench.aggregate_throughput(None, 8192.0, 0.25, "cpu")
    assert v == pytest.approx(32768.0) and t == 0.25


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1"],
                       env=env, capture_output=True, text=True, timeout=120)
    assert p.returncode == 0
    assert p.stdout.strip() == ""


@pytest.mark.slow
def test_reference_arm_prints_one_json_line():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3", "--workload", "tiny"], env=env, capture_output=True, text=True,
                       timeout=300)
    assert p.returncode == 0, p.stderr
    lines = [l for l in p.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == "CCE fwd+bwd tokens/s" and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
