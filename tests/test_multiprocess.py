"""Host logic of the multi-rank bench on CPU: gloo process groups of two ranks.

The hot path shards by (batch, head) problem: every rank runs its own copy of
the workload with no collective on the data path, and the bench only uses the
process group for barriers and for the max-over-ranks timing.  These tests run
that plumbing with world size 2 on the CPU (no GPU), and the reference arm's
rank protocol under torchrun (rank 0 measures and prints, other ranks exit 0).
"""

import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    w, r, local = bench.dist_setup(world)
    assert (w, r, local) == (world, rank, rank)
    assert dist.get_backend() == "gloo"
    bench.barrier(w)
    slowest = bench.max_over_ranks(10.0 + rank, w)  # rank 1 is the slower one
    value = bench.aggregate_tokens_per_s(w, 1024, 4, slowest)
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump({"max": slowest, "value": value}, f)
    dist.destroy_process_group()


def test_two_rank_barrier_and_max_over_ranks(tmp_path):
    world, port = 2, _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    got = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for g in got:
        assert g["max"] == 11.0  # every rank sees the slowest rank's time
        # two replicas of 1024 tokens x 4 steps in 11 ms
        assert g["value"] == pytest.approx(2 * 1024 * 4 / 0.011)


def test_aggregate_is_weak_scaling():
    sys.path.insert(0, ROOT)
    import bench
    one = bench.aggregate_tokens_per_s(1, 4096, 10, 5.0)
    assert bench.aggregate_tokens_per_s(8, 4096, 10, 5.0) == pytest.approx(8 * one)
    # a slower rank lowers the whole job's figure
    assert bench.aggregate_tokens_per_s(2, 4096, 10, 10.0) == pytest.approx(one)


def test_reference_arm_under_torchrun_prints_once(tmp_path):
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes", "1", "--nproc-per-node",
           "2", "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2", "--steps", "1",
           "--warmup", "0", "--workload", "fwd_f32_L1024", "--ref-seconds", "1"]
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    res = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, res.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0


# ---------------------------------------------------------------------------
# one problem's heads split over the ranks (lsh_attention_long_b200.shard)
# ---------------------------------------------------------------------------

def test_head_ranges_cover_every_head_once():
    from lsh_attention_long_b200.shard import head_range
    for n in (0, 1, 7, 8, 16, 64, 65, 1000):
        for world in (1, 2, 3, 4, 8, 13):
            seen = []
            sizes = []
            for r in range(world):
                h0, h1 = head_range(n, world, r)
                assert 0 <= h0 <= h1 <= n
                seen += list(range(h0, h1))
                sizes.append(h1 - h0)
            assert seen == list(range(n))           # contiguous, in order, once each
            assert max(sizes) - min(sizes) <= 1      # balanced
    with pytest.raises(ValueError):
        head_range(8, 2, 2)


def _oracle_forward(q, v, rot, nb, chunk, causal):
    """The single-device forward for the CPU ranks: the fp64 oracle."""
    import torch
    from oracle import oracle as o
    f = o.lsh_forward(q.double().numpy(), v.double().numpy(), rot.double().numpy(), nb, chunk,
                      causal)
    return {"O": torch.from_numpy(f["O"]), "lse": torch.from_numpy(f["lse"]),
            "keys": torch.from_numpy(f["keys"].astype("int64")),
            "perm": torch.from_numpy(f["perm"].astype("int64"))}


def _shard_rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist
    from lsh_attention_long_b200 import workloads as W
    from lsh_attention_long_b200.shard import forward_sharded
    dist.init_process_group("gloo")
    inp = W.make_random(2, 3, 256, 64, 16, 2, torch.float32, seed=17)
    out = forward_sharded(inp["Q"], inp["V"], inp["rot"], 16, 64, True, world, rank,
                          forward=_oracle_forward, gather=True)
    torch.save({"O_full": out["O_full"], "lse_full": out["lse_full"], "O": out["O"]},
               os.path.join(out_dir, f"shard{rank}.pt"))
    dist.destroy_process_group()


def test_two_rank_head_shards_reassemble_the_one_rank_result(tmp_path, oracle):
    """B*H = 6 heads over two gloo ranks (3 each): every rank's slice is its
    heads' forward, and the all-gathered O and lse equal the one-rank result
    on all heads, bit for bit (the oracle is deterministic per head)."""
    import torch
    from lsh_attention_long_b200 import workloads as W
    world, port = 2, _free_port()
    mp.start_processes(_shard_rank_main, args=(world, port, str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    inp = W.make_random(2, 3, 256, 64, 16, 2, torch.float32, seed=17)
    ref = _oracle_forward(inp["Q"], inp["V"], inp["rot"], 16, 64, True)
    got = [torch.load(tmp_path / f"shard{r}.pt") for r in range(world)]
    for g in got:
        assert torch.equal(g["O_full"], ref["O"])
        assert torch.equal(g["lse_full"], ref["lse"])
    flat = ref["O"].reshape(1, 6, 256, 64)
    assert torch.equal(got[0]["O"], flat[:, 0:3])
    assert torch.equal(got[1]["O"], flat[:, 3:6])


def test_one_rank_gather_needs_no_process_group(oracle):
    """A world of one rank holds every head: the gather returns the forward's
    O and lse in [B, H, ...] shape without touching torch.distributed."""
    import torch
    import torch.distributed as dist
    from lsh_attention_long_b200 import workloads as W
    from lsh_attention_long_b200.shard import forward_sharded
    assert not dist.is_initialized()
    inp = W.make_random(2, 3, 256, 64, 16, 2, torch.float32, seed=17)
    out = forward_sharded(inp["Q"], inp["V"], inp["rot"], 16, 64, True, 1, 0,
                          forward=_oracle_forward, gather=True)
    ref = _oracle_forward(inp["Q"], inp["V"], inp["rot"], 16, 64, True)
    assert torch.equal(out["O_full"], ref["O"])
    assert torch.equal(out["lse_full"], ref["lse"])
