"""bench.py's multi-rank timing on CPU: world size 2 over gloo.

Under torchrun each rank runs an independent replica of the workload (the
path shards by replica, with no collective on the data path); the reported
time is the slowest rank's, which every rank must agree on.
"""
import os
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks(1.5 + 2.0 * rank, world, torch.device("cpu"))
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(90)
    assert all(p.exitcode == 0 for p in procs)
    got = dict(q.get(timeout=5) for _ in range(2))
    assert got == {0: 3.5, 1: 3.5}


def test_max_over_ranks_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(2.25, 1, torch.device("cpu")) == 2.25


def test_layer_count_puts_the_kv_caches_past_l2():
    """bench.py steps NL layers with their own KV caches so that the caches
    together exceed twice the L2 (at least 2, at most 8 layers)."""
    sys.path.insert(0, ROOT)
    import bench
    from block_diffusion_attention_flashblock_b200 import workloads as wl
    for name, spec in wl.SPECS.items():
        nl = bench.n_layers(spec)
        kv = 2 * spec.B * spec.Hkv * spec.lcap * spec.D * (4 if spec.dtype == "f32" else 2)
        assert 2 <= nl <= 8, name
        assert nl == 8 or nl * kv >= 2 * bench.L2_BYTES, name
    assert bench.n_layers(wl.get_spec("dllm_8k")) == 8
    assert bench.n_layers(wl.get_spec("dllm_64k_b4")) == 2
