"""The multi-process plumbing on CPU: world size 2 over gloo (no GPU, no data-path collective)."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import synth


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    from decoding_interleaved_rans_b200 import dist
    try:
        w, r, _ = dist.init("gloo", timeout_s=30)
        sizes = [t.numel for t in synth.WORKLOADS["llama2_7b"].tensors]
        mine = dist.shard_tensors(sizes, w, r)
        load = sum(sizes[i] for i in mine)
        dist.barrier()
        slowest = dist.max_over_ranks(1.0 + r)
        total = dist.sum_over_ranks(load)
        q.put((r, mine, load, slowest, total))
    finally:
        dist.shutdown()


def test_two_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    res = sorted(q.get(timeout=120) for _ in ps)
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    sizes = [t.numel for t in synth.WORKLOADS["llama2_7b"].tensors]
    (r0, m0, l0, s0, t0), (r1, m1, l1, s1, t1) = res
    assert sorted(m0 + m1) == list(range(len(sizes)))        # every tensor exactly once
    assert abs(l0 - l1) <= max(sizes)                          # balanced
    assert s0 == s1 == 2.0                                     # the slowest rank's time
    assert t0 == t1 == sum(sizes)


@pytest.mark.parametrize("world", [1, 3, 8])
def test_shard_plan_covers_everything(world):
    from decoding_interleaved_rans_b200 import dist
    sizes = [t.numel for t in synth.WORKLOADS["llama2_7b"].tensors]
    parts = [dist.shard_tensors(sizes, world, r) for r in range(world)]
    assert sorted(i for p in parts for i in p) == list(range(len(sizes)))
    loads = [sum(sizes[i] for i in p) for p in parts]
    assert max(loads) - min(loads) <= max(sizes)
    with pytest.raises(ValueError):
        dist.shard_tensors(sizes, world, world)
