"""Host-side tests of ring attention (context parallelism): the ring schedule
and the shard exchange over a ring of gloo ranks on the CPU. The attention
and merge arithmetic run only in the CUDA kernels (tests/test_ring_gpu.py)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _schedule():
    from exact_attention_ring_b200.ring import DIAG, FULL, SKIP, ring_schedule
    return ring_schedule, FULL, DIAG, SKIP


@pytest.mark.parametrize("world", [1, 2, 3, 4, 7])
@pytest.mark.parametrize("causal", [False, True])
def test_schedule_covers_each_block_once(world, causal):
    ring_schedule, FULL, DIAG, SKIP = _schedule()
    seen = {}
    for r in range(world):
        sched = ring_schedule(r, world, causal)
        assert len(sched) == world
        for s, (src, kind) in enumerate(sched):
            assert src == (r - s) % world  # shards move one rank on per step
            assert (r, src) not in seen
            seen[(r, src)] = kind
    assert len(seen) == world * world
    for (r, src), kind in seen.items():
        if not causal:
            assert kind == FULL
        else:
            # query shard r sees key shard src entirely if it lies earlier, its
            # own shard under the causal mask, and nothing of a later shard
            assert kind == (FULL if src < r else DIAG if src == r else SKIP)
    # step 0 is always the rank's own shard, never skipped
    assert all(ring_schedule(r, world, causal)[0] == (r, DIAG if causal else FULL) for r in range(world))


def test_schedule_rejects_bad_rank():
    ring_schedule, *_ = _schedule()
    with pytest.raises(ValueError):
        ring_schedule(3, 3, False)
    with pytest.raises(ValueError):
        ring_schedule(0, 0, True)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _exchange_worker(rank, world, port, causal, q):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from exact_attention_ring_b200.ring import ring_exchange, ring_schedule
        # this rank's "shards": tensors that identify their owner in every element
        k = torch.full((2, 3, 5, 4), float(rank))
        v = torch.full((2, 1, 5, 4), 100.0 + rank)
        landing = [(torch.empty_like(k), torch.empty_like(v)) for _ in range(min(2, world - 1))]
        cur, held = (k, v), []
        for s, (src, _) in enumerate(ring_schedule(rank, world, causal)):
            reqs = []
            if s + 1 < world:
                nxt = landing[s % 2]
                reqs = ring_exchange(list(cur), list(nxt))
            held.append((src, bool(torch.all(cur[0] == src)), bool(torch.all(cur[1] == 100.0 + src))))
            for r in reqs:
                r.wait()
            if s + 1 < world:
                cur = nxt
        q.put((rank, held, bool(torch.all(k == rank)), bool(torch.all(v == 100.0 + rank))))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_ring_exchange_moves_shards_around_the_ring(world):
    """Every rank holds, in step s, exactly the shard the schedule names; its own
    inputs are left untouched."""
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    mp.start_processes(_exchange_worker, args=(world, _free_port(), True, q), nprocs=world, join=True,
                       start_method="spawn")
    results = sorted(q.get() for _ in range(world))
    for rank, held, k_intact, v_intact in results:
        assert k_intact and v_intact
        assert [src for src, _, _ in held] == [(rank - s) % world for s in range(world)]
        assert all(kok and vok for _, kok, vok in held), held


def test_ring_compute_has_no_cpu_path():
    """The per-rank step refuses CPU tensors instead of computing on the host."""
    from exact_attention_ring_b200.ring import FULL, _RankState
    q = torch.zeros(1, 2, 8, 64, dtype=torch.bfloat16)
    st = _RankState.__new__(_RankState)
    st.q, st.scale, st.merged = q, 0.125, 0
    st.o_acc = torch.zeros(1, 2, 8, 64)
    st.lse = torch.zeros(1, 2, 8)
    st.o_blk = torch.zeros(1, 2, 8, 64, dtype=torch.bfloat16)
    st.lse_blk = torch.zeros(1, 2, 8)
    with pytest.raises(ValueError):
        st.add(q, q, FULL)
