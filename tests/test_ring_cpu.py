"""Host-side tests of ring attention (context parallelism): the ring schedule,
and ring_attention itself over a ring of gloo ranks on the CPU with its
per-step attention + merge replaced by a recorder. The attention and merge
arithmetic run only in the CUDA kernels (tests/test_ring_gpu.py)."""
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


def _ring_worker(rank, world, port, causal, q):
    """Runs the shipped ring_attention on this gloo rank with the per-step
    attention + merge replaced by a recorder: the loop, the exchange, the
    landing buffers and the choice of the step that writes O are the product's
    own code."""
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import exact_attention_ring_b200.ring as ring
        calls = []

        def record(self, k, v, kind, out=None, stream=None):
            # the key/value shard this step holds is identified by its contents
            k0, v0 = float(k.flatten()[0]), float(v.flatten()[0])
            calls.append((k0, bool(torch.all(k == k0)), v0, bool(torch.all(v == v0)), kind, out is not None))

        ring._RankState.add = record
        qs = torch.zeros(2, 4, 5, 8, dtype=torch.bfloat16)
        k = torch.full((2, 2, 5, 8), float(rank), dtype=torch.bfloat16)
        v = torch.full((2, 2, 5, 8), 100.0 + rank, dtype=torch.bfloat16)
        o, lse = ring.ring_attention(qs, k, v, causal=causal)
        q.put((rank, calls, bool(torch.all(k == rank)), bool(torch.all(v == 100.0 + rank)),
               tuple(o.shape), tuple(lse.shape)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("causal", [False, True])
def test_ring_attention_steps_on_gloo_ranks(world, causal):
    """ring_attention itself, on a ring of gloo ranks: in step s every rank holds
    exactly the shard the schedule names (with its kind), the last step that is
    not skipped alone writes O, and the caller's K and V are left untouched."""
    ring_schedule, FULL, DIAG, SKIP = _schedule()
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    mp.start_processes(_ring_worker, args=(world, _free_port(), causal, q), nprocs=world, join=True,
                       start_method="spawn")
    results = sorted(q.get() for _ in range(world))
    assert [r[0] for r in results] == list(range(world))
    for rank, calls, k_intact, v_intact, o_shape, lse_shape in results:
        assert k_intact and v_intact
        assert o_shape == (2, 4, 5, 8) and lse_shape == (2, 4, 5)
        sched = ring_schedule(rank, world, causal)
        assert len(calls) == world
        for (k0, k_uni, v0, v_uni, kind, wrote), (src, skind) in zip(calls, sched):
            assert k_uni and v_uni
            assert (k0, v0, kind) == (float(src), 100.0 + src, skind)
        last = max(s for s, (_, kind) in enumerate(sched) if kind != SKIP)
        assert [wrote for *_, wrote in calls] == [s == last for s in range(world)]


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
