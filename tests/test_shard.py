"""Head sharding of one layer (host logic, CPU): the head blocks partition the heads, and two gloo
ranks that each run the oracle on their own block and all-gather the outputs and final states get
exactly the oracle's whole-layer result.  Heads never interact, so sharding changes no value."""
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from linear_attention_10_b200.shard import gather_heads, head_range, shard_heads
from linear_attention_10_b200.workloads import make_prefill_inputs


@pytest.mark.parametrize("H,world", [(32, 2), (32, 4), (32, 8), (5, 2), (7, 3), (3, 3), (1, 1)])
def test_head_blocks_partition_the_heads(H, world):
    blocks = [head_range(r, world, H) for r in range(world)]
    assert blocks[0][0] == 0 and blocks[-1][1] == H
    for (a0, a1), (b0, b1) in zip(blocks, blocks[1:]):
        assert a1 == b0 and a1 > a0
    sizes = [b - a for a, b in blocks]
    assert max(sizes) - min(sizes) <= 1


def test_head_range_rejects_bad_arguments():
    with pytest.raises(ValueError):
        head_range(2, 2, 32)
    with pytest.raises(ValueError):
        head_range(0, 4, 3)


def test_shard_heads_slices_every_head_axis():
    inp = make_prefill_inputs([20, 9], H=6, dk=16, dv=8, dtype="fp32", seed=3, state_std=0.05)
    part = shard_heads(inp, 1, 2)
    assert part["cu_seqlens"] is inp["cu_seqlens"]
    for n in ("q", "k", "v", "g", "beta", "state_in"):
        assert part[n].is_contiguous()
        assert torch.equal(part[n], inp[n][:, 3:6])


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_main(rank, world, port, q):
    import torch.distributed as dist

    import oracle
    dist.init_process_group("gloo", init_method="tcp://127.0.0.1:%d" % port, rank=rank, world_size=world)
    try:
        inp = make_prefill_inputs([40, 25], H=4, dk=16, dv=8, dtype="fp32", seed=11, state_std=0.05)
        mine = shard_heads(inp, rank, world)
        f = lambda t: t.numpy().astype(np.float64)
        o, s = oracle.recurrence(f(mine["q"]), f(mine["k"]), f(mine["v"]), f(mine["g"]), f(mine["beta"]),
                                 cu_seqlens=inp["cu_seqlens"].numpy(), state_in=f(mine["state_in"]))
        o_all = gather_heads(torch.from_numpy(np.ascontiguousarray(o)), world)
        s_all = gather_heads(torch.from_numpy(np.ascontiguousarray(s)), world)
        q.put((rank, o_all.numpy(), s_all.numpy()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_gather_the_whole_layer():
    import oracle
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=180) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    inp = make_prefill_inputs([40, 25], H=4, dk=16, dv=8, dtype="fp32", seed=11, state_std=0.05)
    f = lambda t: t.numpy().astype(np.float64)
    o_ref, s_ref = oracle.recurrence(f(inp["q"]), f(inp["k"]), f(inp["v"]), f(inp["g"]), f(inp["beta"]),
                                     cu_seqlens=inp["cu_seqlens"].numpy(), state_in=f(inp["state_in"]))
    for _, o_all, s_all in res:
        assert np.array_equal(o_all, o_ref) and np.array_equal(s_all, s_ref)


def _uneven_rank_main(rank, world, port, q):
    import torch.distributed as dist
    dist.init_process_group("gloo", init_method="tcp://127.0.0.1:%d" % port, rank=rank, world_size=world)
    try:
        h0, h1 = head_range(rank, world, 3)          # 2 heads on rank 0, 1 on rank 1
        local = torch.full((5, h1 - h0, 4), float(rank))
        try:
            gather_heads(local, world)
            q.put((rank, "gathered"))
        except ValueError as e:
            q.put((rank, "ValueError: %s" % e))
    finally:
        dist.destroy_process_group()


def test_gather_heads_refuses_unequal_blocks_on_every_rank():
    """3 heads over 2 ranks: both ranks raise ValueError before the data all-gather (none hangs)."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_uneven_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert sorted(res) == [0, 1]
    for r in (0, 1):
        assert res[r].startswith("ValueError") and "equal head blocks" in res[r], res[r]
