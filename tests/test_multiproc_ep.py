"""The expert-parallel exchange (routed_expert_ffn_renorm_b200.ep.exchange)
on world-size-2 and -3 gloo process groups on CPU: variable-size row blocks
reach their ranks in source-rank order, several tensors travel with the same
split, zero-row blocks work, and sending the received rows back with the
received counts returns every rank its own rows in its send order -- the
round trip EPLayer.forward makes."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from routed_expert_ffn_renorm_b200.ep import exchange
        # rank r sends (r + d) % 3 rows to rank d (some blocks empty), row i of the block to d
        # holding the value 1000 r + 100 d + i
        counts = [(rank + d) % 3 for d in range(world)]
        rows = torch.cat([torch.tensor([[1000 * rank + 100 * d + i] * 4 for i in range(c)], dtype=torch.float32)
                          .reshape(c, 4) for d, c in enumerate(counts)])
        ids = rows[:, 0].to(torch.int32)
        recv_counts, (got, got_ids) = exchange(counts, [rows, ids])
        want = [(s + rank) % 3 for s in range(world)]
        assert recv_counts == want, (recv_counts, want)
        exp = [1000 * s + 100 * rank + i for s in range(world) for i in range(want[s])]
        assert got[:, 0].tolist() == exp and got_ids.tolist() == exp and (got == got[:, :1]).all()
        # and back: every rank gets its own rows, in its send order
        back_counts, (back,) = exchange(recv_counts, [got])
        assert back_counts == counts and torch.equal(back, rows)
        q.put((rank, "ok"))
    except Exception as e:  # reported to the parent
        q.put((rank, repr(e)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_exchange_round_trip(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
    assert all(v == "ok" for v in res.values()), res
