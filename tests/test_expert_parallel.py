"""Host logic of expert parallelism (no GPU): the exchange plan, and the dispatch / return
exchange itself between two gloo ranks on CPU, with tagged rows standing for the dispatched
activations and a tag-transforming stand-in for the experts."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from sparse_moe_layer_softmax_b200 import expert_parallel as ep


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_expert_ranges():
    assert ep.expert_ranges(256, 8)[3] == (96, 128)
    assert ep.expert_ranges(16, 1) == [(0, 16)]
    with pytest.raises(ValueError):
        ep.expert_ranges(10, 4)


def test_send_counts_split_offsets_by_owner():
    offsets = np.array([0, 3, 3, 7, 9, 12, 12, 13, 20])  # 8 experts
    c = ep.send_counts(offsets, 2)
    assert c.tolist() == [[3, 0, 4, 2], [3, 0, 1, 7]]
    assert c.sum() == 20


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_regroup_rows_is_expert_major_permutation(seed):
    rng = np.random.default_rng(seed)
    world, n_local = 3, 5
    counts = rng.integers(0, 6, size=(world, n_local))
    rows, offs = ep.regroup_rows(counts)
    total = counts.sum()
    assert sorted(rows.tolist()) == list(range(total))          # a permutation
    assert offs[-1] == total and np.all(np.diff(offs) == counts.sum(0))
    # received buffer: source-major, then expert; tag each received row with (src, expert)
    tags = [(s, e) for s in range(world) for e in range(n_local) for _ in range(counts[s, e])]
    grouped = [tags[r] for r in rows]
    assert grouped == sorted(grouped, key=lambda se: (se[1], se[0]))  # expert-major, then source
    inv = ep.inverse_rows(rows)
    assert np.array_equal(rows[inv], np.arange(total))


def _exchange_worker(rank, world, port, n_experts, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        rng = np.random.default_rng(100 + rank)
        T, k = 40, 3
        # a rank's canonical dispatch: rows grouped by expert ascending, token ascending within
        experts = np.stack([rng.choice(n_experts, size=k, replace=False) for _ in range(T)])
        slots = sorted((int(experts[t, j]), t, j) for t in range(T) for j in range(k))
        offsets = np.searchsorted([e for e, _, _ in slots], np.arange(n_experts + 1))
        # row tag: (source rank, expert, token, slot)
        x_perm = torch.tensor([[rank, e, t, j] for e, t, j in slots], dtype=torch.int64)
        counts = ep.send_counts(offsets, world)
        exchange = ep.dist_exchange()
        recv_counts = ep.dist_exchange_counts(world)(counts, torch.device("cpu"))
        recv = exchange(x_perm, counts.sum(1), recv_counts.sum(1))
        lo, hi = ep.expert_ranges(n_experts, world)[rank]
        rows, offs = ep.regroup_rows(recv_counts)
        grouped = recv.index_select(0, torch.from_numpy(rows).long())
        # the owner sees exactly its experts, grouped by expert, then source rank, then token
        g = grouped.numpy()
        ok_range = bool(np.all((g[:, 1] >= lo) & (g[:, 1] < hi)))
        ok_order = bool(np.all(np.diff(g[:, 1] * 1_000_000 + g[:, 0] * 1000 + g[:, 2]) > 0))
        ok_offs = [int(x) for x in offs] == [int(np.searchsorted(g[:, 1], lo + e))
                                             for e in range(hi - lo)] + [len(g)]
        # stand-in experts: mark the row as processed by this owner
        done = grouped.clone()
        done[:, 3] += 100 * (rank + 1)
        back = done.index_select(0, torch.from_numpy(ep.inverse_rows(rows)).long())
        returned = exchange(back, recv_counts.sum(1), counts.sum(1))
        r = returned.numpy()
        # every row came back to its source in canonical order, processed by its expert's owner
        owner = np.searchsorted([h for _, h in ep.expert_ranges(n_experts, world)], r[:, 1],
                                side="right")
        ok_back = bool(np.array_equal(r[:, :3], x_perm.numpy()[:, :3]) and
                       np.array_equal(r[:, 3] - 100 * (owner + 1), x_perm.numpy()[:, 3]))
        out[rank] = (ok_range, ok_order, ok_offs, ok_back, int(len(g)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_dispatch_and_return_over_gloo(world):
    n_experts = 12
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_exchange_worker, args=(world, _free_port(), n_experts, out), nprocs=world,
                 join=True)
        res = dict(out)
    assert sorted(res) == list(range(world))
    for rank, (ok_range, ok_order, ok_offs, ok_back, n) in res.items():
        assert ok_range and ok_order and ok_offs and ok_back, (rank, res[rank])
    assert sum(v[4] for v in res.values()) == world * 40 * 3  # every dispatched row exchanged
