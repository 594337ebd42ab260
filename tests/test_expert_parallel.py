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


class _TaggedRank:
    """A CPU stand-in for ExpertParallelRank with the same dispatch / compute / finish contract:
    rows are integer tags (source rank, expert, token, slot) and an expert marks the rows it
    processes, so forward()'s exchanges can be checked row by row on gloo ranks."""

    def __init__(self, rank, world, n_experts, T, k):
        self.rank, self.world, self.n, self.T, self.k = rank, world, n_experts, T, k
        self.lo, self.hi = ep.expert_ranges(n_experts, world)[rank]

    def dispatch(self, u):
        rng = np.random.default_rng(200 + self.rank)
        experts = np.stack([rng.choice(self.n, size=self.k, replace=False) for _ in range(self.T)])
        slots = sorted((int(experts[t, j]), t, j) for t in range(self.T) for j in range(self.k))
        offsets = np.searchsorted([e for e, _, _ in slots], np.arange(self.n + 1))
        x_perm = torch.tensor([[self.rank, e, t, j] for e, t, j in slots], dtype=torch.int64)
        return ep.Dispatched(u=u, w=None, inv=None, x_perm=x_perm,
                             counts=ep.send_counts(offsets, self.world))

    def compute(self, recv, recv_counts):
        rows, offs = ep.regroup_rows(recv_counts)
        grouped = recv.index_select(0, torch.from_numpy(rows).long())
        for e in range(self.hi - self.lo):  # expert lo + e marks its rows
            seg = grouped[offs[e]:offs[e + 1]]
            assert bool((seg[:, 1] == self.lo + e).all())
            seg[:, 3] += 100 * (self.lo + e + 1)
        return grouped.index_select(0, torch.from_numpy(ep.inverse_rows(rows)).long())

    def recv_buffer(self, rows):  # the rank's own buffers for the two exchanges
        return torch.full((rows, 4), -1, dtype=torch.int64)

    def return_buffer(self, rows):
        return torch.full((rows, 4), -1, dtype=torch.int64)

    def finish(self, d, out_perm, out=None):
        return d.x_perm, out_perm


def _forward_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r = _TaggedRank(rank, world, n_experts=8, T=24, k=2)
        sent, back = ep.forward(r, torch.zeros(24, 1), ep.dist_exchange(),
                                ep.dist_exchange_counts(world))
        s, b = sent.numpy(), back.numpy()
        out[rank] = bool(np.array_equal(s[:, :3], b[:, :3]) and
                         np.array_equal(b[:, 3] - 100 * (s[:, 1] + 1), s[:, 3]))
    finally:
        dist.destroy_process_group()


def test_forward_orchestration_over_gloo():
    """expert_parallel.forward itself (counts exchange, dispatch, owner compute, return) between
    two gloo ranks: every dispatched row comes back in its canonical place, processed once by the
    expert it was routed to."""
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_forward_worker, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    assert res == {0: True, 1: True}
