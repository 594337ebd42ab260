"""Expert parallelism for the MoE layer: one process per GPU, each rank holding n_experts / R of
the experts (a contiguous range) and its own tokens.

Per forward, on every rank:
  1. route, then the dispatch permutation of the rank's own tokens (moe_route, moe_permute);
     its per-expert offsets go to pinned host memory by an asynchronous copy that overlaps the
     latent down-projection (moe_latent_down), and the rows are dispatched (moe_dispatch_rows).
     The dispatched rows come out grouped by expert, hence by the rank that owns each expert;
  2. exchange: the rows for owner rank d are sent to d (all-to-all), with the per-expert counts;
  3. on the owner: the received rows, ordered (source rank, expert, token), are regrouped by
     expert (moe_gather_rows), the rank's experts run on them (moe_expert_ffn), and the outputs
     are put back in received order (moe_gather_rows);
  4. exchange back: every row returns to the rank it came from, in the order it was sent, which is
     the canonical dispatch order there; then combine and latent up-projection (moe_combine,
     moe_latent_up).

The exchange is a callable, so that the same stages run over torch.distributed
(all_to_all_single: NCCL between GPUs, gloo between CPU processes) or with all ranks emulated in
one process.  Every arithmetic step is one of the library's kernels; this module only plans the
exchange (integer bookkeeping on the host) and moves rows.  A rank keeps its buffers between
forwards (the ones whose size depends on the rows received grow when a forward needs more), so a
steady stream of forwards allocates nothing; the host reads the expert counts once per forward,
while the latent down-projection runs.
"""
from __future__ import annotations

import dataclasses

import numpy as np

from . import (Config, moe_combine, moe_dispatch_rows, moe_expert_ffn, moe_gather_rows,
               moe_latent_down, moe_latent_up, moe_permute, moe_route, workspace_size, MOE_BF16)


# ---------------------------------------------------------------- exchange plan (host integers)

def expert_ranges(n_experts: int, world: int) -> list[tuple[int, int]]:
    """The contiguous expert range [lo, hi) owned by each rank."""
    if world <= 0 or n_experts % world:
        raise ValueError(f"{n_experts} experts do not split evenly over {world} ranks")
    per = n_experts // world
    return [(r * per, (r + 1) * per) for r in range(world)]


def send_counts(offsets: np.ndarray, world: int) -> np.ndarray:
    """Rows of a rank's dispatch (expert offsets [n+1], canonical order) for each owner rank:
    [world, n_local] counts per (owner, local expert)."""
    n = len(offsets) - 1
    counts = np.diff(np.asarray(offsets, dtype=np.int64))
    return counts.reshape(world, n // world)


def regroup_rows(recv_counts: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Plan of the owner's regrouping.  recv_counts [world_src, n_local]: rows received from each
    source rank for each local expert; the received buffer holds them source-major, then expert.
    Returns (rows, local_offsets): grouped row g (expert-major, then source) is received row
    rows[g]; local_offsets [n_local + 1] are the experts' row offsets in the grouped order."""
    recv_counts = np.asarray(recv_counts, dtype=np.int64)
    world, n_local = recv_counts.shape
    flat = recv_counts.reshape(-1)
    # received index of each (source, expert) block, then the blocks in (expert, source) order
    starts = (np.cumsum(flat) - flat).reshape(world, n_local).T.reshape(-1)
    lens = recv_counts.T.reshape(-1)
    total = int(lens.sum())
    grouped_starts = np.cumsum(lens) - lens
    rows = (np.repeat(starts - grouped_starts, lens) + np.arange(total)).astype(np.int32)
    local_offsets = np.concatenate([[0], np.cumsum(recv_counts.sum(0))]).astype(np.int64)
    return rows, local_offsets


def inverse_rows(rows: np.ndarray) -> np.ndarray:
    """inv with inv[rows[g]] = g: gathering the grouped outputs by inv restores received order."""
    inv = np.empty_like(rows)
    inv[rows] = np.arange(len(rows), dtype=rows.dtype)
    return inv


# ---------------------------------------------------------------- exchange over torch.distributed

def dist_exchange(group=None):
    """An exchange callable over torch.distributed: exchange(send, send_splits, recv_splits, out)
    sends rows send[sum(send_splits[:d]) : ...] to rank d and returns the rows received, ordered by
    source rank, in `out` (a buffer of exactly sum(recv_splits) rows) or a new tensor."""
    import torch
    import torch.distributed as dist

    def exchange(send, send_splits, recv_splits, out=None):
        rows = int(sum(recv_splits))
        recv = out if out is not None else torch.empty(
            (rows,) + tuple(send.shape[1:]), dtype=send.dtype, device=send.device)
        dist.all_to_all_single(recv, send.contiguous(), [int(x) for x in recv_splits],
                               [int(x) for x in send_splits], group=group)
        return recv
    return exchange


def dist_exchange_counts(world: int, group=None):
    """counts exchange over torch.distributed: [world, n_local] sent counts -> received counts
    [world_src, n_local] (host int64 arrays; the collective runs on `device`)."""
    import torch
    import torch.distributed as dist

    def exchange_counts(counts: np.ndarray, device) -> np.ndarray:
        send = torch.from_numpy(np.ascontiguousarray(counts, dtype=np.int64)).to(device).reshape(-1)
        recv = torch.empty_like(send)
        dist.all_to_all_single(recv, send, group=group)
        return recv.cpu().numpy().reshape(world, -1)
    return exchange_counts


# ---------------------------------------------------------------- the rank's stages (GPU)

@dataclasses.dataclass
class Dispatched:
    """A rank's state between its dispatch and its finish."""
    u: object            # [T, d_model] the rank's tokens (also the residual)
    w: object            # [T, k] routing weights
    inv: object          # [T*k] inverse permutation (dispatch row of slot (t, j))
    x_perm: object       # [T*k, E_in] dispatched rows, canonical order (expert, token)
    counts: np.ndarray   # [world, n_local] rows for each (owner rank, owner's local expert)


class _Grow:
    """A buffer kept between forwards and reallocated only when a forward needs a larger one."""

    def __init__(self, dtype, device, pin: bool = False):
        self.dtype, self.device, self.pin = dtype, device, pin
        self.buf = None

    def get(self, *shape):
        import math
        import torch
        numel = max(1, math.prod(shape))
        if self.buf is None or self.buf.numel() < numel:
            numel = max(numel, 2 * (0 if self.buf is None else self.buf.numel()))
            if self.pin:
                self.buf = torch.empty(numel, dtype=self.dtype, pin_memory=True)
            else:
                self.buf = torch.empty(numel, dtype=self.dtype, device=self.device)
        return self.buf[:math.prod(shape)].view(*shape)


class ExpertParallelRank:
    """One rank of an expert-parallel layer.

    cfg: the layer's configuration with T = this rank's tokens and n_experts = all experts.
    weights: as for MoELayer, except that w_gu and w_down hold only this rank's experts
    ([n_local, ...], experts [lo, hi) of expert_ranges); the router and latent weights are whole.
    Supported: bf16; no decoder wrap (input_norm / post_norm); a router_f32 router must be given
    as its bf16 split (moe_router_split_weights).

    The rank owns its buffers: the dispatch-side ones (fixed by T) are made here, the ones sized
    by the rows a forward receives grow on demand.  A forward's Dispatched state and its
    exchanged rows live in these buffers until the next forward."""

    def __init__(self, cfg: Config, weights: dict, rank: int, world: int):
        import torch
        if cfg.dtype != MOE_BF16 or cfg.input_norm or cfg.post_norm:
            raise ValueError("expert parallelism supports the bf16 layer without the decoder wrap")
        self.cfg, self.weights, self.rank, self.world = cfg, weights, rank, world
        self.lo, self.hi = expert_ranges(cfg.n_experts, world)[rank]
        self.n_local = self.hi - self.lo
        if weights["w_gu"].shape[0] != self.n_local or weights["w_down"].shape[0] != self.n_local:
            raise ValueError("w_gu / w_down must hold exactly this rank's experts")
        dev = weights["w_gu"].device
        dt = weights["w_gu"].dtype
        T, k, n = cfg.T, cfg.top_k, cfg.n_experts
        E = cfg.d_latent if cfg.d_latent > 0 else cfg.d_model
        self.workspace = torch.empty(workspace_size(cfg), dtype=torch.uint8, device=dev)
        self.logits = torch.empty((T, n), dtype=torch.float32, device=dev)
        self.idx = torch.empty((T, k), dtype=torch.int32, device=dev)
        self.wt = torch.empty((T, k), dtype=torch.float32, device=dev)
        self.z = torch.empty((T, E), dtype=dt, device=dev) if cfg.d_latent > 0 else None
        self.offsets = torch.empty(n + 1, dtype=torch.int32, device=dev)
        self.perm = torch.empty(T * k, dtype=torch.int32, device=dev)
        self.inv = torch.empty(T * k, dtype=torch.int32, device=dev)
        self.x_perm = torch.empty((T * k, E), dtype=dt, device=dev)
        self.y = torch.empty((T, E), dtype=dt, device=dev)
        self.offsets_host = torch.empty(n + 1, dtype=torch.int32, pin_memory=True)
        self.offsets_ready = torch.cuda.Event()
        self.plan_done = torch.cuda.Event()
        self.plan_done.record()
        # sized by the rows received (and sent back) in a forward
        self.recv = _Grow(dt, dev)
        self.back_recv = _Grow(dt, dev)
        self.grouped = _Grow(dt, dev)
        self.expert_out = _Grow(dt, dev)
        self.back = _Grow(dt, dev)
        self.plan_host = _Grow(torch.int32, None, pin=True)
        self.plan_dev = _Grow(torch.int32, dev)
        self.expert_ws = _Grow(torch.uint8, dev)
        self.E = E

    def _local_cfg(self, rows: int) -> Config:
        """The expert FFN's configuration on this rank: `rows` received rows over n_local experts."""
        c = Config.from_buffer_copy(self.cfg)
        c.T, c.top_k, c.n_experts = rows, 1, self.n_local
        return c

    def recv_buffer(self, rows: int):
        """Buffer for the rows this rank receives in a forward's dispatch exchange."""
        return self.recv.get(rows, self.E)

    def return_buffer(self, rows: int):
        """Buffer for the rows that come back to this rank in a forward's return exchange."""
        return self.back_recv.get(rows, self.E)

    def dispatch(self, u) -> Dispatched:
        c, w = self.cfg, self.weights
        moe_route(c, u, w["w_router"], w.get("logit_bias"), self.logits, self.idx, self.wt,
                  correction_bias=w.get("correction_bias"))
        # the permutation first: its expert offsets cross to the host while the latent
        # down-projection runs, then the rows are dispatched
        moe_permute(c, self.idx, self.offsets, self.perm, self.inv, workspace=self.workspace)
        self.offsets_host.copy_(self.offsets, non_blocking=True)
        self.offsets_ready.record()
        x = u
        if c.d_latent > 0:
            moe_latent_down(c, u, w["p_down"], self.z)
            x = self.z
        moe_dispatch_rows(c, self.inv, x, w.get("gamma_pre") if c.pre_norm else None, self.x_perm)
        self.offsets_ready.synchronize()
        return Dispatched(u=u, w=self.wt, inv=self.inv, x_perm=self.x_perm,
                          counts=send_counts(self.offsets_host.numpy(), self.world))

    def compute(self, recv, recv_counts: np.ndarray):
        """The rank's experts on the rows it received (source-major, then expert); returns their
        outputs in the same order."""
        rows, local_offsets = regroup_rows(recv_counts)
        n = len(rows)
        # the whole plan (regroup rows, their inverse, the local expert offsets) crosses to the
        # device in one asynchronous copy from pinned memory; each part starts on a 16-byte
        # boundary (the library's alignment rule).  The pinned buffer is rewritten only after the
        # previous forward's copy out of it has completed.
        m = (n + 3) // 4 * 4
        size = 2 * m + self.n_local + 1
        self.plan_done.synchronize()
        plan = self.plan_host.get(size)
        pv = plan.numpy()
        pv[:n] = rows
        pv[m:m + n] = inverse_rows(rows)
        pv[2 * m:] = local_offsets
        plan_d = self.plan_dev.get(size)
        plan_d.copy_(plan, non_blocking=True)
        self.plan_done.record()
        grouped = self.grouped.get(n, self.E)
        moe_gather_rows(recv, plan_d[:n], grouped)
        c = self._local_cfg(n)
        out = self.expert_out.get(n, self.E)
        ws = self.expert_ws.get(workspace_size(c))
        moe_expert_ffn(c, grouped, plan_d[2 * m:], self.weights["w_gu"], self.weights["w_down"],
                       self.weights.get("gamma_expert") if self.cfg.expert_norm else None, out, ws)
        back = self.back.get(n, self.E)
        moe_gather_rows(out, plan_d[m:m + n], back)
        return back

    def finish(self, d: Dispatched, out_perm, out=None):
        """Combine and latent up-projection of the rank's tokens into `out` (a new tensor when
        None), from their expert outputs out_perm in dispatch order."""
        import torch
        c, w = self.cfg, self.weights
        moe_combine(c, out_perm, d.inv, d.w, self.y)
        if c.d_latent == 0:
            if out is None:
                return self.y.clone()
            out.copy_(self.y)
            return out
        if out is None:
            out = torch.empty_like(d.u)
        moe_latent_up(c, self.y, w["p_up"], d.u, w.get("resid_g"), out)
        return out


def forward(rank: ExpertParallelRank, u, exchange, exchange_counts, out=None):
    """One expert-parallel forward of this rank's tokens (every rank calls it together); the
    exchanged rows land in the rank's own buffers."""
    d = rank.dispatch(u)
    recv_counts = exchange_counts(d.counts, u.device)
    send_splits = d.counts.sum(1)
    recv_splits = recv_counts.sum(1)
    recv = exchange(d.x_perm, send_splits, recv_splits,
                    out=rank.recv_buffer(int(recv_splits.sum())))
    back = rank.compute(recv, recv_counts)
    out_perm = exchange(back, recv_splits, send_splits,
                        out=rank.return_buffer(int(send_splits.sum())))
    return rank.finish(d, out_perm, out)


def emulated_forward(ranks: list, us: list, timer=None) -> list:
    """All ranks' forwards in one process: the exchanges become slicing and concatenation of the
    ranks' buffers (no collective).  Same stages and kernels as forward().  timer, if given, is
    called as timer(stage, rank, fn) for each stage ("dispatch", "compute", "finish") of each rank
    and must return fn()."""
    import torch
    run = timer or (lambda stage, r, fn: fn())
    world = len(ranks)
    ds = [run("dispatch", i, lambda r=r, u=u: r.dispatch(u)) for i, (r, u) in
          enumerate(zip(ranks, us))]
    # sender s's block for owner o: rows [start_s[o], start_s[o] + sum counts[o]) of its x_perm
    starts = [np.concatenate([[0], np.cumsum(d.counts.sum(1))]) for d in ds]
    backs = []
    for o in range(world):
        recv_counts = np.stack([ds[s].counts[o] for s in range(world)])
        recv = torch.cat([ds[s].x_perm[starts[s][o]:starts[s][o + 1]] for s in range(world)])
        back = run("compute", o, lambda o=o, recv=recv, rc=recv_counts: ranks[o].compute(recv, rc))
        backs.append((back, np.concatenate([[0], np.cumsum(recv_counts.sum(1))])))
    outs = []
    for s in range(world):
        out_perm = torch.cat([backs[o][0][backs[o][1][s]:backs[o][1][s + 1]] for o in range(world)])
        outs.append(run("finish", s, lambda s=s, op=out_perm: ranks[s].finish(ds[s], op)))
    return outs
