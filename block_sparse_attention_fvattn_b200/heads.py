"""Head-sharded execution of one attention layer across ranks, with Runtime
Load Balancing (RLB) and Slack-Aware Sparse Augmentation (SASA).

The method runs sequence-parallel video DiTs where, after the all-to-all,
every rank holds a shard of the heads. Top-p routing leaves heads with very
different kept work, so the most loaded rank sets the critical path. RLB
measures each head's actual work after routing and moves a few heavy heads
between ranks over point-to-point links (each rank sending and receiving at
most one); SASA then lets each rank below the critical path spend its slack
on extra high-probability blocks without lengthening that path
(ai-feeds.com FVAttn summary, "Key modules" 2 and 3; hotpaper.ai summary,
RLB and SASA bullets).

One step of rank r (every computation is a C-ABI call of the library):
  1. route its static shard of heads [r*H/W, (r+1)*H/W) and measure each
     head's work (fvattn_route, fvattn_head_cost);
  2. all-gather the H head costs (one collective of H int64 values);
  3. the same migration plan on every rank (fvattn_rlb_plan, host code);
  4. send the Q, K, V of the head it gives away and receive the one it takes
     (point-to-point), route the received head;
  5. optionally augment its lists within its slack, the critical rank's load
     minus its own (fvattn_augment);
  6. schedule and attend its final heads (fvattn_schedule,
     fvattn_sparse_attn);
  7. send the output of the received head back to its owner and receive the
     output of the head it gave away.
The output of rank r is O for its own shard, in shard order.

Slots. A rank's buffers hold S+1 heads: its S own heads and one spare.
A received head lands in the spare slot; if the rank also gave a head away,
the received head is moved into the freed slot, and if it only gave one
away, its last head fills the hole -- so its final heads are always the
contiguous slots [0, F) and run as one problem, and step 7 restores the
shard order of the outputs.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional, Sequence, Tuple

import torch


def shard_range(H: int, world: int, rank: int) -> Tuple[int, int]:
    """Static shard of rank `rank`: heads [rank*H/world, (rank+1)*H/world)."""
    return rank * H // world, (rank + 1) * H // world


@dataclass
class Plan:
    owner_in: List[int]
    owner_out: List[int]
    costs: List[int]
    load_static: List[int]
    load_after: List[int]

    @property
    def critical(self) -> int:
        return max(self.load_after) if self.load_after else 0


def _loads(costs, owner, world):
    out = [0] * world
    for h, c in enumerate(costs):
        out[owner[h]] += int(c)
    return out


def make_plan(costs: Sequence[int], world: int, balance: bool = True, max_moves: int = 1) -> Plan:
    from . import fvattn as fa
    H = len(costs)
    owner_in = [r for r in range(world) for _ in range(*shard_range(H, world, r))]
    if balance:
        owner_out, load = fa.rlb_plan(list(costs), world, None, max_moves)
    else:
        owner_out, load = list(owner_in), _loads(costs, owner_in, world)
    return Plan(owner_in, owner_out, [int(c) for c in costs], _loads(costs, owner_in, world), load)


class GpuBackend:
    """The library's kernels on CUDA tensors; problems are [1, F, N, D] views."""

    def __init__(self, geo, p: float, k_min: int, device, num_ctas: int = 0):
        from . import fvattn as fa
        self.fa = fa
        self.geo1, self.p, self.k_min = geo, float(p), int(k_min)
        self.dev = torch.device(device)
        self.num_ctas = num_ctas if num_ctas > 0 else fa.default_num_ctas()
        self.nb = fa.num_blocks(self.geo(1))
        self._ws = {}
        self.work = None
        self.cta_range = torch.zeros(self.num_ctas + 1, dtype=torch.int32, device=self.dev)

    def geo(self, F: int):
        g = self.geo1
        return self.fa.Geometry(1, F, g.D, g.grid, g.block, g.softmax_scale, g.dtype)

    def ws(self, F: int):
        if F not in self._ws:
            w = torch.zeros(max(self.fa.workspace_size(self.geo(F), self.num_ctas), 256), dtype=torch.uint8,
                            device=self.dev)
            self.fa.workspace_init(w)
            self._ws[F] = w
        return self._ws[F]

    def alloc(self, slots: int):
        g = self.geo1
        N, D, nb = g.N, g.D, self.nb
        mk = lambda *s, dt=g.dtype: torch.zeros(s, dtype=dt, device=self.dev)  # noqa: E731
        return dict(q=mk(slots, N, D), k=mk(slots, N, D), v=mk(slots, N, D), o=mk(slots, N, D),
                    cnt=mk(slots, nb, dt=torch.int32), idx=mk(slots, nb, nb, dt=torch.int32),
                    probs=mk(slots, nb, nb, dt=torch.float32))

    def route(self, buf, a: int, b: int):
        F = b - a
        if F <= 0:
            return
        v = lambda t: t[a:b].unsqueeze(0)  # noqa: E731
        self.fa.route(self.geo(F), v(buf["q"]), v(buf["k"]), self.p, self.k_min, v(buf["cnt"]), v(buf["idx"]),
                      self.ws(F), v(buf["probs"]))

    def head_cost(self, buf, F: int) -> torch.Tensor:
        out = torch.zeros(max(F, 1), dtype=torch.int64, device=self.dev)
        if F > 0:
            self.fa.head_cost(self.geo(F), buf["cnt"][:F].unsqueeze(0), buf["idx"][:F].unsqueeze(0), out[:F])
        return out[:F]

    def augment(self, buf, F: int, budget: int):
        added = torch.zeros(1, dtype=torch.int64, device=self.dev)
        mass = torch.zeros(1, dtype=torch.float64, device=self.dev)
        if F > 0:
            self.fa.augment(self.geo(F), buf["probs"][:F].unsqueeze(0), int(budget), buf["cnt"][:F].unsqueeze(0),
                            buf["idx"][:F].unsqueeze(0), self.ws(F), added, mass)
        return added, mass

    def attend(self, buf, F: int):
        if F <= 0:
            return
        g = self.geo(F)
        need = F * self.nb
        if self.work is None or self.work.numel() < need:
            self.work = torch.zeros(need, dtype=torch.int32, device=self.dev)
        v = lambda t: t[:F].unsqueeze(0)  # noqa: E731
        ws = self.ws(F)
        self.fa.schedule(g, v(buf["cnt"]), v(buf["idx"]), False, self.num_ctas, self.work[:need], self.cta_range,
                         ws)
        self.fa.sparse_attn(g, v(buf["q"]), v(buf["k"]), v(buf["v"]), v(buf["cnt"]), v(buf["idx"]),
                            self.work[:need], self.cta_range, self.num_ctas, False, v(buf["o"]), ws)

    def copy_slot(self, buf, src: int, dst: int, names=("q", "k", "v", "cnt", "idx", "probs")):
        for n in names:
            buf[n][dst].copy_(buf[n][src])


@dataclass
class RankState:
    """Buffers and per-step bookkeeping of one rank."""
    rank: int
    world: int
    H: int
    backend: object
    sasa: bool = False
    balance: bool = True
    h0: int = 0
    h1: int = 0
    buf: dict = field(default_factory=dict)
    plan: Optional[Plan] = None
    send_head: Optional[int] = None
    recv_head: Optional[int] = None
    F: int = 0
    slot_head: List[int] = field(default_factory=list)
    added_pairs: object = None
    added_mass: object = None

    def __post_init__(self):
        self.h0, self.h1 = shard_range(self.H, self.world, self.rank)
        self.buf = self.backend.alloc(self.S + 1)

    @property
    def S(self) -> int:
        return self.h1 - self.h0

    # -- step 1
    def route_and_cost(self):
        self.backend.route(self.buf, 0, self.S)
        return self.backend.head_cost(self.buf, self.S)

    # -- step 3
    def set_plan(self, plan: Plan):
        self.plan = plan
        self.send_head = self.recv_head = None
        for h in range(self.H):
            if plan.owner_in[h] == self.rank and plan.owner_out[h] != self.rank:
                self.send_head = h
            if plan.owner_out[h] == self.rank and plan.owner_in[h] != self.rank:
                self.recv_head = h

    # -- step 4
    def migration(self):
        """(sends, recvs): lists of (peer, tensor) for the point-to-point exchange."""
        sends, recvs = [], []
        if self.send_head is not None:
            m = self.send_head - self.h0
            dst = self.plan.owner_out[self.send_head]
            sends += [(dst, self.buf[n][m]) for n in ("q", "k", "v")]
        if self.recv_head is not None:
            src = self.plan.owner_in[self.recv_head]
            recvs += [(src, self.buf[n][self.S]) for n in ("q", "k", "v")]
        return sends, recvs

    def after_migration(self):
        S = self.S
        heads = list(range(self.h0, self.h1))
        if self.recv_head is not None:
            self.backend.route(self.buf, S, S + 1)
        if self.send_head is not None and self.recv_head is not None:
            m = self.send_head - self.h0
            self.backend.copy_slot(self.buf, S, m)
            heads[m] = self.recv_head
            self.F = S
        elif self.send_head is not None:
            m = self.send_head - self.h0
            if m != S - 1:
                self.backend.copy_slot(self.buf, S - 1, m)
                heads[m] = heads[S - 1]
            heads = heads[:S - 1]
            self.F = S - 1
        elif self.recv_head is not None:
            heads.append(self.recv_head)
            self.F = S + 1
        else:
            self.F = S
        self.slot_head = heads

    # -- step 5
    def budget(self) -> int:
        if not self.sasa or self.plan is None:
            return 0
        return self.plan.critical - self.plan.load_after[self.rank]

    def augment(self):
        self.added_pairs, self.added_mass = self.backend.augment(self.buf, self.F, self.budget())

    # -- step 6
    def attend(self):
        self.backend.attend(self.buf, self.F)

    # -- step 7
    def returns(self):
        sends, recvs = [], []
        S = self.S
        if self.recv_head is not None:
            slot = self.slot_head.index(self.recv_head)
            sends.append((self.plan.owner_in[self.recv_head], self.buf["o"][slot]))
        if self.send_head is not None:
            recvs.append((self.plan.owner_out[self.send_head], self.buf["o"][S]))
        return sends, recvs

    def after_returns(self):
        S = self.S
        if self.send_head is None:
            return
        m = self.send_head - self.h0
        o = self.buf["o"]
        if self.recv_head is None and m != S - 1:
            o[S - 1].copy_(o[m])        # the last own head ran in slot m
        o[m].copy_(o[S])

    def output(self) -> torch.Tensor:
        """O of the rank's own shard, [S, N, D], in shard order."""
        return self.buf["o"][:self.S]


class TorchComm:
    """torch.distributed (NCCL on GPUs, gloo on CPUs): one all-gather of the
    head costs and batched point-to-point exchanges."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group

    def all_gather_costs(self, own: torch.Tensor, H: int, world: int) -> List[int]:
        smax = max(shard_range(H, world, r)[1] - shard_range(H, world, r)[0] for r in range(world))
        pad = torch.zeros(smax, dtype=torch.int64, device=own.device)
        pad[:own.numel()] = own
        parts = [torch.zeros_like(pad) for _ in range(world)]
        self.dist.all_gather(parts, pad, group=self.group)
        out = []
        for r in range(world):
            a, b = shard_range(H, world, r)
            out += [int(x) for x in parts[r][:b - a].cpu().tolist()]
        return out

    def exchange(self, sends, recvs):
        if not sends and not recvs:
            return
        if self.dist.get_backend(self.group) == "nccl":
            # one NCCL group for all the transfers of this phase
            ops = [self.dist.P2POp(self.dist.isend, t, peer, self.group) for peer, t in sends]
            ops += [self.dist.P2POp(self.dist.irecv, t, peer, self.group) for peer, t in recvs]
            works = self.dist.batch_isend_irecv(ops)
        else:
            works = [self.dist.isend(t, peer, group=self.group) for peer, t in sends]
            works += [self.dist.irecv(t, peer, group=self.group) for peer, t in recvs]
        for w in works:
            w.wait()


def step_distributed(st: RankState, comm: TorchComm) -> RankState:
    """One layer step of this rank; every rank calls it with the same H."""
    own = st.route_and_cost()
    costs = comm.all_gather_costs(own, st.H, st.world)
    st.set_plan(make_plan(costs, st.world, balance=st.balance))
    comm.exchange(*st.migration())
    st.after_migration()
    if st.sasa:
        st.augment()
    st.attend()
    comm.exchange(*st.returns())
    st.after_returns()
    return st


def step_emulated(states: List[RankState], timer=None) -> Plan:
    """One layer step of every rank in this process (one GPU or CPU): the same
    phases in the same order, each rank's compute run one rank after another,
    point-to-point transfers done as copies. `timer(rank, fn)` may wrap each
    rank's attention (step 6) to time it."""
    world = len(states)
    H = states[0].H
    costs = []
    for st in states:
        costs += [int(x) for x in st.route_and_cost().cpu().tolist()]
    plan = make_plan(costs, world, balance=states[0].balance)
    for st in states:
        st.set_plan(plan)

    _p2p(states, lambda st: st.migration())
    for st in states:
        st.after_migration()
        if st.sasa:
            st.augment()
    for st in states:
        if timer is not None:
            timer(st.rank, st.attend)
        else:
            st.attend()
    _p2p(states, lambda st: st.returns())
    for st in states:
        st.after_returns()
    return plan


def _p2p(states, phase):
    """Deliver every rank's sends of one phase to the matching receives: the
    k-th receive of rank r from peer s takes the k-th send of s to r."""
    posted = [phase(st) for st in states]
    for r, (_, recvs) in enumerate(posted):
        taken = {}
        for src, t in recvs:
            k = taken.get(src, 0)
            sends = [x for peer, x in posted[src][0] if peer == r]
            t.copy_(sends[k])
            taken[src] = k + 1
