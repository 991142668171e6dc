"""Sequence-parallel Ring Self-Attention across GPUs: one chunk of the sequence per rank.

"Sequence Parallelism: Making 4D Parallelism Possible" (Li, Xue et al., 2021; review page,
Abstract and "Proposed method", points 1-3 and 6): the sequence is split into P chunks, one per
device; each device keeps the queries of its chunk and the key and value chunks travel around
a ring of devices, so that after P - 1 steps each device has computed its chunk's scores
against the whole sequence (ring pass 1), the softmax over the full key length, and the
weighted sum of every value chunk (ring pass 2). The backward pass runs on the same ring: the
partial key and value gradients of a chunk travel with it and collect every device's
contribution before they reach the chunk's owner. The computation of each step overlaps the
transfer of the next chunk (the overlap of computation and communication named in the review
of "Maximizing Parallelism in Distributed Training for Huge Neural Networks").

Rank r of P holds rows [r c, (r + 1) c), c = L / P: its queries Q_r, O_r, dO_r [B, H, c, d] and
full-length key and value buffers Kfull, Vfull [B, H, L, d] whose chunk r is its own and into
which the ring delivers the others (each (b, h) slice of a chunk is contiguous, so it is sent
and received in place). Schedule on rank r, with m the chunk at hand:

    forward, s = 0 .. P-1:   m = (r + s) mod P;  send chunk m of K, V to r - 1 and receive
                             chunk m + 1 from r + 1 while S_r[:, m] = Q_r K_m^T is computed
    then:                    softmax over the whole row and O_r = sum over the ring P V
    backward:                dQ_r over every chunk (no transfer: Kfull, Vfull are complete);
                             s = 0 .. P-1: m = (r - 1 - s) mod P;  this rank's contribution to
                             dK_m, dV_m is added to the fp32 accumulator received from r - 1 and
                             sent on to r + 1; at s = P - 1 the accumulator of chunk r is whole

The schedules are generators that yield once per ring step, after the step's transfer has been
posted and its computation enqueued. A process per rank drives its generator to the end
(`run`); `run_lockstep` drives the generators of every rank of an emulated ring in one process
step by step, which is how the ring's exchange is exercised on one device: no kernel of one
emulated rank ever waits for another's, the ranks only take turns on the host.

The arithmetic of a step belongs to a compute object: `Kernels` runs the library's per-rank
steps (include/rsa_sp.h) on the GPU. The exchange belongs to a ring object: `DistRing` sends
and receives with torch.distributed point-to-point operations (NCCL over NVLink on GPUs,
gloo on the CPU), `LocalRing` copies between the ranks of an emulated ring.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch
import torch.distributed as dist

from . import rsa

# ----------------------------------------------------------------------------- the exchange


class DistRing:
    """Ring of the ranks of a process group (all ranks by default): rank i sends to i - 1 and
    receives from i + 1 for the chunk exchange of the forward, and sends to i + 1 and receives
    from i - 1 for the accumulators of the backward. Every transfer is a point-to-point
    operation posted together with the others of its step (batch_isend_irecv)."""

    def __init__(self, group=None):
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        ranks = dist.get_process_group_ranks(group) if group is not None else list(range(self.world))
        self.prev = ranks[(self.rank - 1) % self.world]
        self.next = ranks[(self.rank + 1) % self.world]

    def _post(self, ops):
        return dist.batch_isend_irecv(ops) if ops else []

    def exchange_chunks(self, fulls, c, send_m, recv_m):
        """Send chunk send_m of every [B, H, L, d] tensor in `fulls` to the previous rank and
        receive chunk recv_m from the next, one contiguous (b, h) slice per message."""
        ops = []
        for t in fulls:
            B, H = t.shape[0], t.shape[1]
            for b in range(B):
                for h in range(H):
                    ops.append(dist.P2POp(dist.isend, t[b, h, send_m * c:(send_m + 1) * c],
                                          self.prev, self.group))
                    ops.append(dist.P2POp(dist.irecv, t[b, h, recv_m * c:(recv_m + 1) * c],
                                          self.next, self.group))
        return self._post(ops)

    def shift(self, send, recv):
        """Send the contiguous tensors `send` to the next rank, receive `recv` from the previous."""
        ops = []
        for a, b in zip(send, recv):
            ops.append(dist.P2POp(dist.isend, a, self.next, self.group))
            ops.append(dist.P2POp(dist.irecv, b, self.prev, self.group))
        return self._post(ops)

    @staticmethod
    def wait(handle):
        for w in handle or []:
            w.wait()


class LocalRing:
    """The ring's exchange between the ranks of an emulated ring held in one process. `states`
    lists every rank's RankState and `rings` every rank's LocalRing, in rank order. A transfer
    is a copy from the neighbour's buffers, made when its handle is waited for; `run_lockstep`
    keeps the ranks in step, so that the data copied is what the neighbour posted."""

    FULLS = ("kfull", "vfull")

    def __init__(self, rank: int, states: list, rings: list):
        self.rank, self.states, self.rings = rank, states, rings
        self.world = len(states)
        self.posted = []  # the tensors each shift sent, in the order the shifts were posted

    def exchange_chunks(self, fulls, c, send_m, recv_m):
        return [("chunk", len(fulls), c, recv_m)]

    def shift(self, send, recv):
        self.posted.append(list(send))
        return [("shift", len(self.posted) - 1, recv)]

    def wait(self, handle):
        for h in handle or []:
            if h[0] == "chunk":
                _, n, c, m = h
                src = self.states[(self.rank + 1) % self.world]
                dst = self.states[self.rank]
                for name in self.FULLS[:n]:
                    getattr(dst, name)[:, :, m * c:(m + 1) * c].copy_(getattr(src, name)[:, :, m * c:(m + 1) * c])
            else:
                _, k, recv = h
                sent = self.rings[(self.rank - 1) % self.world].posted[k]
                for a, b in zip(sent, recv):
                    b.copy_(a)


# ----------------------------------------------------------------------------- per-rank state


@dataclass
class RankState:
    """One rank's tensors. q, o, do, dq, dk, dv: [B, H, c, d]; lse [B, H, c]; kfull, vfull
    [B, H, L, d] (chunk `rank` filled by the caller, the rest by the ring)."""
    q: torch.Tensor
    kfull: torch.Tensor
    vfull: torch.Tensor
    causal: bool
    o: torch.Tensor | None = None
    lse: torch.Tensor | None = None
    do: torch.Tensor | None = None
    dq: torch.Tensor | None = None
    dk: torch.Tensor | None = None
    dv: torch.Tensor | None = None


def forward_steps(st: RankState, ring, comp):
    """Ring pass 1 with the K/V exchange overlapped, then the softmax and ring pass 2."""
    P, r = ring.world, ring.rank
    c = st.q.shape[2]
    for s in range(P):
        m = (r + s) % P
        h = ring.exchange_chunks([st.kfull, st.vfull], c, m, (m + 1) % P) if s < P - 1 else None
        comp.scores(st, r, P, m)
        yield
        ring.wait(h)
    if st.o is None:
        st.o = torch.empty_like(st.q)
    if st.lse is None:
        st.lse = torch.empty(st.q.shape[:3], dtype=torch.float32, device=st.q.device)
    comp.softmax_pv(st, r, P)


def backward_steps(st: RankState, ring, comp):
    """dQ of the rank's rows, then the dK/dV accumulators around the ring."""
    P, r = ring.world, ring.rank
    for name in ("dq", "dk", "dv"):
        if getattr(st, name) is None:
            setattr(st, name, torch.empty_like(st.q))
    comp.backward_rows(st, r, P)
    acc = [comp.new_acc(st.q), comp.new_acc(st.q)]      # dK, dV accumulators in hand
    nxt = [comp.new_acc(st.q), comp.new_acc(st.q)]      # where the next ones arrive
    h = None
    for s in range(P):
        m = (r - 1 - s) % P
        parts = comp.backward_keys(st, r, P, m)          # None when no row of r sees chunk m
        ring.wait(h)                                     # the accumulators of chunk m are here
        if s > 0:
            acc, nxt = nxt, acc
        last = s == P - 1
        comp.accumulate(acc[0], parts and parts[0], st.dk if last else None, s == 0)
        comp.accumulate(acc[1], parts and parts[1], st.dv if last else None, s == 0)
        h = None
        if not last:
            h = ring.shift(acc, nxt)
        yield
    ring.wait(h)


def run(gen):
    """Drive one rank's schedule to the end (one process per rank)."""
    for _ in gen:
        pass


def run_lockstep(gens):
    """Drive the schedules of every rank of an emulated ring one step at a time."""
    live = list(gens)
    while live:
        nxt = []
        for g in live:
            try:
                next(g)
                nxt.append(g)
            except StopIteration:
                pass
        live = nxt


# ----------------------------------------------------------------------------- GPU steps


class Kernels:
    """The per-rank steps through the library's C ABI (include/rsa_sp.h), bf16 on one GPU.
    Workspaces are allocated once per rank state and shape and reused by every step."""

    def __init__(self):
        self.lib = rsa.load_library()
        self._ws = {}
        self._parts = {}
        L = self.lib
        vp, i, sz, ll = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_longlong
        L.rsa_sp_workspace_size.argtypes = [i, i, i, i, i, i, i]
        L.rsa_sp_workspace_size.restype = sz
        L.rsa_sp_scores.argtypes = [vp, vp, i, i, i, i, i, i, i, i, vp, sz, vp]
        L.rsa_sp_softmax_pv.argtypes = [vp, vp, vp, i, i, i, i, i, i, i, vp, sz, vp]
        L.rsa_sp_backward_rows.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, vp, sz, vp]
        L.rsa_sp_backward_keys.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, vp, sz, vp]
        L.rsa_sp_accumulate.argtypes = [vp, vp, vp, ll, i, vp]
        for n in ("rsa_sp_scores", "rsa_sp_softmax_pv", "rsa_sp_backward_rows",
                  "rsa_sp_backward_keys", "rsa_sp_accumulate"):
            getattr(L, n).restype = i

    @staticmethod
    def _dims(st, P):
        B, H, c, d = st.q.shape
        return B, H, c * P, d

    def _workspace(self, st, P, bwd):
        """The rank's own workspace (its score slab, its rows' statistics): one per rank state,
        so that the ranks of an emulated ring never share one."""
        B, H, L, d = self._dims(st, P)
        key = (id(st), B, H, L, d, P, bool(st.causal), bwd, st.q.device)
        if key not in self._ws:
            n = self.lib.rsa_sp_workspace_size(B, H, L, d, P, int(st.causal), int(bwd))
            if n == 0:
                raise rsa.RSAError(rsa.RSA_ERR_UNSUPPORTED, "rsa_sp_workspace_size")
            self._ws[key] = torch.empty(n, dtype=torch.uint8, device=st.q.device)
        return self._ws[key]

    @staticmethod
    def _p(t):
        return ctypes.c_void_p(t.data_ptr()) if t is not None else None

    @staticmethod
    def _stream(st):
        return ctypes.c_void_p(torch.cuda.current_stream(st.q.device).cuda_stream)

    @staticmethod
    def _check(rc, what):
        if rc != rsa.RSA_OK:
            raise rsa.RSAError(rc, what)

    def scores(self, st, r, P, m):
        B, H, L, d = self._dims(st, P)
        ws = self._workspace(st, P, False)
        with torch.cuda.device(st.q.device):
            self._check(self.lib.rsa_sp_scores(self._p(st.q), self._p(st.kfull), B, H, L, d, P, r, m,
                                               int(st.causal), self._p(ws), ws.numel(),
                                               self._stream(st)), "rsa_sp_scores")

    def softmax_pv(self, st, r, P):
        B, H, L, d = self._dims(st, P)
        ws = self._workspace(st, P, False)
        with torch.cuda.device(st.q.device):
            self._check(self.lib.rsa_sp_softmax_pv(self._p(st.vfull), self._p(st.o), self._p(st.lse),
                                                   B, H, L, d, P, r, int(st.causal), self._p(ws),
                                                   ws.numel(), self._stream(st)), "rsa_sp_softmax_pv")

    def backward_rows(self, st, r, P):
        B, H, L, d = self._dims(st, P)
        ws = self._workspace(st, P, True)
        with torch.cuda.device(st.q.device):
            self._check(self.lib.rsa_sp_backward_rows(
                self._p(st.q), self._p(st.kfull), self._p(st.vfull), self._p(st.o), self._p(st.do),
                self._p(st.lse), self._p(st.dq), B, H, L, d, P, r, int(st.causal), self._p(ws),
                ws.numel(), self._stream(st)), "rsa_sp_backward_rows")

    def backward_keys(self, st, r, P, m):
        if st.causal and m > r:
            return None
        B, H, L, d = self._dims(st, P)
        ws = self._workspace(st, P, True)
        key = (st.q.shape, st.q.device, id(st))
        if key not in self._parts:
            self._parts[key] = (torch.empty_like(st.q), torch.empty_like(st.q))
        dk, dv = self._parts[key]
        with torch.cuda.device(st.q.device):
            self._check(self.lib.rsa_sp_backward_keys(
                self._p(st.q), self._p(st.kfull), self._p(st.vfull), self._p(st.do), self._p(dk),
                self._p(dv), B, H, L, d, P, r, m, int(st.causal), self._p(ws), ws.numel(),
                self._stream(st)), "rsa_sp_backward_keys")
        return dk, dv

    @staticmethod
    def new_acc(q):
        return torch.empty(q.shape, dtype=torch.float32, device=q.device)

    def accumulate(self, acc, part, out, first):
        with torch.cuda.device(acc.device):
            s = ctypes.c_void_p(torch.cuda.current_stream(acc.device).cuda_stream)
            self._check(self.lib.rsa_sp_accumulate(self._p(acc), self._p(part), self._p(out),
                                                   acc.numel(), int(first), s), "rsa_sp_accumulate")


# ----------------------------------------------------------------------------- rings of ranks


def ring_groups(world: int, ring_size: int, create: bool = True):
    """Ranks 0 .. world-1 as world / ring_size rings of consecutive ranks: rank g * ring_size + s
    is position s of ring g. With head parallelism ("4-D": heads split over the rings, the
    sequence over the ranks of a ring), ring g holds head group g. Returns the rank lists, or
    with `create` the process groups of the rings (every rank must call this, in the same
    order, as torch.distributed.new_group requires)."""
    if ring_size <= 0 or world % ring_size:
        raise ValueError(f"{world} ranks do not split into rings of {ring_size}")
    lists = [list(range(g * ring_size, (g + 1) * ring_size)) for g in range(world // ring_size)]
    if not create:
        return lists
    return [dist.new_group(ranks) for ranks in lists]


# ----------------------------------------------------------------------------- user entry


def full_buffer(local: torch.Tensor, rank: int, world: int) -> torch.Tensor:
    """A [B, H, L, d] buffer holding this rank's chunk `local` [B, H, c, d] at rows
    [rank c, (rank + 1) c); the ring fills the other rows."""
    B, H, c, d = local.shape
    full = torch.empty((B, H, c * world, d), dtype=local.dtype, device=local.device)
    full[:, :, rank * c:(rank + 1) * c].copy_(local)
    return full


def attention(q, k, v, causal: bool = False, ring=None, comp=None) -> RankState:
    """Sequence-parallel forward on this rank: q, k, v are the rank's chunk [B, H, c, d].
    Returns the rank's state (O, lse, and the full K/V buffers the backward reuses)."""
    ring = ring or DistRing()
    comp = comp or Kernels()
    st = RankState(q=q, kfull=full_buffer(k, ring.rank, ring.world),
                   vfull=full_buffer(v, ring.rank, ring.world), causal=causal)
    run(forward_steps(st, ring, comp))
    return st


def attention_backward(st: RankState, do, ring=None, comp=None) -> RankState:
    """Sequence-parallel backward on this rank: fills st.dq, st.dk, st.dv ([B, H, c, d])."""
    ring = ring or DistRing()
    comp = comp or Kernels()
    st.do = do
    run(backward_steps(st, ring, comp))
    return st
