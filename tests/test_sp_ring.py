"""Sequence-parallel Ring Self-Attention across ranks (one chunk of the sequence per rank):
the ring's schedule and exchange, checked against the fp64 oracle on the whole sequence.

* On the CPU (no GPU needed): the schedule in `sequence_ring_self_b200.ring` runs with a
  stand-in for the GPU's per-rank steps (`Fp64Steps` below, the attention definition on one
  rank's rows in fp64), once as an emulated ring in one process (`run_lockstep`, `LocalRing`)
  and once as real processes exchanging their chunks with torch.distributed (gloo, world
  sizes 2 and 4). The result of every rank is compared with `oracle.forward` / `backward` on
  the whole sequence: this checks which chunk each step sees, the ring order of the exchange,
  and the travelling dK/dV accumulators.
* On the GPU (`-m gpu`): the same schedule with the library's per-rank kernels
  (`ring.Kernels`, include/rsa_sp.h) on an emulated ring on one device, against the oracle with
  the bf16 bounds, and against the single-device forward/backward.
* Head parallelism combined with the ring ("4-D"): world 4 = 2 head groups x 2-rank rings.
"""
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from sequence_ring_self_b200 import ring
from sequence_ring_self_b200.inputs import make_inputs

BF16_MAXABS, BF16_RELL2 = 2e-2, 1e-2


class Fp64Steps:
    """One rank's steps in fp64 on the CPU, written from the attention definition (test
    stand-in for the GPU kernels): the scores of a key chunk into the rank's c x L slab, the
    softmax over the assembled rows and P V, dQ of the rank's rows, and the rank's
    contribution to dK and dV of one key chunk."""

    def __init__(self):
        self.slab = {}

    @staticmethod
    def _mask(st, r, m, c):
        i = r * c + torch.arange(c).view(c, 1)
        j = m * c + torch.arange(c).view(1, c)
        return j > i

    def scores(self, st, r, P, m):
        B, H, c, d = st.q.shape
        sl = self.slab.setdefault(id(st), torch.full((B, H, c, c * P), float("nan"), dtype=torch.float64))
        if st.causal and m > r:
            return
        s = st.q @ st.kfull[:, :, m * c:(m + 1) * c].transpose(-1, -2) / math.sqrt(d)
        if st.causal:
            s = s.masked_fill(self._mask(st, r, m, c), float("-inf"))
        sl[:, :, :, m * c:(m + 1) * c] = s

    def _probs(self, st, r, P):
        B, H, c, d = st.q.shape
        s = st.q @ st.kfull.transpose(-1, -2) / math.sqrt(d)
        if st.causal:
            i = r * c + torch.arange(c).view(c, 1)
            s = s.masked_fill(torch.arange(c * P).view(1, -1) > i, float("-inf"))
        return torch.softmax(s, dim=-1)

    def softmax_pv(self, st, r, P):
        s = self.slab[id(st)]
        if st.causal:  # chunks right of the diagonal were never visited
            B, H, c, L = s.shape
            s = s.clone()
            s[:, :, :, (r + 1) * c:] = float("-inf")
        assert not torch.isnan(s).any(), "a chunk of the slab was never computed"
        st.lse = torch.logsumexp(s, dim=-1)
        st.o = torch.softmax(s, dim=-1) @ st.vfull

    def backward_rows(self, st, r, P):
        d = st.q.shape[-1]
        p = self._probs(st, r, P)
        dp = st.do @ st.vfull.transpose(-1, -2)
        D = (st.do * st.o).sum(-1, keepdim=True)
        st.dq.copy_((p * (dp - D)) @ st.kfull / math.sqrt(d))

    def backward_keys(self, st, r, P, m):
        if st.causal and m > r:
            return None
        B, H, c, d = st.q.shape
        p = self._probs(st, r, P)[:, :, :, m * c:(m + 1) * c]
        dp = st.do @ st.vfull[:, :, m * c:(m + 1) * c].transpose(-1, -2)
        D = (st.do * st.o).sum(-1, keepdim=True)
        ds = p * (dp - D)
        return ds.transpose(-1, -2) @ st.q / math.sqrt(d), p.transpose(-1, -2) @ st.do

    @staticmethod
    def new_acc(q):
        return torch.empty(q.shape, dtype=torch.float64)

    @staticmethod
    def accumulate(acc, part, out, first):
        if first:
            acc.zero_()
        if part is not None:
            acc += part
        if out is not None:
            out.copy_(acc)


def _t(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))


def _lockstep(x, P, causal, comp, get=None):
    """Every rank of a P-rank ring in one process; returns the assembled O, lse, dQ, dK, dV.
    get(name) gives the whole input tensor (fp64 on the CPU by default)."""
    B, H, L, d = x.q.shape
    c = L // P
    get = get or (lambda n: _t(getattr(x, n)))
    q, k, v, do = (get(n) for n in ("q", "k", "v", "do"))
    states = [ring.RankState(q=q[:, :, r * c:(r + 1) * c].contiguous(),
                             kfull=ring.full_buffer(k[:, :, r * c:(r + 1) * c].contiguous(), r, P),
                             vfull=ring.full_buffer(v[:, :, r * c:(r + 1) * c].contiguous(), r, P),
                             causal=causal)
              for r in range(P)]
    rings = []
    rings.extend(ring.LocalRing(r, states, rings) for r in range(P))
    ring.run_lockstep([ring.forward_steps(states[r], rings[r], comp) for r in range(P)])
    for r, st in enumerate(states):
        st.do = do[:, :, r * c:(r + 1) * c].contiguous()
    ring.run_lockstep([ring.backward_steps(states[r], rings[r], comp) for r in range(P)])
    out = {}
    for n in ("o", "lse", "dq", "dk", "dv"):
        out[n] = torch.cat([getattr(st, n) for st in states], dim=2).to("cpu", torch.float64).numpy()
    return out


def _compare_exact(orc, x, got, causal, tol=1e-10):
    o, lse = orc.forward(x.q, x.k, x.v, causal)
    dq, dk, dv = orc.backward(x.q, x.k, x.v, x.do, causal)
    for n, ref in (("o", o), ("lse", lse), ("dq", dq), ("dk", dk), ("dv", dv)):
        np.testing.assert_allclose(got[n], ref, rtol=0, atol=tol, err_msg=n)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("P", [1, 2, 3, 4])
def test_lockstep_ring_schedule_matches_the_oracle(orc, P, causal):
    x = make_inputs(1, 2, 8 * P, 4, seed=500 + P, dtype="f32")
    _compare_exact(orc, x, _lockstep(x, P, causal, Fp64Steps()), causal)


def test_every_chunk_reaches_every_rank_in_ring_order():
    """The chunks a rank's steps see, in order, are its own and then its successors'."""
    P, c = 4, 2
    seen = {r: [] for r in range(P)}

    class Probe(Fp64Steps):
        def scores(self, st, r, P, m):
            # the chunk must already be in this rank's buffer when its step runs
            assert torch.equal(st.kfull[:, :, m * c:(m + 1) * c], full_k[:, :, m * c:(m + 1) * c])
            seen[r].append(m)
            super().scores(st, r, P, m)

    x = make_inputs(1, 1, P * c, 4, seed=9, dtype="f32")
    full_k = _t(x.k)
    _lockstep(x, P, False, Probe())
    for r in range(P):
        assert seen[r] == [(r + s) % P for s in range(P)]


# ----------------------------------------------------------------------------- gloo ranks

def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _gloo_worker(rank, world, port, heads_groups, causal, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    import datetime

    import torch.distributed as dist

    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        sp = world // heads_groups
        rings = ring.ring_groups(world, sp)
        hg, sr = divmod(rank, sp)
        rg = ring.DistRing(rings[hg])
        assert (rg.rank, rg.world) == (sr, sp)
        x = make_inputs(1, 2 * heads_groups, 8 * sp, 4, seed=700 + world, dtype="f32")
        c = 8
        hs = slice(2 * hg, 2 * hg + 2)
        q, k, v, do = (_t(getattr(x, n))[:, hs, sr * c:(sr + 1) * c].contiguous()
                       for n in ("q", "k", "v", "do"))
        comp = Fp64Steps()
        st = ring.attention(q, k, v, causal, ring=rg, comp=comp)
        ring.attention_backward(st, do, ring=rg, comp=comp)
        out.put((rank, {n: getattr(st, n).numpy() for n in ("o", "lse", "dq", "dk", "dv")}))
    finally:
        dist.destroy_process_group()


def _gloo_run(world, heads_groups, causal):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_gloo_worker, args=(r, world, port, heads_groups, causal, q))
             for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return res


@pytest.mark.parametrize("world,causal", [(2, False), (2, True), (4, False), (4, True)])
def test_gloo_ring_matches_the_oracle(orc, world, causal):
    """Real processes, one per rank, exchanging K/V chunks and dK/dV accumulators over gloo."""
    res = _gloo_run(world, 1, causal)
    x = make_inputs(1, 2, 8 * world, 4, seed=700 + world, dtype="f32")
    got = {n: np.concatenate([res[r][n] for r in range(world)], axis=2)
           for n in ("o", "lse", "dq", "dk", "dv")}
    _compare_exact(orc, x, got, causal)


@pytest.mark.parametrize("causal", [False, True])
def test_head_parallel_times_sequence_parallel(orc, causal):
    """4 ranks = 2 head groups x 2-rank sequence rings ("4-D"): rank (g, s) holds heads of
    group g and rows of chunk s; the rings run within each head group."""
    world, groups = 4, 2
    res = _gloo_run(world, groups, causal)
    x = make_inputs(1, 2 * groups, 16, 4, seed=700 + world, dtype="f32")
    sp = world // groups
    got = {}
    for n in ("o", "lse", "dq", "dk", "dv"):
        per_group = [np.concatenate([res[g * sp + s][n] for s in range(sp)], axis=2)
                     for g in range(groups)]
        got[n] = np.concatenate(per_group, axis=1)
    _compare_exact(orc, x, got, causal)


def test_ring_groups_partition_the_ranks():
    gs = ring.ring_groups(8, 4, create=False)
    assert gs == [[0, 1, 2, 3], [4, 5, 6, 7]]
    assert ring.ring_groups(6, 3, create=False) == [[0, 1, 2], [3, 4, 5]]
    with pytest.raises(ValueError):
        ring.ring_groups(6, 4, create=False)


# ----------------------------------------------------------------------------- GPU kernels

SP_GPU = [  # (B, H, L, d, P)
    (1, 2, 512, 64, 4),
    (2, 3, 1024, 128, 2),
    (1, 4, 2048, 64, 8),
    (1, 2, 768, 128, 3),   # chunk of 256 keys: window tiles end exactly at the chunk's end
    (1, 2, 384, 64, 3),    # chunk of 128 keys: a 256-key tile reaches past the window
    (1, 2, 512, 64, 4, "unscaled"),   # score std ~1: wrong scores or statistics would show
    (1, 2, 768, 128, 3, "unscaled"),
]


@pytest.mark.gpu
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", SP_GPU)
def test_gpu_ring_kernels_match_the_oracle(orc, shape, causal):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    from sequence_ring_self_b200 import build, rsa

    build.build()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    B, H, L, d, P = shape[:5]
    unscaled = len(shape) > 5
    x = make_inputs(B, H, L, d, seed=800 + L + P, dtype="bf16",
                    qkv_scale=1.0 if unscaled else None)
    got = _lockstep(x, P, causal, ring.Kernels(), get=lambda n: x.torch(n, dev))
    torch.cuda.synchronize()
    assert rsa.last_device_status() == rsa.RSA_OK
    o, lse = orc.forward(x.q, x.k, x.v, causal)
    refs = dict(zip(("o", "dq", "dk", "dv"), (o,) + orc.backward(x.q, x.k, x.v, x.do, causal)))
    for n, ref in refs.items():
        err = np.abs(got[n] - ref).max()
        rel = np.linalg.norm(got[n] - ref) / np.linalg.norm(ref)
        # unscaled inputs give outputs beyond 8 (one bf16 ulp 0.0625): max-abs relative to the
        # tensor's largest magnitude, as in the single-device sharp-attention cases
        bound = BF16_MAXABS * (max(1.0, float(np.abs(ref).max())) if unscaled else 1.0)
        assert err <= bound and rel <= BF16_RELL2, (n, err, rel)
    np.testing.assert_allclose(got["lse"], lse, rtol=1e-3 if unscaled else 0, atol=1e-3)
    # against the single-device path on the same inputs
    q, k, v, do = (x.torch(n, dev) for n in ("q", "k", "v", "do"))
    o1, lse1 = rsa.forward(q, k, v, P, causal)
    dq1, dk1, dv1 = rsa.backward(q, k, v, o1, do, lse1, P, causal)
    np.testing.assert_allclose(got["lse"], lse1.cpu().numpy(), rtol=1e-5, atol=1e-5)
    # both paths are within the bf16 bound of the oracle (checked above), so they are within
    # twice that bound of each other (two bf16 roundings can differ by a whole ulp, 0.03125
    # for values in [4, 8))
    for n, t in (("o", o1), ("dq", dq1), ("dk", dk1), ("dv", dv1)):
        ref = t.to("cpu", torch.float64).numpy()
        err = np.abs(got[n] - ref).max()
        rel = np.linalg.norm(got[n] - ref) / np.linalg.norm(ref)
        bound = 2 * BF16_MAXABS * (max(1.0, float(np.abs(ref).max())) if unscaled else 1.0)
        assert err <= bound and rel <= 2 * BF16_RELL2, (n, err, rel)
