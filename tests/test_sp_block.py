"""The Transformer block under sequence parallelism (the block's linear layers around the
attention): each rank's linear layers on its own rows, Ring Self-Attention across the ranks,
against the fp64 oracle composed on the whole sequence (oracle.linear and oracle.forward).

* CPU: real gloo processes (world 2, causal and not) run `block.block_forward` with fp64
  stand-ins for the per-rank steps; this checks the composition (head split of the projection,
  head merge of the attention output, residuals, GELU) and the ring around it.
* GPU (`-m gpu`): the library's linear kernel against oracle.linear on plain, head-split and
  head-merged layouts, ragged column tiles, GELU and residual; and the whole block on an
  emulated ring (lockstep) on one device against the oracle.
"""
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from sequence_ring_self_b200 import block, ring
from sequence_ring_self_b200.inputs import normals, round_to_bf16

from test_sp_ring import Fp64Steps

BF16_MAXABS, BF16_RELL2 = 2e-2, 1e-2


def block_inputs(L, hidden, H, d, ffn, seed):
    """Seeded X [L, hidden] ~ N(0, 1) and weights ~ N(0, 1/fan_in), biases ~ N(0, 0.01), all
    rounded to bf16 (biases kept as the fp32 values of the bf16 numbers)."""
    shapes = [("x", (L, hidden), 1.0), ("wqkv", (3 * H * d, hidden), hidden ** -0.5),
              ("bqkv", (3 * H * d,), 0.1), ("wo", (hidden, H * d), (H * d) ** -0.5),
              ("bo", (hidden,), 0.1), ("w1", (ffn, hidden), hidden ** -0.5), ("b1", (ffn,), 0.1),
              ("w2", (hidden, ffn), ffn ** -0.5), ("b2", (hidden,), 0.1)]
    out, start = {}, 0
    for name, shape, scale in shapes:
        n = int(np.prod(shape))
        out[name] = round_to_bf16(normals(seed, start, n).reshape(shape) * scale)
        start += n
    return out


def oracle_block(orc, w, H, d, causal):
    """The block on the whole sequence in fp64: linear layers and attention from the oracle."""
    L = w["x"].shape[0]
    qkv = orc.linear(w["x"], w["wqkv"], w["bqkv"])                     # [L, 3 H d]
    heads = qkv.reshape(L, 3, H, d).transpose(1, 2, 0, 3)             # [3, H, L, d]
    o, _ = orc.forward(heads[0][None], heads[1][None], heads[2][None], causal)
    merged = o[0].transpose(1, 0, 2).reshape(L, H * d)
    y = orc.linear(merged, w["wo"], w["bo"], r=w["x"])
    h = orc.linear(y, w["w1"], w["b1"], gelu=True)
    return orc.linear(h, w["w2"], w["b2"], r=y)


def fp64_linear(x, w, bias=None, residual=None, gelu=False, x_kin=None, y_kin=None):
    """CPU stand-in for the GPU linear layer with the same layouts (fp64 torch tensors)."""
    if x.dim() == 3:  # [H, M, d] read as [M, H d]
        x = x.permute(1, 0, 2).reshape(x.shape[1], -1)
    y = x @ w.T
    if bias is not None:
        y = y + bias
    if gelu:
        y = 0.5 * y * (1 + torch.erf(y / math.sqrt(2.0)))
    if residual is not None:
        y = y + residual
    if y_kin is not None and y_kin != y.shape[1]:  # [M, N] -> [N / y_kin, M, y_kin]
        y = y.reshape(y.shape[0], -1, y_kin).permute(1, 0, 2).contiguous()
    return y


def _weights(w, H, d, to):
    return block.BlockWeights(wqkv=to(w["wqkv"]), bqkv=to(w["bqkv"], True), wo=to(w["wo"]),
                              bo=to(w["bo"], True), w1=to(w["w1"]), b1=to(w["b1"], True),
                              w2=to(w["w2"]), b2=to(w["b2"], True), heads=H, head_dim=d)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


CPU_SHAPE = dict(L=32, hidden=16, H=2, d=4, ffn=24)


def _gloo_block_worker(rank, world, port, causal, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    import datetime

    import torch.distributed as dist

    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        s = CPU_SHAPE
        w = block_inputs(s["L"], s["hidden"], s["H"], s["d"], s["ffn"], seed=900)
        c = s["L"] // world
        to = lambda a, bias=False: torch.from_numpy(np.ascontiguousarray(a))
        wts = _weights(w, s["H"], s["d"], to)
        x = torch.from_numpy(w["x"][rank * c:(rank + 1) * c].copy())
        z, _ = block.block_forward(x, wts, causal, ring=ring.DistRing(), comp=Fp64Steps(),
                                   lin=fp64_linear)
        out.put((rank, z.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("causal", [False, True])
def test_gloo_block_matches_the_oracle(orc, causal):
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_gloo_block_worker, args=(r, world, port, causal, q))
             for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    s = CPU_SHAPE
    w = block_inputs(s["L"], s["hidden"], s["H"], s["d"], s["ffn"], seed=900)
    ref = oracle_block(orc, w, s["H"], s["d"], causal)
    got = np.concatenate([res[r] for r in range(world)], axis=0)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-10)


# ----------------------------------------------------------------------------- GPU


def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    from sequence_ring_self_b200 import build

    build.build()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    return dev


def _check_bf16(got, ref, name):
    err = np.abs(got - ref).max()
    rel = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30)
    bound = BF16_MAXABS * max(1.0, float(np.abs(ref).max()))
    assert err <= bound and rel <= BF16_RELL2, (name, err, bound, rel)


LINEAR_CASES = [  # (M, N, K, x_kin, y_kin, gelu, bias, residual)
    (128, 64, 64, None, None, False, False, False),    # one tile, ragged columns
    (256, 768, 512, None, None, True, True, False),    # three column tiles, GELU
    (384, 320, 128, None, None, False, True, True),    # ragged last column tile, residual
    (256, 768, 256, None, 64, False, True, False),     # query/key/value projection, d = 64
    (128, 768, 256, None, 128, False, True, False),    # the same, d = 128
    (256, 512, 256, 64, None, False, True, True),      # attention output read as [M, H d]
    (128, 256, 512, 128, None, True, False, False),    # the same, d = 128, GELU
]


@pytest.mark.gpu
@pytest.mark.parametrize("case", LINEAR_CASES)
def test_gpu_linear_matches_the_oracle(orc, case):
    from sequence_ring_self_b200 import rsa

    dev = _gpu()
    M, N, K, xk, yk, gelu, with_b, with_r = case
    rng_seed = 1000 + M + N + K
    x = round_to_bf16(normals(rng_seed, 0, M * K).reshape(M, K))
    w = round_to_bf16(normals(rng_seed, M * K, N * K).reshape(N, K) / math.sqrt(K))
    b = normals(rng_seed + 1, 0, N) * 0.1 if with_b else None
    r = round_to_bf16(normals(rng_seed + 2, 0, M * N).reshape(M, N)) if with_r else None
    bf = lambda a: torch.from_numpy(a.astype(np.float32)).to(torch.bfloat16).to(dev)
    if xk is None:
        xt = bf(x)
    else:  # the same matrix stored as [K / xk, M, xk]
        xt = bf(x.reshape(M, K // xk, xk).transpose(1, 0, 2).copy())
    bt = torch.from_numpy(b.astype(np.float32)).to(dev) if b is not None else None
    b_used = bt.double().cpu().numpy() if bt is not None else None  # the fp32 bias the GPU adds
    y = rsa.linear(xt, bf(w), bt, bf(r) if r is not None else None, gelu, x_kin=xk, y_kin=yk)
    torch.cuda.synchronize()
    assert rsa.last_device_status() == rsa.RSA_OK
    got = y.to("cpu", torch.float64).numpy()
    if yk is not None:  # [N / yk, M, yk] -> [M, N]
        got = got.transpose(1, 0, 2).reshape(M, N)
    ref = orc.linear(x, w, b_used, r, gelu)
    _check_bf16(got, ref, "linear")


@pytest.mark.gpu
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("P,d", [(2, 64), (4, 64), (2, 128)])
def test_gpu_block_on_an_emulated_ring_matches_the_oracle(orc, P, d, causal):
    """Every rank's linear layers on its rows, the attention on a lockstep ring of P ranks on
    one device (the library's per-rank kernels), against the oracle's block on the sequence."""
    from sequence_ring_self_b200 import rsa

    dev = _gpu()
    H, hidden, ffn, c = 4, 256, 512, 256
    L = P * c
    w = block_inputs(L, hidden, H, d, ffn, seed=950 + P + d)

    def to(a, bias=False):
        t = torch.from_numpy(np.ascontiguousarray(a.astype(np.float32))).to(dev)
        return t if bias else t.to(torch.bfloat16)

    wts = _weights(w, H, d, to)
    xs = [to(w["x"][r * c:(r + 1) * c]) for r in range(P)]
    # the projections of every rank (no exchange), then the ring in lockstep, then the rest
    qkv = [rsa.linear(x, wts.wqkv, wts.bqkv, y_kin=d) for x in xs]
    states = [ring.RankState(q=qkv[r][0:H].unsqueeze(0),
                             kfull=ring.full_buffer(qkv[r][H:2 * H].unsqueeze(0), r, P),
                             vfull=ring.full_buffer(qkv[r][2 * H:].unsqueeze(0), r, P), causal=causal)
              for r in range(P)]
    rings = []
    rings.extend(ring.LocalRing(r, states, rings) for r in range(P))
    comp = ring.Kernels()
    ring.run_lockstep([ring.forward_steps(states[r], rings[r], comp) for r in range(P)])
    zs = []
    for r in range(P):
        y = rsa.linear(states[r].o[0], wts.wo, wts.bo, xs[r], x_kin=d)
        h = rsa.linear(y, wts.w1, wts.b1, gelu=True)
        zs.append(rsa.linear(h, wts.w2, wts.b2, y))
    torch.cuda.synchronize()
    assert rsa.last_device_status() == rsa.RSA_OK
    got = torch.cat(zs).to("cpu", torch.float64).numpy()
    ref = oracle_block(orc, w, H, d, causal)
    _check_bf16(got, ref, "block")
