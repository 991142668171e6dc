"""GPU parity: the CUDA path (through the C ABI) against the fp64 CPU oracle on the same seeded
inputs.

Tolerances (fixed by the method's target precision): fp32 max-abs <= 1e-5; bf16 inputs with
fp32 accumulation: max-abs <= 2e-2 and relative L2 <= 1e-2, on O, dQ, dK and dV.

Workloads: the five transformer-shaped configurations of the method's evaluation (the pages
quote only end-to-end results, so synthetic inputs of these shapes stand in), plus ragged,
degenerate and sharp-attention edge cases. Large problems are compared on sampled heads, rows
or keys that the oracle computes one by one, and through N-invariance (the ring result must
not depend on the chunk count beyond rounding).
"""
import types

import ctypes

import numpy as np
import pytest
import torch

from sequence_ring_self_b200 import build, rsa
from sequence_ring_self_b200.inputs import make_inputs

pytestmark = pytest.mark.gpu

F32_MAXABS = 1e-5
BF16_MAXABS = 2e-2
BF16_RELL2 = 1e-2


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    build.build()
    rsa.load_library()
    torch.cuda.set_device(0)


def np64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def rel_l2(a, b):
    den = np.linalg.norm(b.ravel())
    return np.linalg.norm((a - b).ravel()) / (den if den > 0 else 1.0)


def check(got, ref, dtype, name, magnitude_scaled=False):
    """magnitude_scaled: for the supplementary unscaled-input cases, whose outputs exceed 8 in
    magnitude (one bf16 ulp is then 0.0625), the max-abs bound is taken relative to the
    tensor's largest magnitude."""
    err = np.abs(got - ref).max() if got.size else 0.0
    if dtype == "f32":
        assert err <= F32_MAXABS, f"{name}: max-abs {err:.3e} > {F32_MAXABS}"
    else:
        r = rel_l2(got, ref)
        bound = BF16_MAXABS * (max(1.0, float(np.abs(ref).max())) if magnitude_scaled else 1.0)
        assert err <= bound and r <= BF16_RELL2, f"{name}: max-abs {err:.3e} (bound {bound:.3e}), rel-L2 {r:.3e}"


def run(x, N, causal, *, bwd=True, ws_budget=0):
    dev = torch.device("cuda", 0)
    q, k, v, do = (x.torch(n, dev) for n in ("q", "k", "v", "do"))
    o, lse = rsa.forward(q, k, v, N, causal, ws_budget=ws_budget)
    out = {"O": o, "lse": lse}
    if bwd:
        dq, dk, dv = rsa.backward(q, k, v, o, do, lse, N, causal, ws_budget=ws_budget)
        out.update(dQ=dq, dK=dk, dV=dv)
    torch.cuda.synchronize()
    assert rsa.last_device_status() == rsa.RSA_OK
    return {n: np64(t) for n, t in out.items()}


def check_full(orc, x, got, causal, bwd=True, magnitude_scaled=False):
    o, lse = orc.forward(x.q, x.k, x.v, causal)
    check(got["O"], o, x.dtype, "O", magnitude_scaled)
    tol = 1e-5 if x.dtype == "f32" else 1e-3
    np.testing.assert_allclose(got["lse"], lse, rtol=tol if magnitude_scaled else 0, atol=tol)
    if bwd:
        for name, ref in zip(("dQ", "dK", "dV"), orc.backward(x.q, x.k, x.v, x.do, causal)):
            check(got[name], ref, x.dtype, name, magnitude_scaled)


def check_sampled(orc, x, got, causal, heads, rows, keys, keys_heads=1):
    for (b, h) in heads:
        o, lse = orc.forward_rows(x.q, x.k, x.v, b, h, rows, causal)
        check(got["O"][b, h, rows], o, x.dtype, f"O[{b},{h}] rows")
        np.testing.assert_allclose(got["lse"][b, h, rows], lse, rtol=0, atol=1e-3)
        dq = orc.backward_rows(x.q, x.k, x.v, x.do, b, h, rows, causal)
        check(got["dQ"][b, h, rows], dq, x.dtype, f"dQ[{b},{h}] rows")
    if keys is not None:
        for (b, h) in heads[:keys_heads]:
            dk, dv = orc.backward_keys(x.q, x.k, x.v, x.do, b, h, keys, causal)
            check(got["dK"][b, h, keys], dk, x.dtype, f"dK[{b},{h}] keys")
            check(got["dV"][b, h, keys], dv, x.dtype, f"dV[{b},{h}] keys")


def sample(L, seed, n=60, edges=(0, 1)):
    """Edge rows plus n seeded-random rows: the relative L2 over a sample stays representative
    of the whole tensor (a handful of hand-picked rows would be dominated by the few causal
    rows that see only one or two keys, where the bf16 rounding of P and O does not average)."""
    rng = np.random.default_rng(seed)
    picks = set(rng.choice(L, size=min(n, L), replace=False).tolist())
    picks |= {e % L for e in edges} | {L - 1, L - 2 if L > 1 else 0}
    return sorted(picks)


def check_invariants(x, got):
    """Properties of the exact result that hold at any size: key gradients sum to zero over the
    keys, value gradients sum to the output gradients (P is row-stochastic)."""
    dk_sum = got["dK"].sum(axis=2)
    dv_sum = got["dV"].sum(axis=2)
    scale_k = np.abs(got["dK"]).sum(axis=2) + 1e-30
    assert np.all(np.abs(dk_sum) <= 2e-2 * scale_k + 1e-6)
    do_sum = x.do.sum(axis=2)
    assert rel_l2(dv_sum, do_sum) <= 1e-2


# ------------------------------------------------------------------ the five configurations

def test_config1_fp32_forward(orc):
    """B=1 H=2 L=256 d=32 N=4 fp32, N(0,1), seed 0; vs oracle and vs the unchunked run."""
    x = make_inputs(1, 2, 256, 32, seed=0, dtype="f32")
    got = run(x, 4, False, bwd=False)
    check_full(orc, x, got, False, bwd=False)
    o_ring, _ = orc.forward_ring(x.q, x.k, x.v, 4)
    check(got["O"], o_ring, "f32", "O vs ring oracle")
    got1 = run(x, 1, False, bwd=False)
    check(got["O"], got1["O"], "f32", "O(N=4) vs O(N=1)")


@pytest.mark.parametrize("causal", [False, True])
def test_config1_fp32_backward(orc, causal):
    x = make_inputs(1, 2, 256, 32, seed=0, dtype="f32")
    got = run(x, 4, causal)
    check_full(orc, x, got, causal)


def test_config2_bert_base(orc):
    """B=8 H=12 L=512 d=64 N=4 bf16, N(0,1)/sqrt(d), dO ~ N(0,1), non-causal, full tensors."""
    x = make_inputs(8, 12, 512, 64, seed=2, dtype="bf16")
    got = run(x, 4, False)
    check_full(orc, x, got, False)
    check_invariants(x, got)


def test_config3_gpt_causal(orc):
    """B=4 H=16 L=4096 d=64 N=8 bf16 causal; four sampled heads compared in full."""
    x = make_inputs(4, 16, 4096, 64, seed=3, dtype="bf16")
    got = run(x, 8, True)
    heads = [(0, 0), (3, 15), (1, 7), (2, 10)]
    sub = types.SimpleNamespace(dtype="bf16")
    for n in ("q", "k", "v", "do"):
        setattr(sub, n, np.stack([getattr(x, n)[b, h] for b, h in heads])[None])
    g = {n: np.stack([got[n][b, h] for b, h in heads])[None] for n in got}
    check_full(orc, sub, g, True)
    check_invariants(x, got)


def test_config4_long_sequence(orc):
    """B=1 H=16 L=16384 d=128 N=16 bf16, forward slab groups in sequence (the default
    workspace holds a fifth of the 17 GB slab): sampled rows and sampled keys of two heads."""
    x = make_inputs(1, 16, 16384, 128, seed=4, dtype="bf16")
    info = rsa.plan_describe(1, 16, 16384, 128, 16, False, torch.bfloat16, False,
                             rsa.workspace_size(1, 16, 16384, 128, 16, False, torch.bfloat16, False))
    assert info["groups"] > 1  # the forward's slab is processed group by group
    got = run(x, 16, False)
    rows = sample(16384, 4, edges=(0, 1, 1023, 1024))
    # 60 random keys plus the edges of the sequence and of a chunk, on both sampled heads
    keys = sample(16384, 40, n=60, edges=(0, 1, 1023, 1024, 8191, 8192))
    check_sampled(orc, x, got, False, [(0, 0), (0, 13)], rows, keys=keys, keys_heads=2)
    check_invariants(x, got)


SWEEP_L = [1024, 2048, 4096, 8192, 16384]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("L", SWEEP_L)
def test_sweep_against_oracle_and_n_invariance(orc, L, causal):
    """B=1 H=16 d=64 bf16: every N in {1,2,4,8,16} agrees with N=1 on every head; the oracle
    checks sampled rows and keys of one head at N=16."""
    idx = SWEEP_L.index(L) * 10 + int(causal)
    x = make_inputs(1, 16, L, 64, seed=5 + idx, dtype="bf16")
    base = run(x, 1, causal)
    for N in (2, 4, 8, 16):
        got = run(x, N, causal)
        for n in ("O", "dQ", "dK", "dV"):
            check(got[n], base[n], "bf16", f"{n} N={N} vs N=1")
    got = run(x, 16, causal)
    check_sampled(orc, x, got, causal, [(0, 5)], sample(L, idx), keys=sample(L, 100 + idx, n=24))


@pytest.mark.parametrize("causal", [False, True])
def test_sweep_maximum_length(orc, causal):
    """The sweep's largest point, L = 32768: every N in {2,4,8,16} agrees with N=1 on every
    head, and at N = 16 sampled rows of one head agree with the oracle."""
    x = make_inputs(1, 16, 32768, 64, seed=60 + int(causal), dtype="bf16")
    base = run(x, 1, causal)
    for N in (2, 4, 8):
        got = run(x, N, causal)
        for n in ("O", "dQ", "dK", "dV"):
            check(got[n], base[n], "bf16", f"{n} N={N} vs N=1")
    got = run(x, 16, causal)
    for n in ("O", "dQ", "dK", "dV"):
        check(got[n], base[n], "bf16", f"{n} N=16 vs N=1")
    check_sampled(orc, x, got, causal, [(0, 3)], sample(32768, 7, edges=(0, 77, 16384)), keys=None)
    check_invariants(x, got)


def test_device_status_word_is_reported_and_cleared():
    """The path a kernel takes when a bounded wait gives up: it posts RSA_ERR_TIMEOUT into the
    device status word, rsa_last_device_status returns it once and clears it. The post here
    comes from the library's injection hook (a one-thread kernel), so no wait runs out."""
    assert rsa.last_device_status() == rsa.RSA_OK
    rsa.debug_report_status(rsa.RSA_ERR_TIMEOUT)
    assert rsa.last_device_status() == rsa.RSA_ERR_TIMEOUT
    assert rsa.last_device_status() == rsa.RSA_OK
    # a later healthy call is unaffected
    x = make_inputs(1, 1, 256, 64, seed=11, dtype="bf16")
    run(x, 2, False)


# ------------------------------------------------------------------ edge cases

EDGE = [  # (B, H, L, d, N)
    (1, 1, 1, 64, 1),      # one token
    (1, 2, 50, 64, 5),     # smaller than one tile, ragged
    (2, 1, 130, 64, 2),    # one full 128-row tile plus a 2-row tail
    (1, 3, 200, 128, 4),   # d = 128, ragged chunks (c = 50)
    (1, 2, 320, 64, 5),    # c = 64
    (1, 1, 700, 128, 7),   # several tiles, ragged tail, c = 100
    (3, 1, 384, 64, 384),  # one row per chunk
]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", EDGE)
def test_edge_shapes_bf16(orc, shape, causal):
    B, H, L, d, N = shape
    x = make_inputs(B, H, L, d, seed=100 + L + d, dtype="bf16")
    got = run(x, N, causal)
    check_full(orc, x, got, causal)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", [(1, 1, 1, 32, 1), (1, 2, 70, 32, 7), (2, 1, 200, 64, 4),
                                   (1, 1, 333, 64, 3)])
def test_edge_shapes_f32(orc, shape, causal):
    B, H, L, d, N = shape
    x = make_inputs(B, H, L, d, seed=200 + L, dtype="f32")
    got = run(x, N, causal)
    check_full(orc, x, got, causal)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("causal", [False, True])
def test_row_range_groups(orc, dtype, causal):
    """A small workspace budget forces groups of 128-row ranges of one head (the last one
    ragged): the forward's slab, and on the fp32 path the backward's, with dK/dV accumulated
    across groups. The bf16 backward keeps no slab and runs as one group."""
    d = 64
    B, H, L, N = 1, 2, 700, 7
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    budget = 300 * 1024
    for bwd in (False, True):
        info = rsa.plan_describe(B, H, L, d, N, causal, tdt, bwd,
                                 rsa.workspace_size(B, H, L, d, N, causal, tdt, bwd, budget))
        if bwd and dtype == "bf16":
            assert info["groups"] == 1
        else:
            assert info["rows_per_group"] < L and info["groups"] > B * H
    x = make_inputs(B, H, L, d, seed=300 + int(causal), dtype=dtype)
    got = run(x, N, causal, ws_budget=budget)
    check_full(orc, x, got, causal)
    whole = run(x, N, causal)
    for n in ("O", "dQ", "dK", "dV"):
        check(got[n], whole[n], dtype, f"{n} row groups vs whole heads")


@pytest.mark.parametrize("kind", ["unscaled", "sharp"])
def test_sharp_attention(orc, kind):
    """Score std ~1 (unscaled inputs) and sharp rows (Q x 8): a wrong scale or a missing
    max-subtraction would show here, not at the configurations' near-uniform attention."""
    extra = 8.0 if kind == "sharp" else 1.0
    x = make_inputs(2, 2, 512, 64, seed=400 + int(extra), dtype="bf16", qkv_scale=1.0,
                    q_extra_scale=extra)
    for causal in (False, True):
        got = run(x, 4, causal)
        check_full(orc, x, got, causal, magnitude_scaled=True)
        o, _ = orc.forward(x.q, x.k, x.v, causal)
        assert rel_l2(got["O"], o) <= BF16_RELL2


def test_deterministic_and_stream_ordered():
    x = make_inputs(2, 4, 1000, 64, seed=7, dtype="bf16")
    a = run(x, 8, True)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        b = run(x, 8, True)
    for n in a:
        np.testing.assert_array_equal(a[n], b[n])


def test_autograd_wrapper_and_host_api(orc):
    x = make_inputs(1, 2, 256, 64, seed=8, dtype="bf16")
    dev = torch.device("cuda", 0)
    q, k, v = (x.torch(n, dev).requires_grad_() for n in ("q", "k", "v"))
    o = rsa.RingSelfAttention.apply(q, k, v, 4, True)
    o.backward(x.torch("do", dev))
    ref = run(x, 4, True)
    np.testing.assert_array_equal(np64(o), ref["O"])
    for t, n in ((q, "dQ"), (k, "dK"), (v, "dV")):
        np.testing.assert_array_equal(np64(t.grad), ref[n])
    host = {n: x.torch(n).pin_memory() for n in ("q", "k", "v", "do")}
    res = rsa.forward_backward_host(host["q"], host["k"], host["v"], host["do"], 4, True)
    torch.cuda.synchronize()
    for n in ("O", "lse", "dQ", "dK", "dV"):
        np.testing.assert_array_equal(res[n].to(torch.float64).numpy(), ref[n])


@pytest.mark.parametrize("shape,chunks", [((2, 3, 384, 64, 3, True), 2),
                                          ((2, 3, 384, 64, 3, True), 6),
                                          ((1, 4, 300, 128, 3, False), 4)])
@pytest.mark.parametrize("recompute", [False, True])
def test_host_api_pipeline_equals_one_call(orc, shape, chunks, recompute):
    """The host-buffer call cut into groups of (batch, head) slices gives the single call's
    results bit for bit, and those agree with the oracle."""
    B, H, L, d, N, causal = shape
    x = make_inputs(B, H, L, d, seed=9 + chunks, dtype="bf16")
    dev = torch.device("cuda", 0)
    q, k, v, do = (x.torch(n, dev) for n in ("q", "k", "v", "do"))
    if recompute:
        o, lse = rsa.forward_recompute(q, k, v, N, causal)
    else:
        o, lse = rsa.forward(q, k, v, N, causal)
    dq, dk, dv = rsa.backward(q, k, v, o, do, lse, N, causal)
    one = {"O": o, "lse": lse, "dQ": dq, "dK": dk, "dV": dv}
    host = {n: x.torch(n).pin_memory() for n in ("q", "k", "v", "do")}
    res = rsa.forward_backward_host(host["q"], host["k"], host["v"], host["do"], N, causal,
                                    chunks=chunks, recompute=recompute)
    torch.cuda.synchronize()
    assert rsa.last_device_status() == rsa.RSA_OK
    for n in one:
        np.testing.assert_array_equal(res[n].to(torch.float64).numpy(), np64(one[n]), err_msg=n)
    check_full(orc, x, {n: res[n].to(torch.float64).numpy() for n in one}, causal)


RECOMPUTE_SHAPES = [  # (B, H, L, d, N, causal)
    (2, 3, 512, 64, 4, False),
    (2, 3, 512, 64, 4, True),
    (1, 3, 200, 128, 4, False),  # d = 128, ragged
    (1, 2, 700, 128, 7, True),
    (1, 1, 1, 64, 1, False),     # one token
    (1, 2, 50, 64, 5, True),     # smaller than one tile
    (2, 1, 130, 64, 2, True),    # one tile plus a 2-row tail
]


@pytest.mark.parametrize("shape", RECOMPUTE_SHAPES)
def test_forward_recompute_matches_oracle_and_slab_forward(orc, shape):
    """The slab-free two-pass forward: O and lse against the oracle, and against the slab
    forward within the bf16 bound; its lse drives the backward like the slab forward's."""
    B, H, L, d, N, causal = shape
    x = make_inputs(B, H, L, d, seed=600 + L + d + int(causal), dtype="bf16")
    dev = torch.device("cuda", 0)
    q, k, v, do = (x.torch(n, dev) for n in ("q", "k", "v", "do"))
    o, lse = rsa.forward_recompute(q, k, v, N, causal)
    dq, dk, dv = rsa.backward(q, k, v, o, do, lse, N, causal)
    torch.cuda.synchronize()
    assert rsa.last_device_status() == rsa.RSA_OK
    o_ref, lse_ref = orc.forward(x.q, x.k, x.v, causal)
    check(np64(o), o_ref, "bf16", "O (recompute)")
    np.testing.assert_allclose(np64(lse), lse_ref, rtol=0, atol=1e-3)
    slab = run(x, N, causal, bwd=False)
    check(np64(o), slab["O"], "bf16", "O recompute vs slab")
    np.testing.assert_allclose(np64(lse), slab["lse"], rtol=0, atol=1e-5)
    for name, ref, got in zip(("dQ", "dK", "dV"), orc.backward(x.q, x.k, x.v, x.do, causal),
                              (dq, dk, dv)):
        check(np64(got), ref, "bf16", f"{name} after the recompute forward")


def test_forward_recompute_rejects_fp32():
    q = torch.zeros(1, 1, 64, 32, dtype=torch.float32, device=torch.device("cuda", 0))
    with pytest.raises(rsa.RSAError) as e:
        rsa.forward_recompute(q, q, q, 1)
    assert e.value.code == rsa.RSA_ERR_UNSUPPORTED


def test_calls_from_a_fresh_thread():
    """A thread that has made no CUDA call yet (as autograd's backward thread may be) can call
    the library: it binds the device's context itself before encoding its tensor maps."""
    import threading
    x = make_inputs(1, 2, 256, 64, seed=9, dtype="bf16")
    ref = run(x, 4, False)
    dev = torch.device("cuda", 0)
    q, k, v, do = (x.torch(n, dev) for n in ("q", "k", "v", "do"))
    o, lse = torch.empty_like(q), torch.empty(1, 2, 256, dtype=torch.float32, device=dev)
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    nf = rsa.workspace_size(1, 2, 256, 64, 4, False, torch.bfloat16, False)
    nb = rsa.workspace_size(1, 2, 256, 64, 4, False, torch.bfloat16, True)
    wf = torch.empty(nf, dtype=torch.uint8, device=dev)
    wb = torch.empty(nb, dtype=torch.uint8, device=dev)
    torch.cuda.synchronize()
    lib = rsa.load_library()
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    rc = []

    def body():
        rc.append(lib.rsa_forward(p(q), p(k), p(v), p(o), p(lse), 1, 2, 256, 64, 4, 0, rsa.RSA_BF16,
                                  p(wf), nf, None))
        rc.append(lib.rsa_backward(p(q), p(k), p(v), p(o), p(do), p(lse), p(dq), p(dk), p(dv),
                                   1, 2, 256, 64, 4, 0, rsa.RSA_BF16, p(wb), nb, None))
        rc.append(lib.rsa_last_device_status(None))

    th = threading.Thread(target=body)
    th.start()
    th.join()
    assert rc == [rsa.RSA_OK] * 3, [rsa.status_string(c) for c in rc]
    torch.cuda.synchronize()
    for n, t in (("O", o), ("dQ", dq), ("dK", dk), ("dV", dv)):
        np.testing.assert_array_equal(np64(t), ref[n])


def test_library_errors_raise():
    dev = torch.device("cuda", 0)
    q = torch.zeros(1, 1, 100, 64, dtype=torch.bfloat16, device=dev)
    with pytest.raises(rsa.RSAError):
        rsa.forward(q, q, q, 3)
    small = torch.empty(1024, dtype=torch.uint8, device=dev)
    q2 = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16, device=dev)
    with pytest.raises(rsa.RSAError) as e:
        rsa.forward(q2, q2, q2, 1, workspace=small)
    assert e.value.code == rsa.RSA_ERR_WORKSPACE


def test_hbm_probe_writes_its_pattern_and_streams():
    """The HBM probe's write kernel covers every 16-byte vector with its documented pattern
    (word k of vector i holds i + k), and both directions stream at a plausible HBM rate."""
    dev = torch.device("cuda", 0)
    lib = rsa.load_library()
    nbytes, blocks = 512 << 20, 148 * 8
    buf = torch.zeros(nbytes, dtype=torch.uint8, device=dev)
    out = torch.zeros(blocks, dtype=torch.int32, device=dev)
    s = torch.cuda.current_stream(dev)
    vp = ctypes.c_void_p
    rates = {}
    for write in (1, 0):
        best = None
        for _ in range(3):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(s)
            rc = lib.rsa_probe_hbm(vp(buf.data_ptr()), nbytes, write, blocks, vp(out.data_ptr()),
                                   vp(s.cuda_stream))
            e1.record(s)
            assert rc == rsa.RSA_OK
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1)
            best = ms if best is None else min(best, ms)
        rates[write] = nbytes / (best / 1e3) / 1e9
    words = buf.view(torch.int32).view(-1, 4).cpu()
    nvec = nbytes // 16
    for i in (0, 1, 12345, nvec // 2 + 7, nvec - 1):
        assert words[i].tolist() == [i, i + 1, i + 2, i + 3], i
    assert int((words[:, 1] - words[:, 0] != 1).sum()) == 0
    for write, gbs in rates.items():
        assert 1000.0 < gbs < 20000.0, (write, gbs)
