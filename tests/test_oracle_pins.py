"""Pins for the fp64 oracle: each test checks the oracle against something other than itself.

* brute force at 50 significant digits (``decimal``), with no max-subtraction, on tiny inputs;
* closed forms (zero queries, one key, a single dominant key, the two-key sigmoid);
* softmax invariants (rows sum to one, masked entries zero, key-shift invariance);
* the chunking invariant of the ring schedule (ring result == unchunked result for every N);
* central finite differences of sum(O * G) for the backward pass, plus invariants that
  follow from P being row-stochastic.

The method: exact softmax attention, S = Q K^T / sqrt(d), P = softmax_row(S), O = P V, the
reading of "Sequence Parallelism: Making 4D Parallelism Possible" (review page, Abstract and
"Proposed method") in which Ring Self-Attention changes only where and in what order the
attention is computed.
"""
import decimal
import math

import numpy as np
import pytest

from sequence_ring_self_b200.inputs import make_inputs


def _rand(B, H, L, d, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    return [rng.standard_normal((B, H, L, d)) * scale for _ in range(4)]


# ---------------------------------------------------------------- brute force, 50 digits

def _decimal_attention(q, k, v, causal):
    """softmax(q k^T / sqrt d) v for one head, in 50-digit decimal arithmetic, without
    subtracting the row maximum."""
    ctx = decimal.Context(prec=50)
    D = decimal.Decimal
    L, d = q.shape
    inv_sqrt_d = ctx.divide(D(1), ctx.sqrt(D(d)))
    O = np.zeros((L, d))
    lse = np.zeros(L)
    for i in range(L):
        w = []
        for j in range(L):
            if causal and j > i:
                w.append(D(0))
                continue
            s = D(0)
            for t in range(d):
                s = ctx.add(s, ctx.multiply(D(float(q[i, t])), D(float(k[j, t]))))
            w.append(ctx.exp(ctx.multiply(s, inv_sqrt_d)))
        z = D(0)
        for x in w:
            z = ctx.add(z, x)
        lse[i] = float(ctx.ln(z))
        for t in range(d):
            acc = D(0)
            for j in range(L):
                acc = ctx.add(acc, ctx.multiply(w[j], D(float(v[j, t]))))
            O[i, t] = float(ctx.divide(acc, z))
    return O, lse


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("L,d,scale", [(1, 1, 1.0), (3, 2, 1.0), (5, 4, 2.0), (8, 4, 3.0),
                                       (7, 3, 0.5)])
def test_forward_matches_decimal_brute_force(orc, L, d, scale, causal):
    q, k, v, _ = _rand(1, 2, L, d, seed=L * 10 + d, scale=scale)
    o, lse = orc.forward(q, k, v, causal)
    for h in range(2):
        ob, lb = _decimal_attention(q[0, h], k[0, h], v[0, h], causal)
        np.testing.assert_allclose(o[0, h], ob, rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(lse[0, h], lb, rtol=1e-13, atol=1e-14)


def test_forward_large_scores_do_not_overflow(orc):
    # scores of order 800: exp would overflow without the row-maximum shift
    q, k, v, _ = _rand(1, 1, 6, 2, seed=3)
    q *= 400.0
    o, lse = orc.forward(q, k, v)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))
    s = q[0, 0] @ k[0, 0].T / math.sqrt(2)
    np.testing.assert_allclose(lse[0, 0], s.max(1) + np.log(np.exp(s - s.max(1, keepdims=True)).sum(1)),
                               rtol=1e-14)


# ---------------------------------------------------------------- closed forms

@pytest.mark.parametrize("causal", [False, True])
def test_zero_queries_give_running_mean(orc, causal):
    _, k, v, _ = _rand(2, 3, 12, 5, seed=7)
    q = np.zeros_like(k)
    o, lse = orc.forward(q, k, v, causal)
    L = 12
    for i in range(L):
        n = i + 1 if causal else L
        np.testing.assert_allclose(o[:, :, i], v[:, :, :n].mean(axis=2), rtol=1e-13, atol=1e-15)
        np.testing.assert_allclose(lse[:, :, i], math.log(n), rtol=1e-14)


def test_single_key_returns_value(orc):
    q, k, v, _ = _rand(2, 2, 1, 6, seed=11)
    o, lse = orc.forward(q, k, v)
    np.testing.assert_array_equal(o, v)
    np.testing.assert_allclose(lse[..., 0], (q * k).sum(-1)[..., 0] / math.sqrt(6), rtol=1e-14)


def test_causal_first_row_is_first_value(orc):
    q, k, v, _ = _rand(1, 2, 9, 4, seed=12)
    o, _ = orc.forward(q, k, v, causal=True)
    np.testing.assert_array_equal(o[:, :, 0], v[:, :, 0])


def test_two_keys_sigmoid(orc):
    # d = 1, L = 2: P_i0 = 1 / (1 + exp(q_i (k_1 - k_0))), a logistic function
    q = np.array([0.7, -1.3]).reshape(1, 1, 2, 1)
    k = np.array([0.4, 1.9]).reshape(1, 1, 2, 1)
    v = np.array([2.0, -5.0]).reshape(1, 1, 2, 1)
    o, _ = orc.forward(q, k, v)
    for i in range(2):
        p0 = 1.0 / (1.0 + math.exp(q[0, 0, i, 0] * (k[0, 0, 1, 0] - k[0, 0, 0, 0])))
        assert o[0, 0, i, 0] == pytest.approx(p0 * 2.0 + (1 - p0) * -5.0, rel=1e-14)


def test_dominant_key_gives_hard_attention(orc):
    L, d = 10, 4
    rng = np.random.default_rng(5)
    k = rng.standard_normal((1, 1, L, d)) * 0.1
    v = rng.standard_normal((1, 1, L, d))
    jstar = 6
    q = np.zeros((1, 1, L, d))
    q[..., 0] = 1.0
    k[0, 0, jstar, 0] = 50.0 * math.sqrt(d)  # score +50 above the rest (which are ~0.05)
    o, _ = orc.forward(q, k, v)
    # the other keys carry weight about exp(-50) each; add fp64 rounding of the sum
    np.testing.assert_allclose(o[0, 0], np.broadcast_to(v[0, 0, jstar], (L, d)), rtol=1e-15, atol=1e-18)


# ---------------------------------------------------------------- softmax invariants

@pytest.mark.parametrize("causal", [False, True])
def test_probabilities_are_row_stochastic_and_masked(orc, causal):
    q, k, _, _ = _rand(2, 2, 16, 8, seed=21, scale=2.0)
    p = orc.probs(q, k, causal)
    assert np.all(p >= 0)
    np.testing.assert_allclose(p.sum(-1), 1.0, atol=1e-14)
    if causal:
        iu = np.triu_indices(16, 1)
        assert np.all(p[..., iu[0], iu[1]] == 0)
    # probabilities reproduce the forward output
    _, k2, v, _ = _rand(2, 2, 16, 8, seed=22)
    o, _ = orc.forward(q, k, v, causal)
    np.testing.assert_allclose(np.einsum("bhij,bhjd->bhid", p, v), o, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("causal", [False, True])
def test_key_shift_invariance(orc, causal):
    # K_j -> K_j + c shifts row i's scores by q_i . c / sqrt d; P and O do not change
    q, k, v, _ = _rand(1, 2, 11, 6, seed=23)
    c = np.random.default_rng(24).standard_normal(6)
    o1, l1 = orc.forward(q, k, v, causal)
    o2, l2 = orc.forward(q, k + c, v, causal)
    np.testing.assert_allclose(o2, o1, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(l2 - l1, (q @ c) / math.sqrt(6), rtol=1e-11, atol=1e-12)


def test_output_linear_in_values(orc):
    q, k, v1, v2 = _rand(1, 2, 9, 3, seed=25)
    o1, _ = orc.forward(q, k, v1)
    o2, _ = orc.forward(q, k, v2)
    o3, _ = orc.forward(q, k, 2.0 * v1 - 3.0 * v2)
    np.testing.assert_allclose(o3, 2.0 * o1 - 3.0 * o2, rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------- chunking invariant

@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("L", [8, 16, 64, 256])
def test_ring_forward_equals_unchunked(orc, L, causal):
    d = 4 if L == 256 else 8
    q, k, v, _ = _rand(1, 2, L, d, seed=L + causal)
    o, lse = orc.forward(q, k, v, causal)
    for N in [n for n in range(1, L + 1) if L % n == 0]:
        o2, l2 = orc.forward_ring(q, k, v, N, causal)
        np.testing.assert_allclose(o2, o, rtol=1e-12, atol=1e-13, err_msg=f"N={N}")
        np.testing.assert_allclose(l2, lse, rtol=1e-12, atol=1e-13, err_msg=f"N={N}")


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("L", [8, 16, 64])
def test_ring_backward_equals_unchunked(orc, L, causal):
    q, k, v, do = _rand(1, 2, L, 4, seed=100 + L + causal)
    ref = orc.backward(q, k, v, do, causal)
    for N in [n for n in range(1, L + 1) if L % n == 0]:
        got = orc.backward_ring(q, k, v, do, N, causal)
        for name, a, b in zip("dQ dK dV".split(), got, ref):
            np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-13, err_msg=f"{name} N={N}")


def test_ring_rejects_indivisible_chunk_count(orc):
    q, k, v, _ = _rand(1, 1, 10, 2, seed=1)
    with pytest.raises(RuntimeError):
        orc.forward_ring(q, k, v, 3)


# ---------------------------------------------------------------- backward

@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("L,d", [(1, 2), (5, 3), (12, 8), (16, 4)])
def test_backward_matches_finite_differences(orc, L, d, causal):
    q, k, v, g = _rand(1, 2, L, d, seed=200 + L + d + causal)
    dq, dk, dv = orc.backward(q, k, v, g, causal)
    h = 1e-6

    def loss(qq, kk, vv):
        return float((orc.forward(qq, kk, vv, causal)[0] * g).sum())

    for which, grad in ((0, dq), (1, dk), (2, dv)):
        fd = np.zeros_like(grad)
        args = [q, k, v]
        for idx in np.ndindex(*grad.shape):
            a = [x.copy() for x in args]
            a[which][idx] += h
            fp = loss(*a)
            a[which][idx] -= 2 * h
            fm = loss(*a)
            fd[idx] = (fp - fm) / (2 * h)
        err = np.abs(fd - grad).max() / max(np.abs(grad).max(), 1e-30)
        assert err <= 1e-6, f"{'QKV'[which]} rel err {err}"


@pytest.mark.parametrize("causal", [False, True])
def test_backward_invariants(orc, causal):
    q, k, v, do = _rand(2, 2, 13, 5, seed=31, scale=1.5)
    dq, dk, dv = orc.backward(q, k, v, do, causal)
    # rows of dS sum to zero, so the key gradients sum to zero
    np.testing.assert_allclose(dk.sum(axis=2), 0.0, atol=1e-12)
    # rows of P sum to one, so the value gradients sum to the output gradients
    np.testing.assert_allclose(dv.sum(axis=2), do.sum(axis=2), rtol=1e-12, atol=1e-12)


def test_backward_permutation_equivariance(orc):
    q, k, v, do = _rand(1, 2, 10, 4, seed=41)
    perm = np.random.default_rng(42).permutation(10)
    dq, dk, dv = orc.backward(q, k, v, do)
    dq2, dk2, dv2 = orc.backward(q, k[:, :, perm], v[:, :, perm], do)
    np.testing.assert_allclose(dq2, dq, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(dk2, dk[:, :, perm], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(dv2, dv[:, :, perm], rtol=1e-12, atol=1e-14)
    o, _ = orc.forward(q, k, v)
    o2, _ = orc.forward(q, k[:, :, perm], v[:, :, perm])
    np.testing.assert_allclose(o2, o, rtol=1e-12, atol=1e-14)


def test_value_gradient_linear_in_output_gradient(orc):
    q, k, v, g1 = _rand(1, 1, 7, 3, seed=51)
    g2 = _rand(1, 1, 7, 3, seed=52)[0]
    a = orc.backward(q, k, v, g1)
    b = orc.backward(q, k, v, g2)
    c = orc.backward(q, k, v, g1 + g2)
    for x, y, z in zip(a, b, c):
        np.testing.assert_allclose(z, x + y, rtol=1e-11, atol=1e-13)


# ---------------------------------------------------------------- sampled rows agree with full

@pytest.mark.parametrize("causal", [False, True])
def test_sampled_rows_and_keys_match_full(orc, causal):
    x = make_inputs(1, 2, 40, 8, seed=9, dtype="bf16")
    o, lse = orc.forward(x.q, x.k, x.v, causal)
    dq, dk, dv = orc.backward(x.q, x.k, x.v, x.do, causal)
    rows = [0, 1, 17, 39]
    orow, lrow = orc.forward_rows(x.q, x.k, x.v, 0, 1, rows, causal)
    np.testing.assert_allclose(orow, o[0, 1, rows], rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(lrow, lse[0, 1, rows], rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(orc.backward_rows(x.q, x.k, x.v, x.do, 0, 1, rows, causal),
                               dq[0, 1, rows], rtol=1e-12, atol=1e-15)
    dkr, dvr = orc.backward_keys(x.q, x.k, x.v, x.do, 0, 1, rows, causal)
    np.testing.assert_allclose(dkr, dk[0, 1, rows], rtol=1e-11, atol=1e-15)
    np.testing.assert_allclose(dvr, dv[0, 1, rows], rtol=1e-11, atol=1e-15)


# ------------------------------------------------------------------ linear layers of the block

def _py_linear(x, w, b, r, gelu):
    """The definition in plain Python floats (math.fsum, math.erf): an independent restatement."""
    M, K = len(x), len(x[0])
    N = len(w)
    y = []
    for m in range(M):
        row = []
        for n in range(N):
            acc = math.fsum(x[m][k] * w[n][k] for k in range(K)) + (b[n] if b is not None else 0.0)
            if gelu:
                acc = 0.5 * acc * (1.0 + math.erf(acc / math.sqrt(2.0)))
            row.append(acc + (r[m][n] if r is not None else 0.0))
        y.append(row)
    return np.array(y)


@pytest.mark.parametrize("gelu", [False, True])
@pytest.mark.parametrize("with_bias,with_res", [(False, False), (True, False), (True, True)])
def test_linear_matches_plain_python(orc, gelu, with_bias, with_res):
    rng = np.random.default_rng(31)
    M, N, K = 3, 5, 7
    x, w = rng.normal(size=(M, K)), rng.normal(size=(N, K))
    b = rng.normal(size=N) if with_bias else None
    r = rng.normal(size=(M, N)) if with_res else None
    got = orc.linear(x, w, b, r, gelu)
    ref = _py_linear(x.tolist(), w.tolist(), None if b is None else b.tolist(),
                     None if r is None else r.tolist(), gelu)
    np.testing.assert_allclose(got, ref, rtol=1e-13, atol=1e-13)


def test_gelu_values_and_symmetry(orc):
    """GELU(x) = x Phi(x): GELU(0) = 0, GELU(x) - GELU(-x) = x (Phi(x) + Phi(-x) = 1),
    GELU(1) = Phi(1) = 0.8413447460685429 (the standard normal CDF at 1), GELU(10) = 10 and
    GELU(-10) = 0 to double precision."""
    xs = np.array([[0.0, 1.0, -1.0, 2.5, -2.5, 10.0, -10.0]])
    eye = np.eye(1)
    y = orc.linear(xs.T, eye, gelu=True)[:, 0]
    assert y[0] == 0.0
    assert y[1] == pytest.approx(0.8413447460685429, abs=1e-15)
    assert y[1] - y[2] == pytest.approx(1.0, abs=1e-15)
    assert y[3] - y[4] == pytest.approx(2.5, abs=1e-15)
    assert y[5] == pytest.approx(10.0, abs=1e-14) and abs(y[6]) < 1e-20


def test_linear_identity_weight_and_residual(orc):
    rng = np.random.default_rng(32)
    x, r = rng.normal(size=(4, 6)), rng.normal(size=(4, 6))
    np.testing.assert_array_equal(orc.linear(x, np.eye(6)), x)
    np.testing.assert_allclose(orc.linear(x, np.eye(6), r=r), x + r, rtol=0, atol=1e-15)
    # the bias adds to every row; the weight is used as out x in (a transposed weight fails)
    w = rng.normal(size=(3, 6))
    b = rng.normal(size=3)
    np.testing.assert_allclose(orc.linear(x, w, b), x @ w.T + b, rtol=1e-13, atol=1e-13)
