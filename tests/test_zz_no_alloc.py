"""rsa_forward_noalloc: the forward pass for callers that cannot allocate device memory.

Some callers may not call cudaMalloc at all, for instance code that runs under another
runtime which owns the device memory pool, or a latency-critical path where an allocation
could synchronise the device. For them the library's rsa_forward_noalloc works in a fixed
scratch array inside the library (RSA_NOALLOC_SCRATCH_BYTES = 32 MiB per GPU) instead of a
caller-supplied workspace. These tests call it through the C ABI and check that it returns
what rsa_forward (with a caller workspace) returns, on two calls in a row, so that a second
call reusing the scratch left by the first still gives the right answer; and that a problem
too large for the scratch is refused before anything runs.

This file is collected last on purpose: if it fails, a run that stops at the first failure
has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from sequence_ring_self_b200 import build, rsa
from sequence_ring_self_b200.inputs import make_inputs

pytestmark = pytest.mark.gpu

SCRATCH = 32 << 20  # RSA_NOALLOC_SCRATCH_BYTES in include/rsa.h


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    build.build()
    torch.cuda.set_device(0)
    return rsa.load_library()


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _close(got, ref, dtype):
    got = got.to("cpu", torch.float64).numpy()
    ref = ref.to("cpu", torch.float64).numpy()
    err = np.abs(got - ref).max()
    if dtype == "f32":
        assert err <= 1e-5, err
    else:
        rel = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30)
        assert err <= 2e-2 and rel <= 1e-2, (err, rel)


@pytest.mark.parametrize("dtype,shape,N,causal", [
    ("bf16", (2, 8, 1024, 64), 4, True),    # several slab groups fit in the scratch
    ("bf16", (1, 2, 700, 128), 7, False),
    ("bf16", (1, 1, 8192, 64), 8, True),    # one head's slab exceeds the scratch: row ranges
    ("f32", (1, 2, 256, 32), 4, False),
])
def test_noalloc_forward_matches_forward_on_two_calls(lib, dtype, shape, N, causal):
    B, H, L, d = shape
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    x = make_inputs(*shape, seed=77, dtype=dtype)
    dev = torch.device("cuda", 0)
    q, k, v = (x.torch(n, dev) for n in ("q", "k", "v"))
    o_ref, lse_ref = rsa.forward(q, k, v, N, causal)  # caller-allocated workspace
    need = lib.rsa_workspace_size(B, H, L, d, N, int(causal), rsa._dtype_code(tdt), 0, SCRATCH)
    assert 0 < need <= SCRATCH
    plan = rsa.plan_describe(B, H, L, d, N, causal, tdt, False, SCRATCH)
    if L == 8192:
        assert plan["rows_per_group"] < L  # the row-range plan is the one exercised
    stream = torch.cuda.current_stream().cuda_stream
    for _ in range(2):
        o = torch.full_like(q, float("nan"))
        lse = torch.full((B, H, L), float("nan"), dtype=torch.float32, device=dev)
        rc = lib.rsa_forward_noalloc(_p(q), _p(k), _p(v), _p(o), _p(lse), B, H, L, d, N,
                                     int(causal), rsa._dtype_code(tdt), ctypes.c_void_p(stream))
        assert rc == rsa.RSA_OK, rsa.status_string(rc)
        torch.cuda.synchronize()
        assert rsa.last_device_status() == rsa.RSA_OK
        _close(o, o_ref, dtype)
        np.testing.assert_allclose(lse.cpu().numpy(), lse_ref.cpu().numpy(), rtol=0, atol=1e-5)


def test_noalloc_refuses_problems_beyond_the_scratch(lib):
    # the smallest plan holds 128 score rows; rows of 70,000 keys need about 36 MB
    B, H, L, d, N = 1, 1, 70000, 64, 1
    assert lib.rsa_workspace_size(B, H, L, d, N, 0, rsa.RSA_BF16, 0, SCRATCH) > SCRATCH
    dev = torch.device("cuda", 0)
    q = torch.zeros(B, H, L, d, dtype=torch.bfloat16, device=dev)
    o = torch.full_like(q, 3.0)
    lse = torch.zeros(B, H, L, dtype=torch.float32, device=dev)
    rc = lib.rsa_forward_noalloc(_p(q), _p(q), _p(q), _p(o), _p(lse), B, H, L, d, N, 0,
                                 rsa.RSA_BF16, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == rsa.RSA_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.all(o == 3.0)  # nothing ran
