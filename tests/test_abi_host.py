"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every function
``include/rsa.h`` declares, rejects bad arguments before launching anything, and plans its
workspace consistently."""
import ctypes
import os
import re

import pytest
import torch

from sequence_ring_self_b200 import build, rsa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return rsa.load_library()


def _declared():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            text = open(os.path.join(ROOT, "include", h)).read()
            names += re.findall(r"RSA_API\s+[\w\s\*]+?\b(rsa_\w+)\s*\(", text)
    return names


def test_header_declares_the_abi():
    assert sorted(_declared()) == sorted(rsa.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for name in _declared():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    assert rsa.status_string(rsa.RSA_OK) == "RSA_OK"
    assert rsa.status_string(rsa.RSA_ERR_WORKSPACE) == "RSA_ERR_WORKSPACE"
    assert rsa.status_string(99) == "RSA_ERR_UNKNOWN"


FAKE = 0x100000  # a 16-byte-aligned non-null pointer that is never dereferenced


def _fwd(lib, B=1, H=1, L=128, d=64, N=1, dt=rsa.RSA_BF16, ptr=FAKE, ws=FAKE, ws_bytes=1 << 30,
         lse=FAKE):
    return lib.rsa_forward(ptr, ptr, ptr, ptr, lse, B, H, L, d, N, 0, dt, ws, ws_bytes, None)


def _bwd(lib, B=1, H=1, L=128, d=64, N=1, dt=rsa.RSA_BF16, ptr=FAKE, ws=FAKE, ws_bytes=1 << 30):
    return lib.rsa_backward(ptr, ptr, ptr, ptr, ptr, ptr, ptr, ptr, ptr, B, H, L, d, N, 0, dt, ws,
                            ws_bytes, None)


@pytest.mark.parametrize("call", [_fwd, _bwd])
def test_argument_errors_are_reported_before_any_launch(lib, call):
    assert call(lib, L=100, N=3) == rsa.RSA_ERR_INVALID_ARG          # L % N != 0
    assert call(lib, B=0) == rsa.RSA_ERR_INVALID_ARG
    assert call(lib, N=0) == rsa.RSA_ERR_INVALID_ARG
    assert call(lib, L=-4) == rsa.RSA_ERR_INVALID_ARG
    assert call(lib, d=96) == rsa.RSA_ERR_UNSUPPORTED                # bf16 head dim
    assert call(lib, d=128, dt=rsa.RSA_F32) == rsa.RSA_ERR_UNSUPPORTED
    assert call(lib, dt=7) == rsa.RSA_ERR_UNSUPPORTED
    assert call(lib, ptr=0) == rsa.RSA_ERR_INVALID_ARG               # null
    assert call(lib, ptr=FAKE + 8) == rsa.RSA_ERR_INVALID_ARG        # misaligned
    assert call(lib, ws_bytes=64) == rsa.RSA_ERR_WORKSPACE           # too small
    assert call(lib, ws=FAKE + 64) == rsa.RSA_ERR_INVALID_ARG        # workspace not 256-aligned
    assert call(lib, ws=0) == rsa.RSA_ERR_INVALID_ARG


@pytest.mark.skipif(torch.cuda.is_available(), reason="needs a machine without a usable GPU")
def test_cuda_failures_are_described(lib):
    # valid arguments: without a GPU the call fails at its first CUDA call, and says which
    assert _bwd(lib) == rsa.RSA_ERR_CUDA
    assert b"failed" in lib.rsa_last_error()
    with pytest.raises(rsa.RSAError, match="failed"):
        raise rsa.RSAError(rsa.RSA_ERR_CUDA, "rsa_backward")


def _fwdr(lib, B=1, H=1, L=128, d=64, N=1, dt=rsa.RSA_BF16, ptr=FAKE, lse=FAKE):
    return lib.rsa_forward_recompute(ptr, ptr, ptr, ptr, lse, B, H, L, d, N, 0, dt, None)


def test_forward_recompute_argument_errors(lib):
    assert _fwdr(lib, L=100, N=3) == rsa.RSA_ERR_INVALID_ARG
    assert _fwdr(lib, B=0) == rsa.RSA_ERR_INVALID_ARG
    assert _fwdr(lib, d=96) == rsa.RSA_ERR_UNSUPPORTED
    assert _fwdr(lib, d=64, dt=rsa.RSA_F32) == rsa.RSA_ERR_UNSUPPORTED  # bf16 only
    assert _fwdr(lib, ptr=0) == rsa.RSA_ERR_INVALID_ARG
    assert _fwdr(lib, lse=0) == rsa.RSA_ERR_INVALID_ARG
    assert _fwdr(lib, ptr=FAKE + 8) == rsa.RSA_ERR_INVALID_ARG


def test_sizes_beyond_the_unit_counters_are_unsupported(lib):
    # 2^24 heads of 2^16 rows: more 128-row units than a 32-bit counter holds
    assert lib.rsa_workspace_size(1 << 12, 1 << 12, 1 << 16, 64, 1, 0, rsa.RSA_BF16, 0, 0) == 0
    assert _fwd(lib, B=1 << 12, H=1 << 12, L=1 << 16) == rsa.RSA_ERR_UNSUPPORTED
    assert _bwd(lib, B=1 << 12, H=1 << 12, L=1 << 16) == rsa.RSA_ERR_UNSUPPORTED
    assert _fwdr(lib, B=1 << 12, H=1 << 12, L=1 << 16) == rsa.RSA_ERR_UNSUPPORTED


def test_forward_rejects_null_lse(lib):
    assert _fwd(lib, lse=0) == rsa.RSA_ERR_INVALID_ARG


def test_workspace_size_invalid_is_zero(lib):
    assert lib.rsa_workspace_size(1, 1, 100, 64, 3, 0, rsa.RSA_BF16, 0, 0) == 0
    assert lib.rsa_workspace_size(1, 1, 128, 80, 1, 0, rsa.RSA_BF16, 0, 0) == 0


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("bwd", [False, True])
def test_plans_fit_their_budget_and_grow_with_it(lib, dtype, bwd):
    d = 64
    B, H, L, N = 2, 3, 1000, 8
    if bwd and dtype == torch.bfloat16:
        # no slab: one group of every head, the padded row statistics only, for any budget
        stats = 2 * B * H * 1024 * 4
        for budget in [1, 1 << 20, 1 << 30, 0]:
            n = rsa.workspace_size(B, H, L, d, N, False, dtype, bwd, budget)
            assert n == stats
            info = rsa.plan_describe(B, H, L, d, N, False, dtype, bwd, n)
            assert info["fits"] and info["groups"] == 1 and info["rows_per_group"] == L
            assert info["heads_per_group"] == B * H
        assert rsa.plan_describe(B, H, L, d, N, False, dtype, bwd, stats - 1)["fits"] is False
        return
    sizes, groups = [], []
    for budget in [1, 1 << 18, 1 << 20, 1 << 22, 1 << 24, 1 << 26, 1 << 30]:
        n = rsa.workspace_size(B, H, L, d, N, False, dtype, bwd, budget)
        info = rsa.plan_describe(B, H, L, d, N, False, dtype, bwd, n)
        assert info["fits"] and info["bytes"] == n
        if n > budget:  # only the minimum plan may exceed the budget
            assert info["rows_per_group"] == 128 and info["heads_per_group"] == 1
        sizes.append(n)
        Lp = info["padded_row"]
        assert Lp % 64 == 0 and Lp >= L
        rows = info["rows_per_group"]
        assert rows == L or rows % 128 == 0
        # every (head, row) is covered exactly once by the groups: rectangles of
        # heads_per_group heads x rows_per_group rows
        assert info["groups"] == -(-B * H // info["heads_per_group"]) * -(-L // rows)
        groups.append(info["groups"])
    assert sizes == sorted(sizes)
    assert groups == sorted(groups, reverse=True)  # a larger budget never needs more groups
    assert rsa.plan_describe(B, H, L, d, N, False, dtype, bwd, sizes[0] - 1)["fits"] is False


def test_forward_groups_fill_whole_rounds(lib):
    """The bf16 forward's slab groups are rectangles of heads x 128-row tiles that fill whole
    rounds of the softmax/PV kernel's CTAs (148 SMs, one CTA each at d = 128): for the
    long-sequence shape (a head's slab is 1.09 GB; the 4 GiB default holds 3.7 heads) the plan
    takes ceil(2048 / 148) = 14 rounds, the fewest possible, and no group is a remainder of a
    few units."""
    B, H, L, d, N = 1, 16, 16384, 128, 16
    n = rsa.workspace_size(B, H, L, d, N, False, torch.bfloat16, False, 0)
    info = rsa.plan_describe(B, H, L, d, N, False, torch.bfloat16, False, n)
    assert info["fits"] and n <= (4 << 30)
    hg, rows = info["heads_per_group"], info["rows_per_group"]
    tiles, rt = -(-L // 128), rows // 128
    per_head = -(-L // rows)
    rounds = 0
    for g in range(info["groups"]):
        heads = min(hg, B * H - (g // per_head) * hg)
        t = min(rt, tiles - (g % per_head) * rt)
        assert heads * t >= 96, (g, heads, t)
        rounds += -(-heads * t // 148)
    assert rounds == -(-B * H * tiles // 148) == 14


def test_default_plan_is_capped_at_one_gib(lib):
    n = rsa.workspace_size(1, 16, 16384, 128, 16, False, torch.bfloat16, True, 0)
    assert n <= (1 << 30)
    info = rsa.plan_describe(1, 16, 16384, 128, 16, False, torch.bfloat16, True, n)
    assert info["fits"]


def _fwdn(lib, B=1, H=1, L=128, d=64, N=1, dt=rsa.RSA_BF16, ptr=FAKE, lse=FAKE):
    return lib.rsa_forward_noalloc(ptr, ptr, ptr, ptr, lse, B, H, L, d, N, 0, dt, None)


@pytest.mark.parametrize("bad", [dict(L=100, N=3), dict(B=0), dict(N=0), dict(d=96),
                                 dict(d=128, dt=rsa.RSA_F32), dict(dt=7), dict(ptr=0),
                                 dict(lse=0), dict(ptr=FAKE + 8), dict(L=(1 << 22) + 1024),
                                 dict(B=1 << 12, H=1 << 12, L=1 << 16)])
def test_noalloc_reports_the_codes_forward_reports(lib, bad):
    """The allocation-free forward checks its arguments like rsa_forward, in the same order, so
    the same bad arguments give the same code (and nothing touches a device)."""
    assert _fwdn(lib, **bad) == _fwd(lib, **bad) != rsa.RSA_OK


def test_noalloc_refuses_rows_beyond_its_scratch_before_any_device_call(lib):
    # rows of 70,000 keys: even one 128-row tile of scores exceeds the 32 MiB scratch
    assert _fwdn(lib, L=70000, N=1) == rsa.RSA_ERR_WORKSPACE


def test_status_hook_rejects_codes_a_kernel_never_reports(lib):
    assert lib.rsa_debug_report_status(rsa.RSA_ERR_CUDA, None) == rsa.RSA_ERR_INVALID_ARG
    assert lib.rsa_debug_report_status(-1, None) == rsa.RSA_ERR_INVALID_ARG


def test_bindings_refuse_outputs_on_another_device():
    cpu = torch.empty(4)
    with pytest.raises(ValueError, match="expected cuda:0"):
        rsa._same_device(torch.device("cuda", 0), None, cpu)


def _lin(lib, M=128, N=64, K=64, xk=64, yk=64, ptr=FAKE, res=None, bias=None):
    return lib.rsa_linear(ptr, ptr, bias, res, ptr, M, N, K, xk, yk, 0, None)


def test_linear_argument_errors(lib):
    assert _lin(lib, ptr=0) == rsa.RSA_ERR_INVALID_ARG
    assert _lin(lib, ptr=FAKE + 8) == rsa.RSA_ERR_INVALID_ARG
    assert _lin(lib, M=0) == rsa.RSA_ERR_INVALID_ARG
    assert _lin(lib, M=100) == rsa.RSA_ERR_UNSUPPORTED            # rows not a multiple of 128
    assert _lin(lib, N=96, yk=96) == rsa.RSA_ERR_UNSUPPORTED      # N not a multiple of 64
    assert _lin(lib, K=96, xk=96) == rsa.RSA_ERR_UNSUPPORTED      # K not a multiple of 64
    assert _lin(lib, K=256, xk=96) == rsa.RSA_ERR_UNSUPPORTED     # head width not dividing K
    assert _lin(lib, N=128, yk=64, res=FAKE) == rsa.RSA_ERR_UNSUPPORTED  # residual, split output


def test_host_pipeline_chunking_rule():
    """Groups of (batch, head) slices for the host-buffer call: at most 8, dividing B H, each
    with at least 8 MB of Q, K, V, dO (the choices measured fastest on the long-sequence,
    GPT-style and BERT-shaped steps: 8, 8 and 3)."""
    from sequence_ring_self_b200.rsa import host_chunks

    assert host_chunks(1, 16, 16384, 128) == 8
    assert host_chunks(4, 16, 4096, 64) == 8
    assert host_chunks(8, 12, 512, 64) == 3
    assert host_chunks(1, 2, 256, 64) == 1
    assert host_chunks(1, 7, 65536, 128) == 7
    for B, H, L, d, e in ((1, 16, 16384, 128, 2), (2, 5, 9000, 64, 4), (3, 5, 7000, 64, 2)):
        c = host_chunks(B, H, L, d, e)
        assert 1 <= c <= 8 and (B * H) % c == 0
        assert c == 1 or 4 * (B * H // c) * L * d * e >= 8e6


@pytest.mark.parametrize("chunks", [0, 3, -2])
def test_host_pipeline_rejects_groups_that_do_not_divide_the_slices(chunks):
    """B H = 4 (batch, head) slices cannot be cut into 0, 3 or -2 groups; the call says so
    before it touches a device."""
    from sequence_ring_self_b200 import rsa

    x = torch.zeros(2, 2, 128, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        rsa.forward_backward_host(x, x, x, x, 4, False, device="cuda:0", chunks=chunks)


def test_hbm_probe_argument_errors(lib):
    """The HBM probe refuses bad buffers, sizes, block counts and modes before any launch."""
    vp = ctypes.c_void_p
    probe = lambda buf=FAKE, n=1 << 20, write=0, blocks=8, out=FAKE: lib.rsa_probe_hbm(
        vp(buf), n, write, blocks, vp(out), vp(0))
    assert probe(buf=0) == rsa.RSA_ERR_INVALID_ARG
    assert probe(buf=FAKE + 8) == rsa.RSA_ERR_INVALID_ARG       # not 16-byte aligned
    assert probe(n=0) == rsa.RSA_ERR_INVALID_ARG
    assert probe(n=(1 << 20) + 8) == rsa.RSA_ERR_INVALID_ARG    # not a multiple of 16
    assert probe(blocks=0) == rsa.RSA_ERR_INVALID_ARG
    assert probe(write=2) == rsa.RSA_ERR_INVALID_ARG
    assert probe(out=0) == rsa.RSA_ERR_INVALID_ARG              # the read probe needs `out`
