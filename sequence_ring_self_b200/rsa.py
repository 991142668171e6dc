"""Python binding of the Ring Self-Attention C ABI (``include/rsa.h``).

Argument marshalling only: tensors are checked for shape, dtype, device and layout, and their
device pointers, sizes and the current CUDA stream are passed to the library; every step of
the computation runs in the library's kernels. PyTorch supplies device memory and streams.
There is no fallback: if the CUDA library is missing or the GPU is not sm_100, calls raise.

Method: "Sequence Parallelism: Making 4D Parallelism Possible" (Li, Xue et al., 2021; review
page, Abstract and "Proposed method"): the sequence is cut into N chunks, each chunk's score
slab is built over a ring of key chunks, normalised by a full-row softmax, and multiplied
with the values over a second ring pass; the backward pass runs the same ring.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "_build", "librsa_b200.so")

RSA_OK, RSA_ERR_INVALID_ARG, RSA_ERR_UNSUPPORTED, RSA_ERR_WORKSPACE, RSA_ERR_CUDA, RSA_ERR_TIMEOUT = range(6)
RSA_F32, RSA_BF16 = 0, 1

EXPORTED = ("rsa_workspace_size", "rsa_forward", "rsa_backward", "rsa_status_string",
            "rsa_last_device_status", "rsa_plan_describe", "rsa_profile_enable",
            "rsa_profile_kinds", "rsa_profile_kind_name", "rsa_profile_read",
            "rsa_forward_noalloc", "rsa_last_error", "rsa_forward_recompute",
            "rsa_probe_ffma", "rsa_probe_ffma_flops_per_thread", "rsa_probe_hbm",
            "rsa_debug_report_status",
            # include/rsa_sp.h
            "rsa_sp_workspace_size", "rsa_sp_scores", "rsa_sp_softmax_pv", "rsa_sp_backward_rows",
            "rsa_sp_backward_keys", "rsa_sp_accumulate", "rsa_linear")

_lib = None
_lock = threading.Lock()


class RSAError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        msg = f"{what}: {status_string(code)} ({code})"
        if code == RSA_ERR_CUDA:
            detail = load_library().rsa_last_error().decode(errors="replace")
            if detail:
                msg += f" [{detail}]"
        super().__init__(msg)


def load_library(path: str | None = None):
    """Load the CUDA library (it must have been built; see ``sequence_ring_self_b200.build``)."""
    global _lib
    with _lock:
        if _lib is not None and path is None:
            return _lib
        p = path or LIB_PATH
        if not os.path.exists(p):
            raise ImportError(f"Ring Self-Attention CUDA library not built: {p} is missing "
                              "(run `python -m sequence_ring_self_b200.build`)")
        lib = ctypes.CDLL(p)
        vp, sz, i = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
        lib.rsa_workspace_size.argtypes = [i, i, i, i, i, i, i, i, sz]
        lib.rsa_workspace_size.restype = sz
        lib.rsa_forward.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, i, vp, sz, vp]
        lib.rsa_forward.restype = i
        lib.rsa_backward.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, vp, sz,
                                     vp]
        lib.rsa_backward.restype = i
        lib.rsa_status_string.argtypes = [i]
        lib.rsa_status_string.restype = ctypes.c_char_p
        lib.rsa_last_error.argtypes = []
        lib.rsa_last_error.restype = ctypes.c_char_p
        lib.rsa_last_device_status.argtypes = [vp]
        lib.rsa_last_device_status.restype = i
        lib.rsa_plan_describe.argtypes = [i, i, i, i, i, i, i, i, sz, ctypes.POINTER(ctypes.c_longlong)]
        lib.rsa_plan_describe.restype = i
        lib.rsa_profile_enable.argtypes = [i]
        lib.rsa_profile_enable.restype = i
        lib.rsa_profile_kinds.argtypes = []
        lib.rsa_profile_kinds.restype = i
        lib.rsa_profile_kind_name.argtypes = [i]
        lib.rsa_profile_kind_name.restype = ctypes.c_char_p
        lib.rsa_profile_read.argtypes = [ctypes.POINTER(ctypes.c_double),
                                         ctypes.POINTER(ctypes.c_longlong)]
        lib.rsa_profile_read.restype = i
        lib.rsa_forward_noalloc.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, i, vp]
        lib.rsa_forward_noalloc.restype = i
        lib.rsa_forward_recompute.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, i, vp]
        lib.rsa_forward_recompute.restype = i
        lib.rsa_probe_ffma.argtypes = [vp, i, i, vp]
        lib.rsa_probe_ffma.restype = i
        lib.rsa_probe_ffma_flops_per_thread.argtypes = [i]
        lib.rsa_probe_ffma_flops_per_thread.restype = ctypes.c_longlong
        lib.rsa_probe_hbm.argtypes = [vp, sz, i, i, vp, vp]
        lib.rsa_probe_hbm.restype = i
        lib.rsa_debug_report_status.argtypes = [i, vp]
        lib.rsa_debug_report_status.restype = i
        lib.rsa_linear.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, vp]
        lib.rsa_linear.restype = i
        if path is None:
            _lib = lib
        return lib


def status_string(code: int) -> str:
    return load_library().rsa_status_string(int(code)).decode()


def _dtype_code(dtype: torch.dtype) -> int:
    if dtype == torch.bfloat16:
        return RSA_BF16
    if dtype == torch.float32:
        return RSA_F32
    raise TypeError(f"unsupported dtype {dtype}; use torch.bfloat16 or torch.float32")


def workspace_size(B: int, H: int, L: int, d: int, N: int, causal: bool, dtype: torch.dtype,
                   for_backward: bool, budget_bytes: int = 0) -> int:
    """Workspace bytes for the plan that fits ``budget_bytes`` (0: the default plan)."""
    n = load_library().rsa_workspace_size(B, H, L, d, N, int(bool(causal)), _dtype_code(dtype),
                                          int(bool(for_backward)), int(budget_bytes))
    if n == 0:
        raise RSAError(RSA_ERR_INVALID_ARG, "rsa_workspace_size")
    return int(n)


def plan_describe(B: int, H: int, L: int, d: int, N: int, causal: bool, dtype: torch.dtype,
                  for_backward: bool, ws_bytes: int) -> dict:
    out = (ctypes.c_longlong * 5)()
    rc = load_library().rsa_plan_describe(B, H, L, d, N, int(bool(causal)), _dtype_code(dtype),
                                          int(bool(for_backward)), int(ws_bytes), out)
    if rc not in (RSA_OK, RSA_ERR_WORKSPACE):
        raise RSAError(rc, "rsa_plan_describe")
    return {"groups": out[0], "heads_per_group": out[1], "rows_per_group": out[2],
            "padded_row": out[3], "bytes": out[4], "fits": rc == RSA_OK}


def last_device_status(stream: torch.cuda.Stream | None = None) -> int:
    """Status the kernels reported on the stream's device (RSA_OK or RSA_ERR_TIMEOUT) since the
    last call; synchronises the stream and clears the status."""
    s = stream if stream is not None else torch.cuda.current_stream()
    with torch.cuda.device(s.device):
        return int(load_library().rsa_last_device_status(ctypes.c_void_p(s.cuda_stream)))


def debug_report_status(code: int, stream: torch.cuda.Stream | None = None) -> None:
    """Post a status code into the device status word from the GPU, as a kernel whose bounded
    wait gave up does (a failure-injection hook for testing the reporting path)."""
    s = stream if stream is not None else torch.cuda.current_stream()
    with torch.cuda.device(s.device):
        rc = load_library().rsa_debug_report_status(int(code), ctypes.c_void_p(s.cuda_stream))
    if rc != RSA_OK:
        raise RSAError(rc, "rsa_debug_report_status")


def profile_enable(on: bool) -> None:
    """Bracket every library kernel launch with CUDA events on its stream (benchmarks)."""
    rc = load_library().rsa_profile_enable(int(bool(on)))
    if rc != RSA_OK:
        raise RSAError(rc, "rsa_profile_enable")


def profile_read() -> dict:
    """{kernel name: (total ms, launches)} accumulated since the last read; waits for the events."""
    lib = load_library()
    n = lib.rsa_profile_kinds()
    ms = (ctypes.c_double * n)()
    cnt = (ctypes.c_longlong * n)()
    rc = lib.rsa_profile_read(ms, cnt)
    if rc != RSA_OK:
        raise RSAError(rc, "rsa_profile_read")
    return {lib.rsa_profile_kind_name(k).decode(): (ms[k], cnt[k]) for k in range(n) if cnt[k]}


def _check_qkv(*ts):
    q = ts[0]
    if q.dim() != 4:
        raise ValueError("tensors must be [B, H, L, d]")
    for t in ts:
        if t.shape != q.shape or t.dtype != q.dtype or t.device != q.device:
            raise ValueError("Q, K, V (and O, dO) must share shape, dtype and device")
        if not t.is_cuda:
            raise ValueError("tensors must be on a CUDA device")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous [B, H, L, d]")


def _workspace(nbytes: int, device, workspace):
    """A caller-supplied workspace is used as it is (the library plans for its size and
    reports RSA_ERR_WORKSPACE if it is below the smallest plan); otherwise one of the size
    the budget asks for is allocated."""
    if workspace is None:
        return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
    if not workspace.is_cuda or workspace.device != device:
        raise ValueError("workspace must be on the tensors' device")
    return workspace


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _same_device(device, *ts):
    """Outputs and workspaces given by the caller must live on the inputs' device."""
    for t in ts:
        if t is not None and t.device != device:
            raise ValueError(f"tensor on {t.device}, expected {device} (the inputs' device)")


def forward(q, k, v, N: int, causal: bool = False, *, ws_budget: int = 0, workspace=None,
            out=None, lse=None, stream: torch.cuda.Stream | None = None):
    """Ring Self-Attention forward. Returns (O [B,H,L,d] in the input dtype, lse [B,H,L] fp32)."""
    _check_qkv(q, k, v)
    _same_device(q.device, out, lse)
    B, H, L, d = q.shape
    dt = _dtype_code(q.dtype)
    lib = load_library()
    nbytes = lib.rsa_workspace_size(B, H, L, d, N, int(bool(causal)), dt, 0, int(ws_budget))
    if nbytes == 0:
        raise RSAError(RSA_ERR_INVALID_ARG, "rsa_forward")
    # the library runs on the current device: make it the tensors' device for the call
    with torch.cuda.device(q.device):
        ws = _workspace(nbytes, q.device, workspace)
        o = torch.empty_like(q) if out is None else out
        ls = torch.empty((B, H, L), dtype=torch.float32, device=q.device) if lse is None else lse
        s = stream if stream is not None else torch.cuda.current_stream(q.device)
        rc = lib.rsa_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(ls), B, H, L, d, N,
                             int(bool(causal)), dt, _ptr(ws), ws.numel() * ws.element_size(),
                             ctypes.c_void_p(s.cuda_stream))
    if rc != RSA_OK:
        raise RSAError(rc, "rsa_forward")
    return o, ls


def forward_recompute(q, k, v, N: int, causal: bool = False, *, out=None, lse=None,
                      stream: torch.cuda.Stream | None = None):
    """Slab-free two-pass forward (bf16): returns (O, lse) like ``forward`` without a workspace."""
    _check_qkv(q, k, v)
    _same_device(q.device, out, lse)
    B, H, L, d = q.shape
    dt = _dtype_code(q.dtype)
    lib = load_library()
    with torch.cuda.device(q.device):
        o = torch.empty_like(q) if out is None else out
        ls = torch.empty((B, H, L), dtype=torch.float32, device=q.device) if lse is None else lse
        s = stream if stream is not None else torch.cuda.current_stream(q.device)
        rc = lib.rsa_forward_recompute(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(ls), B, H, L, d, N,
                                       int(bool(causal)), dt, ctypes.c_void_p(s.cuda_stream))
    if rc != RSA_OK:
        raise RSAError(rc, "rsa_forward_recompute")
    return o, ls


def backward(q, k, v, o, do, lse, N: int, causal: bool = False, *, ws_budget: int = 0,
             workspace=None, dq=None, dk=None, dv=None, stream: torch.cuda.Stream | None = None):
    """Ring Self-Attention backward. Returns (dQ, dK, dV) in the input dtype."""
    _check_qkv(q, k, v, o, do)
    _same_device(q.device, lse, dq, dk, dv)
    B, H, L, d = q.shape
    if lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, L) or not lse.is_contiguous():
        raise ValueError("lse must be contiguous fp32 [B, H, L]")
    dt = _dtype_code(q.dtype)
    lib = load_library()
    nbytes = lib.rsa_workspace_size(B, H, L, d, N, int(bool(causal)), dt, 1, int(ws_budget))
    if nbytes == 0:
        raise RSAError(RSA_ERR_INVALID_ARG, "rsa_backward")
    with torch.cuda.device(q.device):
        ws = _workspace(nbytes, q.device, workspace)
        dq = torch.empty_like(q) if dq is None else dq
        dk = torch.empty_like(q) if dk is None else dk
        dv = torch.empty_like(q) if dv is None else dv
        s = stream if stream is not None else torch.cuda.current_stream(q.device)
        rc = lib.rsa_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse), _ptr(dq),
                              _ptr(dk), _ptr(dv), B, H, L, d, N, int(bool(causal)), dt, _ptr(ws),
                              ws.numel() * ws.element_size(), ctypes.c_void_p(s.cuda_stream))
    if rc != RSA_OK:
        raise RSAError(rc, "rsa_backward")
    return dq, dk, dv


def forward_noalloc(q, k, v, N: int, causal: bool = False, *, out=None, lse=None,
                    stream: torch.cuda.Stream | None = None):
    """rsa_forward without a caller workspace: the library works in its own fixed scratch
    array (RSA_NOALLOC_SCRATCH_BYTES per GPU), for callers that may not allocate device
    memory. Pass `out` and `lse` to allocate nothing here either. Calls on one device share
    the scratch, so calls that overlap on the GPU must not be issued."""
    _check_qkv(q, k, v)
    _same_device(q.device, out, lse)
    B, H, L, d = q.shape
    with torch.cuda.device(q.device):
        o = torch.empty_like(q) if out is None else out
        ls = torch.empty((B, H, L), dtype=torch.float32, device=q.device) if lse is None else lse
        s = stream if stream is not None else torch.cuda.current_stream(q.device)
        rc = load_library().rsa_forward_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(ls), B, H,
                                                L, d, N, int(bool(causal)), _dtype_code(q.dtype),
                                                ctypes.c_void_p(s.cuda_stream))
    if rc != RSA_OK:
        raise RSAError(rc, "rsa_forward_noalloc")
    return o, ls


class RingSelfAttention(torch.autograd.Function):
    """autograd wrapper: ``RingSelfAttention.apply(q, k, v, N, causal)`` -> O."""

    @staticmethod
    def forward(ctx, q, k, v, N, causal=False):
        o, lse = forward(q, k, v, N, causal)
        ctx.save_for_backward(q, k, v, o, lse)
        ctx.N, ctx.causal = N, causal
        return o

    @staticmethod
    def backward(ctx, do):
        q, k, v, o, lse = ctx.saved_tensors
        dq, dk, dv = backward(q, k, v, o, do.contiguous(), lse, ctx.N, ctx.causal)
        return dq, dk, dv, None, None


def host_chunks(B: int, H: int, L: int, d: int, elsize: int = 2) -> int:
    """How many groups of (batch, head) slices ``forward_backward_host`` pipelines: the most,
    up to 8, that divides B H and still gives each group at least 8 MB of Q, K, V and dO to
    copy. Issuing a group costs the host about a quarter of a millisecond, about what 8 MB
    takes over PCIe, so smaller groups would leave the GPU waiting for the host."""
    BH = B * H
    for c in range(min(8, BH), 1, -1):
        if BH % c == 0 and 4 * (BH // c) * L * d * elsize >= 8e6:
            return c
    return 1


def forward_backward_host(q, k, v, do, N: int, causal: bool = False, *, ws_budget: int = 0,
                          device=None, results=None, recompute: bool = False,
                          chunks: int | None = None):
    """One forward + backward from host (ideally pinned) tensors: copies Q, K, V, dO to the
    device, runs the library's forward and backward there, and copies O, lse, dQ, dK, dV
    back into host tensors (``results`` if given, a dict of pinned tensors by name).
    ``recompute`` selects the slab-free forward.

    Attention is independent across the B H (batch, head) slices, so the call runs as a
    pipeline over ``chunks`` groups of slices (default ``host_chunks``): the copies of group
    c + 1 to the device (one side stream) overlap the forward of group c, dO arrives while the
    forwards run, and O, lse and the gradients of each group go back to the host (a second
    side stream, the other PCIe direction) while the next group computes. Every group is one
    library call on [1, B H / chunks, L, d] views, so the results equal those of a single call
    bit for bit. All work is ordered before the current stream's later work: synchronising the
    current stream covers the results."""
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    B, H, L, d = q.shape
    BH = B * H
    C = host_chunks(B, H, L, d, q.element_size()) if chunks is None else int(chunks)
    if C < 1 or BH % C:
        raise ValueError(f"chunks = {C} must divide B H = {BH}")
    n = BH // C
    flat = lambda t: t.reshape(BH, *t.shape[2:])
    piece = lambda t, c: flat(t)[c * n:(c + 1) * n]
    with torch.cuda.device(dev):
        main = torch.cuda.current_stream(dev)
        h2d, d2h = _side_streams(dev)
        if results is None:
            results = {nm: torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
                       for nm in ("O", "dQ", "dK", "dV")}
            results["lse"] = torch.empty((B, H, L), dtype=torch.float32, pin_memory=True)
        # device buffers belong to the current stream; the side streams finish with them
        # before it goes on (it waits on their events below and on d2h at the end)
        qd, kd, vd, dod, o, dq, dk, dv = (torch.empty(q.shape, dtype=q.dtype, device=dev)
                                          for _ in range(8))
        lse = torch.empty((B, H, L), dtype=torch.float32, device=dev)
        h2d.wait_stream(main)  # host and device buffers may still be in use by earlier work
        d2h.wait_stream(main)
        in_ready, do_ready = [], []
        with torch.cuda.stream(h2d):
            for c in range(C):
                for src, dst in ((q, qd), (k, kd), (v, vd)):
                    piece(dst, c).copy_(piece(src, c), non_blocking=True)
                in_ready.append(torch.cuda.Event())
                in_ready[-1].record(h2d)
            for c in range(C):
                piece(dod, c).copy_(piece(do, c), non_blocking=True)
                do_ready.append(torch.cuda.Event())
                do_ready[-1].record(h2d)
        view = lambda t, c: piece(t, c).unsqueeze(0)  # [1, n, L, d] or [1, n, L]
        for c in range(C):
            main.wait_event(in_ready[c])
            if recompute:
                forward_recompute(view(qd, c), view(kd, c), view(vd, c), N, causal,
                                  out=view(o, c), lse=view(lse, c))
            else:
                forward(view(qd, c), view(kd, c), view(vd, c), N, causal, ws_budget=ws_budget,
                        out=view(o, c), lse=view(lse, c))
            done = torch.cuda.Event()
            done.record(main)
            d2h.wait_event(done)
            with torch.cuda.stream(d2h):
                piece(results["O"], c).copy_(piece(o, c), non_blocking=True)
                piece(results["lse"], c).copy_(piece(lse, c), non_blocking=True)
        for c in range(C):
            main.wait_event(do_ready[c])
            backward(view(qd, c), view(kd, c), view(vd, c), view(o, c), view(dod, c),
                     view(lse, c), N, causal, ws_budget=ws_budget, dq=view(dq, c),
                     dk=view(dk, c), dv=view(dv, c))
            done = torch.cuda.Event()
            done.record(main)
            d2h.wait_event(done)
            with torch.cuda.stream(d2h):
                for nm, t in (("dQ", dq), ("dK", dk), ("dV", dv)):
                    piece(results[nm], c).copy_(piece(t, c), non_blocking=True)
        main.wait_stream(d2h)
    return results


_SIDE = {}


def _side_streams(dev):
    """Two side streams per device (host-to-device and device-to-host copies), made once."""
    key = dev.index if dev.index is not None else torch.cuda.current_device()
    if key not in _SIDE:
        _SIDE[key] = (torch.cuda.Stream(dev), torch.cuda.Stream(dev))
    return _SIDE[key]

def linear(x, w, bias=None, residual=None, gelu: bool = False, *, x_kin: int | None = None,
           y_kin: int | None = None, out=None, stream: torch.cuda.Stream | None = None):
    """Y = act(X W^T + bias) + residual on M rows (include/rsa_sp.h, rsa_linear), bf16.

    x: [M, K] bf16, or (x_kin = d) the [H, M, d] output of attention read as [M, H d];
    w: [N, K] bf16; bias: [N] fp32 or None; residual: [M, N] bf16 or None.
    Returns Y [M, N], or with y_kin = d the [N / d, M, d] layout (the query/key/value
    projection written for attention)."""
    if x.dtype != torch.bfloat16 or w.dtype != torch.bfloat16:
        raise TypeError("linear takes bf16 X and W")
    if not (x.is_contiguous() and w.is_contiguous()):
        raise ValueError("X and W must be contiguous")
    N, K = w.shape
    if x.dim() == 2:
        M = x.shape[0]
        xk = K if x_kin is None else x_kin
        if x.shape[1] != K or xk != K:
            raise ValueError("X [M, K] must match W [N, K]")
    elif x.dim() == 3:
        M = x.shape[1]
        xk = x.shape[2]
        if x_kin not in (None, xk) or x.shape[0] * xk != K:
            raise ValueError("X [H, M, d] must have H d = K")
    else:
        raise ValueError("X must be [M, K] or [H, M, d]")
    yk = N if y_kin is None else y_kin
    if bias is not None and (bias.dtype != torch.float32 or tuple(bias.shape) != (N,)):
        raise ValueError("bias must be fp32 [N]")
    if residual is not None and (residual.dtype != torch.bfloat16 or tuple(residual.shape) != (M, N)
                                 or not residual.is_contiguous()):
        raise ValueError("residual must be contiguous bf16 [M, N]")
    _same_device(x.device, w, bias, residual, out)
    shape = (M, N) if yk == N else (N // yk, M, yk)
    with torch.cuda.device(x.device):
        y = torch.empty(shape, dtype=torch.bfloat16, device=x.device) if out is None else out
        s = stream if stream is not None else torch.cuda.current_stream(x.device)
        rc = load_library().rsa_linear(_ptr(x), _ptr(w), _ptr(bias) if bias is not None else None,
                                       _ptr(residual) if residual is not None else None, _ptr(y),
                                       M, N, K, xk, yk, int(bool(gelu)), ctypes.c_void_p(s.cuda_stream))
    if rc != RSA_OK:
        raise RSAError(rc, "rsa_linear")
    return y
