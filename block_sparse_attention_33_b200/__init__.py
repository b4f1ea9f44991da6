"""Python binding of libspattn (routed block-sparse attention for B200).

Argument marshalling only: every step of the path runs in the CUDA kernels of
``libspattn.so``.  Tensors may be passed as torch tensors (their device
pointer is used, after their dtype, device, contiguity and size are checked
against the plan, so that a wrong tensor is refused before a kernel reads
past it) or as raw integer addresses (passed through unchecked).  There is
no fallback: if the library is missing, importing a function raises.

The functions carry the names of the C entry points in ``include/spattn.h``.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libspattn.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, ERR_TIMEOUT, ERR_DEVICE = range(7)
STATUS_NAMES = {0: "OK", 1: "INVALID_ARG", 2: "UNSUPPORTED", 3: "WORKSPACE", 4: "CUDA",
                5: "TIMEOUT", 6: "DEVICE"}

ROUTING_CENTROID, ROUTING_PAMA = 0, 1
SELECT_THRESHOLD = 16   # OR into routing: tau is the per-block threshold theta on p
SELECT_INLINE = 32      # OR into routing: the attention kernel selects (no routing launch)

EXPORTS = ("spattn_plan", "spattn_plan_ex", "spattn_plan_destroy", "spattn_plan_info", "spattn_pool",
           "spattn_route", "spattn_attend", "spattn_forward", "spattn_means", "spattn_check",
           "spattn_hilbert_perm", "spattn_route_static", "spattn_host_staging_bytes",
           "spattn_forward_host", "spattn_probe_scratch_bytes", "spattn_probe_correct",
           "spattn_last_error")


class SpAttnError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"spattn status {STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


_lib = None
# plan handle -> (B, H, N, d, nb, col_capacity, workspace_bytes), for the
# tensor checks of the calls that take a handle
_PLANS = {}


def lib():
    """Load libspattn.so (built in-tree by build.build()); raise if absent."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -c 'import __graft_entry__ as g; g.build()'`")
    L = ctypes.CDLL(LIB_PATH)
    P, I, F, S, I32P, SZP = (ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t,
                             ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_size_t))
    sig = {
        "spattn_plan": [ctypes.POINTER(P), I, I, I, I, I, F, I, I, I, P, SZP],
        "spattn_plan_ex": [ctypes.POINTER(P), I, I, I, I, I, F, I, I, I, P, I, SZP],
        "spattn_plan_destroy": [P],
        "spattn_plan_info": [P, ctypes.POINTER(I), ctypes.POINTER(ctypes.c_int64)],
        "spattn_pool": [P, P, P, P, P, P],
        "spattn_route": [P, P, P, P, P, P, P, P],
        "spattn_attend": [P, P, P, P, P, P, P, P, P],
        "spattn_forward": [P, P, P, P, P, P, P],
        "spattn_means": [P, P, P, P, P, P],
        "spattn_check": [P, P, P],
        "spattn_hilbert_perm": [I, I, I, P],
        "spattn_route_static": [I, I, I, I, I, F, I, I, P, P, P, P, P, P],
        "spattn_host_staging_bytes": [P, I, SZP],
        "spattn_forward_host": [P, P, P, P, P, P, P, I, P],
        "spattn_probe_scratch_bytes": [P, I, SZP],
        "spattn_probe_correct": [P, P, P, P, P, P, I, F, I, P, P, P],
    }
    for name, args in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = ctypes.c_int
    L.spattn_last_error.argtypes = []
    L.spattn_last_error.restype = ctypes.c_char_p
    _lib = L
    return L


def _devs(*specs):
    """Pointers of device arguments, each spec (x, name, dtype, numel, exact).
    A torch tensor must be a contiguous CUDA tensor of `dtype` ("bfloat16",
    "float32", "int32" or "uint8") holding at least (exactly, if `exact`)
    `numel` elements; raw addresses and None pass through.  Every argument's
    dtype, layout and size are checked before any argument's device."""
    for x, name, dtype, numel, exact in specs:
        if x is None or isinstance(x, int):
            continue
        if not hasattr(x, "data_ptr"):
            raise TypeError(f"{name}: expected a torch CUDA tensor or an address, got {type(x)}")
        if str(x.dtype) != "torch." + dtype:
            raise ValueError(f"{name}: dtype must be torch.{dtype}, got {x.dtype}")
        if not x.is_contiguous():
            raise ValueError(f"{name}: must be contiguous")
        n = x.numel()
        if (n != numel) if exact else (n < numel):
            raise ValueError(f"{name}: needs {'exactly' if exact else 'at least'} {numel} "
                             f"elements, has {n}")
    out = []
    for x, name, *_ in specs:
        if x is None or isinstance(x, int):
            out.append(x)
            continue
        if not x.is_cuda:
            raise ValueError(f"{name}: must be a CUDA tensor")
        out.append(x.data_ptr())
    return out


def _hosts(*specs):
    """Pointers of host arguments, each spec (x, name, dtype, numel): a torch
    CPU tensor of `dtype`, contiguous, with exactly `numel` elements (pinned
    memory lets the library's copies run asynchronously); raw addresses pass
    through."""
    out = []
    for x, name, dtype, numel in specs:
        if isinstance(x, int):
            out.append(x)
            continue
        if not hasattr(x, "data_ptr"):
            raise TypeError(f"{name}: expected a torch CPU tensor or an address, got {type(x)}")
        if x.is_cuda:
            raise ValueError(f"{name}: must be a host (CPU) tensor")
        if str(x.dtype) != "torch." + dtype:
            raise ValueError(f"{name}: dtype must be torch.{dtype}, got {x.dtype}")
        if not x.is_contiguous():
            raise ValueError(f"{name}: must be contiguous")
        if x.numel() != numel:
            raise ValueError(f"{name}: needs exactly {numel} elements, has {x.numel()}")
        out.append(x.data_ptr())
    return out


def _shape(plan):
    try:
        return _PLANS[plan]
    except KeyError:
        raise ValueError("unknown or destroyed plan handle") from None


def _tokens(plan, **xs):
    """Specs of bf16 [B, H, N, d] arguments of a plan."""
    B, H, N, d = _shape(plan)[:4]
    return [(x, k, "bfloat16", B * H * N * d, True) for k, x in xs.items()]


def _workspace(plan, ws):
    return (ws, "workspace", "uint8", _shape(plan)[6], False)


def _csr(plan, row_ptr, col_idx, col_min):
    B, H, _, _, nb = _shape(plan)[:5]
    return [(row_ptr, "row_ptr", "int32", B * H * nb + 1, False),
            (col_idx, "col_idx", "int32", col_min, False)]


def _stream(s) -> Optional[int]:
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(st: int):
    if st != OK:
        raise SpAttnError(st, lib().spattn_last_error().decode())


def spattn_last_error() -> str:
    return lib().spattn_last_error().decode()


def spattn_plan(B, H, N, d, b, tau, kmin, kmax, residual, perm=None):
    """Create a plan; returns (handle, workspace_bytes).  perm: host int32 array or None."""
    return spattn_plan_ex(B, H, N, d, b, tau, kmin, kmax, residual, perm, ROUTING_CENTROID)


def spattn_plan_ex(B, H, N, d, b, tau, kmin, kmax, residual, perm=None, routing=ROUTING_CENTROID):
    """spattn_plan with a routing estimate (ROUTING_CENTROID or ROUTING_PAMA),
    optionally | SELECT_THRESHOLD (tau is then the per-block threshold)."""
    import numpy as np
    h = ctypes.c_void_p()
    ws = ctypes.c_size_t()
    pp = None
    if perm is not None:
        perm = np.ascontiguousarray(perm, dtype=np.int32)
        pp = perm.ctypes.data
    _check(lib().spattn_plan_ex(ctypes.byref(h), B, H, N, d, b, float(tau), kmin, kmax, residual,
                                pp, int(routing), ctypes.byref(ws)))
    nb = (N + b - 1) // b
    _PLANS[h.value] = (B, H, N, d, nb, B * H * nb * min(kmax, nb), ws.value)
    return h.value, ws.value


def spattn_plan_destroy(plan):
    _check(lib().spattn_plan_destroy(plan))
    _PLANS.pop(plan, None)


def spattn_plan_info(plan):
    nb = ctypes.c_int()
    cap = ctypes.c_int64()
    _check(lib().spattn_plan_info(plan, ctypes.byref(nb), ctypes.byref(cap)))
    return nb.value, cap.value


def spattn_pool(plan, Q, K, V, workspace, stream=None):
    q, k, v, w = _devs(*_tokens(plan, Q=Q, K=K, V=V), _workspace(plan, workspace))
    _check(lib().spattn_pool(plan, q, k, v, w, _stream(stream)))


def spattn_route(plan, Q, K, V, workspace, row_ptr=None, col_idx=None, stream=None):
    q, k, v, w, rp, ci = _devs(*_tokens(plan, Q=Q, K=K, V=V), _workspace(plan, workspace),
                               *_csr(plan, row_ptr, col_idx, _shape(plan)[5]))
    _check(lib().spattn_route(plan, q, k, v, w, rp, ci, _stream(stream)))


def spattn_attend(plan, Q, K, V, O, workspace, row_ptr=None, col_idx=None, stream=None):
    """row_ptr/col_idx: None (the workspace's kept lists) or a caller CSR;
    col_idx must hold every entry that row_ptr points at (not checked here)."""
    q, k, v, o, w, rp, ci = _devs(*_tokens(plan, Q=Q, K=K, V=V, O=O), _workspace(plan, workspace),
                                  *_csr(plan, row_ptr, col_idx, 0))
    _check(lib().spattn_attend(plan, q, k, v, rp, ci, o, w, _stream(stream)))


def spattn_forward(plan, Q, K, V, O, workspace, stream=None):
    q, k, v, o, w = _devs(*_tokens(plan, Q=Q, K=K, V=V, O=O), _workspace(plan, workspace))
    _check(lib().spattn_forward(plan, q, k, v, o, w, _stream(stream)))


def spattn_host_staging_bytes(plan, chunk_heads) -> int:
    n = ctypes.c_size_t()
    _check(lib().spattn_host_staging_bytes(plan, int(chunk_heads), ctypes.byref(n)))
    return n.value


def spattn_forward_host(plan, Q, K, V, O, workspace, staging, chunk_heads, stream=None):
    """spattn_forward on host tensors, copies overlapped over chunks of
    chunk_heads (batch, head) pairs; synchronise the stream before reading O."""
    B, H, N, d = _shape(plan)[:4]
    q, k, v, o = _hosts(*[(x, n, "bfloat16", B * H * N * d)
                          for n, x in (("Q", Q), ("K", K), ("V", V), ("O", O))])
    w, st = _devs(_workspace(plan, workspace),
                  (staging, "staging", "uint8", spattn_host_staging_bytes(plan, chunk_heads), False))
    _check(lib().spattn_forward_host(plan, q, k, v, o, w, st, int(chunk_heads), _stream(stream)))


def spattn_probe_scratch_bytes(plan, M) -> int:
    n = ctypes.c_size_t()
    _check(lib().spattn_probe_scratch_bytes(plan, int(M), ctypes.byref(n)))
    return n.value


def spattn_probe_correct(plan, Q, K, V, O, probes, M, lam, r, workspace, scratch, stream=None):
    """Probe-fitted residual correction of the routed output O, in place.
    probes: int32 device tensor [B, H, M] of token indices."""
    B, H = _shape(plan)[:2]
    q, k, v, o, pr, w, st = _devs(*_tokens(plan, Q=Q, K=K, V=V, O=O),
                                  (probes, "probes", "int32", B * H * int(M), True),
                                  _workspace(plan, workspace),
                                  (scratch, "scratch", "uint8", spattn_probe_scratch_bytes(plan, M),
                                   False))
    _check(lib().spattn_probe_correct(plan, q, k, v, o, pr, int(M), float(lam), int(r), w, st,
                                      _stream(stream)))


def spattn_means(plan, workspace, Qbar=None, Kbar=None, Vbar=None, stream=None):
    B, H, _, d, nb = _shape(plan)[:5]
    w, *bars = _devs(_workspace(plan, workspace),
                     *[(x, n, "float32", B * H * nb * d, False)
                       for n, x in (("Qbar", Qbar), ("Kbar", Kbar), ("Vbar", Vbar))])
    _check(lib().spattn_means(plan, w, *bars, _stream(stream)))


def spattn_check(plan, workspace, stream=None) -> int:
    """Synchronise and return the device status code (does not raise)."""
    (w,) = _devs(_workspace(plan, workspace))
    return lib().spattn_check(plan, w, _stream(stream))


def spattn_hilbert_perm(T, Hs, W):
    """perm[new] = old for a T x Hs x W grid along the library's 3D Hilbert curve."""
    import numpy as np
    out = np.empty(T * Hs * W, dtype=np.int32)
    _check(lib().spattn_hilbert_perm(T, Hs, W, out.ctypes.data))
    return out


def spattn_route_static(B, H, N, d, b, tau, kmin, kmax, Q, K, row_ptr, col_idx, perm=None,
                        stream=None):
    """Routing with no device allocation (scratch in the library's static
    device array); same CSR as spattn_route.  perm: None or a device int32
    tensor of N entries."""
    nb = (N + b - 1) // b
    tok = B * H * N * d
    q, k, rp, ci, pp = _devs((Q, "Q", "bfloat16", tok, True), (K, "K", "bfloat16", tok, True),
                             (row_ptr, "row_ptr", "int32", B * H * nb + 1, False),
                             (col_idx, "col_idx", "int32", B * H * nb * min(max(kmax, 0), nb), False),
                             (perm, "perm", "int32", N, True))
    _check(lib().spattn_route_static(B, H, N, d, b, float(tau), kmin, kmax, pp, q, k, rp, ci,
                                     _stream(stream)))


def default_chunk_heads(bh: int) -> int:
    """Heads per chunk of the host pipeline: the copies of the first chunk in
    and the last chunk out are exposed (they grow with the chunk), and so is
    the last wave of every chunk's attention (it grows with the number of
    chunks); about sqrt(BH / 5) balances the two.  Measured on one B200 for
    24 heads of the HunyuanVideo-like layer: 903, 933, 932, 921, 910 and 890
    TFLOP/s end to end for 1, 2, 3, 4, 6 and 8 heads per chunk."""
    return max(1, min(bh, int(round((bh / 5.0) ** 0.5))))


class Plan:
    """Owning wrapper: a plan plus its device workspace (torch allocation)."""

    def __init__(self, B, H, N, d, b, tau, kmin, kmax, residual, perm=None, device="cuda",
                 routing=ROUTING_CENTROID):
        import torch
        self.shape = (B, H, N, d)
        self.handle, self.ws_bytes = spattn_plan_ex(B, H, N, d, b, tau, kmin, kmax, residual, perm,
                                                    routing)
        self.nb, self.col_capacity = spattn_plan_info(self.handle)
        self.workspace = torch.empty(max(self.ws_bytes, 256), dtype=torch.uint8, device=device)

    def forward(self, Q, K, V, O, stream=None):
        spattn_forward(self.handle, Q, K, V, O, self.workspace, stream)

    def probe_correct(self, Q, K, V, O, probes, lam, r, stream=None):
        """Probe-fitted residual correction of O (the output of forward on the
        same inputs), in place.  probes: int32 device tensor [B, H, M]."""
        import torch
        M = probes.shape[-1]
        need = spattn_probe_scratch_bytes(self.handle, M)
        if getattr(self, "probe_scratch", None) is None or self.probe_scratch.numel() < need:
            self.probe_scratch = torch.empty(need, dtype=torch.uint8, device=self.workspace.device)
        spattn_probe_correct(self.handle, Q, K, V, O, probes, M, lam, r, self.workspace,
                             self.probe_scratch, stream)

    def forward_host(self, Q, K, V, O, chunk_heads=None, stream=None):
        """Forward on host tensors (pinned for overlap); the device staging
        is allocated on first use.  Default chunk: default_chunk_heads."""
        import torch
        B, H = self.shape[:2]
        c = chunk_heads or default_chunk_heads(B * H)
        need = spattn_host_staging_bytes(self.handle, c)
        if getattr(self, "staging", None) is None or self.staging.numel() < need:
            self.staging = torch.empty(need, dtype=torch.uint8, device=self.workspace.device)
        spattn_forward_host(self.handle, Q, K, V, O, self.workspace, self.staging, c, stream)

    def route(self, Q, K, V, row_ptr=None, col_idx=None, stream=None):
        spattn_route(self.handle, Q, K, V, self.workspace, row_ptr, col_idx, stream)

    def attend(self, Q, K, V, O, row_ptr=None, col_idx=None, stream=None):
        spattn_attend(self.handle, Q, K, V, O, self.workspace, row_ptr, col_idx, stream)

    def pool(self, Q, K, V, stream=None):
        spattn_pool(self.handle, Q, K, V, self.workspace, stream)

    def check(self, stream=None) -> int:
        return spattn_check(self.handle, self.workspace, stream)

    def close(self):
        if self.handle:
            spattn_plan_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
