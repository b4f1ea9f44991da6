"""spattn_route_static: routing for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc -- their device memory belongs to another
allocator, or they are handed only their inputs and outputs, or they run in
loops that must not pay cudaMalloc's implicit synchronisation.  For them the
library routes with scratch held in one static device array.  These tests
check, through the C ABI, that the allocation-free entry point writes the same
CSR as the workspace-based spattn_route on two consecutive calls (the second
call reuses the array the first one left behind), and that a problem larger
than the array is refused up front.

This file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest

import block_sparse_attention_33_b200 as sp
from workloads import get_config, make_qkv


def _dev(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _route_both(w, perm=None):
    import torch
    Q, K, V = make_qkv(w)
    q, k, v = _dev(Q), _dev(K), _dev(V)
    plan = sp.Plan(w.B, w.H, w.N, w.d, w.b, w.tau, w.kmin, w.kmax, w.residual, perm)
    try:
        rows = w.B * w.H * plan.nb
        rp_ref = torch.zeros(rows + 1, dtype=torch.int32, device="cuda")
        ci_ref = torch.full((plan.col_capacity,), -1, dtype=torch.int32, device="cuda")
        plan.route(q, k, v, rp_ref, ci_ref)
        rp = torch.full((rows + 1,), -5, dtype=torch.int32, device="cuda")
        ci = torch.full((plan.col_capacity,), -5, dtype=torch.int32, device="cuda")
        perm_dev = None if perm is None else torch.from_numpy(np.asarray(perm, np.int32)).cuda()
        st = sp.lib().spattn_route_static(w.B, w.H, w.N, w.d, w.b, float(w.tau), w.kmin, w.kmax,
                                          None if perm_dev is None else perm_dev.data_ptr(),
                                          q.data_ptr(), k.data_ptr(),
                                          rp.data_ptr(), ci.data_ptr(),
                                          torch.cuda.current_stream().cuda_stream)
        assert st == sp.OK, sp.spattn_last_error()
        torch.cuda.synchronize()
        nnz = int(rp_ref[-1].item())
        return (rp_ref.cpu().numpy(), ci_ref[:nnz].cpu().numpy(),
                rp.cpu().numpy(), ci[:nnz].cpu().numpy())
    finally:
        plan.close()


@pytest.mark.gpu
def test_static_route_matches_workspace_route_twice(gpu_required):
    sp.lib()
    # first call: medium layer (d = 128); second call: a smaller, permuted,
    # d = 64 problem that reuses the scratch the first call left behind
    w1 = get_config("medium")
    w2 = get_config("tiny", tau=0.7, kmax=5)
    rng = np.random.default_rng(3)
    for w, perm in ((w1, None), (w2, rng.permutation(w2.N))):
        rp_ref, ci_ref, rp, ci = _route_both(w, perm)
        assert np.array_equal(rp, rp_ref)
        assert np.array_equal(ci, ci_ref)
        assert rp[-1] > 0


def test_static_route_rejects_problems_beyond_the_scratch():
    L = sp.lib()
    w = get_config("hunyuan")           # ~0.1 GB of routing scratch
    st = L.spattn_route_static(w.B, w.H, w.N, w.d, w.b, 0.9, 1, w.kmax, None, 16, 16, 16, 16, None)
    assert st == sp.ERR_UNSUPPORTED
    assert "static scratch" in sp.spattn_last_error()


def _scratch_need(B, H, N, d, b, kmax):
    """The scratch size spattn_route_static documents in include/spattn.h."""
    up = lambda x: (x + 255) // 256 * 256
    nb = -(-N // b)
    R = B * H * nb
    return 256 + 2 * up(R * d * 4) + 2 * up(R * 4) + up(R * min(kmax, nb) * 4)


def test_static_route_size_check_follows_the_documented_formula():
    """Shapes on both sides of the limit: the size check comes before the
    pointer checks, so a call with NULL buffers is refused for its size
    (UNSUPPORTED) or, when it fits, for its pointers (INVALID_ARG); nothing
    reaches the device either way."""
    L = sp.lib()
    limit = 32 << 20
    N, d, b, kmax = 32760, 128, 128, 256
    for H in range(60, 68):
        st = L.spattn_route_static(1, H, N, d, b, 0.9, 1, kmax, None, None, None, None, None, None)
        fits = _scratch_need(1, H, N, d, b, kmax) <= limit
        assert st == (sp.ERR_INVALID_ARG if fits else sp.ERR_UNSUPPORTED), (H, st)
    assert _scratch_need(1, 63, N, d, b, kmax) <= limit < _scratch_need(1, 64, N, d, b, kmax)


def test_static_route_path_calls_no_device_allocator():
    """The routing path of spattn_route_static (its own file, the pooling and
    routing launchers and the shared-memory attribute helper) names no device
    allocator, so a later edit that adds one fails here."""
    import os
    import re
    csrc = os.path.join(os.path.dirname(sp.__file__), "csrc")

    def code(path):
        s = open(os.path.join(csrc, path)).read()
        s = re.sub(r"/\*.*?\*/", "", s, flags=re.S)
        return re.sub(r"//[^\n]*", "", s)

    api = code("api.cu")
    start = api.index("cudaError_t ensure_dyn_smem(")
    helper = api[start:api.index("\n}\n", start)]
    alloc = re.compile(r"\b(cudaMalloc\w*|cudaFree\w*|cudaHostAlloc|cuMemAlloc\w*|cuMemCreate|"
                       r"cudaMemPool\w*|cudaMallocAsync)\b")
    for name, text in (("route_static.cu", code("route_static.cu")), ("pool.cu", code("pool.cu")),
                       ("route.cu", code("route.cu")), ("api.cu:ensure_dyn_smem", helper)):
        assert not alloc.findall(text), (name, alloc.findall(text))
