"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every symbol the header declares, validates arguments before touching CUDA,
sizes workspaces, and builds the same Hilbert order as the oracle."""
import ctypes
import os
import re

import numpy as np
import pytest

import block_sparse_attention_33_b200 as sp
import oracle
from workloads import get_config

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from block_sparse_attention_33_b200 import build
    build.build()
    return sp.lib()


def header_functions():
    src = open(os.path.join(ROOT, "include", "spattn.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(spattn_\w+)\s*\(", src)))


def test_library_exports_every_declared_symbol(L):
    names = header_functions()
    assert set(names) == set(sp.EXPORTS)
    for n in names:
        assert hasattr(L, n), n


def plan_status(*args, perm=None):
    h = ctypes.c_void_p()
    ws = ctypes.c_size_t()
    p = None
    if perm is not None:
        perm = np.ascontiguousarray(perm, dtype=np.int32)
        p = perm.ctypes.data
    st = sp.lib().spattn_plan(ctypes.byref(h), *args, p, ctypes.byref(ws))
    return st, h.value, ws.value


@pytest.mark.parametrize("args,code", [
    ((0, 1, 64, 64, 64, 0.9, 1, 4, 1), sp.ERR_INVALID_ARG),      # B = 0
    ((1, 1, 0, 64, 64, 0.9, 1, 4, 1), sp.ERR_INVALID_ARG),       # N = 0
    ((1, 1, 64, 96, 64, 0.9, 1, 4, 1), sp.ERR_UNSUPPORTED),      # d = 96
    ((1, 1, 64, 64, 32, 0.9, 1, 4, 1), sp.ERR_UNSUPPORTED),      # b = 32
    ((1, 1, 64, 64, 64, float("nan"), 1, 4, 1), sp.ERR_INVALID_ARG),
    ((1, 1, 64, 64, 64, float("inf"), 1, 4, 1), sp.ERR_INVALID_ARG),
    ((1, 1, 64, 64, 64, 0.9, 0, 4, 1), sp.ERR_INVALID_ARG),      # kmin = 0
    ((1, 1, 64, 64, 64, 0.9, 5, 4, 1), sp.ERR_INVALID_ARG),      # kmin > kmax
    ((1, 1, 64, 64, 64, 0.9, 1, 4, 2), sp.ERR_INVALID_ARG),      # residual = 2
    ((1, 1, 2049 * 64, 64, 64, 0.9, 1, 4, 1), sp.ERR_UNSUPPORTED),  # nb > 2048
])
def test_plan_rejects_bad_arguments(L, args, code):
    st, h, _ = plan_status(*args)
    assert st == code and not h
    assert L.spattn_last_error().decode()


def test_plan_rejects_non_bijective_perm(L):
    perm = np.arange(100)
    perm[5] = 6
    st, h, _ = plan_status(1, 1, 100, 64, 64, 0.9, 1, 4, 1, perm=perm)
    assert st == sp.ERR_INVALID_ARG and "bijection" in L.spattn_last_error().decode()
    st, h, _ = plan_status(1, 1, 100, 64, 64, 0.9, 1, 4, 1, perm=np.arange(1, 101))
    assert st == sp.ERR_INVALID_ARG


def test_plan_without_perm_needs_no_cuda_and_sizes_workspace(L):
    w = get_config("wan")
    st, h, ws = plan_status(w.B, w.H, w.N, w.d, w.b, w.tau, w.kmin, w.kmax, w.residual)
    assert st == sp.OK and h
    nb, cap = sp.spattn_plan_info(h)
    assert nb == 256 and cap == w.H * 256 * 256
    # means (3 x fp32 + 2 x bf16) + CSR + lists dominate; no token copies
    cen = w.H * nb * w.d
    assert ws >= cen * (3 * 4 + 2 * 2) + 2 * cap * 4
    assert ws < cen * (3 * 4 + 2 * 2) + 2 * cap * 4 + (1 << 20)
    assert ws % 256 == 0
    sp.spattn_plan_destroy(h)


def test_calls_reject_null_arguments(L):
    st, h, ws = plan_status(1, 1, 256, 64, 64, 0.9, 1, 4, 1)
    assert st == sp.OK
    f = L.spattn_forward
    assert f(None, 16, 16, 16, 16, 256, None) == sp.ERR_INVALID_ARG
    assert f(h, None, 16, 16, 16, 256, None) == sp.ERR_INVALID_ARG
    assert f(h, 16, 16, 16, 16, None, None) == sp.ERR_WORKSPACE
    assert f(h, 16, 16, 16, 16, 257, None) == sp.ERR_WORKSPACE      # misaligned workspace
    assert f(h, 8, 16, 16, 16, 256, None) == sp.ERR_INVALID_ARG     # misaligned Q
    assert L.spattn_attend(h, 16, 16, 16, 16, None, 16, 256, None) == sp.ERR_INVALID_ARG
    assert L.spattn_attend(h, 16, 16, 16, None, None, None, 256, None) == sp.ERR_INVALID_ARG
    sp.spattn_plan_destroy(h)
    assert L.spattn_plan_destroy(None) == sp.OK


@pytest.mark.parametrize("grid", [(4, 16, 16), (21, 30, 52), (1, 1, 5), (3, 1, 7), (8, 8, 8)])
def test_library_hilbert_matches_oracle(L, grid):
    assert np.array_equal(sp.spattn_hilbert_perm(*grid), oracle.hilbert_perm(grid))


def test_hilbert_rejects_bad_grid(L):
    buf = np.empty(4, np.int32)
    assert L.spattn_hilbert_perm(0, 2, 2, buf.ctypes.data) == sp.ERR_INVALID_ARG
    assert L.spattn_hilbert_perm(2, 2, 1, None) == sp.ERR_INVALID_ARG


def test_plan_ex_routing_argument(L):
    """spattn_plan_ex accepts the two routing estimates, each with or without
    the threshold selection flag, and the inline selection flag with the
    centroid estimate (no CUDA needed without a permutation); it rejects
    anything else, the inline flag with PAMA among them, before any CUDA
    call."""
    T, I = sp.SELECT_THRESHOLD, sp.SELECT_INLINE
    for routing, code in ((sp.ROUTING_CENTROID, sp.OK), (sp.ROUTING_PAMA, sp.OK),
                          (sp.ROUTING_CENTROID | T, sp.OK), (sp.ROUTING_PAMA | T, sp.OK),
                          (sp.ROUTING_CENTROID | I, sp.OK), (sp.ROUTING_CENTROID | T | I, sp.OK),
                          (sp.ROUTING_PAMA | I, sp.ERR_INVALID_ARG),
                          (sp.ROUTING_PAMA | T | I, sp.ERR_INVALID_ARG),
                          (2, sp.ERR_INVALID_ARG), (-1, sp.ERR_INVALID_ARG), (2 | T, sp.ERR_INVALID_ARG),
                          (64, sp.ERR_INVALID_ARG)):
        h = ctypes.c_void_p()
        ws = ctypes.c_size_t()
        st = L.spattn_plan_ex(ctypes.byref(h), 1, 2, 1000, 64, 64, 0.9, 1, 8, 1, None, routing,
                              ctypes.byref(ws))
        assert st == code, (routing, st, L.spattn_last_error())
        if st == sp.OK:
            assert h.value and ws.value > 0
            assert L.spattn_plan_destroy(h) == sp.OK
        else:
            assert not h.value and b"routing" in L.spattn_last_error()


def test_hilbert_rejects_a_side_beyond_the_key_width(L):
    buf = np.empty(1, np.int32)
    assert L.spattn_hilbert_perm((1 << 21) + 1, 1, 1, buf.ctypes.data) == sp.ERR_UNSUPPORTED
    assert b"2^21" in L.spattn_last_error()


def test_binding_refuses_wrong_tensors_before_any_call(L):
    """The binding checks dtype, contiguity, size and device of torch tensors
    against the plan before the library sees a pointer (no CUDA needed: the
    device check comes last, so host tensors reach every other check)."""
    import torch
    B, H, N, d, b = 1, 2, 256, 64, 64
    h, ws = sp.spattn_plan(B, H, N, d, b, 0.9, 1, 4, 1)
    x = torch.zeros(B * H * N * d, dtype=torch.bfloat16)
    w = torch.zeros(ws, dtype=torch.uint8)
    cases = [
        ((x.float(), x, x, x, w), "dtype"),
        ((x, x[:-1], x, x, w), "exactly"),
        ((x, x, x.view(2, -1).t(), x, w), "contiguous"),
        ((x, x, x, x, w[:-1]), "at least"),
        ((x, x, x, x, w), "CUDA tensor"),
    ]
    for args, msg in cases:
        with pytest.raises(ValueError, match=msg):
            sp.spattn_forward(h, *args)
    rp = torch.zeros(B * H * 4 + 1, dtype=torch.int32)
    with pytest.raises(ValueError, match="col_idx"):
        sp.spattn_route(h, x, x, x, w, rp, torch.zeros(B * H * 4 * 4 - 1, dtype=torch.int32))
    with pytest.raises(ValueError, match="row_ptr"):
        sp.spattn_route(h, x, x, x, w, rp[:-1], torch.zeros(B * H * 4 * 4, dtype=torch.int32))
    with pytest.raises(ValueError, match="Kbar"):
        sp.spattn_means(h, w, None, torch.zeros(B * H * 4 * d - 1), None)
    with pytest.raises(ValueError, match="col_idx"):
        sp.spattn_route_static(B, H, N, d, b, 0.9, 1, 4, x, x, rp,
                               torch.zeros(B * H * 4 * 4 - 1, dtype=torch.int32))
    sp.spattn_plan_destroy(h)
    with pytest.raises(ValueError, match="unknown or destroyed"):
        sp.spattn_forward(h, x, x, x, x, w)


def test_plan_rejects_a_kept_list_capacity_beyond_int32(L):
    """B*H*nb*min(kmax, nb) must fit the int32 CSR offsets: 600 heads of 2048
    blocks keeping up to 2048 blocks each would need 2.5e9 entries."""
    N = 2048 * 128
    st, h, ws = plan_status(1, 600, N, 64, 128, 0.9, 1, 2048, 1)
    assert st == sp.ERR_UNSUPPORTED and b"2^31" in L.spattn_last_error()
    st, h, ws = plan_status(1, 600, N, 64, 128, 0.9, 1, 1024, 1)   # 1.26e9 entries: fits
    assert st == sp.OK
    assert L.spattn_plan_destroy(h) == sp.OK


def test_host_forward_staging_size_and_argument_checks(L):
    """spattn_host_staging_bytes: two slots of four tensors of the chunk,
    each rounded up to 256 bytes; spattn_forward_host refuses NULL and
    misaligned arguments before any CUDA call."""
    B, H, N, d = 1, 5, 1000, 64
    st, h, ws = plan_status(B, H, N, d, 64, 0.9, 1, 4, 1)
    assert st == sp.OK
    up = lambda x: (x + 255) // 256 * 256
    n = ctypes.c_size_t()
    for c, eff in ((1, 1), (2, 2), (5, 5), (9, 5)):
        assert L.spattn_host_staging_bytes(h, c, ctypes.byref(n)) == sp.OK
        assert n.value == 8 * up(eff * N * d * 2)
    assert L.spattn_host_staging_bytes(h, 0, ctypes.byref(n)) == sp.ERR_INVALID_ARG
    f = L.spattn_forward_host
    assert f(h, None, 16, 16, 16, 256, 256, 2, None) == sp.ERR_INVALID_ARG
    assert f(h, 16, 16, 16, 16, 256, 256, 0, None) == sp.ERR_INVALID_ARG
    assert f(h, 16, 16, 16, 16, None, 256, 2, None) == sp.ERR_WORKSPACE
    assert f(h, 16, 16, 16, 16, 256, None, 2, None) == sp.ERR_WORKSPACE
    assert f(h, 16, 16, 16, 16, 256, 272, 2, None) == sp.ERR_WORKSPACE   # misaligned staging
    assert L.spattn_plan_destroy(h) == sp.OK


def test_binding_checks_host_tensors_of_the_host_forward(L):
    import torch
    B, H, N, d = 1, 2, 256, 64
    h, ws = sp.spattn_plan(B, H, N, d, 64, 0.9, 1, 4, 1)
    x = torch.zeros(B * H * N * d, dtype=torch.bfloat16)
    w = torch.zeros(ws, dtype=torch.uint8)
    stg = torch.zeros(sp.spattn_host_staging_bytes(h, 1), dtype=torch.uint8)
    for args, msg in (((x.float(), x, x, x), "dtype"), ((x, x, x, x[:-1]), "exactly"),
                      ((x, x.view(2, -1).t(), x, x), "contiguous")):
        with pytest.raises(ValueError, match=msg):
            sp.spattn_forward_host(h, *args, w, stg, 1)
    with pytest.raises(ValueError, match="staging"):
        sp.spattn_forward_host(h, x, x, x, x, torch.zeros(ws, dtype=torch.uint8), stg[:-1], 1)
    with pytest.raises(ValueError, match="CUDA tensor"):       # host tensors pass; the workspace must be on the device
        sp.spattn_forward_host(h, x, x, x, x, w, stg, 1)
    sp.spattn_plan_destroy(h)


def test_probe_correct_argument_checks(L):
    """spattn_probe_scratch_bytes sizes the exact rows, the fit, B P, b P, the
    gathered probe queries (whole 128-row tiles), the subspace basis, one
    Gram matrix of [1, x, R] per head (width 1 + 2 d padded to a multiple of
    4, whatever the number of probes), and up to 8 key ranges of the exact
    rows with their log2 masses; spattn_probe_correct refuses bad arguments
    before any CUDA call."""
    B, H, N, d = 1, 3, 1000, 64
    st, h, ws = plan_status(B, H, N, d, 64, 0.9, 1, 4, 1)
    assert st == sp.OK
    up = lambda x: (x + 255) // 256 * 256
    n = ctypes.c_size_t()
    zw = (1 + 2 * d + 3) // 4 * 4
    for M in (300, 48):
        assert L.spattn_probe_scratch_bytes(h, M, ctypes.byref(n)) == sp.OK
        assert n.value == (up(B * H * M * d * 4) + up(B * H * (d + 1) * d * 4)
                           + up(B * H * d * d * 4) + up(B * H * d * 4)
                           + up(B * H * ((M + 127) // 128 * 128) * d * 2) + up(B * H * d * d * 4)
                           + up(B * H * zw * zw * 4)
                           + up(8 * B * H * M * d * 4) + up(8 * B * H * M * 4))
    assert L.spattn_probe_scratch_bytes(h, 0, ctypes.byref(n)) == sp.ERR_INVALID_ARG
    f = L.spattn_probe_correct
    ok = dict(Q=16, K=16, V=16, O=16, probes=16, M=M, lam=100.0, r=8, ws=256, scratch=256)

    def call(**kw):
        a = dict(ok, **kw)
        return f(h, a["Q"], a["K"], a["V"], a["O"], a["probes"], a["M"], a["lam"], a["r"],
                 a["ws"], a["scratch"], None)
    assert call(O=None) == sp.ERR_INVALID_ARG
    assert call(O=8) == sp.ERR_INVALID_ARG                      # misaligned O
    assert call(probes=None) == sp.ERR_INVALID_ARG
    assert call(M=0) == sp.ERR_INVALID_ARG
    assert call(lam=-1.0) == sp.ERR_INVALID_ARG
    assert call(lam=float("nan")) == sp.ERR_INVALID_ARG
    assert call(r=-1) == sp.ERR_INVALID_ARG and call(r=d + 1) == sp.ERR_INVALID_ARG
    assert call(scratch=None) == sp.ERR_WORKSPACE and call(scratch=272) == sp.ERR_WORKSPACE
    assert call(ws=None) == sp.ERR_WORKSPACE
    assert L.spattn_plan_destroy(h) == sp.OK


def test_binding_checks_the_probe_tensor(L):
    import torch
    B, H, N, d = 1, 2, 256, 64
    h, ws = sp.spattn_plan(B, H, N, d, 64, 0.9, 1, 4, 1)
    x = torch.zeros(B * H * N * d, dtype=torch.bfloat16)
    w = torch.zeros(ws, dtype=torch.uint8)
    stg = torch.zeros(sp.spattn_probe_scratch_bytes(h, 8), dtype=torch.uint8)
    with pytest.raises(ValueError, match="probes: dtype"):
        sp.spattn_probe_correct(h, x, x, x, x, torch.zeros(B * H * 8, dtype=torch.int64), 8, 1.0, 4, w, stg)
    with pytest.raises(ValueError, match="probes: needs exactly"):
        sp.spattn_probe_correct(h, x, x, x, x, torch.zeros(B * H * 8 - 1, dtype=torch.int32), 8, 1.0, 4, w, stg)
    with pytest.raises(ValueError, match="scratch"):
        sp.spattn_probe_correct(h, x, x, x, x, torch.zeros(B * H * 8, dtype=torch.int32), 8, 1.0, 4, w, stg[:-1])
    sp.spattn_plan_destroy(h)


def test_injected_allocation_failure_returns_an_error_and_no_plan(L, monkeypatch):
    """Host-side fault injection: the permutation's device allocation reports
    out-of-memory (SPATTN_TEST_FAIL_ALLOC=1); the plan call returns
    SPATTN_ERR_CUDA, leaves no plan and names the failing call."""
    monkeypatch.setenv("SPATTN_TEST_FAIL_ALLOC", "1")
    perm = np.arange(256, dtype=np.int32)[::-1].copy()
    st, h, ws = plan_status(1, 2, 256, 64, 64, 0.9, 1, 4, 1, perm=perm)
    assert st == sp.ERR_CUDA and not h
    msg = L.spattn_last_error()
    assert b"cudaMalloc(perm)" in msg and b"out of memory" in msg
    with pytest.raises(sp.SpAttnError) as ei:
        sp.Plan(1, 2, 256, 64, 64, 0.9, 1, 4, 1, perm=perm, device="cpu")
    assert ei.value.status == sp.ERR_CUDA


C_PROGRAM = r"""
#include <stdio.h>
#include <stdlib.h>
#include "spattn.h"

int main(void) {
  spattn_plan_t plan = NULL;
  size_t ws = 0;
  int nb = 0;
  int64_t cap = 0;
  int32_t perm[2 * 3 * 4];
  if (spattn_plan(&plan, 1, 2, 1000, 64, 64, 0.9f, 1, 4, 1, NULL, &ws) != SPATTN_OK) return 1;
  if (spattn_plan_info(plan, &nb, &cap) != SPATTN_OK || nb != 16 || cap != 2 * 16 * 4) return 2;
  if (spattn_plan_destroy(plan) != SPATTN_OK) return 3;
  if (spattn_plan(&plan, 1, 2, 1000, 96, 64, 0.9f, 1, 4, 1, NULL, &ws) != SPATTN_ERR_UNSUPPORTED) return 4;
  if (spattn_last_error()[0] == 0) return 5;
  if (spattn_hilbert_perm(2, 3, 4, perm) != SPATTN_OK) return 6;
  printf("ok %zu %d\n", ws, perm[0]);
  return 0;
}
"""


def test_header_is_c_and_the_library_links_from_c(L, tmp_path):
    """The boundary is a C ABI: a C99 program built with gcc against
    include/spattn.h and libspattn.so runs the host-side calls."""
    import subprocess
    from block_sparse_attention_33_b200 import build
    src = tmp_path / "use.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "use"
    libdir = os.path.dirname(build.LIB)
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                        str(src), "-o", str(exe), "-L", libdir, "-lspattn",
                        f"-Wl,-rpath,{libdir}"], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.startswith("ok "), (r.returncode, r.stdout, r.stderr)


def test_plan_rejects_more_than_65535_heads(L):
    st, h, ws = plan_status(1, 65536, 64, 64, 64, 0.9, 1, 4, 1)
    assert st == sp.ERR_UNSUPPORTED and b"65535" in L.spattn_last_error()
    st, h, ws = plan_status(3, 21845, 64, 64, 64, 0.9, 1, 4, 1)      # 65535 pairs: accepted
    assert st == sp.OK
    assert L.spattn_plan_destroy(h) == sp.OK
    assert L.spattn_route_static(2, 40000, 64, 64, 64, 0.9, 1, 4, None, 16, 16, 16, 16, None) \
        == sp.ERR_UNSUPPORTED


def test_build_stamp_tells_variant_builds_apart(L):
    """The library on disk records its extra compiler flags: the default build
    is up to date for no extra flags and not for others, so a variant build
    is never mistaken for the default one (and vice versa)."""
    from block_sparse_attention_33_b200 import build
    build.build()
    assert build.up_to_date(())
    assert not build.up_to_date(("-DSPATTN_EXP_EMU=2",))
    with open(build.STAMP) as f:
        assert f.read() == ""


def test_default_chunk_heads():
    """The host pipeline's default chunk balances the exposed first/last
    copies against the last attention wave of every chunk: about
    sqrt(BH / 5) heads, at least 1 and at most BH."""
    f = sp.default_chunk_heads
    assert [f(x) for x in (1, 2, 8, 24, 40, 80)] == [1, 1, 1, 2, 3, 4]
    assert all(1 <= f(x) <= x for x in range(1, 200))
