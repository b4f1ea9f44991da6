"""spattn_forward_host: the whole path on host-resident tensors, with the
copies in and out overlapped over chunks of heads.  Heads are independent
through pooling, routing and attention, so every chunking must reproduce
spattn_forward on device tensors bit for bit."""
import numpy as np
import pytest

from workloads import get_config, make_qkv

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu(gpu_required):
    import block_sparse_attention_33_b200 as sp
    sp.lib()


def _host(bits, pinned):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.pin_memory() if pinned else t.clone()


CASES = [
    ("medium, chunks of 3 (3+3+2)", "medium", dict(), 3, True),
    ("medium, one chunk", "medium", dict(), 64, True),
    ("medium, pageable host memory", "medium", dict(H=4, tau=0.8), 2, False),
    ("tiny b=64 (warp-MMA attention), chunks of 1", "tiny", dict(H=3), 1, True),
    ("stress with Hilbert permutation, chunks of 1", "stress", dict(H=3), 1, True),
    ("wan 8 heads, chunks of 3 (3+3+2)", "wan", dict(H=8), 3, True),
]


@pytest.mark.parametrize("desc,name,ov,chunk,pinned", CASES, ids=[c[0] for c in CASES])
def test_host_forward_equals_device_forward(desc, name, ov, chunk, pinned):
    import torch
    import block_sparse_attention_33_b200 as sp
    w = get_config(name, **ov)
    Q, K, V = make_qkv(w)
    perm = sp.spattn_hilbert_perm(*w.grid) if w.hilbert else None
    plan = sp.Plan(w.B, w.H, w.N, w.d, w.b, w.tau, w.kmin, w.kmax, w.residual, perm)
    try:
        qh, kh, vh = (_host(x, pinned) for x in (Q, K, V))
        q, k, v = qh.cuda(), kh.cuda(), vh.cuda()
        o = torch.zeros_like(q)
        plan.forward(q, k, v, o)
        assert plan.check() == sp.OK
        oh = _host(np.full(Q.shape, 0x7FC0, np.uint16), pinned)    # NaN fill: every element must be written
        plan.forward_host(qh, kh, vh, oh, chunk_heads=chunk)
        torch.cuda.current_stream().synchronize()
        assert plan.check() == sp.OK
        assert torch.equal(oh.view(torch.int16), o.cpu().view(torch.int16))
    finally:
        plan.close()
