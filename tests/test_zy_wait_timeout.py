"""Failure detection on the GPU without a fault: a device wait that runs out.

With SPATTN_TEST_WAIT_TIMEOUT=1 in the environment when a plan is made, the
first CTA of the tcgen05 attention waits on an mbarrier phase that nothing
completes.  Its bounded wait gives up after about two seconds, the CTA's roles
leave their loops and drain their copies and MMAs, TMEM is freed, and
spattn_check reports SPATTN_ERR_TIMEOUT.  The context stays usable: a new plan
on the same inputs matches the oracle."""
import numpy as np
import pytest

from tests.harness import MAX_ABS, REL_L2, oracle_check, run_library, to_dev
from workloads import get_config, make_qkv

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_reports_timeout_and_context_survives(gpu_required, monkeypatch):
    import torch
    import block_sparse_attention_33_b200 as sp
    w = get_config("medium", H=2)
    Q, K, V = make_qkv(w)
    monkeypatch.setenv("SPATTN_TEST_WAIT_TIMEOUT", "1")
    plan = sp.Plan(w.B, w.H, w.N, w.d, w.b, w.tau, w.kmin, w.kmax, w.residual)
    monkeypatch.delenv("SPATTN_TEST_WAIT_TIMEOUT")
    try:
        q, k, v = to_dev(Q), to_dev(K), to_dev(V)
        o = torch.zeros_like(q)
        plan.route(q, k, v)
        plan.attend(q, k, v, o)
        st = plan.check()
        msg = sp.spattn_last_error()
    finally:
        plan.close()
    assert st == sp.ERR_TIMEOUT, (st, msg)
    assert "gave up" in msg
    # same process, same device: a fresh plan computes the right answer
    res = run_library(w, Q, K, V)
    assert res["status"] == 0
    fig = oracle_check(w, Q, K, V, res)
    assert fig["bad"] == 0 and fig["max_abs"] < MAX_ABS and fig["rel_l2"] < REL_L2, fig
