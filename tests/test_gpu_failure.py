"""Failure detection on the GPU without a fault: a bounded wait that runs out.

With THIN_ATTN_INJECT_WAIT_TIMEOUT set, the attention kernel's first CTA withholds its first
key tile, so its MMA issuer's bounded wait gives up (~0.2 s).  The CTA records the site in the
handle's status word and exits through its normal path (tensor memory freed, no copy in flight);
thin_attn_check must report THIN_ATTN_ETIMEOUT, and the next forward on the same context must
run and match the oracle-checked result.
"""
import os

import pytest
import torch

import thinned_softmax_attention_b200 as TA
import workloads as W

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("kernel", ["two_cta", "ping_pong"])
def test_bounded_wait_reports_timeout_and_context_survives(kernel, monkeypatch):
    """Both persistent attention kernels: the two-CTA one (this shape's default) and the ping-pong
    one (forced), whose withheld key tile is the first of the K ring."""
    if kernel == "ping_pong":
        monkeypatch.setenv("THIN_ATTN_PP", "1")
    w = W.WORKLOADS["express32k"].with_(H=2, n_exact=256, batch=256)
    q, k, v = (x.cuda() for x in W.make_qkv(w, T=1024))
    h = TA.ThinAttention(w.B, 1024, 1024, w.H, w.E, w.D, w.torch_dtype, n_exact=256, batch=256)
    good = h.forward(q, k, v, causal=True, g=2, seed=3)["out"].clone()
    h.check()
    os.environ["THIN_ATTN_INJECT_WAIT_TIMEOUT"] = "1"
    try:
        h.forward(q, k, v, causal=True, g=2, seed=3)
        with pytest.raises(TA.ThinAttnError, match="ETIMEOUT") as ei:
            h.check()
        assert "query tile" in str(ei.value)      # the site of the wait that gave up is reported
    finally:
        del os.environ["THIN_ATTN_INJECT_WAIT_TIMEOUT"]
    again = h.forward(q, k, v, causal=True, g=2, seed=3)["out"]
    h.check()
    assert torch.equal(again, good)


def test_scheduler_dependency_wait_reports_timeout_and_context_survives():
    """The persistent halving launch: with THIN_ATTN_INJECT_SCHED_TIMEOUT set, one work item waits on a
    completion flag that nothing sets; its bounded wait gives up (~0.2 s), the status word stops every
    other CTA at its next item, and thin_attn_check reports THIN_ATTN_ETIMEOUT naming the scheduler.
    The next forward on the same context (a new epoch for the flags, counters reset by the last CTA)
    is exact."""
    w = W.WORKLOADS["express32k"].with_(H=2)
    q, k, v = (x.cuda() for x in W.make_qkv(w, T=8192))
    h = TA.ThinAttention(w.B, 8192, 8192, w.H, w.E, w.D, w.torch_dtype, n_exact=w.n_exact, batch=w.batch)
    assert len(h.sched_layout(True, 2)[0]) > 0
    good = h.forward(q, k, v, causal=True, g=2, seed=3, return_coreset=True)
    good = {key: t.clone() for key, t in good.items()}
    h.check()
    os.environ["THIN_ATTN_INJECT_SCHED_TIMEOUT"] = "1"
    try:
        h.forward(q, k, v, causal=True, g=2, seed=3)
        with pytest.raises(TA.ThinAttnError, match="ETIMEOUT") as ei:
            h.check()
        assert "scheduler" in str(ei.value)
    finally:
        del os.environ["THIN_ATTN_INJECT_SCHED_TIMEOUT"]
    again = h.forward(q, k, v, causal=True, g=2, seed=3, return_coreset=True)
    h.check()
    assert torch.equal(again["out"], good["out"]) and torch.equal(again["coreset"], good["coreset"])
