"""Batch-, head- and sequence-parallel shards on one GPU, through the C ABI.

A shard is a handle over batch rows [b0, b0 + B) and heads [h0, h0 + H) of a larger problem
(config fields b0, h0, H_total): its Philox counters are keyed on the whole problem's (b,h), so its
decisions, coresets, outputs and log-sum-exps must equal the whole problem's run on the same GPU
bit for bit -- the shards of a multi-GPU run compute exactly what one GPU would.  The shards run one
after the other here (no kernel waits on another); the oracle of the whole problem checks one shard
on its own as well.
"""
import numpy as np
import pytest
import torch

import thinned_softmax_attention_b200 as TA
import workloads as W
from oracle import express, express_a, thinformer

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda", 0)


def _run(w, q, k, v, shard=(0, 0, 0)):
    B, T, H = q.shape[0], q.shape[1], q.shape[2]
    S = k.shape[1]
    h = TA.ThinAttention(B, T, S, H, w.E, w.D, w.torch_dtype, n_exact=w.n_exact, batch=w.batch, shard=shard)
    r = h.forward(q.to(DEV), k.to(DEV), v.to(DEV), causal=w.mode, g=w.g, seed=w.seed, return_lse=True,
                  return_coreset=True, return_trace=True)
    torch.cuda.synchronize()
    h.check()
    r["decisions"] = TA.decode_trace(r["trace"], h.trace_layout(w.mode, w.g))
    r["H"] = H
    return r


def _assert_shard_equals_whole(whole, part, bsel, hsel, b0, h0):
    assert torch.equal(part["out"], whole["out"][bsel][:, :, hsel])
    assert torch.equal(part["lse"], whole["lse"][bsel][:, hsel])
    assert torch.equal(part["coreset"], whole["coreset"][bsel][:, hsel])
    Hw, Hp = whole["H"], part["H"]
    n = 0
    for (bh, rid), bits in part["decisions"].items():
        g_bh = (b0 + bh // Hp) * Hw + h0 + bh % Hp
        np.testing.assert_array_equal(bits, whole["decisions"][(g_bh, rid)])
        n += 1
    assert n > 0


CASES = {
    "vit": W.WORKLOADS["vit"].with_(B=4),
    "biggan": W.WORKLOADS["biggan"].with_(B=2, T=1024),
    "express": W.WORKLOADS["express32k"].with_(H=4, T=12 * 1024),
    "express_a": W.WORKLOADS["express32k_a"].with_(H=4, T=12 * 1024),
}


@pytest.mark.parametrize("name", ["vit", "biggan"])
def test_batch_shards_equal_the_whole_problem(name):
    w = CASES[name]
    q, k, v = W.make_qkv(w)
    whole = _run(w, q, k, v)
    for b0, b1 in [(0, 1), (1, w.B)]:
        part = _run(w, q[b0:b1].contiguous(), k[b0:b1].contiguous(), v[b0:b1].contiguous(), shard=(b0, 0, 0))
        _assert_shard_equals_whole(whole, part, slice(b0, b1), slice(0, w.H), b0, 0)


@pytest.mark.parametrize("name", ["express", "express_a"])
def test_head_shards_equal_the_whole_problem(name):
    w = CASES[name]
    q, k, v = W.make_qkv(w)
    whole = _run(w, q, k, v)
    for h0, h1 in [(0, 1), (1, 4)]:
        sl = (slice(None), slice(None), slice(h0, h1))
        part = _run(w, q[sl].contiguous(), k[sl].contiguous(), v[sl].contiguous(), shard=(0, h0, w.H))
        _assert_shard_equals_whole(whole, part, slice(0, w.B), slice(h0, h1), 0, h0)


def test_unsharded_stream_differs():
    """Without its offsets a shard draws the stream of (b,h) = (0,0): its decisions differ."""
    w = CASES["express"]
    q, k, v = W.make_qkv(w, heads=[2])
    right = _run(w, q, k, v, shard=(0, 2, w.H))
    wrong = _run(w, q, k, v)
    assert not torch.equal(right["coreset"], wrong["coreset"])


@pytest.mark.parametrize("name", ["vit", "express", "express_a"])
def test_shard_matches_the_oracle(name):
    """One shard (batch row 1, or heads 2..3) against the oracle run with the shard's offsets."""
    w = CASES[name]
    if w.causal:
        b0, hs = 0, [2, 3]
        q, k, v = W.make_qkv(w.with_(B=1), heads=hs)
        shard = (0, hs[0], w.H)
    else:
        b0, hs = 1, list(range(w.H))
        q, k, v = W.make_qkv(w.with_(B=1), b0=b0)
        shard = (b0, 0, w.H)
    r = _run(w, q, k, v, shard=shard)
    Hp = len(hs)
    follow = {((b0 + bh // Hp) * w.H + hs[bh % Hp], rid): bits for (bh, rid), bits in r["decisions"].items()}
    rows = np.sort(np.random.default_rng(3).choice(w.T, 256, replace=False))
    kw = dict(follow=follow, rows=rows, heads=(w.H, hs), b0=b0)
    if w.mode == 2:
        ref = express_a(q, k, v, w.n_exact, w.g, w.seed, **kw)
    elif w.mode == 1:
        ref = express(q, k, v, w.n_exact, w.batch, w.g, w.seed, **kw)
    else:
        ref = thinformer(q, k, v, w.g, w.seed, **kw)
    assert ref.stats.mismatches == 0
    assert np.array_equal(r["coreset"].cpu().numpy(), ref.coreset)
    o = r["out"].float().cpu().numpy()[:, rows]
    err = np.abs(o - ref.out).max(axis=(1, 3)) / np.abs(ref.out).max(axis=(1, 3))
    assert float(err.max()) <= 1e-2
    lse = r["lse"].cpu().numpy()[:, :, rows]
    assert float(np.abs(lse - ref.lse).max()) <= 2e-3


SEQ_CASES = {
    "express": (W.WORKLOADS["express32k"].with_(H=4, T=12 * 1024), [0, 1024, 4096, 4224, 12 * 1024]),
    "express_ragged": (W.WORKLOADS["express32k"].with_(T=3000, H=3, n_exact=200, batch=300), [0, 128, 1152, 2048, 3000]),
    "express_a": (W.WORKLOADS["express32k_a"].with_(H=4, T=8192), [0, 512, 2048, 8192]),
    "vit": (W.WORKLOADS["vit"].with_(B=4), [0, 1024, 1152, 3136]),
}


@pytest.mark.parametrize("form", ["default", "ping_pong"])
@pytest.mark.parametrize("name", sorted(SEQ_CASES))
def test_query_row_shards_equal_the_whole_problem(name, form, monkeypatch):
    """Sequence-parallel shards (config q_begin, q_end): every shard thins all keys and attends only
    its query rows; its rows of out and lse equal the whole run's bit for bit, its coreset and
    decisions are the whole run's, and the rows outside its range keep what the buffers held (a
    sentinel).  Range ends fall inside tiles where the exact phase and the batches are not multiples
    of 128 rows (the ragged shape), so clipped tiles are covered; the ping-pong form rebuilds its tile
    pairs inside each range."""
    if form == "ping_pong":
        monkeypatch.setenv("THIN_ATTN_PP", "1")
    w, cuts = SEQ_CASES[name]
    q, k, v = (x.to(DEV) for x in W.make_qkv(w))
    S = w.T if w.causal else w.S
    whole = _run(w, q, k, v)
    for q0, q1 in zip(cuts[:-1], cuts[1:]):
        h = TA.ThinAttention(w.B, w.T, S, w.H, w.E, w.D, w.torch_dtype, n_exact=w.n_exact, batch=w.batch,
                             q_range=(q0, q1))
        out = torch.full((w.B, w.T, w.H, w.D), 7.0, dtype=w.torch_dtype, device=DEV)
        lse = torch.full((w.B, w.H, w.T), -3.0, dtype=torch.float32, device=DEV)
        r = h.forward(q, k, v, causal=w.mode, g=w.g, seed=w.seed, out=out, lse=lse, return_coreset=True)
        torch.cuda.synchronize()
        h.check()
        assert torch.equal(out[:, q0:q1], whole["out"][:, q0:q1])
        assert torch.equal(lse[:, :, q0:q1], whole["lse"][:, :, q0:q1])
        assert bool((out[:, :q0] == 7.0).all()) and bool((out[:, q1:] == 7.0).all())
        assert bool((lse[:, :, :q0] == -3.0).all()) and bool((lse[:, :, q1:] == -3.0).all())
        assert torch.equal(r["coreset"], whole["coreset"])


@pytest.mark.parametrize("name", ["express", "express_ragged"])
def test_split_thinning_sequence_shards_equal_the_whole_problem(name):
    """Sequence shards that split the thinning too (thin_split): each emulated rank thins only the
    batches whose last token lies in its range (phase 1), the batch coresets are exchanged between the
    ranks (export, import), and each rank runs every merge and its rows' attention (phase 2).  Every
    rank's rows, the full node coresets and every halving decision equal the whole run's bit for
    bit; the ragged shape gives one range that owns no batch."""
    w, cuts = SEQ_CASES[name]
    q, k, v = (x.to(DEV) for x in W.make_qkv(w))
    whole = _run(w, q, k, v)
    ranges = list(zip(cuts[:-1], cuts[1:]))
    hs = [TA.ThinAttention(w.B, w.T, w.T, w.H, w.E, w.D, w.torch_dtype, n_exact=w.n_exact, batch=w.batch, q_range=r,
                           thin_split=True) for r in ranges]
    owned = [h.nodes_layout(w.g)[:2] for h in hs]
    n_b = hs[0].nodes_layout(w.g)[2]
    assert owned[0][0] == 0 and owned[-1][1] == n_b and n_b > 0        # the ranges' batches partition them
    assert all(a[1] == b[0] for a, b in zip(owned[:-1], owned[1:]))
    traces1 = [h.forward_phase(q, k, v, phase=1, g=w.g, seed=w.seed, return_trace=True)["trace"] for h in hs]
    TA.exchange_batch_coresets(hs, w.g)
    for h, (q0, q1), tr1 in zip(hs, ranges, traces1):
        out = torch.full((w.B, w.T, w.H, w.D), 7.0, dtype=w.torch_dtype, device=DEV)
        lse = torch.full((w.B, w.H, w.T), -3.0, dtype=torch.float32, device=DEV)
        r = h.forward_phase(q, k, v, phase=2, g=w.g, seed=w.seed, out=out, lse=lse, return_coreset=True,
                            return_trace=True)
        torch.cuda.synchronize()
        h.check()
        assert torch.equal(out[:, q0:q1], whole["out"][:, q0:q1])
        assert torch.equal(lse[:, :, q0:q1], whole["lse"][:, :, q0:q1])
        assert bool((out[:, :q0] == 7.0).all()) and bool((out[:, q1:] == 7.0).all())
        assert torch.equal(r["coreset"], whole["coreset"])
        # phase 1 recorded the batches' decisions, phase 2 the merges' (disjoint words of the trace)
        mine = TA.decode_trace(r["trace"] | tr1, h.trace_layout(w.mode, w.g))
        assert len(mine) > 0 or h.nodes_layout(w.g)[0] == h.nodes_layout(w.g)[1]
        for key, bits in mine.items():
            np.testing.assert_array_equal(bits, whole["decisions"][key])


def test_split_thinning_refuses_the_one_call_forward():
    w, _ = SEQ_CASES["express"]
    h = TA.ThinAttention(w.B, w.T, w.T, w.H, w.E, w.D, w.torch_dtype, n_exact=w.n_exact, batch=w.batch, q_range=(0, 1024),
                         thin_split=True)
    x = torch.zeros(w.B, w.T, w.H, w.E, dtype=w.torch_dtype, device=DEV)
    with pytest.raises(TA.ThinAttnError, match="EINVAL"):
        h.forward(x, x, x, causal=True, g=w.g, seed=w.seed)
