"""Parity of the CUDA path (through the C ABI) with the fp64 CPU oracle.

For every case the library runs with its decision trace; the oracle then
replays the same thinning in follow mode: a decision whose swap margin is
below 1e-4 of the instance's kernel scale is a near tie and takes the GPU's
choice, every other decision must agree (mismatches == 0).  Given identical
coresets the outputs must agree within 1e-2 (bf16) / 1e-5 (fp32) max relative
error per (b,h) slice (max |o_gpu - o_ref| / max |o_ref|).  The same error per query
row (max_d |o_gpu - o_ref| / max_d |o_ref| of that row) is bounded too, so that a row
whose outputs are small beside its slice's largest cannot hide a large relative error.
"""
import math

import numpy as np
import pytest
import torch

import thinned_softmax_attention_b200 as TA
import workloads as W
from oracle import express, express_a, thinformer

pytestmark = pytest.mark.gpu

TOL = {"fp32": 1e-5, "bf16": 1e-2}
ROW_TOL = {"fp32": 1e-4, "bf16": 2e-2}
LSE_TOL = {"fp32": 1e-5, "bf16": 2e-3}


def _rel_err_per_slice(o, ref):
    """max over (b,h) of max|o - ref| / max|ref| on (B, rows, H, D) arrays."""
    err = np.abs(o - ref).max(axis=(1, 3))
    scale = np.abs(ref).max(axis=(1, 3))
    return float((err / scale).max())


def _rel_err_per_row(o, ref):
    """max over (b, row, h) of max_d |o - ref| / max_d |ref| on (B, rows, H, D) arrays."""
    return float((np.abs(o - ref).max(axis=3) / np.abs(ref).max(axis=3)).max())


def run_case(w, T=None, S=None, heads=None, rows=None, g=None, seed=None, check_heads=None):
    """Run GPU + oracle on workload ``w`` (optionally resized); returns a dict of measurements."""
    T = w.T if T is None else T
    S = (T if w.causal else w.S) if S is None else S
    g = w.g if g is None else g
    seed = w.seed if seed is None else seed
    q, k, v = W.make_qkv(w, T=T, S=S)
    dev = torch.device("cuda", 0)
    h = TA.ThinAttention(w.B, T, S, w.H, w.E, w.D, w.torch_dtype, n_exact=w.n_exact, batch=w.batch)
    r = h.forward(q.to(dev), k.to(dev), v.to(dev), causal=w.mode, g=g, seed=seed, return_lse=True,
                  return_coreset=True, return_trace=True)
    torch.cuda.synchronize()
    h.check()
    follow = TA.decode_trace(r["trace"], h.trace_layout(w.mode, g))
    hs = list(range(w.H)) if check_heads is None else list(check_heads)
    rsel = np.arange(T) if rows is None else np.sort(np.asarray(rows))
    qh, kh, vh = q[:, :, hs], k[:, :, hs], v[:, :, hs]
    if w.causal and w.cache == "A":
        ref = express_a(qh, kh, vh, w.n_exact, g, seed, follow=follow, rows=rsel, heads=(w.H, hs))
    elif w.causal:
        ref = express(qh, kh, vh, w.n_exact, w.batch, g, seed, follow=follow, rows=rsel, heads=(w.H, hs))
    else:
        ref = thinformer(qh, kh, vh, g, seed, follow=follow, rows=rsel, heads=(w.H, hs))
    o = r["out"].float().cpu().numpy()[:, rsel][:, :, hs]
    lse = r["lse"].cpu().numpy()[:, hs][:, :, rsel]
    cs = r["coreset"].cpu().numpy()[:, hs]
    return {
        "mismatches": ref.stats.mismatches,
        "near_ties": ref.stats.near_ties,
        "decisions": ref.stats.decisions,
        "coreset_equal": bool(np.array_equal(cs, ref.coreset)),
        "coreset_shape": cs.shape,
        "out_err": _rel_err_per_slice(o, ref.out),
        "row_err": _rel_err_per_row(o, ref.out),
        "lse_err": float(np.abs(lse - ref.lse).max()),
        "ref": ref,
        "gpu": r,
    }


def assert_parity(res, dtype):
    assert res["mismatches"] == 0, res
    assert res["coreset_equal"]
    assert res["out_err"] <= TOL[dtype], res["out_err"]
    assert res["row_err"] <= ROW_TOL[dtype], res["row_err"]
    assert res["lse_err"] <= LSE_TOL[dtype], res["lse_err"]


# ------------------------------------------------------------------ non-causal


def test_tiny_fp32_full():
    w = W.WORKLOADS["tiny"]
    res = run_case(w)
    assert res["coreset_shape"] == (1, 1, 64)
    assert_parity(res, "fp32")


@pytest.mark.parametrize("name,B", [("vit", 2), ("biggan", 2)])
def test_reduced_batch_full_length(name, B):
    w = W.WORKLOADS[name].with_(B=B)
    res = run_case(w)
    assert_parity(res, w.dtype)


@pytest.mark.parametrize("name", ["vit", "biggan"])
def test_full_workload_sampled_rows(name):
    """The full workload in the launch configuration the bench times; outputs checked on sampled rows."""
    w = W.WORKLOADS[name]
    rows = np.random.default_rng(0).choice(w.T, 192, replace=False)
    res = run_case(w, rows=rows)
    assert_parity(res, w.dtype)


@pytest.mark.parametrize("B,H,T,S,E,D,g,dtype", [
    (2, 3, 77, 1000, 64, 128, 2, "bf16"),    # ragged: S' = 960, groups of 60 (m = 30, not a multiple of 32)
    (1, 2, 130, 200, 64, 64, 0, "bf16"),     # g = 0: r clamped so leaves are non-empty
    (1, 1, 40, 64, 64, 64, 3, "fp32"),       # S <= 4^g: coreset = all keys, exact attention
    (2, 2, 300, 513, 128, 128, 1, "fp32"),   # odd S, fp32
    (1, 1, 1, 4096, 64, 64, 2, "bf16"),      # a single query
    (1, 2, 64, 2000, 128, 128, 2, "bf16"),   # last level 224 points: partial second 128-row block
    (1, 2, 64, 3000, 256, 64, 2, "bf16"),    # last level 352 points (257..512), E = 256, D = 64
])
def test_noncausal_edge_cases(B, H, T, S, E, D, g, dtype):
    w = W.Workload("edge", B, H, T, S, E, D, dtype, False, g, 11, 5, "iid")
    res = run_case(w)
    assert_parity(res, dtype)


@pytest.mark.parametrize("S,g,E,D", [
    (16384, 4, 64, 64),      # levels of 1024, 2048 and 4096 points: tensor-core Gram + the long walk
    (8192, 3, 128, 128),     # levels of 128 .. 512 points fused, the last (1024 points) three launches
    (10000, 4, 64, 128),     # subsampled (S' = 9984): 624, 1248 and 2496 points, m not a multiple of 32
])
def test_bf16_instances_above_512_points(S, g, E, D):
    """bf16 halving instances of more than 512 points take the pair-Gram kernel and the long walk
    (three launches per level); sampled query rows of every (b,h) against the oracle."""
    w = W.Workload("large", 1, 2, 512, S, E, D, "bf16", False, g, 13, 21, "iid")
    rows = np.random.default_rng(4).choice(w.T, 96, replace=False)
    res = run_case(w, rows=rows)
    assert res["coreset_shape"][-1] == {16384: 2048, 8192: 512, 10000: 1248}[S]
    assert_parity(res, "bf16")


def test_coreset_equal_to_full_set_is_exact_attention():
    w = W.Workload("exact", 1, 2, 50, 60, 64, 64, "fp32", False, 3, 1, 9, "iid")
    res = run_case(w)
    q, k, v = W.make_qkv(w)
    ex = torch.nn.functional.scaled_dot_product_attention(
        q.double().transpose(1, 2), k.double().transpose(1, 2), v.double().transpose(1, 2)).transpose(1, 2)
    o = res["gpu"]["out"].double().cpu()
    assert float((o - ex).abs().max() / ex.abs().max()) < 1e-5


# ------------------------------------------------------------------ causal (Express)


def test_express_reduced():
    w = W.WORKLOADS["express32k"].with_(H=2, n_exact=512, batch=512)
    res = run_case(w, T=4608)   # 7 batches + a trailing partial batch; one level-1 merge
    assert_parity(res, "bf16")


@pytest.mark.parametrize("T,n_e,bsz,g,dtype", [
    (300, 512, 256, 2, "bf16"),     # T < n_e: everything in the exact phase
    (1000, 0, 64, 1, "bf16"),       # no exact phase; 15 batches, three level-1 merges
    (700, 100, 16, 2, "fp32"),      # batch <= 4^g: batches are stored whole, merges still halve
    (2048, 256, 96, 2, "bf16"),     # batch not a power of 4: subsample inside every batch
])
def test_express_edge_cases(T, n_e, bsz, g, dtype):
    w = W.Workload("edge", 1, 2, T, T, 128 if dtype == "bf16" else 64, 128 if dtype == "bf16" else 64, dtype,
                   True, g, 7, 4, "rope", n_exact=n_e, batch=bsz)
    res = run_case(w)
    assert_parity(res, dtype)


def test_express_exact_phase_equals_exact_causal_attention():
    w = W.WORKLOADS["express32k"].with_(H=2, n_exact=256, batch=256)
    q, k, v = W.make_qkv(w, T=1024)
    res = run_case(w, T=1024)
    ex = torch.nn.functional.scaled_dot_product_attention(
        q.double().transpose(1, 2), k.double().transpose(1, 2), v.double().transpose(1, 2),
        is_causal=True).transpose(1, 2)
    o = res["gpu"]["out"].double().cpu()
    # exact phase and the first batch (no node exists yet) are exact causal attention
    assert float((o[:, :512] - ex[:, :512]).abs().max() / ex[:, :512].abs().max()) < 1e-2


def test_express32k_full_sampled_rows():
    w = W.WORKLOADS["express32k"]
    rows = np.random.default_rng(1).choice(w.T, 256, replace=False)
    res = run_case(w, rows=rows, check_heads=[0, 7, 31])
    assert_parity(res, "bf16")


@pytest.mark.slow
def test_express128k_full_sampled_rows():
    w = W.WORKLOADS["express128k"]
    rows = np.random.default_rng(2).choice(w.T, 128, replace=False)
    res = run_case(w, rows=rows, check_heads=[5, 30])
    assert_parity(res, "bf16")


# ------------------------------------------------------------------ API paths


def test_host_buffer_entry_point_matches_device_path():
    w = W.WORKLOADS["biggan"].with_(B=2)
    q, k, v = W.make_qkv(w)
    h = TA.ThinAttention(w.B, w.T, w.S, w.H, w.E, w.D, w.torch_dtype)
    dev = torch.device("cuda", 0)
    r = h.forward(q.to(dev), k.to(dev), v.to(dev), causal=False, g=w.g, seed=w.seed, return_lse=True)
    out = torch.empty(w.B, w.T, w.H, w.D, dtype=w.torch_dtype).pin_memory()
    lse = torch.empty(w.B, w.H, w.T, dtype=torch.float32).pin_memory()
    h.forward_host(q.pin_memory(), k.pin_memory(), v.pin_memory(), out, causal=False, g=w.g, seed=w.seed, lse=lse)
    assert torch.equal(out, r["out"].cpu())
    assert torch.equal(lse, r["lse"].cpu())


def test_repeat_calls_are_deterministic():
    w = W.WORKLOADS["express32k"].with_(H=2, n_exact=256, batch=256)
    q, k, v = (x.cuda() for x in W.make_qkv(w, T=2048))
    h = TA.ThinAttention(w.B, 2048, 2048, w.H, w.E, w.D, w.torch_dtype, n_exact=256, batch=256)
    a = h.forward(q, k, v, causal=True, g=2, seed=3, return_coreset=True)
    b = h.forward(q, k, v, causal=True, g=2, seed=3, return_coreset=True)
    c = h.forward(q, k, v, causal=True, g=2, seed=4, return_coreset=True)
    assert torch.equal(a["out"], b["out"]) and torch.equal(a["coreset"], b["coreset"])
    assert not torch.equal(a["coreset"], c["coreset"])


def test_dropin_call_returns_output_and_none():
    w = W.WORKLOADS["tiny"]
    q, k, v = (x.cuda() for x in W.make_qkv(w))
    out, weights = TA.thinformer_attention(q, k, v, g=2, seed=1)
    assert weights is None and out.shape == (1, 256, 1, 64)
    # the README's layer object: the same call, non-causal and causal
    layer = TA.ThinformerAttention(g=2, seed=1)
    out2, weights2 = layer(q, k, v)
    assert weights2 is None and torch.equal(out, out2)
    we = W.WORKLOADS["express32k"].with_(H=2)
    qe, ke, ve = (x.cuda() for x in W.make_qkv(we, T=4096))
    h = TA.ThinAttention(1, 4096, 4096, 2, we.E, we.D, we.torch_dtype, n_exact=1024, batch=1024)
    ref = h.forward(qe, ke, ve, causal=True, g=2, seed=1)["out"]
    out3, weights3 = layer(qe, ke, ve, causal=True)
    assert weights3 is None and torch.equal(out3, ref)


@pytest.mark.parametrize("name,mode", [("express", 1), ("express_a", 2), ("vit", 0)])
def test_pipelined_host_path_equals_device_path(name, mode):
    """Inputs of 64 MB and more go through the host path in four shards (heads, or batch rows when H
    does not divide), copies overlapping the other shards' compute; outputs and LSE equal the
    device-resident forward's bit for bit."""
    w = {"express": W.WORKLOADS["express32k"].with_(T=16384, H=8),
         "express_a": W.WORKLOADS["express32k_a"].with_(T=16384, H=8),
         "vit": W.WORKLOADS["vit"].with_(B=64)}[name]
    S = w.T if w.causal else w.S
    q, k, v = W.make_qkv(w)
    assert (q.numel() + k.numel() + v.numel()) * 2 >= 64 << 20
    h = TA.ThinAttention(w.B, w.T, S, w.H, w.E, w.D, w.torch_dtype, n_exact=w.n_exact, batch=w.batch)
    dev = h.forward(q.cuda(), k.cuda(), v.cuda(), causal=mode, g=w.g, seed=w.seed, return_lse=True)
    torch.cuda.synchronize()
    out = torch.empty(w.B, w.T, w.H, w.D, dtype=w.torch_dtype).pin_memory()
    lse = torch.empty(w.B, w.H, w.T, dtype=torch.float32).pin_memory()
    for _ in range(2):   # the second call reuses the shards, streams and staging
        out.zero_()
        h.forward_host(q.pin_memory(), k.pin_memory(), v.pin_memory(), out, causal=mode, g=w.g, seed=w.seed, lse=lse)
        assert torch.equal(out, dev["out"].cpu())
        assert torch.equal(lse, dev["lse"].cpu())


@pytest.mark.parametrize("case", ["causal", "noncausal", "ragged224", "ragged352"])
def test_fused_and_three_launch_halving_agree(case, monkeypatch):
    """The one-launch halving kernels (up to 512 points) and the c^2 / Gram / walk launches take the
    same decisions (same arithmetic), so traces, coresets, outputs and LSE are bit-identical."""
    causal = case == "causal"
    if causal:
        w = W.WORKLOADS["express32k"].with_(T=8192, H=4)
        S = w.T
    elif case == "noncausal":
        w = W.WORKLOADS["express32k"].with_(T=512, H=2, B=2, causal=False, S=1024)
        S = 1024
    else:
        S = 2000 if case == "ragged224" else 3000
        w = W.WORKLOADS["express32k"].with_(T=256, H=3, B=1, causal=False, S=S, E=128 if S == 2000 else 256,
                                            D=128 if S == 2000 else 64)
    q, k, v = (x.cuda() for x in W.make_qkv(w, T=w.T, S=S))
    res = []
    for unfused in (False, True):
        if unfused:
            monkeypatch.setenv("THIN_ATTN_UNFUSED_HALVING", "1")
        else:
            monkeypatch.delenv("THIN_ATTN_UNFUSED_HALVING", raising=False)
        h = TA.ThinAttention(w.B, w.T, S, w.H, w.E, w.D, w.torch_dtype, n_exact=w.n_exact, batch=w.batch)
        r = h.forward(q, k, v, causal=causal, g=w.g, seed=w.seed, return_lse=True, return_coreset=True,
                      return_trace=True)
        torch.cuda.synchronize()
        h.check()
        res.append(r)
    for key in ("trace", "coreset", "out", "lse"):
        assert torch.equal(res[0][key], res[1][key]), key


@pytest.mark.parametrize("name", ["express", "express_long", "express_ragged", "express_a"])
def test_scheduled_and_levelwise_halving_agree(name, monkeypatch):
    """The persistent halving launch (the last batch level and every HALVE merge as work items waiting
    on their inputs) and one launch per step run the
    same instance kernels: traces, coresets, outputs and LSE are bit-identical, on two forwards in a
    row (the completion flags of the first must not satisfy the second's waits)."""
    w = {"express": W.WORKLOADS["express32k"].with_(T=8192, H=4),
         "express_long": W.WORKLOADS["express128k"].with_(T=40960, H=2),
         "express_ragged": W.WORKLOADS["express32k"].with_(T=22000, H=2, n_exact=100, batch=600),
         "express_a": W.WORKLOADS["express32k_a"].with_(T=16384, H=2)}[name]
    S = w.T if w.causal else w.S
    q, k, v = (x.cuda() for x in W.make_qkv(w))
    res = []
    for levelwise in (False, True):
        if levelwise:
            monkeypatch.setenv("THIN_ATTN_LEVELWISE", "1")
        else:
            monkeypatch.delenv("THIN_ATTN_LEVELWISE", raising=False)
        h = TA.ThinAttention(w.B, w.T, S, w.H, w.E, w.D, w.torch_dtype, n_exact=w.n_exact, batch=w.batch)
        if not levelwise:
            assert len(h.sched_layout(w.mode, w.g)[0]) > 0
        for _ in range(2):
            r = h.forward(q, k, v, causal=w.mode, g=w.g, seed=w.seed, return_lse=True, return_coreset=True,
                          return_trace=True)
            torch.cuda.synchronize()
            h.check()
            res.append(r)
    for r in res[1:]:
        for key in ("trace", "coreset", "out", "lse"):
            assert torch.equal(res[0][key], r[key]), key


@pytest.mark.parametrize("name", ["vit", "express", "express_a", "express_ragged", "vit_e64_d128", "vit_e128_d64"])
def test_attention_launch_forms_agree(name, monkeypatch):
    """The ping-pong kernel (two query tiles of a head against one K/V stream, one CTA per SM), the
    two-CTA persistent kernel (items from a work counter), its one-CTA-per-tile form, and the
    persistent kernel launched as several dependent waves on a side stream (each launch takes and
    resets the same counter) run the same per-tile arithmetic: outputs and LSE are bit-identical.
    ViT's 25 query tiles per head leave one tile unpaired; the ragged Express shape has batches of
    three tiles, so pairs cross from the exact phase into batches and some tiles run alone.  The two
    ViT variants with unequal head dims take the ping-pong kernel's other ring layouts (4 K stages)."""
    w = {"vit": W.WORKLOADS["vit"].with_(B=8),
         "vit_e64_d128": W.WORKLOADS["vit"].with_(B=4, D=128),
         "vit_e128_d64": W.WORKLOADS["vit"].with_(B=4, E=128),
         "express": W.WORKLOADS["express32k"].with_(T=8192, H=4),
         "express_a": W.WORKLOADS["express32k_a"].with_(T=8192, H=4),
         "express_ragged": W.WORKLOADS["express32k"].with_(T=3000, H=3, n_exact=200, batch=300)}[name]
    S = w.T if w.causal else w.S
    q, k, v = (x.cuda() for x in W.make_qkv(w))
    forms = [{"THIN_ATTN_PP": "1"}, {"THIN_ATTN_TC2P": "1"}, {"THIN_ATTN_TC2_PER_TILE": "1"}, {"THIN_ATTN_OVERLAP": "1"}]
    res = []
    for env in forms:
        for key in ("THIN_ATTN_PP", "THIN_ATTN_TC2P", "THIN_ATTN_TC2_PER_TILE", "THIN_ATTN_OVERLAP"):
            if key in env:
                monkeypatch.setenv(key, env[key])
            else:
                monkeypatch.delenv(key, raising=False)
        h = TA.ThinAttention(w.B, w.T, S, w.H, w.E, w.D, w.torch_dtype, n_exact=w.n_exact, batch=w.batch)
        outs = []
        for _ in range(2):   # a second forward on the same handle starts from a reset counter
            r = h.forward(q, k, v, causal=w.mode, g=w.g, seed=w.seed, return_lse=True)
            torch.cuda.synchronize()
            h.check()
            outs.append(r)
        assert torch.equal(outs[0]["out"], outs[1]["out"])
        res.append(outs[0])
    for r in res[1:]:
        assert torch.equal(res[0]["out"], r["out"])
        assert torch.equal(res[0]["lse"], r["lse"])


def test_profile_steps_cover_the_halving_phases():
    w = W.WORKLOADS["express32k"].with_(T=8192, H=4)
    q, k, v = (x.cuda() for x in W.make_qkv(w))
    h = TA.ThinAttention(w.B, w.T, w.T, w.H, w.E, w.D, w.torch_dtype, n_exact=w.n_exact, batch=w.batch)
    h.forward(q, k, v, causal=True, g=w.g, seed=w.seed)
    h.profile(True)
    for _ in range(2):
        h.forward(q, k, v, causal=True, g=w.g, seed=w.seed)
    h.profile(False)
    ph = h.profile_read()
    sp = h.profile_steps()
    assert ph["calls"] == 2 and sp["calls"] == 2
    steps = sp["steps"]
    # steps that ran in the persistent halving launch report its time on the first of them, 0 after
    grouped = set()
    ent, _ = h.sched_layout(True, w.g)
    if ent:
        lay = h.trace_layout(True, w.g)
        rounds = {(lay[e][0], lay[e][1]) for e in ent}
        grouped = {i for i, s in enumerate(steps) if s["n"] > 128}
        assert len(rounds) > 0
    assert len(steps) > 0 and all(s["n_inst"] > 0 and s["n"] >= 2 for s in steps)
    assert all(s["ms"] > 0 for i, s in enumerate(steps) if i not in grouped or i == min(grouped))
    assert all(s["ms"] == 0 for i, s in enumerate(steps) if i in grouped and i != min(grouped))
    total = sum(s["ms"] for s in steps)
    assert abs(total - (ph["thin_ms"] + ph["merge_ms"])) <= 0.05 * total + 1e-3
    again = h.profile_steps()
    assert again["calls"] == 0 and all(s["ms"] == 0 for s in again["steps"])



# ---------------------------------------------------------------- Express with the page-literal cache
@pytest.mark.parametrize("T,n_out,g,dtype", [
    (2048, 32, 1, "bf16"),     # levels 0..2 (batches of 32, 128, 512 -> subsampled to 256), H_1, H_2
    (1500, 64, 2, "bf16"),     # level 2 a partial batch: H_2 over the three thinned level-1 batches
    (700, 16, 0, "fp32"),      # fp32 path, g = 0 (leaves of one point)
    (200, 64, 2, "bf16"),      # shorter than 4 n_out: exact attention throughout
])
def test_express_a_reduced(T, n_out, g, dtype):
    w = W.WORKLOADS["express32k_a"].with_(T=T, H=2, n_exact=n_out, g=g, dtype=dtype,
                                          E=128 if dtype == "bf16" else 64, D=128 if dtype == "bf16" else 64)
    res = run_case(w)
    assert_parity(res, dtype)


def test_express_a_32k_sampled_rows():
    w = W.WORKLOADS["express32k_a"]
    rows = np.sort(np.random.default_rng(3).choice(w.T, 128, replace=False))
    res = run_case(w, rows=rows, check_heads=[0, 17])
    assert_parity(res, "bf16")
