"""The C-ABI library loads, exports what include/thin_attn.h declares, and plans on the host.

No GPU: handles are created and planned only (thin_attn_create and the plan
queries touch no device); no compute entry point is called.
"""
import ctypes
import os
import re
import subprocess

import numpy as np
import torch
import pytest

import thinned_softmax_attention_b200 as T
import workloads as W
from oracle import compress_sizes, express_layout, round_batch, round_merge, round_noncausal

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "thin_attn.h")


def _declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"\b(thin_attn_[a-z_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    T.lib()
    out = subprocess.run(["nm", "-D", "--defined-only", T.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (thin_attn_\w+)", out))
    declared = set(_declared())
    assert declared, "no declarations parsed"
    assert declared <= exported, declared - exported
    assert set(T.EXPORTS) <= exported
    # nothing else leaks out of the library (hidden visibility)
    assert all(s.startswith("thin_attn_") for s in exported)


def test_version_and_error_strings():
    assert b"thin_attn" in T.lib().thin_attn_version()
    assert T.lib().thin_attn_last_error() is not None


def _handle(w, **kw):
    return T.ThinAttention(w.B, w.T, w.T if w.causal else w.S, w.H, w.E, w.D, w.torch_dtype,
                           n_exact=w.n_exact, batch=w.batch, **kw)


@pytest.mark.parametrize("name", ["tiny", "vit", "biggan"])
def test_noncausal_plan_matches_oracle_sizes(name):
    w = W.WORKLOADS[name]
    h = _handle(w)
    p = h.plan(False, w.g)
    r, L, Ss, C = compress_sizes(w.S, w.g)
    assert (p["levels"], p["leaf"], p["subsampled"], p["coreset_rows"]) == (r, L, Ss, C)
    assert p["coreset_idx_elems"] == w.B * w.H * C
    lay = h.trace_layout(False, w.g)
    # one entry per (b,h, level, group); every (b,h, level) covers all its pairs exactly once
    pairs = {}
    for bh, rid, pair0, m, off in lay:
        pairs.setdefault((bh, rid), []).append((pair0, m))
    assert len(pairs) == w.B * w.H * r
    for (bh, rid), parts in pairs.items():
        lv = rid
        assert rid == round_noncausal(lv) and 1 <= lv <= r
        parts.sort()
        assert parts[0][0] == 0 and all(a[0] + a[1] == b[0] for a, b in zip(parts, parts[1:]))
        assert parts[-1][0] + parts[-1][1] == Ss >> lv
    offs = sorted(e[4] for e in lay)
    assert len(set(offs)) == len(offs) and p["trace_words"] >= offs[-1] + 1


@pytest.mark.parametrize("name", ["express32k", "express128k"])
def test_express_plan_matches_oracle_layout(name):
    w = W.WORKLOADS[name]
    h = _handle(w)
    p = h.plan(True, w.g)
    n_b, slots = express_layout(w.T, w.n_exact, w.batch)
    r, L, Ss, c = compress_sizes(w.batch, w.g)
    assert (p["n_batches"], p["n_nodes"], p["coreset_rows"], p["levels"]) == (n_b, len(slots), c, r)
    assert p["coreset_idx_elems"] == w.B * w.H * len(slots) * c
    lay = h.trace_layout(True, w.g)
    rounds = {rid for _, rid, _, _, _ in lay}
    want = {round_batch(k, lv) for k in range(n_b) for lv in range(1, r + 1)}
    lv = 0
    while n_b // 4 ** (lv + 1):
        want |= {round_merge(lv + 1, j, s) for j in range(n_b // 4 ** (lv + 1)) for s in (0, 1)}
        lv += 1
    assert rounds == want
    assert len({e[0] for e in lay}) == w.B * w.H


def test_bad_arguments_are_rejected_on_the_host():
    w = W.WORKLOADS["tiny"]
    with pytest.raises(T.ThinAttnError, match="EINVAL"):
        T.ThinAttention(1, 8, 8, 1, 12, 64, w.torch_dtype)          # E not a multiple of 8
    h = _handle(w)
    for g in (-1, 7):
        with pytest.raises(T.ThinAttnError, match="EINVAL"):
            h.plan(False, g)
    with pytest.raises(T.ThinAttnError, match="EINVAL"):
        h.plan(True, 2)                                              # causal needs batch >= 1
    cfg = T.Config(0, 1, 8, 8, 1, 64, 64, 0.0, 0, 0, 0)
    hh = ctypes.c_void_p()
    assert T.lib().thin_attn_create(None, ctypes.byref(cfg)) == 1
    assert T.lib().thin_attn_create(ctypes.byref(hh), None) == 1
    assert T.lib().thin_attn_forward(None, None, None, None, None, 0, 2, 0, None, None, None, None) == 1
    assert T.lib().thin_attn_destroy(None) == 0


def test_shard_offsets_are_checked_on_the_host():
    w = W.WORKLOADS["express32k"]
    mk = lambda shard: T.ThinAttention(1, 4096, 4096, 4, w.E, w.D, w.torch_dtype, n_exact=1024, batch=1024,
                                       shard=shard)
    for bad in [(0, 2, 4), (-1, 0, 0), (0, -1, 8), (0, 0, 2), (1 << 30, 0, 8)]:
        with pytest.raises(T.ThinAttnError, match="EINVAL"):
            mk(bad)
    h = mk((3, 4, 8))                    # batch row 3, heads 4..7 of an 8-head problem
    assert h.trace_layout(True, 2) == mk((0, 0, 0)).trace_layout(True, 2)   # same instances, local (b,h)


def test_decode_trace_bit_order():
    lay = [(3, 7, 0, 40, 0), (3, 7, 40, 40, 2)]
    words = np.array([0b101, 1 << 7, 1, 0], dtype=np.uint32)
    d = T.decode_trace(words, lay)
    bits = d[(3, 7)]
    assert bits.shape == (80,)
    assert list(np.nonzero(bits)[0]) == [0, 2, 39, 40]


def _plan_pairs(h, causal, g):
    """(b*H+h, round id) -> pairs, from the plan's trace layout; each key's pair ranges tile 0..m."""
    parts = {}
    for bh, rid, pair0, m, _ in h.trace_layout(causal, g):
        parts.setdefault((bh, rid), []).append((pair0, m))
    out = {}
    for key, ps in parts.items():
        ps.sort()
        assert ps[0][0] == 0 and all(a[0] + a[1] == b[0] for a, b in zip(ps, ps[1:])), key
        out[key] = ps[-1][0] + ps[-1][1]
    return out


# (mode, B, H, T, S, g, n_exact, batch): mode 0 Thinformer, 1 Express, 2 Express with the page-literal cache
_PLAN_SWEEP = [
    (0, 1, 2, 4, 1, 2, 0, 0), (0, 1, 1, 4, 17, 0, 0, 0), (0, 2, 1, 4, 100, 1, 0, 0), (0, 1, 1, 4, 300, 2, 0, 0),
    (0, 1, 2, 4, 1000, 2, 0, 0), (0, 1, 1, 4, 3136, 2, 0, 0), (0, 1, 1, 4, 1024, 3, 0, 0), (0, 1, 1, 4, 4097, 5, 0, 0),
    (1, 1, 2, 700, 700, 2, 100, 64), (1, 1, 1, 1000, 1000, 1, 0, 64), (1, 1, 1, 2048, 2048, 2, 256, 96),
    (1, 1, 1, 300, 300, 2, 512, 256), (1, 1, 1, 700, 700, 2, 100, 16), (1, 1, 1, 5000, 5000, 2, 64, 64),
    (2, 1, 1, 700, 700, 2, 16, 0), (2, 1, 2, 2000, 2000, 1, 32, 0), (2, 1, 1, 3000, 3000, 2, 64, 0),
    (2, 1, 1, 100, 100, 2, 128, 0),
]


@pytest.mark.parametrize("mode,B,H,T_,S,g,n_e,bsz", _PLAN_SWEEP)
def test_plan_halvings_are_the_oracles(mode, B, H, T_, S, g, n_e, bsz):
    """The planner's halvings -- every (b,h, Philox round) and its pair count -- are exactly those the
    oracle's run of the same problem takes, in all three modes."""
    from oracle import express, express_a, thinformer
    rng = np.random.default_rng(mode * 1000 + S + g)
    L = S if mode == 0 else T_
    q = rng.normal(size=(B, T_, H, 8))
    k = rng.normal(size=(B, L, H, 8))
    v = rng.normal(size=(B, L, H, 8))
    if mode == 0:
        ref = thinformer(q, k, v, g, 3, rows=[0])
    elif mode == 1:
        ref = express(q, k, v, n_e, bsz, g, 3, rows=[0])
    else:
        ref = express_a(q, k, v, n_e, g, 3, rows=[0])
    h = T.ThinAttention(B, T_, L, H, 8, 8, W.WORKLOADS["tiny"].torch_dtype, n_exact=n_e, batch=bsz)
    assert _plan_pairs(h, mode, g) == {key: len(bits) for key, bits in ref.trace.items()}
    # and the coreset index output has the oracle's layout: (B,H,|C|), or (B,H,n_nodes,c) when causal
    p = h.plan(mode, g)
    assert p["coreset_idx_elems"] == ref.coreset.size
    if mode == 0:
        assert ref.coreset.shape == (B, H, p["coreset_rows"])
    else:
        assert ref.coreset.shape[:3] == (B, H, p["n_nodes"])
        assert p["n_nodes"] == 0 or ref.coreset.shape[3] == p["coreset_rows"]


def test_empty_inputs_and_the_largest_instance():
    """B, T, H = 0 or S = 0 are rejected on the host; the largest halving instance is 4096 points
    (the last level halves 2|C| points), one level beyond it is EUNSUPPORTED."""
    bf16 = W.WORKLOADS["vit"].torch_dtype
    for B_, T_, H_ in [(0, 4, 1), (1, 0, 1), (1, 4, 0)]:
        with pytest.raises(T.ThinAttnError, match="EINVAL"):
            T.ThinAttention(B_, T_, 4, H_, 64, 64, bf16)
    with pytest.raises(T.ThinAttnError, match="EINVAL"):
        T.ThinAttention(1, 4, 0, 1, 64, 64, bf16).plan(False, 2)
    for S, g, ok in [(16384, 4, True), (65536, 4, False), (16384, 5, False), (4096, 6, True)]:
        C = compress_sizes(S, g)[3]
        h = T.ThinAttention(1, 4, S, 1, 64, 64, bf16)
        assert ok == (compress_sizes(S, g)[0] == 0 or 2 * C <= 4096)
        if ok:
            assert h.plan(False, g)["coreset_rows"] == C
        else:
            with pytest.raises(T.ThinAttnError, match="EUNSUPPORTED"):
                h.plan(False, g)


def test_decode_cache_arguments_are_checked_on_the_host():
    bf16 = W.WORKLOADS["vit"].torch_dtype
    for kw in (dict(g=7), dict(g=-1), dict(batch=0), dict(n_exact=-1)):
        args = dict(capacity=4096, n_exact=1024, batch=1024, g=2)
        args.update(kw)
        with pytest.raises(T.ThinAttnError, match="EINVAL"):
            T.ThinAttentionCache(1, 4, 64, 64, bf16, **args)
    with pytest.raises(T.ThinAttnError, match="EINVAL"):
        T.ThinAttentionCache(1, 4, 12, 64, bf16, capacity=4096, n_exact=1024, batch=1024)   # E % 8


def _round_kind(rid):
    """(kind, fields) of a Philox round id: ('batch', k, level) / ('merge', level, node, step) / ('level', l)."""
    if rid & 0xC0000000 == 0x40000000:
        return ("batch", (rid >> 4) & 0x3FFFFFF, rid & 0xF)
    if rid & 0xC0000000 == 0x80000000:
        return ("merge", (rid >> 24) & 0x3F, (rid >> 1) & 0x7FFFFF, rid & 1)
    return ("level", rid)


@pytest.mark.parametrize("T,n_e,bsz,H", [(32768, 1024, 1024, 32), (8192, 1024, 1024, 4), (22000, 100, 600, 2)])
def test_sched_layout_merges_wait_for_their_children(T, n_e, bsz, H):
    """The persistent halving launch of an Express plan: the last level of every batch and both steps
    of every HALVE merge; the queue order is topological; the first step of merge (l, j) waits for
    exactly the four items that write its children (the last level of batches 4j..4j+3, or the second
    steps of merges (l-1, 4j..4j+3)) of the same (b,h), its second step for exactly its first."""
    w = W.WORKLOADS["express32k"].with_(T=T, H=H, n_exact=n_e, batch=bsz)
    h = _handle(w)
    ent, preds = h.sched_layout(True, w.g)
    lay = h.trace_layout(True, w.g)
    assert len(ent) > 0
    assert all(q < i for i, ps in enumerate(preds) for q in ps)
    last = h.plan(True, w.g)["levels"]
    keys = [(lay[e][0],) + _round_kind(lay[e][1]) for e in ent]
    where = {k: i for i, k in enumerate(keys)}
    assert len(where) == len(keys)
    n_merge = 0
    for i, k in enumerate(keys):
        bh, kind = k[0], k[1]
        if kind == "batch":
            assert k[3] == last and preds[i] == []
            continue
        assert kind == "merge"
        lv, j, step = k[2], k[3], k[4]
        if step == 1:
            assert preds[i] == [where[(bh, "merge", lv, j, 0)]]
            continue
        n_merge += 1
        if lv == 1:
            want = {where[(bh, "batch", 4 * j + c, last)] for c in range(4)}
        else:
            want = {where[(bh, "merge", lv - 1, 4 * j + c, 1)] for c in range(4)}
        assert set(preds[i]) == want
    n_b = (T - n_e) // bsz
    assert n_merge == H * sum(n_b >> (2 * lv) for lv in range(1, 8))


def test_sched_layout_noncausal_has_none():
    """The persistent halving launch is planned only where HALVE merges follow the last thinning level:
    a Thinformer compress (ViT's 192- and 384-point levels, BigGAN's) runs one launch per level."""
    for name in ("vit", "biggan"):
        w = W.WORKLOADS[name]
        assert _handle(w).sched_layout(False, w.g) == ([], [])


@pytest.mark.parametrize("kw", [dict(E=64), dict(D=256), dict(dtype="fp32", E=128, D=128), dict(H=129)])
def test_fp8_qk_refuses_unsupported_shapes(kw):
    """e4m3 QK^T is built for bf16 handles with E = 128 and D = 64 or 128: anything else is refused at
    creation, before any device work."""
    w = W.WORKLOADS["express32k"].with_(**kw)
    with pytest.raises(T.ThinAttnError, match="EUNSUPPORTED"):
        T.ThinAttention(w.B, w.T, w.T, w.H, w.E, w.D, w.torch_dtype, n_exact=w.n_exact, batch=w.batch, qk_fp8=True)


@pytest.mark.parametrize("mode,T_,S,ne,bsz", [(1, 3000, 3000, 200, 300), (1, 8192, 8192, 1024, 1024),
                                             (0, 3136, 3136, 0, 0), (2, 8192, 8192, 128, 0)])
def test_query_ranges_cover_every_row_once(mode, T_, S, ne, bsz):
    """Query-row shards (sequence parallelism): each range's plan attends exactly its rows, and ranges
    that partition [0, T) cover every row once -- also where the tiles do not start on multiples of
    128 (200 exact tokens, batches of 300), so tiles are clipped at the range ends."""
    dt = W.WORKLOADS["express32k"].torch_dtype
    full = T.ThinAttention(1, T_, S, 2, 128, 128, dt, n_exact=ne, batch=bsz).plan(mode, 2)
    assert full["attn_rows"] == T_
    cuts = [0, 1024, 1152, 2048, T_]
    total = 0
    for r in zip(cuts[:-1], cuts[1:]):
        h = T.ThinAttention(1, T_, S, 2, 128, 128, dt, n_exact=ne, batch=bsz, q_range=r)
        p = h.plan(mode, 2)
        assert p["attn_rows"] == r[1] - r[0]
        # the thinning is the whole run's: same halvings, same coreset layout
        assert p["n_halvings"] == full["n_halvings"] and p["coreset_idx_elems"] == full["coreset_idx_elems"]
        total += p["attn_rows"]
    assert total == T_


@pytest.mark.parametrize("r", [(100, 384), (0, 100), (256, 128), (-128, 128), (0, 3128), (128, 128)])
def test_query_range_must_be_aligned_and_inside(r):
    with pytest.raises(T.ThinAttnError, match="EINVAL"):
        T.ThinAttention(1, 3000, 3000, 2, 128, 128, W.WORKLOADS["express32k"].torch_dtype, n_exact=200, batch=300,
                        q_range=r)


def test_query_range_is_refused_by_the_host_path_and_the_cache():
    dt = W.WORKLOADS["express32k"].torch_dtype
    h = T.ThinAttention(1, 3000, 3000, 1, 128, 128, dt, n_exact=200, batch=300, q_range=(0, 1024))
    x = torch.zeros(1, 3000, 1, 128, dtype=dt)
    o = torch.zeros_like(x)
    p = ctypes.c_void_p
    st = T.lib().thin_attn_forward_host(h._h, p(x.data_ptr()), p(x.data_ptr()), p(x.data_ptr()), p(o.data_ptr()), 1, 2,
                                        ctypes.c_uint64(1), None, None)
    assert st == 5, st   # THIN_ATTN_EUNSUPPORTED, refused before any copy
    cfg = T.Config(T.BF16, 1, 64, 64, 1, 128, 128, 0.0, 16, 16, 0, 0, 0, 0, 0, 0, 64)
    c = ctypes.c_void_p()
    assert T.lib().thin_attn_cache_create(ctypes.byref(c), ctypes.byref(cfg), 2, ctypes.c_uint64(1)) != 0


@pytest.mark.parametrize("T_,ne,bsz,cuts", [(8192, 1024, 1024, [0, 2048, 4224, 8192]),
                                            (3000, 200, 300, [0, 128, 1152, 2048, 3000])])
def test_split_thinning_ranges_own_every_batch_once(T_, ne, bsz, cuts):
    """thin_split: batch k belongs to the range holding its last token; the ranges' batches partition
    the completed batches, and each plan holds its batches' halvings plus every merge."""
    dt = W.WORKLOADS["express32k"].torch_dtype
    full = T.ThinAttention(1, T_, T_, 2, 128, 128, dt, n_exact=ne, batch=bsz)
    n_full = full.plan(True, 2)["n_halvings"]
    hs = [T.ThinAttention(1, T_, T_, 2, 128, 128, dt, n_exact=ne, batch=bsz, q_range=r, thin_split=True)
          for r in zip(cuts[:-1], cuts[1:])]
    lays = [h.nodes_layout(2) for h in hs]
    n_b = (T_ - ne) // bsz
    assert [lay[2] for lay in lays] == [n_b] * len(hs)
    assert lays[0][0] == 0 and lays[-1][1] == n_b and all(a[1] == b[0] for a, b in zip(lays[:-1], lays[1:]))
    for (q0, q1), (k0, k1, _, _) in zip(zip(cuts[:-1], cuts[1:]), lays):
        assert all(q0 <= ne + (kk + 1) * bsz - 1 < q1 for kk in range(k0, k1))
    # a plan holds owned x P batch halvings plus every merge's M: solve P, M from two plans, then the
    # plans together hold the whole run's halvings with the merges counted once per plan
    counts = [h.plan(True, 2)["n_halvings"] for h in hs]
    owned = [k1 - k0 for k0, k1, _, _ in lays]
    i, j = min(range(len(hs)), key=owned.__getitem__), max(range(len(hs)), key=owned.__getitem__)
    P = (counts[j] - counts[i]) // (owned[j] - owned[i])
    M = counts[i] - owned[i] * P
    assert all(c == o * P + M for c, o in zip(counts, owned))
    assert sum(counts) - (len(hs) - 1) * M == n_full
    with pytest.raises(T.ThinAttnError, match="EUNSUPPORTED"):
        T.ThinAttention(1, T_, T_, 2, 128, 128, dt, n_exact=ne, batch=bsz, q_range=(0, 1024), thin_split=True).plan(2, 2)
