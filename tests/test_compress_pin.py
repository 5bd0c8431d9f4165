"""Pin of the oracle's KH-Compress tree and Express node tree against an independent recursion.

``tests/plain_kh.py`` builds the coreset by the recursion of Shetty, Dwivedi & Mackey ("Distribution
Compression in Near-linear Time": split into four contiguous quarters, compress each, concatenate in
order, halve), with its own Philox on Python integers, its own systematic subsample and the
plain-loop walk that evaluates psi from the points.  The oracle (``kh_compress`` / ``halve_level``)
works level by level on index arrays.  On every case below the two must give the same coreset
indices, with no decision taken differently outside a near tie (the oracle replays the plain walk's
decision only where its own swap margin is below 1e-4 of the kernel scale).

The pin must catch the mistakes a level-by-level tree invites; each is planted in a copy of the
oracle and must fail it: a pair counter that restarts in every group, groups taken with a stride
instead of contiguously, groups concatenated in the wrong order, and Express children merged in the
wrong order.
"""
import math

import numpy as np
import pytest

import oracle.thin_oracle as O
from tests.plain_kh import plain_compress, plain_express_nodes

# (S, g): S a power of 4, and S that is not L 4^r (a systematic subsample first)
CASES = [(16, 0), (16, 1), (64, 0), (64, 1), (64, 2), (256, 0), (256, 1), (256, 2), (256, 3),
         (20, 1), (50, 0), (50, 1), (77, 1), (100, 1), (100, 2), (200, 1), (200, 2), (300, 2),
         (1000, 3), (150, 0), (90, 2), (36, 0), (130, 2), (500, 2)]

E, D = 4, 3


def _points(S, seed, B=1, H=2, T=2):
    rng = np.random.default_rng(seed)
    k = rng.normal(size=(B, S, H, E)) * 0.8
    v = rng.normal(size=(B, S, H, D))
    q = rng.normal(size=(B, T, H, E))
    return q, k, v


def _follow(trace):
    """Plain trace {(bh, rid): {node position: flags}} -> the oracle's {(bh, rid): flags of the level}."""
    return {key: np.array([f for pos in sorted(d) for f in d[pos]], dtype=bool) for key, d in trace.items()}


def _compress_case(mod, S, g, seed=7):
    """True when the oracle module ``mod`` reproduces the plain recursion on this case."""
    q, k, v = _points(S, 1000 * S + g)
    Htot, hs, b0 = 5, [1, 3], 2                # Philox (b,h) words 11 and 13
    scale = 1 / math.sqrt(E)
    want, trace = [], {}
    for j, h in enumerate(hs):
        bh = b0 * Htot + h
        want.append(plain_compress(k[0, :, j].tolist(), v[0, :, j].tolist(), scale, g, seed, bh,
                                   lambda d: d, 0xC0000000, trace))
    ref = mod.thinformer(q, k, v, g, seed, follow=_follow(trace), heads=(Htot, hs), b0=b0)
    ok = ref.stats.mismatches == 0 and np.array_equal(ref.coreset[0], np.array(want))
    return ok, ref.stats.near_ties


def _express_case(mod, T, n_e, bsz, g, seed=3):
    q, k, v = _points(T, 17 * T + bsz, T=T)
    Htot, hs = 4, [0, 2]
    scale = 1 / math.sqrt(E)
    trace, want = {}, []
    for j, h in enumerate(hs):
        want.append(plain_express_nodes(k[0, :, j].tolist(), v[0, :, j].tolist(), scale, n_e, bsz, g, seed, h,
                                        trace))
    ref = mod.express(q, k, v, n_e, bsz, g, seed, follow=_follow(trace), rows=[0], heads=(Htot, hs))
    _, slots = mod.express_layout(T, n_e, bsz)
    got = ref.coreset[0]
    ok = ref.stats.mismatches == 0 and all(
        np.array_equal(got[j, s], np.array(want[j][slot])) for j in range(len(hs)) for s, slot in enumerate(slots))
    return ok, ref.stats.near_ties


EXPRESS_CASES = [(1280, 128, 64, 2), (900, 50, 100, 2), (700, 0, 40, 1), (1100, 60, 16, 1)]


@pytest.mark.parametrize("S,g", CASES)
def test_compress_tree_equals_plain_recursion(S, g):
    ok, near = _compress_case(O, S, g)
    assert ok
    assert near <= 2


@pytest.mark.parametrize("T,n_e,bsz,g", EXPRESS_CASES)
def test_express_nodes_equal_plain_recursion(T, n_e, bsz, g):
    ok, near = _express_case(O, T, n_e, bsz, g)
    assert ok
    assert near <= 2


def _planted(old, new):
    src = open(O.__file__).read()
    bad = src.replace(old, new)
    assert bad != src, old
    ns = {}
    exec(compile(bad, "planted_oracle", "exec"), ns)

    class M:
        pass

    m = M()
    for key in ("thinformer", "express", "express_layout"):
        setattr(m, key, ns[key])
    return m


PLANTS = {
    # the Philox pair counter restarts at 0 in every group of a level
    "restarting_counter": ("pair = np.arange(G * m, dtype=np.uint64)[None, :]",
                           "pair = np.tile(np.arange(m, dtype=np.uint64), G)[None, :]"),
    # group gi takes points gi, gi + G, gi + 2G, ... instead of a contiguous run
    "strided_groups": ("rows = np.arange(I)[:, None]\n",
                       "rows = np.arange(I)[:, None]\n"
                       "    idx = idx.reshape(I, n_group, G).transpose(0, 2, 1).reshape(I, n_cur)\n"),
    # the halved groups are concatenated last group first
    "reversed_concatenation": ("return np.where(keep, first, second)",
                               "return np.where(keep, first, second).reshape(I, G, m)[:, ::-1].reshape(I, G * m)"),
}


@pytest.mark.parametrize("plant", sorted(PLANTS))
def test_compress_pin_catches_a_planted_tree_mistake(plant):
    mod = _planted(*PLANTS[plant])
    failed = sum(not _compress_case(mod, S, g)[0] for S, g in CASES)
    assert failed >= 15, failed      # only the single-group trees (r = 1) cannot show it


def test_express_pin_catches_children_merged_out_of_order():
    mod = _planted("idx = np.concatenate([nodes[(lv, 4 * j + t)] for t in range(4)], axis=1)",
                   "idx = np.concatenate([nodes[(lv, 4 * j + t)] for t in (1, 0, 2, 3)], axis=1)")
    assert not all(_express_case(mod, *c)[0] for c in EXPRESS_CASES)
