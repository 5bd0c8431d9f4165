"""The relations the Express summary prints for its cache (tests/golden/express_methodology.txt),
checked on the page-literal cache of the oracle (express_a, reading A).

The page fixes: the first n_out points are kept exactly; when the cache reaches 4 n_out it is
halved twice back to n_out; the cache never holds more than 6 n_out points.
"""
import os

import numpy as np
import torch

import workloads as W
from oracle import express_a
from oracle.thin_oracle import express_a_layout, round_merge

HERE = os.path.dirname(os.path.abspath(__file__))


def _golden():
    out = {}
    for line in open(os.path.join(HERE, "golden", "express_methodology.txt")):
        line = line.split("#")[0].strip()
        if line:
            key, val = (x.strip() for x in line.split("="))
            out[key] = int(val)
    return out


def _cache_sizes(T, n_out):
    """Points of the weighted cache over the stream under reading A, sampled after every batch: the
    exact tokens, then per level the HALVE output (n_out) and the level's completed thinned batches."""
    sizes = [min(T, n_out)]
    cache = min(T, n_out)
    level = 0
    for lv, s, start, length in express_a_layout(T, n_out):
        if lv != level:              # entering level lv: the cache was halved twice to n_out
            cache = n_out
            level = lv
        if length == 4 ** lv * n_out:
            cache += n_out           # a completed batch enters thinned to n_out points
        sizes.append(cache)
    return sizes


def test_cache_relations_of_the_page():
    g = _golden()
    for n_out in (16, 64, 128):
        for T in (n_out, 4 * n_out, 4 * n_out + 1, 16 * n_out + 7, 256 * n_out):
            sizes = _cache_sizes(T, n_out)
            assert max(sizes) <= g["cache_bound"] * n_out
            assert max(sizes) <= g["halve_threshold"] * n_out
            L = express_a_layout(T, n_out)
            # the exact phase: tokens [0, n_out) come before the first batch
            assert not L or L[0][2] == g["exact_phase_points"] * n_out


def test_halve_is_two_halvings_to_n_out():
    g = _golden()
    w = W.WORKLOADS["express32k"].with_(E=16, D=16)
    n_out, T = 16, 16 * 16 + 40
    q, k, v = W.make_qkv(w, T=T, heads=[0])
    o = express_a(q, k, v, n_out, 1, 5, heads=(w.H, [0]))
    # H_1 and H_2: two halvings each (steps 0 and 1 of round_merge(i, 0, t))
    for i in (1, 2):
        steps = [key for key in o.trace if key[1] in (round_merge(i, 0, 0), round_merge(i, 0, 1))]
        assert len(steps) == g["halvings_per_halve"]
        sizes = sorted(len(o.trace[key]) for key in steps)
        # 4 n_out points -> 2 n_out (2 n_out pairs), 2 n_out -> n_out (n_out pairs)
        assert sizes == [g["halve_output"] * n_out, 2 * n_out]
