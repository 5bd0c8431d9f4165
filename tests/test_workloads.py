"""The seeded input generator shared by the oracle and the CUDA path (no method arithmetic in it).

RoPE follows its definition: rows rotated pairwise by position-dependent angles, so inner
products depend only on the distance between positions. Slices are pure functions of
(workload, b, h), so a shard's draw is the matching slice of the whole problem's draw.
"""
import math

import numpy as np
import torch

import workloads as W


def test_rope_closed_form():
    """Row t, pair i = (2i, 2i+1) is rotated by the angle t * 10000^(-2i/E)."""
    E, T = 4, 3
    x = torch.tensor([[1.0, 2.0, 3.0, 4.0]]).repeat(T, 1)
    r = W._rope(x).double()
    for t in range(T):
        for i, (a, b) in enumerate(((1.0, 2.0), (3.0, 4.0))):
            ang = t * 10000.0 ** (-2.0 * i / E)
            want = (a * math.cos(ang) - b * math.sin(ang), a * math.sin(ang) + b * math.cos(ang))
            np.testing.assert_allclose(r[t, 2 * i:2 * i + 2].numpy(), want, rtol=1e-6, atol=1e-6)


def test_rope_inner_products_depend_on_distance_only():
    E, T = 16, 40
    g = torch.Generator().manual_seed(5)
    x, y = torch.randn(E, generator=g), torch.randn(E, generator=g)
    rx, ry = W._rope(x.repeat(T, 1)).double(), W._rope(y.repeat(T, 1)).double()
    np.testing.assert_allclose(rx.norm(dim=1).numpy(), float(x.norm()), rtol=1e-5)
    for d in (0, 3, 17):
        dots = (rx[d:] * ry[:T - d]).sum(dim=1).numpy()
        np.testing.assert_allclose(dots, dots[0], rtol=1e-4, atol=1e-4)


def test_slices_are_deterministic_and_distinct():
    w = W.WORKLOADS["express32k"].with_(T=64, H=2)
    a, b = W.slice_qkv(w, 0, 1), W.slice_qkv(w, 0, 1)
    assert all(torch.equal(x, y) for x, y in zip(a, b))
    c = W.slice_qkv(w, 0, 0)
    assert not torch.equal(a[0], c[0])


def test_shard_draw_is_a_slice_of_the_whole():
    for name in ("vit", "express32k"):
        w = W.WORKLOADS[name].with_(B=3, H=4, T=64, S=64)
        whole = W.make_qkv(w)
        part = W.make_qkv(w.with_(B=2), heads=[1, 3], b0=1)
        for x, y in zip(whole, part):
            assert torch.equal(x[1:3][:, :, [1, 3]], y)


def test_workload_shapes_and_scales():
    """Keys and queries of the rank-8 and RoPE recipes are scaled by E^(-1/4), values are N(0,1)."""
    for name in ("vit", "express32k", "biggan"):
        w = W.WORKLOADS[name].with_(T=512, S=512, B=1, H=1)
        q, k, v = W.slice_qkv(w, 0, 0)
        assert q.shape == (512, w.E) and k.shape == (512, w.E) and v.shape == (512, w.D)
        assert q.dtype == w.torch_dtype
        kv = k.double().pow(2).mean().item()
        want = 1.0 if w.kind == "iid" else (1.0 + 0.25) / math.sqrt(w.E) if w.kind == "rank8" else 1.0 / math.sqrt(w.E)
        assert abs(kv / want - 1) < 0.1, (name, kv, want)
        assert abs(v.double().pow(2).mean().item() - 1) < 0.1
