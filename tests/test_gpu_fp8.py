"""e4m3 QK^T (thin_attn_config::qk_fp8) against the fp64 oracle run with the same e4m3-rounded operands.

The library copies q, k and the coreset keys to e4m3 with one scale per (b,h) and tensor (448 / the
slice's largest |x|, in fp32), multiplies the e4m3 values on the tensor cores and undoes the scales in
the softmax; the thinning keeps the bf16 keys.  The oracle reference rounds q and k the same way (an
fp32 product with the same fp32 scale, then torch's round-to-nearest-even e4m3 cast), divides the
scale back out in fp64 and attends with those operands (attn_q / attn_k), so the comparison isolates
the kernel's arithmetic: the decisions and coresets must match as in bf16 (the keys of the thinning are
the same) and the outputs within the bf16 tolerance.  The distance to the bf16 path's outputs is
reported (the e4m3 rounding of q and k itself; ~5e-3 per slice on Express shapes).
"""
import numpy as np
import pytest
import torch

import thinned_softmax_attention_b200 as TA
import workloads as W
from oracle import express, express_a, thinformer

pytestmark = pytest.mark.gpu


def _e4m3_rounded(x):
    """x (B, L, H, E) bf16 -> e4m3(x scale) / scale in fp64, scale = 448 / max|x| per (b,h) in fp32."""
    xf = x.float()
    amax = xf.abs().amax(dim=(1, 3), keepdim=True)
    scale = torch.where(amax > 0, torch.tensor(448.0, dtype=torch.float32) / amax, torch.ones_like(amax))
    return (xf * scale).to(torch.float8_e4m3fn).double() / scale.double()


def _rel(o, r):
    d = np.abs(o - r)
    return float((d.max(axis=(1, 3)) / np.abs(r).max(axis=(1, 3))).max()), float((d.max(axis=3) / np.abs(r).max(axis=3)).max())


def _run(w, T, S, rows, heads=None):
    q, k, v = W.make_qkv(w, T=T, S=S)
    dev = torch.device("cuda", 0)
    res = {}
    for fp8 in (True, False):
        h = TA.ThinAttention(w.B, T, S, w.H, w.E, w.D, w.torch_dtype, n_exact=w.n_exact, batch=w.batch, qk_fp8=fp8)
        r = h.forward(q.to(dev), k.to(dev), v.to(dev), causal=w.mode, g=w.g, seed=w.seed, return_lse=True,
                      return_coreset=True, return_trace=True)
        torch.cuda.synchronize()
        h.check()
        res[fp8] = (h, r)
    h, r = res[True]
    follow = TA.decode_trace(r["trace"], h.trace_layout(w.mode, w.g))
    hs = list(range(w.H)) if heads is None else list(heads)
    qh, kh, vh = q[:, :, hs], k[:, :, hs], v[:, :, hs]
    qa, ka = _e4m3_rounded(q)[:, :, hs], _e4m3_rounded(k)[:, :, hs]
    kw = dict(follow=follow, rows=rows, heads=(w.H, hs), attn_q=qa, attn_k=ka)
    if not w.causal:
        ref = thinformer(qh, kh, vh, w.g, w.seed, **kw)
    elif w.cache == "A":
        ref = express_a(qh, kh, vh, w.n_exact, w.g, w.seed, **kw)
    else:
        ref = express(qh, kh, vh, w.n_exact, w.batch, w.g, w.seed, **kw)
    assert ref.stats.mismatches == 0
    assert np.array_equal(r["coreset"].cpu().numpy()[:, hs], ref.coreset)
    assert torch.equal(r["coreset"], res[False][1]["coreset"])
    o = r["out"].float().cpu().numpy()[:, rows][:, :, hs]
    slice_err, row_err = _rel(o, ref.out)
    assert slice_err <= 1e-2, slice_err
    assert row_err <= 2e-2, row_err
    lse = r["lse"].cpu().numpy()[:, hs][:, :, rows]
    assert np.abs(lse - ref.lse).max() <= 2e-3
    ob = res[False][1]["out"].float().cpu().numpy()[:, rows][:, :, hs]
    return slice_err, _rel(o, ob)[0]


@pytest.mark.parametrize("case", ["express", "express_ragged", "express_a", "noncausal"])
def test_fp8_qk_matches_oracle_with_rounded_operands(case):
    w = {"express": W.WORKLOADS["express32k"].with_(H=2),
         "express_ragged": W.WORKLOADS["express32k"].with_(H=3, n_exact=200, batch=300),
         "express_a": W.WORKLOADS["express32k_a"].with_(H=2),
         "noncausal": W.WORKLOADS["express32k"].with_(causal=False, B=2, H=2, g=2)}[case]
    T, S = {"express": (8192, 8192), "express_ragged": (3000, 3000), "express_a": (8192, 8192),
            "noncausal": (600, 5000)}[case]
    rows = np.sort(np.random.default_rng(5).choice(T, 160, replace=False))
    err, vs_bf16 = _run(w, T, S, rows)
    assert vs_bf16 <= 3e-2, vs_bf16


def test_fp8_qk_express32k_sampled_rows():
    """The full Express 32K workload in the bench's launch configuration, sampled rows of three heads."""
    w = W.WORKLOADS["express32k"]
    rows = np.sort(np.random.default_rng(6).choice(w.T, 128, replace=False))
    _run(w, w.T, w.T, rows, heads=[0, 16, 31])
