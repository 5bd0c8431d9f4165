"""Express decode cache (the pages' updatable weighted cache object) against the fp64 oracle.

Decoding the tokens of a sequence one at a time must reproduce the oracle's Express prefill: token t
attends to the cache held after token t (exact prefix, the nodes of the completed batches, its own
batch), which is exactly what query t of the prefill sees.  Checked directly against
``oracle.express``: every node of the cache (token indices, bit for bit), every decoded row within
the bf16 / fp32 tolerance per (b,h) slice and per row, and every LSE.  The oracle replays the
thinning in follow mode on the decision trace of a prefill of the same tokens (taken only where a
decision is a near tie; any other disagreement fails).  The cache must also equal the library's
prefill bit for bit (same Philox rounds, same points, same halving kernels).
"""
import numpy as np
import pytest
import torch

import thinned_softmax_attention_b200 as TA
import workloads as W
from oracle import express

pytestmark = pytest.mark.gpu

TOL = {"fp32": 1e-5, "bf16": 1e-2}
ROW_TOL = {"fp32": 1e-4, "bf16": 2e-2}
LSE_TOL = {"fp32": 1e-5, "bf16": 2e-3}


@pytest.mark.parametrize("T,n_e,bsz,g,dtype,tiles", [
    (1152, 128, 64, 2, "bf16", False),   # 16 batches: level-1 merges and one level-2 merge
    (1152, 128, 64, 2, "bf16", True),    # the same through the query-tile attention kernels
    (700, 100, 96, 2, "bf16", False),    # batch not a power of 4 (subsample), trailing partial batch
    (300, 40, 16, 2, "fp32", False),     # batches stored whole (no thinning), fp32 path
])
def test_decode_matches_oracle(T, n_e, bsz, g, dtype, tiles, monkeypatch):
    """Few (b,h) rows take the split-key decode kernels; `tiles` forces the query-tile kernels."""
    if tiles:
        monkeypatch.setenv("THIN_ATTN_DECODE_TILES", "1")
    E = D = 128 if dtype == "bf16" else 64
    w = W.Workload("decode", 1, 2, T, T, E, D, dtype, True, g, 9, 6, "rope", n_exact=n_e, batch=bsz)
    qc, kc, vc = W.make_qkv(w)
    q, k, v = (x.cuda() for x in (qc, kc, vc))
    pre = TA.ThinAttention(w.B, T, T, w.H, E, D, w.torch_dtype, n_exact=n_e, batch=bsz)
    pf = pre.forward(q, k, v, causal=True, g=g, seed=w.seed, return_coreset=True, return_trace=True)
    torch.cuda.synchronize()
    follow = TA.decode_trace(pf["trace"], pre.trace_layout(True, g))
    ref = express(qc, kc, vc, n_e, bsz, g, w.seed, follow=follow, heads=(w.H, [0, 1]))
    assert ref.stats.mismatches == 0
    cache = TA.ThinAttentionCache(w.B, w.H, E, D, w.torch_dtype, capacity=T, n_exact=n_e, batch=bsz, g=g, seed=w.seed)
    outs, lses = [], []
    for t in range(T):
        lse = torch.empty(w.B, w.H, dtype=torch.float32, device="cuda")
        o = cache.decode(q[:, t:t + 1].contiguous(), k[:, t:t + 1].contiguous(), v[:, t:t + 1].contiguous(), lse=lse)
        outs.append(o)
        lses.append(lse)
    cache.check()
    assert len(cache) == T
    nodes = cache.nodes().cpu().numpy()
    assert np.array_equal(nodes, ref.coreset)
    assert torch.equal(cache.nodes(), pf["coreset"])
    o = torch.cat(outs, dim=1).float().cpu().numpy()
    d = np.abs(o - ref.out)
    slice_err = (d.max(axis=(1, 3)) / np.abs(ref.out).max(axis=(1, 3))).max()
    row_err = (d.max(axis=3) / np.abs(ref.out).max(axis=3)).max()
    assert slice_err <= TOL[dtype], slice_err
    assert row_err <= ROW_TOL[dtype], row_err
    lse = torch.stack(lses, dim=2).cpu().numpy()
    assert np.abs(lse - ref.lse).max() <= LSE_TOL[dtype]


@pytest.mark.parametrize("chunks", [[1, 7, 64, 200, 500, 380], [1152]])
def test_decode_n_equals_token_by_token(chunks):
    """Several tokens per call (batch boundaries, merges and the exact phase crossed inside a call):
    outputs, LSE and coresets bit-identical to one call per token."""
    T, n_e, bsz, g = 1152, 128, 64, 2
    w = W.Workload("decode", 1, 2, T, T, 128, 128, "bf16", True, g, 9, 6, "rope", n_exact=n_e, batch=bsz)
    q, k, v = (x.cuda() for x in W.make_qkv(w))
    one = TA.ThinAttentionCache(1, 2, 128, 128, w.torch_dtype, capacity=T, n_exact=n_e, batch=bsz, g=g, seed=w.seed)
    outs, lses = [], []
    for t in range(T):
        lse = torch.empty(1, 2, dtype=torch.float32, device="cuda")
        outs.append(one.decode(q[:, t:t + 1].contiguous(), k[:, t:t + 1].contiguous(), v[:, t:t + 1].contiguous(),
                               lse=lse))
        lses.append(lse)
    many = TA.ThinAttentionCache(1, 2, 128, 128, w.torch_dtype, capacity=T, n_exact=n_e, batch=bsz, g=g, seed=w.seed)
    got, got_lse, t0 = [], [], 0
    for n in chunks:
        lse = torch.empty(1, 2, n, dtype=torch.float32, device="cuda")
        got.append(many.decode_n(q[:, t0:t0 + n].contiguous(), k[:, t0:t0 + n].contiguous(),
                                 v[:, t0:t0 + n].contiguous(), lse=lse))
        got_lse.append(lse)
        t0 += n
    torch.cuda.synchronize()
    one.check()
    many.check()
    assert t0 == T and len(many) == T
    assert torch.equal(torch.cat(outs, dim=1), torch.cat(got, dim=1))
    assert torch.equal(torch.stack(lses, dim=2), torch.cat(got_lse, dim=2))
    assert torch.equal(one.nodes(), many.nodes())


def test_cache_refuses_tokens_beyond_capacity():
    w = W.WORKLOADS["express32k"].with_(H=1)
    cache = TA.ThinAttentionCache(1, 1, w.E, w.D, w.torch_dtype, capacity=2, n_exact=1, batch=1, g=0, seed=1)
    x = torch.zeros(1, 1, 1, w.E, dtype=w.torch_dtype, device="cuda")
    cache.decode(x, x, x)
    cache.decode(x, x, x)
    with pytest.raises(TA.ThinAttnError, match="capacity"):
        cache.decode(x, x, x)
