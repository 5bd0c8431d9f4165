"""Express decode cache (the pages' updatable weighted cache object) against the prefill.

Decoding the tokens of a sequence one at a time must reproduce the prefill: the same coresets
(token indices, bit for bit: same Philox rounds, same points, same kernels) and, for every token t,
the prefill's output row t within the bf16 / fp32 tolerance, since query t of the prefill attends
to exactly the cache the decoder holds after token t.
"""
import pytest
import torch

import thinned_softmax_attention_b200 as TA
import workloads as W

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T,n_e,bsz,g,dtype,tiles", [
    (1152, 128, 64, 2, "bf16", False),   # 16 batches: level-1 merges and one level-2 merge
    (1152, 128, 64, 2, "bf16", True),    # the same through the query-tile attention kernels
    (700, 100, 96, 2, "bf16", False),    # batch not a power of 4 (subsample), trailing partial batch
    (300, 40, 16, 2, "fp32", False),     # batches stored whole (no thinning), fp32 path
])
def test_decode_matches_prefill(T, n_e, bsz, g, dtype, tiles, monkeypatch):
    """Few (b,h) rows take the split-key decode kernels; `tiles` forces the query-tile kernels."""
    if tiles:
        monkeypatch.setenv("THIN_ATTN_DECODE_TILES", "1")
    E = D = 128 if dtype == "bf16" else 64
    w = W.Workload("decode", 1, 2, T, T, E, D, dtype, True, g, 9, 6, "rope", n_exact=n_e, batch=bsz)
    q, k, v = (x.cuda() for x in W.make_qkv(w))
    pre = TA.ThinAttention(w.B, T, T, w.H, E, D, w.torch_dtype, n_exact=n_e, batch=bsz)
    ref = pre.forward(q, k, v, causal=True, g=g, seed=w.seed, return_coreset=True, return_lse=True)
    cache = TA.ThinAttentionCache(w.B, w.H, E, D, w.torch_dtype, capacity=T, n_exact=n_e, batch=bsz, g=g, seed=w.seed)
    outs, lses = [], []
    for t in range(T):
        lse = torch.empty(w.B, w.H, dtype=torch.float32, device="cuda")
        o = cache.decode(q[:, t:t + 1].contiguous(), k[:, t:t + 1].contiguous(), v[:, t:t + 1].contiguous(), lse=lse)
        outs.append(o)
        lses.append(lse)
    cache.check()
    assert len(cache) == T
    assert torch.equal(cache.nodes(), ref["coreset"])
    o = torch.cat(outs, dim=1).float()
    r = ref["out"].float()
    err = ((o - r).abs().amax(dim=(1, 3)) / r.abs().amax(dim=(1, 3))).max().item()
    assert err <= (1e-2 if dtype == "bf16" else 1e-5), err
    lse = torch.stack(lses, dim=2)
    assert (lse - ref["lse"]).abs().max().item() <= (2e-3 if dtype == "bf16" else 1e-5)


def test_cache_refuses_tokens_beyond_capacity():
    w = W.WORKLOADS["express32k"].with_(H=1)
    cache = TA.ThinAttentionCache(1, 1, w.E, w.D, w.torch_dtype, capacity=2, n_exact=1, batch=1, g=0, seed=1)
    x = torch.zeros(1, 1, 1, w.E, dtype=w.torch_dtype, device="cuda")
    cache.decode(x, x, x)
    cache.decode(x, x, x)
    with pytest.raises(TA.ThinAttnError, match="capacity"):
        cache.decode(x, x, x)
