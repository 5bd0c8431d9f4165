"""thin_attn_halve_noalloc: Kernel Halving with no device allocation, checked against thin_attn_forward.

Some callers cannot allocate device memory while they run (their memory belongs to a pool of
their own, or an allocation's device-wide synchronisation and possible failure is not
acceptable mid-run).  The no-allocation entry point keeps its scratch in a fixed array inside
the library.  Here it must reproduce, bit for bit, the first halving level of the regular
entry point (same Philox counters, same kernel, same walk) on two calls in a row, the second
of which finds the scratch holding the first call's contents.

This file is collected last so that a stop at the first failure has run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import thinned_softmax_attention_b200 as TA
import workloads as W

pytestmark = pytest.mark.gpu


def _noalloc_fn():
    f = TA.lib().thin_attn_halve_noalloc
    vp, i = ctypes.c_void_p, ctypes.c_int
    f.argtypes = [i, vp, vp, i, i, i, i, ctypes.c_float, ctypes.c_uint64, ctypes.c_uint32, vp, vp, vp, vp, vp]
    f.restype = ctypes.c_int
    return f


def _call(Ks, Vs, seed, round_id):
    BH, n, E = Ks.shape
    D = Vs.shape[2]
    m = n // 2
    Ko = torch.empty(BH, m, E, dtype=Ks.dtype, device=Ks.device)
    Vo = torch.empty(BH, m, D, dtype=Vs.dtype, device=Vs.device)
    idx = torch.empty(BH, m, dtype=torch.int32, device=Ks.device)
    words = (n + 63) // 64
    bits = torch.zeros(BH * words, dtype=torch.int32, device=Ks.device)
    dt = 0 if Ks.dtype == torch.float32 else 1
    st = _noalloc_fn()(dt, Ks.data_ptr(), Vs.data_ptr(), BH, n, E, D, 0.0, seed, round_id, Ko.data_ptr(),
                       Vo.data_ptr(), idx.data_ptr(), bits.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == 0, TA.lib().thin_attn_last_error().decode()
    torch.cuda.synchronize()
    return Ko, Vo, idx, bits


@pytest.mark.parametrize("S,g,E,D,dtype,B,H", [
    (64, 2, 64, 128, "bf16", 2, 3), (256, 3, 128, 128, "bf16", 2, 3), (128, 3, 64, 64, "fp32", 2, 3),
    (1024, 4, 64, 64, "bf16", 2, 3),     # 6 sets of 1024 points: 6 MiB of pair differences
    (2048, 5, 64, 128, "bf16", 1, 3),    # 3 sets of 2048 points: 12 MiB, near the scratch's limit
])
def test_noalloc_matches_forward_twice(S, g, E, D, dtype, B, H):
    # S with 4^g < S <= 4^(g+1) and S = 4L: KH-Compress is a single halving of all S keys of each
    # (b,h) with Philox round id 1 and counter word b*H+h -- the instance index below.
    w = W.Workload("noalloc", B, H, 16, S, E, D, dtype, False, g, 5, 8, "iid")
    q, k, v = (x.cuda() for x in W.make_qkv(w))
    h = TA.ThinAttention(w.B, w.T, S, w.H, E, D, w.torch_dtype)
    plan = h.plan(False, g)
    assert plan["levels"] == 1 and plan["coreset_rows"] == S // 2
    ref = h.forward(q, k, v, causal=False, g=g, seed=w.seed, return_coreset=True, return_trace=True)
    torch.cuda.synchronize()
    BH = w.B * w.H
    ref_idx = ref["coreset"].reshape(BH, S // 2)
    ref_bits = ref["trace"][: BH * ((S + 63) // 64)]
    Ks = k.permute(0, 2, 1, 3).reshape(BH, S, E).contiguous()
    Vs = v.permute(0, 2, 1, 3).reshape(BH, S, D).contiguous()
    for _ in range(2):
        Ko, Vo, idx, bits = _call(Ks, Vs, w.seed, 1)
        assert torch.equal(idx, ref_idx)
        assert torch.equal(bits, ref_bits)
        rows = torch.arange(BH, device="cuda")[:, None]
        assert torch.equal(Ko, Ks[rows, idx.long()])
        assert torch.equal(Vo, Vs[rows, idx.long()])
        # one point of every pair
        assert torch.equal(idx.long() // 2, torch.arange(S // 2, device="cuda").expand(BH, -1))


def test_noalloc_rejects_requests_beyond_its_scratch():
    f = _noalloc_fn()
    x = torch.empty(16, dtype=torch.float32, device="cuda")
    # 4096 sets of 4096 points would need 4096 * 2048^2 * 4 bytes of pair differences
    st = f(0, x.data_ptr(), x.data_ptr(), 4096, 4096, 8, 8, 0.0, 1, 1, x.data_ptr(), x.data_ptr(),
           x.data_ptr(), None, None)
    assert st == 1
    assert "maximum" in TA.lib().thin_attn_last_error().decode()
