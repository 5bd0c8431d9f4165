"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: a library
routine (torch SDPA / logsumexp, Triton's Philox run by its CPU interpreter), a
closed form, an invariant, an independent plain-loop implementation, or a
statistical property of Kernel Halving.  No GPU is needed.
"""
import json
import math
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import workloads as W
from oracle import (compress_sizes, exact_attention, express, express_a, express_a_layout, express_a_sizes,
                    express_layout, kappa_att,
                    kernel_halving, philox4x32_10, philox_uniform, round_batch, round_merge,
                    snapshot_nodes, subsample_indices, thinformer, weighted_attention)
from tests.plain_kh import plain_kernel_halving

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# ---------------------------------------------------------------- Philox


_TRITON_SNIPPET = r"""
import os, sys, json
os.environ["TRITON_INTERPRET"] = "1"
import torch, triton, triton.language as tl
from triton.language.random import philox_impl
@triton.jit
def kern(out, c, k):
    i = tl.arange(0, 1)
    a, b, cc, d = philox_impl(tl.load(c + 0 + i), tl.load(c + 1 + i), tl.load(c + 2 + i), tl.load(c + 3 + i),
                              tl.load(k + 0 + i), tl.load(k + 1 + i), 10)
    tl.store(out + 0 + i, a); tl.store(out + 1 + i, b); tl.store(out + 2 + i, cc); tl.store(out + 3 + i, d)
res = []
for c, k in json.loads(sys.stdin.read()):
    ct = torch.tensor(c, dtype=torch.int64).to(torch.uint32)
    kt = torch.tensor(k, dtype=torch.int64).to(torch.uint32)
    o = torch.zeros(4, dtype=torch.uint32)
    kern[(1,)](o, ct, kt)
    res.append([int(x) & 0xFFFFFFFF for x in o.view(torch.int32).tolist()])
print(json.dumps(res))
"""


def test_philox_matches_triton_interpreter():
    """Philox4x32-10 equals Triton's independent implementation (run on the CPU interpreter)."""
    rng = np.random.default_rng(0)
    cases = [([0, 0, 0, 0], [0, 0]), ([0xFFFFFFFF] * 4, [0xFFFFFFFF] * 2)]
    cases += [(rng.integers(0, 2 ** 32, 4).tolist(), rng.integers(0, 2 ** 32, 2).tolist()) for _ in range(14)]
    # the counter layouts the method uses: (pair, round id, b*H+h, 0)
    cases += [([5, round_batch(3, 2), 77, 0], [123456789, 0]), ([0, round_merge(2, 1, 1), 31, 0], [1, 0])]
    p = subprocess.run([sys.executable, "-c", _TRITON_SNIPPET], input=json.dumps(cases),
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert p.returncode == 0, p.stderr[-2000:]
    ref = json.loads(p.stdout.strip().splitlines()[-1])
    for (c, k), r in zip(cases, ref):
        got = [int(x) for x in philox4x32_10(*c, *k)]
        assert got == r, (c, k, [hex(x) for x in got], [hex(x) for x in r])


def test_philox_uniform_exact_and_uniform():
    u = philox_uniform(12345, 7, 3, np.arange(200_000, dtype=np.uint64))
    assert u.min() > 0.0 and u.max() < 1.0
    # u = (j + 1/2) 2^-23 for an integer j < 2^23: 24 significant bits, exact in fp32 and fp64
    j = u * 2.0 ** 23 - 0.5
    assert np.all(j == np.floor(j)) and np.all(u.astype(np.float32).astype(np.float64) == u)
    hist = np.histogram(u, bins=20, range=(0, 1))[0]
    chi2 = ((hist - len(u) / 20) ** 2 / (len(u) / 20)).sum()
    assert chi2 < 50.0     # 19 dof: p ~ 1e-4


def test_philox_streams_differ_by_counter_field():
    base = philox_uniform(1, 0, 1, np.arange(64, dtype=np.uint64))
    for other in (philox_uniform(1, 1, 1, np.arange(64, dtype=np.uint64)),
                  philox_uniform(1, 0, 2, np.arange(64, dtype=np.uint64)),
                  philox_uniform(2, 0, 1, np.arange(64, dtype=np.uint64))):
        assert not np.any(base == other)


# ---------------------------------------------------------------- attention


def _sdpa64(q, k, v, causal=False):
    """torch SDPA in float64 on the CPU; (T,E),(S,E),(S,D) -> (T,D)."""
    qt, kt, vt = (torch.as_tensor(x, dtype=torch.float64)[None, None] for x in (q, k, v))
    return torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=causal)[0, 0].numpy()


@pytest.mark.parametrize("T,S,E,D,causal", [(7, 7, 4, 4, False), (16, 40, 8, 24, False),
                                            (33, 33, 16, 8, True)])
def test_weighted_attention_matches_sdpa(T, S, E, D, causal):
    rng = np.random.default_rng(T * S)
    q, k, v = rng.normal(size=(T, E)), rng.normal(size=(S, E)), rng.normal(size=(S, D))
    mask = (np.arange(S)[None, :] <= np.arange(T)[:, None]) if causal else None
    o, lse = weighted_attention(q, k, v, 1 / math.sqrt(E), None, mask)
    np.testing.assert_allclose(o, _sdpa64(q, k, v, causal), rtol=1e-12, atol=1e-12)
    z = torch.as_tensor(q @ k.T / math.sqrt(E))
    if causal:
        z = z.masked_fill(~torch.as_tensor(mask), -math.inf)
    np.testing.assert_allclose(lse, torch.logsumexp(z, dim=1).numpy(), rtol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_exact_attention_matches_sdpa_per_batch_and_head(causal):
    """The (B,T,H,E) wrapper: every (b,h) slice and any subset of query rows equals torch's SDPA in
    fp64 on the (B,H,T,E) layout, with LSE from logsumexp."""
    rng = np.random.default_rng(21 + causal)
    B, T, H, E, D = 2, 19, 3, 8, 5
    q, k, v = rng.normal(size=(B, T, H, E)), rng.normal(size=(B, T, H, E)), rng.normal(size=(B, T, H, D))
    rows = np.array([0, 4, 11, 18])
    out, lse = exact_attention(q, k, v, causal=causal, rows=rows)
    qt, kt, vt = (torch.as_tensor(x).transpose(1, 2) for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=causal).transpose(1, 2)
    np.testing.assert_allclose(out, ref.numpy()[:, rows], rtol=1e-12, atol=1e-12)
    z = qt @ kt.transpose(-1, -2) / math.sqrt(E)
    if causal:
        z = z.masked_fill(torch.triu(torch.ones(T, T, dtype=torch.bool), 1), -math.inf)
    np.testing.assert_allclose(lse, torch.logsumexp(z, dim=-1).numpy()[:, :, rows], rtol=1e-12)


def test_weight_is_multiplicity():
    """A key of weight 2 is the same as that key listed twice (weights multiply exp(s q.k))."""
    rng = np.random.default_rng(1)
    q, k, v = rng.normal(size=(5, 6)), rng.normal(size=(4, 6)), rng.normal(size=(4, 3))
    logw = np.log(np.array([1.0, 2.0, 1.0, 3.0]))
    o, l = weighted_attention(q, k, v, 0.4, logw)
    kk = np.concatenate([k, k[[1, 3, 3]]])
    vv = np.concatenate([v, v[[1, 3, 3]]])
    o2, l2 = weighted_attention(q, kk, vv, 0.4)
    np.testing.assert_allclose(o, o2, rtol=1e-12)
    np.testing.assert_allclose(l, l2, rtol=1e-12)


def test_closed_forms_of_attention():
    rng = np.random.default_rng(2)
    v = rng.normal(size=(9, 5))
    k = np.tile(rng.normal(size=(1, 4)), (9, 1))         # all keys equal -> mean of v
    o, l = weighted_attention(rng.normal(size=(3, 4)), k, v, 0.5)
    np.testing.assert_allclose(o, np.tile(v.mean(0), (3, 1)), rtol=1e-12)
    k = np.zeros((9, 4)); k[4] = 100.0                     # one dominant key -> its value
    o, _ = weighted_attention(np.ones((2, 4)), k, v, 1.0)
    np.testing.assert_allclose(o, np.tile(v[4], (2, 1)), rtol=1e-12)


# ---------------------------------------------------------------- kappa_att


def test_kappa_matches_feature_expansion():
    """kappa = <phi(k,v), phi(k',v')> with the exponential kernel expanded in its Taylor
    features (E=1) and the augmented value (v, c): an independent route to the kernel."""
    rng = np.random.default_rng(3)
    K = rng.normal(size=(5, 1)); V = rng.normal(size=(5, 2)); s = 0.7; c = 1.9

    def feat(kx, vx):
        ex = np.array([math.sqrt(s ** n / math.factorial(n)) * kx ** n for n in range(40)])
        return np.kron(ex, np.append(vx, c))

    F = np.stack([feat(K[i, 0], V[i]) for i in range(5)])
    np.testing.assert_allclose(kappa_att(K, V, K, V, s, c * c), F @ F.T, rtol=1e-12)


def test_kappa_gram_symmetric_psd():
    rng = np.random.default_rng(4)
    K, V = rng.normal(size=(40, 8)), rng.normal(size=(40, 6))
    G = kappa_att(K, V, K, V, 1 / math.sqrt(8), np.abs(V).max() ** 2)
    np.testing.assert_allclose(G, G.T, rtol=1e-13)
    assert np.linalg.eigvalsh(G).min() > -1e-9 * np.abs(G).max()


# ---------------------------------------------------------------- Kernel Halving


def _rand_instances(I, n, E, D, seed, spread=1.0):
    rng = np.random.default_rng(seed)
    return rng.normal(size=(I, n, E)) * spread, rng.normal(size=(I, n, D)), rng.uniform(size=(I, n // 2))


def test_kh_one_survivor_per_pair():
    K, V, u = _rand_instances(20, 64, 8, 8, 5)
    r = kernel_halving(K, V, 0.35, u)
    assert r.keep_first.shape == (20, 32)     # exactly m decisions: one point of each pair survives


@pytest.mark.parametrize("n,E,D,spread", [(8, 3, 2, 1.0), (16, 4, 5, 1.5), (32, 2, 2, 0.5), (24, 6, 3, 2.0)])
def test_kh_agrees_with_plain_loop(n, E, D, spread):
    """Bit-identical decisions with the independent plain-loop walk (which evaluates psi from the points)."""
    K, V, u = _rand_instances(25, n, E, D, n * 7 + E, spread)
    s = 1 / math.sqrt(E)
    ref = []
    for i in range(K.shape[0]):
        keep, _, _ = plain_kernel_halving(K[i].tolist(), V[i].tolist(), s, u[i].tolist())
        ref.append(keep)
    ref = np.array(ref)
    r = kernel_halving(K, V, s, u, follow=ref)
    assert r.mismatch.sum() == 0
    assert (r.keep_first != ref).sum() == 0


def test_kh_first_pair_is_a_fair_coin():
    """Pair 0 has alpha = 0 and sigma = 0, so a = b^2 and p+ = 1/2: keep x iff u < 1/2."""
    K, V, _ = _rand_instances(6, 8, 3, 3, 6)
    for uval, want in ((0.25, True), (0.75, False), (2.0 ** -25, True), (1 - 2.0 ** -25, False)):
        u = np.full((6, 4), uval)
        assert np.all(kernel_halving(K, V, 0.5, u).keep_first[:, 0] == want)


def test_kh_follow_mode_replays_only_near_ties():
    """Near-tie follow mode. Pair 0 has alpha = 0 and a = b^2, so u = 1/2 puts its decision exactly on
    the swap boundary (margin 0). Following "keep x" there must give the walk that u = 1/4 gives
    (only pair 0's decision differs between the two, and it feeds alpha of every later pair);
    a followed decision that disagrees away from a near tie is flagged and not taken."""
    K, V, _ = _rand_instances(8, 32, 4, 4, 11)
    rng = np.random.default_rng(12)
    u = rng.uniform(0.05, 0.95, size=(8, 16))
    for first, u0 in ((True, 0.25), (False, 0.75)):
        ua, ub = u.copy(), u.copy()
        ua[:, 0], ub[:, 0] = u0, 0.5
        ref = kernel_halving(K, V, 0.5, ua)
        assert not ref.near[:, 0].any() and np.all(ref.keep_first[:, 0] == first)
        own = kernel_halving(K, V, 0.5, ub)
        assert own.near[:, 0].all()
        fol = kernel_halving(K, V, 0.5, ub, follow=ref.keep_first)
        assert np.array_equal(fol.keep_first, ref.keep_first)
        assert not fol.mismatch.any()
        assert np.array_equal(fol.near[:, 1:], ref.near[:, 1:])
    # a disagreement away from a near tie: flagged, and the walk keeps its own decision
    ref = kernel_halving(K, V, 0.5, u)
    bad = ref.keep_first.copy()
    far = ~ref.near
    far[:, :5] = False
    i, j = np.argwhere(far)[0]
    bad[i, j] = ~bad[i, j]
    fol = kernel_halving(K, V, 0.5, u, follow=bad)
    assert fol.mismatch.sum() == 1 and fol.mismatch[i, j]
    assert np.array_equal(fol.keep_first, ref.keep_first)


def _mmd2(G, sel):
    n = G.shape[0]
    w = -np.ones(n) / n
    w[sel] += 1.0 / len(sel)
    return w @ G @ w


def _mmd_ratio_vs_uniform(halving_fn, E=2, D=1, spread=0.3, n=512, I=60):
    """Mean MMD^2(kept half, all) of ``halving_fn`` over that of uniformly random halves.

    Low-dimensional points (E=2, D=1, small keys) give the kernel a small effective
    dimension; there the walk can balance its pair differences and must beat a coin flip.
    (In high dimension pair differences are nearly orthogonal and no rule can.)"""
    rng = np.random.default_rng(7)
    K = rng.normal(size=(I, n, E)) * spread
    V = rng.normal(size=(I, n, D))
    u = rng.uniform(size=(I, n // 2))
    s = 1 / math.sqrt(E)
    r = halving_fn(K, V, s, u)
    kh, un = [], []
    for i in range(I):
        G = kappa_att(K[i], V[i], K[i], V[i], s, np.abs(V[i]).max() ** 2)
        kh.append(_mmd2(G, np.where(r.keep_first[i], np.arange(0, n, 2), np.arange(1, n, 2))))
        un.append(_mmd2(G, np.where(rng.uniform(size=n // 2) < 0.5, np.arange(0, n, 2), np.arange(1, n, 2))))
    return np.mean(kh) / np.mean(un), r.clipped.mean()


def test_kh_beats_uniform_halving_in_mmd():
    """Kernel Halving's kept half is closer in MMD to the full set than a random half, and the
    walk almost never clips its swap probability (|alpha| <= a except with probability <= delta)."""
    ratio, clipped = _mmd_ratio_vs_uniform(kernel_halving)
    assert ratio < 0.4 and clipped <= 0.05


def test_mmd_pin_catches_an_inverted_swap_rule():
    """Plant a sign error in a copy of the oracle (keep x with probability (1 + alpha/a)/2):
    the MMD pin above must fail on it."""
    import oracle.thin_oracle as O
    src = open(O.__file__).read()
    bad = src.replace("pplus = np.clip(0.5 * (1.0 - alpha / a)", "pplus = np.clip(0.5 * (1.0 + alpha / a)")
    assert bad != src
    ns = {}
    exec(compile(bad, "planted_oracle", "exec"), ns)
    ratio, clipped = _mmd_ratio_vs_uniform(ns["kernel_halving"])
    assert ratio > 1.0 and clipped > 0.5


def test_kh_psi_norm_is_n2_mmd2():
    """For the kept half, n^2 MMD^2(kept, all) = ||psi_m||^2 with psi_m = sum_kept k - sum_discarded k."""
    K, V, u = _rand_instances(5, 32, 4, 4, 9)
    r = kernel_halving(K, V, 0.5, u)
    for i in range(5):
        G = kappa_att(K[i], V[i], K[i], V[i], 0.5, np.abs(V[i]).max() ** 2)
        sgn = np.where(np.repeat(r.keep_first[i], 2) == np.tile([True, False], 16), 1.0, -1.0)
        sel = np.nonzero(sgn > 0)[0]
        assert math.isclose(32 ** 2 * _mmd2(G, sel), sgn @ G @ sgn, rel_tol=1e-9)


def test_kh_duplicate_pair_keeps_first():
    K, V, u = _rand_instances(3, 8, 3, 3, 10)
    K[:, 3], V[:, 3] = K[:, 2], V[:, 2]       # pair 1 is two copies of one point: b^2 = 0
    r = kernel_halving(K, V, 0.5, np.full((3, 4), 0.999))
    assert np.all(r.keep_first[:, 1])


# ---------------------------------------------------------------- KH-Compress


def test_compress_sizes_of_the_workloads():
    # (S, g) -> (levels, leaf size, subsampled S', coreset size)
    assert compress_sizes(256, 2) == (2, 16, 256, 64)          # tiny: "coreset 2^g sqrt(S) = 64"
    assert compress_sizes(3136, 2) == (4, 12, 3072, 192)       # T2T-ViT shape
    assert compress_sizes(1024, 3) == (2, 64, 1024, 256)       # BigGAN shape
    assert compress_sizes(1024, 2) == (3, 16, 1024, 128)       # Express batch of 1024
    assert compress_sizes(2048, 2) == (4, 8, 2048, 128)        # Express batch of 2048
    for S, g in [(4 ** 5, 1), (4 ** 6, 2), (4 ** 4, 0)]:
        assert compress_sizes(S, g)[3] == 2 ** g * math.isqrt(S)
    for S in range(1, 300):
        for g in range(0, 4):
            r, L, Ss, C = compress_sizes(S, g)
            assert 1 <= L and Ss <= S and C == L * 2 ** r and (r == 0 or g == 0 or L <= 4 ** g)


def test_subsample_indices_are_distinct_increasing():
    for S, Ss in [(3136, 3072), (17, 16), (100, 64)]:
        for U in (0, 1, Ss - 1):
            idx = subsample_indices(S, Ss, np.array([U]))[0]
            assert len(idx) == Ss and idx[0] >= 0 and idx[-1] < S and np.all(np.diff(idx) >= 1)


@pytest.mark.parametrize("S,Ss", [(17, 16), (100, 64), (150, 64), (3136, 3072)])
def test_subsample_is_evenly_spread(S, Ss):
    """Systematic sampling with start U in [0, S'): every gap between kept indices is floor(S/S') or
    ceil(S/S'), index 0 is always kept, and over all U a token is kept between max(0, 2S' - S) and S'
    times (a window of S' starts can overlap at most one skipped run of S - S'), S'^2 times in all."""
    U = np.arange(Ss)
    idx = subsample_indices(S, Ss, U)
    gaps = np.unique(np.diff(idx, axis=1))
    assert set(gaps.tolist()) <= {S // Ss, -(-S // Ss)}
    assert np.all(idx[:, 0] == 0) and np.all(idx[:, -1] < S)
    counts = np.bincount(idx.ravel(), minlength=S)
    assert counts.sum() == Ss * Ss
    assert counts.min() >= max(0, 2 * Ss - S) and counts.max() <= Ss


@pytest.mark.parametrize("S,g", [(16, 2), (60, 3), (64, 3)])
def test_coreset_equal_full_set_is_exact_attention(S, g):
    """S <= 4^g: the coreset is every point (weight 1), so Thinformer is exact attention."""
    w = W.WORKLOADS["tiny"]
    q, k, v = W.make_qkv(w, T=24, S=S)
    o = thinformer(q, k, v, g, 1)
    assert o.coreset.shape[-1] == S
    ex = np.stack([_sdpa64(q[0, :, 0].double(), k[0, :, 0].double(), v[0, :, 0].double())])
    np.testing.assert_allclose(o.out[0, :, 0], ex[0], rtol=1e-11, atol=1e-12)


def test_thinformer_coreset_and_mass():
    w = W.WORKLOADS["tiny"]
    q, k, v = W.make_qkv(w)
    o = thinformer(q, k, v, w.g, w.seed)
    assert o.coreset.shape == (1, 1, 64)
    assert len(np.unique(o.coreset)) == 64
    # q = 0: every logit is ln(S/|C|), so lse = ln(|C| * S/|C|) = ln S
    oz = thinformer(torch.zeros_like(q), k, v, w.g, w.seed)
    np.testing.assert_allclose(oz.lse, math.log(256), rtol=1e-13)
    np.testing.assert_array_equal(oz.coreset, o.coreset)     # thinning ignores queries


def test_thinformer_is_better_than_uniform_coreset():
    """On clustered keys the KH coreset approximates attention better than a uniform subsample."""
    w = W.WORKLOADS["vit"].with_(B=4)
    q, k, v = W.make_qkv(w, T=512, S=1024)
    o = thinformer(q, k, v, w.g, w.seed)
    ex, _ = exact_attention(q, k, v)
    err_kh = np.abs(o.out - ex).mean()
    rng = np.random.default_rng(0)
    C = o.coreset.shape[-1]
    errs = []
    for b in range(4):
        sel = np.sort(rng.choice(1024, C, replace=False))
        ou, _ = weighted_attention(q[b, :, 0].double().numpy(), k[b, sel, 0].double().numpy(),
                                   v[b, sel, 0].double().numpy(), w.scale)
        errs.append(np.abs(ou - ex[b, :, 0]).mean())
    assert err_kh < np.mean(errs)


# ---------------------------------------------------------------- Express


def _small_express(T=1280, n_e=128, bsz=64, g=2, H=2, seed=5):
    w = W.WORKLOADS["express32k"]
    q, k, v = W.make_qkv(w, T=T, heads=range(H))
    return w, (q, k, v), express(q, k, v, n_e, bsz, g, seed, heads=(w.H, list(range(H))))


def test_express_exact_phase_is_exact_causal():
    w, (q, k, v), o = _small_express()
    ex, _ = exact_attention(q, k, v, causal=True)
    np.testing.assert_allclose(o.out[:, :128], ex[:, :128], rtol=1e-11, atol=1e-13)
    # first batch after the exact phase sees no node yet: exact causal too
    np.testing.assert_allclose(o.out[:, 128:192], ex[:, 128:192], rtol=1e-11, atol=1e-13)
    assert np.abs(o.out[:, 192:] - ex[:, 192:]).max() > 1e-6


def test_express_without_complete_batch_is_exact():
    w = W.WORKLOADS["express32k"]
    q, k, v = W.make_qkv(w, T=300, heads=[0])
    o = express(q, k, v, 100, 256, 2, 3, heads=(w.H, [0]))
    ex, _ = exact_attention(q, k, v, causal=True)
    np.testing.assert_allclose(o.out, ex, rtol=1e-11, atol=1e-13)


def test_express_mass_is_token_count():
    """q = 0: lse_t = ln(sum of weights seen by t) = ln(t+1) -- each node of level l stands for 4^l b tokens."""
    w = W.WORKLOADS["express32k"]
    q, k, v = W.make_qkv(w, T=64 + 64 * 21 + 30, heads=[0])
    o = express(torch.zeros_like(q), k, v, 64, 64, 1, 2, heads=(w.H, [0]))
    np.testing.assert_allclose(o.lse[0, 0], np.log(np.arange(q.shape[1]) + 1.0), rtol=1e-12)


def test_express_node_structure_and_cache_bound():
    w, (q, k, v), o = _small_express()
    n_b, slots = express_layout(1280, 128, 64)
    assert n_b == 18 and len(slots) == 18 + 4 + 1
    c = 32        # compress_sizes(64, 2) = (1, 16, 64, 32)
    assert o.coreset.shape == (1, 2, len(slots), c)
    for s, (lv, j) in enumerate(slots):
        node = o.coreset[0, 0, s]
        lo, hi = 128 + j * 4 ** lv * 64, 128 + (j + 1) * 4 ** lv * 64
        assert np.all((node >= lo) & (node < hi)) and len(np.unique(node)) == c
        assert o.weights[s] == 4 ** lv * 64 / c
    for kb in range(n_b + 1):
        nodes = snapshot_nodes(kb)
        assert len(nodes) == sum(int(d) for d in np.base_repr(kb, 4)) if kb else len(nodes) == 0
        levels = max(1, len(np.base_repr(max(kb, 1), 4)))
        assert 128 + c * len(nodes) + 64 <= 128 + 3 * c * levels + 64


def test_express_merges_only_equal_levels():
    for kb in range(1, 200):
        nodes = snapshot_nodes(kb)
        # consecutive batch ranges, oldest first, covering exactly batches [0, kb)
        covered = sorted((j * 4 ** lv, (j + 1) * 4 ** lv) for lv, j in nodes)
        assert covered[0][0] == 0 and covered[-1][1] == kb
        assert all(a[1] == b[0] for a, b in zip(covered, covered[1:]))
        assert all(sum(1 for x in nodes if x[0] == lv) <= 3 for lv, _ in nodes)


# ---------------------------------------------------------------- Express, page-literal cache (reading A)
def test_express_a_sizes():
    """Thinning N = m n_out tokens to n_out: S' = L 4^r = n_out 2^r, capped by N and by the COMPRESS2(g)
    input size n_out^2 / 4^g (leaves of at least 4^g points)."""
    assert express_a_sizes(128, 128, 2) == (0, 128, 128)       # inflation 1: kept whole
    assert express_a_sizes(512, 128, 2) == (2, 32, 512)        # 512 -> 256 -> 128, no subsample
    assert express_a_sizes(2048, 128, 2) == (3, 16, 1024)      # subsample to 1024 = 128^2 / 16
    assert express_a_sizes(8192, 128, 2) == (3, 16, 1024)
    for n_out in (16, 64, 128, 512):
        for g in (0, 1, 2):
            for i in range(5):
                N = 4 ** i * n_out
                r, L, S = express_a_sizes(N, n_out, g)
                assert S == L * 4 ** r == n_out * 2 ** r and S <= N and L * 2 ** r == n_out
                assert S <= max(n_out, n_out * n_out // 4 ** g)


def test_express_a_layout():
    L = express_a_layout(32768, 128)
    assert [b[3] for b in L] == [128] * 3 + [512] * 3 + [2048] * 3 + [8192] * 3
    assert all(b[2] == 128 + sum(x[3] for x in L[:j]) for j, b in enumerate(L))
    Lp = express_a_layout(5000, 128)    # last batch partial
    assert Lp[-1][2] + Lp[-1][3] == 5000 and Lp[-1][3] < 4 ** Lp[-1][0] * 128


def _small_express_a(T=16 * 64 + 100, zero_q=False, plant=None):
    w = W.WORKLOADS["express32k"].with_(E=16, D=16)
    q, k, v = W.make_qkv(w, T=T, heads=[0, 1])
    if zero_q:
        q = torch.zeros_like(q)
    return (q, k, v), express_a(q, k, v, 16, 1, 5, heads=(w.H, [0, 1]), _plant=plant)


def test_express_a_is_exact_until_the_first_halve():
    """With inflation 1 a batch of n_out tokens is kept whole: tokens [0, 4 n_out) are attended exactly."""
    (q, k, v), o = _small_express_a()
    ex, _ = exact_attention(q, k, v, causal=True)
    np.testing.assert_allclose(o.out[:, :64], ex[:, :64], rtol=1e-11, atol=1e-13)
    assert np.abs(o.out[:, 64:] - ex[:, 64:]).max() > 1e-6


def test_express_a_mass_is_token_count():
    """q = 0: lse_t = ln(total weight seen by t) = ln(t+1): the HALVE outputs and the thinned batches
    of level i weigh 4^i each, the raw tokens of the batch in progress 1."""
    (q, k, v), o = _small_express_a(zero_q=True)
    np.testing.assert_allclose(o.lse[0, 0], np.log(np.arange(q.shape[1]) + 1.0), rtol=1e-12)
    np.testing.assert_allclose(o.lse[0, 1], np.log(np.arange(q.shape[1]) + 1.0), rtol=1e-12)


def test_express_a_mass_pin_catches_a_wrong_weight():
    (q, k, v), o = _small_express_a(zero_q=True, plant="weight")
    assert np.abs(o.lse[0, 0] - np.log(np.arange(q.shape[1]) + 1.0)).max() > 0.1


def test_express_a_node_structure():
    """T = 1124, n_out = 16: levels 1 and 2 complete, level 3 a partial batch -> slots H_1, B(1,1..3),
    H_2, B(2,1..3), H_3; every node n_out distinct tokens in time order, inside its batch (thinned
    batches) or inside the tokens its HALVE consumed (H_i: tokens [0, 4^i n_out))."""
    T = 16 * 64 + 100
    (q, k, v), o = _small_express_a(T=T)
    L = express_a_layout(T, 16)
    assert o.coreset.shape == (1, 2, 9, 16)
    np.testing.assert_array_equal(o.weights, [4, 4, 4, 4, 16, 16, 16, 16, 64])
    ranges = ([(0, 64)] + [(b[2], b[2] + b[3]) for b in L if b[0] == 1] + [(0, 256)] +
              [(b[2], b[2] + b[3]) for b in L if b[0] == 2] + [(0, 1024)])
    for sl, (lo, hi) in enumerate(ranges):
        for h in range(2):
            node = o.coreset[0, h, sl]
            assert len(node) == 16 and np.all(np.diff(node) > 0) and node[0] >= lo and node[-1] < hi


def test_attention_operands_leave_the_thinning_alone():
    """Attention with separately given q and k (the e4m3 QK^T path attends with rounded copies) keeps
    the coresets and the decisions of the original keys; given the inputs themselves it is the default
    run bit for bit; and its outputs are the weighted attention of those operands over the same keys."""
    w = W.WORKLOADS["express32k"].with_(T=1280, H=2, n_exact=128, batch=128)
    q, k, v = W.make_qkv(w)
    rows = np.arange(0, 1280, 53)
    base = express(q, k, v, 128, 128, 2, 4, rows=rows)
    same = express(q, k, v, 128, 128, 2, 4, rows=rows, attn_q=q, attn_k=k)
    assert np.array_equal(base.out, same.out) and np.array_equal(base.lse, same.lse)
    qa, ka = q.double() * 1.5, k.double().flip(-1)
    alt = express(q, k, v, 128, 128, 2, 4, rows=rows, attn_q=qa, attn_k=ka)
    assert np.array_equal(alt.coreset, base.coreset) and alt.trace.keys() == base.trace.keys()
    assert all(np.array_equal(alt.trace[key], base.trace[key]) for key in base.trace)
    # exact-phase rows (t < n_e): plain causal attention of the given operands
    t = rows[rows < 128]
    o, _ = weighted_attention(qa[0, t, 1].numpy(), ka[0, :128, 1].numpy(), v[0, :128, 1].double().numpy(), w.scale,
                              None, np.arange(128)[None, :] <= t[:, None])
    np.testing.assert_allclose(alt.out[0, :len(t), 1], o, rtol=1e-12, atol=1e-14)
    # Thinformer likewise
    wt = W.WORKLOADS["tiny"]
    qt, kt, vt = W.make_qkv(wt)
    b0 = thinformer(qt, kt, vt, 2, 1)
    b1 = thinformer(qt, kt, vt, 2, 1, attn_q=qt * 2.0, attn_k=kt)
    assert np.array_equal(b0.coreset, b1.coreset) and not np.allclose(b0.out, b1.out)
