"""Plain fp64 CPU oracle of Thinformer and Thinformer Express attention.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
legs of ``bench.py`` may import this module.  The CUDA library never calls it,
and it shares no code, tables or helpers with the CUDA path; the only common
code is the seeded input generator in ``workloads.py``.

What the pages fix, and what is a reading of them
-------------------------------------------------
The sources are the Thinformer README ("Getting Started": layouts and API) and
the summary "Express Language Modeling" (Methodology: "The EXPRESS
Meta-Procedure" and "Thinformer Express").  They name the pieces but print no
algorithm, so each step below states the reading it takes:

* exact softmax attention, optionally weighted (a weight w_j multiplies
  exp(s q.k_j) in numerator and denominator)                      -- fixed
* the key-value attention kernel kappa_att                        -- reading:
  kappa((k,v),(k',v')) = exp(s<k,k'>) * (<v,v'> + c^2), c = max |v| of the
  halving instance
* Kernel Halving (Dwivedi & Mackey, "Kernel Thinning", self-balancing
  walk with delta = 1/2, delta_i = delta/m)                        -- reading
* KH-Compress (Shetty, Dwivedi & Mackey, "Distribution Compression in
  Near-linear Time": 4-way split, compress, concatenate, halve), with a
  systematic uniform subsample when S is not L*4^r                 -- reading
* Philox4x32-10 (Salmon, Moraes, Dror & Shaw, SC'11) keyed on the seed,
  counter (pair, round id, b*H+h, 0), u = ((x0 >> 9) + 1/2) 2^-23  -- reading
  (24 significant bits, so u is exact in fp32 as well as fp64)
* Express: exact phase of n_e tokens; fixed batches of b tokens thinned to
  c points of weight b/c; a 4-ary counter merges four equal-level coresets
  by two halvings into one of 4x the weight ("HALVE" phase)      -- reading

The oracle is pinned by ``tests/test_oracle_pins.py`` (library routines,
closed forms, invariants, statistics, an independent plain-loop walk) and
``tests/test_golden.py`` (the cache relations the Express summary prints).
The exact sequence of KH decisions has no printed value to check against: it
is pinned only by the invariants and by the independent plain-loop walk.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Callable, Dict, Optional, Tuple

import numpy as np

# --------------------------------------------------------------------------
# Philox4x32-10 (Salmon et al., "Parallel random numbers: as easy as 1, 2, 3",
# SC'11): ten rounds of two 32x32->64 multiplies; the key is bumped by the
# Weyl constants between rounds.
# --------------------------------------------------------------------------
_MASK = np.uint64(0xFFFFFFFF)
_M0 = np.uint64(0xD2511F53)
_M1 = np.uint64(0xCD9E8D57)
_W0 = np.uint64(0x9E3779B9)
_W1 = np.uint64(0xBB67AE85)
_S32 = np.uint64(32)


def philox4x32_10(c0, c1, c2, c3, k0, k1):
    """Vectorised Philox4x32-10; arguments are integer arrays holding 32-bit words."""
    c0, c1, c2, c3, k0, k1 = (np.asarray(x, dtype=np.uint64) & _MASK
                              for x in (c0, c1, c2, c3, k0, k1))
    for r in range(10):
        if r:
            k0 = (k0 + _W0) & _MASK
            k1 = (k1 + _W1) & _MASK
        p0 = c0 * _M0          # exact: both factors < 2^32
        p1 = c2 * _M1
        c0, c1, c2, c3 = ((p1 >> _S32) ^ c1 ^ k0,
                          p1 & _MASK,
                          (p0 >> _S32) ^ c3 ^ k1,
                          p0 & _MASK)
    return c0, c1, c2, c3


def round_noncausal(level: int) -> int:
    return level


def round_batch(k: int, level: int) -> int:
    return 0x40000000 | (k << 4) | level


def round_merge(level: int, node: int, step: int) -> int:
    return 0x80000000 | (level << 24) | (node << 1) | step


def round_subsample(k: int) -> int:
    return 0xC0000000 | k


def philox_word(seed: int, bh, round_id, pair):
    """First output word x0 of Philox4x32-10 at counter (pair, round, bh, 0)."""
    x0, _, _, _ = philox4x32_10(pair, round_id, bh, 0, seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF)
    return x0


def philox_uniform(seed: int, bh, round_id, pair):
    """u = ((x0 >> 9) + 0.5) * 2^-23 in (0, 1): an odd multiple of 2^-24, exact in fp32 and fp64."""
    x0 = philox_word(seed, bh, round_id, pair)
    return ((x0 >> np.uint64(9)).astype(np.float64) + 0.5) * 2.0 ** -23


# --------------------------------------------------------------------------
# Exact (weighted) softmax attention -- the quantity being approximated
# (Express summary, "Problem Statement"; README layouts).
# --------------------------------------------------------------------------
def weighted_attention(q, K, V, scale, logw=None, mask=None):
    """o_t = sum_j w_j e^{s q_t.k_j} v_j / sum_j w_j e^{s q_t.k_j};  lse_t = ln sum_j w_j e^{s q_t.k_j}.

    q (T,E), K (N,E), V (N,D), logw (N,) = ln w_j, mask (T,N) bool (True = visible).
    """
    z = scale * (q @ K.T)
    if logw is not None:
        z = z + logw[None, :]
    if mask is not None:
        z = np.where(mask, z, -np.inf)
    mu = z.max(axis=1, keepdims=True)
    p = np.exp(z - mu)
    den = p.sum(axis=1, keepdims=True)
    return (p @ V) / den, (mu + np.log(den))[:, 0]


# --------------------------------------------------------------------------
# Key-value attention kernel (Thinformer Express section names kappa_att).
# --------------------------------------------------------------------------
def kappa_att(K1, V1, K2, V2, scale, c2):
    """kappa((k,v),(k',v')) = exp(s <k,k'>) (<v,v'> + c^2) for all row pairs (batched over a leading axis)."""
    return np.exp(scale * (K1 @ np.swapaxes(K2, -1, -2))) * (V1 @ np.swapaxes(V2, -1, -2) + c2)


# --------------------------------------------------------------------------
# Kernel Halving: self-balancing walk over consecutive pairs.
# --------------------------------------------------------------------------
NEAR_TIE_REL = 1e-4


@dataclasses.dataclass
class HalvingOut:
    keep_first: np.ndarray   # (I, m) bool: pair i keeps its first point
    near: np.ndarray         # (I, m) bool: |alpha - a(1-2u)| < 1e-4 * kernel scale
    mismatch: np.ndarray     # (I, m) bool: follow mode only; decided differently outside a near tie
    clipped: np.ndarray      # (I,) bool: some step had |alpha| > a (probability clipped)


def kernel_halving(K, V, scale, u, follow=None, chunk_elems=1 << 25):
    """Halve each instance of n points (n = 2m) to m points, one per consecutive pair.

    K (I,n,E), V (I,n,D) float64; u (I,m) uniforms of the pairs.
    For pair i = (x, y) = (p_{2i}, p_{2i+1}) (0-based):
      b^2   = k(x,x) + k(y,y) - 2k(x,y)
      alpha = sum_{j<i} eta_j [k(x_j,x) - k(y_j,x) - k(x_j,y) + k(y_j,y)]
      a     = max(b sigma sqrt(2 ln(2/delta_i)), b^2),  delta_i = (1/2)/m
      p+    = clip((1 - alpha/a)/2, 0, 1); eta = +1 (keep x) iff u < p+
      sigma^2 <- sigma^2 + b^2 max(0, 1 + (b^2 - 2a) sigma^2 / a^2)
    A pair with b^2 <= 0 keeps x and leaves sigma unchanged.
    ``follow`` (I,m) bool: decisions of another implementation; where this
    walk's own decision is a near tie the followed one is taken instead.
    """
    I, n, _ = K.shape
    per = max(1, chunk_elems // max(1, n * n))
    if I > per:
        parts = [kernel_halving(K[s:s + per], V[s:s + per], scale, u[s:s + per],
                                None if follow is None else follow[s:s + per], chunk_elems)
                 for s in range(0, I, per)]
        return HalvingOut(*(np.concatenate([getattr(p, f.name) for p in parts])
                            for f in dataclasses.fields(HalvingOut)))
    m = n // 2
    c2 = np.abs(V).max(axis=(1, 2)) ** 2
    G = kappa_att(K, V, K, V, scale, c2[:, None, None])          # (I,n,n)
    kscale = np.diagonal(G, axis1=1, axis2=2).max(axis=1)
    # Delta[j, i] = k(x_j,x_i) - k(y_j,x_i) - k(x_j,y_i) + k(y_j,y_i)
    Delta = G[:, 0::2, 0::2] - G[:, 1::2, 0::2] - G[:, 0::2, 1::2] + G[:, 1::2, 1::2]
    C = math.sqrt(2.0 * math.log(2.0 / (0.5 / m)))
    eta = np.zeros((I, m))
    sigma2 = np.zeros(I)
    keep = np.zeros((I, m), dtype=bool)
    near = np.zeros((I, m), dtype=bool)
    mism = np.zeros((I, m), dtype=bool)
    clipped = np.zeros(I, dtype=bool)
    for i in range(m):
        alpha = np.einsum("ij,ij->i", eta[:, :i], Delta[:, :i, i])
        b2 = Delta[:, i, i]
        tie = b2 <= 0.0
        a = np.maximum(np.sqrt(np.where(tie, 0.0, b2)) * np.sqrt(sigma2) * C, b2)
        a = np.where(tie, 1.0, a)
        ui = u[:, i]
        pplus = np.clip(0.5 * (1.0 - alpha / a), 0.0, 1.0)
        own = tie | (ui < pplus)
        margin = np.where(tie, np.inf, np.abs(alpha - a * (1.0 - 2.0 * ui)))
        nt = margin < NEAR_TIE_REL * kscale
        clipped |= ~tie & (np.abs(alpha) > a)
        if follow is not None:
            f = follow[:, i]
            mism[:, i] = ~nt & (f != own)
            dec = np.where(nt, f, own)
        else:
            dec = own
        keep[:, i] = dec
        near[:, i] = nt
        eta[:, i] = np.where(dec, 1.0, -1.0)
        sigma2 = np.where(tie, sigma2,
                          sigma2 + b2 * np.maximum(0.0, 1.0 + (b2 - 2.0 * a) * sigma2 / (a * a)))
    return HalvingOut(keep, near, mism, clipped)


# --------------------------------------------------------------------------
# KH-Compress with a systematic uniform subsample.
# --------------------------------------------------------------------------
def compress_sizes(S: int, g: int) -> Tuple[int, int, int, int]:
    """(r, L, S', |C|): r halving levels over 4^r leaves of L points, S' = L 4^r, |C| = L 2^r.

    r is the least integer with 4^(g+r) >= S, lowered (only possible when g = 0)
    until 4^r <= S so that every leaf holds at least one point.  When S = 4^(g+r)
    the coreset has exactly 2^g sqrt(S) points.
    """
    if S <= 0:
        return 0, 0, 0, 0
    r = 0
    while 4 ** (g + r) < S:
        r += 1
    while r > 0 and 4 ** r > S:
        r -= 1
    L = S // 4 ** r
    return r, L, L * 4 ** r, L * 2 ** r


def subsample_indices(S: int, S_sub: int, U: np.ndarray) -> np.ndarray:
    """Systematic subsample: idx_i = floor((i S + U) / S') for i < S', U in [0, S'); shape (I, S')."""
    i = np.arange(S_sub, dtype=np.int64)
    return (i[None, :] * S + U.astype(np.int64)[:, None]) // S_sub


Trace = Dict[Tuple[int, int], np.ndarray]


@dataclasses.dataclass
class Stats:
    near_ties: int = 0
    mismatches: int = 0
    decisions: int = 0
    clipped_instances: int = 0

    def add(self, h: HalvingOut):
        self.near_ties += int(h.near.sum())
        self.mismatches += int(h.mismatch.sum())
        self.decisions += int(h.keep_first.size)
        self.clipped_instances += int(h.clipped.sum())


def halve_level(Kall, Vall, idx, n_group, scale, seed, bh, round_ids, trace, follow, stats):
    """One halving level of every instance row of ``idx`` (I, n_cur), groups of ``n_group`` points.

    Pair p of (bh, round) is counted across the whole level: group gi, local pair i -> gi*(n_group/2)+i.
    Kall (I,S,E), Vall (I,S,D): the points the indices refer to.
    """
    I, n_cur = idx.shape
    G = n_cur // n_group
    m = n_group // 2
    rows = np.arange(I)[:, None]
    Kg = Kall[rows, idx].reshape(I * G, n_group, -1)
    Vg = Vall[rows, idx].reshape(I * G, n_group, -1)
    pair = np.arange(G * m, dtype=np.uint64)[None, :]
    u = philox_uniform(seed, bh.astype(np.uint64)[:, None], round_ids.astype(np.uint64)[:, None], pair)
    fol = None
    if follow is not None:
        fol = np.stack([follow[(int(b), int(r))] for b, r in zip(bh, round_ids)]).reshape(I * G, m)
    res = kernel_halving(Kg, Vg, scale, u.reshape(I * G, m), fol)
    stats.add(res)
    keep = res.keep_first.reshape(I, G * m)
    for t in range(I):
        trace[(int(bh[t]), int(round_ids[t]))] = keep[t].copy()
    first = idx[:, 0::2]
    second = idx[:, 1::2]
    return np.where(keep, first, second)


def kh_compress(Kall, Vall, scale, g, seed, bh, round_of_level: Callable[[int], np.ndarray],
                sub_round: np.ndarray, trace: Trace, follow: Optional[Trace], stats: Stats,
                sizes: Optional[Tuple[int, int, int]] = None):
    """KH-Compress of I independent point sets of S points each -> (I, |C|) indices into the S points.

    ``sizes`` = (r, L, S'): the tree to use instead of compress_sizes(S, g)."""
    I, S, _ = Kall.shape
    r, L, S_sub = sizes if sizes is not None else compress_sizes(S, g)[:3]
    if S_sub < S:
        U = philox_word(seed, bh.astype(np.uint64), sub_round.astype(np.uint64), 0) % np.uint64(S_sub)
        idx = subsample_indices(S, S_sub, U)
    else:
        idx = np.broadcast_to(np.arange(S, dtype=np.int64), (I, S)).copy()
    for level in range(1, r + 1):
        n_group = 4 * L * 2 ** (level - 1)
        idx = halve_level(Kall, Vall, idx, n_group, scale, seed, bh, round_of_level(level),
                          trace, follow, stats)
    return idx


def _f64(x):
    import torch
    if isinstance(x, torch.Tensor):
        return x.detach().to("cpu", dtype=torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


# --------------------------------------------------------------------------
# Thinformer (non-causal)
# --------------------------------------------------------------------------
@dataclasses.dataclass
class OracleOut:
    out: Optional[np.ndarray]      # (B,T,H,D) or rows-only (B,len(rows),H,D)
    lse: Optional[np.ndarray]      # (B,H,T) or (B,H,len(rows))
    coreset: np.ndarray            # non-causal (B,H,|C|); causal (B,H,n_nodes,c) original token indices
    trace: Trace
    stats: Stats
    weights: Optional[np.ndarray] = None   # causal: (n_nodes,) node weights


def _attn_operands(q, k, attn_q, attn_k):
    """The q and k the attention step uses: by default the inputs themselves; the e4m3 QK^T path of
    the library attends with e4m3-rounded copies (passed here, dequantised) while the thinning keeps
    the original keys."""
    return (q if attn_q is None else _f64(attn_q)), (k if attn_k is None else _f64(attn_k))


def thinformer(q, k, v, g, seed, scale=None, follow=None, rows=None, heads=None, b0=0, attn_q=None, attn_k=None):
    """Non-causal Thinformer: per (b,h), KH-Compress the S keys/values to a coreset C,
    then weighted attention of every query against C with weight S/|C| per point.

    q (B,T,H,E), k (B,S,H,E), v (B,S,H,D) (torch or numpy; read as fp64).
    ``rows``: optional query rows to evaluate (all by default). ``heads``: global
    head ids of the H axis when the tensors hold a subset, ``b0``: the whole problem's
    index of batch row 0 (Philox (b,h) word = (b0 + b)*H_total + h).  ``attn_q``, ``attn_k``:
    the query and key tensors of the attention step when they differ from q, k (same shapes).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    qa, ka = _attn_operands(q, k, attn_q, attn_k)
    B, T, H, E = q.shape
    S = k.shape[1]
    scale = 1.0 / math.sqrt(E) if scale is None else scale
    hs = np.arange(H) if heads is None else np.asarray(heads[1])
    Htot = H if heads is None else heads[0]
    bh = ((b0 + np.arange(B))[:, None] * Htot + hs[None, :]).reshape(-1)
    Kall = k.transpose(0, 2, 1, 3).reshape(B * H, S, E)
    Vall = v.transpose(0, 2, 1, 3).reshape(B * H, S, -1)
    trace: Trace = {}
    stats = Stats()
    n_bh = B * H
    cidx = kh_compress(Kall, Vall, scale, g, seed, bh,
                       lambda lv: np.full(n_bh, round_noncausal(lv), dtype=np.int64),
                       np.full(n_bh, round_subsample(0), dtype=np.int64), trace, follow, stats)
    C = cidx.shape[1]
    rsel = np.arange(T) if rows is None else np.asarray(rows)
    D = v.shape[3]
    out = np.zeros((B, len(rsel), H, D))
    lse = np.zeros((B, H, len(rsel)))
    logw = np.full(C, math.log(S / C)) if C > 0 else None
    for i in range(n_bh):
        b, h = divmod(i, H)
        Kc, Vc = ka[b, :, h][cidx[i]], Vall[i, cidx[i]]
        o, l = weighted_attention(qa[b, rsel, h], Kc, Vc, scale, logw)
        out[b, :, h], lse[b, h] = o, l
    return OracleOut(out, lse, cidx.reshape(B, H, C), trace, stats)


# --------------------------------------------------------------------------
# Thinformer Express (causal)
# --------------------------------------------------------------------------
def express_layout(T: int, n_e: int, bsz: int):
    """Batch count and node slots: level-0 nodes k < n_b, then level-1 nodes j < n_b//4, ...

    Returns (n_b, [(level, j), ...]) in slot order.  Level-l node j summarises
    batches [j 4^l, (j+1) 4^l).
    """
    n_b = (T - n_e) // bsz if T > n_e and bsz > 0 else 0
    slots = []
    lv = 0
    while n_b // 4 ** lv > 0:
        slots += [(lv, j) for j in range(n_b // 4 ** lv)]
        lv += 1
    return n_b, slots


def snapshot_nodes(k: int):
    """Nodes present after k completed batches: base-4 digit d_l of k gives d_l nodes at level l."""
    nodes = []
    lv = 0
    while 4 ** lv <= k:
        d = (k // 4 ** lv) % 4
        base = (k // 4 ** (lv + 1)) * 4
        nodes += [(lv, base + j) for j in range(d)]
        lv += 1
    return nodes


def express(q, k, v, n_e, bsz, g, seed, scale=None, follow=None, rows=None, heads=None, b0=0, attn_q=None,
            attn_k=None):
    """Thinformer Express prefill (causal).

    * tokens [0, n_e): kept exactly (weight 1) -- exact phase;
    * batch k = tokens [n_e + k b, n_e + (k+1) b), k < n_b = floor((T - n_e)/b),
      is KH-Compressed to c points of weight b/c -- thin phase;
    * whenever four nodes of level l exist they are concatenated in time order
      (4c points) and halved twice (4c -> 2c -> c) into one level-(l+1) node of
      4x the weight -- HALVE phase;
    * query t < n_e: exact causal attention; query t in batch k (k may be n_b for
      a trailing partial batch): the exact prefix, the nodes after k completed
      batches, and tokens [n_e + k b, t] of its own batch (weight 1).
    ``attn_q``, ``attn_k``: as for thinformer.
    """
    q, k_, v = _f64(q), _f64(k), _f64(v)
    qa, ka = _attn_operands(q, k_, attn_q, attn_k)
    B, T, H, E = q.shape
    D = v.shape[3]
    scale = 1.0 / math.sqrt(E) if scale is None else scale
    hs = np.arange(H) if heads is None else np.asarray(heads[1])
    Htot = H if heads is None else heads[0]
    n_bh = B * H
    bh = ((b0 + np.arange(B))[:, None] * Htot + hs[None, :]).reshape(-1)
    Kall = k_.transpose(0, 2, 1, 3).reshape(n_bh, T, E)
    Vall = v.transpose(0, 2, 1, 3).reshape(n_bh, T, D)
    Qall = qa.transpose(0, 2, 1, 3).reshape(n_bh, T, E)
    Kattn = ka.transpose(0, 2, 1, 3).reshape(n_bh, T, E)
    n_b, slots = express_layout(T, n_e, bsz)
    trace: Trace = {}
    stats = Stats()
    nodes: Dict[Tuple[int, int], np.ndarray] = {}     # (level, j) -> (n_bh, c) token indices
    c = compress_sizes(bsz, g)[3] if bsz > 0 else 0
    # thin phase: every batch compressed independently (batch k depends on its tokens only)
    if n_b:
        Kb = Kall[:, n_e:n_e + n_b * bsz].reshape(n_bh * n_b, bsz, E)
        Vb = Vall[:, n_e:n_e + n_b * bsz].reshape(n_bh * n_b, bsz, D)
        bhb = np.repeat(bh, n_b)
        kk = np.tile(np.arange(n_b), n_bh)
        loc = kh_compress(Kb, Vb, scale, g, seed, bhb,
                          lambda lv: np.array([round_batch(int(x), lv) for x in kk], dtype=np.int64),
                          np.array([round_subsample(int(x)) for x in kk], dtype=np.int64),
                          trace, follow, stats)
        tok = loc.reshape(n_bh, n_b, c) + (n_e + np.arange(n_b) * bsz)[None, :, None]
        for j in range(n_b):
            nodes[(0, j)] = tok[:, j]
    # HALVE phase: 4-ary counter, level by level (a merge needs only its four children)
    lv = 0
    while n_b // 4 ** (lv + 1) > 0:
        nj = n_b // 4 ** (lv + 1)
        for j in range(nj):
            idx = np.concatenate([nodes[(lv, 4 * j + t)] for t in range(4)], axis=1)   # (n_bh, 4c)
            for step in range(2):
                rid = np.full(n_bh, round_merge(lv + 1, j, step), dtype=np.int64)
                idx = halve_level(Kall, Vall, idx, idx.shape[1], scale, seed, bh, rid, trace, follow, stats)
            nodes[(lv + 1, j)] = idx
        lv += 1
    weight = {s: float(4 ** s[0] * bsz / c) for s in slots} if n_b else {}
    # attention
    rsel = np.arange(T) if rows is None else np.sort(np.asarray(rows))
    out = np.zeros((B, len(rsel), H, D))
    lse = np.zeros((B, H, len(rsel)))
    batch_of = np.where(rsel < n_e, -1, (rsel - n_e) // max(bsz, 1))
    if n_b == 0:
        batch_of[:] = -1
    for grp in np.unique(batch_of):
        sel = np.nonzero(batch_of == grp)[0]
        tq = rsel[sel]
        for i in range(n_bh):
            b, h = divmod(i, H)
            if grp < 0:
                hi = int(tq.max()) + 1
                key = np.arange(hi)
                logw = np.zeros(hi)
                mask = key[None, :] <= tq[:, None]
            else:
                start = n_e + int(grp) * bsz
                end = min(start + bsz, T)
                parts = [np.arange(n_e)]
                lw = [np.zeros(n_e)]
                for nd in snapshot_nodes(int(grp)):
                    parts.append(nodes[nd][i])
                    lw.append(np.full(c, math.log(weight[nd])))
                n_fixed = sum(len(p) for p in parts)
                parts.append(np.arange(start, end))
                lw.append(np.zeros(end - start))
                key = np.concatenate(parts)
                logw = np.concatenate(lw)
                mask = np.ones((len(tq), len(key)), dtype=bool)
                mask[:, n_fixed:] = np.arange(start, end)[None, :] <= tq[:, None]
            o, l = weighted_attention(Qall[i, tq], Kattn[i, key], Vall[i, key], scale, logw, mask)
            out[b, sel, h] = o
            lse[b, h, sel] = l
    coreset = (np.stack([nodes[s] for s in slots], axis=1).reshape(B, H, len(slots), c)
               if slots else np.zeros((B, H, 0, c), dtype=np.int64))
    wts = np.array([weight[s] for s in slots]) if slots else np.zeros(0)
    return OracleOut(out, lse, coreset, trace, stats, wts)


# --------------------------------------------------------------------------
# Thinformer Express, page-literal cache ("reading A").
# --------------------------------------------------------------------------
def express_a_sizes(N: int, n_out: int, g: int) -> Tuple[int, int, int]:
    """(r, L, S') thinning a batch of N points to n_out: S' = L 4^r = n_out 2^r points (a uniform
    subsample when S' < N) through r KH-Compress levels over leaves of L = n_out / 2^r points.

    2^r is the largest power of two with 2^r <= N / n_out and 2^r <= n_out / 4^g, i.e. S' never
    exceeds N nor the COMPRESS2(g) input size n_out^2 / 4^g (the leaves hold at least 4^g points).
    """
    r = 0
    while 2 ** (r + 1) * n_out <= N and 2 ** (r + 1) * 4 ** g <= n_out and n_out % 2 ** (r + 1) == 0:
        r += 1
    L = n_out // 2 ** r
    return r, L, L * 4 ** r


def express_a_layout(T: int, n_out: int):
    """Batches after the exact phase: (level i, s in 1..3, start, length), batch size 4^i n_out.

    Level 0 covers tokens [n_out, 4 n_out) (inflation 1: three batches of n_out tokens), level i
    the next 3 4^i n_out tokens; the last batch may be partial.
    """
    out, start, i = [], n_out, 0
    while start < T:
        for s in range(1, 4):
            if start >= T:
                break
            size = 4 ** i * n_out
            out.append((i, s, start, min(size, T - start)))
            start += size
        i += 1
    return out


def express_a(q, k, v, n_out, g, seed, scale=None, follow=None, rows=None, heads=None, b0=0, _plant=None,
              attn_q=None, attn_k=None):
    """Thinformer Express prefill with the page-literal cache (reading A).

    The cache holds points of one weight m, the inflation factor (m = 1 at the start):
      * exact phase: tokens [0, n_out) enter the cache with weight 1;
      * thin phase: the following tokens come in batches of m n_out; a completed batch is thinned to
        n_out points (express_a_sizes: a systematic uniform subsample to S' points, then r
        KH-Compress levels) of weight m and appended to the cache;
      * HALVE phase: when the cache holds 4 n_out points they are halved twice (4 n_out -> 2 n_out ->
        n_out, in time order) and m <- 4 m.
    With m = 1 a batch of n_out tokens is kept whole, so tokens [0, 4 n_out) are attended exactly.
    Query t in a batch of level i >= 1 attends to the cache at the start of its batch (the HALVE
    output H_i and the thinned batches of level i before its own, all of weight 4^i) and to tokens
    [batch start, t] of its own batch (weight 1).
    Philox rounds: batch number kb (0-based, level 0 included) level l -> round_batch(kb, l),
    subsample -> round_subsample(kb); HALVE H_j step t -> round_merge(j, 0, t).
    Coreset slots, in order: for i = 1, 2, ...: H_i, then the thinned batches of level i, each
    present only if a query uses it (directly or through a later HALVE).
    ``_plant`` (test hook): "weight" gives the thinned points the weight of the previous level.
    ``attn_q``, ``attn_k``: as for thinformer.
    """
    q, k_, v = _f64(q), _f64(k), _f64(v)
    qa, ka = _attn_operands(q, k_, attn_q, attn_k)
    B, T, H, E = q.shape
    D = v.shape[3]
    scale = 1.0 / math.sqrt(E) if scale is None else scale
    hs = np.arange(H) if heads is None else np.asarray(heads[1])
    Htot = H if heads is None else heads[0]
    n_bh = B * H
    bh = ((b0 + np.arange(B))[:, None] * Htot + hs[None, :]).reshape(-1)
    Kall = k_.transpose(0, 2, 1, 3).reshape(n_bh, T, E)
    Vall = v.transpose(0, 2, 1, 3).reshape(n_bh, T, D)
    Qall = qa.transpose(0, 2, 1, 3).reshape(n_bh, T, E)
    Kattn = ka.transpose(0, 2, 1, 3).reshape(n_bh, T, E)
    layout = express_a_layout(T, n_out)
    trace: Trace = {}
    stats = Stats()
    levels = sorted({b[0] for b in layout})
    # which nodes are needed: H_i for every level i >= 1 with a batch; thinned batch (i, s) if batch
    # (i, s+1) exists (its queries see it) or H_{i+1} is needed
    have = {(b[0], b[1]): b for b in layout}
    need_h = {i for i in levels if i >= 1}
    need_b = set()
    for (i, s), b in have.items():
        if i >= 1 and ((i, s + 1) in have or (i + 1) in need_h):
            need_b.add((i, s))
    nodes: Dict[Tuple[str, int, int], np.ndarray] = {}
    for kb, (i, s, start, length) in enumerate(layout):
        if (i, s) not in need_b:
            continue
        r, L, S_sub = express_a_sizes(length, n_out, g)
        Kb = Kall[:, start:start + length]
        Vb = Vall[:, start:start + length]
        loc = kh_compress(Kb, Vb, scale, g, seed, bh,
                          lambda lv: np.full(n_bh, round_batch(kb, lv), dtype=np.int64),
                          np.full(n_bh, round_subsample(kb), dtype=np.int64), trace, follow, stats,
                          sizes=(r, L, S_sub))
        nodes[("b", i, s)] = loc + start
    for i in sorted(need_h):
        if i == 1:
            idx = np.broadcast_to(np.arange(4 * n_out, dtype=np.int64), (n_bh, 4 * n_out)).copy()
        else:
            idx = np.concatenate([nodes[("h", i - 1, 0)]] + [nodes[("b", i - 1, s)] for s in (1, 2, 3)], axis=1)
        for step in range(2):
            rid = np.full(n_bh, round_merge(i, 0, step), dtype=np.int64)
            idx = halve_level(Kall, Vall, idx, idx.shape[1], scale, seed, bh, rid, trace, follow, stats)
        nodes[("h", i, 0)] = idx
    slots = []
    for i in sorted(need_h):
        slots.append(("h", i, 0))
        slots += [("b", i, s) for s in (1, 2, 3) if ("b", i, s) in nodes]
    wlev = (lambda i: 4 ** (i - 1)) if _plant == "weight" else (lambda i: 4 ** i)
    # attention
    rsel = np.arange(T) if rows is None else np.sort(np.asarray(rows))
    out = np.zeros((B, len(rsel), H, D))
    lse = np.zeros((B, H, len(rsel)))
    bat = np.full(len(rsel), -1)
    for kb, (i, s, start, length) in enumerate(layout):
        if i >= 1:
            bat[(rsel >= start) & (rsel < start + length)] = kb
    for grp in np.unique(bat):
        sel = np.nonzero(bat == grp)[0]
        tq = rsel[sel]
        for n in range(n_bh):
            b, h = divmod(n, H)
            if grp < 0:
                hi = int(tq.max()) + 1
                key = np.arange(hi)
                logw = np.zeros(hi)
                mask = key[None, :] <= tq[:, None]
            else:
                i, s, start, length = layout[grp]
                parts = [nodes[("h", i, 0)][n]] + [nodes[("b", i, s2)][n] for s2 in range(1, s)]
                n_fixed = sum(len(p) for p in parts)
                w_i = wlev(i)
                h_w = 4 ** i
                lw = [np.full(n_out, math.log(h_w))] + [np.full(n_out, math.log(w_i)) for _ in range(1, s)]
                parts.append(np.arange(start, start + length))
                lw.append(np.zeros(length))
                key = np.concatenate(parts)
                logw = np.concatenate(lw)
                mask = np.ones((len(tq), len(key)), dtype=bool)
                mask[:, n_fixed:] = np.arange(start, start + length)[None, :] <= tq[:, None]
            o, l = weighted_attention(Qall[n, tq], Kattn[n, key], Vall[n, key], scale, logw, mask)
            out[b, sel, h] = o
            lse[b, h, sel] = l
    coreset = (np.stack([nodes[sl] for sl in slots], axis=1).reshape(B, H, len(slots), n_out)
               if slots else np.zeros((B, H, 0, n_out), dtype=np.int64))
    wts = np.array([float(4 ** sl[1]) for sl in slots]) if slots else np.zeros(0)
    return OracleOut(out, lse, coreset, trace, stats, wts)


def exact_attention(q, k, v, causal=False, scale=None, rows=None):
    """Exact softmax attention (B,T,H,E) x (B,S,H,E) x (B,S,H,D) in fp64: the baseline the method approximates."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, T, H, E = q.shape
    S = k.shape[1]
    scale = 1.0 / math.sqrt(E) if scale is None else scale
    rsel = np.arange(T) if rows is None else np.asarray(rows)
    out = np.zeros((B, len(rsel), H, v.shape[3]))
    lse = np.zeros((B, H, len(rsel)))
    for b in range(B):
        for h in range(H):
            mask = (np.arange(S)[None, :] <= rsel[:, None]) if causal else None
            o, l = weighted_attention(q[b, rsel, h], k[b, :, h], v[b, :, h], scale, None, mask)
            out[b, :, h], lse[b, h] = o, l
    return out, lse
