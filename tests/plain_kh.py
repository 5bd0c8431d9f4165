"""Independent plain-loop Kernel Halving, KH-Compress and Express tree for tiny inputs (pure Python).

Written from the same definitions as the oracle but without Gram or pair-difference
matrices: alpha is evaluated as psi(x) - psi(y) with psi = sum over kept points of
kappa(p, .) minus the sum over discarded points, recomputed from the points at
every step.  Used only by the oracle pin tests.
"""
import math


def _dot(a, b):
    return sum(x * y for x, y in zip(a, b))


def plain_kernel_halving(K, V, scale, u):
    """K, V: lists of n rows; u: list of m uniforms.  Returns (keep_first list, margins, kernel scale)."""
    n = len(K)
    m = n // 2
    c2 = max(abs(x) for row in V for x in row) ** 2

    def kap(a, b):
        return math.exp(scale * _dot(K[a], K[b])) * (_dot(V[a], V[b]) + c2)

    kscale = max(kap(i, i) for i in range(n))
    kept, disc = [], []
    sigma2 = 0.0
    C = math.sqrt(2.0 * math.log(4.0 * m))       # sqrt(2 ln(2/delta_i)), delta_i = 1/(2m)
    keep, margins = [], []
    for i in range(m):
        x, y = 2 * i, 2 * i + 1

        def psi(z):
            return sum(kap(p, z) for p in kept) - sum(kap(p, z) for p in disc)

        alpha = psi(x) - psi(y)
        b2 = kap(x, x) + kap(y, y) - 2.0 * kap(x, y)
        if b2 <= 0.0:
            keep.append(True)
            margins.append(math.inf)
            kept.append(x)
            disc.append(y)
            continue
        a = max(math.sqrt(b2) * math.sqrt(sigma2) * C, b2)
        p = min(1.0, max(0.0, 0.5 * (1.0 - alpha / a)))
        kx = u[i] < p
        keep.append(kx)
        margins.append(abs(alpha - a * (1.0 - 2.0 * u[i])))
        if kx:
            kept.append(x)
            disc.append(y)
        else:
            kept.append(y)
            disc.append(x)
        sigma2 = sigma2 + b2 * max(0.0, 1.0 + (b2 - 2.0 * a) * sigma2 / (a * a))
    return keep, margins, kscale


# ---------------------------------------------------------------------------------------------
# Independent plain-loop KH-Compress and Express node tree (pure Python ints and floats).
#
# Written from the definitions, not from the oracle's level-by-level arrays: Philox4x32-10 on
# Python integers (Salmon, Moraes, Dror & Shaw, SC'11), the systematic subsample, and COMPRESS as
# the recursion of Shetty, Dwivedi & Mackey ("Distribution Compression in Near-linear Time"):
# a node splits its points into four contiguous quarters, compresses each, concatenates the four
# results in order and halves the concatenation.  The Philox pair counter of a halving is the
# node's position among the nodes of its depth times its pair count, plus the local pair index,
# so the nodes of one (b,h) and round draw distinct numbers.
# ---------------------------------------------------------------------------------------------
_M32 = 0xFFFFFFFF


def plain_philox_x0(seed, c0, c1, c2, c3=0):
    """First output word of Philox4x32-10 at counter (c0, c1, c2, c3), key (seed low, seed high)."""
    k0, k1 = seed & _M32, (seed >> 32) & _M32
    x = [c0 & _M32, c1 & _M32, c2 & _M32, c3 & _M32]
    for _ in range(10):
        hi_a, lo_a = divmod(0xD2511F53 * x[0], 1 << 32)
        hi_b, lo_b = divmod(0xCD9E8D57 * x[2], 1 << 32)
        x = [hi_b ^ x[1] ^ k0, lo_b, hi_a ^ x[3] ^ k1, lo_a]
        k0 = (k0 + 0x9E3779B9) & _M32
        k1 = (k1 + 0xBB67AE85) & _M32
    return x[0]


def plain_uniform(seed, bh, round_id, pair):
    """The uniform of a pair: the top 23 bits of the first Philox word, centred in its cell."""
    return ((plain_philox_x0(seed, pair, round_id, bh) >> 9) + 0.5) / float(1 << 23)


def plain_tree_sizes(S, g):
    """Levels r (least with 4^(g+r) >= S, lowered until 4^r <= S) and leaf size L = floor(S / 4^r)."""
    r = 0
    while 4 ** (g + r) < S:
        r += 1
    while r > 0 and 4 ** r > S:
        r -= 1
    return r, S // 4 ** r


def plain_compress(K, V, scale, g, seed, bh, level_round, sub_round, trace=None):
    """KH-Compress of the point list (K[i], V[i]), i < S: returns the coreset's point indices.

    ``level_round(l)`` is the Philox round id of tree depth l (leaves are depth 0);
    ``trace`` (dict) receives {(bh, round id): {node position: [keep-first flags]}}.
    """
    S = len(K)
    r, L = plain_tree_sizes(S, g)
    n_sub = L * 4 ** r
    if n_sub < S:
        U = plain_philox_x0(seed, 0, sub_round, bh) % n_sub
        pts = [(i * S + U) // n_sub for i in range(n_sub)]
    else:
        pts = list(range(S))

    def node(start, length, depth):
        if depth == 0:
            return pts[start:start + length]
        quarter = length // 4
        kids = []
        for c in range(4):
            kids += node(start + c * quarter, quarter, depth - 1)
        m = len(kids) // 2
        pos = start // length
        rid = level_round(depth)
        u = [plain_uniform(seed, bh, rid, pos * m + i) for i in range(m)]
        keep, _, _ = plain_kernel_halving([K[p] for p in kids], [V[p] for p in kids], scale, u)
        if trace is not None:
            trace.setdefault((bh, rid), {})[pos] = keep
        return [kids[2 * i] if keep[i] else kids[2 * i + 1] for i in range(m)]

    return node(0, n_sub, r)


def plain_express_nodes(K, V, scale, n_e, bsz, g, seed, bh, trace=None):
    """Coresets of the Express prefill of one (b,h): {(level, j): token indices}.

    Batch k (tokens n_e + k bsz .. n_e + (k+1) bsz - 1, complete batches only) is compressed with
    round ids 0x40000000 | k << 4 | depth and subsample round 0xC0000000 | k; four level-l nodes
    4j .. 4j+3, concatenated oldest first, are halved twice (round 0x80000000 | (l+1) << 24 | j << 1
    | step, pairs counted from 0 in each halving) into node (l+1, j).
    """
    T = len(K)
    n_b = (T - n_e) // bsz if T > n_e and bsz > 0 else 0
    nodes = {}
    for kb in range(n_b):
        lo = n_e + kb * bsz
        loc = plain_compress(K[lo:lo + bsz], V[lo:lo + bsz], scale, g, seed, bh,
                             lambda d, kb=kb: 0x40000000 | (kb << 4) | d, 0xC0000000 | kb, trace)
        nodes[(0, kb)] = [lo + p for p in loc]
    lv = 0
    while n_b // 4 ** (lv + 1) > 0:
        for j in range(n_b // 4 ** (lv + 1)):
            pts = []
            for t in range(4):
                pts += nodes[(lv, 4 * j + t)]
            for step in range(2):
                rid = 0x80000000 | ((lv + 1) << 24) | (j << 1) | step
                m = len(pts) // 2
                u = [plain_uniform(seed, bh, rid, i) for i in range(m)]
                keep, _, _ = plain_kernel_halving([K[p] for p in pts], [V[p] for p in pts], scale, u)
                if trace is not None:
                    trace.setdefault((bh, rid), {})[0] = keep
                pts = [pts[2 * i] if keep[i] else pts[2 * i + 1] for i in range(m)]
            nodes[(lv + 1, j)] = pts
        lv += 1
    return nodes
