"""Pins for the float64 oracle: facts the pages and plain mathematics fix,
computed here by routes that do not share the oracle's arithmetic.

Each test names what pins it.  A plausible slip in the oracle (a dropped
1/n, a transposed operand, a wrong region/token index, a missing scale, a
wrong tie-break, a softmax over the wrong set) fails at least one of them.
"""
import itertools
import math

import numpy as np
import pytest

import bra_inputs as bi
import oracle

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def fmap(B, H, W, C, S, seed, stream):
    """float64 region-correlated map (the workloads' recipe, no rounding)."""
    return bi.feature_map(bi.BraShape(B, H, W, C, 1, S, 1, "f32"), seed, stream)


def qkv(B, H, W, C, S, seed):
    return [fmap(B, H, W, C, S, seed, s) for s in range(3)]


def region_indicator(H, W, S):
    """[R, HW] matrix with 1/n where token u lies in region r."""
    reg = bi.region_map(H, W, S).reshape(-1)
    R, n = S * S, (H // S) * (W // S)
    P = np.zeros((R, H * W))
    P[reg, np.arange(H * W)] = 1.0 / n
    return P


def heads_view(x, heads):
    """[B,H,W,C] -> [B, heads, HW, d]."""
    B, H, W, C = x.shape
    return x.reshape(B, H * W, heads, C // heads).transpose(0, 2, 1, 3)


def dense_attention(q, k, v, heads, mask=None):
    """Textbook softmax(Q K^T / sqrt(d)) V per head over all HW tokens,
    optionally with a boolean [B, heads, HW, HW] mask of allowed pairs."""
    B, H, W, C = q.shape
    d = C // heads
    Q, K, V = heads_view(q, heads), heads_view(k, heads), heads_view(v, heads)
    s = Q @ K.transpose(0, 1, 3, 2) / math.sqrt(d)
    if mask is not None:
        s = np.where(mask, s, -np.inf)
    s = s - s.max(axis=-1, keepdims=True)
    p = np.exp(s)
    p /= p.sum(axis=-1, keepdims=True)
    o = p @ V  # [B, heads, HW, d]
    return o.transpose(0, 2, 1, 3).reshape(B, H, W, C)


# ---------------------------------------------------------------- pooling --

def test_region_pool_is_block_mean():
    """Q^r is the mean of the region's tokens (blog Part 2 section 2.2, step 3):
    computed here by reshaping the map into (S, H/S, S, W/S) blocks."""
    B, H, W, C, heads, S = 2, 12, 8, 6, 3, 4
    x = fmap(B, H, W, C, S, 7, 0)
    got = oracle.region_pool(x, heads, S)
    blocks = x.reshape(B, S, H // S, S, W // S, C).mean(axis=(2, 4))  # [B, S, S, C]
    want = blocks.reshape(B, S * S, heads, C // heads).transpose(0, 2, 1, 3)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-13)


def test_affinity_equals_average_token_affinity():
    """Affinity of the region means equals the mean of all token-pair
    affinities between the two regions (paperlayer summary, section 6: the
    region-average affinity identity).  Computed as P (Q K^T) P^T."""
    B, H, W, C, heads, S = 2, 8, 12, 8, 2, 4
    q, k, _ = qkv(B, H, W, C, S, 11)
    qr, kr = oracle.region_pool(q, heads, S), oracle.region_pool(k, heads, S)
    a = oracle.region_affinity(qr, kr)
    P = region_indicator(H, W, S)
    Q, K = heads_view(q, heads), heads_view(k, heads)
    want = P @ (Q @ K.transpose(0, 1, 3, 2)) @ P.T
    np.testing.assert_allclose(a, want, rtol=1e-12, atol=1e-12)


def test_affinity_is_not_scaled_and_not_transposed():
    """A^r[r, s] = <Q^r[r], K^r[s]> with no scale: a hand example where
    every entry is a distinct integer, so a transpose or a scale shows."""
    qr = np.array([[[[1.0, 0.0], [0.0, 2.0], [3.0, 1.0]]]])
    kr = np.array([[[[1.0, 1.0], [2.0, 0.0], [0.0, 5.0]]]])
    a = oracle.region_affinity(qr, kr)
    want = np.array([[1, 2, 0], [2, 0, 10], [4, 6, 5]], dtype=float)
    np.testing.assert_array_equal(a[0, 0], want)


# ---------------------------------------------------------------- routing --

def brute_force_route(row, k):
    """Enumerate every k-subset; keep the one whose members all precede all
    non-members under (value descending, index ascending); order it the same way."""
    R = len(row)

    def before(i, j):
        return row[i] > row[j] or (row[i] == row[j] and i < j)

    winners = []
    for T in itertools.combinations(range(R), k):
        rest = [j for j in range(R) if j not in T]
        if all(before(i, j) for i in T for j in rest):
            winners.append(T)
    assert len(winners) == 1
    T = list(winners[0])
    for a in range(len(T)):  # selection sort with the same relation
        for b in range(a + 1, len(T)):
            if before(T[b], T[a]):
                T[a], T[b] = T[b], T[a]
    return T


@pytest.mark.parametrize("R", [1, 3, 4, 7, 9])
@pytest.mark.parametrize("ties", [False, True])
def test_topk_matches_subset_enumeration(R, ties):
    """Row-wise top-k (blog section 2.2 step 3) against enumeration of all
    C(R, k) subsets; with ``ties`` the affinities take 3 values only, so the
    lower-index rule decides most of the choice."""
    rng = np.random.default_rng(R * 10 + ties)
    a = rng.integers(0, 3, size=(2, 1, R, R)).astype(float) if ties \
        else rng.standard_normal((2, 1, R, R))
    for k in range(1, R + 1):
        idx = oracle.topk_routing(a, k)
        for b in range(2):
            for r in range(R):
                assert list(idx[b, 0, r]) == brute_force_route(list(a[b, 0, r]), k)


def test_topk_all_zero_affinity_takes_lowest_indices():
    """Q = 0 makes every affinity 0; the tie rule then routes every region to
    regions 0..k-1 in that order."""
    B, H, W, C, heads, S, k = 1, 8, 8, 4, 2, 4, 3
    _, kk, v = qkv(B, H, W, C, S, 3)
    _, idx = oracle.bra_forward(np.zeros_like(kk), kk, v, heads, S, k)
    assert (idx == np.arange(k)).all()


def test_topk_duplicate_region_lower_index_first():
    """Two regions with identical keys tie exactly; the lower index must be
    listed first and both are taken when k = 2."""
    B, H, W, C, S = 1, 8, 8, 2, 4
    q, k, v = qkv(B, H, W, C, S, 5)
    n = 2
    # make region 9's tokens a copy of region 2's, and make them the best match
    big = np.array([40.0, 40.0])
    k[:, 0:2, 4:6, :] = big          # region 2 = rows 0-1, cols 4-5
    k[:, 4:6, 2:4, :] = big          # region 9 = rows 4-5, cols 2-3
    q[...] = np.abs(q) + 1.0         # all region means positive
    _, idx = oracle.bra_forward(q, k, v, 1, S, 2)
    assert (idx[0, 0, :, 0] == 2).all() and (idx[0, 0, :, 1] == 9).all()
    del n


# -------------------------------------------------------------- attention --

@pytest.mark.parametrize("heads", [1, 2])
def test_full_topk_is_dense_attention(heads):
    """topk = S^2 routes every region to every region, so the method is full
    attention (blog Part 4 section 4.3: the last stage's k = S^2 "defaults to
    full attention")."""
    B, H, W, C, S = 2, 8, 8, 8, 4
    q, k, v = qkv(B, H, W, C, S, 21)
    o, idx = oracle.bra_forward(q, k, v, heads, S, S * S)
    np.testing.assert_allclose(o, dense_attention(q, k, v, heads), rtol=0, atol=1e-12)
    assert (np.sort(idx, axis=-1) == np.arange(S * S)).all()


def test_single_region_is_dense_attention():
    """S = 1: one region, the only route is itself; full attention again."""
    B, H, W, C, heads = 2, 6, 10, 8, 2
    q, k, v = qkv(B, H, W, C, 1, 22)
    o, idx = oracle.bra_forward(q, k, v, heads, 1, 1)
    np.testing.assert_allclose(o, dense_attention(q, k, v, heads), rtol=0, atol=1e-12)
    assert (idx == 0).all()


@pytest.mark.parametrize("cfg", [(2, 8, 8, 8, 2, 4, 1), (1, 12, 8, 6, 3, 4, 3),
                                 (2, 8, 8, 4, 1, 2, 2)])
def test_gather_equals_region_masked_dense(cfg):
    """Second formulation of the token step (blog section 2.2 step 4): dense
    scores over all tokens with a mask that keeps key u for query t iff
    region(u) is routed from region(t).  Same routing, independent gather."""
    B, H, W, C, heads, S, k = cfg
    q, kk, v = qkv(B, H, W, C, S, 30 + k)
    o, idx = oracle.bra_forward(q, kk, v, heads, S, k)
    reg = bi.region_map(H, W, S).reshape(-1)
    routed = np.zeros((B, heads, S * S, S * S), dtype=bool)
    for m in range(k):
        np.put_along_axis(routed, idx[..., m:m + 1].astype(np.int64), True, axis=-1)
    mask = routed[:, :, reg][:, :, :, reg]  # [B, heads, HW(query), HW(key)]
    np.testing.assert_allclose(o, dense_attention(q, kk, v, heads, mask), rtol=0, atol=1e-12)


@pytest.mark.parametrize("heads", [1, 2])
def test_repeated_routes_attend_the_union(heads):
    """A caller-given routing may list a region more than once; the query
    attends over the union of its routed tokens (each token once), which is
    the region-masked dense formulation with the mask built from the set of
    listed regions."""
    B, H, W, C, S, k = 1, 8, 8, 8, 4, 3
    q, kk, v = qkv(B, H, W, C, S, 35 + heads)
    rng = np.random.default_rng(heads)
    idx = rng.integers(0, S * S, size=(B, heads, S * S, k)).astype(np.int32)
    idx[0, 0, :4] = [[2, 2, 2], [5, 1, 5], [0, 0, 7], [9, 3, 3]]
    o = oracle.token_attention(q, kk, v, idx, heads, S)
    reg = bi.region_map(H, W, S).reshape(-1)
    routed = np.zeros((B, heads, S * S, S * S), dtype=bool)
    for m in range(k):
        np.put_along_axis(routed, idx[..., m:m + 1].astype(np.int64), True, axis=-1)
    mask = routed[:, :, reg][:, :, :, reg]
    np.testing.assert_allclose(o, dense_attention(q, kk, v, heads, mask), rtol=0, atol=1e-12)
    # a region listed three times gives what the same region listed once gives
    once = np.ascontiguousarray(idx[..., :1])  # row 0 of head 0 is [2]
    o1 = oracle.token_attention(q, kk, v, once, heads, S)
    d = C // heads
    in_region0 = (reg == 0).reshape(H, W)
    assert np.array_equal(o[0][in_region0][:, :d], o1[0][in_region0][:, :d])


def test_constant_values_give_constant_output():
    """softmax weights sum to one: V = c everywhere gives O = c."""
    B, H, W, C, heads, S, k = 1, 8, 8, 8, 2, 4, 2
    q, kk, _ = qkv(B, H, W, C, S, 40)
    c = np.linspace(-2, 3, C)
    v = np.broadcast_to(c, q.shape).copy()
    o, _ = oracle.bra_forward(q, kk, v, heads, S, k)
    np.testing.assert_allclose(o, v, rtol=0, atol=1e-13)


def test_zero_query_averages_routed_values():
    """Q = 0: all logits are equal, so each output is the plain mean of the
    values of the routed tokens; routing is regions 0..k-1 (tie rule)."""
    B, H, W, C, heads, S, k = 1, 8, 8, 4, 1, 4, 2
    _, kk, v = qkv(B, H, W, C, S, 41)
    o, _ = oracle.bra_forward(np.zeros_like(v), kk, v, heads, S, k)
    reg = bi.region_map(H, W, S)
    want = v[0][(reg == 0) | (reg == 1)].mean(axis=0)
    np.testing.assert_allclose(o[0].reshape(-1, C), np.broadcast_to(want, (H * W, C)), atol=1e-13)


def test_identical_keys_give_uniform_weights():
    """All keys equal: every logit equal again, so O is the routed V mean
    whatever Q is."""
    B, H, W, C, heads, S, k = 1, 8, 8, 4, 1, 4, 3
    q, _, v = qkv(B, H, W, C, S, 42)
    kk = np.ones_like(q)
    o, idx = oracle.bra_forward(q, kk, v, heads, S, k)
    reg = bi.region_map(H, W, S).reshape(-1)
    vf = v[0].reshape(-1, C)
    for t in range(H * W):
        want = vf[np.isin(reg, idx[0, 0, reg[t]])].mean(axis=0)
        np.testing.assert_allclose(o[0].reshape(-1, C)[t], want, atol=1e-13)


def test_worked_example_by_hand():
    """A 2x2 map with S = 2 (four one-token regions), C = d = 2, topk = 2,
    solved by hand.  Region means are the tokens themselves, so
      A = q k^T = [[2,0,1,0],[0,2,0,0],[2,2,1,0],[-2,0,-1,0]]
    and the routes (ties to the lower index) are
      r0 -> [0,2], r1 -> [1,0], r2 -> [0,1], r3 -> [1,3].
    Each output is the two-term softmax blend
      o = v_a * sigma(x) + v_b * (1 - sigma(x)),  x = (s_a - s_b) / sqrt(2)."""
    q = np.array([[1, 0], [0, 1], [1, 1], [-1, 0]], dtype=float).reshape(1, 2, 2, 2)
    k = np.array([[2, 0], [0, 2], [1, 0], [0, 0]], dtype=float).reshape(1, 2, 2, 2)
    v = np.array([[1, 0], [0, 1], [3, 3], [-1, 2]], dtype=float).reshape(1, 2, 2, 2)
    o, idx = oracle.bra_forward(q, k, v, 1, 2, 2)
    assert idx[0, 0].tolist() == [[0, 2], [1, 0], [0, 1], [1, 3]]
    sig = lambda x: 1.0 / (1.0 + math.exp(-x))
    r2 = math.sqrt(2.0)
    vv = v.reshape(4, 2)
    want = np.array([
        vv[0] * sig((2 - 1) / r2) + vv[2] * (1 - sig((2 - 1) / r2)),   # token 0: s = (2, 1)
        vv[1] * sig((2 - 0) / r2) + vv[0] * (1 - sig((2 - 0) / r2)),   # token 1: s = (2, 0)
        vv[0] * sig((2 - 2) / r2) + vv[1] * (1 - sig((2 - 2) / r2)),   # token 2: s = (2, 2)
        vv[1] * sig((0 - 0) / r2) + vv[3] * (1 - sig((0 - 0) / r2)),   # token 3: s = (0, 0)
    ])
    np.testing.assert_allclose(o.reshape(4, 2), want, rtol=0, atol=1e-14)


# ------------------------------------------------------------ equivariance --

def move_regions(x, S, perm):
    """Place region r's block at region perm[r] (blocks keep their inner order)."""
    B, H, W, C = x.shape
    hs, ws = H // S, W // S
    out = np.empty_like(x)
    for r in range(S * S):
        i, j = divmod(r, S)
        pi, pj = divmod(perm[r], S)
        out[:, pi * hs:(pi + 1) * hs, pj * ws:(pj + 1) * ws] = x[:, i * hs:(i + 1) * hs, j * ws:(j + 1) * ws]
    return out


def test_region_permutation_equivariance():
    """Moving whole regions around moves the outputs the same way and relabels
    the routes (away from affinity ties)."""
    B, H, W, C, heads, S, k = 2, 8, 12, 8, 2, 4, 3
    q, kk, v = qkv(B, H, W, C, S, 50)
    perm = np.random.default_rng(0).permutation(S * S)
    o, idx, a = oracle.bra_forward(q, kk, v, heads, S, k, want_affinity=True)
    o2, idx2 = oracle.bra_forward(*(move_regions(t, S, perm) for t in (q, kk, v)), heads, S, k)
    np.testing.assert_allclose(o2, move_regions(o, S, perm), rtol=0, atol=1e-12)
    srt = -np.sort(-a, axis=-1)
    for b in range(B):
        for h in range(heads):
            for r in range(S * S):
                if abs(srt[b, h, r, k - 1] - srt[b, h, r, k]) > 1e-9:
                    assert set(perm[idx[b, h, r]]) == set(idx2[b, h, perm[r]])


def test_token_permutation_inside_regions():
    """Shuffling tokens inside each region jointly in K and V leaves O alone;
    shuffling Q tokens inside a region shuffles O the same way."""
    B, H, W, C, heads, S, k = 1, 8, 8, 4, 2, 2, 2
    q, kk, v = qkv(B, H, W, C, S, 60)
    o, idx = oracle.bra_forward(q, kk, v, heads, S, k)
    hs = H // S
    rng = np.random.default_rng(1)
    k2, v2, q2, o_perm = kk.copy(), v.copy(), q.copy(), o.copy()
    for i in range(S):
        for j in range(S):
            sl = (slice(None), slice(i * hs, (i + 1) * hs), slice(j * hs, (j + 1) * hs))
            blk = rng.permutation(hs * hs)
            for src, dst in ((kk, k2), (v, v2)):
                dst[sl] = src[sl].reshape(B, hs * hs, C)[:, blk].reshape(B, hs, hs, C)
            blq = rng.permutation(hs * hs)
            q2[sl] = q[sl].reshape(B, hs * hs, C)[:, blq].reshape(B, hs, hs, C)
            o_perm[sl] = o[sl].reshape(B, hs * hs, C)[:, blq].reshape(B, hs, hs, C)
    o_kv, idx_kv = oracle.bra_forward(q, k2, v2, heads, S, k)
    assert (idx_kv == idx).all()
    np.testing.assert_allclose(o_kv, o, rtol=0, atol=1e-12)
    o_q, _ = oracle.bra_forward(q2, kk, v, heads, S, k)
    np.testing.assert_allclose(o_q, o_perm, rtol=0, atol=1e-12)


# ------------------------------------------------------------- brute force --

def brute_force_bra(q, k, v, heads, S, topk):
    """Everything in plain Python loops with math.exp, straight from the
    definition, for inputs of a few dozen numbers."""
    B, H, W, C = q.shape
    d, hs, ws = C // heads, H // S, W // S
    toks = lambda r: [((r // S) * hs + t // ws, (r % S) * ws + t % ws) for t in range(hs * ws)]
    o = np.zeros_like(q)
    routes = np.zeros((B, heads, S * S, topk), dtype=int)
    for b in range(B):
        for h in range(heads):
            ch = range(h * d, (h + 1) * d)
            mean = lambda x, r: [sum(x[b, y, xx, c] for y, xx in toks(r)) / (hs * ws) for c in ch]
            qm = [mean(q, r) for r in range(S * S)]
            km = [mean(k, r) for r in range(S * S)]
            for r in range(S * S):
                aff = [sum(qm[r][c] * km[s][c] for c in range(d)) for s in range(S * S)]
                order = sorted(range(S * S), key=lambda s: (-aff[s], s))[:topk]
                routes[b, h, r] = order
                keys = [p for s in order for p in toks(s)]
                for (y, x) in toks(r):
                    logits = [sum(q[b, y, x, c] * k[b, yy, xx, c] for c in ch) / math.sqrt(d)
                              for (yy, xx) in keys]
                    mx = max(logits)
                    w = [math.exp(s - mx) for s in logits]
                    for c in ch:
                        o[b, y, x, c] = sum(wi * v[b, yy, xx, c] for wi, (yy, xx) in zip(w, keys)) / sum(w)
    return o, routes


@pytest.mark.parametrize("heads", [1, 2])
@pytest.mark.parametrize("topk", [1, 2, 3, 4])
def test_brute_force_tiny(heads, topk):
    B, H, W, C, S = 1, 4, 4, 4, 2
    q, k, v = qkv(B, H, W, C, S, 70 + topk)
    o, idx = oracle.bra_forward(q, k, v, heads, S, topk)
    o_bf, idx_bf = brute_force_bra(q, k, v, heads, S, topk)
    assert (idx == idx_bf).all()
    np.testing.assert_allclose(o, o_bf, rtol=0, atol=1e-12)


# ----------------------------------------------------------------- errors --

@pytest.mark.parametrize("bad", [dict(S=3), dict(topk=0), dict(topk=17), dict(heads=3)])
def test_oracle_rejects_bad_shapes(bad):
    """S must divide the map (blog Part 3: S is a clean divisor, no padding),
    1 <= topk <= S^2, heads must divide C."""
    args = dict(heads=2, S=4, topk=2)
    args.update(bad)
    q = np.zeros((1, 8, 8, 8))
    with pytest.raises(ValueError):
        oracle.bra_forward(q, q, q, args["heads"], args["S"], args["topk"])


@pytest.mark.parametrize("bad", [np.nan, np.inf, -np.inf])
def test_non_finite_inputs_are_rejected(bad):
    # Non-finite maps are outside the contract: the oracle refuses them instead
    # of returning a result no reading of the pages defines.
    q = np.random.default_rng(0).standard_normal((1, 4, 4, 4))
    q[0, 1, 2, 3] = bad
    with pytest.raises(ValueError):
        oracle.region_pool(q, 1, 2)
    with pytest.raises(ValueError):
        oracle.qkv_projection(q, np.eye(4).repeat(3, axis=0))
