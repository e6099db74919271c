"""The facts the GPU selection's shortcuts rest on, checked on the CPU by brute force.

The kernels (select_fast.cuh, select_group.cuh, select.cuh) take the product-key route of
"Sparse Delta Memory: Scaling the State of Linear RNNs through Sparsity" (paper.rainbus.top
summary, method step 1; ai-paper-analysis.pages.dev SDM write-up, 步骤 1) with three
shortcuts of their own.  Each is a claim about any input, tested here on random and
tie-heavy rows against the top-K of all S1*S2 outer sums:

- rank-pair pruning: only the pairs of half ranks with (r1+1)(r2+1) <= K can reach the top K,
  and there are sum_{r=1..K} floor(K/r) of them (280 for K = 64);
- candidate bracket: A[K-1] + B[0] and A[0] + B[K-1] are at most the K-th largest candidate
  sum, and A[0] + B[0] is the largest;
- per-lane bracket: when n lanes each keep their P = ceil(K/n) largest keys, the smallest of
  the lanes' P-th largest keys is at most the K-th largest key.

Sums are fp32, as the method's scores are.  The rows of the first tests keep every fp32 sum
exact (bf16 halves with nonzero exponents less than 16 apart).  When a sum rounds, the pruning
alone can miss a tie: a pair outside the pruned set whose sum rounds onto the K-th largest sum
T may have a lower slot index than the tie the pruned set kept.  The kernels therefore check
for that case and repair the ties at T over all K*K candidate pairs; `repaired_topk` below is
that procedure, tested against the route on rows built to make sums collide.
"""

import json
import os

import numpy as np
import pytest


def order(scores, idx):
    """Positions of (score descending, index ascending); -0 and +0 compare equal."""
    s = np.asarray(scores, np.float64) + 0.0
    return np.lexsort((idx, -s))


def to_bf16(x):
    """Round float32 values to the nearest bf16 (ties to even), returned as float32."""
    u = np.asarray(x, np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32)


def half_sorted(h):
    o = order(h, np.arange(h.size))
    return h[o], o


def brute_topk(a, b, K):
    s = np.add.outer(a, b).astype(np.float32).ravel()
    flat = np.arange(s.size)
    o = order(s, flat)[:K]
    return flat[o], s[o]


def pruned_topk(a, b, K):
    """Top-K over the rank pairs (r1+1)(r2+1) <= K of the sorted halves only."""
    A, ia = half_sorted(a)
    B, ib = half_sorted(b)
    r1, r2 = np.meshgrid(np.arange(min(K, a.size)), np.arange(min(K, b.size)), indexing="ij")
    keep = (r1 + 1) * (r2 + 1) <= K
    r1, r2 = r1[keep], r2[keep]
    s = (A[r1] + B[r2]).astype(np.float32)
    flat = ia[r1].astype(np.int64) * b.size + ib[r2]
    o = order(s, flat)[:K]
    return flat[o], s[o], s


def rows(rng, S1, S2, kind):
    if kind == "normal":
        x = rng.standard_normal(S1 + S2)
    elif kind == "palette":
        x = rng.choice(np.array([-1.0, -0.0, 0.0, 0.5, 1.0, 1.0, 2.0, 0.25]), S1 + S2)
    elif kind == "skewed":  # the long-prefill bias that makes low indices hot
        j = np.concatenate([np.arange(S1), np.arange(S2)])
        x = rng.standard_normal(S1 + S2) - 0.5 * np.log1p(j)
    elif kind == "hyperbola":  # sums order as -(r1+1)(r2+1): the top K hug the pruning edge
        x = -np.log2(np.concatenate([rng.permutation(S1), rng.permutation(S2)]) + 1.0)
        x = x + 1e-3 * rng.standard_normal(S1 + S2)
    else:  # "dominant1" / "dominant2": one half's best value dwarfs the rest, so the top K
        # is that value plus the other half's K best (ranks up to K - 1 on one side)
        x = 0.01 * rng.standard_normal(S1 + S2)
        x[rng.integers(0, S1) if kind == "dominant1" else S1 + rng.integers(0, S2)] = 6.0
    # magnitudes in [2^-12, 8] or zero: every exponent within 16 of every other, so every
    # fp32 sum of two of these bf16 values is exact
    x = np.where(np.abs(x) < 2.0 ** -12, 0.0, np.clip(x, -8.0, 8.0))
    x = to_bf16(x.astype(np.float32))
    return x[:S1], x[S1:]


def route_topk(a, b, K):
    """The product-key route as the method states it: the top K of each half, then the top K
    of all K*K candidate sums (fp32), in (score descending, index ascending) order."""
    A, ia = half_sorted(a)
    B, ib = half_sorted(b)
    A, ia, B, ib = A[:K], ia[:K], B[:K], ib[:K]
    s = np.add.outer(A, B).astype(np.float32).ravel()
    flat = (ia.astype(np.int64)[:, None] * b.size + ib[None, :]).ravel()
    o = order(s, flat)[:K]
    return flat[o], s[o]


def bf16_sums_exact(A, B):
    """True when every fp32 sum of a value of A and a value of B (bf16 values) is exact: the
    nonzero values' exponent fields (subnormals counted as 1) span at most 15 and stay below
    254, so a sum needs at most 24 significant bits and cannot overflow."""
    v = np.concatenate([A, B]).astype(np.float32)
    e = (v.view(np.uint32) >> 23) & 0xFF
    e = np.maximum(e[v != 0], 1)
    return e.size == 0 or (int(e.max()) - int(e.min()) <= 15 and int(e.max()) < 254)


def repaired_topk(a, b, K, bf16=False):
    """The kernels' selection: the rank-pair pruned top K, then, unless every sum is exact,
    a check of the first pruned-away pair of every rank row; if one of them sums to the K-th
    largest sum T, the ties at T are refilled from all K*K pairs, lowest slot index first.

    Returns (slots, sums, repaired)."""
    A, ia = half_sorted(a)
    B, ib = half_sorted(b)
    A, ia, B, ib = A[:K], ia[:K], B[:K], ib[:K]
    got_idx, got_s, _ = pruned_topk(a, b, K)
    T = got_s[K - 1]
    if bf16 and bf16_sums_exact(A, B):
        return got_idx, got_s, False
    hit = False
    for r1 in range(1, K):
        c0 = K // (r1 + 1)  # the first column the pruning drops in rank row r1
        if c0 < K and np.float32(A[r1] + B[c0]) == T:
            hit = True
    if not hit:
        return got_idx, got_s, False
    ngt = int(np.sum(got_s > T))
    ties = []
    for r1 in range(K):
        row = (A[r1] + B).astype(np.float32)  # weakly decreasing along the row
        cs = int(np.sum(row > T))             # first column at or below T
        ce = int(np.sum(row >= T))            # first column below T
        ties.extend(int(ia[r1]) * b.size + int(ib[c]) for c in range(cs, ce))
    ties = sorted(ties)[: K - ngt]
    idx = np.concatenate([got_idx[:ngt], np.array(ties, np.int64)])
    s = np.concatenate([got_s[:ngt], np.full(K - ngt, T, np.float32)])
    return idx, s, True


def collision_rows(rng, S1, S2, K, kind, bf16):
    """Rows whose candidate sums round onto one another.

    One half ("big") draws from a small palette, so its top K repeats a few values; the
    other ("small") has K + 3 chosen values above a negative floor:
    absorb1 / absorb2: the chosen values are tiny (2^-30 .. 2^-24) and vanish in every sum
      (absorb2 puts them in the second half);
    mixed: about a third of the chosen values are of order one, the rest tiny;
    near: the chosen values are distinct in [1, 2) and the big half sits near 2^17, where
      the fp32 spacing (2^-6) merges several of them."""
    small_first = kind != "absorb2"
    n_s = S1 if small_first else S2
    n_b = S1 + S2 - n_s
    if kind == "near":
        big = 2.0 ** 17 * rng.choice([1.0, 1.0, 1.0, 1.0 + 2.0 ** -7, 0.5], n_b)
    else:
        big = rng.choice([2.0, 2.0, 1.5, 1.0, 0.5, -1.0], n_b)
    small = -rng.uniform(1.0, 3.0, n_s)
    pos = rng.choice(n_s, min(n_s, K + 3), replace=False)
    tiny = 2.0 ** rng.uniform(-30, -24, pos.size)
    if kind in ("absorb1", "absorb2"):
        small[pos] = tiny
    elif kind == "mixed":
        small[pos] = np.where(rng.random(pos.size) < 0.3, rng.uniform(0.5, 1.5, pos.size), tiny)
    else:
        step = 2.0 ** -7 if bf16 else 2.0 ** -12
        pop = min(int(1 / step), 2 * pos.size)  # dense enough to collide
        small[pos] = 1.0 + step * rng.choice(pop, pos.size, replace=pos.size > pop)
    x = np.concatenate([small, big] if small_first else [big, small]).astype(np.float32)
    if bf16:
        x = to_bf16(x)
    return x[:S1].copy(), x[S1:].copy()


COLLISION_KINDS = ["absorb1", "absorb2", "mixed", "near"]


def test_pruning_alone_misses_a_rounded_tie():
    """a = [1e-8, 2e-8], b = [1, 1], K = 2: every sum rounds to 1.0f, so the top 2 are the
    two lowest slot indices, 0 and 1.  The rank pairs (r1+1)(r2+1) <= 2 are (0,0) -> slot 2,
    (0,1) -> slot 3 and (1,0) -> slot 0: the pruning alone returns [0, 2]."""
    a = np.array([1e-8, 2e-8], np.float32)
    b = np.array([1.0, 1.0], np.float32)
    np.testing.assert_array_equal(pruned_topk(a, b, 2)[0], [0, 2])
    np.testing.assert_array_equal(route_topk(a, b, 2)[0], [0, 1])
    idx, _, repaired = repaired_topk(a, b, 2)
    assert repaired
    np.testing.assert_array_equal(idx, [0, 1])


def test_hand_derived_collisions():
    """The hand-derived rows of tests/golden/route_collisions.json: the pruning alone gives
    the recorded wrong slots, the repaired pruning the route's."""
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "route_collisions.json")))
    for c in g["cases"]:
        a = np.array(c["a"], np.float32)
        b = np.array(c["b"], np.float32)
        np.testing.assert_array_equal(pruned_topk(a, b, c["K"])[0], c["expect_pruned_only"])
        np.testing.assert_array_equal(route_topk(a, b, c["K"])[0], c["expect_route"])
        np.testing.assert_array_equal(repaired_topk(a, b, c["K"])[0], c["expect_route"])


@pytest.mark.parametrize("bf16", [False, True])
@pytest.mark.parametrize("kind", COLLISION_KINDS)
@pytest.mark.parametrize("S1,S2,K", [(16, 16, 8), (24, 40, 8), (256, 256, 64), (128, 96, 64),
                                     (128, 128, 128), (200, 136, 128)])
def test_repaired_pruning_equals_the_route_on_collisions(kind, bf16, S1, S2, K):
    rng = np.random.default_rng(S1 * 31 + S2 * 7 + K + 1000 * bf16 + 97 * len(kind))
    missed = 0
    for _ in range(12):
        a, b = collision_rows(rng, S1, S2, K, kind, bf16)
        ref_idx, ref_s = route_topk(a, b, K)
        got_idx, got_s, _ = repaired_topk(a, b, K, bf16)
        np.testing.assert_array_equal(got_idx, ref_idx)
        np.testing.assert_array_equal(got_s + 0.0, ref_s + 0.0)
        missed += not np.array_equal(pruned_topk(a, b, K)[0], ref_idx)
    if kind == "absorb1" or (kind == "near" and not bf16):
        # (tiny values in the second half cannot defeat the pruning: the flat index is
        # first-half major, so rank row 0, which the pruning keeps whole, holds every winner)
        assert missed > 0, "these rows are built to defeat the pruning alone"


@pytest.mark.parametrize("kind", ["normal", "palette", "skewed", "hyperbola", "dominant1",
                                  "dominant2"])
@pytest.mark.parametrize("S1,S2,K", [(16, 16, 8), (64, 64, 64), (256, 256, 128)])
def test_repaired_pruning_equals_the_route_on_exact_rows(kind, S1, S2, K):
    """On rows whose sums are exact the check must not change the result, whether or not it
    takes the repair (exact ties at T make it take the repair on fp32 rows)."""
    rng = np.random.default_rng(S1 + K + 11)
    for _ in range(6):
        a, b = rows(rng, S1, S2, kind)
        ref_idx, _ = route_topk(a, b, K)
        for bf16 in (False, True):
            np.testing.assert_array_equal(repaired_topk(a, b, K, bf16)[0], ref_idx)


@pytest.mark.parametrize("kind", COLLISION_KINDS)
def test_bf16_exactness_check_is_sound(kind):
    """Whenever the exponent-span check passes, every candidate sum is exact (checked in
    double), so the pruning alone gives the route's result."""
    rng = np.random.default_rng(len(kind))
    for K in (8, 64, 128):
        for _ in range(20):
            a, b = collision_rows(rng, 160, 160, K, kind, True)
            # shrink the span of some rows so that both outcomes of the check occur
            if rng.random() < 0.5:
                a = to_bf16(np.where(np.abs(a) < 2.0 ** -10, 0.0, a).astype(np.float32))
                b = to_bf16(np.where(np.abs(b) > 2.0 ** 10, 3.0, b).astype(np.float32))
            A, _ = half_sorted(a)
            B, _ = half_sorted(b)
            if bf16_sums_exact(A[:K], B[:K]):
                s32 = np.add.outer(A[:K], B[:K]).astype(np.float32).astype(np.float64)
                s64 = np.add.outer(A[:K].astype(np.float64), B[:K].astype(np.float64))
                np.testing.assert_array_equal(s32, s64)
                np.testing.assert_array_equal(pruned_topk(a, b, K)[0], route_topk(a, b, K)[0])


@pytest.mark.parametrize("K", [1, 2, 5, 16, 64, 100, 128])
def test_candidate_count_is_the_number_of_rank_pairs(K):
    pairs = sum(1 for r1 in range(K) for r2 in range(K) if (r1 + 1) * (r2 + 1) <= K)
    assert pairs == sum(K // r for r in range(1, K + 1))
    if K == 64:
        assert pairs == 280


@pytest.mark.parametrize("kind", ["normal", "palette", "skewed", "hyperbola", "dominant1",
                                  "dominant2"])
@pytest.mark.parametrize("S1,S2,K", [(16, 16, 8), (32, 24, 17), (64, 64, 64), (128, 96, 64),
                                     (200, 136, 100), (256, 256, 128)])
def test_rank_pair_pruning_keeps_the_top_k(kind, S1, S2, K):
    rng = np.random.default_rng(S1 * 1000 + S2 + K)
    for _ in range(6):
        a, b = rows(rng, S1, S2, kind)
        ref_idx, ref_s = brute_topk(a, b, K)
        got_idx, got_s, _ = pruned_topk(a, b, K)
        np.testing.assert_array_equal(got_idx, ref_idx)
        np.testing.assert_array_equal(got_s + 0.0, ref_s + 0.0)


@pytest.mark.parametrize("kind", ["normal", "palette", "skewed", "hyperbola", "dominant1",
                                  "dominant2"])
@pytest.mark.parametrize("S,K", [(64, 16), (512, 64), (1024, 64), (256, 128)])
def test_candidate_bracket_bounds_the_kth_sum(kind, S, K):
    rng = np.random.default_rng(S + K)
    for _ in range(6):
        a, b = rows(rng, S, S, kind)
        A, _ = half_sorted(a)
        B, _ = half_sorted(b)
        _, top_s, cand = pruned_topk(a, b, K)
        kth = top_s[K - 1]
        lo = max(np.float32(A[K - 1] + B[0]), np.float32(A[0] + B[K - 1]))
        assert lo <= kth
        assert np.float32(A[0] + B[0]) == cand.max() == top_s[0]


@pytest.mark.parametrize("lanes,per_lane", [(32, 8), (32, 16), (32, 32), (64, 8), (64, 16)])
@pytest.mark.parametrize("K", [1, 16, 33, 64, 128])
def test_lane_bracket_bounds_the_kth_key(lanes, per_lane, K):
    """Lane l holds values l*8 .. l*8+7 of every round of lanes*8 values (the load layout of
    the kernels); P = ceil(K / lanes)."""
    n = lanes * per_lane
    if K > n:
        pytest.skip("K beyond the values")
    rng = np.random.default_rng(lanes * 7 + per_lane + K)
    P = -(-K // lanes)
    for kind in ("normal", "palette", "skewed", "hyperbola"):
        x, _ = rows(rng, n, 1, kind)
        keys = np.sort(x)[::-1]
        kth = keys[K - 1]
        rounds = x.reshape(per_lane // 8, lanes, 8)
        per = rounds.transpose(1, 0, 2).reshape(lanes, per_lane)  # lane -> its values
        pth = np.sort(per, axis=1)[:, ::-1][:, P - 1]
        assert pth.min() <= kth
        assert per.max() == keys[0]


def test_bf16_sums_used_here_are_exact():
    """fp32 sums of two bf16 values whose exponents differ by less than 16 are exact: the
    condition under which the product-key route gives the top-K of all N sums."""
    rng = np.random.default_rng(5)
    a = to_bf16(rng.standard_normal(200000).astype(np.float32) * 4)
    b = to_bf16(rng.standard_normal(200000).astype(np.float32) * 4)
    ea = np.frexp(a)[1]
    eb = np.frexp(b)[1]
    ok = (np.abs(ea - eb) < 16) & (a != 0) & (b != 0)
    s32 = (a[ok] + b[ok]).astype(np.float32).astype(np.float64)
    exact = a[ok].astype(np.float64) + b[ok].astype(np.float64)
    np.testing.assert_array_equal(s32, exact)
