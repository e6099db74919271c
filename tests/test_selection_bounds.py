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

Sums are fp32, as the method's scores are.  The bf16 halves used keep every fp32 sum exact
(nonzero exponents less than 16 apart), the condition under which the route is exact.
"""

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
