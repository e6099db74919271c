"""Pins of the CPU oracle against facts fixed by the method's statement and by
mathematics, not by the oracle itself: brute force over all outer sums, closed forms
of the write and read, the dense matrix form y_t = M_t^T q_t, hand-derived values and
the worked candidate count printed with the product-key selection.

The method's statement: "Sparse Delta Memory: Scaling the State of Linear RNNs
through Sparsity" (paper.rainbus.top summary), method steps 1-4, and the SDM write-up
on ai-paper-analysis.pages.dev, sections 步骤 1-4.
"""

import json
import math
import os

import numpy as np
import pytest
import scipy.special

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------- helpers
def brute_force_topk(row, S1, K):
    """Top-K of all S1*S2 fp32 outer sums, (score desc, slot asc), independent of the oracle."""
    a = np.asarray(row[:S1], np.float32)
    b = np.asarray(row[S1:], np.float32)
    s = np.add.outer(a, b).astype(np.float32).ravel()  # fp32 sums, slot = i1*S2 + i2
    s = s + np.float32(0.0)  # -0 -> +0
    flat = np.arange(s.size)
    order = np.lexsort((flat, -s.astype(np.float64)))
    sel = order[:K]
    return sel.astype(np.int32), s[sel]


def dense_reference(idx_w, wt_w, idx_r, wt_r, v, alpha, beta, M0):
    """The pass in dense matrix form: M_t = D_t M_{t-1} + b_t v_t^T with D_t diagonal
    (1 off the write set, alpha(1 - beta k_i) on it) and b_t = beta k; y_t = M_t^T q_t."""
    T = idx_w.shape[0]
    M = M0.astype(np.float64).copy()
    N = M.shape[0]
    ys = []
    for t in range(T):
        d = np.ones(N)
        bvec = np.zeros(N)
        d[idx_w[t]] = alpha[t] * (1.0 - beta[t] * wt_w[t])
        bvec[idx_w[t]] = beta[t] * wt_w[t]
        M = d[:, None] * M + np.outer(bvec, v[t].astype(np.float64))
        q = np.zeros(N)
        q[idx_r[t]] = wt_r[t]
        ys.append(M.T @ q)
    return np.array(ys), M


def rand_unit(rng, T, S1, S2, d_v, dtype=np.float32):
    kp = rng.standard_normal((1, T, 1, S1 + S2)).astype(dtype)
    qp = rng.standard_normal((1, T, 1, S1 + S2)).astype(dtype)
    v = rng.standard_normal((1, T, 1, d_v)).astype(np.float32)
    alpha = rng.uniform(0.05, 1.0, (1, T, 1)).astype(np.float32)
    beta = rng.uniform(0.0, 1.0, (1, T, 1)).astype(np.float32)
    M0 = (0.02 * rng.standard_normal((1, S1 * S2, d_v))).astype(np.float32)
    return kp, qp, v, alpha, beta, M0


# ------------------------------------------------------- the undo log of the in-place update
def test_undo_log_is_the_state_each_write_found():
    """Log entry (t, j) is written slot j's row after tokens [0, t): the final state of the
    pass cut at t, rounded to fp32 the same way, bit for bit; a log of the decayed row or of
    the row after the write differs."""
    rng = np.random.default_rng(31)
    T, S1, S2, d_v, W = 20, 4, 3, 5, 3
    kp, qp, v, alpha, beta, M0 = rand_unit(rng, T, S1, S2, d_v)
    r = oracle.run_unit(kp, qp, v, alpha, beta, M0, 0, 0, S1=S1, W=W, R=2, want_log=True)
    assert len(set(r["idx_w"].ravel().tolist())) < T * W  # slots written more than once
    for t in (0, 1, 7, T - 1):
        cut = oracle.run_unit(kp, qp, v, alpha, beta, M0, 0, 0, S1=S1, W=W, R=2, t_end=t)
        rows = cut["M"][r["idx_w"][t]]
        np.testing.assert_array_equal(r["wlog"][t].astype(np.float32), rows)


def test_undo_restores_the_starting_state():
    """Replaying the log backwards gives back the state the pass started from, exactly:
    from M0 and from a continued state, with slots written many times over."""
    rng = np.random.default_rng(32)
    T, S1, S2, d_v = 40, 3, 3, 4
    kp = rng.standard_normal((2, T, 2, S1 + S2)).astype(np.float32)
    qp = rng.standard_normal((2, T, 2, S1 + S2)).astype(np.float32)
    v = rng.standard_normal((2, T, 2, d_v)).astype(np.float32)
    alpha = rng.uniform(0.05, 1.0, (2, T, 2)).astype(np.float32)
    beta = rng.uniform(0.0, 1.0, (2, T, 2)).astype(np.float32)
    M0 = rng.standard_normal((2, S1 * S2, d_v)).astype(np.float32)
    M1 = rng.standard_normal((2, 2, S1 * S2, d_v)).astype(np.float32)
    for M_init in (M0, M1):
        r = oracle.forward(kp, qp, v, alpha, beta, M_init, S1=S1, W=3, R=2, want_log=True)
        start = np.broadcast_to(M_init, r["M"].shape) if M_init.ndim == 3 else M_init
        assert not np.array_equal(r["M"], start)
        np.testing.assert_array_equal(oracle.undo(r["M"], r["idx_w"], r["wlog"]),
                                      start.astype(np.float64))


def test_undo_of_three_decays_of_one_slot():
    """W = 1, beta = 0, alpha = 1/2: tokens 0-2 write slot 0 (8 -> 4 -> 2 -> 1), token 3
    writes slot 3 (8 -> 4).  The log holds 8, 4, 2, 8 (the row each write found) and the
    undo gives back 8 everywhere."""
    kp = np.tile(np.array([5.0, 0.0, 5.0, 0.0], np.float32), (1, 4, 1, 1))
    kp[0, 3, 0] = [0.0, 5.0, 0.0, 5.0]
    v = np.ones((1, 4, 1, 1), np.float32)
    alpha = np.full((1, 4, 1), 0.5, np.float32)
    beta = np.zeros((1, 4, 1), np.float32)
    M0 = np.full((1, 4, 1), 8.0, np.float32)
    r = oracle.forward(kp, kp, v, alpha, beta, M0, S1=2, W=1, R=1, want_log=True)
    assert r["idx_w"].ravel().tolist() == [0, 0, 0, 3]
    assert r["wlog"].ravel().tolist() == [8.0, 4.0, 2.0, 8.0]
    assert r["M"][0, 0, :, 0].tolist() == [1.0, 8.0, 8.0, 4.0]
    assert oracle.undo(r["M"], r["idx_w"], r["wlog"])[0, 0, :, 0].tolist() == [8.0] * 4


# ------------------------------------------------------------------ step 1: selection
@pytest.mark.parametrize("S1,S2", [(3, 5), (4, 4), (8, 16), (16, 16), (7, 9), (1, 6)])
def test_select_equals_brute_force_random(S1, S2):
    rng = np.random.default_rng(1000 + S1 * 31 + S2)
    for trial in range(40):
        row = rng.standard_normal(S1 + S2).astype(np.float32)
        for K in sorted({1, 2, min(S1, S2), max(1, min(S1, S2) // 2)}):
            want_idx, want_s = brute_force_topk(row, S1, K)
            for mode in ("product_key", "brute_force"):
                idx, wt = oracle.select(row[None], S1, K, mode=mode)
                np.testing.assert_array_equal(idx[0], want_idx, err_msg=f"{mode} K={K}")
                np.testing.assert_allclose(wt[0], scipy.special.softmax(want_s.astype(np.float64)),
                                           rtol=1e-12, atol=0)


@pytest.mark.parametrize("S1,S2", [(4, 4), (6, 3), (8, 8)])
def test_select_ties_and_signed_zeros(S1, S2):
    """Many equal half scores and both zeros: order falls back on the lowest slot."""
    rng = np.random.default_rng(7 + S1 + S2)
    palette = np.array([-1.0, -0.0, 0.0, 0.5, 1.0, 1.0, 2.0], np.float32)
    for trial in range(60):
        row = palette[rng.integers(0, palette.size, S1 + S2)]
        for K in range(1, min(S1, S2) + 1):
            want_idx, _ = brute_force_topk(row, S1, K)
            idx, wt = oracle.select(row[None], S1, K)
            np.testing.assert_array_equal(idx[0], want_idx)
    # all scores equal (a mix of -0 and +0): slots 0..K-1, equal weights
    row = np.array([-0.0, 0.0, 0.0, -0.0, 0.0, -0.0, -0.0, 0.0], np.float32)
    idx, wt = oracle.select(row[None], 4, 4)
    np.testing.assert_array_equal(idx[0], [0, 1, 2, 3])
    np.testing.assert_array_equal(wt[0], [0.25] * 4)


def test_select_non_square_keys_beyond_half():
    """K larger than one half (S1=1): the candidate set is the full second half."""
    row = np.array([0.5, 3.0, -1.0, 2.0, 2.0], np.float32)
    idx, _ = oracle.select(row[None], 1, 4)
    np.testing.assert_array_equal(idx[0], [0, 2, 3, 1])


def test_worked_candidate_count():
    g = json.load(open(os.path.join(GOLDEN, "pkm_worked_count.json")))
    rng = np.random.default_rng(3)
    row = rng.standard_normal(g["S1"] + g["S2"]).astype(np.float32)
    idx, wt, scored = oracle.select(row[None], g["S1"], g["K"], return_scored=True)
    assert g["S1"] * g["S2"] == g["N"]
    assert scored == g["candidate_sums"]
    want_idx, _ = brute_force_topk(row, g["S1"], g["K"])
    np.testing.assert_array_equal(idx[0], want_idx)


def test_select_sample_tokens_of_tiny_and_small_workloads():
    """The product-key route against brute force on real workload rows."""
    import torch
    import sdm_synth
    for name, ntok in (("tiny", 64), ("small", 24)):
        wl = sdm_synth.WORKLOADS[name]
        if name == "tiny":
            kp = sdm_synth.make_inputs(wl)["kp"]
        else:
            S = wl.S1 + wl.S2
            kp = sdm_synth.draw(wl.seed, sdm_synth.TID_KP, (ntok, S), wl.in_dtype)
        rows = kp.float().reshape(-1, wl.S1 + wl.S2).numpy()[:ntok]
        idx, _ = oracle.select(rows, wl.S1, wl.W)
        for r in range(rows.shape[0]):
            want_idx, _ = brute_force_topk(rows[r], wl.S1, wl.W)
            np.testing.assert_array_equal(idx[r], want_idx)


def test_select_route_when_sums_round():
    """Hand-derived rows whose candidate sums round onto one another
    (tests/golden/route_collisions.json): the oracle's product-key route keeps the top K of
    every half, then the lowest slots among equal candidate sums; the definition mode takes
    the top K of all sums.  The fixture also records what the rank-pair pruning alone gives,
    which the selection kernels must not return."""
    g = json.load(open(os.path.join(GOLDEN, "route_collisions.json")))
    for c in g["cases"]:
        a = np.array(c["a"], np.float32)
        b = np.array(c["b"], np.float32)
        row = np.concatenate([a, b])[None]
        idx, wt = oracle.select(row, a.size, c["K"])
        np.testing.assert_array_equal(idx[0], c["expect_route"])
        np.testing.assert_array_equal(wt[0], c["expect_wt"])
        idx_all, _ = oracle.select(row, a.size, c["K"], mode="brute_force")
        np.testing.assert_array_equal(idx_all[0], c["expect_all_sums"])
        want_all, _ = brute_force_topk(row[0], a.size, c["K"])
        np.testing.assert_array_equal(idx_all[0], want_all)
        assert c["expect_pruned_only"] != c["expect_route"]


# ------------------------------------------------------- the coupled delta rule
def test_coupled_rule_with_every_slot_selected_is_the_gated_delta_rule():
    """SDM write-up on ai-paper-analysis.pages.dev and the m.163.com article: SDM reduces to
    the gated delta rule when every slot is selected.  With the coupled prediction and
    W = R = N, the pass must equal the dense recurrence M_t = alpha_t (I - beta_t k k^T)
    M_{t-1} + beta_t k v_t^T, y_t = M_t^T q, written here with numpy matrices (k, q: the
    slot weights scattered over all N slots).  The per-slot write does not reduce to it."""
    rng = np.random.default_rng(12)
    S1 = S2 = 4
    N = S1 * S2
    T, d_v = 9, 5
    kp, qp, v, alpha, beta, M0 = rand_unit(rng, T, S1, S2, d_v)
    M0 = (0.3 * rng.standard_normal((1, N, d_v))).astype(np.float32)
    r = oracle.forward(kp, qp, v, alpha, beta, M0, S1=S1, W=N, R=N, coupled=True)
    M = M0[0].astype(np.float64)
    for t in range(T):
        k = np.zeros(N)
        q = np.zeros(N)
        k[r["idx_w"][0, t, 0]] = r["wt_w"][0, t, 0]
        q[r["idx_r"][0, t, 0]] = r["wt_r"][0, t, 0]
        a_t, b_t = float(alpha[0, t, 0]), float(beta[0, t, 0])
        M = a_t * (np.eye(N) - b_t * np.outer(k, k)) @ M + b_t * np.outer(k, v[0, t, 0])
        np.testing.assert_allclose(r["y"][0, t, 0], M.T @ q, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(r["M"][0, 0], M.astype(np.float32), rtol=1e-6, atol=1e-7)
    per_slot = oracle.forward(kp, qp, v, alpha, beta, M0, S1=S1, W=N, R=N)
    assert np.abs(per_slot["y"] - r["y"]).max() > 1e-3


def test_coupled_rule_with_one_write_slot_is_the_per_slot_rule():
    """With W = 1 the shared prediction is the one written row, k alpha M[i] with k = 1:
    the two readings coincide, bit for bit."""
    rng = np.random.default_rng(13)
    kp, qp, v, alpha, beta, M0 = rand_unit(rng, 30, 8, 8, 6)
    a = oracle.forward(kp, qp, v, alpha, beta, M0, S1=8, W=1, R=5, coupled=True)
    b = oracle.forward(kp, qp, v, alpha, beta, M0, S1=8, W=1, R=5)
    np.testing.assert_array_equal(a["y"], b["y"])
    np.testing.assert_array_equal(a["M"], b["M"])


def test_coupled_rule_needs_every_written_row_tracked():
    rng = np.random.default_rng(14)
    kp, qp, v, alpha, beta, M0 = rand_unit(rng, 4, 8, 8, 4)
    with pytest.raises(ValueError):
        oracle.run_unit(kp, qp, v, alpha, beta, M0, 0, 0, S1=8, W=4, R=4, rows=[0, 1],
                        want_y=np.zeros(4, bool), coupled=True)


# -------------------------------------------------------------- slot weights (softmax)
def test_weights_are_softmax_over_selected_set():
    rng = np.random.default_rng(11)
    rows = (1000.0 + rng.standard_normal((20, 32))).astype(np.float32)  # exp(1000) overflows
    idx, wt = oracle.select(rows, 16, 8)
    assert np.all(np.isfinite(wt))
    np.testing.assert_allclose(wt.sum(axis=1), 1.0, rtol=1e-14)
    assert np.all(np.diff(wt, axis=1) <= 0)  # selection order = weight order
    # a dominant pair: weight 1 up to exp(-gap)
    row = np.zeros(8, np.float32)
    row[2] = 60.0
    row[4 + 1] = 60.0
    idx, wt = oracle.select(row[None], 4, 3)
    assert idx[0, 0] == 2 * 4 + 1
    assert abs(wt[0, 0] - 1.0) < 1e-25 + 2 * math.exp(-60.0)


def test_selection_shift_invariance():
    """Adding an integer to every score of one half shifts all sums equally (exact
    for small integers), so slots and weights do not change."""
    rng = np.random.default_rng(5)
    row = rng.integers(-8, 8, 24).astype(np.float32)
    idx0, wt0 = oracle.select(row[None], 12, 5)
    shifted = row.copy()
    shifted[:12] += 37.0
    idx1, wt1 = oracle.select(shifted[None], 12, 5)
    np.testing.assert_array_equal(idx0, idx1)
    np.testing.assert_allclose(wt0, wt1, rtol=1e-15)


# ----------------------------------------------------------- steps 2-3: write and read
def test_hand_worked_example():
    g = json.load(open(os.path.join(GOLDEN, "tiny_worked_example.json")))
    T, S1, d_v = g["T"], g["S1"], g["d_v"]
    kp = np.array(g["kp"], np.float32).reshape(1, T, 1, -1)
    qp = np.array(g["qp"], np.float32).reshape(1, T, 1, -1)
    v = np.array(g["v"], np.float32).reshape(1, T, 1, d_v)
    alpha = np.array(g["alpha"], np.float32).reshape(1, T, 1)
    beta = np.array(g["beta"], np.float32).reshape(1, T, 1)
    M0 = np.array(g["M0"], np.float32)[None]
    r = oracle.forward(kp, qp, v, alpha, beta, M0, S1=S1, W=g["W"], R=g["R"], gate=None,
                       eps=0.0, act="identity")
    np.testing.assert_array_equal(r["idx_w"][0, :, 0], g["expect_idx_w"])
    np.testing.assert_array_equal(r["idx_r"][0, :, 0], g["expect_idx_r"])
    np.testing.assert_array_equal(r["wt_w"][0, :, 0], g["expect_wt"])
    np.testing.assert_array_equal(r["y"][0, :, 0], g["expect_y"])
    np.testing.assert_array_equal(r["M"][0, 0], g["expect_M"])


def test_beta_zero_is_pure_decay_and_unselected_rows_untouched():
    rng = np.random.default_rng(21)
    T, S1, S2, d_v = 12, 8, 7, 3
    kp, qp, v, alpha, beta, M0 = rand_unit(rng, T, S1, S2, d_v)
    beta[:] = 0.0
    r = oracle.run_unit(kp, qp, v, alpha, beta, M0, 0, 0, S1=S1, W=3, R=2)
    assert len(set(r["idx_w"].ravel().tolist())) < T * 3  # some slot written twice
    decay = np.ones(S1 * S2)
    for t in range(T):
        decay[r["idx_w"][t]] *= np.float64(alpha[0, t, 0])
    want = (decay[:, None] * M0[0].astype(np.float64)).astype(np.float32)
    np.testing.assert_allclose(r["M"], want, rtol=1e-6, atol=0)
    untouched = np.setdiff1d(np.arange(S1 * S2), r["idx_w"].ravel())
    assert untouched.size > 0
    assert r["M"][untouched].tobytes() == M0[0][untouched].tobytes()  # bit-identical


def test_unit_write_weight_and_beta_one_sets_slot_to_v():
    """W = 1 gives k = 1; with beta = 1 the written slot becomes v_t exactly."""
    rng = np.random.default_rng(22)
    T, S1, S2, d_v = 30, 4, 4, 5
    kp, qp, v, alpha, beta, M0 = rand_unit(rng, T, S1, S2, d_v)
    beta[:] = 1.0
    r = oracle.run_unit(kp, qp, v, alpha, beta, M0, 0, 0, S1=S1, W=1, R=1)
    assert np.all(r["wt_w"] == 1.0)
    last = {}
    for t in range(T):
        last[int(r["idx_w"][t, 0])] = t
    for slot, t in last.items():
        np.testing.assert_array_equal(r["M"][slot], v[0, t, 0])


def test_read_sees_this_tokens_write():
    """q' = k' makes the read set the write set; with W = R = 1 and beta = 1, y_t = v_t.
    A read taken before the write would return the old row instead."""
    rng = np.random.default_rng(23)
    T, S1, S2, d_v = 25, 4, 4, 4
    kp, qp, v, alpha, beta, M0 = rand_unit(rng, T, S1, S2, d_v)
    qp = kp.copy()
    beta[:] = 1.0
    r = oracle.run_unit(kp, qp, v, alpha, beta, M0, 0, 0, S1=S1, W=1, R=1)
    np.testing.assert_allclose(r["y"], v[0, :, 0].astype(np.float64), rtol=1e-15, atol=1e-300)


def test_two_writes_compose_affinely():
    """Two writes of one slot: M = a2 (a1 M0 + b1 v0) + b2 v1, a = alpha(1 - beta k),
    b = beta k (the step form expanded by hand)."""
    S1 = S2 = 2
    kp = np.array([[[[3.0, 0.0, 2.0, 0.0]]], [[[3.0, 0.0, 2.0, 0.0]]]], np.float32)
    kp = kp.reshape(1, 2, 1, 4)
    qp = kp.copy()
    v = np.array([[1.0, -2.0], [0.5, 4.0]], np.float32).reshape(1, 2, 1, 2)
    alpha = np.array([0.9, 0.7], np.float32).reshape(1, 2, 1)
    beta = np.array([0.6, 0.3], np.float32).reshape(1, 2, 1)
    M0 = np.array([[0.1, 0.2], [0.3, 0.4], [0.5, 0.6], [0.7, 0.8]], np.float32)[None]
    r = oracle.run_unit(kp, qp, v, alpha, beta, M0, 0, 0, S1=S1, W=2, R=2)
    # sums: slot0 = 5, slot1 = 3, slot2 = 2, slot3 = 0  -> top-2 = slots 0, 1
    np.testing.assert_array_equal(r["idx_w"], [[0, 1], [0, 1]])
    k0 = 1.0 / (1.0 + math.exp(-2.0))  # softmax of (5, 3)
    al = alpha[0, :, 0].astype(np.float64)
    be = beta[0, :, 0].astype(np.float64)
    a = al * (1.0 - be * k0)
    b = be * k0
    m0 = M0[0, 0].astype(np.float64)
    want = a[1] * (a[0] * m0 + b[0] * v[0, 0, 0]) + b[1] * v[0, 1, 0]
    np.testing.assert_allclose(r["M"][0], want.astype(np.float32), rtol=2e-7)


def test_matches_dense_matrix_form():
    """The sparse pass equals the dense form y_t = M_t^T q_t with a diagonal-plus-rank-1
    state update (the pages' y_t = M_t^T q_t written with dense q_t)."""
    rng = np.random.default_rng(31)
    T, S1, S2, d_v = 50, 5, 6, 7
    kp, qp, v, alpha, beta, M0 = rand_unit(rng, T, S1, S2, d_v)
    r = oracle.run_unit(kp, qp, v, alpha, beta, M0, 0, 0, S1=S1, W=4, R=3)
    y_d, M_d = dense_reference(r["idx_w"], r["wt_w"], r["idx_r"], r["wt_r"], v[0, :, 0],
                               alpha[0, :, 0].astype(np.float64),
                               beta[0, :, 0].astype(np.float64), M0[0])
    np.testing.assert_allclose(r["y"], y_d, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(r["M"], M_d.astype(np.float32), rtol=1e-6, atol=1e-9)


def test_read_of_every_slot():
    """W = R = N on a tiny memory: every slot is written and read each token."""
    rng = np.random.default_rng(32)
    T, S1, S2, d_v = 12, 2, 2, 3
    kp, qp, v, alpha, beta, M0 = rand_unit(rng, T, S1, S2, d_v)
    r = oracle.run_unit(kp, qp, v, alpha, beta, M0, 0, 0, S1=S1, W=4, R=4)
    for t in range(T):
        assert sorted(r["idx_r"][t]) == [0, 1, 2, 3]
    y_d, _ = dense_reference(r["idx_w"], r["wt_w"], r["idx_r"], r["wt_r"], v[0, :, 0],
                             alpha[0, :, 0].astype(np.float64),
                             beta[0, :, 0].astype(np.float64), M0[0])
    np.testing.assert_allclose(r["y"], y_d, rtol=1e-12, atol=1e-15)


def test_per_slot_recurrence_replay():
    """Each slot follows its own first-order recurrence M <- a M + b v over the tokens
    that write it; replaying it slot by slot reproduces the token-ordered pass."""
    rng = np.random.default_rng(33)
    T, S1, S2, d_v = 200, 4, 4, 6
    kp, qp, v, alpha, beta, M0 = rand_unit(rng, T, S1, S2, d_v)
    r = oracle.run_unit(kp, qp, v, alpha, beta, M0, 0, 0, S1=S1, W=3, R=3)
    M = M0[0].astype(np.float64).copy()
    for slot in range(S1 * S2):
        for t in range(T):
            hit = np.nonzero(r["idx_w"][t] == slot)[0]
            if hit.size:
                k = r["wt_w"][t, hit[0]]
                a = alpha[0, t, 0] * (1.0 - beta[0, t, 0] * k)
                b = beta[0, t, 0] * k
                M[slot] = a * M[slot] + b * v[0, t, 0]
    np.testing.assert_allclose(r["M"], M.astype(np.float32), rtol=1e-6, atol=1e-9)


def test_tracked_subset_equals_full_pass():
    rng = np.random.default_rng(34)
    T, S1, S2, d_v = 60, 8, 8, 4
    kp, qp, v, alpha, beta, M0 = rand_unit(rng, T, S1, S2, d_v)
    full = oracle.run_unit(kp, qp, v, alpha, beta, M0, 0, 0, S1=S1, W=4, R=4)
    want_t = np.zeros(T, bool)
    want_t[[5, 17, 59]] = True
    rows = np.unique(np.concatenate([full["idx_r"][want_t].ravel(), [0, 63]]))
    sub = oracle.run_unit(kp, qp, v, alpha, beta, M0, 0, 0, S1=S1, W=4, R=4, rows=rows,
                          want_y=want_t)
    np.testing.assert_array_equal(sub["y"][want_t], full["y"][want_t])
    np.testing.assert_array_equal(sub["M"], full["M"][rows])
    with pytest.raises(ValueError):  # a wanted read row that is not tracked
        oracle.run_unit(kp, qp, v, alpha, beta, M0, 0, 0, S1=S1, W=4, R=4, rows=rows[:1],
                        want_y=want_t)


def test_continue_equals_one_long_pass():
    """Running tokens [0, T1) then continuing from the state over [T1, T) equals one pass."""
    rng = np.random.default_rng(35)
    T, T1, S1, S2, d_v = 48, 19, 6, 6, 4
    kp, qp, v, alpha, beta, M0 = rand_unit(rng, T, S1, S2, d_v)
    full = oracle.forward(kp, qp, v, alpha, beta, M0, S1=S1, W=3, R=3)
    a = oracle.forward(kp[:, :T1], qp[:, :T1], v[:, :T1], alpha[:, :T1], beta[:, :T1], M0,
                       S1=S1, W=3, R=3)
    b = oracle.forward(kp[:, T1:], qp[:, T1:], v[:, T1:], alpha[:, T1:], beta[:, T1:], a["M"],
                       S1=S1, W=3, R=3)
    np.testing.assert_allclose(np.concatenate([a["y"], b["y"]], axis=1), full["y"],
                               rtol=1e-6, atol=1e-9)
    np.testing.assert_allclose(b["M"], full["M"], rtol=1e-6, atol=1e-9)


# ----------------------------------------------------------- step 4: RMSNorm and gate
@pytest.mark.parametrize("c", [0.3, -2.0, 1e-3])
def test_norm_gate_constant_vector(c):
    d_v, eps = 8, 1e-6
    y = np.full((1, d_v), c)
    gamma = np.linspace(0.5, 2.0, d_v).astype(np.float32)
    g = np.zeros((1, d_v), np.float32)
    base = np.sign(c) * gamma.astype(np.float64) / math.sqrt(1.0 + eps / (c * c))
    np.testing.assert_allclose(oracle.norm_gate(y, g, gamma, eps, "sigmoid")[0], 0.5 * base,
                               rtol=1e-14)
    np.testing.assert_allclose(oracle.norm_gate(y, g, gamma, eps, "silu")[0], 0.0, atol=0)
    g3 = np.full((1, d_v), math.log(3.0), np.float32)  # sigmoid(ln 3) = 3/4
    x = float(np.float32(math.log(3.0)))
    sig = 1.0 / (1.0 + math.exp(-x))
    np.testing.assert_allclose(oracle.norm_gate(y, g3, gamma, eps, "silu")[0], x * sig * base,
                               rtol=1e-14)
    np.testing.assert_allclose(oracle.norm_gate(y, g3, gamma, eps, "identity")[0], x * base,
                               rtol=1e-14)
    assert abs(sig - 0.75) < 1e-7


def test_norm_gate_pythagorean_and_scale_invariance():
    y = np.array([[3.0, 4.0]])
    o = oracle.norm_gate(y, None, None, 0.0, "identity")
    np.testing.assert_allclose(o[0], [3.0 / math.sqrt(12.5), 4.0 / math.sqrt(12.5)], rtol=1e-15)
    rng = np.random.default_rng(41)
    y = rng.standard_normal((5, 16))
    np.testing.assert_allclose(oracle.norm_gate(7.5 * y, None, None, 0.0),
                               oracle.norm_gate(y, None, None, 0.0), rtol=1e-13)
    o = oracle.norm_gate(y, None, None, 0.0)
    np.testing.assert_allclose(np.mean(o ** 2, axis=1), 1.0, rtol=1e-13)
