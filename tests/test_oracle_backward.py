"""Pins of the backward-pass oracle (oracle/backward.py): its float64 forward against the pass
oracle, its gradients against central finite differences of the forward for every input and
every gate activation, and the state its backward walk leaves (the undo of every write gives
back the starting state exactly)."""

import numpy as np
import pytest

import oracle
from oracle import backward as BW

S1 = S2 = 4
T, W, R, D = 7, 3, 3, 5


def problem(seed, act="silu"):
    rng = np.random.default_rng(seed)
    x = dict(kp=rng.standard_normal((T, S1 + S2)).astype(np.float32),
             qp=rng.standard_normal((T, S1 + S2)).astype(np.float32),
             v=rng.standard_normal((T, D)),
             alpha=rng.uniform(0.3, 1.0, T),
             beta=rng.uniform(0.1, 0.9, T),
             M_init=rng.standard_normal((S1 * S2, D)),
             gate=rng.standard_normal((T, D)),
             gamma=rng.uniform(0.5, 1.5, D))
    idx_w, idx_r = BW.selection(x["kp"], x["qp"], S1, W, R)
    do = rng.standard_normal((T, D))
    return x, idx_w, idx_r, do


def loss(x, idx_w, idx_r, do, act):
    o = BW.unit_forward(x["kp"], x["qp"], x["v"], x["alpha"], x["beta"], x["M_init"], x["gate"],
                        x["gamma"], idx_w, idx_r, S1=S1, act=act)["o"]
    return float(np.sum(do * o))


def test_forward_matches_the_pass_oracle():
    x, idx_w, idx_r, _ = problem(1)
    f32 = lambda a: np.asarray(a, np.float32)  # noqa: E731
    r = oracle.run_unit(x["kp"][None, :, None], x["qp"][None, :, None], f32(x["v"])[None, :, None],
                        f32(x["alpha"])[None, :, None], f32(x["beta"])[None, :, None],
                        f32(x["M_init"])[None], 0, 0, S1=S1, W=W, R=R)
    np.testing.assert_array_equal(r["idx_w"], idx_w)
    # the pass oracle takes fp32 inputs; the same fp32 values through the float64 forward
    g = BW.unit_forward(x["kp"], x["qp"], f32(x["v"]).astype(np.float64),
                        f32(x["alpha"]).astype(np.float64), f32(x["beta"]).astype(np.float64),
                        f32(x["M_init"]).astype(np.float64), x["gate"], x["gamma"], idx_w, idx_r,
                        S1=S1)
    np.testing.assert_allclose(g["y"], r["y"], rtol=1e-6, atol=1e-9)
    np.testing.assert_allclose(g["M"], r["M"], rtol=1e-6, atol=1e-7)


@pytest.mark.parametrize("act", ["silu", "sigmoid", "identity"])
def test_gradients_match_finite_differences(act):
    x, idx_w, idx_r, do = problem(2, act)
    g = BW.unit_backward(x["kp"], x["qp"], x["v"], x["alpha"], x["beta"], x["M_init"],
                         x["gate"], x["gamma"], do, idx_w, idx_r, S1=S1, act=act)
    names = {"kp": "dkp", "qp": "dqp", "v": "dv", "alpha": "dalpha", "beta": "dbeta",
             "M_init": "dM_init", "gate": "dgate", "gamma": "dgamma"}
    for name, gname in names.items():
        base = np.asarray(x[name], np.float64)
        fd = np.zeros_like(base)
        for e in np.ndindex(base.shape):
            h = 1e-6 * max(1.0, abs(base[e]))
            for sign in (1, -1):
                y = dict(x)
                arr = base.copy()
                arr[e] += sign * h
                y[name] = arr
                fd[e] += sign * loss(y, idx_w, idx_r, do, act) / (2 * h)
        np.testing.assert_allclose(g[gname], fd, rtol=2e-5, atol=2e-7,
                                   err_msg=f"d{name} ({act})")


def test_the_backward_walk_undoes_every_write():
    x, idx_w, idx_r, do = problem(3)
    assert len(set(idx_w.ravel().tolist())) < idx_w.size  # slots written more than once
    g = BW.unit_backward(x["kp"], x["qp"], x["v"], x["alpha"], x["beta"], x["M_init"],
                         x["gate"], x["gamma"], do, idx_w, idx_r, S1=S1)
    np.testing.assert_array_equal(g["M_restored"], x["M_init"])
