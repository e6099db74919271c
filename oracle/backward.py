"""CPU oracle of the backward pass -- TEST INFRASTRUCTURE.

Gradients of the SDM memory pass (per-slot rule) for one (sequence, head) unit, computed the
way the m.163.com article on SDM (section 八, the memory-efficiency paragraph) trains: the
state is updated in place during the forward pass, and the backward pass walks the tokens
from the last to the first, undoing each token's writes from the undo log to recover the
state that the token saw.  Everything is float64; the selected slots are fixed by the
forward pass (the selection is piecewise constant), so the scores receive gradient through
the slot weights (a softmax over the selected sums) and each sum passes it to its two halves.

The method (paper.rainbus.top summary, method steps 1-4; ai-paper-analysis.pages.dev
write-up, 步骤 1-4), restated for token t with write slots I_w, weights k, read slots I_r,
weights q:  M[i] <- a_i M[i] + b_i v_t with a_i = alpha_t (1 - beta_t k_i), b_i = beta_t k_i;
y_t = sum_j q_j M[j] (after the write); o_t = y_t r_t gamma act(g_t) with
r_t = (mean(y_t^2) + eps)^(-1/2).

Only the test-suite may import this module; the product path never does.
"""

from __future__ import annotations

import numpy as np

from oracle import run_unit


def _act(g, act):
    if act == "silu":
        s = 1.0 / (1.0 + np.exp(-g))
        return g * s, s * (1.0 + g * (1.0 - s))
    if act == "sigmoid":
        s = 1.0 / (1.0 + np.exp(-g))
        return s, s * (1.0 - s)
    return g, np.ones_like(g)


def _weights(halves, idx, S1, S2):
    """Softmax, over the selected set, of the selected sums of halves [T, S1+S2] (float64)."""
    i1, i2 = idx // S2, idx % S2
    s = np.take_along_axis(halves[:, :S1], i1, 1) + np.take_along_axis(halves[:, S1:], i2, 1)
    e = np.exp(s - s.max(axis=1, keepdims=True))
    return e / e.sum(axis=1, keepdims=True)


def selection(kp, qp, S1, W, R):
    """The forward pass's selected slots of one unit (the oracle's product-key route on the
    fp32 halves).  kp, qp [T, S1+S2]."""
    T, S = kp.shape
    d = np.zeros((1, T, 1, 1), np.float32)
    kp32 = np.asarray(kp, np.float32)[None, :, None]
    qp32 = np.asarray(qp, np.float32)[None, :, None]
    r = run_unit(kp32, qp32, d, d[..., 0], d[..., 0],
                 np.zeros((1, S1 * (S - S1), 1), np.float32), 0, 0, S1=S1, W=W, R=R)
    return r["idx_w"].astype(np.int64), r["idx_r"].astype(np.int64)


def unit_forward(kp, qp, v, alpha, beta, M_init, gate, gamma, idx_w, idx_r, *, S1, eps=1e-6,
                 act="silu", want_log=False):
    """The pass in float64 with the given selected slots: returns o [T, d_v], y, the final
    state and, with want_log, the undo log [T, W, d_v] (each written row before its write)."""
    T, S = kp.shape
    S2 = S - S1
    k = _weights(np.asarray(kp, np.float64), idx_w, S1, S2)
    q = _weights(np.asarray(qp, np.float64), idx_r, S1, S2)
    M = np.array(M_init, np.float64, copy=True)
    y = np.zeros((T, v.shape[1]))
    wlog = np.zeros(idx_w.shape + (v.shape[1],)) if want_log else None
    for t in range(T):
        for j, i in enumerate(idx_w[t]):
            if want_log:
                wlog[t, j] = M[i]
            a = alpha[t] * (1.0 - beta[t] * k[t, j])
            M[i] = a * M[i] + beta[t] * k[t, j] * v[t]
        y[t] = q[t] @ M[idx_r[t]]
    r = 1.0 / np.sqrt(np.mean(y * y, axis=1, keepdims=True) + eps)
    A, _ = _act(np.asarray(gate, np.float64), act)
    o = y * r * gamma * A
    return dict(o=o, y=y, M=M, k=k, q=q, wlog=wlog)


def unit_backward(kp, qp, v, alpha, beta, M_init, gate, gamma, do, idx_w, idx_r, *, S1,
                  eps=1e-6, act="silu"):
    """Gradients of L = sum_t <do_t, o_t> with respect to kp, qp, v, alpha, beta, M_init,
    gate and gamma.  The forward keeps only the final state and the undo log; the backward
    restores each token's state by undoing its writes, in place, last token first.  Returns
    a dict of gradients and the state left after the walk ("M_restored", equal to M_init)."""
    T, S = kp.shape
    S2 = S - S1
    v = np.asarray(v, np.float64)
    alpha = np.asarray(alpha, np.float64)
    beta = np.asarray(beta, np.float64)
    gamma = np.asarray(gamma, np.float64)
    f = unit_forward(kp, qp, v, alpha, beta, M_init, gate, gamma, idx_w, idx_r, S1=S1, eps=eps,
                     act=act, want_log=True)
    y, k, q, M, wlog = f["y"], f["k"], f["q"], f["M"], f["wlog"]
    d_v = y.shape[1]
    # step 4: o = y r gamma A
    A, dA = _act(np.asarray(gate, np.float64), act)
    r = 1.0 / np.sqrt(np.mean(y * y, axis=1, keepdims=True) + eps)
    u = do * gamma * A                       # d o / d(y r) contracted with do
    dy = r * u - (r ** 3 / d_v) * y * np.sum(u * y, axis=1, keepdims=True)
    dgamma = np.sum(do * y * r * A, axis=0)
    dgate = do * y * r * gamma * dA
    # steps 2-3, last token first, undoing the writes as we go
    dM = np.zeros_like(M)
    dv = np.zeros_like(v)
    dalpha = np.zeros(T)
    dbeta = np.zeros(T)
    dk = np.zeros(idx_w.shape)
    dq = np.zeros(idx_r.shape)
    for t in range(T - 1, -1, -1):
        # the read saw the state after token t's writes: M, as it stands now
        for j, i in enumerate(idx_r[t]):
            dq[t, j] = dy[t] @ M[i]
            dM[i] += q[t, j] * dy[t]
        for j, i in enumerate(idx_w[t]):
            old = wlog[t, j]
            g = dM[i].copy()
            kj = k[t, j]
            a = alpha[t] * (1.0 - beta[t] * kj)
            b = beta[t] * kj
            da = g @ old
            db = g @ v[t]
            dv[t] += b * g
            dalpha[t] += da * (1.0 - beta[t] * kj)
            dbeta[t] += -da * alpha[t] * kj + db * kj
            dk[t, j] = -da * alpha[t] * beta[t] + db * beta[t]
            dM[i] = a * g
            M[i] = old  # undo the write
    # step 1: softmax over the selected set, then each sum to its two halves
    dsw = k * (dk - np.sum(k * dk, axis=1, keepdims=True))
    dsr = q * (dq - np.sum(q * dq, axis=1, keepdims=True))
    dkp = np.zeros((T, S))
    dqp = np.zeros((T, S))
    for dh, ds, idx in ((dkp, dsw, idx_w), (dqp, dsr, idx_r)):
        rows = np.repeat(np.arange(T), idx.shape[1])
        np.add.at(dh, (rows, (idx // S2).ravel()), ds.ravel())
        np.add.at(dh, (rows, S1 + (idx % S2).ravel()), ds.ravel())
    return dict(dkp=dkp, dqp=dqp, dv=dv, dalpha=dalpha, dbeta=dbeta, dM_init=dM,
                dgate=dgate, dgamma=dgamma, M_restored=M)
