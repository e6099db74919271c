"""Helpers of the GPU parity tests: tolerance, device inputs and sampled oracle checks."""

from __future__ import annotations

import os

import numpy as np
import torch

import oracle

# fp32 state, y and o against the double-precision oracle
TOL_ABS = 2e-4
TOL_REL = 1e-3
# slot weights (fp32 softmax against double)
WT_ABS = 2e-7
WT_REL = 4e-6

THREADS = max(1, min(64, os.cpu_count() or 1))


def assert_close(got, ref, what, atol=TOL_ABS, rtol=TOL_REL):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    err = np.abs(got - ref)
    bad = err > atol + rtol * np.abs(ref)
    if bad.any():
        i = np.unravel_index(np.argmax(err - rtol * np.abs(ref)), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} outside tolerance; "
                             f"worst at {i}: got {got[i]!r} ref {ref[i]!r}")


def host(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy()


def device_status_ok():
    import sparse_memory_linear_b200 as sdm
    assert sdm.sdm_get_device_status() == 0


def sel_views(sel: torch.Tensor, B, T, H, W, R):
    n = B * T * H
    sw = sel[: n * W].view(B, T, H, W)
    sr = sel[n * W: n * (W + R)].view(B, T, H, R)
    return sw, sr


def sampled_unit_check(wl, g: dict, out: dict, M: torch.Tensor, b: int, h: int, toks,
                       extra_rows, act="silu", eps=1e-6, gamma=None):
    """Checks one (b, h) of a GPU prefill against the oracle on sampled tokens and rows.

    The oracle selects the write slots of every token (needed for the state), the read
    slots of the sampled tokens only, and carries the tracked rows through the whole
    sequence.  Checks: selected slots of the sampled tokens bit-exact; y and o at the
    sampled tokens; the final state at the tracked rows.
    """
    T = wl.T
    toks = np.array(sorted(set(int(t) for t in toks)), np.int64)
    kp_u = host(g["kp"][b, :, h])
    qp_s = host(g["qp"][b, toks, h])
    idx_w, wt_w = oracle.select(kp_u, wl.S1, wl.W, threads=THREADS)
    idx_r = np.zeros((T, wl.R), np.int32)
    wt_r = np.zeros((T, wl.R), np.float64)
    ir, wr = oracle.select(qp_s, wl.S1, wl.R)
    idx_r[toks], wt_r[toks] = ir, wr
    rows = np.unique(np.concatenate([ir.ravel(), np.asarray(extra_rows, np.int64).ravel()]))
    want = np.zeros(T, bool)
    want[toks] = True
    v_u = host(g["v"][b, :, h])[None, :, None, :]
    a_u = host(g["alpha"][b, :, h])[None, :, None]
    be_u = host(g["beta"][b, :, h])[None, :, None]
    M0_h = host(g["M0"][h])[None]
    r = oracle.run_unit(kp_u[None, :, None, :], None, v_u, a_u, be_u, M0_h, 0, 0, S1=wl.S1,
                        W=wl.W, R=wl.R, rows=rows, want_y=want,
                        selection=(idx_w, wt_w, idx_r, wt_r))
    sw, sr = sel_views(out["sel"], wl.B, T, wl.H, wl.W, wl.R)
    np.testing.assert_array_equal(sw[b, toks, h].cpu().numpy(), idx_w[toks],
                                  err_msg=f"write slots of unit {(b, h)}")
    np.testing.assert_array_equal(sr[b, toks, h].cpu().numpy(), ir,
                                  err_msg=f"read slots of unit {(b, h)}")
    assert_close(host(out["y"][b, toks, h]), r["y"][toks], f"y of unit {(b, h)}")
    if out.get("o") is not None:
        gate = host(g["gate"][b, toks, h]) if "gate" in g else None
        o_ref = oracle.norm_gate(r["y"][toks], gate,
                                 None if gamma is None else host(gamma), eps, act)
        assert_close(host(out["o"][b, toks, h]), o_ref, f"o of unit {(b, h)}")
    assert_close(host(M[b, h, torch.as_tensor(rows, device=M.device)]), r["M"],
                 f"final M rows of unit {(b, h)}")
    return idx_w
