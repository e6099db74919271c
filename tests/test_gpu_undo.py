"""The logged prefill and the undo (sdm_scan_forward_logged, sdm_state_undo, through the C
ABI) against the oracle's undo log and backward replay: the logged pass computes what the
plain pass does (selections and state bit for bit), its log matches the oracle's log within
the pass's tolerance, and the undo gives back the starting state bit for bit, on both
engines, over several time chunks, from M0 and from a continued state, and on the long
skewed layer at 1/8 of its tokens."""

import numpy as np
import pytest
import torch

import oracle
import sdm_synth
from tests._parity import THREADS, assert_close, device_status_ok, host, sel_views

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
F32, BF16 = torch.float32, torch.bfloat16


@pytest.fixture(scope="module")
def sdm():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import __graft_entry__
    __graft_entry__.build()
    import sparse_memory_linear_b200 as m
    torch.cuda.set_device(0)
    return m


def inputs(wl):
    return {k: t.to(DEV) for k, t in sdm_synth.make_inputs(wl).items()}


def logged_then_undone(sdm, wl, g, engine, M_start, init):
    M = M_start.clone()
    out = sdm.sdm_scan_forward_logged(g["kp"], g["qp"], g["v"], g["alpha"], g["beta"], M,
                                      W=wl.W, R=wl.R, S1=wl.S1, M0=g["M0"], init=init,
                                      gate=g["gate"], engine=engine)
    torch.cuda.synchronize()
    device_status_ok()
    M_after = M.clone()
    sdm.sdm_state_undo(M, out["sel"], out["wlog"], W=wl.W, S1=wl.S1)
    torch.cuda.synchronize()
    device_status_ok()
    return out, M_after, M


@pytest.mark.parametrize("engine", ["seq", "slot"])
@pytest.mark.parametrize("name", ["tiny", "small"])
def test_log_matches_the_oracle_and_undo_restores_m0(sdm, name, engine):
    wl = sdm_synth.WORKLOADS[name]
    g = inputs(wl)
    M_start = torch.empty((wl.B, wl.H, wl.N, wl.d_v), dtype=F32, device=DEV)
    out, M_after, M_undone = logged_then_undone(sdm, wl, g, engine, M_start, "m0")
    f = host
    ref = oracle.forward(f(g["kp"]), f(g["qp"]), f(g["v"]), f(g["alpha"]), f(g["beta"]),
                         f(g["M0"]), S1=wl.S1, W=wl.W, R=wl.R, gate=f(g["gate"]),
                         threads=THREADS, want_log=True)
    sw, sr = sel_views(out["sel"], wl.B, wl.T, wl.H, wl.W, wl.R)
    np.testing.assert_array_equal(sw.cpu().numpy(), ref["idx_w"])
    np.testing.assert_array_equal(sr.cpu().numpy(), ref["idx_r"])
    assert_close(host(out["y"]), ref["y"], "y")
    assert_close(host(M_after), ref["M"], "M after the pass")
    assert_close(host(out["wlog"]), ref["wlog"], "undo log")
    start = g["M0"].unsqueeze(0).expand_as(M_undone)
    assert torch.equal(M_undone, start), "undo did not give back M0"
    # the plain pass computes the same selections and state
    M_plain = torch.empty_like(M_after)
    plain = sdm.sdm_scan_forward(g["kp"], g["qp"], g["v"], g["alpha"], g["beta"], M_plain,
                                 W=wl.W, R=wl.R, S1=wl.S1, M0=g["M0"], gate=g["gate"],
                                 want_sel=True, engine=engine)
    torch.cuda.synchronize()
    assert torch.equal(plain["sel"], out["sel"]) and torch.equal(M_plain, M_after)


@pytest.mark.parametrize("schedule", [1, 2])
def test_undo_over_several_chunks_from_a_continued_state(sdm, schedule):
    """The slot engine over 3 time chunks (128 + 128 + 44 tokens of 64 wide rows), serial
    and pipelined selection, starting from a state that is not M0."""
    wl = sdm_synth.WORKLOADS["tiny"].replace(B=8, H=8, T=300, S1=16, S2=16, W=8, R=8,
                                            d_v=1024, in_dtype=BF16, seed=62)
    g = inputs(wl)
    gen = torch.Generator(device=DEV).manual_seed(7)
    M_start = torch.randn((wl.B, wl.H, wl.N, wl.d_v), generator=gen, device=DEV)
    sdm.sdm_set_option("select_schedule", schedule)
    try:
        out, M_after, M_undone = logged_then_undone(sdm, wl, g, "slot", M_start, "continue")
    finally:
        sdm.sdm_set_option("select_schedule", 0)
    assert not torch.equal(M_after, M_start)
    assert torch.equal(M_undone, M_start)
    # log entries of a few units against the oracle's, all rows tracked
    f = host
    for b, h in ((0, 0), (5, 3), (7, 7)):
        r = oracle.run_unit(f(g["kp"]), f(g["qp"]), f(g["v"]), f(g["alpha"]), f(g["beta"]),
                            f(M_start), b, h, S1=wl.S1, W=wl.W, R=wl.R, threads=THREADS,
                            want_log=True)
        assert_close(host(out["wlog"][b, :, h]), r["wlog"], f"undo log of unit {(b, h)}")


def test_long_skew_undo_and_sampled_log(sdm):
    """The long skewed layer at 32768 tokens (4 time chunks, hot slots written thousands of
    times): the undo gives back M0 bit for bit; log entries of sampled tokens of head 1
    match the oracle's state at those tokens (tracked rows)."""
    wl = sdm_synth.WORKLOADS["long_skew"].replace(T=32768)
    g = inputs(wl)
    M_start = torch.empty((wl.B, wl.H, wl.N, wl.d_v), dtype=F32, device=DEV)
    out, M_after, M_undone = logged_then_undone(sdm, wl, g, "slot", M_start, "m0")
    assert torch.equal(M_undone, g["M0"].unsqueeze(0).expand_as(M_undone))
    b, h = 0, 1
    toks = [0, 5, 4095, 8191, 8192, 9000, 20000]
    sw, _ = sel_views(out["sel"], wl.B, wl.T, wl.H, wl.W, wl.R)
    kp_u = host(g["kp"][b, :, h])
    idx_w, wt_w = oracle.select(kp_u, wl.S1, wl.W, threads=THREADS)
    np.testing.assert_array_equal(sw[b, toks, h].cpu().numpy(), idx_w[toks])
    v_u = host(g["v"][b, :, h])[None, :, None, :]
    a_u = host(g["alpha"][b, :, h])[None, :, None]
    be_u = host(g["beta"][b, :, h])[None, :, None]
    M0_h = host(g["M0"][h])[None]
    dummy_r = np.zeros((wl.T, wl.R), np.int32), np.zeros((wl.T, wl.R), np.float64)
    for t in toks:
        rows = np.unique(idx_w[t])
        r = oracle.run_unit(kp_u[None, :, None, :], None, v_u, a_u, be_u, M0_h, 0, 0,
                            S1=wl.S1, W=wl.W, R=wl.R, rows=rows, t_end=t,
                            want_y=np.zeros(max(t, 1), bool),
                            selection=(idx_w[:t], wt_w[:t], dummy_r[0][:t], dummy_r[1][:t]))
        pos = np.searchsorted(rows, idx_w[t])
        assert_close(host(out["wlog"][b, t, h]), r["M"][pos], f"undo log at token {t}")
