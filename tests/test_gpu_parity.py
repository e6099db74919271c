"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Selected slots must match bit for bit; y, o and the state within
|d| <= 2e-4 + 1e-3 |ref|; slot weights within 2e-7 + 4e-6 |ref|.
"""

import numpy as np
import pytest
import torch

import oracle
import sdm_synth
from tests._parity import (THREADS, WT_ABS, WT_REL, assert_close, device_status_ok, host,
                           sampled_unit_check, sel_views)

pytestmark = pytest.mark.gpu

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


DEV = "cuda:0"


# --------------------------------------------------------------------------- step 1
SELECT_CASES = [
    (16, 16, 8, F32), (256, 256, 64, BF16), (512, 512, 64, BF16), (1024, 1024, 64, BF16),
    (7, 9, 7, F32), (33, 17, 17, BF16), (100, 37, 37, F32), (1, 1, 1, F32), (2, 3, 2, BF16),
    (64, 64, 1, BF16), (128, 128, 128, BF16), (4096, 4096, 128, BF16), (300, 500, 100, F32),
]


@pytest.mark.parametrize("S1,S2,K,dt", SELECT_CASES)
def test_select_matches_oracle(sdm, S1, S2, K, dt):
    n = 200 if S1 * S2 < (1 << 22) else 40
    x = sdm_synth.draw(17 + S1 + S2 + K, 1, (n, S1 + S2), dt)
    idx, wt = sdm.sdm_select(x.to(DEV), K, S1=S1)
    torch.cuda.synchronize()
    device_status_ok()
    ref_idx, ref_wt = oracle.select(host(x), S1, K, threads=THREADS)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref_idx)
    assert_close(wt.cpu().numpy(), ref_wt, "weights", atol=WT_ABS, rtol=WT_REL)
    if S1 * S2 <= 4096:
        bf_idx, _ = oracle.select(host(x), S1, K, mode="brute_force")
        np.testing.assert_array_equal(idx.cpu().numpy(), bf_idx)


@pytest.mark.parametrize("S1,S2,K", [(1024, 1024, 64), (512, 512, 64), (256, 200, 33),
                                     (1000, 24, 17), (8, 8, 8), (128, 130, 128)])
def test_select_fast_path_equals_general_path(sdm, S1, S2, K):
    """bf16 rows take the register-resident path; forcing the general path must give the
    same slots bit for bit and the same weights."""
    x = sdm_synth.draw(5 + S1 + K, 1, (300, S1 + S2), BF16).to(DEV)
    idx_f, wt_f = sdm.sdm_select(x, K, S1=S1)
    sdm.sdm_set_option("select_general", 1)
    try:
        idx_g, wt_g = sdm.sdm_select(x, K, S1=S1)
    finally:
        sdm.sdm_set_option("select_general", 0)
    torch.cuda.synchronize()
    assert torch.equal(idx_f, idx_g)
    assert_close(wt_f.cpu().numpy(), wt_g.cpu().numpy(), "weights", atol=1e-7, rtol=1e-6)


@pytest.mark.parametrize("dt", [F32, BF16])
@pytest.mark.parametrize("S1,S2,K", [(8, 8, 8), (16, 12, 5), (64, 64, 64), (40, 40, 9)])
def test_select_ties_and_signed_zeros(sdm, S1, S2, K, dt):
    rng = np.random.default_rng(S1 * 7 + K)
    palette = np.array([-1.0, -0.0, 0.0, 0.5, 1.0, 1.0, 2.0, 0.25], np.float32)
    x = palette[rng.integers(0, palette.size, (300, S1 + S2))]
    x[:20] = 0.0
    x[20:40] = -0.0
    xt = torch.from_numpy(x).to(dt)
    idx, wt = sdm.sdm_select(xt.to(DEV), K, S1=S1)
    ref_idx, ref_wt = oracle.select(host(xt), S1, K, mode="brute_force")
    np.testing.assert_array_equal(idx.cpu().numpy(), ref_idx)
    assert_close(wt.cpu().numpy(), ref_wt, "weights", atol=WT_ABS, rtol=WT_REL)


def test_select_skewed_halves(sdm):
    """Long-prefill halves (per-index bias): many hot low indices."""
    wl = sdm_synth.WORKLOADS["long_skew"]
    x = sdm_synth.draw(wl.seed, sdm_synth.TID_KP, (500, wl.S1 + wl.S2), BF16,
                       transform=sdm_synth._skew_transform(wl.S1, wl.S2))
    idx, wt = sdm.sdm_select(x.to(DEV), wl.W, S1=wl.S1)
    ref_idx, ref_wt = oracle.select(host(x), wl.S1, wl.W, threads=THREADS)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref_idx)
    assert_close(wt.cpu().numpy(), ref_wt, "weights", atol=WT_ABS, rtol=WT_REL)


# --------------------------------------------------------------------- steps 1-4
def run_scan(sdm, wl, g, *, gamma=None, act="silu", eps=1e-6, engine="auto", init="m0",
             M=None, want_o=True):
    if M is None:
        M = torch.empty((wl.B, wl.H, wl.N, wl.d_v), dtype=F32, device=DEV)
    out = sdm.sdm_scan_forward(g["kp"], g["qp"], g["v"], g["alpha"], g["beta"], M, W=wl.W,
                               R=wl.R, S1=wl.S1, M0=g.get("M0"), init=init,
                               gate=g.get("gate"), gamma=gamma, eps=eps, act=act,
                               want_o=want_o, want_sel=True, engine=engine)
    torch.cuda.synchronize()
    device_status_ok()
    return out, M


def full_check(wl, g, out, M, *, gamma=None, act="silu", eps=1e-6, M_init=None):
    f = host
    ref = oracle.forward(f(g["kp"]), f(g["qp"]), f(g["v"]), f(g["alpha"]), f(g["beta"]),
                         f(g["M0"]) if M_init is None else M_init, S1=wl.S1, W=wl.W, R=wl.R,
                         gate=None if g.get("gate") is None else f(g["gate"]),
                         gamma=None if gamma is None else f(gamma), eps=eps, act=act,
                         threads=THREADS)
    sw, sr = sel_views(out["sel"], wl.B, wl.T, wl.H, wl.W, wl.R)
    np.testing.assert_array_equal(sw.cpu().numpy(), ref["idx_w"], err_msg="write slots")
    np.testing.assert_array_equal(sr.cpu().numpy(), ref["idx_r"], err_msg="read slots")
    assert_close(host(out["y"]), ref["y"], "y")
    if out["o"] is not None:
        assert_close(host(out["o"]), ref["o"], "o")
    assert_close(host(M), ref["M"], "final M")
    return ref


def device_inputs(wl, **kw):
    return {k: t.to(DEV) for k, t in sdm_synth.make_inputs(wl, **kw).items()}


ENGINES = ["seq", "slot", "chunk"]


@pytest.mark.parametrize("engine", ENGINES)
@pytest.mark.parametrize("act", ["silu", "sigmoid", "identity"])
def test_scan_tiny_full(sdm, act, engine):
    wl = sdm_synth.WORKLOADS["tiny"]
    g = device_inputs(wl, with_gamma=True)
    out, M = run_scan(sdm, wl, g, gamma=g["gamma"], act=act, engine=engine)
    ref = full_check(wl, g, out, M, gamma=g["gamma"], act=act)
    # rows never written keep M0 bit for bit
    untouched = np.setdiff1d(np.arange(wl.N), ref["idx_w"].ravel())
    assert untouched.size > 0
    assert (host(M[0, 0])[untouched].tobytes() == host(g["M0"][0])[untouched].tobytes())


@pytest.mark.parametrize("engine", ENGINES)
def test_scan_small_full(sdm, engine):
    wl = sdm_synth.WORKLOADS["small"]
    g = device_inputs(wl)
    out, M = run_scan(sdm, wl, g, engine=engine)
    full_check(wl, g, out, M)


@pytest.mark.parametrize("kw", [
    dict(B=2, H=3, T=37, S1=24, S2=40, W=5, R=11, d_v=16, in_dtype=F32),   # ragged, W != R
    dict(B=1, H=2, T=50, S1=64, S2=64, W=16, R=48, d_v=8, in_dtype=BF16),  # narrowest bf16
    dict(B=3, H=1, T=40, S1=32, S2=32, W=8, R=8, d_v=4, in_dtype=F32),     # d_v = 4
    dict(B=1, H=1, T=1, S1=16, S2=16, W=1, R=1, d_v=32, in_dtype=BF16),    # one token, K = 1
    dict(B=2, H=2, T=65, S1=128, S2=128, W=128, R=128, d_v=256, in_dtype=BF16),  # K = 128
    dict(B=1, H=2, T=30, S1=8, S2=8, W=8, R=8, d_v=512, in_dtype=BF16),    # every slot hit
])
@pytest.mark.parametrize("engine", ENGINES)
def test_scan_edge_shapes(sdm, kw, engine):
    wl = sdm_synth.WORKLOADS["tiny"].replace(**kw, seed=99 + kw["T"])
    g = device_inputs(wl, with_gamma=True)
    out, M = run_scan(sdm, wl, g, gamma=g["gamma"], engine=engine)
    full_check(wl, g, out, M, gamma=g["gamma"])


@pytest.mark.parametrize("engine", ENGINES)
def test_scan_without_gate_or_output(sdm, engine):
    """No gate, and no output o: y and the state are those of the run with o.  The state is
    deterministic in every engine; the slot engine adds each read into y with float atomics,
    whose order (and so y's last bits) may change from run to run."""
    wl = sdm_synth.WORKLOADS["tiny"].replace(B=2, T=20, seed=5)
    g = device_inputs(wl, with_gate=False)
    out, M = run_scan(sdm, wl, g, eps=0.0, engine=engine)
    full_check(wl, g, out, M, eps=0.0)
    out2, M2 = run_scan(sdm, wl, g, want_o=False, engine=engine)
    assert out2["o"] is None
    assert torch.equal(M2, M)
    if engine in ("seq", "chunk"):
        assert torch.equal(out2["y"], out["y"])
    else:
        assert_close(host(out2["y"]), host(out["y"]), "y", atol=1e-7, rtol=1e-6)


@pytest.mark.parametrize("engine", ENGINES)
def test_scan_all_scores_equal(sdm, engine):
    """Every token selects the same slots (all sums tie): each token's rows were written
    by every token before it (the sequential engine forwards them from shared memory;
    the slot engine sees one long segment per slot)."""
    wl = sdm_synth.WORKLOADS["tiny"].replace(B=1, H=2, T=70, S1=32, S2=32, W=16, R=16,
                                            d_v=64, in_dtype=BF16, seed=7)
    g = device_inputs(wl)
    g["kp"].zero_()
    g["qp"].zero_()
    g["qp"][..., 0] = 1.0
    out, M = run_scan(sdm, wl, g, engine=engine)
    full_check(wl, g, out, M)


@pytest.mark.parametrize("engine", ENGINES)
def test_scan_continue_equals_one_pass(sdm, engine):
    wl = sdm_synth.WORKLOADS["small"].replace(B=1, T=300, seed=11)
    g = device_inputs(wl)
    out, M = run_scan(sdm, wl, g, engine=engine)
    T1 = 113
    first = {k: (t[:, :T1].contiguous() if k not in ("M0",) else t) for k, t in g.items()}
    second = {k: (t[:, T1:].contiguous() if k not in ("M0",) else t) for k, t in g.items()}
    w1, w2 = wl.replace(T=T1), wl.replace(T=wl.T - T1)
    o1, M1 = run_scan(sdm, w1, first, engine=engine)
    o2, M1 = run_scan(sdm, w2, second, init="continue", M=M1, engine=engine)
    assert_close(host(torch.cat([o1["y"], o2["y"]], 1)), host(out["y"]), "y split", atol=1e-6,
                 rtol=1e-5)
    assert_close(host(M1), host(M), "M split", atol=1e-6, rtol=1e-5)


def test_scan_zero_tokens_only_initialises(sdm):
    wl = sdm_synth.WORKLOADS["tiny"].replace(B=2, seed=3)
    g = device_inputs(wl)
    M = torch.full((wl.B, wl.H, wl.N, wl.d_v), 7.0, dtype=F32, device=DEV)
    empty = {k: (t[:, :0] if k != "M0" else t) for k, t in g.items()}
    sdm.sdm_scan_forward(empty["kp"], empty["qp"], empty["v"], empty["alpha"], empty["beta"],
                         M, W=wl.W, R=wl.R, M0=g["M0"], gate=empty["gate"])
    torch.cuda.synchronize()
    assert torch.equal(M, g["M0"].expand_as(M))


@pytest.mark.parametrize("engine", ["auto"] + ENGINES)
def test_scan_layer1p4b_sampled(sdm, engine):
    """The 1.4B-like layer at full size, launched as the benchmark launches it."""
    wl = sdm_synth.WORKLOADS["layer1p4b"]
    g = device_inputs(wl)
    out, M = run_scan(sdm, wl, g, engine=engine)
    rng = np.random.default_rng(1)
    for (b, h) in [(0, 0), (3, 7), (2, 5)]:
        toks = [0, 1, 2, wl.T - 1] + list(rng.integers(0, wl.T, 12))
        extra = np.concatenate([rng.integers(0, wl.N, 64), [0, wl.N - 1]])
        idx_w = sampled_unit_check(wl, g, out, M, b, h, toks, extra)
        # rows that no token wrote still hold M0, bit for bit
        untouched = np.setdiff1d(rng.integers(0, wl.N, 4096), idx_w.ravel())
        ut = torch.as_tensor(untouched, device=DEV)
        assert torch.equal(M[b, h, ut], g["M0"][h, ut])


@pytest.mark.parametrize("engine", ["auto", "seq", "slot"])
def test_scan_long_skew_sampled(sdm, engine):
    """The long skewed prefill at full size (hot slots written thousands of times).  The
    chunk-wise engine, a CTA per (head, column slice) through 8192 chunks here, is checked at
    full size on the 1.4B-like layer instead."""
    wl = sdm_synth.WORKLOADS["long_skew"]
    g = device_inputs(wl)
    out, M = run_scan(sdm, wl, g, engine=engine)
    rng = np.random.default_rng(2)
    for (b, h) in [(0, 1)]:
        toks = [0, 1, wl.T // 2, wl.T - 1] + list(rng.integers(0, wl.T, 12))
        extra = np.concatenate([rng.integers(0, wl.N, 64), [0, 1, 1024, 1025, wl.N - 1]])
        sampled_unit_check(wl, g, out, M, b, h, toks, extra)


# ------------------------------------------------------------------------- decode
def decode_steps(sdm, wl, steps, M, gamma=None, chained=False):
    """One sdm_decode_step per step, or with chained=True one sdm_decode_step_chained per
    step over inputs staged on the device before the first launch."""
    ys, os_, sels = [], [], []
    staged = [{k: t.to(DEV) for k, t in s.items() if k != "M0"} for s in steps] if chained \
        else None
    if chained:
        torch.cuda.synchronize()
    for i, s in enumerate(steps):
        gs = staged[i] if chained else {k: t.to(DEV) for k, t in s.items() if k != "M0"}
        out = sdm.sdm_decode_step(gs["kp"], gs["qp"], gs["v"], gs["alpha"], gs["beta"], M,
                                  W=wl.W, R=wl.R, S1=wl.S1, gate=gs.get("gate"), gamma=gamma,
                                  want_sel=True, chained=chained)
        ys.append(out["y"])
        os_.append(out["o"])
        sels.append(out["sel"])
    torch.cuda.synchronize()
    device_status_ok()
    return torch.stack(ys, 1), torch.stack(os_, 1), sels


@pytest.mark.parametrize("kw", [
    dict(B=3, H=2, S1=64, S2=64, W=16, R=16, d_v=64, in_dtype=BF16),
    dict(B=2, H=3, S1=20, S2=12, W=7, R=3, d_v=12, in_dtype=F32),
    dict(B=1, H=1, S1=256, S2=256, W=128, R=64, d_v=256, in_dtype=BF16),
    dict(B=2, H=1, S1=64, S2=64, W=16, R=16, d_v=1024, in_dtype=BF16),
    dict(B=2, H=2, S1=1024, S2=1024, W=64, R=32, d_v=128, in_dtype=BF16),
    dict(B=1, H=3, S1=200, S2=136, W=100, R=128, d_v=32, in_dtype=BF16),
])
def test_decode_matches_oracle(sdm, kw):
    wl = sdm_synth.WORKLOADS["decode"].replace(T=6, seed=21, **kw)
    steps = [sdm_synth.make_inputs(wl, step=s, with_gamma=True) for s in range(wl.T)]
    M0 = steps[0]["M0"]
    gamma = steps[0]["gamma"].to(DEV)
    M = M0.to(DEV).unsqueeze(0).expand(wl.B, -1, -1, -1).contiguous()
    y, o, sels = decode_steps(sdm, wl, steps, M, gamma=gamma)
    st = lambda k: np.stack([host(s[k]) for s in steps], 1)  # noqa: E731  [B, T, H, ...]
    ref = oracle.forward(st("kp"), st("qp"), st("v"), st("alpha"), st("beta"), host(M0),
                         S1=wl.S1, W=wl.W, R=wl.R, gate=st("gate"), gamma=host(gamma))
    for t, sel in enumerate(sels):
        nw = wl.B * wl.H * wl.W
        np.testing.assert_array_equal(sel[:nw].view(wl.B, wl.H, wl.W).cpu().numpy(),
                                      ref["idx_w"][:, t])
        np.testing.assert_array_equal(sel[nw:].view(wl.B, wl.H, wl.R).cpu().numpy(),
                                      ref["idx_r"][:, t])
    assert_close(host(y), ref["y"], "decode y")
    assert_close(host(o), ref["o"], "decode o")
    assert_close(host(M), ref["M"], "decode M")


@pytest.mark.parametrize("S1,S2,W,R", [(64, 64, 16, 16), (512, 512, 64, 64),
                                         (128, 160, 128, 100)])
def test_decode_ties_and_signed_zeros(sdm, S1, S2, W, R):
    """Decode selection on scores drawn from a small palette (many equal sums, -0 and +0):
    equal scores take the lowest indices, exactly as the oracle orders them."""
    wl = sdm_synth.WORKLOADS["decode"].replace(B=3, H=2, T=3, S1=S1, S2=S2, W=W, R=R,
                                               d_v=64, seed=29)
    rng = np.random.default_rng(S1 + W)
    palette = np.array([-1.0, -0.0, 0.0, 0.5, 1.0, 1.0, 2.0, 0.25], np.float32)
    steps = []
    for s in range(wl.T):
        st = sdm_synth.make_inputs(wl, step=s)
        for k in ("kp", "qp"):
            x = palette[rng.integers(0, palette.size, tuple(st[k].shape))]
            if s == 1:
                x[0] = 0.0
                x[1] = -0.0
            st[k] = torch.from_numpy(x).to(BF16)
        steps.append(st)
    M0 = steps[0]["M0"]
    M = M0.to(DEV).unsqueeze(0).expand(wl.B, -1, -1, -1).contiguous()
    y, o, sels = decode_steps(sdm, wl, steps, M)
    st = lambda k: np.stack([host(s[k]) for s in steps], 1)  # noqa: E731
    ref = oracle.forward(st("kp"), st("qp"), st("v"), st("alpha"), st("beta"), host(M0),
                         S1=wl.S1, W=wl.W, R=wl.R, gate=st("gate"))
    for t, sel in enumerate(sels):
        nw = wl.B * wl.H * wl.W
        np.testing.assert_array_equal(sel[:nw].view(wl.B, wl.H, wl.W).cpu().numpy(),
                                      ref["idx_w"][:, t])
        np.testing.assert_array_equal(sel[nw:].view(wl.B, wl.H, wl.R).cpu().numpy(),
                                      ref["idx_r"][:, t])
    assert_close(host(y), ref["y"], "decode ties y")
    assert_close(host(M), ref["M"], "decode ties M")


def test_decode_equals_scan(sdm):
    wl = sdm_synth.WORKLOADS["decode"].replace(B=4, H=2, T=16, S1=128, S2=128, seed=23)
    steps = [sdm_synth.make_inputs(wl, step=s) for s in range(wl.T)]
    M0 = steps[0]["M0"].to(DEV)
    Md = M0.unsqueeze(0).expand(wl.B, -1, -1, -1).contiguous()
    y_d, o_d, _ = decode_steps(sdm, wl, steps, Md)
    g = {k: torch.stack([s[k] for s in steps], 1).to(DEV) for k in steps[0] if k != "M0"}
    g["M0"] = M0
    out, Ms = run_scan(sdm, wl, g)
    assert_close(host(y_d), host(out["y"]), "decode vs scan y", atol=1e-6, rtol=1e-5)
    assert_close(host(o_d), host(out["o"]), "decode vs scan o", atol=1e-6, rtol=1e-5)
    assert_close(host(Md), host(Ms), "decode vs scan M", atol=1e-6, rtol=1e-5)


def test_decode_chained_equals_plain(sdm):
    """Chained launches (each step's selection overlapping the step before) give the plain
    launches' results bit for bit."""
    wl = sdm_synth.WORKLOADS["decode"].replace(B=16, T=12, S1=256, S2=256, seed=31)
    steps = [sdm_synth.make_inputs(wl, step=s) for s in range(wl.T)]
    M0 = steps[0]["M0"].to(DEV)
    Mp = M0.unsqueeze(0).expand(wl.B, -1, -1, -1).contiguous()
    Mc = Mp.clone()
    y_p, o_p, sel_p = decode_steps(sdm, wl, steps, Mp)
    y_c, o_c, sel_c = decode_steps(sdm, wl, steps, Mc, chained=True)
    for a, b in zip(sel_p, sel_c):
        assert torch.equal(a, b)
    assert torch.equal(y_p, y_c) and torch.equal(o_p, o_c) and torch.equal(Mp, Mc)


def test_decode_full_size_sampled(sdm):
    """The batched-decode workload at full size (64 GB state), a few chained steps."""
    wl = sdm_synth.WORKLOADS["decode"]
    nsteps = 3
    steps = [{k: t.to(DEV) for k, t in sdm_synth.make_inputs(wl, step=s).items()}
             for s in range(nsteps)]
    M0 = steps[0]["M0"]
    M = torch.empty((wl.B, wl.H, wl.N, wl.d_v), dtype=F32, device=DEV)
    sdm.sdm_state_init(M0, M)
    y, o, sels = decode_steps(sdm, wl, steps, M, chained=True)
    st = lambda k, b, h: np.stack([host(s[k][b, h]) for s in steps], 0)  # noqa: E731
    for (b, h) in [(0, 0), (63, 7), (17, 3)]:
        kp = st("kp", b, h)[None, :, None]
        r = oracle.run_unit(kp, st("qp", b, h)[None, :, None], st("v", b, h)[None, :, None],
                            st("alpha", b, h)[None, :, None], st("beta", b, h)[None, :, None],
                            host(M0[h])[None], 0, 0, S1=wl.S1, W=wl.W, R=wl.R)
        o_ref = oracle.norm_gate(r["y"], st("gate", b, h), None, 1e-6, "silu")
        assert_close(host(y[b, :, h]), r["y"], f"decode y {(b, h)}")
        assert_close(host(o[b, :, h]), o_ref, f"decode o {(b, h)}")
        touched = np.unique(np.concatenate([r["idx_w"].ravel(), r["idx_r"].ravel()]))
        tt = torch.as_tensor(touched, device=DEV)
        assert_close(host(M[b, h, tt]), r["M"][touched], f"decode M {(b, h)}")


# --------------------------------------------------------------------------- step 4
@pytest.mark.parametrize("act", ["silu", "sigmoid", "identity"])
@pytest.mark.parametrize("dt", [F32, BF16])
def test_norm_gate(sdm, act, dt):
    rng = np.random.default_rng(4)
    y = torch.from_numpy(rng.standard_normal((3, 50, 256)).astype(np.float32))
    y[0, 0] = 0.0
    y[0, 1] = 1e-4
    g = torch.from_numpy(rng.standard_normal((3, 50, 256)).astype(np.float32)).to(dt)
    gamma = torch.from_numpy(rng.uniform(0.5, 1.5, 256).astype(np.float32))
    o = sdm.sdm_norm_gate(y.to(DEV), gate=g.to(DEV), gamma=gamma.to(DEV), eps=1e-6, act=act)
    ref = oracle.norm_gate(y.numpy(), host(g), gamma.numpy(), 1e-6, act)
    assert_close(host(o), ref, "o")
    o2 = sdm.sdm_norm_gate(y.to(DEV), eps=0.5)
    assert_close(host(o2), oracle.norm_gate(y.numpy(), None, None, 0.5), "o ungated")


def test_slot_engine_cta_stats_account_for_every_event(sdm):
    """With per-CTA statistics on, the slot engine's CTAs together apply every event of the
    step exactly once (short segments plus long, hot-slot segments); with them off nothing is
    recorded.  Skewed halves make hot slots, so both kinds occur."""
    wl = sdm_synth.WORKLOADS["long_skew"].replace(T=4096, H=1, seed=41)
    g = device_inputs(wl)
    sdm.sdm_slot_cta_stats(reset=True)
    sdm.sdm_set_option("slot_cta_stats", 1)
    try:
        out, M = run_scan(sdm, wl, g, engine="slot", want_o=False)
    finally:
        sdm.sdm_set_option("slot_cta_stats", 0)
    st = sdm.sdm_slot_cta_stats(reset=True)
    events = wl.B * wl.T * wl.H * (wl.W + wl.R)
    assert int(st[:, 0].sum() + st[:, 1].sum()) == events
    assert st[:, 1].sum() > 0 and st[:, 2].sum() > 0 and st[:, 3].sum() > 0
    run_scan(sdm, wl, g, engine="slot", want_o=False)
    assert int(sdm.sdm_slot_cta_stats(reset=True).sum()) == 0


@pytest.mark.parametrize("schedule", ["serial", "pipelined"])
@pytest.mark.parametrize("dt", [BF16, F32])
def test_scan_slot_engine_over_several_chunks(sdm, dt, schedule):
    """Many wide (sequence, head) rows per token make the slot engine's time chunks short
    (here 128 tokens: 128 + 128 + 44), so the state carries over between chunks; the result
    is the oracle's all the same, with the whole selection first and with each chunk's
    selection pipelined beside the chunk before (bf16 rows take the fast selection, fp32 rows
    the general one; both select a chunk of all 8 sequences through a strided window)."""
    wl = sdm_synth.WORKLOADS["tiny"].replace(B=8, H=8, T=300, S1=16, S2=16, W=8, R=8,
                                            d_v=1024, in_dtype=dt, seed=61)
    g = device_inputs(wl)
    sdm.sdm_set_option("select_schedule", 1 if schedule == "serial" else 2)
    try:
        out, M = run_scan(sdm, wl, g, engine="slot")
    finally:
        sdm.sdm_set_option("select_schedule", 0)
    full_check(wl, g, out, M)


def test_pipelined_schedule_equals_serial_schedule(sdm):
    """Both schedules of the slot engine's selection on the long skewed shape at 1/32 of its
    tokens (4 time chunks): the same selections and final state bit for bit, y within
    rounding (reads are added with float atomics), and again on a second call that
    continues from the first call's state."""
    wl = sdm_synth.WORKLOADS["long_skew"].replace(T=32768)
    g = device_inputs(wl)
    res = {}
    for sched in (1, 2):
        M = torch.empty((wl.B, wl.H, wl.N, wl.d_v), dtype=F32, device=DEV)
        sdm.sdm_set_option("select_schedule", sched)
        try:
            out1, M = run_scan(sdm, wl, g, engine="slot", want_o=False, M=M)
            sel1, y1 = out1["sel"].clone(), out1["y"].clone()
            out2, M = run_scan(sdm, wl, g, engine="slot", want_o=False, M=M, init="continue")
        finally:
            sdm.sdm_set_option("select_schedule", 0)
        res[sched] = (sel1, y1, out2["sel"], out2["y"], M)
    a, b = res[1], res[2]
    assert torch.equal(a[0], b[0]) and torch.equal(a[2], b[2])
    assert torch.equal(a[4], b[4])
    for ya, yb in ((a[1], b[1]), (a[3], b[3])):
        assert_close(host(yb), host(ya).astype(np.float64), "y", atol=1e-5, rtol=1e-5)
