"""The coupled delta rule on the GPU against the oracle's coupled mode.

The SDM write-up on ai-paper-analysis.pages.dev and the m.163.com article state that SDM
reduces exactly to the gated delta rule when every slot is selected; that holds when the
token's written rows share one prediction p = sum_j k_j alpha M[j] and each becomes
alpha M[i] + beta k_i (v - p) (sdm_scan_forward_coupled, sdm_decode_step_coupled).  The
oracle's coupled mode is pinned against the dense gated delta recurrence
(tests/test_oracle_pins.py); here the sequential engine and the decode kernel must match it:
slots bit for bit, y, o and the state within |d| <= 2e-4 + 1e-3 |ref|.
"""

import numpy as np
import pytest
import torch

import oracle
import sdm_synth
from tests._parity import THREADS, assert_close, device_status_ok, host, sel_views

pytestmark = pytest.mark.gpu

F32, BF16 = torch.float32, torch.bfloat16
DEV = "cuda:0"


@pytest.fixture(scope="module")
def sdm():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import __graft_entry__
    __graft_entry__.build()
    import sparse_memory_linear_b200 as m
    torch.cuda.set_device(0)
    return m


def inputs(wl, **kw):
    return {k: t.to(DEV) for k, t in sdm_synth.make_inputs(wl, **kw).items()}


def ref_forward(wl, g, gamma=None, M_init=None):
    f = host
    return oracle.forward(f(g["kp"]), f(g["qp"]), f(g["v"]), f(g["alpha"]), f(g["beta"]),
                          f(g["M0"]) if M_init is None else M_init, S1=wl.S1, W=wl.W, R=wl.R,
                          gate=None if g.get("gate") is None else f(g["gate"]),
                          gamma=None if gamma is None else f(gamma), threads=THREADS,
                          coupled=True)


SHAPES = [
    dict(),                                                                    # tiny, fp32
    dict(B=2, H=3, T=37, S1=24, S2=40, W=5, R=11, d_v=16),                     # ragged, W != R
    dict(B=2, H=2, T=120, S1=64, S2=64, W=16, R=16, d_v=32, in_dtype=BF16),    # bf16
    dict(B=1, H=2, T=50, S1=64, S2=64, W=64, R=48, d_v=8, in_dtype=BF16),      # W = S
    dict(B=3, H=1, T=40, S1=32, S2=32, W=8, R=8, d_v=4),                       # d_v = 4
    dict(B=1, H=1, T=33, S1=128, S2=128, W=128, R=128, d_v=64, in_dtype=BF16),  # K = 128
]


@pytest.mark.parametrize("kw", SHAPES)
@pytest.mark.parametrize("engine", ["auto", "seq"])
def test_scan_coupled_matches_oracle(sdm, kw, engine):
    wl = sdm_synth.WORKLOADS["tiny"].replace(**kw, seed=200 + len(kw) + (kw.get("T", 0)))
    g = inputs(wl, with_gamma=True)
    M = torch.empty((wl.B, wl.H, wl.N, wl.d_v), dtype=F32, device=DEV)
    out = sdm.sdm_scan_forward_coupled(g["kp"], g["qp"], g["v"], g["alpha"], g["beta"], M,
                                       W=wl.W, R=wl.R, S1=wl.S1, M0=g["M0"], gate=g["gate"],
                                       gamma=g["gamma"], want_sel=True, engine=engine)
    torch.cuda.synchronize()
    device_status_ok()
    ref = ref_forward(wl, g, g["gamma"])
    sw, sr = sel_views(out["sel"], wl.B, wl.T, wl.H, wl.W, wl.R)
    np.testing.assert_array_equal(sw.cpu().numpy(), ref["idx_w"])
    np.testing.assert_array_equal(sr.cpu().numpy(), ref["idx_r"])
    assert_close(host(out["y"]), ref["y"], "y")
    assert_close(host(out["o"]), ref["o"], "o")
    assert_close(host(M), ref["M"], "final M")


def test_scan_coupled_continue_and_small_workload(sdm):
    """The small workload in two calls (SDM_CONTINUE) against one oracle pass."""
    wl = sdm_synth.WORKLOADS["small"].replace(T=256, seed=211)
    g = inputs(wl)
    M = torch.empty((wl.B, wl.H, wl.N, wl.d_v), dtype=F32, device=DEV)
    half = wl.T // 2
    parts = []
    for t0, t1, init in ((0, half, "m0"), (half, wl.T, "continue")):
        sl = {k: (t[:, t0:t1].contiguous() if k != "M0" else t) for k, t in g.items()}
        parts.append(sdm.sdm_scan_forward_coupled(sl["kp"], sl["qp"], sl["v"], sl["alpha"],
                                                  sl["beta"], M, W=wl.W, R=wl.R, S1=wl.S1,
                                                  M0=g["M0"], init=init, gate=sl["gate"]))
    torch.cuda.synchronize()
    device_status_ok()
    ref = ref_forward(wl, g)
    y = torch.cat([p["y"] for p in parts], 1)
    assert_close(host(y), ref["y"], "y")
    assert_close(host(M), ref["M"], "final M")


def test_slot_engine_refuses_the_coupled_rule(sdm):
    wl = sdm_synth.WORKLOADS["tiny"]
    g = inputs(wl)
    M = torch.empty((wl.B, wl.H, wl.N, wl.d_v), dtype=F32, device=DEV)
    n = sdm.sdm_launch_count()
    with pytest.raises(sdm.SdmError) as e:
        sdm.sdm_scan_forward_coupled(g["kp"], g["qp"], g["v"], g["alpha"], g["beta"], M,
                                     W=wl.W, R=wl.R, M0=g["M0"], engine="slot")
    assert e.value.status == 2 and sdm.sdm_launch_count() == n


def decode_run(sdm, wl, steps, M, chained=False):
    ys, os_, sels = [], [], []
    for s in steps:
        d = {k: t.to(DEV) for k, t in s.items() if k != "M0"}
        out = sdm.sdm_decode_step(d["kp"], d["qp"], d["v"], d["alpha"], d["beta"], M, W=wl.W,
                                  R=wl.R, S1=wl.S1, gate=d["gate"], want_sel=True,
                                  chained=chained, coupled=True)
        ys.append(out["y"].clone())
        os_.append(out["o"].clone())
        sels.append(out["sel"].clone())
    torch.cuda.synchronize()
    device_status_ok()
    return torch.stack(ys, 1), torch.stack(os_, 1), sels


@pytest.mark.parametrize("kw", [
    dict(B=8, H=2, T=6, S1=128, S2=128, W=32, R=32, d_v=64),                         # group path
    dict(B=4, H=2, T=5, S1=512, S2=512, W=64, R=64, d_v=128),                        # bench shape
    dict(B=4, H=2, T=5, S1=16, S2=16, W=8, R=8, d_v=16, in_dtype=F32),               # warp path
    dict(B=2, H=2, T=4, S1=1024, S2=1024, W=128, R=96, d_v=128),                     # K = 128
])
def test_decode_coupled_matches_oracle(sdm, kw):
    wl = sdm_synth.WORKLOADS["decode"].replace(**kw, seed=230 + kw["S1"])
    steps = [sdm_synth.make_inputs(wl, step=s) for s in range(wl.T)]
    M0 = steps[0]["M0"].to(DEV)
    M = M0.unsqueeze(0).expand(wl.B, -1, -1, -1).contiguous()
    y, o, sels = decode_run(sdm, wl, steps, M)
    st = {k: torch.stack([s[k] for s in steps], 1) for k in steps[0] if k != "M0"}
    ref = oracle.forward(host(st["kp"]), host(st["qp"]), host(st["v"]), host(st["alpha"]),
                         host(st["beta"]), host(steps[0]["M0"]), S1=wl.S1, W=wl.W, R=wl.R,
                         gate=host(st["gate"]), threads=THREADS, coupled=True)
    for t, sel in enumerate(sels):
        s = sel.cpu().numpy()
        n = wl.B * wl.H
        np.testing.assert_array_equal(s[: n * wl.W].reshape(wl.B, wl.H, wl.W), ref["idx_w"][:, t])
        np.testing.assert_array_equal(s[n * wl.W:].reshape(wl.B, wl.H, wl.R), ref["idx_r"][:, t])
    assert_close(host(y), ref["y"], "y")
    assert_close(host(o), ref["o"], "o")
    assert_close(host(M), ref["M"], "final M")


def test_decode_coupled_equals_scan_and_chained_equals_plain(sdm):
    wl = sdm_synth.WORKLOADS["decode"].replace(B=4, H=2, T=12, S1=128, S2=128, seed=241)
    steps = [sdm_synth.make_inputs(wl, step=s) for s in range(wl.T)]
    M0 = steps[0]["M0"].to(DEV)
    Mp = M0.unsqueeze(0).expand(wl.B, -1, -1, -1).contiguous()
    Mc = Mp.clone()
    y_p, o_p, sel_p = decode_run(sdm, wl, steps, Mp)
    y_c, o_c, sel_c = decode_run(sdm, wl, steps, Mc, chained=True)
    for a, b in zip(sel_p, sel_c):
        assert torch.equal(a, b)
    assert torch.equal(y_p, y_c) and torch.equal(o_p, o_c) and torch.equal(Mp, Mc)
    g = {k: torch.stack([s[k] for s in steps], 1).to(DEV) for k in steps[0] if k != "M0"}
    Ms = torch.empty_like(Mp)
    out = sdm.sdm_scan_forward_coupled(g["kp"], g["qp"], g["v"], g["alpha"], g["beta"], Ms,
                                       W=wl.W, R=wl.R, S1=wl.S1, M0=M0, gate=g["gate"])
    torch.cuda.synchronize()
    assert_close(host(y_p), host(out["y"]), "decode vs scan y", atol=1e-6, rtol=1e-5)
    assert_close(host(Mp), host(Ms), "decode vs scan M", atol=1e-6, rtol=1e-5)


def test_decode_coupled_refuses_rows_beyond_shared_memory(sdm):
    """W * d_v * 4 > 64 KB: the coupled step would need its write rows in registers."""
    wl = sdm_synth.WORKLOADS["decode"].replace(B=1, H=1, T=1, S1=128, S2=128, W=64, R=8,
                                               d_v=512, seed=251)
    s = {k: t.to(DEV) for k, t in sdm_synth.make_inputs(wl, step=0).items()}
    M = s["M0"].unsqueeze(0).contiguous()
    n = sdm.sdm_launch_count()
    with pytest.raises(sdm.SdmError) as e:
        sdm.sdm_decode_step_coupled(s["kp"], s["qp"], s["v"], s["alpha"], s["beta"], M,
                                    W=wl.W, R=wl.R, S1=wl.S1, gate=s["gate"])
    assert e.value.status == 2 and sdm.sdm_launch_count() == n
