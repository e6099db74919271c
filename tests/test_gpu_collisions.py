"""Selection parity on rows whose fp32 candidate sums round onto one another.

The method's selection ("Sparse Delta Memory: Scaling the State of Linear RNNs through
Sparsity", paper.rainbus.top summary, method step 1; ai-paper-analysis.pages.dev SDM
write-up, 步骤 1) takes the top K of each score half, then the top K of the K*K candidate
sums.  The kernels score only the rank pairs (r1+1)(r2+1) <= K and must still return the
route's slots when rounding merges unequal sums (a tiny half score vanishing in its sum, or
near-equal scores next to a large one).  These rows are built to hit that case
(tests/test_selection_bounds.py::collision_rows); every selection kernel is compared with
the oracle's product-key route bit for bit: the bf16 register path, the general path (fp32
halves, halves longer than 1024), both prefill engines and both decode selections.
"""

import json
import os

import numpy as np
import pytest
import torch

import oracle
from tests._parity import (THREADS, WT_ABS, WT_REL, assert_close, device_status_ok, host,
                           sel_views)
from tests.test_selection_bounds import COLLISION_KINDS, collision_rows

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


def collision_matrix(n, S1, S2, K, dt, seed):
    """n score rows cycling through the collision kinds, as a CPU tensor of dtype dt."""
    rng = np.random.default_rng(seed)
    rows = [np.concatenate(collision_rows(rng, S1, S2, K, COLLISION_KINDS[i % 4], dt == BF16))
            for i in range(n)]
    return torch.from_numpy(np.stack(rows).astype(np.float32)).to(dt)


SELECT_CASES = [
    (16, 16, 8, F32), (16, 16, 8, BF16), (24, 40, 8, BF16), (256, 256, 64, BF16),
    (256, 256, 64, F32), (128, 128, 128, BF16), (200, 136, 128, F32), (1024, 1024, 64, BF16),
    (1024, 1024, 128, BF16), (2048, 2048, 64, BF16),
]


@pytest.mark.parametrize("S1,S2,K,dt", SELECT_CASES)
def test_select_collisions_match_oracle(sdm, S1, S2, K, dt):
    x = collision_matrix(96, S1, S2, K, dt, S1 * 3 + S2 + K)
    idx, wt = sdm.sdm_select(x.to(DEV), K, S1=S1)
    torch.cuda.synchronize()
    device_status_ok()
    ref_idx, ref_wt = oracle.select(host(x), S1, K, threads=THREADS)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref_idx)
    assert_close(wt.cpu().numpy(), ref_wt, "weights", atol=WT_ABS, rtol=WT_REL)


def test_select_hand_derived_collisions(sdm):
    """tests/golden/route_collisions.json: the route's slots, never the pruning-only ones."""
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "route_collisions.json")))
    for c in g["cases"]:
        row = torch.tensor([c["a"] + c["b"]], dtype=F32)
        dts = [F32] + ([BF16] if torch.equal(row.to(BF16).float(), row) else [])
        for dt in dts:
            idx, wt = sdm.sdm_select(row.to(dt).to(DEV), c["K"], S1=len(c["a"]))
            np.testing.assert_array_equal(idx.cpu().numpy()[0], c["expect_route"])
            assert_close(wt.cpu().numpy()[0], c["expect_wt"], "weights", atol=WT_ABS, rtol=WT_REL)


def scan_inputs(B, T, H, S1, S2, K, d_v, dt, seed):
    rng = np.random.default_rng(seed)
    S = S1 + S2
    kp = collision_matrix(B * T * H, S1, S2, K, dt, seed + 1).view(B, T, H, S)
    qp = collision_matrix(B * T * H, S1, S2, K, dt, seed + 2).view(B, T, H, S)
    f = lambda a: torch.from_numpy(np.asarray(a, np.float32))
    return dict(kp=kp, qp=qp,
                v=f(rng.standard_normal((B, T, H, d_v))).to(dt),
                gate=f(rng.standard_normal((B, T, H, d_v))).to(dt),
                alpha=f(rng.uniform(0.3, 1.0, (B, T, H))),
                beta=f(rng.uniform(0.0, 1.0, (B, T, H))),
                M0=f(0.02 * rng.standard_normal((H, S1 * S2, d_v))))


def oracle_forward(g, S1, W, R):
    return oracle.forward(host(g["kp"]), host(g["qp"]), host(g["v"]), host(g["alpha"]),
                          host(g["beta"]), host(g["M0"]), S1=S1, W=W, R=R,
                          gate=host(g["gate"]), threads=THREADS)


@pytest.mark.parametrize("engine", ["seq", "slot"])
@pytest.mark.parametrize("S1,S2,K,dt", [(16, 16, 8, F32), (256, 256, 64, BF16),
                                        (128, 128, 128, BF16)])
def test_scan_collisions_match_oracle(sdm, engine, S1, S2, K, dt):
    B, T, H, d_v = 2, 24, 2, 16
    g = scan_inputs(B, T, H, S1, S2, K, d_v, dt, S1 + K)
    d = {k: t.to(DEV) for k, t in g.items()}
    M = torch.empty((B, H, S1 * S2, d_v), dtype=F32, device=DEV)
    out = sdm.sdm_scan_forward(d["kp"], d["qp"], d["v"], d["alpha"], d["beta"], M, W=K, R=K,
                               S1=S1, M0=d["M0"], gate=d["gate"], want_sel=True, engine=engine)
    torch.cuda.synchronize()
    device_status_ok()
    ref = oracle_forward(g, S1, K, K)
    sw, sr = sel_views(out["sel"], B, T, H, K, K)
    np.testing.assert_array_equal(sw.cpu().numpy(), ref["idx_w"], err_msg="write slots")
    np.testing.assert_array_equal(sr.cpu().numpy(), ref["idx_r"], err_msg="read slots")
    assert_close(host(out["y"]), ref["y"], "y")
    assert_close(host(out["o"]), ref["o"], "o")
    assert_close(host(M), ref["M"], "final M")


@pytest.mark.parametrize("S1,S2,K,dt", [(16, 16, 8, F32), (256, 256, 64, BF16),
                                        (512, 512, 64, BF16), (1024, 1024, 128, BF16)])
def test_decode_collisions_match_oracle(sdm, S1, S2, K, dt):
    """bf16 halves of up to 1024 take the group selection, fp32 halves the warp path."""
    B, H, d_v = 8, 2, 32
    g = scan_inputs(B, 1, H, S1, S2, K, d_v, dt, 3 * S1 + K)
    d = {k: t.to(DEV) for k, t in g.items()}
    M = torch.empty((B, H, S1 * S2, d_v), dtype=F32, device=DEV)
    sdm.sdm_state_init(d["M0"], M)
    out = sdm.sdm_decode_step(d["kp"][:, 0], d["qp"][:, 0], d["v"][:, 0], d["alpha"][:, 0],
                              d["beta"][:, 0], M, W=K, R=K, S1=S1, gate=d["gate"][:, 0],
                              want_sel=True)
    torch.cuda.synchronize()
    device_status_ok()
    ref = oracle_forward(g, S1, K, K)
    sel = out["sel"].cpu().numpy()
    np.testing.assert_array_equal(sel[: B * H * K].reshape(B, H, K), ref["idx_w"][:, 0],
                                  err_msg="write slots")
    np.testing.assert_array_equal(sel[B * H * K:].reshape(B, H, K), ref["idx_r"][:, 0],
                                  err_msg="read slots")
    assert_close(host(out["y"]), ref["y"][:, 0], "y")
    assert_close(host(out["o"]), ref["o"][:, 0], "o")
    assert_close(host(M), ref["M"], "final M")
