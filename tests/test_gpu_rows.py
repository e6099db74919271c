"""Parity of the checkpoint-row kernels (sdm_state_pack / sdm_state_unpack, through the C ABI)
with the CPU oracle of oracle/rows.py: codes and scales bit for bit, unpacked rows bit for
bit, on random rows of several widths and magnitudes, rows built to hit E4M3 and int4
rounding midpoints, zero and single-value rows, a ragged row count, and rows sampled from a
full-size (4 GB) state."""

import numpy as np
import pytest
import torch

import sdm_synth
from oracle import rows as R
from tests._parity import device_status_ok

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
FMTS = ["bf16", "e4m3", "int4"]


@pytest.fixture(scope="module")
def sdm():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import __graft_entry__
    __graft_entry__.build()
    import sparse_memory_linear_b200 as m
    torch.cuda.set_device(0)
    return m


def codes_np(codes, fmt):
    c = codes.cpu()
    return c.view(torch.int16).numpy().view(np.uint16) if fmt == "bf16" else c.numpy()


def check(sdm, M, fmt):
    d_v = M.shape[-1]
    codes, scales = sdm.sdm_state_pack(M.to(DEV), fmt)
    back = sdm.sdm_state_unpack(codes, scales, d_v, fmt)
    torch.cuda.synchronize()
    device_status_ok()
    ref_codes, ref_scales = R.pack(M.numpy().reshape(-1, d_v), fmt)
    np.testing.assert_array_equal(codes_np(codes, fmt), ref_codes, err_msg=f"{fmt} codes")
    if fmt != "bf16":
        np.testing.assert_array_equal(scales.cpu().numpy().view(np.uint32),
                                      ref_scales.view(np.uint32), err_msg=f"{fmt} scales")
    ref_back = R.unpack(ref_codes, ref_scales, fmt, d_v)
    np.testing.assert_array_equal(back.cpu().numpy().view(np.uint32), ref_back.view(np.uint32),
                                  err_msg=f"{fmt} unpacked")


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("rows,d_v", [(1, 4), (37, 64), (300, 256), (77, 512), (1000, 128),
                                      (5, 12)])
def test_random_rows(sdm, fmt, rows, d_v):
    g = torch.Generator().manual_seed(rows * 1000 + d_v)
    mag = 10.0 ** torch.randint(-6, 4, (rows, 1), generator=g).float()
    M = torch.randn(rows, d_v, generator=g) * mag
    check(sdm, M, fmt)


@pytest.mark.parametrize("fmt", FMTS)
def test_rounding_midpoints_zero_rows_and_single_values(sdm, fmt):
    """With amax = 448 (E4M3) or 7 (int4) the scale is 1 and x / s = x exactly, so rows of
    grid midpoints test ties to even; also all-zero rows, a single nonzero value, values that
    round to -0, and subnormal E4M3 codes."""
    grid = np.array([R.e4m3_value(c) for c in range(127)])
    mids = ((grid[:-1] + grid[1:]) / 2).astype(np.float32)  # exact in fp32
    rows = []
    for sign in (1, -1):
        r = np.zeros(128, np.float32)
        r[0] = 448.0
        r[1:127] = sign * mids
        r[127] = sign * 2.0 ** -12
        rows.append(r)
    r = np.zeros(128, np.float32)
    r[0] = 7.0
    r[1:15] = np.arange(-6.5, 7.0, 1.0, dtype=np.float32)  # int4 midpoints
    rows.append(r)
    rows.append(np.zeros(128, np.float32))
    r = np.zeros(128, np.float32)
    r[77] = -3.25
    rows.append(r)
    r = np.full(128, -1e-30, np.float32)
    r[5] = 1.0
    rows.append(r)
    check(sdm, torch.from_numpy(np.stack(rows)), fmt)


@pytest.mark.parametrize("fmt", ["e4m3", "int4"])
def test_full_size_state_sampled(sdm, fmt):
    """The long skewed layer's state (4 heads x 2^20 slots x 256, 4 GB) after a few hundred
    tokens of the pass: packed and unpacked on the GPU in full, 2000 sampled rows against the
    oracle bit for bit."""
    wl = sdm_synth.WORKLOADS["long_skew"].replace(T=256)
    g = {k: t.to(DEV) for k, t in sdm_synth.make_inputs(wl, device=DEV).items()}
    M = torch.empty((wl.B, wl.H, wl.N, wl.d_v), dtype=torch.float32, device=DEV)
    sdm.sdm_scan_forward(g["kp"], g["qp"], g["v"], g["alpha"], g["beta"], M, W=wl.W, R=wl.R,
                         S1=wl.S1, M0=g["M0"], init="m0", want_o=False)
    codes, scales = sdm.sdm_state_pack(M, fmt)
    back = sdm.sdm_state_unpack(codes, scales, wl.d_v, fmt)
    torch.cuda.synchronize()
    device_status_ok()
    rows = M.numel() // wl.d_v
    pick = torch.from_numpy(np.random.default_rng(3).choice(rows, 2000, replace=False))
    Mh = M.view(rows, wl.d_v)[pick.to(DEV)].cpu().numpy()
    ref_codes, ref_scales = R.pack(Mh, fmt)
    np.testing.assert_array_equal(codes[pick.to(DEV)].cpu().numpy(), ref_codes)
    np.testing.assert_array_equal(scales[pick.to(DEV)].cpu().numpy(), ref_scales)
    np.testing.assert_array_equal(back[pick.to(DEV)].cpu().numpy(),
                                  R.unpack(ref_codes, ref_scales, fmt, wl.d_v))


def test_zero_rows_is_a_no_op(sdm):
    M = torch.empty((0, 64), dtype=torch.float32, device=DEV)
    before = sdm.sdm_launch_count()
    codes, scales = sdm.sdm_state_pack(M, "e4m3")
    sdm.sdm_state_unpack(codes, scales, 64, "e4m3")
    assert sdm.sdm_launch_count() == before and codes.numel() == 0
