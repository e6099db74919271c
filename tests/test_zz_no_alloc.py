"""The prefill entry point that allocates nothing, through the C ABI.

sdm_scan_forward_noalloc serves callers that cannot allocate device memory while the pass
runs (an engine that owns all device memory in its own pool, a plugin interface without a
workspace argument, a loop that must not call the CUDA allocator once running): it takes
its scratch from a fixed device array inside the library.  Its results must equal those of
sdm_scan_forward with a caller workspace and those of the CPU oracle, call after call, even
though every call reuses the same array; and once the first call on the device has looked
up the array's address, a call must not change the memory the process holds on the device.
"""

import ctypes

import numpy as np
import pytest
import torch

import oracle
import sdm_synth
from tests._parity import THREADS, TOL_ABS, TOL_REL, assert_close, host

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import __graft_entry__
    __graft_entry__.build()
    import sparse_memory_linear_b200 as sdm
    torch.cuda.set_device(0)
    L = ctypes.CDLL(sdm.library_path)
    P, I, F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float
    L.sdm_scan_forward_noalloc.argtypes = [P, P, P, P, P, P, P, I, P, P, P, F, I, P, P,
                                           sdm.SdmShape, P]
    L.sdm_scan_forward_noalloc.restype = I
    return sdm, L


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def test_noalloc_equals_workspace_entry_point_twice(lib):
    sdm, L = lib
    wl = sdm_synth.WORKLOADS["small"].replace(T=1024, seed=77)
    g = {k: t.to(DEV) for k, t in sdm_synth.make_inputs(wl, with_gamma=True).items()}
    shape = sdm.shape_of(wl.B, wl.T, wl.H, wl.S1, wl.S2, wl.W, wl.R, wl.d_v, sdm.SDM_BF16)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)

    M_ref = torch.empty((wl.B, wl.H, wl.N, wl.d_v), dtype=torch.float32, device=DEV)
    ref = sdm.sdm_scan_forward(g["kp"], g["qp"], g["v"], g["alpha"], g["beta"], M_ref, W=wl.W,
                               R=wl.R, M0=g["M0"], gate=g["gate"], gamma=g["gamma"],
                               want_sel=True, engine="seq")
    torch.cuda.synchronize()

    for call in range(2):
        M = torch.full_like(M_ref, float("nan"))
        y = torch.full_like(ref["y"], float("nan"))
        o = torch.full_like(ref["o"], float("nan"))
        sel = torch.full_like(ref["sel"], -1)
        if call == 0:  # the C entry point itself
            rc = L.sdm_scan_forward_noalloc(
                _p(g["kp"]), _p(g["qp"]), _p(g["v"]), _p(g["alpha"]), _p(g["beta"]),
                _p(g["M0"]), _p(M), 0, _p(y), _p(g["gate"]), _p(g["gamma"]), 1e-6, 0, _p(o),
                _p(sel), shape, stream)
            assert rc == 0, sdm.sdm_status_string(rc)
        else:  # through the Python binding of the same name
            sdm.sdm_scan_forward_noalloc(g["kp"], g["qp"], g["v"], g["alpha"], g["beta"], M,
                                         W=wl.W, R=wl.R, M0=g["M0"], y=y, gate=g["gate"],
                                         gamma=g["gamma"], o=o, sel_out=sel)
        torch.cuda.synchronize()
        assert sdm.sdm_get_device_status() == 0
        assert torch.equal(sel, ref["sel"]), f"call {call}: selected slots differ"
        assert_close(y.cpu().numpy(), ref["y"].cpu().numpy(), f"call {call}: y",
                     atol=TOL_ABS, rtol=TOL_REL)
        assert_close(o.cpu().numpy(), ref["o"].cpu().numpy(), f"call {call}: o",
                     atol=TOL_ABS, rtol=TOL_REL)
        assert_close(M.cpu().numpy(), M_ref.cpu().numpy(), f"call {call}: M",
                     atol=TOL_ABS, rtol=TOL_REL)


def _noalloc(sdm, g, wl, M, y, o, sel):
    sdm.sdm_scan_forward_noalloc(g["kp"], g["qp"], g["v"], g["alpha"], g["beta"], M, W=wl.W,
                                 R=wl.R, M0=g["M0"], y=y, gate=g["gate"], gamma=g["gamma"],
                                 o=o, sel_out=sel)


def test_noalloc_matches_the_oracle_on_consecutive_calls(lib):
    """Two calls in a row (the second over the first one's scratch) against the oracle."""
    sdm, _ = lib
    wl = sdm_synth.WORKLOADS["small"].replace(T=192, seed=78)
    cpu = sdm_synth.make_inputs(wl, with_gamma=True)
    g = {k: t.to(DEV) for k, t in cpu.items()}
    ref = oracle.forward(host(cpu["kp"]), host(cpu["qp"]), host(cpu["v"]), host(cpu["alpha"]),
                         host(cpu["beta"]), host(cpu["M0"]), S1=wl.S1, W=wl.W, R=wl.R,
                         gate=host(cpu["gate"]), gamma=host(cpu["gamma"]), threads=THREADS)
    n = wl.B * wl.T * wl.H
    for call in range(2):
        M = torch.full((wl.B, wl.H, wl.N, wl.d_v), float("nan"), device=DEV)
        y = torch.full((wl.B, wl.T, wl.H, wl.d_v), float("nan"), device=DEV)
        o = torch.full_like(y, float("nan"))
        sel = torch.full((n * (wl.W + wl.R),), -1, dtype=torch.int32, device=DEV)
        _noalloc(sdm, g, wl, M, y, o, sel)
        torch.cuda.synchronize()
        assert sdm.sdm_get_device_status() == 0
        s = sel.cpu().numpy()
        np.testing.assert_array_equal(s[: n * wl.W].reshape(ref["idx_w"].shape), ref["idx_w"])
        np.testing.assert_array_equal(s[n * wl.W:].reshape(ref["idx_r"].shape), ref["idx_r"])
        assert_close(host(y), ref["y"], f"call {call}: y")
        assert_close(host(o), ref["o"], f"call {call}: o")
        assert_close(host(M), ref["M"], f"call {call}: M")


def test_noalloc_calls_hold_no_new_device_memory(lib):
    """After the first call on the device (which looks up the array's address), further
    calls leave torch's allocation count and the device's free memory where they were.
    (The free-memory check assumes no other process allocates on this GPU meanwhile.)"""
    sdm, _ = lib
    wl = sdm_synth.WORKLOADS["small"].replace(T=512, seed=79)
    g = {k: t.to(DEV) for k, t in sdm_synth.make_inputs(wl, with_gamma=True).items()}
    M = torch.empty((wl.B, wl.H, wl.N, wl.d_v), device=DEV)
    y = torch.empty((wl.B, wl.T, wl.H, wl.d_v), device=DEV)
    o = torch.empty_like(y)
    sel = torch.empty((wl.B * wl.T * wl.H * (wl.W + wl.R),), dtype=torch.int32, device=DEV)
    _noalloc(sdm, g, wl, M, y, o, sel)
    torch.cuda.synchronize()
    held = torch.cuda.memory_allocated()
    free0, _ = torch.cuda.mem_get_info()
    launches = sdm.sdm_launch_count()
    for _ in range(3):
        _noalloc(sdm, g, wl, M, y, o, sel)
    torch.cuda.synchronize()
    assert sdm.sdm_launch_count() > launches  # the calls did run
    assert torch.cuda.memory_allocated() == held
    free1, _ = torch.cuda.mem_get_info()
    assert free1 >= free0 - (1 << 20), (free0, free1)
    assert sdm.sdm_get_device_status() == 0
