"""The prefill entry point that allocates nothing, through the C ABI.

sdm_scan_forward_noalloc serves callers that cannot allocate device memory while the pass
runs (an engine that owns all device memory in its own pool, a plugin interface without a
workspace argument, a loop that must not call the CUDA allocator once running): it takes
its scratch from a fixed device array inside the library.  Its results must equal those of
sdm_scan_forward with a caller workspace, call after call, even though every call reuses
the same array.
"""

import ctypes

import numpy as np
import pytest
import torch

import sdm_synth
from tests._parity import TOL_ABS, TOL_REL, assert_close

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


def test_noalloc_rejects_shapes_beyond_its_scratch(lib):
    sdm, L = lib
    # 4 x 8192 x 8 rows with W = R = 64 need 128 MiB of scratch, beyond the fixed 16 MiB
    big = sdm.shape_of(4, 8192, 8, 512, 512, 64, 64, 128, sdm.SDM_BF16)
    assert sdm.sdm_workspace_size(big, "seq") > (16 << 20)
    fake = ctypes.c_void_p(0x10000)
    rc = L.sdm_scan_forward_noalloc(fake, fake, fake, fake, fake, ctypes.c_void_p(0x2000000000),
                                    fake, 0, fake, None, None, 1e-6, 0, None, None, big, None)
    assert rc == 1  # SDM_ERR_INVALID_ARG, nothing launched
    np.testing.assert_equal(sdm.sdm_get_device_status(), 0)
