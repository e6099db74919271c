"""The C ABI without a GPU: the library loads, exports every entry point the header
declares, sizes its scratch, and rejects bad arguments on the host before any launch.

The rejection tests pass made-up device addresses, which validation turns down before any
launch; every one also checks that the library's launch counter did not move.  They run
only where no CUDA device is visible, so that a regression in validation could never put a
kernel on such an address.  The host code they exercise is the same on a GPU machine."""

import ctypes
import os
import re

import pytest
import torch

host_only = pytest.mark.skipif(torch.cuda.is_available(),
                               reason="made-up device addresses are passed only without a GPU")

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def sdm():
    from sparse_memory_linear_b200.build import build_library
    build_library()
    import sparse_memory_linear_b200 as m
    m.library()
    return m


def declared_functions():
    src = open(os.path.join(ROOT, "include", "sdm.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(sdm_\w+)\s*\(", src)))


def test_exports_every_declared_symbol(sdm):
    names = declared_functions()
    assert "sdm_scan_forward" in names and "sdm_decode_step" in names
    lib = ctypes.CDLL(sdm.library_path)
    for n in names:
        assert hasattr(lib, n), n


def declared_parameter_counts():
    src = open(os.path.join(ROOT, "include", "sdm.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    out = {}
    for name, params in re.findall(r"\b(sdm_\w+)\s*\(([^)]*)\)\s*;", src):
        params = params.strip()
        out[name] = 0 if params in ("", "void") else params.count(",") + 1
    return out


def test_binding_has_every_declared_call_with_its_signature(sdm):
    """Each call of the header has a Python function of the same name, and the ctypes
    prototype the binding gives it has the header's number of parameters."""
    import sparse_memory_linear_b200 as pkg
    counts = declared_parameter_counts()
    assert set(counts) == set(declared_functions())
    lib = sdm.library()
    for name, n in counts.items():
        assert callable(getattr(pkg, name, None)), name
        assert len(getattr(lib, name).argtypes) == n, name


def test_library_is_the_in_tree_build(sdm):
    sdm.library()
    maps = open("/proc/self/maps").read()
    assert sdm.library_path in maps


def good_shape(sdm, **kw):
    d = dict(B=2, T=16, H=3, S1=32, S2=32, W=8, R=8, d_v=64, in_dtype=sdm.SDM_BF16)
    d.update(kw)
    return sdm.shape_of(**d)


def test_workspace_size(sdm):
    s = good_shape(sdm, W=6, R=8)
    rows = 2 * 16 * 3
    # four regions (idx and weights of writes and reads), rows padded to 4 entries
    def r256(x):
        return (x + 255) // 256 * 256
    want = r256(rows * 8 * 4) * 2 + r256(rows * 8 * 4) * 2
    assert sdm.sdm_workspace_size(s, "seq") == want
    # the slot engine adds double-buffered events (12 B each), the radix histogram and the
    # chunk offsets; AUTO reserves room for either engine
    events = rows * (6 + 8)
    slot = sdm.sdm_workspace_size(s, "slot")
    assert slot >= want + 2 * events * 12
    assert sdm.sdm_workspace_size(s) == slot
    assert sdm.sdm_workspace_size(good_shape(sdm, W=40)) == 0  # W > S
    assert sdm.sdm_workspace_size(good_shape(sdm, d_v=12)) == 0  # bf16 needs d_v % 8 == 0
    # the chunk-wise engine keeps only the selections, as the sequential one
    assert sdm.sdm_workspace_size(s, "chunk") == want
    assert sdm.library().sdm_workspace_size(s, 4) == 0  # no such engine


FAKE = 0x10000  # aligned, never dereferenced: validation rejects the call first


class no_launch:
    """Asserts that the library launched no kernel inside the block."""

    def __init__(self, sdm):
        self.sdm = sdm

    def __enter__(self):
        self.n = self.sdm.sdm_launch_count()

    def __exit__(self, *exc):
        assert self.sdm.sdm_launch_count() == self.n, "a rejected call launched a kernel"


def scan(sdm, shape, **over):
    with no_launch(sdm):
        return _scan(sdm, shape, **over)


def _scan(sdm, shape, **over):
    args = dict(kp=FAKE, qp=FAKE, v=FAKE, alpha=FAKE, beta=FAKE, M0=FAKE + 0x100000000,
                M=FAKE, init=0, y=FAKE, gate=None, gamma=None, eps=1e-6, act=0, o=None,
                sel=None, engine=0, ws=FAKE, ws_bytes=1 << 40)
    args.update(over)
    P = ctypes.c_void_p
    return sdm.library().sdm_scan_forward(
        P(args["kp"]), P(args["qp"]), P(args["v"]), P(args["alpha"]), P(args["beta"]),
        P(args["M0"]), P(args["M"]), args["init"], P(args["y"]), P(args["gate"]),
        P(args["gamma"]), args["eps"], args["act"], P(args["o"]), P(args["sel"]),
        args["engine"], P(args["ws"]), args["ws_bytes"], shape, None)


@host_only
@pytest.mark.parametrize("bad", [
    dict(kp=None), dict(qp=None), dict(v=None), dict(alpha=None), dict(beta=None),
    dict(M=None), dict(y=None), dict(ws=None), dict(M0=None),
    dict(kp=FAKE + 4), dict(M=FAKE + 8), dict(ws=FAKE + 16), dict(gate=FAKE + 2),
    dict(ws_bytes=16), dict(init=7), dict(engine=9), dict(act=3), dict(eps=-1.0),
    dict(M0=FAKE),  # M0 overlaps M
])
def test_scan_rejects_bad_arguments(sdm, bad):
    assert scan(sdm, good_shape(sdm), **bad) == 1


@host_only
@pytest.mark.parametrize("kw", [
    dict(W=0), dict(R=0), dict(W=33), dict(R=40), dict(S1=0), dict(S2=5000), dict(B=0),
    dict(H=0), dict(T=-1), dict(d_v=12), dict(d_v=0), dict(d_v=2048), dict(in_dtype=5),
    dict(S1=256, S2=256, W=129, R=8),
])
def test_scan_rejects_bad_shapes(sdm, kw):
    assert scan(sdm, good_shape(sdm, **kw)) == 1


@host_only
def test_decode_and_select_and_norm_reject_bad_arguments(sdm):
    with no_launch(sdm):
        _decode_select_norm_reject(sdm)


def _decode_select_norm_reject(sdm):
    lib = sdm.library()
    P = ctypes.c_void_p
    s = good_shape(sdm)
    # decode, plain and chained: missing M, then misaligned v
    for fn in (lib.sdm_decode_step, lib.sdm_decode_step_chained):
        assert fn(P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE), None, P(FAKE),
                  None, None, 1e-6, 0, None, None, s, None) == 1
        assert fn(P(FAKE), P(FAKE), P(FAKE + 4), P(FAKE), P(FAKE), P(FAKE),
                  P(FAKE), None, None, 1e-6, 0, None, None, s, None) == 1
    # select: K out of range, null output
    assert lib.sdm_select(P(FAKE), s, 0, P(FAKE), P(FAKE), None) == 1
    assert lib.sdm_select(P(FAKE), s, 33, P(FAKE), P(FAKE), None) == 1
    assert lib.sdm_select(P(FAKE), s, 8, None, P(FAKE), None) == 1
    # norm: bad activation, null y
    assert lib.sdm_norm_gate(P(FAKE), None, None, 1e-6, 5, s, P(FAKE), None) == 1
    assert lib.sdm_norm_gate(None, None, None, 1e-6, 0, s, P(FAKE), None) == 1
    # state init: overlapping M and M0
    assert lib.sdm_state_init(P(FAKE), P(FAKE), s, None) == 1


def test_state_rows_bytes(sdm):
    assert sdm.sdm_state_rows_bytes(1000, 256, "bf16") == 512000
    assert sdm.sdm_state_rows_bytes(1000, 256, "e4m3") == 256000
    assert sdm.sdm_state_rows_bytes(1000, 256, "int4") == 128000
    assert sdm.sdm_state_rows_bytes(0, 4, "int4") == 0
    lib = sdm.library()
    for rows, d_v, fmt in ((-1, 64, 2), (10, 2, 2), (10, 6, 2), (10, 516, 3), (10, 64, 0),
                           (10, 64, 4)):
        assert lib.sdm_state_rows_bytes(rows, d_v, fmt) == 0


@host_only
def test_state_pack_and_unpack_reject_bad_arguments(sdm):
    """Unknown format, d_v out of range, missing or misaligned buffers, a missing scale
    array, overlapping buffers: SDM_ERR_INVALID_ARG before any launch; rows = 0 is a no-op."""
    lib = sdm.library()
    P = ctypes.c_void_p
    big = FAKE + (1 << 30)
    with no_launch(sdm):
        for fn, args in ((lib.sdm_state_pack, lambda M, r, d, f, c, s: (M, r, d, f, c, s, None)),
                         (lib.sdm_state_unpack, lambda M, r, d, f, c, s: (c, s, r, d, f, M, None))):
            assert fn(*args(P(FAKE), 8, 64, 0, P(big), P(big * 2))) == 1      # format
            assert fn(*args(P(FAKE), 8, 66, 2, P(big), P(big * 2))) == 1      # d_v % 4
            assert fn(*args(P(FAKE), 8, 1024, 2, P(big), P(big * 2))) == 1    # d_v > 512
            assert fn(*args(None, 8, 64, 2, P(big), P(big * 2))) == 1         # no M
            assert fn(*args(P(FAKE), 8, 64, 2, None, P(big * 2))) == 1        # no codes
            assert fn(*args(P(FAKE), 8, 64, 2, P(big + 4), P(big * 2))) == 1  # misaligned
            assert fn(*args(P(FAKE), 8, 64, 3, P(big), None)) == 1            # no scales
            assert fn(*args(P(FAKE), 8, 64, 2, P(FAKE + 256), P(big * 2))) == 1  # overlap
            assert fn(*args(P(FAKE), -1, 64, 2, P(big), P(big * 2))) == 1     # rows < 0
            assert fn(*args(None, 0, 64, 2, None, None)) == 0                 # nothing to do


@host_only
def test_logged_pass_and_undo_reject_bad_arguments(sdm):
    """The logged prefill needs its log (16-byte aligned, apart from M and y); the undo needs
    M, the write slots, the log and a large enough aligned workspace, none overlapping."""
    lib = sdm.library()
    P = ctypes.c_void_p
    s = good_shape(sdm)  # B2 T16 H3 S32x32 W8 R8 d_v64
    GB = 1 << 30
    M, y, wlog, ws = FAKE, FAKE + GB, FAKE + 2 * GB, FAKE + 4 * GB
    need = sdm.sdm_workspace_size(s, "auto")
    with no_launch(sdm):
        def logged(wl, ys=y):
            return lib.sdm_scan_forward_logged(
                P(FAKE + 8 * GB), P(FAKE + 9 * GB), P(FAKE + 10 * GB), P(FAKE + 11 * GB),
                P(FAKE + 12 * GB), None, P(M), 1, P(ys), None, None, 1e-6, 0, None, None, 0,
                P(ws), need, s, wl, None)
        assert logged(None) == 1                      # no log
        assert logged(P(wlog + 4)) == 1               # misaligned log
        assert logged(P(M + 4096)) == 1               # log over M
        assert logged(P(y)) == 1                      # log over y
        need_u = lib.sdm_undo_workspace_size(s)
        assert need_u == 2 * 3 * 1024 * 4
        sel = FAKE + 6 * GB
        undo = lib.sdm_state_undo
        assert undo(None, P(sel), P(wlog), s, P(ws), need_u, None) == 1
        assert undo(P(M), None, P(wlog), s, P(ws), need_u, None) == 1
        assert undo(P(M), P(sel), None, s, P(ws), need_u, None) == 1
        assert undo(P(M), P(sel), P(wlog), s, P(ws), need_u - 1, None) == 1   # small ws
        assert undo(P(M), P(sel), P(wlog), s, P(ws + 16), need_u, None) == 1  # ws alignment
        assert undo(P(M), P(sel), P(M + 256), s, P(ws), need_u, None) == 1    # log over M
        assert undo(P(M), P(sel), P(wlog), s, P(wlog + 64), need_u, None) == 1  # ws over log
        t0 = sdm.shape_of(2, 0, 3, 32, 32, 8, 8, 64, sdm.SDM_BF16)
        assert undo(None, None, None, t0, None, 0, None) == 0                 # T = 0: nothing


@host_only
def test_noalloc_rejects_shapes_beyond_its_scratch(sdm):
    """4 x 8192 x 8 rows with W = R = 64 need 128 MiB of scratch, beyond the fixed 16 MiB
    of sdm_scan_forward_noalloc: SDM_ERR_INVALID_ARG before any CUDA call or launch."""
    lib = sdm.library()
    big = sdm.shape_of(4, 8192, 8, 512, 512, 64, 64, 128, sdm.SDM_BF16)
    assert sdm.sdm_workspace_size(big, "seq") > (16 << 20)
    ok = sdm.shape_of(1, 1024, 8, 512, 512, 64, 64, 128, sdm.SDM_BF16)
    assert sdm.sdm_workspace_size(ok, "seq") <= (16 << 20)
    P = ctypes.c_void_p
    with no_launch(sdm):
        rc = lib.sdm_scan_forward_noalloc(P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE),
                                          P(FAKE + 0x100000000), P(FAKE), 0, P(FAKE), None,
                                          None, 1e-6, 0, None, None, big, None)
    assert rc == 1


def test_options_are_explicit_and_validated(sdm):
    """Launch options come only from sdm_set_option: unknown options and values out of
    range are refused and change nothing; every option reads back and resets to 0."""
    lib = sdm.library()
    for name, code in sdm.OPTION.items():
        assert sdm.sdm_get_option(name) == 0
    good = {"no_pdl": 1, "select_general": 1, "select_ctas_per_sm": 3, "slot_ctas_per_sm": 2,
            "seq_columns": 16, "seq_depth": 8, "slot_cta_stats": 1, "select_schedule": 2}
    bad = {"no_pdl": 2, "select_general": -1, "select_ctas_per_sm": 65,
           "slot_ctas_per_sm": -2, "seq_columns": 12, "seq_depth": 5, "slot_cta_stats": 3,
           "select_schedule": 3}
    try:
        for name in sdm.OPTION:
            assert lib.sdm_set_option(sdm.OPTION[name], bad[name]) == 1
            assert sdm.sdm_get_option(name) == 0
            sdm.sdm_set_option(name, good[name])
            assert sdm.sdm_get_option(name) == good[name]
    finally:
        for name in sdm.OPTION:
            sdm.sdm_set_option(name, 0)
    assert lib.sdm_set_option(0, 0) == 1 and lib.sdm_set_option(99, 0) == 1
    assert lib.sdm_slot_cta_stats(None, 4, 0) == 1  # no output buffer: refused before any CUDA call
    assert lib.sdm_get_option(0) == -1 and lib.sdm_get_option(99) == -1
    csrc = os.path.join(ROOT, "sparse_memory_linear_b200", "csrc")
    for f in os.listdir(csrc):
        assert "getenv" not in open(os.path.join(csrc, f)).read(), f"{f} reads the environment"


@host_only
def test_coupled_prefill_refuses_the_slot_engine_before_any_launch(sdm):
    lib = sdm.library()
    P = ctypes.c_void_p
    with no_launch(sdm):
        rc = lib.sdm_scan_forward_coupled(P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE),
                                          P(FAKE + 0x100000000), P(FAKE), 0, P(FAKE), None,
                                          None, 1e-6, 0, None, None, 2, P(FAKE), 1 << 40,
                                          good_shape(sdm), None)
    assert rc == 2  # SDM_ERR_UNSUPPORTED


@host_only
def test_chunk_engine_refuses_the_coupled_rule_and_the_undo_log(sdm):
    """The chunk-wise engine computes the per-slot rule and keeps no log: the coupled and the
    logged prefill refuse it (SDM_ERR_UNSUPPORTED) before any launch; an unknown engine is an
    invalid argument."""
    lib = sdm.library()
    P = ctypes.c_void_p
    s = good_shape(sdm)
    GB = 1 << 30
    need = sdm.sdm_workspace_size(s, "chunk")
    args = (P(FAKE), P(FAKE + GB), P(FAKE + 2 * GB), P(FAKE + 3 * GB), P(FAKE + 4 * GB), None,
            P(FAKE + 5 * GB), 1, P(FAKE + 6 * GB), None, None, 1e-6, 0, None, None)
    with no_launch(sdm):
        assert lib.sdm_scan_forward_coupled(*args, 3, P(FAKE + 8 * GB), need, s, None) == 2
        assert lib.sdm_scan_forward_logged(*args, 3, P(FAKE + 8 * GB), need, s,
                                           P(FAKE + 16 * GB), None) == 2
        assert lib.sdm_scan_forward(*args, 4, P(FAKE + 8 * GB), need, s, None) == 1


def test_status_strings(sdm):
    assert sdm.sdm_status_string(0) == "SDM_OK"
    assert sdm.sdm_status_string(4) == "SDM_ERR_DEVICE_CHECK"
    assert sdm.sdm_status_string(99) == "SDM_ERR_UNKNOWN"


def test_missing_library_raises_instead_of_falling_back(monkeypatch, tmp_path):
    """Without the built library every call raises: there is no CPU or torch fallback."""
    import sparse_memory_linear_b200._binding as B
    monkeypatch.setattr(B, "_lib", None)
    monkeypatch.setattr(B, "library_path", str(tmp_path / "libsdm.so"))
    with pytest.raises(RuntimeError, match="missing"):
        B.library()


C_PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "sdm.h"

int main(void) {
    sdm_shape s = {2, 16, 3, 32, 32, 8, 8, 64, SDM_BF16};
    if (sdm_workspace_size(s, SDM_ENGINE_SEQ) == 0) return 1;
    sdm_shape bad = s;
    bad.W = 40;  /* beyond S1 */
    if (sdm_workspace_size(bad, SDM_ENGINE_AUTO) != 0) return 2;
    int32_t idx[8];
    float wt[8];
    /* validation rejects these before anything touches a pointer or the GPU */
    if (sdm_select((const void *)0x10000, s, 0, idx, wt, NULL) != SDM_ERR_INVALID_ARG) return 3;
    if (sdm_decode_step((const void *)0x10000, (const void *)0x10000, (const void *)0x10000,
                        (const float *)0x10000, (const float *)0x10000, NULL,
                        (float *)0x10000, NULL, NULL, 1e-6f, SDM_GATE_SILU, NULL, NULL, s,
                        NULL) != SDM_ERR_INVALID_ARG) return 4;
    if (strcmp(sdm_status_string(SDM_ERR_INVALID_ARG), "SDM_ERR_INVALID_ARG") != 0) return 5;
    printf("ok\n");
    return 0;
}
"""


@host_only
def test_plain_c_program_builds_links_and_calls_the_abi(sdm, tmp_path):
    """The boundary is usable from C alone: a C99 program including sdm.h links against
    libsdm.so and calls it (host-side calls only), and the header also parses as C++."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    src = tmp_path / "use_sdm.c"
    src.write_text(C_PROGRAM)
    libdir = os.path.dirname(sdm.library_path)
    exe = tmp_path / "use_sdm"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I",
                    os.path.join(ROOT, "include"), str(src), "-L", libdir, "-lsdm",
                    f"-Wl,-rpath,{libdir}", "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0 and out.stdout.strip() == "ok", (out.returncode, out.stderr)
    if shutil.which("g++"):
        subprocess.run(["g++", "-std=c++17", "-fsyntax-only", "-x", "c++", "-I",
                        os.path.join(ROOT, "include"), str(src)], check=True)


def test_binding_refuses_tensors_that_do_not_match_the_call(sdm):
    """The C ABI sees bare pointers, so the binding checks every tensor against the shape
    of the call before anything reaches the library.  The first case is a decode run's
    step-major stack [T, B, H, S] passed as a prefill's [B, T, H, S] with a state sized for
    B sequences: the library would read it as T sequences and run off the end of the state."""
    f = torch.float32
    B, T, H, S1, d_v, W = 4, 16, 2, 16, 8, 4
    N = S1 * S1
    kp = torch.zeros(T, B, H, 2 * S1)
    good = dict(qp=kp, v=torch.zeros(T, B, H, d_v), alpha=torch.zeros(T, B, H),
                beta=torch.zeros(T, B, H))
    with no_launch(sdm), pytest.raises(ValueError, match=r"M has shape"):
        sdm.sdm_scan_forward(kp, good["qp"], good["v"], good["alpha"], good["beta"],
                             torch.zeros(B, H, N, d_v), W=W, R=W)
    kp = torch.zeros(B, T, H, 2 * S1)
    args = dict(qp=kp, v=torch.zeros(B, T, H, d_v), alpha=torch.zeros(B, T, H),
                beta=torch.zeros(B, T, H), M=torch.zeros(B, H, N, d_v))
    bad = [("qp", torch.zeros(B, T, H, 2 * S1 + 2)), ("v", torch.zeros(B, T, H + 1, d_v)),
           ("alpha", torch.zeros(B, T)), ("beta", torch.zeros(B, T, H, 1)),
           ("M", torch.zeros(B, H, N + 1, d_v))]
    for name, t in bad:
        a = dict(args)
        a[name] = t
        with no_launch(sdm), pytest.raises(ValueError, match=name):
            sdm.sdm_scan_forward(kp, a["qp"], a["v"], a["alpha"], a["beta"], a["M"], W=W, R=W)
    for kw in (dict(y=torch.zeros(B, T, H, d_v + 1)), dict(o=torch.zeros(1)),
               dict(M0=torch.zeros(H + 1, N, d_v)), dict(gate=torch.zeros(B, T, H, 2)),
               dict(gamma=torch.zeros(d_v + 1)), dict(sel_out=torch.zeros(3, dtype=torch.int32))):
        with no_launch(sdm), pytest.raises(ValueError, match="shape|elements"):
            sdm.sdm_scan_forward(kp, args["qp"], args["v"], args["alpha"], args["beta"],
                                 args["M"], W=W, R=W, **kw)
    # consistent shapes get as far as the device check (no GPU tensors here)
    with no_launch(sdm), pytest.raises(ValueError, match="CUDA"):
        sdm.sdm_scan_forward(kp, args["qp"], args["v"], args["alpha"], args["beta"], args["M"],
                             W=W, R=W)
    # decode, state init, selection and norm/gate
    dk = torch.zeros(B, H, 2 * S1)
    with no_launch(sdm), pytest.raises(ValueError, match="M has shape"):
        sdm.sdm_decode_step(dk, dk, torch.zeros(B, H, d_v), torch.zeros(B, H), torch.zeros(B, H),
                            torch.zeros(2 * B, H, N, d_v), W=W, R=W)
    with no_launch(sdm), pytest.raises(ValueError, match="M0 has shape"):
        sdm.sdm_state_init(torch.zeros(H, N, 2 * d_v), torch.zeros(B, H, N, d_v))
    with no_launch(sdm), pytest.raises(ValueError, match="idx has shape"):
        sdm.sdm_select(torch.zeros(5, 2 * S1), W, idx=torch.zeros(5, W + 1, dtype=torch.int32))
    with no_launch(sdm), pytest.raises(ValueError, match="o has shape"):
        sdm.sdm_norm_gate(torch.zeros(5, d_v, dtype=f), o=torch.zeros(5, d_v + 4))
