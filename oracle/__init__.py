"""CPU oracle of the SDM memory pass -- TEST INFRASTRUCTURE.

Plain, slow, double-precision restatement of the four steps of Sparse Delta Memory
(selection, gated delta write, sparse read, RMSNorm + output gate), written in C
(``sdm_oracle.c``) and driven through ctypes.  Only the test-suite, the smoke check
and the benchmark's CPU-baseline leg may import this package; the product path never
does, and the oracle imports nothing from the product package.

Array conventions (all numpy, C-contiguous; half scores already widened to float32,
which is exact for bf16 inputs):

    kp, qp  [B, T, H, S1 + S2]   write / read score halves (k'_1 | k'_2)
    v       [B, T, H, d_v]
    alpha, beta [B, T, H]
    M_init  [H, N, d_v]  (the learnable M0, shared by every sequence)  or
            [B, H, N, d_v] (a state to continue from)
    gate    [B, T, H, d_v] or None;  gamma [d_v] or None
"""

from __future__ import annotations

import ctypes
import os
import subprocess
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sdm_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle_sdm.so")

ACT = {"silu": 0, "sigmoid": 1, "identity": 2}
_MODE = {"product_key": 0, "brute_force": 1}

_lib = None


def build(force: bool = False) -> str:
    """Compile sdm_oracle.c into liboracle_sdm.so (plain gcc, no FMA contraction)."""
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-std=c99", "-O2", "-fPIC", "-shared", "-ffp-contract=off",
               "-fno-fast-math", "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        L = ctypes.c_long
        I = ctypes.c_int
        lib.sdm_oracle_select.argtypes = [P, L, L, I, I, I, I, P, P, P]
        lib.sdm_oracle_select.restype = I
        lib.sdm_oracle_pass.argtypes = [I, I, I, I, I, P, P, P, P, P, L, P, P, L, I, P, P,
                                        P, P, P]
        lib.sdm_oracle_pass.restype = I
        lib.sdm_oracle_pass_coupled.argtypes = lib.sdm_oracle_pass.argtypes
        lib.sdm_oracle_pass_coupled.restype = I
        lib.sdm_oracle_pass_logged.argtypes = lib.sdm_oracle_pass.argtypes + [P]
        lib.sdm_oracle_pass_logged.restype = I
        lib.sdm_oracle_norm_gate.argtypes = [L, I, P, P, P, ctypes.c_double, I, P]
        lib.sdm_oracle_norm_gate.restype = I
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data


def select(halves, S1: int, K: int, mode: str = "product_key", return_scored: bool = False,
           threads: int = 1):
    """Top-K slot selection of every row of ``halves`` [..., S1+S2] (float32).

    Returns (idx int32 [..., K], wt float64 [..., K]) in selection order, and the
    number of candidate sums scored per row when ``return_scored``.  Rows are
    independent; ``threads`` splits them into that many chunks.
    """
    h = np.ascontiguousarray(halves, dtype=np.float32)
    S = h.shape[-1]
    S2 = S - S1
    rows = h.reshape(-1, S)
    n = rows.shape[0]
    idx = np.empty((n, K), np.int32)
    wt = np.empty((n, K), np.float64)
    scored = ctypes.c_long(0)
    lib = _load()

    def chunk(rng):
        r0, r1 = rng
        rc = lib.sdm_oracle_select(rows[r0:].ctypes.data, r1 - r0, S, S1, S2, K, _MODE[mode],
                                   idx[r0:].ctypes.data, wt[r0:].ctypes.data,
                                   ctypes.byref(scored))
        if rc != 0:
            raise ValueError(f"sdm_oracle_select failed ({rc})")

    nt = max(1, min(int(threads), n))
    bounds = [(n * i // nt, n * (i + 1) // nt) for i in range(nt)]
    if nt > 1:
        with ThreadPoolExecutor(nt) as ex:
            list(ex.map(chunk, bounds))
    elif n:
        chunk(bounds[0])
    out = (idx.reshape(h.shape[:-1] + (K,)), wt.reshape(h.shape[:-1] + (K,)))
    return out + (scored.value,) if return_scored else out


def norm_gate(y, g=None, gamma=None, eps: float = 1e-6, act: str | int = "silu"):
    """RMSNorm over the last axis, weight gamma, times act(g). Returns float64."""
    y64 = np.ascontiguousarray(y, dtype=np.float64)
    d_v = y64.shape[-1]
    g32 = None if g is None else np.ascontiguousarray(g, dtype=np.float32)
    gm = None if gamma is None else np.ascontiguousarray(gamma, dtype=np.float32)
    o = np.empty_like(y64)
    a = ACT[act] if isinstance(act, str) else int(act)
    rc = _load().sdm_oracle_norm_gate(y64.size // d_v, d_v, _ptr(y64), _ptr(g32), _ptr(gm),
                                      float(eps), a, _ptr(o))
    if rc != 0:
        raise ValueError(f"sdm_oracle_norm_gate failed ({rc})")
    return o


def run_unit(kp, qp, v, alpha, beta, M_init, b: int, h: int, *, S1: int, W: int, R: int,
             rows=None, want_y=None, t_end=None, select_mode: str = "product_key",
             threads: int = 1, selection=None, coupled: bool = False,
             want_log: bool = False):
    """Steps 1-3 for one (sequence b, head h) over tokens [0, t_end).

    want_log: also return "wlog" [t_end, W, d_v] float64, the undo log of the in-place
    update: written slot j of token t as the write found it (sdm_oracle_pass_logged; NaN for
    untracked rows).

    coupled: the coupled delta rule (one prediction shared by the token's written rows,
    sdm_oracle_pass_coupled) instead of the per-slot write; every written row must then be
    tracked.

    rows: tracked slot rows (int array) or None for all N rows.
    want_y: bool array [t_end] of tokens whose read result is wanted, or None (all).
    threads: token chunks of the selection (independent per token) run on this many
    threads.  selection: a previous result's (idx_w, wt_w, idx_r, wt_r) to reuse.
    Returns dict(idx_w, wt_w, idx_r, wt_r, y [t_end, d_v] float64 (NaN where unwanted),
    M [n_rows, d_v] float32, rows).
    """
    B, T, H, S = kp.shape
    S2 = S - S1
    N = S1 * S2
    d_v = v.shape[-1]
    t_end = T if t_end is None else int(t_end)
    lib = _load()

    def sel(x, K):
        idx = np.empty((t_end, K), np.int32)
        wt = np.empty((t_end, K), np.float64)
        xs = np.ascontiguousarray(x[b, :t_end, h, :], dtype=np.float32)

        def chunk(rng):
            t0, t1 = rng
            rc = lib.sdm_oracle_select(xs[t0:].ctypes.data, t1 - t0, S, S1, S2, K,
                                       _MODE[select_mode], idx[t0:].ctypes.data,
                                       wt[t0:].ctypes.data, None)
            if rc != 0:
                raise ValueError(f"sdm_oracle_select failed ({rc})")

        n = max(1, min(threads, t_end))
        bounds = [(t_end * i // n, t_end * (i + 1) // n) for i in range(n)]
        if n > 1:
            with ThreadPoolExecutor(n) as ex:
                list(ex.map(chunk, bounds))
        else:
            chunk(bounds[0])
        return idx, wt

    if selection is None:
        idx_w, wt_w = sel(kp, W)
        idx_r, wt_r = sel(qp, R)
    else:
        idx_w, wt_w, idx_r, wt_r = selection

    v_u = np.ascontiguousarray(v[b, :t_end, h, :], dtype=np.float32)
    a_u = np.ascontiguousarray(alpha[b, :t_end, h], dtype=np.float32)
    be_u = np.ascontiguousarray(beta[b, :t_end, h], dtype=np.float32)
    M_src = M_init[h] if M_init.ndim == 3 else M_init[b, h]
    if rows is None:
        rows_arr = None
        n_rows = N
        M_in = np.ascontiguousarray(M_src, dtype=np.float32)
    else:
        rows_arr = np.ascontiguousarray(np.asarray(rows, dtype=np.int32))
        n_rows = rows_arr.size
        M_in = np.ascontiguousarray(M_src[rows_arr], dtype=np.float32)
    wy = None if want_y is None else np.ascontiguousarray(want_y, dtype=np.uint8)
    y = np.full((t_end, d_v), np.nan, np.float64)
    M_out = np.empty((n_rows, d_v), np.float32)
    args = (t_end, N, d_v, W, R, _ptr(idx_w), _ptr(wt_w), _ptr(idx_r), _ptr(wt_r), _ptr(v_u),
            d_v, _ptr(a_u), _ptr(be_u), 1, n_rows, _ptr(rows_arr), _ptr(M_in), _ptr(wy),
            _ptr(y), _ptr(M_out))
    wlog = None
    if want_log:
        if coupled:
            raise ValueError("the undo log is kept for the per-slot rule")
        wlog = np.empty((t_end, W, d_v), np.float64)
        rc = lib.sdm_oracle_pass_logged(*args, _ptr(wlog))
    else:
        rc = (lib.sdm_oracle_pass_coupled if coupled else lib.sdm_oracle_pass)(*args)
    if rc != 0:
        raise ValueError(f"sdm_oracle_pass failed ({rc})")
    out = dict(idx_w=idx_w, wt_w=wt_w, idx_r=idx_r, wt_r=wt_r, y=y, M=M_out, rows=rows_arr)
    if want_log:
        out["wlog"] = wlog
    return out


def forward(kp, qp, v, alpha, beta, M_init, *, S1: int, W: int, R: int, gate=None,
            gamma=None, eps: float = 1e-6, act="silu", select_mode: str = "product_key",
            threads: int = 1, coupled: bool = False, want_log: bool = False):
    """The whole pass over every (b, h) and every token, all rows tracked.

    Returns dict(idx_w [B,T,H,W], idx_r [B,T,H,R], wt_w, wt_r, y [B,T,H,d_v] float64,
    o [B,T,H,d_v] float64, M [B,H,N,d_v] float32), and with want_log the undo log
    wlog [B,T,H,W,d_v] float64 (run_unit).
    """
    B, T, H, S = kp.shape
    N = S1 * (S - S1)
    d_v = v.shape[-1]
    idx_w = np.empty((B, T, H, W), np.int32)
    idx_r = np.empty((B, T, H, R), np.int32)
    wt_w = np.empty((B, T, H, W), np.float64)
    wt_r = np.empty((B, T, H, R), np.float64)
    y = np.empty((B, T, H, d_v), np.float64)
    M = np.empty((B, H, N, d_v), np.float32)
    wlog = np.empty((B, T, H, W, d_v), np.float64) if want_log else None
    units = [(b, h) for b in range(B) for h in range(H)]

    def one(u):
        b, h = u
        r = run_unit(kp, qp, v, alpha, beta, M_init, b, h, S1=S1, W=W, R=R,
                     select_mode=select_mode, coupled=coupled, want_log=want_log)
        if want_log:
            wlog[b, :, h] = r["wlog"]
        idx_w[b, :, h], wt_w[b, :, h] = r["idx_w"], r["wt_w"]
        idx_r[b, :, h], wt_r[b, :, h] = r["idx_r"], r["wt_r"]
        y[b, :, h] = r["y"]
        M[b, h] = r["M"]

    if threads > 1:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(one, units))
    else:
        for u in units:
            one(u)
    g = None if gate is None else np.asarray(gate, dtype=np.float32)
    o = norm_gate(y, g, gamma, eps, act)
    out = dict(idx_w=idx_w, idx_r=idx_r, wt_w=wt_w, wt_r=wt_r, y=y, o=o, M=M)
    if want_log:
        out["wlog"] = wlog
    return out


def undo(M, idx_w, wlog):
    """Undoes a pass's in-place writes [m.163.com article on SDM, section 八, the
    memory-efficiency paragraph]: replays the undo log backwards, from the last token to the
    first, putting back each written row as its write found it.

    M [B,H,N,d_v] the state after the pass; idx_w [B,T,H,W]; wlog [B,T,H,W,d_v].  Returns the
    restored state (float64).
    """
    out = np.array(M, dtype=np.float64, copy=True)
    B, T, H, W = idx_w.shape
    for b in range(B):
        for h in range(H):
            for t in range(T - 1, -1, -1):
                for j in range(W):
                    out[b, h, idx_w[b, t, h, j]] = wlog[b, t, h, j]
    return out
