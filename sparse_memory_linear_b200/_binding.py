"""ctypes binding of libsdm.so (C ABI in include/sdm.h): argument marshalling only."""

from __future__ import annotations

import ctypes
import math
import os

import torch

SDM_F32, SDM_BF16 = 0, 1
ENGINE = {"auto": 0, "seq": 1, "slot": 2, "chunk": 3}
INIT = {"m0": 0, "continue": 1}
ACT = {"silu": 0, "sigmoid": 1, "identity": 2}
_STATUS = {0: "SDM_OK", 1: "SDM_ERR_INVALID_ARG", 2: "SDM_ERR_UNSUPPORTED", 3: "SDM_ERR_CUDA",
           4: "SDM_ERR_DEVICE_CHECK", 5: "SDM_ERR_TIMEOUT"}

_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "libsdm.so")


class SdmShape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("B", "T", "H", "S1", "S2", "W", "R", "d_v",
                                               "in_dtype")]

    def __repr__(self):
        return "SdmShape(" + ", ".join(f"{n}={getattr(self, n)}" for n, _ in self._fields_) + ")"


class SdmError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = int(status)
        super().__init__(f"{what}: {_STATUS.get(self.status, self.status)}")


_lib = None


def library():
    """The loaded libsdm.so.  Raises if it has not been built: there is no other path."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(library_path):
        raise RuntimeError(
            f"{library_path} is missing; build it with "
            "`python -c 'import __graft_entry__ as g; g.build()'` (nvcc, sm_100a)")
    lib = ctypes.CDLL(library_path)
    P, I, F, Z = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
    S = SdmShape
    sig = {
        "sdm_select": ([P, S, I, P, P, P], I),
        "sdm_workspace_size": ([S, I], Z),
        "sdm_state_init": ([P, P, S, P], I),
        "sdm_scan_forward": ([P, P, P, P, P, P, P, I, P, P, P, F, I, P, P, I, P, Z, S, P], I),
        "sdm_decode_step": ([P, P, P, P, P, P, P, P, P, F, I, P, P, S, P], I),
        "sdm_decode_step_chained": ([P, P, P, P, P, P, P, P, P, F, I, P, P, S, P], I),
        "sdm_decode_step_coupled": ([P, P, P, P, P, P, P, P, P, F, I, P, P, S, P], I),
        "sdm_decode_step_coupled_chained": ([P, P, P, P, P, P, P, P, P, F, I, P, P, S, P], I),
        "sdm_scan_forward_coupled": ([P, P, P, P, P, P, P, I, P, P, P, F, I, P, P, I, P, Z, S, P],
                                     I),
        "sdm_scan_forward_noalloc": ([P, P, P, P, P, P, P, I, P, P, P, F, I, P, P, S, P], I),
        "sdm_scan_forward_logged": ([P, P, P, P, P, P, P, I, P, P, P, F, I, P, P, I, P, Z, S, P,
                                     P], I),
        "sdm_undo_workspace_size": ([S], Z),
        "sdm_state_undo": ([P, P, P, S, P, Z, P], I),
        "sdm_norm_gate": ([P, P, P, F, I, S, P, P], I),
        "sdm_get_device_status": ([P], I),
        "sdm_status_string": ([I], ctypes.c_char_p),
        "sdm_profile_enable": ([I], I),
        "sdm_profile_read": ([P, P], I),
        "sdm_launch_count": ([], ctypes.c_uint64),
        "sdm_set_option": ([I, I], I),
        "sdm_get_option": ([I], I),
        "sdm_slot_cta_stats": ([P, I, I], I),
        "sdm_state_rows_bytes": ([ctypes.c_int64, I, I], Z),
        "sdm_state_pack": ([P, ctypes.c_int64, I, I, P, P, P], I),
        "sdm_state_unpack": ([P, P, ctypes.c_int64, I, I, P, P], I),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    _lib = lib
    return lib


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream, device=None):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _check(rc: int, what: str):
    if rc != 0:
        raise SdmError(rc, what)


def _in_dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return SDM_BF16
    if t.dtype == torch.float32:
        return SDM_F32
    raise TypeError(f"inputs must be bfloat16 or float32, got {t.dtype}")


def _need(t, name, dtype=None, device=None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    return t


def _expect(t, name, shape=None, numel=None):
    """Raises ValueError unless tensor t (None passes) has this shape or element count.
    The C ABI receives bare pointers and cannot see buffer sizes, so every tensor is
    checked against the call's shape here, before any pointer reaches the library."""
    if t is None:
        return
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if numel is not None and t.numel() != numel:
        raise ValueError(f"{name} has {t.numel()} elements, expected {numel}")


def shape_of(B, T, H, S1, S2, W, R, d_v, in_dtype) -> SdmShape:
    return SdmShape(int(B), int(T), int(H), int(S1), int(S2), int(W), int(R), int(d_v),
                    int(in_dtype))


def sdm_status_string(status: int) -> str:
    return library().sdm_status_string(int(status)).decode()


def sdm_workspace_size(shape: SdmShape, engine: str = "auto") -> int:
    return int(library().sdm_workspace_size(shape, ENGINE[engine]))


def sdm_select(halves: torch.Tensor, K: int, *, S1: int | None = None, idx=None, wt=None,
               stream=None):
    """Top-K product-key selection of every row of ``halves`` [..., S1+S2].
    Returns (idx int32 [..., K], wt float32 [..., K])."""
    S = halves.shape[-1]
    S1 = S // 2 if S1 is None else int(S1)
    rows = halves.numel() // S if S else 0
    lead = tuple(halves.shape[:-1])
    _expect(idx, "idx", lead + (K,))
    _expect(wt, "wt", lead + (K,))
    _need(halves, "halves")
    idx = torch.empty(lead + (K,), dtype=torch.int32, device=halves.device) if idx is None else idx
    wt = torch.empty(lead + (K,), dtype=torch.float32, device=halves.device) if wt is None else wt
    _need(idx, "idx", torch.int32, halves.device)
    _need(wt, "wt", torch.float32, halves.device)
    shape = shape_of(rows, 1, 1, S1, S - S1, 1, 1, 8, _in_dtype(halves))
    _check(library().sdm_select(_p(halves), shape, int(K), _p(idx), _p(wt),
                                _stream(stream, halves.device)), "sdm_select")
    return idx, wt


def sdm_state_init(M0: torch.Tensor, M: torch.Tensor, *, d_v: int | None = None, stream=None):
    """M[b, h] = M0[h] for every b.  M0 [H, N, d_v], M [B, H, N, d_v] float32."""
    if M.dim() != 4:
        raise ValueError(f"M has shape {tuple(M.shape)}, expected [B, H, N, d_v]")
    B, H, N, dv = M.shape
    _expect(M0, "M0", (H, N, dv))
    _need(M0, "M0", torch.float32)
    _need(M, "M", torch.float32, M0.device)
    shape = shape_of(B, 1, H, 1, N, 1, 1, dv, SDM_F32)
    _check(library().sdm_state_init(_p(M0), _p(M), shape, _stream(stream, M.device)),
           "sdm_state_init")
    return M


def _scan_outputs(kp, qp, v, alpha, beta, M, W, R, S1, M0, y, gate, gamma, o, want_o,
                  sel_out, want_sel):
    """Checks the prefill arguments and allocates the missing outputs; returns
    (shape, y, o, sel_out)."""
    dev = kp.device
    if kp.dim() != 4:
        raise ValueError(f"kp has shape {tuple(kp.shape)}, expected [B, T, H, S1 + S2]")
    B, T, H, S = kp.shape
    S1 = S // 2 if S1 is None else int(S1)
    d_v = v.shape[-1]
    N = S1 * (S - S1)
    for t, name, shp in ((qp, "qp", (B, T, H, S)), (v, "v", (B, T, H, d_v)),
                         (gate, "gate", (B, T, H, d_v)), (alpha, "alpha", (B, T, H)),
                         (beta, "beta", (B, T, H)), (M, "M", (B, H, N, d_v)),
                         (M0, "M0", (H, N, d_v)), (gamma, "gamma", (d_v,)),
                         (y, "y", (B, T, H, d_v)), (o, "o", (B, T, H, d_v))):
        _expect(t, name, shp)
    _expect(sel_out, "sel_out", numel=B * T * H * (W + R))
    _need(kp, "kp", device=dev)
    dt = kp.dtype
    _need(qp, "qp", dt, dev)
    _need(v, "v", dt, dev)
    _need(gate, "gate", dt, dev)
    _need(alpha, "alpha", torch.float32, dev)
    _need(beta, "beta", torch.float32, dev)
    _need(M, "M", torch.float32, dev)
    _need(M0, "M0", torch.float32, dev)
    _need(gamma, "gamma", torch.float32, dev)
    shape = shape_of(B, T, H, S1, S - S1, W, R, d_v, _in_dtype(kp))
    if y is None:
        y = torch.empty((B, T, H, d_v), dtype=torch.float32, device=dev)
    if o is None and want_o:
        o = torch.empty((B, T, H, d_v), dtype=torch.float32, device=dev)
    if sel_out is None and want_sel:
        sel_out = torch.empty(B * T * H * (W + R), dtype=torch.int32, device=dev)
    _need(y, "y", torch.float32, dev)
    _need(o, "o", torch.float32, dev)
    _need(sel_out, "sel_out", torch.int32, dev)
    return shape, y, o, sel_out


def sdm_scan_forward(kp, qp, v, alpha, beta, M, *, W: int, R: int, S1: int | None = None,
                     M0=None, init: str = "m0", y=None, gate=None, gamma=None,
                     eps: float = 1e-6, act: str = "silu", o=None, want_o: bool = True,
                     sel_out=None, want_sel: bool = False, engine: str = "auto", ws=None,
                     stream=None, coupled: bool = False):
    """Prefill over T tokens.  kp, qp [B,T,H,S1+S2]; v, gate [B,T,H,d_v]; alpha, beta
    [B,T,H]; M [B,H,N,d_v] (in/out); M0 [H,N,d_v] (init="m0").  coupled=True calls
    sdm_scan_forward_coupled (the coupled delta rule).
    Returns dict(y, o, sel): sel holds [B,T,H,W] write slots then [B,T,H,R] read slots."""
    dev = kp.device
    shape, y, o, sel_out = _scan_outputs(kp, qp, v, alpha, beta, M, W, R, S1, M0, y, gate,
                                         gamma, o, want_o, sel_out, want_sel)
    need = sdm_workspace_size(shape, engine)
    if ws is None:
        ws = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    _need(ws, "ws", torch.uint8, dev)
    name = "sdm_scan_forward_coupled" if coupled else "sdm_scan_forward"
    _check(getattr(library(), name)(
        _p(kp), _p(qp), _p(v), _p(alpha), _p(beta), _p(M0), _p(M), INIT[init], _p(y), _p(gate),
        _p(gamma), float(eps), ACT[act], _p(o), _p(sel_out), ENGINE[engine], _p(ws),
        ws.numel(), shape, _stream(stream, dev)), name)
    return dict(y=y, o=o, sel=sel_out)


def sdm_scan_forward_coupled(kp, qp, v, alpha, beta, M, **kw):
    """sdm_scan_forward(..., coupled=True): the token's written rows share one prediction."""
    return sdm_scan_forward(kp, qp, v, alpha, beta, M, coupled=True, **kw)


def sdm_scan_forward_logged(kp, qp, v, alpha, beta, M, *, W: int, R: int, S1: int | None = None,
                            M0=None, init: str = "m0", y=None, gate=None, gamma=None,
                            eps: float = 1e-6, act: str = "silu", o=None, want_o: bool = True,
                            sel_out=None, engine: str = "auto", ws=None, wlog=None,
                            stream=None):
    """sdm_scan_forward that also keeps the undo log of its in-place writes: returns
    dict(y, o, sel, wlog) with wlog [B,T,H,W,d_v] fp32, written row j of token (b, t, h) as
    its write found it; sel (the write slots, then the read slots) is always returned, since
    sdm_state_undo needs it."""
    dev = kp.device
    shape, y, o, sel_out = _scan_outputs(kp, qp, v, alpha, beta, M, W, R, S1, M0, y, gate,
                                         gamma, o, want_o, sel_out, True)
    B, T, H = kp.shape[:3]
    d_v = v.shape[-1]
    _expect(wlog, "wlog", (B, T, H, W, d_v))
    if wlog is None:
        wlog = torch.empty((B, T, H, W, d_v), dtype=torch.float32, device=dev)
    _need(wlog, "wlog", torch.float32, dev)
    need = sdm_workspace_size(shape, engine)
    if ws is None:
        ws = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    _need(ws, "ws", torch.uint8, dev)
    _check(library().sdm_scan_forward_logged(
        _p(kp), _p(qp), _p(v), _p(alpha), _p(beta), _p(M0), _p(M), INIT[init], _p(y), _p(gate),
        _p(gamma), float(eps), ACT[act], _p(o), _p(sel_out), ENGINE[engine], _p(ws),
        ws.numel(), shape, _p(wlog), _stream(stream, dev)), "sdm_scan_forward_logged")
    return dict(y=y, o=o, sel=sel_out, wlog=wlog)


def sdm_undo_workspace_size(shape: SdmShape) -> int:
    return int(library().sdm_undo_workspace_size(shape))


def sdm_state_undo(M, sel, wlog, *, W: int, S1: int | None = None, ws=None, stream=None):
    """Undoes a logged pass in place: M [B,H,N,d_v] gets back, for every slot the pass wrote,
    the row its first write found.  sel: the pass's sel output (its first B*T*H*W entries
    are the write slots); wlog [B,T,H,W,d_v] its undo log."""
    if M.dim() != 4 or wlog.dim() != 5:
        raise ValueError("M must be [B, H, N, d_v] and wlog [B, T, H, W, d_v]")
    B, H, N, d_v = M.shape
    _, T, _, _, _ = wlog.shape
    _expect(wlog, "wlog", (B, T, H, W, d_v))
    if sel.numel() < B * T * H * W:
        raise ValueError(f"sel has {sel.numel()} entries, fewer than the {B * T * H * W} "
                         "write slots of the pass")
    S1 = int(math.isqrt(N)) if S1 is None else int(S1)
    if S1 < 1 or N % S1:
        raise ValueError(f"S1 = {S1} does not divide N = {N}")
    dev = M.device
    _need(M, "M", torch.float32, dev)
    _need(sel, "sel", torch.int32, dev)
    _need(wlog, "wlog", torch.float32, dev)
    shape = shape_of(B, T, H, S1, N // S1, W, W, d_v, SDM_F32)
    need = sdm_undo_workspace_size(shape)
    if ws is None:
        ws = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    _need(ws, "ws", torch.uint8, dev)
    _check(library().sdm_state_undo(_p(M), _p(sel), _p(wlog), shape, _p(ws), ws.numel(),
                                    _stream(stream, dev)), "sdm_state_undo")
    return M


def sdm_scan_forward_noalloc(kp, qp, v, alpha, beta, M, *, W: int, R: int,
                             S1: int | None = None, M0=None, init: str = "m0", y=None,
                             gate=None, gamma=None, eps: float = 1e-6, act: str = "silu",
                             o=None, want_o: bool = True, sel_out=None, want_sel: bool = False,
                             stream=None):
    """sdm_scan_forward with the sequential engine and the library's own fixed scratch array
    instead of a workspace (no device allocation by the library; at most 16384 rows of
    (sequence, token, head) with W = R = 64).  Outputs that are not given are allocated
    here, before the call."""
    dev = kp.device
    shape, y, o, sel_out = _scan_outputs(kp, qp, v, alpha, beta, M, W, R, S1, M0, y, gate,
                                         gamma, o, want_o, sel_out, want_sel)
    _check(library().sdm_scan_forward_noalloc(
        _p(kp), _p(qp), _p(v), _p(alpha), _p(beta), _p(M0), _p(M), INIT[init], _p(y), _p(gate),
        _p(gamma), float(eps), ACT[act], _p(o), _p(sel_out), shape, _stream(stream, dev)),
        "sdm_scan_forward_noalloc")
    return dict(y=y, o=o, sel=sel_out)


def sdm_decode_step(kp, qp, v, alpha, beta, M, *, W: int, R: int, S1: int | None = None,
                    y=None, gate=None, gamma=None, eps: float = 1e-6, act: str = "silu", o=None,
                    want_o: bool = True, sel_out=None, want_sel: bool = False, stream=None,
                    chained: bool = False, coupled: bool = False):
    """One token for each (b, h).  kp, qp [B,H,S1+S2]; v, gate [B,H,d_v]; alpha, beta [B,H];
    M [B,H,N,d_v] in/out.  Returns dict(y, o, sel).  chained=True calls
    sdm_decode_step_chained: only when the kernel launched right before on the stream writes
    none of this step's inputs (a chain of steps over inputs already on the device)."""
    dev = kp.device
    if kp.dim() != 3:
        raise ValueError(f"kp has shape {tuple(kp.shape)}, expected [B, H, S1 + S2]")
    B, H, S = kp.shape
    S1 = S // 2 if S1 is None else int(S1)
    d_v = v.shape[-1]
    N = S1 * (S - S1)
    for t, name, shp in ((qp, "qp", (B, H, S)), (v, "v", (B, H, d_v)), (gate, "gate", (B, H, d_v)),
                         (alpha, "alpha", (B, H)), (beta, "beta", (B, H)),
                         (M, "M", (B, H, N, d_v)), (gamma, "gamma", (d_v,)),
                         (y, "y", (B, H, d_v)), (o, "o", (B, H, d_v))):
        _expect(t, name, shp)
    _expect(sel_out, "sel_out", numel=B * H * (W + R))
    _need(kp, "kp", device=dev)
    dt = kp.dtype
    _need(qp, "qp", dt, dev)
    _need(v, "v", dt, dev)
    _need(gate, "gate", dt, dev)
    _need(alpha, "alpha", torch.float32, dev)
    _need(beta, "beta", torch.float32, dev)
    _need(M, "M", torch.float32, dev)
    _need(gamma, "gamma", torch.float32, dev)
    shape = shape_of(B, 1, H, S1, S - S1, W, R, d_v, _in_dtype(kp))
    if y is None:
        y = torch.empty((B, H, d_v), dtype=torch.float32, device=dev)
    if o is None and want_o:
        o = torch.empty((B, H, d_v), dtype=torch.float32, device=dev)
    if sel_out is None and want_sel:
        sel_out = torch.empty(B * H * (W + R), dtype=torch.int32, device=dev)
    name = "sdm_decode_step" + ("_coupled" if coupled else "") + ("_chained" if chained else "")
    _check(getattr(library(), name)(
        _p(kp), _p(qp), _p(v), _p(alpha), _p(beta), _p(M), _p(y), _p(gate), _p(gamma),
        float(eps), ACT[act], _p(o), _p(sel_out), shape, _stream(stream, dev)), name)
    return dict(y=y, o=o, sel=sel_out)


def sdm_decode_step_coupled(kp, qp, v, alpha, beta, M, **kw):
    """sdm_decode_step(..., coupled=True): one step of the coupled delta rule."""
    return sdm_decode_step(kp, qp, v, alpha, beta, M, coupled=True, **kw)


def sdm_decode_step_coupled_chained(kp, qp, v, alpha, beta, M, **kw):
    """sdm_decode_step(..., coupled=True, chained=True)."""
    return sdm_decode_step(kp, qp, v, alpha, beta, M, coupled=True, chained=True, **kw)


def sdm_decode_step_chained(kp, qp, v, alpha, beta, M, **kw):
    """sdm_decode_step(..., chained=True): the launch may overlap the kernel ahead of it,
    which must write none of this step's inputs."""
    return sdm_decode_step(kp, qp, v, alpha, beta, M, chained=True, **kw)


def sdm_norm_gate(y, *, gate=None, gamma=None, eps: float = 1e-6, act: str = "silu", o=None,
                  stream=None):
    """o = y * rsqrt(mean(y^2) + eps) * gamma * act(gate) over the last axis of y."""
    d_v = y.shape[-1]
    _expect(gate, "gate", tuple(y.shape))
    _expect(o, "o", tuple(y.shape))
    _expect(gamma, "gamma", (d_v,))
    _need(y, "y", torch.float32)
    _need(gate, "gate", device=y.device)
    _need(gamma, "gamma", torch.float32, y.device)
    rows = y.numel() // d_v
    o = torch.empty_like(y) if o is None else o
    _need(o, "o", torch.float32, y.device)
    dt = _in_dtype(gate) if gate is not None else SDM_F32
    shape = shape_of(rows, 1, 1, 1, 1, 1, 1, d_v, dt)
    _check(library().sdm_norm_gate(_p(y), _p(gate), _p(gamma), float(eps), ACT[act], shape,
                                   _p(o), _stream(stream, y.device)), "sdm_norm_gate")
    return o


ROW_FORMAT = {"bf16": 1, "e4m3": 2, "int4": 3}


def _row_codes_shape(rows: int, d_v: int, fmt: str):
    if fmt == "bf16":
        return (rows, d_v), torch.int16
    if fmt == "e4m3":
        return (rows, d_v), torch.uint8
    if fmt == "int4":
        return (rows, d_v // 2), torch.uint8
    raise ValueError(f"unknown row format {fmt!r}; one of {sorted(ROW_FORMAT)}")


def sdm_state_rows_bytes(rows: int, d_v: int, fmt: str = "e4m3") -> int:
    """Bytes of the checkpoint codes of `rows` rows of d_v values (0: invalid arguments)."""
    return int(library().sdm_state_rows_bytes(int(rows), int(d_v), ROW_FORMAT[fmt]))


def sdm_state_pack(M, fmt: str = "e4m3", *, codes=None, scales=None, stream=None):
    """Checkpoint rows of M [..., d_v] (fp32): (codes, scales).  codes: int16 [rows, d_v]
    (bf16 bit patterns), uint8 [rows, d_v] (E4M3) or uint8 [rows, d_v / 2] (int4, two per
    byte); scales: fp32 [rows] (None for bf16)."""
    d_v = M.shape[-1]
    rows = M.numel() // d_v if d_v else 0
    cshape, cdt = _row_codes_shape(rows, d_v, fmt)
    _expect(codes, "codes", cshape)
    _expect(scales, "scales", (rows,))
    _need(M, "M", torch.float32)
    if codes is None:
        codes = torch.empty(cshape, dtype=cdt, device=M.device)
    _need(codes, "codes", cdt, M.device)
    if fmt != "bf16":
        if scales is None:
            scales = torch.empty(rows, dtype=torch.float32, device=M.device)
        _need(scales, "scales", torch.float32, M.device)
    else:
        scales = None
    _check(library().sdm_state_pack(_p(M), rows, d_v, ROW_FORMAT[fmt], _p(codes), _p(scales),
                                    _stream(stream, M.device)), "sdm_state_pack")
    return codes, scales


def sdm_state_unpack(codes, scales, d_v: int, fmt: str = "e4m3", *, out=None, stream=None):
    """fp32 rows [rows, d_v] from checkpoint codes (+ scales) made by sdm_state_pack."""
    rows = codes.shape[0]
    cshape, cdt = _row_codes_shape(rows, d_v, fmt)
    _expect(codes, "codes", cshape)
    _expect(out, "out", None, rows * d_v)
    _need(codes, "codes", cdt)
    if fmt != "bf16":
        _expect(scales, "scales", (rows,))
        _need(scales, "scales", torch.float32, codes.device)
    out = torch.empty((rows, d_v), dtype=torch.float32, device=codes.device) if out is None \
        else out
    _need(out, "out", torch.float32, codes.device)
    _check(library().sdm_state_unpack(_p(codes), _p(scales if fmt != "bf16" else None), rows,
                                      d_v, ROW_FORMAT[fmt], _p(out),
                                      _stream(stream, codes.device)), "sdm_state_unpack")
    return out


KERNEL_KINDS = ("state_init", "select", "scan_seq", "scan_slot", "norm_gate", "decode",
                "slot_sort", "state_rows", "undo", "scan_chunk")


def sdm_profile_enable(on: bool = True):
    """Brackets every library launch with CUDA events on its stream (off by default)."""
    _check(library().sdm_profile_enable(1 if on else 0), "sdm_profile_enable")


def sdm_profile_read() -> dict:
    """{kind: (total ms, launches)} of the launches recorded since the last enable/read."""
    ms = (ctypes.c_double * 16)()
    n = (ctypes.c_int64 * 16)()
    _check(library().sdm_profile_read(ctypes.cast(ms, ctypes.c_void_p),
                                      ctypes.cast(n, ctypes.c_void_p)), "sdm_profile_read")
    return {k: (ms[i], n[i]) for i, k in enumerate(KERNEL_KINDS)}


OPTION = {"no_pdl": 1, "select_general": 2, "select_ctas_per_sm": 3, "slot_ctas_per_sm": 4,
          "seq_columns": 5, "seq_depth": 6, "slot_cta_stats": 7, "select_schedule": 8}
SLOT_STATS_CTAS = 1024


def sdm_slot_cta_stats(max_ctas: int = SLOT_STATS_CTAS, reset: bool = True):
    """Per-CTA work of the slot engine recorded while option "slot_cta_stats" is 1: an int64
    array [max_ctas, 4] of (short-segment events, long-segment events, spans, busy warp-ns)."""
    import numpy as np
    out = np.zeros((int(max_ctas), 4), np.uint64)
    _check(library().sdm_slot_cta_stats(ctypes.c_void_p(out.ctypes.data), int(max_ctas),
                                        1 if reset else 0), "sdm_slot_cta_stats")
    return out.astype(np.int64)


def sdm_set_option(option: str, value: int):
    """Sets a process-wide launch option of include/sdm.h (sdm_option), by name."""
    _check(library().sdm_set_option(OPTION[option], int(value)), f"sdm_set_option({option})")


def sdm_get_option(option: str) -> int:
    return int(library().sdm_get_option(OPTION[option]))


def sdm_launch_count() -> int:
    """Kernels launched by the library in this process so far."""
    return int(library().sdm_launch_count())


def sdm_get_device_status(stream=None) -> int:
    """Synchronises the stream and returns (and clears) the device status code."""
    return int(library().sdm_get_device_status(_stream(stream)))
