"""Seeded synthetic inputs for the SDM memory pass.

This module holds the workload shapes and a counter-based random generator, and
nothing of the method's arithmetic.  Both the CUDA path (tests, benchmark) and the
CPU oracle consume what it produces; neither side's code lives here.

Generator.  Every element is a pure function of (seed, tensor id, element index), so
the values do not depend on device, chunking or thread count:

  * a 32-bit mixing function ``mix32`` (the "lowbias32" integer hash published by
    C. Wellons in hash-prospector: xorshift 16, multiply 0x7feb352d, xorshift 15,
    multiply 0x846ca68b, xorshift 16), evaluated in int64 tensor arithmetic with
    16-bit limbs so no intermediate exceeds 2^49;
  * two 32-bit words per element, w1 = mix32(mix32(e + k1) + k2) and the same with
    keys k3, k4, which are bijections of the element index e < 2^32;
  * Box-Muller in float64: z = sqrt(-2 ln u1) cos(2 pi u2), u1 = (w1 + 1) / 2^32,
    u2 = w2 / 2^32;
  * rounding float64 -> float32 -> bfloat16, each round-to-nearest-even.

Distributions (the five workloads):
  score halves k', q' ~ N(0, 1) (the long skewed prefill adds -0.5 ln(1 + j) to
  element j of each half before rounding); v, gate ~ N(0, 1); alpha = exp(-softplus(z)),
  beta = sigmoid(z') with z, z' ~ N(0, 1); M0 ~ N(0, 0.02^2) in float32.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

M32 = 0xFFFFFFFF

# tensor ids of the generator streams
TID_KP, TID_QP, TID_V, TID_ALPHA, TID_BETA, TID_GATE, TID_M0, TID_GAMMA = 1, 2, 3, 4, 5, 6, 7, 8
STEP_STRIDE = 64  # decode step s of a tensor uses tensor id tid + STEP_STRIDE * (s + 1)


@dataclass(frozen=True)
class Workload:
    """Shape and dtype of one synthetic workload."""
    name: str
    B: int
    H: int
    T: int
    S1: int
    S2: int
    W: int
    R: int
    d_v: int
    in_dtype: torch.dtype
    skew: bool = False
    decode: bool = False          # T successive single-token steps
    seed: int = 0x5D3
    note: str = field(default="", compare=False)

    @property
    def N(self) -> int:
        return self.S1 * self.S2

    def replace(self, **kw) -> "Workload":
        d = {k: getattr(self, k) for k in self.__dataclass_fields__}
        d.update(kw)
        return Workload(**d)


WORKLOADS = {
    "tiny": Workload("tiny", B=1, H=1, T=64, S1=16, S2=16, W=8, R=8, d_v=16,
                     in_dtype=torch.float32, seed=0x5D3 + 0,
                     note="B1 H1 T64 N256 W=R=8 d_v16 fp32"),
    "small": Workload("small", B=2, H=4, T=2048, S1=256, S2=256, W=64, R=64, d_v=64,
                      in_dtype=torch.bfloat16, seed=0x5D3 + 1,
                      note="B2 H4 T2048 N65536 W=R=64 d_v64 bf16"),
    "layer1p4b": Workload("layer1p4b", B=4, H=8, T=8192, S1=512, S2=512, W=64, R=64,
                          d_v=128, in_dtype=torch.bfloat16, seed=0x5D3 + 2,
                          note="B4 H8 T8192 N262144 W=R=64 d_v128 bf16"),
    "long_skew": Workload("long_skew", B=1, H=4, T=262144, S1=1024, S2=1024, W=64, R=64,
                          d_v=256, in_dtype=torch.bfloat16, skew=True, seed=0x5D3 + 3,
                          note="B1 H4 T262144 N1048576 W=R=64 d_v256 bf16, skewed halves"),
    "decode": Workload("decode", B=64, H=8, T=256, S1=512, S2=512, W=64, R=64, d_v=128,
                       in_dtype=torch.bfloat16, decode=True, seed=0x5D3 + 4,
                       note="64 seq H8 N262144 W=R=64 d_v128 bf16, 256 decode steps"),
}


def mix32_int(x: int) -> int:
    """lowbias32 on a Python int (used for the scalar keys)."""
    x &= M32
    x ^= x >> 16
    x = (x * 0x7FEB352D) & M32
    x ^= x >> 15
    x = (x * 0x846CA68B) & M32
    x ^= x >> 16
    return x


def _mul32(x: torch.Tensor, c: int) -> torch.Tensor:
    """(x * c) mod 2^32 for int64 x in [0, 2^32), with 16-bit limbs of c."""
    lo = x * (c & 0xFFFF)
    hi = (x * (c >> 16)) & 0xFFFF
    return (lo + (hi << 16)) & M32


def mix32(x: torch.Tensor) -> torch.Tensor:
    """lowbias32 on an int64 tensor holding values in [0, 2^32)."""
    x = x ^ (x >> 16)
    x = _mul32(x, 0x7FEB352D)
    x = x ^ (x >> 15)
    x = _mul32(x, 0x846CA68B)
    x = x ^ (x >> 16)
    return x


def _keys(seed: int, tid: int):
    base = mix32_int(mix32_int(seed) ^ mix32_int(tid * 0x9E3779B1 + 0x632BE5AB))
    return [mix32_int(base + 0x85EBCA77 * (j + 1)) for j in range(4)]


def _words(e: torch.Tensor, ka: int, kb: int) -> torch.Tensor:
    return mix32((mix32((e + ka) & M32) + kb) & M32)


def normal_f64(seed: int, tid: int, start: int, count: int, device) -> torch.Tensor:
    """float64 N(0,1) draws for element indices [start, start + count)."""
    if start + count > (1 << 32):
        raise ValueError("element index beyond 2^32 in one generator stream")
    k = _keys(seed, tid)
    e = torch.arange(start, start + count, dtype=torch.int64, device=device)
    w1 = _words(e, k[0], k[1])
    w2 = _words(e, k[2], k[3])
    del e
    u1 = (w1.to(torch.float64) + 1.0) * (1.0 / 4294967296.0)
    u2 = w2.to(torch.float64) * (1.0 / 4294967296.0)
    del w1, w2
    return torch.sqrt(-2.0 * torch.log(u1)) * torch.cos((2.0 * math.pi) * u2)


def draw(seed: int, tid: int, shape, dtype: torch.dtype, device="cpu", scale: float = 1.0,
         transform=None, chunk: int = 1 << 24) -> torch.Tensor:
    """A tensor of ``shape`` filled element-by-element (row-major order) from the stream.

    transform(z, flat_index) may map the float64 draws before rounding to ``dtype``.
    """
    shape = tuple(int(s) for s in shape)
    n = 1
    for s in shape:
        n *= s
    out = torch.empty(n, dtype=dtype, device=device)
    for s0 in range(0, n, chunk):
        c = min(chunk, n - s0)
        z = normal_f64(seed, tid, s0, c, device)
        if scale != 1.0:
            z = z * scale
        if transform is not None:
            z = transform(z, s0)
        z32 = z.to(torch.float32)
        out[s0:s0 + c] = z32.to(dtype) if dtype != torch.float32 else z32
    return out.view(shape)


def _skew_transform(S1: int, S2: int):
    """Adds -0.5 ln(1 + j) to element j of each half of a [.., S1 + S2] score row."""
    def f(z: torch.Tensor, s0: int) -> torch.Tensor:
        pos = torch.arange(s0, s0 + z.numel(), dtype=torch.int64, device=z.device) % (S1 + S2)
        j = torch.where(pos < S1, pos, pos - S1).to(torch.float64)
        return z - 0.5 * torch.log1p(j)
    return f


def _alpha_from(z: torch.Tensor, s0: int) -> torch.Tensor:
    return torch.exp(-torch.nn.functional.softplus(z))


def _beta_from(z: torch.Tensor, s0: int) -> torch.Tensor:
    return torch.sigmoid(z)


def make_inputs(wl: Workload, device="cpu", with_gate: bool = True, with_gamma: bool = False,
                step: int | None = None) -> dict:
    """All inputs of one workload.

    Prefill layout: kp/qp [B,T,H,S1+S2], v/gate [B,T,H,d_v], alpha/beta [B,T,H].
    Decode workloads (``wl.decode``) with ``step`` given: one step's inputs,
    kp/qp [B,H,S1+S2], v/gate [B,H,d_v], alpha/beta [B,H]; with ``step`` None the whole
    run stacked step-major: kp [T,B,H,S1+S2] etc.
    M0 is [H, N, d_v] float32 (omitted for a decode step other than the first).
    """
    S = wl.S1 + wl.S2
    seed = wl.seed
    if wl.decode and step is not None:
        lead = (wl.B, wl.H)
        off = STEP_STRIDE * (step + 1)
    elif wl.decode:
        # stacked: each step's block comes from its own stream so that a single step
        # drawn alone equals the matching slice of the stack
        steps = [make_inputs(wl, device, with_gate, with_gamma, step=s) for s in range(wl.T)]
        out = {k: torch.stack([st[k] for st in steps]) for k in steps[0] if k not in ("M0",)}
        out["M0"] = steps[0]["M0"]
        if with_gamma:
            out["gamma"] = steps[0]["gamma"]
        return out
    else:
        lead = (wl.B, wl.T, wl.H)
        off = 0
    tr = _skew_transform(wl.S1, wl.S2) if wl.skew else None
    d = {}
    d["kp"] = draw(seed, TID_KP + off, lead + (S,), wl.in_dtype, device, transform=tr)
    d["qp"] = draw(seed, TID_QP + off, lead + (S,), wl.in_dtype, device, transform=tr)
    d["v"] = draw(seed, TID_V + off, lead + (wl.d_v,), wl.in_dtype, device)
    d["alpha"] = draw(seed, TID_ALPHA + off, lead, torch.float32, device, transform=_alpha_from)
    d["beta"] = draw(seed, TID_BETA + off, lead, torch.float32, device, transform=_beta_from)
    if with_gate:
        d["gate"] = draw(seed, TID_GATE + off, lead + (wl.d_v,), wl.in_dtype, device)
    if not wl.decode or step in (None, 0):
        d["M0"] = draw(seed, TID_M0, (wl.H, wl.N, wl.d_v), torch.float32, device, scale=0.02)
    if with_gamma:
        d["gamma"] = draw(seed, TID_GAMMA, (wl.d_v,), torch.float32, device,
                          transform=lambda z, s0: 1.0 + 0.1 * z)
    return d
