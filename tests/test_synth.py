"""The seeded input recipe (sdm_synth): counter-based, shape-independent streams with the
distributions the workloads state.

The recipe: score halves k', q' ~ N(0, 1), with the long skewed prefill adding
-0.5 ln(1 + j) to element j of each half; v, gate ~ N(0, 1); alpha = exp(-softplus(z)),
beta = sigmoid(z') with z, z' ~ N(0, 1); M0 ~ N(0, 0.02^2) in float32; bf16 where the
workload says so.  Every element is a pure function of (seed, tensor id, element index).
"""

import math

import numpy as np
import pytest
import torch

import sdm_synth as S


def test_tensor_hash_equals_the_scalar_hash():
    """The 16-bit-limb int64 evaluation of lowbias32 equals the plain integer one."""
    rng = np.random.default_rng(0)
    xs = np.concatenate([rng.integers(0, 2 ** 32, 4000, dtype=np.uint64),
                         np.array([0, 1, 0xFFFF, 0x10000, 2 ** 31, 2 ** 32 - 1], np.uint64)])
    got = S.mix32(torch.from_numpy(xs.astype(np.int64))).numpy()
    want = np.array([S.mix32_int(int(x)) for x in xs], np.int64)
    np.testing.assert_array_equal(got, want)


def test_scalar_hash_follows_its_published_steps():
    """lowbias32: xorshift 16, multiply 0x7feb352d, xorshift 15, multiply 0x846ca68b,
    xorshift 16, all modulo 2^32, restated here with numpy uint32 arithmetic."""
    x = np.arange(0, 1 << 20, 4099, dtype=np.uint32)
    with np.errstate(over="ignore"):
        y = x ^ (x >> np.uint32(16))
        y = y * np.uint32(0x7FEB352D)
        y = y ^ (y >> np.uint32(15))
        y = y * np.uint32(0x846CA68B)
        y = y ^ (y >> np.uint32(16))
    np.testing.assert_array_equal(y, [S.mix32_int(int(v)) for v in x])


def test_normal_draws_have_unit_moments():
    z = S.normal_f64(0x5D3, 1, 0, 1 << 20, "cpu").numpy()
    assert abs(z.mean()) < 5e-3
    assert abs(z.var() - 1.0) < 5e-3
    tail = np.mean(np.abs(z) > 3.0)
    assert abs(tail - math.erfc(3.0 / math.sqrt(2.0))) < 5e-4
    assert np.isfinite(z).all()


def test_streams_do_not_depend_on_chunking_or_offset():
    a = S.draw(7, 3, (5, 1000), torch.float32, chunk=1 << 24)
    b = S.draw(7, 3, (5, 1000), torch.float32, chunk=333)
    assert torch.equal(a, b)
    whole = S.normal_f64(7, 3, 0, 5000, "cpu")
    part = S.normal_f64(7, 3, 1234, 777, "cpu")
    assert torch.equal(whole[1234:1234 + 777], part)
    assert not torch.equal(S.normal_f64(7, 4, 0, 100, "cpu"), whole[:100])  # another stream


def test_distributions_of_a_workload():
    wl = S.WORKLOADS["small"].replace(T=64, S1=64, S2=64)
    d = S.make_inputs(wl, with_gamma=True)
    assert d["kp"].dtype == torch.bfloat16 and d["alpha"].dtype == torch.float32
    assert d["kp"].shape == (wl.B, wl.T, wl.H, wl.S1 + wl.S2)
    assert d["M0"].shape == (wl.H, wl.N, wl.d_v) and d["M0"].dtype == torch.float32
    a, b = d["alpha"], d["beta"]
    assert bool(((a > 0) & (a < 1)).all()) and bool(((b > 0) & (b < 1)).all())
    # alpha = exp(-softplus(z)) = sigmoid(-z); beta = sigmoid(z'): both have mean 1/2 by
    # symmetry of z
    assert abs(float(a.mean()) - 0.5) < 0.03 and abs(float(b.mean()) - 0.5) < 0.03
    assert abs(float(d["M0"].std()) - 0.02) < 2e-4
    assert abs(float(d["kp"].float().std()) - 1.0) < 0.02
    # bf16 values are exactly representable: the float32 copies round-trip
    assert torch.equal(d["v"].float().to(torch.bfloat16), d["v"])


def test_skew_adds_the_stated_bias_per_half():
    base = S.WORKLOADS["long_skew"].replace(T=4, H=2, S1=16, S2=8, in_dtype=torch.float32)
    skew = S.make_inputs(base, with_gate=False)["kp"].double()
    flat = S.make_inputs(base.replace(skew=False), with_gate=False)["kp"].double()
    j = torch.cat([torch.arange(16), torch.arange(8)]).double()
    np.testing.assert_allclose((skew - flat).numpy(),
                               np.broadcast_to(-0.5 * np.log1p(j.numpy()), skew.shape),
                               atol=1e-6)


def test_first_sequence_prefix_does_not_depend_on_the_length():
    """The CPU baseline draws sequence 0's first tokens alone: they equal the same tokens
    of the full workload."""
    wl = S.WORKLOADS["small"].replace(T=32, S1=16, S2=16, d_v=16)
    full = S.make_inputs(wl)
    short = S.make_inputs(wl.replace(B=1, T=8))
    for k in ("kp", "qp", "v", "alpha", "beta", "gate"):
        assert torch.equal(short[k], full[k][:1, :8]), k
    assert torch.equal(short["M0"], full["M0"])


@pytest.mark.parametrize("step", [0, 3])
def test_a_decode_step_equals_its_slice_of_the_stacked_run(step):
    wl = S.WORKLOADS["decode"].replace(B=2, H=2, T=4, S1=16, S2=16, d_v=16)
    one = S.make_inputs(wl, step=step)
    stack = S.make_inputs(wl)
    for k in ("kp", "qp", "v", "alpha", "beta", "gate"):
        assert torch.equal(one[k], stack[k][step]), k
    assert ("M0" in one) == (step == 0)
