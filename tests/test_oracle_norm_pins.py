"""Pins of the oracle's pre-RMSNorm layer variant (CPU).

The reading (a DeepSeek-style decoder block without its attention, which the
pages do not give): a layer with a norm gain g routes and runs its experts on
x = bf16(RMSNorm(h) * g) and adds the MoE output to the un-normalised
residual, h' = bf16(h + MoE(x)).  Rows of +-1 have RMS exactly 1, so there
RMSNorm is the identity up to eps (which bf16 rounding absorbs): that fixes
the variant against the plain layer, the gain, and which tensor the residual
takes.
"""
import numpy as np
import pytest

from moe_decoder_speculative_b200 import workloads as wl


def bf(a):
    return wl.f32_to_bf16_bits(np.asarray(a, np.float32))


@pytest.fixture(scope="module")
def setup():
    w = wl.workload(0)
    inp = wl.make_inputs(w, norm=True)
    rng = np.random.default_rng(3)
    signs = bf(np.where(rng.random((w.T, w.H)) < 0.5, -1.0, 1.0))   # every row has RMS exactly 1
    return w, inp, signs


def test_unit_gain_on_unit_rms_rows_equals_the_plain_layer(oracle_mod, setup):
    w, inp, signs = setup
    lay = dict(inp["layers"][0])
    lay["norm_gain"] = bf(np.ones(w.H))
    plain = dict(lay)
    plain.pop("norm_gain")
    a = oracle_mod.moe_stack(signs, [lay], w.k)
    b = oracle_mod.moe_stack(signs, [plain], w.k)
    np.testing.assert_array_equal(a["h"], b["h"])
    np.testing.assert_array_equal(a["layers"][0]["idx"], b["layers"][0]["idx"])


def test_gain_reaches_router_and_experts_but_not_the_residual(oracle_mod, setup):
    """Gain 2 on unit-RMS rows: x = 2h exactly, so the layer equals routing and
    experts on 2h with the residual h."""
    w, inp, signs = setup
    lay = dict(inp["layers"][0])
    lay["norm_gain"] = bf(np.full(w.H, 2.0))
    got = oracle_mod.moe_stack(signs, [lay], w.k)
    x2 = bf(2.0 * wl.bf16_bits_to_f32(signs))
    idx, tw, _, _ = oracle_mod.router(x2, lay["w_router"], w.k)
    _, expect = oracle_mod.moe_ffn(x2, lay, idx, tw, residual=signs)
    np.testing.assert_array_equal(got["layers"][0]["idx"], idx)
    np.testing.assert_array_equal(got["h"], expect)


def test_a_zero_layer_returns_the_unnormalised_rows(oracle_mod, setup):
    w, inp, _ = setup
    lay = {k: (np.zeros_like(v) if isinstance(v, np.ndarray) and k != "norm_gain" else v)
           for k, v in inp["layers"][0].items()}
    h = wl.normal_bf16(np.random.SeedSequence(8), (w.T, w.H), 3.0)   # RMS far from 1
    got = oracle_mod.moe_stack(h, [lay], w.k)
    np.testing.assert_array_equal(got["h"], h)


def test_routing_does_not_see_the_scale_of_the_rows(oracle_mod, setup):
    w, inp, _ = setup
    lay = inp["layers"][0]
    h = wl.normal_bf16(np.random.SeedSequence(9), (w.T, w.H), 1.0)
    h4 = bf(4.0 * wl.bf16_bits_to_f32(h))
    a = oracle_mod.moe_stack(h, [lay], w.k)["layers"][0]
    b = oracle_mod.moe_stack(h4, [lay], w.k)["layers"][0]
    clear = (a["gap"] > 1e-3) & (b["gap"] > 1e-3)
    assert clear.mean() > 0.5
    for r in np.nonzero(clear)[0]:
        assert set(a["idx"][r]) == set(b["idx"][r])
