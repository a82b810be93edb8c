"""Pins for the text-fusion part of the oracle (NEXT row: Krea2TextFusion + txt_in)."""
import numpy as np

import krea2_inputs as KI
from oracle import krea2_oracle as O
from test_oracle_pins import _textbook_block

R = np.random.default_rng(77)
TD = KI.TINY_TEXT


def _args(td=TD):
    return dict(H=td.H, Hkv=td.Hkv, D=td.D, eps=td.eps)


def test_fusion_block_is_a_textbook_prenorm_block_without_positions():
    bd = TD.block_dims()
    w = KI.block_weights(bd, 3)
    x = R.standard_normal((2, 5, TD.Dt))
    kv = np.ones((2, 5), dtype=bool)
    kv[1, 3:] = False
    got = O.text_fusion_block(x, w, kv, **_args())
    ref = _textbook_block(bd, x, w, np.zeros((5, 3)), kv)   # zero positions: RoPE is the identity
    np.testing.assert_allclose(got, ref, rtol=1e-10, atol=1e-10)


def test_layer_projection_picks_the_weighted_layer_stack():
    ehs = R.standard_normal((2, 4, TD.L, TD.Dt))
    lw = np.zeros(TD.L)
    lw[1] = 1.0
    out = O.text_fusion(ehs, None, [], lw, [], **_args())
    np.testing.assert_array_equal(out, ehs[:, :, 1])
    lw = R.standard_normal(TD.L)
    out = O.text_fusion(ehs, None, [], lw, [], **_args())
    np.testing.assert_allclose(out, (ehs * lw[None, None, :, None]).sum(axis=2), rtol=1e-12)


def test_layerwise_stage_treats_tokens_independently():
    w = KI.text_fusion_weights(TD)
    ehs = R.standard_normal((1, 4, TD.L, TD.Dt))
    out = O.text_fusion(ehs, None, w["layerwise"], w["layer_w"], [], **_args())
    ehs2 = ehs.copy()
    ehs2[0, 2] = R.standard_normal((TD.L, TD.Dt)) * 3
    out2 = O.text_fusion(ehs2, None, w["layerwise"], w["layer_w"], [], **_args())
    np.testing.assert_allclose(out2[0, [0, 1, 3]], out[0, [0, 1, 3]], rtol=1e-12, atol=1e-12)


def test_layerwise_stage_has_no_positions_along_the_layer_axis():
    # no RoPE: permuting the stacked layers (and the projection weights with them) changes nothing
    w = KI.text_fusion_weights(TD)
    ehs = R.standard_normal((1, 3, TD.L, TD.Dt))
    perm = R.permutation(TD.L)
    a = O.text_fusion(ehs, None, w["layerwise"], w["layer_w"], [], **_args())
    b = O.text_fusion(ehs[:, :, perm], None, w["layerwise"], w["layer_w"][perm], [], **_args())
    np.testing.assert_allclose(a, b, rtol=1e-10, atol=1e-10)


def test_refiner_ignores_padded_tokens():
    w = KI.text_fusion_weights(TD)
    ehs = R.standard_normal((1, 6, TD.L, TD.Dt))
    mask = np.array([[True, True, True, True, False, False]])
    out = O.text_fusion(ehs, mask, w["layerwise"], w["layer_w"], w["refiner"], **_args())
    ehs2 = ehs.copy()
    ehs2[0, 4:] = R.standard_normal((2, TD.L, TD.Dt)) * 4
    out2 = O.text_fusion(ehs2, mask, w["layerwise"], w["layer_w"], w["refiner"], **_args())
    np.testing.assert_allclose(out2[0, :4], out[0, :4], rtol=1e-10, atol=1e-10)


def test_txt_in_is_a_linear_with_bias():
    w = KI.text_fusion_weights(TD)
    x = R.standard_normal((2, 3, TD.Dt))
    out = O.txt_in(x, w["txt_in_w"], w["txt_in_b"])
    assert out.shape == (2, 3, TD.C)
    np.testing.assert_allclose(out[1, 2], w["txt_in_w"] @ x[1, 2] + w["txt_in_b"], rtol=1e-12)
