"""Pins for the CPU oracle: closed forms, invariants, library special cases, brute force.

Each test ties one oracle function to something other than the oracle itself, so that a
dropped term, a wrong sign or index, or a transposed operand fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as Fn

import krea2_inputs as KI
from oracle import krea2_oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden")
R = np.random.default_rng(1234)


def _load(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


# ----------------------------------------------------------------------------- config

def test_defaults_match_api_page():
    g = _load("config_defaults.json")
    d = KI.FULL
    assert d.in_ch == g["in_channels"] and d.n_layers == g["num_layers"]
    assert d.D == g["attention_head_dim"] and d.H == g["num_attention_heads"]
    assert d.Hkv == g["num_key_value_heads"] and d.F == g["intermediate_size"]
    assert d.t_dim == g["timestep_embed_dim"] and list(d.axes) == g["axes_dims_rope"]
    assert d.theta == g["rope_theta"] and d.eps == g["norm_eps"]
    assert d.C == g["hidden_size"] == d.H * d.D and d.H // d.Hkv == g["gqa_group"]
    assert sum(d.axes) == d.D


def test_dim_and_position_checks_raise():
    with pytest.raises(ValueError):
        O.check_dims(128, (32, 48, 40), 48, 12)
    with pytest.raises(ValueError):
        O.check_dims(128, (32, 48, 48), 48, 10)
    O.check_dims(128, (32, 48, 48), 48, 12)
    with pytest.raises(ValueError):
        O.check_positions(np.zeros((10, 2)))
    with pytest.raises(ValueError):
        O.check_positions(np.zeros((10, 3, 1)))
    with pytest.raises(ValueError):
        O.check_positions(np.zeros((10, 3)), S=11)


# ----------------------------------------------------------------------------- P1 RMSNorm

def test_rmsnorm_mean_square_closed_form():
    # with w = 0 each output row has mean square ms / (ms + eps)
    eps = 1e-5
    for scale in (1e-3, 1.0, 37.0):
        x = R.standard_normal((3, 64)) * scale
        ms = np.mean(x * x, axis=-1)
        y = O.rms_norm(x, np.zeros(64), eps)
        np.testing.assert_allclose(np.mean(y * y, axis=-1), ms / (ms + eps), rtol=1e-12)
        # direction is kept: y is a positive multiple of x per row
        ratio = y / x
        assert np.all(ratio > 0)
        np.testing.assert_allclose(ratio, ratio[:, :1] * np.ones_like(ratio), rtol=1e-12)


def test_rmsnorm_weight_is_one_plus_w_against_torch():
    x = R.standard_normal((5, 48))
    w = R.standard_normal(48) * 0.3
    ref = Fn.rms_norm(torch.tensor(x), (48,), weight=1.0 + torch.tensor(w), eps=1e-5).numpy()
    np.testing.assert_allclose(O.rms_norm(x, w, 1e-5), ref, rtol=1e-12, atol=1e-14)


# ----------------------------------------------------------------------------- P2 RoPE

def test_rope_angles_hand_values():
    g = _load("rope_hand_values.json")
    for case in g["cases"]:
        ang = O.rope_angles(np.array([case["pos"]], dtype=np.float64), (32, 48, 48), 1000.0)
        assert ang.shape == (1, 64)
        assert abs(ang[0, case["pair"]] - case["angle"]) < 1e-12, case


def test_rope_axis_blocks_touch_only_their_dims():
    x = R.standard_normal((3, 2, 128))
    pos = np.array([[5, 0, 0], [0, 5, 0], [0, 0, 5]], dtype=np.float64)
    c, s = O.rope_cos_sin(pos, (32, 48, 48), 1000.0)
    y = O.apply_rope(x, c, s)
    spans = [(0, 32), (32, 80), (80, 128)]
    for r, (lo, hi) in enumerate(spans):
        changed = np.nonzero(np.any(np.abs(y[r] - x[r]) > 1e-12, axis=0))[0]
        assert changed.min() >= lo and changed.max() < hi, (r, changed)


def test_rope_preserves_norm_and_is_identity_at_zero():
    x = R.standard_normal((7, 3, 128))
    pos = R.integers(0, 64, size=(7, 3)).astype(np.float64)
    c, s = O.rope_cos_sin(pos, (32, 48, 48), 1000.0)
    y = O.apply_rope(x, c, s)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-12)
    c0, s0 = O.rope_cos_sin(np.zeros((7, 3)), (32, 48, 48), 1000.0)
    np.testing.assert_array_equal(O.apply_rope(x, c0, s0), x)


def test_rope_matches_complex_rotation():
    # pair p as the complex number x_{2p} + i x_{2p+1}, multiplied by exp(i * angle)
    x = R.standard_normal((4, 1, 64))
    pos = R.integers(0, 30, size=(4, 3)).astype(np.float64)
    ang = O.rope_angles(pos, (16, 24, 24), 1000.0)
    z = (x[..., 0::2] + 1j * x[..., 1::2]) * np.exp(1j * ang)[:, None, :]
    ref = np.empty_like(x)
    ref[..., 0::2] = z.real
    ref[..., 1::2] = z.imag
    c, s = O.rope_cos_sin(pos, (16, 24, 24), 1000.0)
    np.testing.assert_allclose(O.apply_rope(x, c, s), ref, rtol=1e-12, atol=1e-12)


def test_rope_is_relative():
    q = R.standard_normal((1, 1, 128))
    k = R.standard_normal((1, 1, 128))
    p = np.array([[0, 3, 11]], dtype=np.float64)
    pk = np.array([[0, 7, 2]], dtype=np.float64)
    for shift in ([0, 5, 0], [0, 0, 9], [2, 1, 13]):
        sh = np.array([shift], dtype=np.float64)
        dots = []
        for off in (0.0, 1.0):
            cq, sq = O.rope_cos_sin(p + off * sh, (32, 48, 48), 1000.0)
            ck, sk = O.rope_cos_sin(pk + off * sh, (32, 48, 48), 1000.0)
            dots.append(float(np.sum(O.apply_rope(q, cq, sq) * O.apply_rope(k, ck, sk))))
        assert abs(dots[0] - dots[1]) < 1e-10


# ----------------------------------------------------------------------------- P3/P5 attention

def _rand_attn(B=2, S=12, H=8, Hkv=2, D=16):
    q = R.standard_normal((B, S, H, D))
    k = R.standard_normal((B, S, Hkv, D))
    v = R.standard_normal((B, S, Hkv, D))
    kv = R.random((B, S)) < 0.7
    kv[:, -1] = True
    return q, k, v, kv


def _sdpa(q, k, v, kv):
    qt = torch.tensor(q).permute(0, 2, 1, 3)
    kt = torch.tensor(k).permute(0, 2, 1, 3)
    vt = torch.tensor(v).permute(0, 2, 1, 3)
    mask = torch.tensor(kv)[:, None, None, :]
    return Fn.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask).permute(0, 2, 1, 3).numpy()


def test_gqa_equals_mha_with_repeat_interleaved_kv():
    q, k, v, kv = _rand_attn()
    G = q.shape[2] // k.shape[2]
    out = O.attention(q, k, v, kv, 1.0 / math.sqrt(q.shape[-1]))
    ref = _sdpa(q, np.repeat(k, G, axis=2), np.repeat(v, G, axis=2), kv)
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-12)
    # negative control: tiled (not interleaved) head order must differ
    bad = _sdpa(q, np.tile(k, (1, 1, G, 1)), np.tile(v, (1, 1, G, 1)), kv)
    assert np.max(np.abs(out - bad)) > 1e-3


def test_attention_brute_force_python_loops():
    B, S, H, Hkv, D = 1, 9, 4, 2, 4
    q, k, v, kv = _rand_attn(B, S, H, Hkv, D)
    out = O.attention(q, k, v, kv, 1.0 / math.sqrt(D))
    for h in range(H):
        j = h // (H // Hkv)
        for i in range(S):
            scores = []
            for t in range(S):
                if kv[0, t]:
                    scores.append((t, sum(q[0, i, h, c] * k[0, t, j, c] for c in range(D)) / math.sqrt(D)))
            mx = max(sc for _, sc in scores)
            wsum = sum(math.exp(sc - mx) for _, sc in scores)
            for c in range(D):
                ref = sum(math.exp(sc - mx) / wsum * v[0, t, j, c] for t, sc in scores)
                assert abs(out[0, i, h, c] - ref) < 1e-12


def test_padded_keys_have_no_effect():
    q, k, v, kv = _rand_attn()
    out = O.attention(q, k, v, kv, 0.25)
    k2, v2 = k.copy(), v.copy()
    k2[~kv] = R.standard_normal(k2[~kv].shape) * 50
    v2[~kv] = R.standard_normal(v2[~kv].shape) * 50
    np.testing.assert_array_equal(O.attention(q, k2, v2, kv, 0.25), out)


# ----------------------------------------------------------------------------- block fixtures

def _tiny_block_inputs(dims=KI.TINY, B=1, T=8, gh=8, gw=8, lengths=(6,)):
    S = T + gh * gw
    h = KI.residual(dims, B, S).astype(np.float64)
    temb = KI.temb(dims, B).astype(np.float64)
    w = KI.block_weights(dims, 0)
    pos = KI.position_ids(T, gh, gw)
    c, s = O.rope_cos_sin(pos, dims.axes, dims.theta)
    kv = O.key_valid_mask(KI.mask_from_lengths(T, lengths), B, T, gh * gw)
    return h, temb, w, c, s, kv, pos


def _blk(dims, h, temb, w, c, s, kv, rows=None, dtype=np.float64):
    return O.block_forward(h, temb, w, c, s, kv, dims.H, dims.Hkv, dims.D, dims.eps, rows=rows, dtype=dtype)


# ----------------------------------------------------------------------------- P4 mask (block level)

def test_block_valid_rows_equal_run_without_padded_tokens():
    d = KI.TINY
    h, temb, w, c, s, kv, pos = _tiny_block_inputs()
    out = _blk(d, h, temb, w, c, s, kv)
    keep = np.nonzero(kv[0])[0]
    c2, s2 = O.rope_cos_sin(pos[keep], d.axes, d.theta)
    out2 = _blk(d, h[:, keep], temb, w, c2, s2, kv[:, keep])
    np.testing.assert_allclose(out[:, keep], out2, rtol=1e-12, atol=1e-12)


def test_block_padded_text_rows_do_not_reach_valid_rows():
    d = KI.TINY
    h, temb, w, c, s, kv, _ = _tiny_block_inputs()
    out = _blk(d, h, temb, w, c, s, kv)
    h2 = h.copy()
    h2[0, ~kv[0]] = R.standard_normal(h2[0, ~kv[0]].shape) * 10
    out2 = _blk(d, h2, temb, w, c, s, kv)
    np.testing.assert_allclose(out2[0, kv[0]], out[0, kv[0]], rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------------------- P6 block special cases

def test_block_zero_gates_is_identity():
    d = KI.TINY
    h, temb, w, c, s, kv, _ = _tiny_block_inputs()
    w = dict(w)
    C = d.C
    table = w["table"].astype(np.float64).copy()
    table[2] = -temb[0, 2 * C:3 * C]
    table[5] = -temb[0, 5 * C:6 * C]
    w["table"] = table
    np.testing.assert_array_equal(_blk(d, h, temb, w, c, s, kv), h)


def _torch_rope(x, pos, axes, theta):
    # x (B, S, heads, D) tensor; complex rotation per adjacent pair, axis blocks t|h|w
    parts = []
    for a, da in enumerate(axes):
        freqs = 1.0 / (theta ** (torch.arange(0, da, 2, dtype=torch.float64) / da))
        parts.append(torch.outer(torch.tensor(pos[:, a], dtype=torch.float64), freqs))
    ang = torch.cat(parts, dim=1)
    rot = torch.polar(torch.ones_like(ang), ang)[None, :, None, :]
    z = torch.view_as_complex(x.reshape(*x.shape[:-1], -1, 2).contiguous())
    return torch.view_as_real(z * rot).reshape(x.shape)


def _textbook_block(d, h, w, pos, kv, scale1=0.0, shift1=0.0, gate1=1.0, scale2=0.0, shift2=0.0, gate2=1.0):
    # textbook pre-norm block with adaLN roles made explicit, written with torch library routines
    C = d.C
    T = lambda a: torch.tensor(np.asarray(a, dtype=np.float64))
    x = T(h)
    B, S, _ = x.shape
    n1 = Fn.rms_norm(x, (C,), weight=1 + T(w["norm1_w"]), eps=d.eps) * (1 + T(scale1)) + T(shift1)
    q = Fn.linear(n1, T(w["wq"])).view(B, S, d.H, d.D)
    k = Fn.linear(n1, T(w["wk"])).view(B, S, d.Hkv, d.D)
    v = Fn.linear(n1, T(w["wv"])).view(B, S, d.Hkv, d.D)
    q = Fn.rms_norm(q, (d.D,), weight=1 + T(w["q_norm_w"]), eps=d.eps)
    k = Fn.rms_norm(k, (d.D,), weight=1 + T(w["k_norm_w"]), eps=d.eps)
    q, k = _torch_rope(q, pos, d.axes, d.theta), _torch_rope(k, pos, d.axes, d.theta)
    G = d.H // d.Hkv
    o = Fn.scaled_dot_product_attention(
        q.transpose(1, 2), k.repeat_interleave(G, 2).transpose(1, 2), v.repeat_interleave(G, 2).transpose(1, 2),
        attn_mask=torch.tensor(kv)[:, None, None, :]).transpose(1, 2).reshape(B, S, C)
    o = o * torch.sigmoid(Fn.linear(n1, T(w["wg"])))
    x1 = x + T(gate1) * Fn.linear(o, T(w["wo"]))
    n2 = Fn.rms_norm(x1, (C,), weight=1 + T(w["norm2_w"]), eps=d.eps) * (1 + T(scale2)) + T(shift2)
    ff = Fn.linear(Fn.silu(Fn.linear(n2, T(w["w_gate"]))) * Fn.linear(n2, T(w["w_up"])), T(w["w_down"]))
    return (x1 + T(gate2) * ff).numpy()


def test_block_reduces_to_textbook_prenorm_block():
    # modulation cancelled by the table (scale = shift = 0, gates = 1): the block becomes
    # x + A(n1(x)), then + M(n2(.)), written here with torch library routines
    d = KI.TINY
    h, temb, w, c, s, kv, pos = _tiny_block_inputs()
    C = d.C
    w = dict(w)
    table = -temb[0].reshape(6, C).astype(np.float64).copy()
    table[2] += 1.0
    table[5] += 1.0
    w["table"] = table
    out = _blk(d, h, temb, w, c, s, kv)
    np.testing.assert_allclose(out, _textbook_block(d, h, w, pos, kv), rtol=1e-10, atol=1e-10)


@pytest.mark.parametrize("chunk,role", [(0, "scale1"), (1, "shift1"), (2, "gate1"),
                                        (3, "scale2"), (4, "shift2"), (5, "gate2")])
def test_block_modulation_chunk_order(chunk, role):
    # one chunk of the (6, C) modulation carries a known vector; it must act in the role the
    # page's unbind order gives it (prescale, preshift, pregate, postscale, postshift, postgate)
    d = KI.TINY
    h, temb, w, c, s, kv, pos = _tiny_block_inputs()
    C = d.C
    w = dict(w)
    table = -temb[0].reshape(6, C).astype(np.float64).copy()
    table[2] += 1.0
    table[5] += 1.0
    probe = 0.5 + 0.25 * np.cos(np.arange(C))
    table[chunk] += probe
    w["table"] = table
    out = _blk(d, h, temb, w, c, s, kv)
    kw = {role: probe + (1.0 if role.startswith("gate") else 0.0)}
    np.testing.assert_allclose(out, _textbook_block(d, h, w, pos, kv, **kw), rtol=1e-10, atol=1e-10)


def test_block_modulation_scale_shift_are_applied():
    # a pure shift (prescale = 0 after the table) must move the norm output by exactly the shift:
    # compare the oracle's xn path through a 1-row identity probe of the gate-only path
    d = KI.TINY
    h, temb, w, c, s, kv, _ = _tiny_block_inputs()
    C = d.C
    base = _blk(d, h, temb, w, c, s, kv)
    w2 = dict(w)
    tb = w["table"].astype(np.float64).copy()
    tb[1] += 0.37      # preshift
    w2["table"] = tb
    assert np.max(np.abs(_blk(d, h, temb, w2, c, s, kv) - base)) > 1e-3
    w3 = dict(w)
    tb3 = w["table"].astype(np.float64).copy()
    tb3[2] *= 2.0      # pregate doubles the attention branch
    w3["table"] = tb3
    assert np.max(np.abs(_blk(d, h, temb, w3, c, s, kv) - base)) > 1e-3


# ----------------------------------------------------------------------------- P7 equivariance / batch

def test_block_image_token_permutation_equivariance():
    d = KI.TINY
    h, temb, w, c, s, kv, pos = _tiny_block_inputs()
    T = 8
    out = _blk(d, h, temb, w, c, s, kv)
    perm = np.concatenate([np.arange(T), T + R.permutation(64)])
    c2, s2 = O.rope_cos_sin(pos[perm], d.axes, d.theta)
    out2 = _blk(d, h[:, perm], temb, w, c2, s2, kv[:, perm])
    np.testing.assert_allclose(out2, out[:, perm], rtol=1e-12, atol=1e-12)


def test_block_batch_rows_are_independent():
    d = KI.TINY
    B, T = 2, 8
    h, temb, w, c, s, kv, _ = _tiny_block_inputs(B=2, lengths=(8, 3))
    out = _blk(d, h, temb, w, c, s, kv)
    for b in range(B):
        ob = _blk(d, h[b:b + 1], temb[b:b + 1], w, c, s, kv[b:b + 1])
        np.testing.assert_allclose(out[b:b + 1], ob, rtol=1e-12, atol=1e-12)


def test_block_row_subset_matches_full():
    d = KI.TINY
    h, temb, w, c, s, kv, _ = _tiny_block_inputs(B=2, lengths=(8, 2))
    out = _blk(d, h, temb, w, c, s, kv)
    rows = [0, 3, 7, 8, 40, 71]
    np.testing.assert_allclose(_blk(d, h, temb, w, c, s, kv, rows=rows), out[:, rows], rtol=1e-12, atol=1e-12)


def test_attention_from_qkvg_row_subset_and_gate():
    d = KI.TINY
    B, T, N = 1, 8, 64
    S = T + N
    x = KI.qkvg_raw(d, B, S).astype(np.float64)
    w = KI.block_weights(d, 0)
    c, s = O.rope_cos_sin(KI.position_ids(T, 8, 8), d.axes, d.theta)
    kv = O.key_valid_mask(KI.mask_from_lengths(T, [6]), B, T, N)
    full = O.attention_from_qkvg(x, B, S, d.H, d.Hkv, d.D, w["q_norm_w"], w["k_norm_w"], d.eps, c, s, kv)
    sub = O.attention_from_qkvg(x, B, S, d.H, d.Hkv, d.D, w["q_norm_w"], w["k_norm_w"], d.eps, c, s, kv, rows=[1, 50])
    np.testing.assert_allclose(sub, full[:, [1, 50]], rtol=1e-12, atol=1e-12)
    # a gate column of -inf-ish logits switches its output element off
    x2 = x.copy()
    x2[:, d.HD + 2 * d.KVD + 5] = -700.0
    out2 = O.attention_from_qkvg(x2, B, S, d.H, d.Hkv, d.D, w["q_norm_w"], w["k_norm_w"], d.eps, c, s, kv)
    assert np.max(np.abs(out2[:, :, 5])) < 1e-300


# ----------------------------------------------------------------------------- P9 cross precision

def test_fp32_oracle_agrees_with_fp64():
    d = KI.TINY
    h, temb, w, c, s, kv, _ = _tiny_block_inputs()
    o64 = _blk(d, h, temb, w, c, s, kv, dtype=np.float64)
    o32 = _blk(d, h.astype(np.float32), temb.astype(np.float32), w, c, s, kv, dtype=np.float32)
    err = np.max(np.abs(o32 - o64)) / np.max(np.abs(o64))
    assert err < 2e-6, err


# ----------------------------------------------------------------------------- time path / final

def test_timestep_embedding_cos_first_and_scale():
    e0 = O.timestep_embedding(np.array([0.0]), 256)
    np.testing.assert_array_equal(e0[0, :128], np.ones(128))
    np.testing.assert_array_equal(e0[0, 128:], np.zeros(128))
    t = math.pi / 2000.0            # 1000 * t * f_0 = pi/2
    e = O.timestep_embedding(np.array([t]), 256)
    assert abs(e[0, 0]) < 1e-12 and abs(e[0, 128] - 1.0) < 1e-12
    # f_64 = exp(-ln(1e4) * 64/128) = 1e-2
    assert abs(e[0, 64] - math.cos(1000 * t * 1e-2)) < 1e-12
    assert abs(e[0, 128 + 64] - math.sin(1000 * t * 1e-2)) < 1e-12


def test_activations_against_torch():
    x = np.linspace(-9, 9, 1001)
    xt = torch.tensor(x)
    np.testing.assert_allclose(O.gelu_tanh(x), Fn.gelu(xt, approximate="tanh").numpy(), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(O.silu(x), Fn.silu(xt).numpy(), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(O.sigmoid(x), torch.sigmoid(xt).numpy(), rtol=1e-12, atol=1e-14)


def test_time_path_against_torch_modules():
    d = KI.TINY
    mw = KI.model_weights(d)
    t = np.array([0.0, 0.25, 0.9])
    temb, e = O.time_path(t, mw, d.t_dim)
    T = lambda a: torch.tensor(np.asarray(a, dtype=np.float64))
    half = 128
    freqs = torch.exp(-math.log(10000.0) * torch.arange(half, dtype=torch.float64) / half)
    args = 1000.0 * T(t)[:, None] * freqs[None]
    emb = torch.cat([torch.cos(args), torch.sin(args)], dim=1)
    x = Fn.gelu(Fn.linear(emb, T(mw["t1_w"]), T(mw["t1_b"])), approximate="tanh")
    e_ref = Fn.gelu(Fn.linear(x, T(mw["t2_w"]), T(mw["t2_b"])), approximate="tanh")
    temb_ref = Fn.linear(e_ref, T(mw["mod_w"]), T(mw["mod_b"]))
    np.testing.assert_allclose(e, e_ref.numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(temb, temb_ref.numpy(), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("chunk", [0, 1])
def test_final_layer_scale_then_shift(chunk):
    d = KI.TINY
    mw = dict(KI.model_weights(d))
    x = R.standard_normal((1, 5, d.C))
    e = R.standard_normal((1, d.C))
    probe = 0.5 + 0.25 * np.sin(np.arange(d.C))
    tb = -np.stack([e[0], e[0]])
    tb[chunk] += probe
    mw["final_table"] = tb
    out = O.final_layer(x, e, mw, d.eps)
    T = lambda a: torch.tensor(np.asarray(a, dtype=np.float64))
    n = Fn.rms_norm(T(x), (d.C,), weight=1 + T(mw["final_norm_w"]), eps=d.eps)
    n = n * (1 + T(probe)) if chunk == 0 else n + T(probe)
    ref = Fn.linear(n, T(mw["final_w"]), T(mw["final_b"])).numpy()
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)


def test_final_layer_reduces_to_norm_and_linear():
    d = KI.TINY
    mw = dict(KI.model_weights(d))
    x = R.standard_normal((2, 5, d.C))
    e = R.standard_normal((2, d.C))
    mw["final_table"] = np.zeros((2, d.C))
    # table cancels e for scale and shift
    mw_c = dict(mw)
    out_c = []
    for b in range(2):
        mw_c["final_table"] = -np.stack([e[b], e[b]])
        out_c.append(O.final_layer(x[b:b + 1], e[b:b + 1], mw_c, d.eps))
    out_c = np.concatenate(out_c)
    T = lambda a: torch.tensor(np.asarray(a, dtype=np.float64))
    ref = Fn.linear(Fn.rms_norm(T(x), (d.C,), weight=1 + T(mw["final_norm_w"]), eps=d.eps),
                    T(mw["final_w"]), T(mw["final_b"])).numpy()
    np.testing.assert_allclose(out_c, ref, rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------------------- backbone

def _backbone(d, B, T, gh, gw, lengths, layers=None, mw=None, zero_gates=False, text=None, dtype=np.float64):
    N = gh * gw
    mw = KI.model_weights(d) if mw is None else mw
    hidden = KI.latents(d, B, N)
    text = KI.text_states(d, B, T) if text is None else text
    pos = KI.position_ids(T, gh, gw)
    mask = KI.mask_from_lengths(T, lengths)
    t = KI.timesteps(B)
    nl = d.n_layers if layers is None else layers
    bw = lambda i: KI.block_weights(d, i, zero_gates=zero_gates)
    return O.backbone_forward(hidden, text, pos, mask, t, mw, bw, nl, d.H, d.Hkv, d.D, d.axes,
                              d.theta, d.eps, d.t_dim, dtype)


def test_img_in_against_torch_linear_with_bias():
    # img_in = nn.Linear(in_channels, C, bias=True) ([ARCH] module list)
    d = KI.TINY
    mw = KI.model_weights(d)
    x = KI.latents(d, 2, 24).astype(np.float64)
    out = O.img_in(x, mw)
    assert out.shape == (2, 24, d.C)
    W, b = torch.from_numpy(mw["img_in_w"].astype(np.float64)), torch.from_numpy(mw["img_in_b"].astype(np.float64))
    ref = Fn.linear(torch.from_numpy(x), W, b).numpy()
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)
    # negative control: the same check sees a dropped bias
    assert np.max(np.abs(Fn.linear(torch.from_numpy(x), W).numpy() - out)) > 0.05


def test_img_in_of_one_hot_latents_is_a_weight_column_plus_bias():
    d = KI.TINY
    mw = KI.model_weights(d)
    out = O.img_in(np.eye(d.in_ch)[None], mw)[0]          # latent k = e_k
    np.testing.assert_allclose(out, mw["img_in_w"].T.astype(np.float64) + mw["img_in_b"], rtol=1e-15, atol=1e-15)
    np.testing.assert_allclose(O.img_in(np.zeros((1, 3, d.in_ch)), mw)[0], np.tile(mw["img_in_b"], (3, 1)),
                               rtol=0, atol=0)


def test_quickstart_output_shape():
    g = _load("quickstart_shape.json")
    d = KI.with_dims(KI.tiny_block(), in_ch=g["in_channels"], n_layers=1).dims
    out = _backbone(d, g["batch"], g["text_seq"], *g["grid"], lengths=[g["text_seq"]])
    assert list(out.shape) == g["output_shape"]
    assert np.all(np.isfinite(out))


def test_backbone_zero_gates_reduces_to_final_of_img_in():
    d = KI.TINY
    mw = dict(KI.model_weights(d))
    C = d.C
    mw["mod_w"] = mw["mod_w"].copy()
    mw["mod_b"] = mw["mod_b"].copy()
    for k in (2, 5):
        mw["mod_w"][k * C:(k + 1) * C] = 0.0
        mw["mod_b"][k * C:(k + 1) * C] = 0.0
    out = _backbone(d, 1, 8, 8, 8, [6], layers=2, mw=mw, zero_gates=True)
    _, e = O.time_path(KI.timesteps(1), mw, d.t_dim)
    ref = O.final_layer(O.img_in(KI.latents(d, 1, 64), mw), e, mw, d.eps)
    np.testing.assert_array_equal(out, ref)


def test_backbone_ignores_padded_text_features():
    # tiny test config of the architecture page (section 六): head_dim 8, 4 heads, 2 KV heads,
    # in_channels 16, 4 text tokens with the last one padded, 2x2 grid
    d = KI.Dims(C=32, H=4, Hkv=2, D=8, F=64, axes=(2, 2, 4), n_layers=2, in_ch=16)
    text = KI.text_states(d, 1, 4)
    out = _backbone(d, 1, 4, 2, 2, [3], text=text)
    assert out.shape == (1, 4, 16)
    text2 = text.copy()
    text2[0, 3] = R.standard_normal(d.C) * 5
    out2 = _backbone(d, 1, 4, 2, 2, [3], text=text2)
    np.testing.assert_allclose(out2, out, rtol=1e-12, atol=1e-12)
    text3 = text.copy()
    text3[0, 1] += 1.0
    assert np.max(np.abs(_backbone(d, 1, 4, 2, 2, [3], text=text3) - out)) > 1e-6
