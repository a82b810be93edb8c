"""GPU parity of krea2_backbone_forward against the oracle backbone."""
import numpy as np
import pytest
import torch

import krea2_inputs as KI
from oracle import krea2_oracle as O
from gpu_util import TOL_BF16, TOL_F32, dev, host, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def K2(cuda_device):
    import flow_matching_stream_b200 as K2
    return K2


def run_backbone(K2, d, B, T, gh, gw, lengths, dtype, mw_h=None, blocks=None, text=None):
    N = gh * gw
    mw_h = KI.model_weights(d) if mw_h is None else mw_h
    if blocks is None:
        blocks = [K2.BlockWeights(KI.block_weights(d, i), dtype, "cuda") for i in range(d.n_layers)]
    mw = K2.ModelWeights(mw_h, blocks, dtype, "cuda")
    hidden = KI.latents(d, B, N)
    text = KI.text_states(d, B, T) if text is None else text
    pos = KI.position_ids(T, gh, gw)
    mask = KI.mask_from_lengths(T, lengths)
    t = KI.timesteps(B)
    vel = torch.empty(B, N, d.in_ch, device="cuda", dtype=dtype)
    ws = torch.empty(K2.workspace_size(d, B, T, N, dtype), dtype=torch.uint8, device="cuda")
    K2.backbone_forward(d, B, T, N, dev(hidden, dtype), dev(text, dtype), dev(pos, torch.float32),
                        dev(mask.astype(np.uint8), torch.uint8) if T else None, dev(t, torch.float32), mw, vel, ws)
    K2.check_device_error()
    return host(vel), (hidden, text, pos, mask, t, mw_h)


def oracle_backbone(d, inputs, dtype):
    hidden, text, pos, mask, t, mw_h = inputs
    return O.backbone_forward(hidden, text, pos, mask, t, mw_h, lambda i: KI.block_weights(d, i), d.n_layers,
                              d.H, d.Hkv, d.D, d.axes, d.theta, d.eps, d.t_dim, dtype)


def test_backbone_tiny_fp32(K2):
    d = KI.TINY  # 2 layers
    vel, inputs = run_backbone(K2, d, 1, 8, 8, 8, [6], torch.float32)
    ref = oracle_backbone(d, inputs, np.float64)
    assert rel_err(vel, ref) < TOL_F32


def test_backbone_full_width_two_layers_bf16(K2):
    d = KI.with_dims(KI.backbone_1024(), n_layers=2).dims
    vel, inputs = run_backbone(K2, d, 2, 48, 8, 8, [48, 20], torch.bfloat16)
    ref = oracle_backbone(d, inputs, np.float32)
    assert rel_err(vel, ref) < TOL_BF16


def test_backbone_28_layers_full_width_live_gates(K2):
    # All 28 full-width blocks, each with its own seeded weights and live gates, on a short sequence
    # (2 batch rows of 64 text tokens, the second padded to 20 valid, plus an 8x8 image) so that the
    # fp32 oracle finishes in seconds. Tolerance: the per-block bf16 bound, unchanged for the stack.
    d = KI.FULL
    B, T, gh, gw, lengths = 2, 64, 8, 8, [64, 20]
    N = gh * gw
    mw_h = KI.model_weights(d)
    blocks = []

    def block_w(i):  # the oracle draws each block once; the same weights go to the device
        w = KI.block_weights(d, i)
        blocks.append(K2.BlockWeights(w, torch.bfloat16, "cuda"))
        return w
    hidden, text = KI.latents(d, B, N), KI.text_states(d, B, T)
    pos, mask, t = KI.position_ids(T, gh, gw), KI.mask_from_lengths(T, lengths), KI.timesteps(B)
    ref = O.backbone_forward(hidden, text, pos, mask, t, mw_h, block_w, d.n_layers, d.H, d.Hkv, d.D, d.axes,
                             d.theta, d.eps, d.t_dim, np.float32)
    assert len(blocks) == d.n_layers == 28
    vel, _ = run_backbone(K2, d, B, T, gh, gw, lengths, torch.bfloat16, mw_h=mw_h, blocks=blocks)
    assert rel_err(vel, ref, "28 layers, live gates") < TOL_BF16
    # the gates are live: the stack moves the velocity far from that of identity blocks
    _, e = O.time_path(t, mw_h, d.t_dim, np.float32)
    identity = O.final_layer(O.img_in(hidden, mw_h, np.float32), e, mw_h, d.eps, np.float32)
    assert rel_err(identity, ref, "identity blocks vs live") > 0.1
    del blocks
    torch.cuda.empty_cache()


def test_backbone_quickstart_shape(K2):
    # 16 text tokens + 8x8 latent grid -> velocity (1, 64, 64) (quick-start example of the pages)
    d = KI.with_dims(KI.backbone_1024(), n_layers=1).dims
    vel, _ = run_backbone(K2, d, 1, 16, 8, 8, [16], torch.bfloat16)
    assert vel.shape == (1, 64, 64) and np.all(np.isfinite(vel))


def test_backbone_full_size_zero_gates_is_final_of_img_in(K2):
    # full 28-layer backbone at 1024^2; with every block gate at zero the blocks are exactly the
    # identity, so the velocity must equal final_layer(img_in(latents)) of the oracle
    wl = KI.backbone_1024()
    d = wl.dims
    mw_h = dict(KI.model_weights(d))
    C = d.C
    mw_h["mod_w"] = mw_h["mod_w"].copy()
    mw_h["mod_b"] = mw_h["mod_b"].copy()
    for k in (2, 5):
        mw_h["mod_w"][k * C:(k + 1) * C] = 0.0
        mw_h["mod_b"][k * C:(k + 1) * C] = 0.0
    g = torch.Generator(device="cuda").manual_seed(0)
    blocks = []
    for _ in range(d.n_layers):
        b = K2.BlockWeights.random(d, torch.bfloat16, "cuda", g)
        b.table[2].zero_()
        b.table[5].zero_()
        blocks.append(b)
    vel, inputs = run_backbone(K2, d, wl.B, wl.T, wl.gh, wl.gw, wl.lengths, torch.bfloat16, mw_h=mw_h, blocks=blocks)
    hidden, text, pos, mask, t, _ = inputs
    _, e = O.time_path(t, mw_h, d.t_dim, np.float32)
    ref = O.final_layer(O.img_in(hidden, mw_h, np.float32), e, mw_h, d.eps, np.float32)
    assert rel_err(vel, ref) < TOL_BF16
    del blocks
    torch.cuda.empty_cache()


def test_backbone_full_size_runs_finite(K2):
    wl = KI.backbone_1024()
    d = wl.dims
    g = torch.Generator(device="cuda").manual_seed(1)
    blocks = [K2.BlockWeights.random(d, torch.bfloat16, "cuda", g) for _ in range(d.n_layers)]
    vel, _ = run_backbone(K2, d, wl.B, wl.T, wl.gh, wl.gw, wl.lengths, torch.bfloat16, blocks=blocks)
    assert vel.shape == (1, 4096, 64) and np.all(np.isfinite(vel))
    del blocks
    torch.cuda.empty_cache()
