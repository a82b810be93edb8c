"""GPU parity of krea2_gqa_attention (raw projection in, gated attention out) against the oracle."""
import numpy as np
import pytest
import torch

import krea2_inputs as KI
from oracle import krea2_oracle as O
from gpu_util import TOL_BF16, TOL_F32, dev, host, rel_err, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def K2(cuda_device):
    import flow_matching_stream_b200 as K2
    return K2


def run_attention(K2, d, B, T, gh, gw, mask, dtype, key=0):
    N = gh * gw
    S = T + N
    x = KI.qkvg_raw(d, B, S, key=key)
    w = KI.block_weights(d, 0)
    pos = KI.position_ids(T, gh, gw)
    cs = torch.empty(S, d.D // 2, device="cuda")
    sn = torch.empty_like(cs)
    K2.rope_tables(d, dev(pos, torch.float32), cs, sn)
    out = torch.empty(B * S, d.HD, device="cuda", dtype=dtype)
    ws_n = K2.attention_workspace_size(d, B, T, N, dtype)
    ws = torch.empty(max(ws_n, 1), dtype=torch.uint8, device="cuda")
    m = dev(mask.astype(np.uint8), torch.uint8) if mask is not None else None
    K2.gqa_attention(d, B, T, N, dev(x, dtype), dev(w["q_norm_w"], torch.float32), dev(w["k_norm_w"], torch.float32),
                     cs, sn, m, out, ws if ws_n else None)
    K2.check_device_error()
    return x, w, pos, host(out).reshape(B, S, d.HD)


def oracle_attention(d, x, w, pos, B, T, N, mask, rows=None, dtype=np.float64):
    c, s = O.rope_cos_sin(pos, d.axes, d.theta)
    kv = O.key_valid_mask(mask, B, T, N)
    return O.attention_from_qkvg(x, B, T + N, d.H, d.Hkv, d.D, w["q_norm_w"], w["k_norm_w"], d.eps, c, s, kv,
                                 rows=rows, dtype=dtype)


def test_attention_tiny_fp32(K2):
    d = KI.TINY
    B, T, gh, gw = 1, 8, 8, 8
    mask = KI.mask_from_lengths(T, [6])
    x, w, pos, out = run_attention(K2, d, B, T, gh, gw, mask, torch.float32)
    ref = oracle_attention(d, x, w, pos, B, T, gh * gw, mask)
    assert rel_err(out, ref) < TOL_F32


@pytest.mark.parametrize("B,T,gh,gw,lengths", [
    (2, 100, 10, 20, [37, 100]),      # ragged: S=300 is no multiple of 32 or 128, partial text tile
    (1, 0, 9, 15, []),               # no text at all
    (2, 256, 8, 16, [1, 129]),       # whole padded text tiles skipped, a tile with a single valid key
    (3, 64, 4, 4, [64, 5, 33]),      # several batch rows, short image
])
def test_attention_bf16_full_heads(K2, B, T, gh, gw, lengths):
    d = KI.FULL
    mask = KI.mask_from_lengths(T, lengths) if T else None
    x, w, pos, out = run_attention(K2, d, B, T, gh, gw, mask, torch.bfloat16)
    ref = oracle_attention(d, x, w, pos, B, T, gh * gw, mask)
    assert rel_err(out, ref) < TOL_BF16


def test_attention_bf16_random_non_prefix_mask(K2):
    d = KI.FULL
    B, T, gh, gw = 2, 300, 12, 12
    mask = KI.random_keep_mask(B, T, 0.3)
    x, w, pos, out = run_attention(K2, d, B, T, gh, gw, mask, torch.bfloat16)
    ref = oracle_attention(d, x, w, pos, B, T, gh * gw, mask)
    assert rel_err(out, ref) < TOL_BF16
    # all text masked except the first token
    mask2 = np.zeros((B, T), dtype=bool)
    mask2[:, 0] = True
    x, w, pos, out = run_attention(K2, d, B, T, gh, gw, mask2, torch.bfloat16, key=1)
    ref = oracle_attention(d, x, w, pos, B, T, gh * gw, mask2)
    assert rel_err(out, ref) < TOL_BF16


def test_attention_bf16_padded_keys_are_ignored(K2):
    # changing padded text k/v in the raw projection must not change any output row
    d = KI.FULL
    B, T, gh, gw = 1, 128, 8, 8
    mask = KI.mask_from_lengths(T, [40])
    S = T + gh * gw
    x, w, pos, out = run_attention(K2, d, B, T, gh, gw, mask, torch.bfloat16)
    x2 = x.copy()
    x2[40:T, d.HD:d.HD + 2 * d.KVD] = 7.0
    cs = torch.empty(S, 64, device="cuda")
    sn = torch.empty_like(cs)
    K2.rope_tables(d, dev(pos, torch.float32), cs, sn)
    out2 = torch.empty(S, d.HD, device="cuda", dtype=torch.bfloat16)
    ws = torch.empty(K2.attention_workspace_size(d, B, T, gh * gw, torch.bfloat16), dtype=torch.uint8, device="cuda")
    K2.gqa_attention(d, B, T, gh * gw, dev(x2, torch.bfloat16), dev(w["q_norm_w"], torch.float32),
                     dev(w["k_norm_w"], torch.float32), cs, sn, dev(mask.astype(np.uint8), torch.uint8), out2, ws)
    np.testing.assert_array_equal(host(out2).reshape(B, S, d.HD), out)


@pytest.mark.parametrize("grid", [32, 64])
def test_attention_sweep_sampled_rows(K2, grid):
    # the attention-only sweep shapes (512 text tokens, random valid length), rows sampled
    wl = KI.attn_sweep(grid)
    d = wl.dims
    mask = wl.mask()
    x, w, pos, out = run_attention(K2, d, wl.B, wl.T, wl.gh, wl.gw, mask, torch.bfloat16)
    rows = sample_rows(wl.T, wl.S)
    ref = oracle_attention(d, x, w, pos, wl.B, wl.T, wl.N, mask, rows=rows, dtype=np.float32)
    assert rel_err(out[:, rows], ref) < TOL_BF16
