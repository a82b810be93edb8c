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


@pytest.mark.parametrize("seed,p_keep", [(3, 0.05), (4, 0.5), (5, 0.9), (6, 0.02)])
def test_attention_bf16_masks_that_split_the_lane_quarters(K2, seed, p_keep):
    # sparse random text masks make the running maxima of different rows grow on different
    # tiles, so some lane quarters rescale O and others do not; the barrier protocol between
    # the softmax warps and the MMA issuer must keep the result exact regardless
    d = KI.FULL
    B, T, gh, gw = 2, 320, 10, 12
    mask = KI.random_keep_mask(B, T, p_keep, key=seed)
    x, w, pos, out = run_attention(K2, d, B, T, gh, gw, mask, torch.bfloat16, key=seed)
    ref = oracle_attention(d, x, w, pos, B, T, gh * gw, mask)
    assert rel_err(out, ref, f"mask seed {seed} keep {p_keep}") < TOL_BF16


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


@pytest.mark.parametrize("grid", [32, 64, 96, 128])
def test_attention_sweep_sampled_rows(K2, grid):
    # the attention-only sweep shapes (512 text tokens, random valid length), rows sampled
    wl = KI.attn_sweep(grid)
    d = wl.dims
    mask = wl.mask()
    x, w, pos, out = run_attention(K2, d, wl.B, wl.T, wl.gh, wl.gw, mask, torch.bfloat16)
    rows = sample_rows(wl.T, wl.S)
    ref = oracle_attention(d, x, w, pos, wl.B, wl.T, wl.N, mask, rows=rows, dtype=np.float32)
    assert rel_err(out[:, rows], ref) < TOL_BF16


@pytest.mark.parametrize("T,length", [(512, 512), (509, 301)])
def test_attention_full_size_whole_cta_tiles(K2, T, length):
    # Full heads at the 1024^2 sequence length: every row (all 48 heads) of the query tiles around the
    # text/image boundary and of the last tiles of the sequence. T = 509 makes S = 4605 ragged: the
    # last tile is partial and a tile straddles the boundary under 32- and 64-position tilings alike.
    d = KI.FULL
    B, gh, gw = 1, 64, 64
    S = T + gh * gw
    mask = KI.mask_from_lengths(T, [length])
    x, w, pos, out = run_attention(K2, d, B, T, gh, gw, mask, torch.bfloat16, key=3)
    lo = (T // 64) * 64
    rows = sorted(set(range(lo - 64, min(lo + 128, S))) | set(range((S // 64) * 64 - 64, S)))
    ref = oracle_attention(d, x, w, pos, B, T, gh * gw, mask, rows=rows, dtype=np.float32)
    assert rel_err(out[:, rows], ref, f"S={S}, {len(rows)} rows") < TOL_BF16


@pytest.mark.parametrize("H,Hkv", [(8, 8), (8, 4), (20, 20)])
def test_attention_bf16_other_group_sizes(K2, H, Hkv):
    # tensor-core path with 1 or 2 query heads per KV head (128 or 64 positions per tile)
    d = KI.Dims(C=H * 128, H=H, Hkv=Hkv, D=128, F=1024, axes=(32, 48, 48))
    B, T, gh, gw = 2, 70, 9, 11
    mask = KI.mask_from_lengths(T, [70, 17])
    x, w, pos, out = run_attention(K2, d, B, T, gh, gw, mask, torch.bfloat16)
    ref = oracle_attention(d, x, w, pos, B, T, gh * gw, mask)
    assert rel_err(out, ref) < TOL_BF16


@pytest.mark.parametrize("segs,lengths", [
    ([("text", 150), ("image", 64), ("text", 30), ("image", 400)], [244, 100]),   # ragged, padded text
    ([("text", 40), ("image", 130), ("image", 70)], [40, 40]),                   # adjacent image blocks
    ([("text", 200)], [200, 1]),                                                  # pure causal text
])
def test_attention_block_causal(K2, segs, lengths):
    d = KI.FULL
    ids = O.image_block_ids(segs)
    S = len(ids)
    B = 2
    T = S  # the whole sequence takes the text mask (image positions marked valid)
    mask = KI.mask_from_lengths(T, lengths)
    for b in range(B):
        mask[b, ids >= 0] = True
    x = KI.qkvg_raw(d, B, S)
    w = KI.block_weights(d, 0)
    pos = np.zeros((S, 3), dtype=np.float32)
    pos[:, 1] = np.arange(S) // 16
    pos[:, 2] = np.arange(S) % 16
    cs = torch.empty(S, 64, device="cuda")
    sn = torch.empty_like(cs)
    K2.rope_tables(d, dev(pos, torch.float32), cs, sn)
    kend = dev(K2.block_causal_key_end(ids), torch.int32)
    out = torch.empty(B * S, d.HD, device="cuda", dtype=torch.bfloat16)
    ws = torch.empty(K2.attention_workspace_size(d, B, T - 1, 1, torch.bfloat16), dtype=torch.uint8, device="cuda")
    # the whole sequence sits under the text mask (T = S, no separate image tokens)
    K2.gqa_attention_block_causal(d, B, T, 0, dev(x, torch.bfloat16), dev(w["q_norm_w"], torch.float32),
                                  dev(w["k_norm_w"], torch.float32), cs, sn, dev(mask.astype(np.uint8), torch.uint8),
                                  kend, out, ws)
    K2.check_device_error()
    c, s = O.rope_cos_sin(pos, d.axes, d.theta)
    xf = x.astype(np.float64).reshape(B, S, -1)
    q = O.apply_rope(O.rms_norm(xf[..., :d.HD].reshape(B, S, d.H, d.D), w["q_norm_w"], d.eps), c, s)
    k = O.apply_rope(O.rms_norm(xf[..., d.HD:d.HD + d.KVD].reshape(B, S, d.Hkv, d.D), w["k_norm_w"], d.eps), c, s)
    v = xf[..., d.HD + d.KVD:d.HD + 2 * d.KVD].reshape(B, S, d.Hkv, d.D)
    g = xf[..., d.HD + 2 * d.KVD:]
    kv = mask
    o = O.masked_attention(q, k, v, O.block_causal_allowed(ids), kv, 1.0 / np.sqrt(d.D))
    ref = o.reshape(B, S, d.HD) * O.sigmoid(g)
    assert rel_err(host(out).reshape(B, S, d.HD), ref) < TOL_BF16


@pytest.mark.parametrize("head,tail,lengths,spare", [
    # the image being denoised after a cached prompt and condition image: every key readable
    ([("text", 300), ("image", 256)], [("image", 1024)], [300, 77], 37),
    # new text and image tokens after the cached prefix: per-token key_end of the pattern
    ([("text", 100), ("image", 128)], [("text", 40), ("image", 200)], [100, 9], 0),
])
def test_attention_kv_cache(K2, head, tail, lengths, spare):
    d = KI.FULL
    ids = O.image_block_ids(head + tail)
    S, P = len(ids), len(O.image_block_ids(head))
    Nq, B = S - P, 2
    cap = S + spare
    last_text = int(np.nonzero(ids < 0)[0].max()) + 1
    T = last_text if tail[0][0] == "image" else S  # keys [0, T) sit under the text mask
    mask = np.ones((B, T), dtype=bool)
    first_text = head[0][1]
    for b, n in enumerate(lengths):
        mask[b, n:first_text] = False  # the prompt is right-padded
    kv = np.ones((B, S), dtype=bool)
    kv[:, :T] = mask
    x = KI.qkvg_raw(d, B, S, key=21)
    w = KI.block_weights(d, 0)
    pos = np.zeros((S, 3), dtype=np.float32)
    pos[:, 1] = np.arange(S) // 32
    pos[:, 2] = np.arange(S) % 32
    cs = torch.empty(S, d.D // 2, device="cuda")
    sn = torch.empty_like(cs)
    K2.rope_tables(d, dev(pos, torch.float32), cs, sn)
    xg = dev(x, torch.bfloat16).view(B, S, -1)
    x_prefix = xg[:, :P].reshape(B * P, -1).contiguous()
    x_new = xg[:, P:].reshape(B * Nq, -1).contiguous()
    qw, kw = dev(w["q_norm_w"], torch.float32), dev(w["k_norm_w"], torch.float32)
    # rows past L hold NaN: a read beyond the cached keys or across batch rows would show
    kc = torch.full((B, cap, d.KVD), float("nan"), device="cuda", dtype=torch.bfloat16)
    vc = torch.full_like(kc, float("nan"))
    K2.kv_cache_append(d, B, P, 0, x_prefix, kw, cs[:P], sn[:P], kc, vc)
    K2.kv_cache_append(d, B, Nq, P, x_new, kw, cs[P:], sn[P:], kc, vc)
    key_end = None if tail == [("image", tail[0][1])] else dev(K2.block_causal_key_end(ids)[P:], torch.int32)
    out = torch.empty(B * Nq, d.HD, device="cuda", dtype=torch.bfloat16)
    ws = torch.empty(K2.kv_cache_attention_workspace_size(d, B, Nq, torch.bfloat16), dtype=torch.uint8, device="cuda")
    K2.gqa_attention_kv_cache(d, B, T, S, Nq, x_new, qw, cs[P:], sn[P:], dev(mask.astype(np.uint8), torch.uint8),
                              kc, vc, key_end, out, ws)
    K2.check_device_error()

    c, s = O.rope_cos_sin(pos, d.axes, d.theta)
    xf = x.astype(np.float64).reshape(B, S, -1)
    q = O.apply_rope(O.rms_norm(xf[..., :d.HD].reshape(B, S, d.H, d.D), w["q_norm_w"], d.eps), c, s)
    k = O.apply_rope(O.rms_norm(xf[..., d.HD:d.HD + d.KVD].reshape(B, S, d.Hkv, d.D), w["k_norm_w"], d.eps), c, s)
    v = xf[..., d.HD + d.KVD:d.HD + 2 * d.KVD].reshape(B, S, d.Hkv, d.D)
    g = xf[:, P:, d.HD + 2 * d.KVD:]
    # the cache: v is the projection copied bit for bit, k the normalised and rotated keys, spare rows untouched
    assert torch.equal(vc[:, :S], xg[..., d.HD + d.KVD:d.HD + 2 * d.KVD])
    assert rel_err(host(kc[:, :S]).reshape(B, S, d.Hkv, d.D), k, "k cache") < TOL_BF16
    assert torch.isnan(kc[:, S:]).all() and torch.isnan(vc[:, S:]).all()
    o = O.cached_step_attention(q[:, P:], k[:, :P], v[:, :P], k[:, P:], v[:, P:], O.block_causal_allowed(ids)[P:],
                                kv, 1.0 / np.sqrt(d.D))
    ref = o.reshape(B, Nq, d.HD) * O.sigmoid(g)
    assert rel_err(host(out).reshape(B, Nq, d.HD), ref, "kv-cache attention") < TOL_BF16
