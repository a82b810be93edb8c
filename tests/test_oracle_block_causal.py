"""Pins for the block-causal attention pattern of the QwenImage 2.1 page (NEXT row f4)."""
import math

import numpy as np
import torch
import torch.nn.functional as Fn

from oracle import krea2_oracle as O

R = np.random.default_rng(11)


def test_block_ids_keep_adjacent_images_apart():
    ids = O.image_block_ids([("text", 3), ("image", 4), ("image", 2), ("text", 1), ("image", 5)])
    assert ids.tolist() == [-1] * 3 + [0] * 4 + [1] * 2 + [-1] + [2] * 5


def test_allowed_pattern_small_case_by_hand():
    ids = O.image_block_ids([("text", 2), ("image", 2)])
    a = O.block_causal_allowed(ids).astype(int)
    # text rows are causal; the image rows read each other both ways
    assert a.tolist() == [[1, 0, 0, 0], [1, 1, 0, 0], [1, 1, 1, 1], [1, 1, 1, 1]]


def test_allowed_keys_form_a_prefix():
    # the pattern is a per-query prefix [0, end(q)): end = q + 1 for text, the block end for image
    for _ in range(20):
        segs = [(("text", "image")[R.integers(2)], int(R.integers(1, 6))) for _ in range(R.integers(1, 7))]
        ids = O.image_block_ids(segs)
        a = O.block_causal_allowed(ids)
        S = len(ids)
        for q in range(S):
            end = q + 1
            if ids[q] >= 0:
                end = int(np.nonzero(ids == ids[q])[0].max()) + 1
            assert a[q].tolist() == [k < end for k in range(S)]


def test_text_only_is_causal_sdpa_and_one_block_is_full_attention():
    B, S, H, D = 1, 7, 2, 4
    q, k, v = (R.standard_normal((B, S, H, D)) for _ in range(3))
    kv = np.ones((B, S), dtype=bool)
    causal = O.masked_attention(q, k, v, O.block_causal_allowed(O.image_block_ids([("text", S)])), kv, 0.5)
    ref = Fn.scaled_dot_product_attention(*(torch.tensor(t).transpose(1, 2) for t in (q, k, v)), is_causal=True,
                                          scale=0.5).transpose(1, 2).numpy()
    np.testing.assert_allclose(causal, ref, rtol=1e-12, atol=1e-12)
    full = O.masked_attention(q, k, v, O.block_causal_allowed(O.image_block_ids([("image", S)])), kv, 0.5)
    np.testing.assert_allclose(full, O.attention(q, k, v, kv, 0.5), rtol=1e-12, atol=1e-12)


def test_fully_masked_row_gives_zeros():
    B, S, H, D = 1, 4, 1, 2
    q, k, v = (R.standard_normal((B, S, H, D)) for _ in range(3))
    kv = np.array([[False, True, True, True]])
    out = O.masked_attention(q, k, v, O.block_causal_allowed(O.image_block_ids([("text", S)])), kv, 1.0)
    assert np.all(out[0, 0] == 0.0) and np.all(out[0, 1:] != 0.0)


def _segments_with_tail(tail):
    head = [("text", 9), ("image", 6), ("text", 3), ("image", 5)]
    return head, head + tail


def test_cached_step_equals_the_full_sequence_rows():
    # the cache only saves recomputing the prefix: the new tokens' rows are those of the full pass
    for tail in ([("image", 7)], [("text", 4), ("image", 6)], [("text", 5)]):
        head, segs = _segments_with_tail(tail)
        ids = O.image_block_ids(segs)
        S, P = len(ids), len(O.image_block_ids(head))
        B, H, Hkv, D = 2, 4, 2, 8
        q = R.standard_normal((B, S, H, D))
        k, v = (R.standard_normal((B, S, Hkv, D)) for _ in range(2))
        kv = R.random((B, S)) > 0.2
        allowed = O.block_causal_allowed(ids)
        full = O.masked_attention(q, k, v, allowed, kv, 0.3)
        step = O.cached_step_attention(q[:, P:], k[:, :P], v[:, :P], k[:, P:], v[:, P:], allowed[P:], kv, 0.3)
        assert np.array_equal(step, full[:, P:])


def test_cached_target_block_is_padded_sdpa_with_kv_heads_repeated():
    # the denoised image is the last block: it reads every earlier token and itself, i.e. plain
    # attention over all keys under the key padding mask (torch SDPA with repeat_interleaved KV heads)
    head, segs = _segments_with_tail([("image", 8)])
    ids = O.image_block_ids(segs)
    S, P = len(ids), len(O.image_block_ids(head))
    B, H, Hkv, D = 2, 4, 2, 8
    q = R.standard_normal((B, S - P, H, D))
    k, v = (R.standard_normal((B, S, Hkv, D)) for _ in range(2))
    kv = np.ones((B, S), dtype=bool)
    kv[0, 2:9] = False
    kv[1, 16:18] = False
    out = O.cached_step_attention(q, k[:, :P], v[:, :P], k[:, P:], v[:, P:], O.block_causal_allowed(ids)[P:], kv,
                                  1.0 / math.sqrt(D))
    t = lambda a: torch.tensor(a).transpose(1, 2)
    kr = t(k).repeat_interleave(H // Hkv, dim=1)
    vr = t(v).repeat_interleave(H // Hkv, dim=1)
    ref = Fn.scaled_dot_product_attention(t(q), kr, vr, attn_mask=torch.tensor(kv)[:, None, None, :])
    np.testing.assert_allclose(out, ref.transpose(1, 2).numpy(), rtol=1e-12, atol=1e-12)


def test_cached_step_reads_valid_cache_entries_only():
    head, segs = _segments_with_tail([("image", 5)])
    ids = O.image_block_ids(segs)
    S, P = len(ids), len(O.image_block_ids(head))
    B, H, Hkv, D = 1, 2, 1, 4
    q = R.standard_normal((B, S - P, H, D))
    k, v = (R.standard_normal((B, S, Hkv, D)) for _ in range(2))
    kv = np.ones((B, S), dtype=bool)
    kv[0, 3] = False
    allowed = O.block_causal_allowed(ids)[P:]
    base = O.cached_step_attention(q, k[:, :P], v[:, :P], k[:, P:], v[:, P:], allowed, kv, 0.5)
    kp, vp = k[:, :P].copy(), v[:, :P].copy()
    kp[0, 3] += 10.0
    vp[0, 3] -= 10.0
    assert np.array_equal(O.cached_step_attention(q, kp, vp, k[:, P:], v[:, P:], allowed, kv, 0.5), base)
    kp[0, 4] += 1.0
    assert not np.allclose(O.cached_step_attention(q, kp, vp, k[:, P:], v[:, P:], allowed, kv, 0.5), base)
