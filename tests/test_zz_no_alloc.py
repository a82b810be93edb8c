"""krea2_gqa_attention_noalloc against krea2_gqa_attention, both called through the C ABI.

The no-allocation entry point serves callers that cannot give the library a workspace, for
example a plugin interface that hands over only input and output buffers, or a runtime whose
allocator owns all device memory. Its q|k scratch is a static device array shared by every
call, so the check runs two calls in a row, the second smaller and with another mask, and
requires each to equal the workspace entry point's result bit for bit: the second call must
not see anything left over from the first.
"""
import ctypes

import numpy as np
import pytest
import torch

import krea2_inputs as KI
from gpu_util import dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def K2(cuda_device):
    import flow_matching_stream_b200 as K2
    return K2


def _inputs(K2, d, B, T, gh, gw, lengths, key):
    N = gh * gw
    S = T + N
    x = dev(KI.qkvg_raw(d, B, S, key=key), torch.bfloat16)
    w = KI.block_weights(d, key)
    qw, kw = dev(w["q_norm_w"], torch.float32), dev(w["k_norm_w"], torch.float32)
    cs = torch.empty(S, d.D // 2, device="cuda")
    sn = torch.empty_like(cs)
    K2.rope_tables(d, dev(KI.position_ids(T, gh, gw), torch.float32), cs, sn)
    mask = dev(KI.mask_from_lengths(T, lengths).astype(np.uint8), torch.uint8)
    return x, qw, kw, cs, sn, mask


def test_noalloc_matches_workspace_entry_point_on_two_calls(K2):
    # Both entry points run the same kernels on the same inputs, so the results must be equal bit for
    # bit. The second call is smaller than the first and has another mask: had it read any scratch left
    # over from the larger call, the outputs would differ.
    d = KI.FULL
    lib = K2.lib()
    dims = K2.dims_struct(d)
    stream = torch.cuda.current_stream().cuda_stream
    cases = ((2, 96, 16, 20, [96, 13], 11), (1, 64, 8, 12, [7], 12))
    for call, (B, T, gh, gw, lengths, key) in enumerate(cases):
        N, S = gh * gw, T + gh * gw
        x, qw, kw, cs, sn, mask = _inputs(K2, d, B, T, gh, gw, lengths, key)
        ref = torch.empty(B * S, d.HD, device="cuda", dtype=torch.bfloat16)
        ws_n = lib.krea2_attention_workspace_size(ctypes.byref(dims), B, T, N, K2.KREA2_BF16)
        ws = torch.empty(ws_n, dtype=torch.uint8, device="cuda")
        rc = lib.krea2_gqa_attention(ctypes.byref(dims), B, T, N, K2.KREA2_BF16, x.data_ptr(), qw.data_ptr(),
                                     kw.data_ptr(), cs.data_ptr(), sn.data_ptr(), mask.data_ptr(), ref.data_ptr(),
                                     ws.data_ptr(), ws_n, stream)
        assert rc == 0, lib.krea2_last_error_string()
        out = torch.full((B * S, d.HD), float("nan"), device="cuda", dtype=torch.bfloat16)
        rc = lib.krea2_gqa_attention_noalloc(ctypes.byref(dims), B, T, N, K2.KREA2_BF16, x.data_ptr(), qw.data_ptr(),
                                             kw.data_ptr(), cs.data_ptr(), sn.data_ptr(), mask.data_ptr(),
                                             out.data_ptr(), stream)
        assert rc == 0, lib.krea2_last_error_string()
        assert lib.krea2_check_device_error(stream) == 0
        assert bool(torch.isfinite(out).all()), f"call {call}"
        assert torch.equal(out, ref), f"call {call}: max |diff| {(out.float() - ref.float()).abs().max().item()}"


def test_noalloc_rejects_shapes_beyond_the_static_scratch(K2):
    d = KI.FULL
    wl = KI.block_1024_cfg()  # 9216 tokens need 141.6 MB of q|k scratch
    lib = K2.lib()
    dims = K2.dims_struct(d)
    out = torch.empty(1, device="cuda")
    rc = lib.krea2_gqa_attention_noalloc(ctypes.byref(dims), wl.B, wl.T, wl.N, K2.KREA2_BF16, out.data_ptr(),
                                         out.data_ptr(), out.data_ptr(), out.data_ptr(), out.data_ptr(), None,
                                         out.data_ptr(), None)
    assert rc == -2
    assert b"static" in lib.krea2_last_error_string()
