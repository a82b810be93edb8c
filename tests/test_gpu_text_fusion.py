"""GPU parity of krea2_text_fusion (Krea2TextFusion + txt_in) against the oracle."""
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


def run(K2, td, B, T, lengths, dtype):
    tw_h = KI.text_fusion_weights(td)
    tw = K2.TextWeights(tw_h, dtype, "cuda")
    ehs = KI.encoder_hidden_states(td, B, T)
    mask = KI.mask_from_lengths(T, lengths)
    out = torch.empty(B, T, td.C, device="cuda", dtype=dtype)
    ws = torch.empty(K2.text_fusion_workspace_size(td, B, T, dtype), dtype=torch.uint8, device="cuda")
    K2.text_fusion(td, B, T, dev(ehs, dtype), dev(mask.astype(np.uint8), torch.uint8), tw, out, ws)
    K2.check_device_error()
    return host(out), (ehs, mask, tw_h)


def oracle(td, inputs, dtype):
    ehs, mask, tw = inputs
    x = O.text_fusion(ehs, mask, tw["layerwise"], tw["layer_w"], tw["refiner"], td.H, td.Hkv, td.D, td.eps, dtype)
    return O.txt_in(x, tw["txt_in_w"], tw["txt_in_b"], dtype)


def test_text_fusion_tiny_fp32(K2):
    td = KI.TINY_TEXT
    out, inputs = run(K2, td, 2, 7, [7, 3], torch.float32)
    assert rel_err(out, oracle(td, inputs, np.float64)) < TOL_F32


def test_text_fusion_full_size_bf16(K2):
    # the pages' sizes: 12 stacked layers of 2560, 20 heads, SwiGLU 6912, 2 + 2 blocks, txt_in to 6144
    td = KI.FULL_TEXT
    out, inputs = run(K2, td, 2, 40, [40, 9], torch.bfloat16)
    ref = oracle(td, inputs, np.float32)
    assert rel_err(out, ref) < TOL_BF16
