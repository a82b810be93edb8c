"""GPU parity of krea2_block_forward against the oracle block."""
import numpy as np
import pytest
import torch

import krea2_inputs as KI
from gpu_util import TOL_BF16, TOL_BF16_DELTA, TOL_F32, BlockCase, rel_err, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu(cuda_device):
    yield


def test_block_tiny_fp32():
    # tiny single block: 4 heads x 64 over 1 KV head, 8 text tokens (last 2 padded), 8x8 grid
    c = BlockCase(KI.tiny_block(), torch.float32)
    out = c.run_gpu()
    ref = c.oracle(dtype=np.float64)
    assert rel_err(out, ref) < TOL_F32
    assert rel_err(out - c.h, ref - c.h) < TOL_F32 * 10


def test_block_tiny_bf16_simt_attention():
    # the bf16 path with head_dim 64 (SIMT attention, tcgen05 projections)
    c = BlockCase(KI.tiny_block(), torch.bfloat16)
    out = c.run_gpu()
    ref = c.oracle(dtype=np.float64)
    assert rel_err(out, ref) < TOL_BF16
    assert rel_err(out - c.h, ref - c.h) < TOL_BF16_DELTA


@pytest.mark.parametrize("B,T,gh,gw,lengths", [(2, 64, 8, 16, [64, 9]), (1, 0, 5, 7, [])])
def test_block_bf16_full_width_small(B, T, gh, gw, lengths):
    wl = KI.Workload("small", KI.FULL, B=B, T=T, gh=gh, gw=gw, lengths=lengths)
    c = BlockCase(wl, torch.bfloat16)
    out = c.run_gpu()
    ref = c.oracle(dtype=np.float32)
    assert rel_err(out, ref) < TOL_BF16
    assert rel_err(out - c.h, ref - c.h) < TOL_BF16_DELTA


@pytest.mark.parametrize("wl_fn", [KI.block_512, KI.block_1024_cfg])
def test_block_bf16_full_size_sampled_rows(wl_fn):
    wl = wl_fn()
    c = BlockCase(wl, torch.bfloat16)
    out = c.run_gpu()
    rows = sample_rows(wl.T, wl.S)
    ref = c.oracle(rows=rows, dtype=np.float32)
    got = out[:, rows]
    h = c.h[:, rows]
    assert np.all(np.isfinite(out))
    assert rel_err(got, ref) < TOL_BF16
    assert rel_err(got - h, ref - h) < TOL_BF16_DELTA
