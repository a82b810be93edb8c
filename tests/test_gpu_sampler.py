"""GPU parity of the sampler row: the Euler + CFG step kernel and the whole device sampling loop
(krea2_sample) against the oracle's loop over its own backbone."""
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


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("guidance", [0.0, 4.5])
def test_euler_cfg_step(K2, dtype, guidance):
    n = 3 * 4096 + 5
    rng = np.random.default_rng(3)
    x = rng.standard_normal(n).astype(np.float32)
    vc = KI.to_bf16(rng.standard_normal(n).astype(np.float32))
    vu = KI.to_bf16(rng.standard_normal(n).astype(np.float32))
    xd = dev(x, torch.float32)
    xm = torch.empty(2 * n, device="cuda", dtype=dtype)
    tt = torch.empty(2, device="cuda")
    K2.euler_cfg_step(xd, dev(vc, dtype), dev(vu, dtype), guidance, 0.75, 0.5, xm, 2, tt)
    ref = O.euler_step(x.astype(np.float64), O.cfg_combine(vc.astype(np.float64), vu.astype(np.float64), guidance),
                       0.75, 0.5)
    assert rel_err(host(xd), ref) < 1e-6
    m = host(xm).reshape(2, n)
    tol = 8e-3 if dtype == torch.bfloat16 else 1e-6
    assert rel_err(m[0], ref) < tol and rel_err(m[1], ref) < tol
    assert np.all(host(tt) == 0.5)


def run_sample(K2, d, T, gh, gw, len_c, len_u, steps, guidance, dtype, mu):
    N = gh * gw
    mw_h = KI.model_weights(d)
    blocks = [K2.BlockWeights(KI.block_weights(d, i), dtype, "cuda") for i in range(d.n_layers)]
    mw = K2.ModelWeights(mw_h, blocks, dtype, "cuda")
    x0 = KI.latents(d, 1, N)[0]
    tc, tu = KI.text_states(d, 1, T, key=0)[0], KI.text_states(d, 1, T, key=1)[0]
    mc, mu_ = KI.mask_from_lengths(T, [len_c])[0], KI.mask_from_lengths(T, [len_u])[0]
    pos = KI.position_ids(T, gh, gw)
    sig = O.shifted_sigmas(steps, mu).astype(np.float32)   # the oracle's schedule drives both sides
    lat = dev(x0, torch.float32)
    ws = torch.empty(K2.sample_workspace_size(d, T, N, dtype, guidance > 0), dtype=torch.uint8, device="cuda")
    K2.sample(d, T, N, lat, dev(tc, dtype), dev(tu, dtype), dev(mc.astype(np.uint8), torch.uint8),
              dev(mu_.astype(np.uint8), torch.uint8), dev(pos, torch.float32), sig, guidance, mw, ws)
    K2.check_device_error()
    return host(lat), (x0, tc, tu, mc, mu_, pos, sig, mw_h)


def oracle_sample(d, inputs, guidance, dtype):
    x0, tc, tu, mc, mu_, pos, sig, mw_h = inputs
    return O.sample(x0, tc, tu, mc, mu_, pos, sig.astype(np.float64), guidance, mw_h,
                    lambda i: KI.block_weights(d, i), d.n_layers, d.H, d.Hkv, d.D, d.axes, d.theta, d.eps, d.t_dim,
                    dtype)


def test_sample_tiny_fp32_cfg(K2):
    d = KI.TINY  # 2 layers
    out, inputs = run_sample(K2, d, 8, 8, 8, 6, 3, 4, 4.5, torch.float32, O.shift_mu(64))
    ref = oracle_sample(d, inputs, 4.5, np.float64)
    assert rel_err(out, ref) < TOL_F32
    assert rel_err(out - inputs[0], ref - inputs[0]) < TOL_F32 * 10


def test_sample_tiny_fp32_distilled_no_guidance(K2):
    d = KI.TINY
    out, inputs = run_sample(K2, d, 8, 8, 8, 8, 8, 3, 0.0, torch.float32, 1.15)
    ref = oracle_sample(d, inputs, 0.0, np.float64)
    assert rel_err(out, ref) < TOL_F32


def test_sample_bf16_full_width_two_layers(K2):
    d = KI.with_dims(KI.backbone_1024(), n_layers=2).dims
    out, inputs = run_sample(K2, d, 32, 8, 8, 32, 5, 3, 4.5, torch.bfloat16, O.shift_mu(64))
    ref = oracle_sample(d, inputs, 4.5, np.float32)
    assert rel_err(out, ref) < TOL_BF16
    assert rel_err(out - inputs[0], ref - inputs[0]) < 3e-2
