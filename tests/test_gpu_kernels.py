"""GPU parity of the row kernels and projections against the oracle (or, for a plain matrix
product, a float64 numpy product of the same bf16 operands)."""
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


@pytest.mark.parametrize("T,gh,gw", [(512, 64, 64), (8, 8, 8), (0, 3, 5), (128, 128, 128)])
def test_rope_tables(K2, T, gh, gw):
    d = KI.FULL
    pos = KI.position_ids(T, gh, gw)
    c_ref, s_ref = O.rope_cos_sin(pos, d.axes, d.theta)
    S = pos.shape[0]
    cs = torch.empty(S, 64, device="cuda")
    sn = torch.empty_like(cs)
    K2.rope_tables(d, dev(pos, torch.float32), cs, sn)
    # fp64 evaluation stored as fp32: only the final rounding differs
    assert np.max(np.abs(host(cs) - c_ref)) < 1e-7
    assert np.max(np.abs(host(sn) - s_ref)) < 1e-7


def _bf(shape, seed, scale=1.0):
    g = np.random.default_rng(seed)
    return KI.to_bf16(g.standard_normal(shape).astype(np.float32) * scale)


@pytest.mark.parametrize("M,N,K", [(300, 512, 256), (1152, 6144, 6144), (129, 384, 640), (1, 128, 64)])
def test_linear_store(K2, M, N, K):
    A, W = _bf((M, K), 1), _bf((N, K), 2, K ** -0.5)
    # the output is the first M rows of a buffer whose 40 sentinel rows must stay untouched
    buf = torch.full((M + 40, N), 7.0, device="cuda", dtype=torch.bfloat16)
    out = buf[:M]
    K2.linear(K2.KREA2_EPI_STORE, dev(A, torch.bfloat16), dev(W, torch.bfloat16), out)
    K2.check_device_error()
    ref = A @ W.T  # fp32 BLAS: ~1e-6 relative, far below the bf16 output rounding
    assert rel_err(host(out), ref) < 8e-3
    assert torch.all(buf[M:] == 7.0).item()


def test_linear_store_unaligned_out_rejected(K2):
    """Outputs are written by TMA stores, which need a 16-byte aligned base address."""
    M, N, K = 64, 128, 64
    A, W = _bf((M, K), 1), _bf((N, K), 2, K ** -0.5)
    buf = torch.zeros(M * N + 1, device="cuda", dtype=torch.bfloat16)
    with pytest.raises(K2.Krea2Error):
        K2.linear(K2.KREA2_EPI_STORE, dev(A, torch.bfloat16), dev(W, torch.bfloat16), buf[1:].view(M, N))
    K2.check_device_error()
    assert torch.count_nonzero(buf).item() == 0


@pytest.mark.parametrize("M,F,K", [(200, 256, 128), (1152, 16384, 6144)])
def test_linear_swiglu(K2, M, F, K):
    A, Wg, Wu = _bf((M, K), 3), _bf((F, K), 4, K ** -0.5), _bf((F, K), 5, K ** -0.5)
    Wgu = K2.interleave_gate_up(dev(Wg, torch.bfloat16), dev(Wu, torch.bfloat16)).contiguous()
    buf = torch.full((M + 40, F), 7.0, device="cuda", dtype=torch.bfloat16)
    out = buf[:M]
    K2.linear(K2.KREA2_EPI_SWIGLU, dev(A, torch.bfloat16), Wgu, out)
    K2.check_device_error()
    assert torch.all(buf[M:] == 7.0).item()
    ref = O.silu(A @ Wg.T) * (A @ Wu.T)
    assert rel_err(host(out), ref) < 8e-3


@pytest.mark.parametrize("B,S,N,K,goff", [
    (2, 150, 256, 512, 0),        # ragged rows; a batch boundary inside a 32-row block
    (2, 150, 256, 512, 1),        # the same with gate rows off 16-byte alignment (scalar gate loads)
    (5, 20, 256, 128, 0),         # one 32-row block spans three batch rows
    (1, 60, 384, 64, 0),          # one ragged row tile: 32-row blocks partly and wholly past M
    (2, 4608, 6144, 16384, 0),    # the backbone's down projection at the 1024^2 CFG shape
])
def test_linear_gated_residual(K2, B, S, N, K, goff):
    M = B * S
    A, W = _bf((M, K), 6), _bf((N, K), 7, K ** -0.5)
    h0 = np.random.default_rng(8).standard_normal((M, N)).astype(np.float32)
    mod = np.random.default_rng(9).standard_normal((B, 6, N + 1)).astype(np.float32)
    # h is the first M rows of a buffer with 40 more sentinel rows, which must stay untouched
    hbuf = dev(np.concatenate([h0, np.full((40, N), 7.0, np.float32)]), torch.float32)
    h = hbuf[:M]
    modd = dev(mod, torch.float32)
    # gate = modulation chunk 2 of each batch row (shifted by goff): base at 2(N+1) + goff, batch
    # stride 6(N+1); the odd stride and offset keep gate rows off 16-byte alignment when goff = 1
    W1 = N + 1
    K2.linear(K2.KREA2_EPI_RESID, dev(A, torch.bfloat16), dev(W, torch.bfloat16), h,
              gate=modd.view(-1)[2 * W1 + goff:], rows_per_batch=S, gate_stride=6 * W1)
    K2.check_device_error()
    acc = (A @ W.T).astype(np.float64)
    gate = np.repeat(mod[:, 2, goff:goff + N], S, axis=0)
    ref_delta = gate * acc
    assert rel_err(host(h) - h0, ref_delta) < 1e-3
    assert torch.all(hbuf[M:] == 7.0).item()


def test_linear_gated_residual_unaligned_out_rejected(K2):
    """The residual is updated by TMA reduce-adds, which need a 16-byte aligned fp32 output."""
    M, N, K = 64, 128, 64
    A, W = _bf((M, K), 6), _bf((N, K), 7, K ** -0.5)
    buf = torch.zeros(M * N + 1, device="cuda", dtype=torch.float32)
    h = buf[1:].view(M, N)
    gate = torch.ones(N, device="cuda", dtype=torch.float32)
    with pytest.raises(K2.Krea2Error):
        K2.linear(K2.KREA2_EPI_RESID, dev(A, torch.bfloat16), dev(W, torch.bfloat16), h, gate=gate,
                  rows_per_batch=M, gate_stride=0)
    K2.check_device_error()
    assert torch.count_nonzero(buf).item() == 0


@pytest.mark.parametrize("dtype,tol", [(torch.bfloat16, 8e-3), (torch.float32, 1e-5)])
@pytest.mark.parametrize("chunk", [0, 3])
@pytest.mark.parametrize("B,S", [(2, 333), (2, 1500)])
def test_modulated_rmsnorm(K2, dtype, tol, chunk, B, S):
    d = KI.FULL
    h = KI.residual(d, B, S)
    temb = KI.temb(d, B)
    table = KI._normal(0, (99, 1), (6, d.C), 0.1)
    nw = KI._normal(0, (99, 2), (d.C,), 0.1)
    out = torch.empty(B * S, d.C, device="cuda", dtype=dtype)
    K2.modulated_rmsnorm(d, B, S, dev(h.reshape(B * S, d.C), torch.float32), dev(nw, torch.float32),
                         dev(temb, torch.float32), dev(table, torch.float32), chunk, out)
    mod = O.modulation(temb, table)
    ref = (1 + mod[:, chunk][:, None]) * O.rms_norm(h, nw, d.eps) + mod[:, chunk + 1][:, None]
    assert rel_err(host(out).reshape(B, S, d.C), ref) < tol


@pytest.mark.parametrize("C", [128, 1152, 2560, 4096, 5120, 7168, 8192])
def test_modulated_rmsnorm_widths(K2, C):
    """The norm kernel keeps ceil(C / 1024) float4 per thread in registers: one instantiation
    per width class, 1 to 8 (C = 6144, the model's, is covered above)."""
    d = KI.Dims(C=C, H=C // 128, Hkv=C // 128, D=128, F=256)
    B, S = 2, 37
    h = KI.residual(d, B, S)
    temb = KI.temb(d, B)
    table = KI._normal(0, (98, 1), (6, C), 0.1)
    nw = KI._normal(0, (98, 2), (C,), 0.1)
    out = torch.empty(B * S, C, device="cuda", dtype=torch.float32)
    K2.modulated_rmsnorm(d, B, S, dev(h.reshape(B * S, C), torch.float32), dev(nw, torch.float32),
                         dev(temb, torch.float32), dev(table, torch.float32), 3, out)
    mod = O.modulation(temb, table)
    ref = (1 + mod[:, 3][:, None]) * O.rms_norm(h, nw, d.eps) + mod[:, 4][:, None]
    assert rel_err(host(out).reshape(B, S, C), ref) < TOL_F32


@pytest.mark.parametrize("dims,dtype,tol", [(KI.FULL, torch.bfloat16, 2e-3), (KI.TINY, torch.float32, TOL_F32)])
def test_time_embed(K2, dims, dtype, tol):
    mw_h = KI.model_weights(dims)
    mw = K2.ModelWeights(mw_h, [], dtype, "cuda")
    t = np.array([0.0, 0.37, 1.0], dtype=np.float32)
    B = len(t)
    temb = torch.empty(B, 6 * dims.C, device="cuda")
    e = torch.empty(B, dims.C, device="cuda")
    scratch = torch.empty(B, dims.C, device="cuda")
    K2.time_embed(dims, dev(t, torch.float32), mw, temb, e, scratch)
    temb_ref, e_ref = O.time_path(t, mw_h, dims.t_dim)
    assert rel_err(host(e), e_ref) < tol
    assert rel_err(host(temb), temb_ref) < tol


@pytest.mark.parametrize("dims,dtype,tol", [(KI.FULL, torch.bfloat16, TOL_BF16), (KI.TINY, torch.float32, TOL_F32)])
def test_final_layer(K2, dims, dtype, tol):
    mw_h = KI.model_weights(dims)
    mw = K2.ModelWeights(mw_h, [], dtype, "cuda")
    B, T, N = 2, 37, 200
    S = T + N
    h = KI.residual(dims, B, S)
    e = KI.temb(dims, B)[:, :dims.C]
    vel = torch.empty(B * N, dims.in_ch, device="cuda", dtype=dtype)
    ws_n = K2.final_layer_workspace_size(dims, B, N, dtype)
    ws = torch.empty(ws_n, dtype=torch.uint8, device="cuda") if ws_n else None
    K2.final_layer(dims, B, T, N, dev(h.reshape(B * S, dims.C), torch.float32), dev(e, torch.float32), mw, vel, ws)
    ref = O.final_layer(h[:, T:], e, mw_h, dims.eps)
    assert rel_err(host(vel).reshape(B, N, dims.in_ch), ref) < tol
