"""The two-rank guidance split (flow_matching_stream_b200.cfg_split) driving the CUDA library.

Two gloo ranks run as processes on the one GPU of the test machine. Each runs its guidance
branch's backbone forward through krea2_backbone_forward (rank 0 the conditional prompt, rank 1
the unconditional one), the velocities are exchanged as host tensors by one all-gather per step,
and each rank applies krea2_euler_cfg_step to its own device latents. No kernel of one rank waits
on the other: the only exchange is the host all-gather. Both ranks must end with the same latents,
within the bf16 tolerance of the oracle's sampling loop ([PIPE] guidance_scale: v = cond +
g (cond - uncond)). The NCCL all-gather over NVLink that the module uses on two GPUs is not run
here: this machine has one GPU.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import krea2_inputs as KI
from oracle import krea2_oracle as O
from gpu_util import TOL_BF16, rel_err

pytestmark = pytest.mark.gpu

T, GH, GW, STEPS, G = 32, 8, 8, 3, 4.5
LENGTHS = (32, 5)  # conditional prompt all valid, unconditional prompt 5 valid tokens


def _dims():
    return KI.with_dims(KI.backbone_1024(), n_layers=2).dims


def _host_inputs(d):
    N = GH * GW
    return dict(x0=KI.latents(d, 1, N)[0], text=[KI.text_states(d, 1, T, key=k)[0] for k in (0, 1)],
                mask=[KI.mask_from_lengths(T, [L])[0] for L in LENGTHS], pos=KI.position_ids(T, GH, GW),
                sigmas=O.shifted_sigmas(STEPS, O.shift_mu(N)).astype(np.float32))


def _rank(rank, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=2)
    try:
        import flow_matching_stream_b200 as K2
        from flow_matching_stream_b200.cfg_split import sample_cfg_split
        torch.cuda.set_device(0)
        d = _dims()
        inp = _host_inputs(d)
        N, bf = GH * GW, torch.bfloat16
        blocks = [K2.BlockWeights(KI.block_weights(d, i), bf, "cuda") for i in range(d.n_layers)]
        mw = K2.ModelWeights(KI.model_weights(d), blocks, bf, "cuda")
        text = torch.from_numpy(inp["text"][rank])[None].to("cuda", bf)
        mask = torch.from_numpy(inp["mask"][rank].astype(np.uint8))[None].to("cuda")
        pos = torch.from_numpy(inp["pos"]).to("cuda")
        ws = torch.empty(K2.workspace_size(d, 1, T, N, bf), dtype=torch.uint8, device="cuda")
        vel = torch.empty(1, N, d.in_ch, device="cuda", dtype=bf)
        tt = torch.empty(1, device="cuda")

        def velocity_fn(x, sigma):  # this rank's branch at timestep sigma, returned on the host
            tt.fill_(sigma)
            K2.backbone_forward(d, 1, T, N, x.to(bf)[None].contiguous(), text, pos, mask, tt, mw, vel, ws)
            return vel[0].float().cpu()

        def step_fn(x, vc, vu, sigma, sigma_next):
            K2.euler_cfg_step(x, vc.to("cuda", bf), vu.to("cuda", bf), G, sigma, sigma_next)
            return x

        x = torch.from_numpy(inp["x0"]).to("cuda")
        out = sample_cfg_split(x, [float(s) for s in inp["sigmas"]], velocity_fn, step_fn)
        K2.check_device_error()
        q.put((rank, out.cpu().numpy()))
    finally:
        dist.destroy_process_group()


def test_cfg_split_two_ranks_through_the_cuda_library():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=600) for _ in procs)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    np.testing.assert_array_equal(res[0], res[1])  # both ranks hold the same latents
    d = _dims()
    inp = _host_inputs(d)
    ref = O.sample(inp["x0"], inp["text"][0], inp["text"][1], inp["mask"][0], inp["mask"][1], inp["pos"],
                   inp["sigmas"].astype(np.float64), G, KI.model_weights(d), lambda i: KI.block_weights(d, i),
                   d.n_layers, d.H, d.Hkv, d.D, d.axes, d.theta, d.eps, d.t_dim, np.float32)
    assert rel_err(res[0], ref, "split latents") < TOL_BF16
    assert rel_err(res[0] - inp["x0"], ref - inp["x0"], "split latent change") < 3e-2
