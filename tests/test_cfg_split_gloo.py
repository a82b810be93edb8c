"""The two-rank guidance split (flow_matching_stream_b200.cfg_split) on CPU ranks over gloo: each
rank runs one guidance branch through the oracle backbone, velocities are exchanged with one
all-gather per step, and both ranks must end with the latents of the single-process loop."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import krea2_inputs as KI
from oracle import krea2_oracle as O

D = KI.TINY
T, GH, GW, STEPS, G = 8, 4, 4, 3, 4.5


def _inputs():
    N = GH * GW
    return dict(x0=KI.latents(D, 1, N)[0].astype(np.float64),
                text=[KI.text_states(D, 1, T, key=0)[0], KI.text_states(D, 1, T, key=1)[0]],
                mask=[KI.mask_from_lengths(T, [8])[0], KI.mask_from_lengths(T, [3])[0]],
                pos=KI.position_ids(T, GH, GW), mw=KI.model_weights(D),
                sigmas=O.shifted_sigmas(STEPS, O.shift_mu(N)))


def _velocity(inp, branch, x, sigma):
    return O.backbone_forward(x[None], inp["text"][branch][None], inp["pos"], inp["mask"][branch][None],
                              np.array([sigma]), inp["mw"], lambda i: KI.block_weights(D, i), D.n_layers, D.H,
                              D.Hkv, D.D, D.axes, D.theta, D.eps, D.t_dim, np.float64)[0]


def _rank(rank, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=2)
    try:
        from flow_matching_stream_b200.cfg_split import sample_cfg_split
        inp = _inputs()
        vel = lambda x, s: torch.from_numpy(_velocity(inp, rank, x.numpy(), s))
        step = lambda x, vc, vu, s, sn: torch.from_numpy(
            O.euler_step(x.numpy(), O.cfg_combine(vc.numpy(), vu.numpy(), G), s, sn))
        out = sample_cfg_split(torch.from_numpy(inp["x0"]), inp["sigmas"], vel, step)
        q.put((rank, out.numpy()))
    finally:
        dist.destroy_process_group()


def test_cfg_split_over_two_gloo_ranks_matches_the_single_process_loop():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    inp = _inputs()
    ref = O.sample(inp["x0"], inp["text"][0], inp["text"][1], inp["mask"][0], inp["mask"][1], inp["pos"],
                   inp["sigmas"], G, inp["mw"], lambda i: KI.block_weights(D, i), D.n_layers, D.H, D.Hkv, D.D,
                   D.axes, D.theta, D.eps, D.t_dim, np.float64)
    np.testing.assert_array_equal(res[0], res[1])             # both ranks hold the same latents
    np.testing.assert_allclose(res[0], ref, rtol=1e-12, atol=1e-12)
