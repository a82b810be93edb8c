"""Classifier-free guidance split across two ranks (one process per GPU).

With guidance the sampler needs two backbone forwards per step, one for the conditional and
one for the unconditional prompt ([PIPE] "Krea 2" page, guidance_scale: v = cond + g (cond -
uncond)). They are independent, so two GPUs can each run one. Rank 0 takes the conditional
branch and rank 1 the unconditional one. After every step one all-gather exchanges the two
velocity tensors ((N, in_ch), 512 KB in bf16 at 1024^2). Both ranks then apply the same
Euler + CFG update and so keep identical latents, with no further exchange.

This module only orchestrates. `velocity_fn` runs the rank's backbone forward and `step_fn`
the Euler + CFG update. On GPUs these are the library's krea2_backbone_forward and
krea2_euler_cfg_step, and the all-gather goes over NCCL on NVLink. No kernel reads another
GPU's memory.
"""
from __future__ import annotations

from typing import Callable, Sequence

import torch
import torch.distributed as dist


def sample_cfg_split(x: torch.Tensor, sigmas: Sequence[float], velocity_fn: Callable[[torch.Tensor, float], torch.Tensor],
                     step_fn: Callable[[torch.Tensor, torch.Tensor, torch.Tensor, float, float], torch.Tensor],
                     group=None) -> torch.Tensor:
    """Run the sampling loop with the two guidance branches on the two ranks of `group`.

    x: the rank's copy of the latents (identical on both ranks at entry). velocity_fn(x, sigma)
    returns this rank's branch velocity: conditional on rank 0, unconditional on rank 1.
    step_fn(x, v_cond, v_uncond, sigma, sigma_next) returns the next latents.
    Returns the final latents (identical on both ranks)."""
    if dist.get_world_size(group) != 2:
        raise ValueError("the guidance split needs exactly two ranks")
    for i in range(len(sigmas) - 1):
        v = velocity_fn(x, float(sigmas[i])).contiguous()
        both = [torch.empty_like(v), torch.empty_like(v)]
        dist.all_gather(both, v, group=group)
        x = step_fn(x, both[0], both[1], float(sigmas[i]), float(sigmas[i + 1]))
    return x
