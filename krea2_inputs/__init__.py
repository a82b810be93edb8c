"""Seeded synthetic inputs for the Krea 2 single-stream block and backbone.

This module is shared by the CPU oracle (``oracle/``), the tests and ``bench.py``.
It only draws random numbers and lays out shapes; it holds none of the model's
arithmetic (no norm, no RoPE, no attention, no projection).

Recipe (numpy PCG64, one independent stream per tensor):

* weights      seed 0   linear weights ~ N(0,1)/sqrt(fan_in); biases, norm weights and
                        modulation tables ~ N(0, 0.1^2)
* activations  seed 1   residual stream / packed latents / text states ~ N(0,1);
                        the shared modulation vector ``temb`` ~ N(0, 0.5^2)
* masks        seed 2   valid text lengths (right padding) or random keep patterns
* timesteps    seed 3   t ~ U[0, 1]

Every floating-point array is rounded to bf16 (round to nearest even) before either
side sees it, so the oracle and the GPU path read identical values.

Shapes follow the Krea2Transformer2DModel API page ("Parámetros", ``forward``):
hidden_states (B, N, in_channels), position_ids (T + N, 3) with zero text rows and
``(0, h, w)`` image rows in row-major grid order (Krea 2 pipeline page,
``prepare_position_ids``), encoder_attention_mask (B, T) bool, timestep (B,) in [0, 1].
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field, replace
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

SEED_WEIGHTS = 0
SEED_ACTIVATIONS = 1
SEED_MASKS = 2
SEED_TIMESTEPS = 3


@dataclass(frozen=True)
class Dims:
    """Model hyper-parameters (Krea2Transformer2DModel constructor defaults)."""

    C: int = 6144            # hidden size = heads * head_dim
    H: int = 48              # query heads
    Hkv: int = 12            # key/value heads
    D: int = 128             # head dim
    F: int = 16384           # SwiGLU intermediate size
    axes: Tuple[int, int, int] = (32, 48, 48)
    theta: float = 1000.0
    eps: float = 1e-5
    n_layers: int = 28
    in_ch: int = 64
    t_dim: int = 256         # sinusoidal timestep width

    @property
    def HD(self) -> int:
        return self.H * self.D

    @property
    def KVD(self) -> int:
        return self.Hkv * self.D

    @property
    def qkvg_cols(self) -> int:
        return 2 * self.H * self.D + 2 * self.Hkv * self.D


FULL = Dims()
TINY = Dims(C=256, H=4, Hkv=1, D=64, F=512, axes=(16, 24, 24), n_layers=2, in_ch=16)


def to_bf16(x) -> np.ndarray:
    """Round float32 values to the nearest bf16 value (ties to even); returns float32.

    Adds 0x7FFF plus the lowest kept bit to the raw bits and clears the low 16 bits, in
    wrapping 32-bit arithmetic (a new array; the input is left unchanged)."""
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    u = x.view(np.uint32)
    r = (u >> np.uint32(16)) & np.uint32(1)
    r += np.uint32(0x7FFF)
    r += u
    r &= np.uint32(0xFFFF0000)
    return r.view(np.float32).reshape(x.shape)


def bf16_bits(x) -> np.ndarray:
    """Raw bf16 bit patterns (uint16) of already bf16-representable float32 values."""
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    return (x.view(np.uint32) >> 16).astype(np.uint16)


def _rng(seed: int, *key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed, spawn_key=tuple(key))))


def _normal(seed: int, key: Sequence[int], shape, std: float) -> np.ndarray:
    g = _rng(seed, *key)
    a = g.standard_normal(int(np.prod(shape)), dtype=np.float32).reshape(shape)
    a *= np.float32(std)
    return to_bf16(a)


# tensor ids inside one block's weight stream
_BLOCK_TENSORS = ("wq", "wk", "wv", "wg", "wo", "w_gate", "w_up", "w_down",
                  "norm1_w", "norm2_w", "q_norm_w", "k_norm_w", "table")


def block_weights(d: Dims, layer: int = 0, seed: int = SEED_WEIGHTS,
                  zero_gates: bool = False) -> Dict[str, np.ndarray]:
    """One block's weights in the model's own (unpacked) layout, float32 bf16-valued.

    Linear weights are (out_features, in_features) like ``nn.Linear``.
    ``zero_gates`` zeroes the pregate/postgate rows of the modulation table (used by
    tests that make a block the identity together with a zero shared ``temb`` gate).
    """
    C, HD, KVD, F, D = d.C, d.HD, d.KVD, d.F, d.D
    shapes = {
        "wq": ((HD, C), C ** -0.5), "wk": ((KVD, C), C ** -0.5), "wv": ((KVD, C), C ** -0.5),
        "wg": ((HD, C), C ** -0.5), "wo": ((C, HD), HD ** -0.5),
        "w_gate": ((F, C), C ** -0.5), "w_up": ((F, C), C ** -0.5), "w_down": ((C, F), F ** -0.5),
        "norm1_w": ((C,), 0.1), "norm2_w": ((C,), 0.1),
        "q_norm_w": ((D,), 0.1), "k_norm_w": ((D,), 0.1), "table": ((6, C), 0.1),
    }
    # every tensor has its own stream, so drawing them on threads (numpy releases the GIL while it
    # fills an array) gives the same values as drawing them in turn
    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        futs = {name: ex.submit(_normal, seed, (layer, i), *shapes[name]) for i, name in enumerate(_BLOCK_TENSORS)}
        out = {name: futs[name].result() for name in _BLOCK_TENSORS}
    if zero_gates:
        out["table"][2] = 0.0
        out["table"][5] = 0.0
    return out


_MODEL_TENSORS = ("img_in_w", "img_in_b", "t1_w", "t1_b", "t2_w", "t2_b",
                  "mod_w", "mod_b", "final_norm_w", "final_table", "final_w", "final_b")


def model_weights(d: Dims, seed: int = SEED_WEIGHTS) -> Dict[str, np.ndarray]:
    """Backbone weights outside the blocks (img_in, time path, final layer)."""
    C = d.C
    shapes = {
        "img_in_w": ((C, d.in_ch), d.in_ch ** -0.5), "img_in_b": ((C,), 0.1),
        "t1_w": ((C, d.t_dim), d.t_dim ** -0.5), "t1_b": ((C,), 0.1),
        "t2_w": ((C, C), C ** -0.5), "t2_b": ((C,), 0.1),
        "mod_w": ((6 * C, C), C ** -0.5), "mod_b": ((6 * C,), 0.1),
        "final_norm_w": ((C,), 0.1), "final_table": ((2, C), 0.1),
        "final_w": ((d.in_ch, C), C ** -0.5), "final_b": ((d.in_ch,), 0.1),
    }
    out = {}
    for i, name in enumerate(_MODEL_TENSORS):
        shape, std = shapes[name]
        out[name] = _normal(seed, (10_000, i), shape, std)
    return out


@dataclass(frozen=True)
class TextDims:
    """Text-fusion hyper-parameters ([API] text_hidden_dim 2560, num_text_layers 12,
    text_num_attention_heads / text_num_key_value_heads 20, text_intermediate_size 6912,
    num_layerwise_text_blocks 2, num_refiner_text_blocks 2); C is the backbone hidden size."""

    Dt: int = 2560
    L: int = 12
    H: int = 20
    Hkv: int = 20
    D: int = 128
    F: int = 6912
    n_layerwise: int = 2
    n_refiner: int = 2
    C: int = 6144
    eps: float = 1e-5

    def block_dims(self) -> Dims:
        # a fusion block has the shapes of a backbone block of hidden size Dt (no RoPE is applied)
        return Dims(C=self.Dt, H=self.H, Hkv=self.Hkv, D=self.D, F=self.F, axes=(self.D // 4, 3 * self.D // 8,
                                                                                  3 * self.D // 8), eps=self.eps)


FULL_TEXT = TextDims()
TINY_TEXT = TextDims(Dt=128, L=3, H=2, Hkv=2, D=64, F=256, n_layerwise=1, n_refiner=1, C=256)


def text_fusion_weights(td: TextDims, seed: int = SEED_WEIGHTS) -> Dict[str, object]:
    """Layerwise and refiner block weights, the layer-axis projection (L,) and txt_in (C, Dt) + bias."""
    bd = td.block_dims()
    layerwise = [block_weights(bd, 20_000 + i, seed) for i in range(td.n_layerwise)]
    refiner = [block_weights(bd, 21_000 + i, seed) for i in range(td.n_refiner)]
    for w in layerwise + refiner:
        del w["table"]
    return {"layerwise": layerwise, "refiner": refiner,
            "layer_w": _normal(seed, (22_000, 0), (td.L,), td.L ** -0.5),
            "txt_in_w": _normal(seed, (22_000, 1), (td.C, td.Dt), td.Dt ** -0.5),
            "txt_in_b": _normal(seed, (22_000, 2), (td.C,), 0.1)}


def encoder_hidden_states(td: TextDims, B: int, T: int, seed: int = SEED_ACTIVATIONS, key: int = 0) -> np.ndarray:
    """Stacked text-encoder hidden states (B, T, L, Dt) ~ N(0, 1)."""
    return _normal(seed, (key, 5), (B, T, td.L, td.Dt), 1.0)


def residual(d: Dims, B: int, S: int, seed: int = SEED_ACTIVATIONS, key: int = 0) -> np.ndarray:
    """Residual stream h (B, S, C) ~ N(0, 1)."""
    return _normal(seed, (key, 0), (B, S, d.C), 1.0)


def temb(d: Dims, B: int, seed: int = SEED_ACTIVATIONS, key: int = 0) -> np.ndarray:
    """Shared modulation vector (B, 6C) ~ N(0, 0.5^2), standing in for the time path output."""
    return _normal(seed, (key, 1), (B, 6 * d.C), 0.5)


def latents(d: Dims, B: int, N: int, seed: int = SEED_ACTIVATIONS, key: int = 0) -> np.ndarray:
    """Packed noisy latents hidden_states (B, N, in_ch) ~ N(0, 1)."""
    return _normal(seed, (key, 2), (B, N, d.in_ch), 1.0)


def text_states(d: Dims, B: int, T: int, seed: int = SEED_ACTIVATIONS, key: int = 0) -> np.ndarray:
    """Post-fusion text features (B, T, C) ~ N(0, 1)."""
    return _normal(seed, (key, 3), (B, T, d.C), 1.0)


def qkvg_raw(d: Dims, B: int, S: int, seed: int = SEED_ACTIVATIONS, key: int = 0) -> np.ndarray:
    """Raw (pre-norm, pre-RoPE) fused projection output (B*S, 2*H*D + 2*Hkv*D) ~ N(0, 1)."""
    return _normal(seed, (key, 4), (B * S, d.qkvg_cols), 1.0)


def timesteps(B: int, seed: int = SEED_TIMESTEPS, key: int = 0) -> np.ndarray:
    g = _rng(seed, key)
    return to_bf16(g.random(B, dtype=np.float64).astype(np.float32))


def mask_from_lengths(T: int, lengths: Sequence[int]) -> np.ndarray:
    """Right-padded text mask (B, T) bool: the first ``lengths[b]`` tokens are valid."""
    m = np.zeros((len(lengths), T), dtype=bool)
    for b, L in enumerate(lengths):
        m[b, :L] = True
    return m


def random_lengths(B: int, lo: int, hi: int, seed: int = SEED_MASKS, key: int = 0) -> List[int]:
    """Valid lengths ~ U{lo, ..., hi} (inclusive)."""
    g = _rng(seed, key)
    return [int(v) for v in g.integers(lo, hi + 1, size=B)]


def random_keep_mask(B: int, T: int, p_keep: float = 0.6, seed: int = SEED_MASKS, key: int = 1) -> np.ndarray:
    """Non-prefix random text mask (B, T) bool, at least one valid token per row."""
    g = _rng(seed, key)
    m = g.random((B, T)) < p_keep
    m[:, 0] = True
    return m


def position_ids(T: int, gh: int, gw: int) -> np.ndarray:
    """(T + gh*gw, 3) float32: text rows (0,0,0), image rows (0, h, w), token n = h*gw + w."""
    pos = np.zeros((T + gh * gw, 3), dtype=np.float32)
    hh, ww = np.meshgrid(np.arange(gh), np.arange(gw), indexing="ij")
    pos[T:, 1] = hh.reshape(-1)
    pos[T:, 2] = ww.reshape(-1)
    return pos


@dataclass
class Workload:
    """A named synthetic workload: shapes plus the mask recipe."""

    name: str
    dims: Dims
    B: int
    T: int
    gh: int
    gw: int
    lengths: List[int] = field(default_factory=list)
    dtype: str = "bf16"

    @property
    def N(self) -> int:
        return self.gh * self.gw

    @property
    def S(self) -> int:
        return self.T + self.N

    @property
    def M(self) -> int:
        return self.B * self.S

    def mask(self) -> np.ndarray:
        if self.T == 0:
            return np.ones((self.B, 0), dtype=bool)
        return mask_from_lengths(self.T, self.lengths)

    def positions(self) -> np.ndarray:
        return position_ids(self.T, self.gh, self.gw)


def tiny_block() -> Workload:
    """Tiny single block, fp32: T=8 with the last 2 text tokens padded, 8x8 image grid."""
    return Workload("tiny_block_fp32", TINY, B=1, T=8, gh=8, gw=8, lengths=[6], dtype="f32")


def block_512() -> Workload:
    """One full-size block at 512^2: 32x32 image tokens + 128 text tokens, valid length ~ U[16,128]."""
    return Workload("block_512sq_b1", FULL, B=1, T=128, gh=32, gw=32,
                    lengths=random_lengths(1, 16, 128))


def block_1024_cfg() -> Workload:
    """One full-size block at 1024^2 with CFG: B=2, 512 text tokens (cond all valid, uncond 8 valid)."""
    return Workload("block_1024sq_cfg_b2", FULL, B=2, T=512, gh=64, gw=64, lengths=[512, 8])


def backbone_1024() -> Workload:
    """Full 28-layer backbone at 1024^2, batch 1, 512 text tokens (all valid)."""
    return Workload("backbone_1024sq_b1", FULL, B=1, T=512, gh=64, gw=64, lengths=[512])


def attn_sweep(grid: int) -> Workload:
    """Attention-only sweep point: grid x grid image tokens + 512 text tokens, random valid length."""
    return Workload(f"attn_{grid}sq", FULL, B=1, T=512, gh=grid, gw=grid,
                    lengths=random_lengths(1, 1, 512, key=grid))


def with_dims(w: Workload, **kw) -> Workload:
    return replace(w, dims=replace(w.dims, **kw))
