"""CPU oracle for the Krea 2 single-stream MMDiT block and 28-layer backbone.

TEST INFRASTRUCTURE ONLY. This is a plain, slow, obviously-correct numpy restatement of
what the pages define. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference leg of ``bench.py`` may import it. The CUDA library never
calls it and shares no code with it; the two meet only through the seeded inputs of
``krea2_inputs``.

Sources (cited below by these short names):

* [API]  page "Krea2Transformer2DModel" (diffusers v0.43.0 API docs): constructor
  defaults, "Parámetros", ``forward`` argument contract.
* [ARCH] page "Diffusers 中的 Krea2Transformer2DModel：Krea 2 单流 MMDiT 流匹配
  Transformer 架构全解": §二 I/O contract, §三 defaults and the head-split check,
  §四 module list and data flow, §四.2 TransformerBlock, §四.3 Attention, §四.4 RMSNorm,
  §四.5 TimestepEmbedding, §四.6 FinalLayer, §七 quick start.
* [PIPE] page "Krea 2" (Krea2Pipeline docs): ``prepare_position_ids``, the scheduler shift,
  guidance and the sampling loop.
* page "QwenImage21Transformer2DModel": the block-causal attention pattern and the key/value
  cache of that variant (cited by name where used).

Precision: ``dtype=np.float64`` runs everything in fp64 (tiny config); ``np.float32``
runs the projections in fp32 and every softmax in fp64 (full size). Softmax is always
an explicit normalised exponential over all valid keys of the row, never tiled.

Readings where the pages are silent or garbled (the extraction of [ARCH] dropped the
``+``, ``=`` operators of its block pseudo-code) are marked READING below.

Parity status: every function here is pinned against closed forms, invariants, library
routines or brute force: the block, backbone and their parts (``img_in`` included) by
``tests/test_oracle_pins.py``, the sampler pieces and the sampling loop (``sample_loop``
against exact flows, ``sample``'s wiring of the two prompts) by
``tests/test_oracle_sampler.py``, text fusion by
``tests/test_oracle_text_fusion.py``, and the block-causal pattern and cached step by
``tests/test_oracle_block_causal.py``. Agreement with the trained
Krea 2 model itself is *unpinned*: no weights or reference outputs are available, and
the RoPE pairing convention (READING in ``apply_rope``) cannot be told apart from the
rotate-half alternative by any invariant.
"""
from __future__ import annotations

import math
from typing import Callable, Dict, Optional, Sequence, Tuple

import numpy as np


def check_dims(D: int, axes: Sequence[int], H: int, Hkv: int) -> None:
    """[ARCH] §三: sum(axes_dims_rope) must equal attention_head_dim, else ValueError.

    GQA also needs H to be a multiple of Hkv ([API] num_key_value_heads).
    """
    if sum(axes) != D:
        raise ValueError(f"sum(axes_dims_rope)={sum(axes)} != attention_head_dim={D}")
    if any(a % 2 for a in axes):
        raise ValueError("every RoPE axis needs an even number of dims")
    if H % Hkv:
        raise ValueError(f"num_attention_heads={H} is not a multiple of num_key_value_heads={Hkv}")


def check_positions(pos: np.ndarray, S: Optional[int] = None) -> None:
    """[ARCH] §二: position_ids must be 2-D with last dim 3, else ValueError."""
    if pos.ndim != 2 or pos.shape[1] != 3:
        raise ValueError(f"position_ids must have shape (T+N, 3), got {pos.shape}")
    if S is not None and pos.shape[0] != S:
        raise ValueError(f"position_ids has {pos.shape[0]} rows, sequence has {S}")


# ----------------------------------------------------------------------------- basics

def rms_norm(x: np.ndarray, w: np.ndarray, eps: float, dtype=np.float64) -> np.ndarray:
    """Krea2RMSNorm ([ARCH] §四.4; eps from [API] norm_eps).

    y = x * (mean(x^2 over the last axis) + eps)^(-1/2) * (1 + w): the effective multiplier
    is ``1 + weight`` (weight zero-initialised in the model), computed in float.
    """
    xf = x.astype(dtype)
    ms = np.mean(xf * xf, axis=-1, keepdims=True)
    return xf / np.sqrt(ms + dtype(eps)) * (dtype(1.0) + w.astype(dtype))


def gelu_tanh(x: np.ndarray) -> np.ndarray:
    """GELU, tanh approximation ([ARCH] §四.5): 0.5x(1 + tanh(sqrt(2/pi)(x + 0.044715x^3)))."""
    c = np.asarray(math.sqrt(2.0 / math.pi), dtype=x.dtype)
    return 0.5 * x * (1.0 + np.tanh(c * (x + np.asarray(0.044715, x.dtype) * x * x * x)))


def silu(x: np.ndarray) -> np.ndarray:
    """SiLU x * sigmoid(x), the gate activation of SwiGLU ([ARCH] §三 intermediate_size)."""
    return x / (1.0 + np.exp(-x))


def sigmoid(x: np.ndarray) -> np.ndarray:
    """Logistic sigmoid used by the attention output gate ([ARCH] §四.3)."""
    return 1.0 / (1.0 + np.exp(-x))


# ----------------------------------------------------------------------------- RoPE

def rope_angles(pos: np.ndarray, axes: Sequence[int], theta: float) -> np.ndarray:
    """Rotation angles (S, D/2) in fp64 for 3-axis (t, h, w) RoPE.

    [API] axes_dims_rope splits head_dim between the axes (t, h, w); rope_theta is the base.
    [ARCH] §一: the rotary embedding is adapted from Flux's FluxPosEmbed.
    READING: axis a with d_a dims owns d_a/2 rotated pairs; pair j of axis a turns by
    pos_a * theta^(-2j/d_a). Axis blocks are laid out in order t, h, w along head_dim.
    """
    pos = np.asarray(pos, dtype=np.float64)
    cols = []
    for a, d_a in enumerate(axes):
        j = np.arange(d_a // 2, dtype=np.float64)
        inv_freq = float(theta) ** (-2.0 * j / d_a)
        cols.append(pos[:, a:a + 1] * inv_freq[None, :])
    return np.concatenate(cols, axis=1)


def rope_cos_sin(pos: np.ndarray, axes: Sequence[int], theta: float) -> Tuple[np.ndarray, np.ndarray]:
    """cos and sin of ``rope_angles`` (S, D/2), fp64."""
    ang = rope_angles(pos, axes, theta)
    return np.cos(ang), np.sin(ang)


def apply_rope(x: np.ndarray, cos: np.ndarray, sin: np.ndarray) -> np.ndarray:
    """Rotate q or k: x (..., S, heads, D), cos/sin (S, D/2).

    READING (FluxPosEmbed convention, [ARCH] §一): adjacent dims (2p, 2p+1) form pair p;
    x'_{2p} = x_{2p} cos - x_{2p+1} sin, x'_{2p+1} = x_{2p+1} cos + x_{2p} sin.
    """
    c = cos.astype(x.dtype)[:, None, :]
    s = sin.astype(x.dtype)[:, None, :]
    x0 = x[..., 0::2]
    x1 = x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = x0 * c - x1 * s
    out[..., 1::2] = x1 * c + x0 * s
    return out


# ----------------------------------------------------------------------------- attention

def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, key_valid: np.ndarray,
              scale: float) -> np.ndarray:
    """Masked grouped-query softmax attention ([ARCH] §四.3).

    q (B, Sq, H, D); k, v (B, S, Hkv, D); key_valid (B, S) bool. Query head h reads KV head
    h // (H/Hkv): the page's processor repeat_interleave's K/V heads, so consecutive query
    heads share a KV head. Masked keys are left out of the softmax entirely (the same as a
    -inf score). READING: scale = 1/sqrt(D) (the SDPA default; the pages give none).
    Returns fp64 (B, Sq, H, D).
    """
    B, Sq, H, D = q.shape
    Hkv = k.shape[2]
    G = H // Hkv
    out = np.empty((B, Sq, H, D), dtype=np.float64)
    for b in range(B):
        idx = np.nonzero(key_valid[b])[0]
        if idx.size == 0:
            raise ValueError("a batch row has no valid key")
        for h in range(H):
            j = h // G
            kk = k[b, idx, j, :]
            vv = v[b, idx, j, :].astype(np.float64)
            s = (q[b, :, h, :] @ kk.T).astype(np.float64) * scale
            s -= s.max(axis=1, keepdims=True)
            p = np.exp(s)
            p /= p.sum(axis=1, keepdims=True)
            out[b, :, h, :] = p @ vv
    return out


def key_valid_mask(text_mask: Optional[np.ndarray], B: int, T: int, N: int) -> np.ndarray:
    """Key mask over the joint [text, image] sequence ([API] encoder_attention_mask).

    Text keys follow the bool mask (None = all valid); image keys are always valid.
    READING: the mask only removes keys; padded text rows are still computed as queries.
    """
    km = np.ones((B, T + N), dtype=bool)
    if text_mask is not None:
        km[:, :T] = np.asarray(text_mask, dtype=bool)
    return km


def attention_from_qkvg(qkvg: np.ndarray, B: int, S: int, H: int, Hkv: int, D: int,
                        q_norm_w: np.ndarray, k_norm_w: np.ndarray, eps: float,
                        cos: np.ndarray, sin: np.ndarray, key_valid: np.ndarray,
                        rows: Optional[Sequence[int]] = None, dtype=np.float64) -> np.ndarray:
    """Krea2AttnProcessor from the fused projection output up to (not incl.) ``to_out``.

    qkvg (B*S, H*D + 2*Hkv*D + H*D) holds [q | k | v | gate] columns, head-major inside
    each block. Steps ([ARCH] §四.3): per-head RMSNorm of q and k over head_dim (weights of
    shape (D,), shared by all heads); RoPE; GQA softmax attention; merge heads; multiply by
    sigmoid(gate). ``rows`` selects query positions (same for every batch row).
    Returns (B, R, H*D) in ``dtype``.
    """
    HD, KVD = H * D, Hkv * D
    x = qkvg.astype(dtype).reshape(B, S, -1)
    qsel = np.arange(S) if rows is None else np.asarray(rows)
    q = x[:, qsel, :HD].reshape(B, len(qsel), H, D)
    k = x[:, :, HD:HD + KVD].reshape(B, S, Hkv, D)
    v = x[:, :, HD + KVD:HD + 2 * KVD].reshape(B, S, Hkv, D)
    g = x[:, qsel, HD + 2 * KVD:]
    q = rms_norm(q, q_norm_w, eps, dtype)
    k = rms_norm(k, k_norm_w, eps, dtype)
    q = apply_rope(q, cos[qsel], sin[qsel])
    k = apply_rope(k, cos, sin)
    o = attention(q, k, v, key_valid, 1.0 / math.sqrt(D)).astype(dtype)
    return o.reshape(B, len(qsel), HD) * sigmoid(g)


# ----------------------------------------------------------------------------- block

MOD_NAMES = ("prescale", "preshift", "pregate", "postscale", "postshift", "postgate")


def modulation(temb: np.ndarray, table: np.ndarray, dtype=np.float64) -> np.ndarray:
    """Shared modulation plus the block's additive table ([ARCH] §一, §四.2).

    temb (B, 6C) is unflattened to (B, 6, C) and the block's scale_shift_table (6, C) is
    added. READING: chunk order prescale, preshift, pregate, postscale, postshift, postgate
    (the unbind order printed in §四.2).
    """
    B = temb.shape[0]
    C = table.shape[1]
    return temb.astype(dtype).reshape(B, 6, C) + table.astype(dtype)[None]


def block_forward(h: np.ndarray, temb: np.ndarray, w: Dict[str, np.ndarray],
                  cos: np.ndarray, sin: np.ndarray, key_valid: np.ndarray,
                  H: int, Hkv: int, D: int, eps: float,
                  rows: Optional[Sequence[int]] = None, dtype=np.float64) -> np.ndarray:
    """Krea2TransformerBlock.forward ([ARCH] §四.2, §四.3).

    READING of the garbled pseudo-code (operators lost in extraction):
      xn   = (1 + prescale) * norm1(h) + preshift
      h1   = h + pregate * attn(xn)
      xn2  = (1 + postscale) * norm2(h1) + postshift
      out  = h1 + postgate * ff(xn2),   ff(x) = W_down(silu(W_gate x) * W_up x)
    attn(x) = W_out(sigmoid(W_g x) * GQA(norm/RoPE(W_q x), norm/RoPE(W_k x), W_v x)).
    READING: the gate projection reads the attention module's input xn, is elementwise
    (C -> H*D), and no block linear has a bias.
    ``rows`` computes only the listed sequence positions of the output (every key is
    still formed from all rows). Returns (B, R, C) in ``dtype``.
    """
    B, S, C = h.shape
    f = dtype
    hf = h.astype(f)
    mod = modulation(temb, w["table"], f)
    prescale, preshift, pregate, postscale, postshift, postgate = (mod[:, i][:, None, :] for i in range(6))
    xn = (1.0 + prescale) * rms_norm(hf, w["norm1_w"], eps, f) + preshift
    qsel = np.arange(S) if rows is None else np.asarray(rows)
    xq = xn[:, qsel]
    q = xq @ w["wq"].astype(f).T
    k = xn @ w["wk"].astype(f).T
    v = xn @ w["wv"].astype(f).T
    g = xq @ w["wg"].astype(f).T
    R = len(qsel)
    q = rms_norm(q.reshape(B, R, H, D), w["q_norm_w"], eps, f)
    k = rms_norm(k.reshape(B, S, Hkv, D), w["k_norm_w"], eps, f)
    q = apply_rope(q, cos[qsel], sin[qsel])
    k = apply_rope(k, cos, sin)
    o = attention(q, k, v.reshape(B, S, Hkv, D), key_valid, 1.0 / math.sqrt(D)).astype(f)
    o = o.reshape(B, R, H * D) * sigmoid(g)
    attn_out = o @ w["wo"].astype(f).T
    h1 = hf[:, qsel] + pregate * attn_out
    xn2 = (1.0 + postscale) * rms_norm(h1, w["norm2_w"], eps, f) + postshift
    u = silu(xn2 @ w["w_gate"].astype(f).T) * (xn2 @ w["w_up"].astype(f).T)
    ff = u @ w["w_down"].astype(f).T
    return h1 + postgate * ff


# ----------------------------------------------------------------------------- time path

def timestep_embedding(t: np.ndarray, dim: int, dtype=np.float64) -> np.ndarray:
    """Krea2TimestepEmbedding sinusoid ([ARCH] §四.5; width from [API] timestep_embed_dim).

    The input time is scaled by 1000 and the cosine half comes first.
    READING: half = dim/2 frequencies f_i = exp(-ln(10000) * i / half), i = 0..half-1.
    """
    half = dim // 2
    i = np.arange(half, dtype=np.float64)
    freqs = np.exp(-math.log(10000.0) * i / half)
    args = 1000.0 * np.asarray(t, dtype=np.float64)[:, None] * freqs[None, :]
    return np.concatenate([np.cos(args), np.sin(args)], axis=1).astype(dtype)


def time_path(t: np.ndarray, mw: Dict[str, np.ndarray], t_dim: int,
              dtype=np.float64) -> Tuple[np.ndarray, np.ndarray]:
    """timestep -> time_embed -> GELU -> time_mod_proj ([ARCH] §四 data flow, §四.5).

    time_embed is a 2-layer MLP with GELU-tanh: Linear(256, C) -> GELU -> Linear(C, C).
    READING: the GELU between time_embed and time_mod_proj is also the tanh form.
    time_mod_proj = Linear(C, 6C, bias=True) ([ARCH] §四 module list).
    Returns temb (B, 6C) and e = GELU(time_embed(t)) (B, C).
    """
    f = dtype
    x = timestep_embedding(t, t_dim, f)
    x = gelu_tanh(x @ mw["t1_w"].astype(f).T + mw["t1_b"].astype(f))
    te = x @ mw["t2_w"].astype(f).T + mw["t2_b"].astype(f)
    e = gelu_tanh(te)
    temb = e @ mw["mod_w"].astype(f).T + mw["mod_b"].astype(f)
    return temb, e


def final_layer(x: np.ndarray, e: np.ndarray, mw: Dict[str, np.ndarray], eps: float,
                dtype=np.float64) -> np.ndarray:
    """Krea2FinalLayer ([ARCH] §四.6): adaptive RMSNorm with a (2, C) table, then Linear(C, in_ch).

    READING: (scale, shift) = table[0:2] + e with e = GELU(time_embed(t)) (B, C), and
    y = (1 + scale) * norm(x) + shift; the projection has a bias (nn.Linear default).
    x (B, N, C) image rows only. Returns (B, N, in_ch).
    """
    f = dtype
    mod = mw["final_table"].astype(f)[None] + e.astype(f)[:, None, :]
    scale, shift = mod[:, 0][:, None, :], mod[:, 1][:, None, :]
    y = (1.0 + scale) * rms_norm(x.astype(f), mw["final_norm_w"], eps, f) + shift
    return y @ mw["final_w"].astype(f).T + mw["final_b"].astype(f)


def img_in(hidden: np.ndarray, mw: Dict[str, np.ndarray], dtype=np.float64) -> np.ndarray:
    """img_in = nn.Linear(in_channels, C, bias=True) on packed latents ([ARCH] §四 module list)."""
    f = dtype
    return hidden.astype(f) @ mw["img_in_w"].astype(f).T + mw["img_in_b"].astype(f)


def backbone_forward(hidden: np.ndarray, text: np.ndarray, pos: np.ndarray,
                     text_mask: Optional[np.ndarray], t: np.ndarray,
                     mw: Dict[str, np.ndarray], block_w: Callable[[int], Dict[str, np.ndarray]],
                     n_layers: int, H: int, Hkv: int, D: int, axes: Sequence[int],
                     theta: float, eps: float, t_dim: int, dtype=np.float64) -> np.ndarray:
    """Krea2Transformer2DModel.forward from post-fusion text features ([ARCH] §四 data flow).

    temb = time path(t); x = cat([text, img_in(hidden)]) along the sequence (text first,
    [API] description); RoPE tables from position_ids; n_layers blocks in order sharing
    temb; drop the text rows ([ARCH] §二); final layer -> velocity (B, N, in_ch).
    ``text`` stands for the text-fusion + txt_in output (B, T, C).
    """
    B, N, _ = hidden.shape
    T = text.shape[1]
    check_dims(D, axes, H, Hkv)
    check_positions(pos, T + N)
    cos, sin = rope_cos_sin(pos, axes, theta)
    temb, e = time_path(t, mw, t_dim, dtype)
    x = np.concatenate([text.astype(dtype), img_in(hidden, mw, dtype)], axis=1)
    kv = key_valid_mask(text_mask, B, T, N)
    for layer in range(n_layers):
        x = block_forward(x, temb, block_w(layer), cos, sin, kv, H, Hkv, D, eps, dtype=dtype)
    return final_layer(x[:, T:], e, mw, eps, dtype)


# ----------------------------------------------------------------------------- sampler (Euler + CFG)

def shift_mu(image_seq_len: int, base_seq_len: int = 256, max_seq_len: int = 6400,
             base_shift: float = 0.5, max_shift: float = 1.15) -> float:
    """Resolution-aware shift parameter ([PIPE] scheduler: use_dynamic_shifting with base_shift 0.5,
    max_shift 1.15, base_image_seq_len 256, max_image_seq_len 6400; `mu` is computed from the
    image resolution unless the checkpoint is distilled, where mu = 1.15).
    READING: mu is the straight line through (256, 0.5) and (6400, 1.15) in image_seq_len."""
    slope = (max_shift - base_shift) / (max_seq_len - base_seq_len)
    return base_shift + slope * (image_seq_len - base_seq_len)


def shifted_sigmas(steps: int, mu: float) -> np.ndarray:
    """Sigma schedule ([PIPE] __call__: default grid linspace(1, 1/N, N); the scheduler applies the
    exponential time shift). READING: sigma' = e^mu / (e^mu + (1/sigma - 1)), followed by the
    terminal sigma 0. Returns steps + 1 values in fp64."""
    s = np.linspace(1.0, 1.0 / steps, steps)
    em = math.exp(mu)
    shifted = em / (em + (1.0 / s - 1.0))
    return np.concatenate([shifted, [0.0]])


def cfg_combine(cond: np.ndarray, uncond: Optional[np.ndarray], guidance: float) -> np.ndarray:
    """Krea 2 guidance convention ([PIPE] guidance_scale): v = cond + g * (cond - uncond), used
    whenever g > 0; g = 0 returns cond."""
    if guidance <= 0 or uncond is None:
        return cond
    return cond + guidance * (cond - uncond)


def euler_step(x: np.ndarray, v: np.ndarray, sigma: float, sigma_next: float) -> np.ndarray:
    """Flow-matching Euler update of FlowMatchEulerDiscreteScheduler ([PIPE] scheduler):
    x <- x + (sigma_next - sigma) * v. The model sees timestep = sigma (t / num_train_timesteps,
    [ARCH] §五)."""
    return x + (sigma_next - sigma) * v


def sample_loop(latents: np.ndarray, sigmas: Sequence[float], guidance: float,
                velocity: Callable[[np.ndarray, float, int], np.ndarray], dtype=np.float64) -> np.ndarray:
    """Sampling loop of [PIPE] __call__ for one image, with the model as a callable.

    For i = 0 .. len(sigmas) - 2 the model is evaluated at the current latents and at timestep
    sigmas[i] (t = sigma, [ARCH] §五): velocity(x, sigmas[i], 0) for the conditional prompt and,
    when guidance > 0, velocity(x, sigmas[i], 1) for the unconditional one, as a separate call.
    cfg_combine merges them and euler_step moves the latents from sigmas[i] to sigmas[i + 1].
    Returns the final latents."""
    x = latents.astype(dtype)
    for i in range(len(sigmas) - 1):
        vc = velocity(x, sigmas[i], 0)
        vu = velocity(x, sigmas[i], 1) if guidance > 0 else None
        x = euler_step(x, cfg_combine(vc, vu, guidance), sigmas[i], sigmas[i + 1])
    return x


def sample(latents: np.ndarray, text_cond: np.ndarray, text_uncond: Optional[np.ndarray],
           mask_cond: Optional[np.ndarray], mask_uncond: Optional[np.ndarray], pos: np.ndarray,
           sigmas: Sequence[float], guidance: float, mw: Dict[str, np.ndarray],
           block_w: Callable[[int], Dict[str, np.ndarray]], n_layers: int, H: int, Hkv: int, D: int,
           axes: Sequence[int], theta: float, eps: float, t_dim: int, dtype=np.float64) -> np.ndarray:
    """sample_loop with the backbone as the model ([PIPE] __call__): branch 0 runs backbone_forward
    on (text_cond, mask_cond), branch 1 on (text_uncond, mask_uncond), each as a batch of one at
    timestep sigma. latents (N, in_ch); text_* (T, C); masks (T) or None. Returns (N, in_ch)."""
    texts, masks = (text_cond, text_uncond), (mask_cond, mask_uncond)

    def velocity(x, sigma, branch):
        m = None if masks[branch] is None else masks[branch][None]
        return backbone_forward(x[None], texts[branch][None], pos, m, np.array([sigma], dtype=np.float64), mw,
                                block_w, n_layers, H, Hkv, D, axes, theta, eps, t_dim, dtype)[0]
    return sample_loop(latents, sigmas, guidance, velocity, dtype)


# ----------------------------------------------------------------------------- text fusion

def text_fusion_block(x: np.ndarray, w: Dict[str, np.ndarray], key_valid: np.ndarray, H: int, Hkv: int,
                      D: int, eps: float, dtype=np.float64) -> np.ndarray:
    """Krea2TextFusionBlock ([ARCH] §四.1): a pre-norm block with no RoPE and no time modulation.

    READING: apart from those two, the same structure as Krea2TransformerBlock:
    x + attn(norm1(x)), then + SwiGLU(norm2(x)), with q/k RMSNorm and the sigmoid-gated
    attention of §四.3 (text heads text_num_attention_heads / text_num_key_value_heads). Written
    as block_forward with a modulation of (scale 0, shift 0, gate 1) twice and a zero rotation,
    which are exact identities. x (B, S, Dt); key_valid (B, S). Returns (B, S, Dt)."""
    B, S, C = x.shape
    unit = np.zeros((6, C))
    unit[2] = 1.0
    unit[5] = 1.0
    wu = dict(w)
    wu["table"] = unit
    ang0 = np.zeros((S, D // 2))
    return block_forward(x, np.zeros((B, 6 * C)), wu, np.cos(ang0), np.sin(ang0), key_valid, H, Hkv, D, eps,
                         dtype=dtype)


def text_fusion(ehs: np.ndarray, text_mask: Optional[np.ndarray], layerwise: Sequence[Dict[str, np.ndarray]],
                layer_w: np.ndarray, refiner: Sequence[Dict[str, np.ndarray]], H: int, Hkv: int, D: int,
                eps: float, dtype=np.float64) -> np.ndarray:
    """Krea2TextFusion ([ARCH] §四.1; sizes from [API] text_* parameters).

    ehs (B, T, L, Dt): L stacked encoder layers per token. Three steps, in the page's order:
    1. layerwise: each token's (L, Dt) stack is its own sequence through the layerwise blocks
       (no mask: every layer is valid);
    2. projection: Linear(L, 1, bias=False) over the layer axis, layer_w (L,);
    3. refiner: the (B, T, Dt) token sequence through the refiner blocks with the text mask.
    Returns (B, T, Dt)."""
    B, T, L, Dt = ehs.shape
    x = ehs.astype(dtype).reshape(B * T, L, Dt)
    all_valid = np.ones((B * T, L), dtype=bool)
    for w in layerwise:
        x = text_fusion_block(x, w, all_valid, H, Hkv, D, eps, dtype)
    x = np.einsum("nld,l->nd", x, layer_w.astype(dtype)).reshape(B, T, Dt)
    kv = np.ones((B, T), dtype=bool) if text_mask is None else np.asarray(text_mask, dtype=bool)
    for w in refiner:
        x = text_fusion_block(x, w, kv, H, Hkv, D, eps, dtype)
    return x


def txt_in(x: np.ndarray, w: np.ndarray, b: np.ndarray, dtype=np.float64) -> np.ndarray:
    """Krea2TextProjection ([ARCH] §四 module list: txt_in(text_hidden_dim -> hidden_size)).
    READING: its internals are not given; a plain Linear(Dt, C) with bias."""
    return x.astype(dtype) @ w.astype(dtype).T + b.astype(dtype)


# ----------------------------------------------------------------------------- block-causal variant

def image_block_ids(segments: Sequence[Tuple[str, int]]) -> np.ndarray:
    """Token metadata of the block-causal variant (page "QwenImage21Transformer2DModel",
    build_token_metadata): the joint sequence as ("text", n) / ("image", n) segments in order;
    -1 at text positions and one id per image block. Block boundaries come from the segment
    sizes, so two adjacent image segments stay two blocks."""
    ids = []
    nxt = 0
    for kind, n in segments:
        if kind == "text":
            ids += [-1] * n
        else:
            ids += [nxt] * n
            nxt += 1
    return np.asarray(ids, dtype=np.int64)


def block_causal_allowed(ids: np.ndarray) -> np.ndarray:
    """Attention pattern of the QwenImage 2.1 page: query q may read key k iff
    (q_idx >= kv_idx) or (q and k lie in the same image block). Returns (S, S) bool."""
    S = len(ids)
    q = np.arange(S)[:, None]
    k = np.arange(S)[None, :]
    same = (ids[:, None] == ids[None, :]) & (ids[:, None] >= 0)
    return (q >= k) | same


def masked_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, allowed: np.ndarray, key_valid: np.ndarray,
                     scale: float) -> np.ndarray:
    """GQA softmax attention where query row i of batch row b reads keys j with
    allowed[i, j] and key_valid[b, j]; a row with no readable key outputs zeros.
    q (B, Sq, H, D); k, v (B, Sk, Hkv, D); allowed (Sq, Sk); key_valid (B, Sk). Returns fp64."""
    B, Sq, H, D = q.shape
    G = H // k.shape[2]
    out = np.zeros((B, Sq, H, D), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            j = h // G
            for i in range(Sq):
                idx = np.nonzero(allowed[i] & key_valid[b])[0]
                if idx.size == 0:
                    continue
                s = (k[b, idx, j, :] @ q[b, i, h, :]).astype(np.float64) * scale
                p = np.exp(s - s.max())
                out[b, i, h, :] = (p / p.sum()) @ v[b, idx, j, :].astype(np.float64)
    return out


def cached_step_attention(q_new: np.ndarray, k_cache: np.ndarray, v_cache: np.ndarray, k_new: np.ndarray,
                          v_new: np.ndarray, allowed_new: np.ndarray, key_valid: np.ndarray,
                          scale: float) -> np.ndarray:
    """One denoising step of the block-causal variant with a key/value cache (page
    "QwenImage21Transformer2DModel", kv_cache with causal_condition): the P prefix tokens are
    not recomputed; their keys and values come from the cache, the Nq new tokens' own keys and
    values follow them, and new token i reads the keys its row of the pattern allows.
    q_new (B, Nq, H, D); k_cache, v_cache (B, P, Hkv, D); k_new, v_new (B, Nq, Hkv, D);
    allowed_new (Nq, P + Nq), the pattern's rows of the new tokens; key_valid (B, P + Nq)."""
    k = np.concatenate([k_cache, k_new], axis=1)
    v = np.concatenate([v_cache, v_new], axis=1)
    return masked_attention(q_new, k, v, allowed_new, key_valid, scale)
