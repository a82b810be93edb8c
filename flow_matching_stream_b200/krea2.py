"""Python binding of libkrea2.so: argument marshalling from torch tensors to the C ABI.

Every function here has the name of a C entry point in ``include/krea2.h`` (without the
``krea2_`` prefix) and does no arithmetic of its own: it checks devices, dtypes and
contiguity, passes raw pointers and the current CUDA stream, and raises ``Krea2Error``
with the library's message when a call fails. Weight containers build the library's
device layout (fused [q|k|v|gate] rows, gate/up rows interleaved in 64-row groups).
"""
from __future__ import annotations

import ctypes
from typing import Dict, List, Optional, Sequence

import numpy as np
import torch

from . import _lib
from ._lib import KREA2_BF16, KREA2_F32, KREA2_EPI_RESID, KREA2_EPI_STORE, KREA2_EPI_SWIGLU  # noqa: F401

__all__ = [
    "Krea2Error", "lib", "dims_struct", "dtype_code", "workspace_size", "attention_workspace_size",
    "rope_tables", "gqa_attention", "gqa_attention_noalloc", "block_causal_key_end", "gqa_attention_block_causal",
    "kv_cache_append", "kv_cache_attention_workspace_size", "gqa_attention_kv_cache", "modulated_rmsnorm", "linear", "time_embed", "final_layer_workspace_size", "final_layer",
    "text_dims_struct", "TextWeights", "text_fusion_workspace_size", "text_fusion",
    "shift_mu", "sigma_schedule", "euler_cfg_step", "sample_workspace_size", "sample",
    "block_forward", "block_forward_traced", "BLOCK_STEPS", "launch_count", "backbone_forward", "check_device_error", "BlockWeights", "ModelWeights",
    "interleave_gate_up", "KREA2_BF16", "KREA2_F32", "KREA2_EPI_STORE", "KREA2_EPI_SWIGLU", "KREA2_EPI_RESID",
]

_LIB = None


class Krea2Error(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"krea2 error {code}: {msg}")
        self.code = code


def lib() -> ctypes.CDLL:
    global _LIB
    if _LIB is None:
        _LIB = _lib.load()
    return _LIB


def _check(rc: int) -> None:
    if rc != 0:
        raise Krea2Error(rc, lib().krea2_last_error_string().decode())


def dims_struct(d) -> _lib.Krea2Dims:
    """Krea2Dims from any object with C, H, Hkv, D, F, axes, theta, eps, n_layers, in_ch, t_dim."""
    s = _lib.Krea2Dims()
    s.C, s.H, s.Hkv, s.D, s.F = d.C, d.H, d.Hkv, d.D, d.F
    s.axes[0], s.axes[1], s.axes[2] = tuple(d.axes)
    s.theta, s.eps = float(d.theta), float(d.eps)
    s.n_layers, s.in_ch, s.t_dim = d.n_layers, d.in_ch, d.t_dim
    return s


def dtype_code(dt: torch.dtype) -> int:
    if dt == torch.bfloat16:
        return KREA2_BF16
    if dt == torch.float32:
        return KREA2_F32
    raise TypeError(f"unsupported dtype {dt}")


def _p(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _s(stream: Optional[torch.cuda.Stream]) -> int:
    return (stream if stream is not None else torch.cuda.current_stream()).cuda_stream


def _want(t: torch.Tensor, dt: torch.dtype, name: str) -> None:
    if t.dtype != dt:
        raise TypeError(f"{name} must be {dt}, got {t.dtype}")


def workspace_size(dims, B: int, T: int, N: int, dtype: torch.dtype) -> int:
    return int(lib().krea2_workspace_size(ctypes.byref(dims_struct(dims)), B, T, N, dtype_code(dtype)))


def attention_workspace_size(dims, B: int, T: int, N: int, dtype: torch.dtype) -> int:
    return int(lib().krea2_attention_workspace_size(ctypes.byref(dims_struct(dims)), B, T, N, dtype_code(dtype)))


def check_device_error(stream=None) -> None:
    _check(lib().krea2_check_device_error(_s(stream)))


def rope_tables(dims, position_ids: torch.Tensor, cos_out: torch.Tensor, sin_out: torch.Tensor, stream=None) -> None:
    for t, n in ((position_ids, "position_ids"), (cos_out, "cos_out"), (sin_out, "sin_out")):
        _want(t, torch.float32, n)
    if position_ids.dim() != 2 or position_ids.shape[1] != 3:
        raise ValueError("position_ids must have shape (T+N, 3)")
    S = position_ids.shape[0]
    _check(lib().krea2_rope_tables(ctypes.byref(dims_struct(dims)), _p(position_ids), S, _p(cos_out), _p(sin_out),
                                   _s(stream)))


def gqa_attention(dims, B: int, T: int, N: int, qkvg: torch.Tensor, q_norm_w: torch.Tensor, k_norm_w: torch.Tensor,
                  cos: torch.Tensor, sin: torch.Tensor, text_mask: Optional[torch.Tensor], out: torch.Tensor,
                  workspace: Optional[torch.Tensor] = None, stream=None) -> None:
    dt = dtype_code(qkvg.dtype)
    _want(out, qkvg.dtype, "out")
    if text_mask is not None:
        _want(text_mask, torch.uint8, "text_mask")
    ws = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().krea2_gqa_attention(ctypes.byref(dims_struct(dims)), B, T, N, dt, _p(qkvg), _p(q_norm_w),
                                     _p(k_norm_w), _p(cos), _p(sin), _p(text_mask), _p(out), _p(workspace), ws,
                                     _s(stream)))


def gqa_attention_noalloc(dims, B: int, T: int, N: int, qkvg: torch.Tensor, q_norm_w: torch.Tensor,
                          k_norm_w: torch.Tensor, cos: torch.Tensor, sin: torch.Tensor,
                          text_mask: Optional[torch.Tensor], out: torch.Tensor, stream=None) -> None:
    """gqa_attention for callers that cannot allocate: the library's static scratch replaces the workspace."""
    _want(out, qkvg.dtype, "out")
    if text_mask is not None:
        _want(text_mask, torch.uint8, "text_mask")
    _check(lib().krea2_gqa_attention_noalloc(ctypes.byref(dims_struct(dims)), B, T, N, dtype_code(qkvg.dtype),
                                             _p(qkvg), _p(q_norm_w), _p(k_norm_w), _p(cos), _p(sin),
                                             _p(text_mask), _p(out), _s(stream)))


def block_causal_key_end(image_ids: np.ndarray) -> np.ndarray:
    """Per-query key prefix of the block-causal pattern (host computation in the library)."""
    ids = np.ascontiguousarray(image_ids, dtype=np.int32)
    out = np.zeros(len(ids), dtype=np.int32)
    _check(lib().krea2_block_causal_key_end(ids.ctypes.data, len(ids), out.ctypes.data))
    return out


def gqa_attention_block_causal(dims, B: int, T: int, N: int, qkvg: torch.Tensor, q_norm_w: torch.Tensor,
                               k_norm_w: torch.Tensor, cos: torch.Tensor, sin: torch.Tensor,
                               text_mask: Optional[torch.Tensor], key_end: torch.Tensor, out: torch.Tensor,
                               workspace: torch.Tensor, stream=None) -> None:
    _want(key_end, torch.int32, "key_end")
    _want(out, qkvg.dtype, "out")
    _check(lib().krea2_gqa_attention_block_causal(
        ctypes.byref(dims_struct(dims)), B, T, N, dtype_code(qkvg.dtype), _p(qkvg), _p(q_norm_w), _p(k_norm_w),
        _p(cos), _p(sin), _p(text_mask), _p(key_end), _p(out), _p(workspace),
        workspace.numel() * workspace.element_size(), _s(stream)))


def kv_cache_append(dims, B: int, n: int, row0: int, qkvg: torch.Tensor, k_norm_w: torch.Tensor, cos: torch.Tensor,
                    sin: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, stream=None) -> None:
    """Keys and values of n tokens into rows [row0, row0 + n) of a (B, capacity, Hkv*D) cache."""
    for t, name in ((k_cache, "k_cache"), (v_cache, "v_cache")):
        _want(t, qkvg.dtype, name)
    if k_cache.shape != v_cache.shape or k_cache.dim() != 3 or k_cache.shape[0] != B:
        raise ValueError("k_cache and v_cache must both be (B, capacity, Hkv*D)")
    _check(lib().krea2_kv_cache_append(ctypes.byref(dims_struct(dims)), B, n, row0, k_cache.shape[1],
                                       dtype_code(qkvg.dtype), _p(qkvg), _p(k_norm_w), _p(cos), _p(sin),
                                       _p(k_cache), _p(v_cache), _s(stream)))


def kv_cache_attention_workspace_size(dims, B: int, Nq: int, dtype: torch.dtype) -> int:
    return int(lib().krea2_kv_cache_attention_workspace_size(ctypes.byref(dims_struct(dims)), B, Nq,
                                                             dtype_code(dtype)))


def gqa_attention_kv_cache(dims, B: int, T: int, L: int, Nq: int, qkvg: torch.Tensor, q_norm_w: torch.Tensor,
                           cos: torch.Tensor, sin: torch.Tensor, text_mask: Optional[torch.Tensor],
                           k_cache: torch.Tensor, v_cache: torch.Tensor, key_end: Optional[torch.Tensor],
                           out: torch.Tensor, workspace: torch.Tensor, stream=None) -> None:
    """Attention of the Nq tokens at key positions [L - Nq, L) over the first L cached keys."""
    if key_end is not None:
        _want(key_end, torch.int32, "key_end")
    _want(out, qkvg.dtype, "out")
    _check(lib().krea2_gqa_attention_kv_cache(
        ctypes.byref(dims_struct(dims)), B, T, L, Nq, dtype_code(qkvg.dtype), _p(qkvg), _p(q_norm_w), _p(cos),
        _p(sin), _p(text_mask), _p(k_cache), _p(v_cache), k_cache.shape[1], _p(key_end), _p(out), _p(workspace),
        workspace.numel() * workspace.element_size(), _s(stream)))


def modulated_rmsnorm(dims, B: int, S: int, h: torch.Tensor, norm_w: torch.Tensor, temb: torch.Tensor,
                      table: torch.Tensor, chunk: int, out: torch.Tensor, stream=None) -> None:
    _check(lib().krea2_modulated_rmsnorm(ctypes.byref(dims_struct(dims)), B, S, dtype_code(out.dtype), _p(h),
                                         _p(norm_w), _p(temb), _p(table), chunk, _p(out), _s(stream)))


def linear(epilogue: int, A: torch.Tensor, W: torch.Tensor, out: torch.Tensor, gate: Optional[torch.Tensor] = None,
           rows_per_batch: int = 1, gate_stride: int = 0, stream=None) -> None:
    M, K = A.shape
    Nw = W.shape[0]
    if W.shape[1] != K:
        raise ValueError("A and W disagree on K")
    _want(W, A.dtype, "W")
    _check(lib().krea2_linear(dtype_code(A.dtype), epilogue, M, Nw, K, _p(A), _p(W), _p(out), _p(gate),
                              rows_per_batch, gate_stride, _s(stream)))


def time_embed(dims, timestep: torch.Tensor, mw: "ModelWeights", temb_out: torch.Tensor, e_out: torch.Tensor,
               scratch: torch.Tensor, stream=None) -> None:
    _check(lib().krea2_time_embed(ctypes.byref(dims_struct(dims)), timestep.shape[0], mw.dtype_code, _p(timestep),
                                  ctypes.byref(mw.struct), _p(temb_out), _p(e_out), _p(scratch), _s(stream)))


def final_layer_workspace_size(dims, B: int, N: int, dtype: torch.dtype) -> int:
    return int(lib().krea2_final_layer_workspace_size(ctypes.byref(dims_struct(dims)), B, N, dtype_code(dtype)))


def final_layer(dims, B: int, T: int, N: int, h: torch.Tensor, e: torch.Tensor, mw: "ModelWeights",
                velocity: torch.Tensor, workspace: Optional[torch.Tensor] = None, stream=None) -> None:
    ws = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().krea2_final_layer(ctypes.byref(dims_struct(dims)), B, T, N, mw.dtype_code, _p(h), _p(e),
                                   ctypes.byref(mw.struct), _p(velocity), _p(workspace), ws, _s(stream)))


def block_forward(dims, B: int, T: int, N: int, h: torch.Tensor, temb: torch.Tensor, bw: "BlockWeights",
                  cos: torch.Tensor, sin: torch.Tensor, text_mask: Optional[torch.Tensor], workspace: torch.Tensor,
                  stream=None) -> None:
    _want(h, torch.float32, "h")
    _check(lib().krea2_block_forward(ctypes.byref(dims_struct(dims)), B, T, N, bw.dtype_code, _p(h), _p(temb),
                                     ctypes.byref(bw.struct), _p(cos), _p(sin), _p(text_mask), _p(workspace),
                                     workspace.numel() * workspace.element_size(), _s(stream)))


def text_dims_struct(td) -> _lib.Krea2TextDims:
    s = _lib.Krea2TextDims()
    for f in ("Dt", "L", "H", "Hkv", "D", "F", "n_layerwise", "n_refiner", "C"):
        setattr(s, f, getattr(td, f))
    s.eps = float(td.eps)
    return s


def text_fusion_workspace_size(td, B: int, T: int, dtype: torch.dtype) -> int:
    return int(lib().krea2_text_fusion_workspace_size(ctypes.byref(text_dims_struct(td)), B, T, dtype_code(dtype)))


def text_fusion(td, B: int, T: int, ehs: torch.Tensor, text_mask: Optional[torch.Tensor], tw: "TextWeights",
                text_out: torch.Tensor, workspace: torch.Tensor, stream=None) -> None:
    _want(ehs, tw.dtype, "ehs")
    _want(text_out, tw.dtype, "text_out")
    _check(lib().krea2_text_fusion(ctypes.byref(text_dims_struct(td)), B, T, tw.dtype_code, _p(ehs), _p(text_mask),
                                   ctypes.byref(tw.struct), _p(text_out), _p(workspace),
                                   workspace.numel() * workspace.element_size(), _s(stream)))


def shift_mu(image_seq_len: int) -> float:
    return float(lib().krea2_shift_mu(image_seq_len))


def sigma_schedule(n_steps: int, mu: float) -> np.ndarray:
    out = np.zeros(n_steps + 1, dtype=np.float32)
    _check(lib().krea2_sigma_schedule(n_steps, mu, out.ctypes.data))
    return out


def euler_cfg_step(x: torch.Tensor, v_cond: torch.Tensor, v_uncond: Optional[torch.Tensor], guidance: float,
                   sigma: float, sigma_next: float, x_model: Optional[torch.Tensor] = None, copies: int = 1,
                   timestep_out: Optional[torch.Tensor] = None, stream=None) -> None:
    _want(x, torch.float32, "x")
    _check(lib().krea2_euler_cfg_step(dtype_code(v_cond.dtype), x.numel(), _p(x), _p(v_cond), _p(v_uncond),
                                      guidance, sigma, sigma_next, _p(x_model), copies, _p(timestep_out),
                                      _s(stream)))


def sample_workspace_size(dims, T: int, N: int, dtype: torch.dtype, cfg: bool) -> int:
    return int(lib().krea2_sample_workspace_size(ctypes.byref(dims_struct(dims)), T, N, dtype_code(dtype), int(cfg)))


def sample(dims, T: int, N: int, latents: torch.Tensor, text_cond: torch.Tensor, text_uncond: Optional[torch.Tensor],
           mask_cond: Optional[torch.Tensor], mask_uncond: Optional[torch.Tensor], position_ids: torch.Tensor,
           sigmas: np.ndarray, guidance: float, mw: "ModelWeights", workspace: torch.Tensor, stream=None) -> None:
    """The device sampling loop (krea2_sample); `sigmas` is a host array of n_steps + 1 values."""
    _want(latents, torch.float32, "latents")
    sg = np.ascontiguousarray(sigmas, dtype=np.float32)
    _check(lib().krea2_sample(ctypes.byref(dims_struct(dims)), T, N, mw.dtype_code, _p(latents), _p(text_cond),
                              _p(text_uncond), _p(mask_cond), _p(mask_uncond), _p(position_ids), sg.ctypes.data,
                              len(sg) - 1, guidance, ctypes.byref(mw.struct), _p(workspace),
                              workspace.numel() * workspace.element_size(), _s(stream)))


BLOCK_STEPS = ("modulation", "norm1", "qkv_proj", "attention", "out_proj_resid", "norm2", "gate_up_swiglu",
               "down_proj_resid")


def block_forward_traced(dims, B: int, T: int, N: int, h: torch.Tensor, temb: torch.Tensor, bw: "BlockWeights",
                         cos: torch.Tensor, sin: torch.Tensor, text_mask: Optional[torch.Tensor],
                         workspace: torch.Tensor, events: Sequence[torch.cuda.Event], stream=None) -> None:
    """block_forward recording events[i] before launch i (BLOCK_STEPS order) and events[8] after."""
    if len(events) != 9:
        raise ValueError("need 9 events")
    st = stream if stream is not None else torch.cuda.current_stream()
    for e in events:
        if not e.cuda_event:
            e.record(st)  # torch creates the CUDA event lazily, on its first record
    arr = (ctypes.c_void_p * 9)(*[e.cuda_event for e in events])
    _want(h, torch.float32, "h")
    _check(lib().krea2_block_forward_traced(ctypes.byref(dims_struct(dims)), B, T, N, bw.dtype_code, _p(h), _p(temb),
                                            ctypes.byref(bw.struct), _p(cos), _p(sin), _p(text_mask),
                                            _p(workspace), workspace.numel() * workspace.element_size(), arr,
                                            _s(stream)))


def launch_count() -> int:
    return int(lib().krea2_launch_count())


def backbone_forward(dims, B: int, T: int, N: int, hidden_states: torch.Tensor, text_states: torch.Tensor,
                     position_ids: torch.Tensor, text_mask: Optional[torch.Tensor], timestep: torch.Tensor,
                     mw: "ModelWeights", velocity: torch.Tensor, workspace: torch.Tensor, stream=None) -> None:
    _check(lib().krea2_backbone_forward(ctypes.byref(dims_struct(dims)), B, T, N, mw.dtype_code, _p(hidden_states),
                                        _p(text_states), _p(position_ids), _p(text_mask), _p(timestep),
                                        ctypes.byref(mw.struct), _p(velocity), _p(workspace),
                                        workspace.numel() * workspace.element_size(), _s(stream)))


# ----------------------------------------------------------------------------- weights

def interleave_gate_up(w_gate: torch.Tensor, w_up: torch.Tensor) -> torch.Tensor:
    """(F, C) gate and up rows -> (2F, C) in 64-row groups [gate 64 | up 64 | gate 64 | ...]."""
    F, C = w_gate.shape
    if F % 64:
        raise ValueError("intermediate size must be a multiple of 64")
    return torch.stack([w_gate.reshape(F // 64, 64, C), w_up.reshape(F // 64, 64, C)], dim=1).reshape(2 * F, C)


def _dev(a, dtype, device) -> torch.Tensor:
    t = a if isinstance(a, torch.Tensor) else torch.from_numpy(np.ascontiguousarray(a))
    return t.to(device=device, dtype=dtype).contiguous()


class BlockWeights:
    """One block's device tensors in the library layout plus the Krea2BlockWeights struct."""

    def __init__(self, w: Dict[str, object], dtype: torch.dtype, device):
        self.dtype = dtype
        self.dtype_code = dtype_code(dtype)
        f32 = torch.float32
        self.w_qkvg = _dev(torch.cat([_dev(w[k], dtype, device) for k in ("wq", "wk", "wv", "wg")], 0), dtype, device)
        self.w_out = _dev(w["wo"], dtype, device)
        self.w_gu = interleave_gate_up(_dev(w["w_gate"], dtype, device), _dev(w["w_up"], dtype, device)).contiguous()
        self.w_down = _dev(w["w_down"], dtype, device)
        self.norm1_w = _dev(w["norm1_w"], f32, device)
        self.norm2_w = _dev(w["norm2_w"], f32, device)
        self.q_norm_w = _dev(w["q_norm_w"], f32, device)
        self.k_norm_w = _dev(w["k_norm_w"], f32, device)
        self.table = _dev(w["table"], f32, device)
        self.struct = _lib.Krea2BlockWeights()
        self.fill(self.struct)

    def fill(self, s: _lib.Krea2BlockWeights) -> None:
        s.w_qkvg, s.w_out, s.w_gu, s.w_down = (_p(self.w_qkvg), _p(self.w_out), _p(self.w_gu), _p(self.w_down))
        s.norm1_w, s.norm2_w = _p(self.norm1_w), _p(self.norm2_w)
        s.q_norm_w, s.k_norm_w = _p(self.q_norm_w), _p(self.k_norm_w)
        s.scale_shift_table = _p(self.table)

    @staticmethod
    def random(dims, dtype: torch.dtype, device, generator: torch.Generator) -> "BlockWeights":
        """Seeded random weights drawn on the device (N(0,1)/sqrt(fan_in) linears, N(0, 0.1^2) rest)."""
        C, HD, KVD, F, D = dims.C, dims.H * dims.D, dims.Hkv * dims.D, dims.F, dims.D

        def n(shape, std):
            return (torch.randn(shape, device=device, generator=generator, dtype=torch.float32) * std).to(dtype)

        w = {"wq": n((HD, C), C ** -0.5), "wk": n((KVD, C), C ** -0.5), "wv": n((KVD, C), C ** -0.5),
             "wg": n((HD, C), C ** -0.5), "wo": n((C, HD), HD ** -0.5), "w_gate": n((F, C), C ** -0.5),
             "w_up": n((F, C), C ** -0.5), "w_down": n((C, F), F ** -0.5),
             "norm1_w": n((C,), 0.1).float(), "norm2_w": n((C,), 0.1).float(), "q_norm_w": n((D,), 0.1).float(),
             "k_norm_w": n((D,), 0.1).float(), "table": n((6, C), 0.1).float()}
        return BlockWeights(w, dtype, device)


class TextWeights:
    """Text-fusion device tensors: layerwise / refiner blocks (no modulation table), the layer-axis
    projection and txt_in."""

    def __init__(self, tw: Dict[str, object], dtype: torch.dtype, device):
        self.dtype = dtype
        self.dtype_code = dtype_code(dtype)
        self.layerwise = [BlockWeights(dict(w, table=np.zeros((6, 1), np.float32)), dtype, device)
                          for w in tw["layerwise"]]
        self.refiner = [BlockWeights(dict(w, table=np.zeros((6, 1), np.float32)), dtype, device)
                        for w in tw["refiner"]]
        self.layer_w = _dev(tw["layer_w"], torch.float32, device)
        self.txt_in_w = _dev(tw["txt_in_w"], dtype, device)
        self.txt_in_b = _dev(tw["txt_in_b"], torch.float32, device)
        self._lw = (_lib.Krea2BlockWeights * max(1, len(self.layerwise)))()
        self._rf = (_lib.Krea2BlockWeights * max(1, len(self.refiner)))()
        for arr, blocks in ((self._lw, self.layerwise), (self._rf, self.refiner)):
            for i, b in enumerate(blocks):
                b.fill(arr[i])
                arr[i].scale_shift_table = None   # fusion blocks carry no time modulation
        s = _lib.Krea2TextWeights()
        s.layerwise = ctypes.cast(self._lw, ctypes.POINTER(_lib.Krea2BlockWeights))
        s.refiner = ctypes.cast(self._rf, ctypes.POINTER(_lib.Krea2BlockWeights))
        s.layer_w, s.txt_in_w, s.txt_in_b = _p(self.layer_w), _p(self.txt_in_w), _p(self.txt_in_b)
        self.struct = s


class ModelWeights:
    """Backbone device tensors (img_in, time path, final layer) plus the block list."""

    def __init__(self, mw: Dict[str, object], blocks: Sequence[BlockWeights], dtype: torch.dtype, device):
        self.dtype = dtype
        self.dtype_code = dtype_code(dtype)
        f32 = torch.float32
        self.tensors = {}
        for k in ("img_in_w", "t1_w", "t2_w", "mod_w", "final_w"):
            self.tensors[k] = _dev(mw[k], dtype, device)
        for k in ("img_in_b", "t1_b", "t2_b", "mod_b", "final_norm_w", "final_table", "final_b"):
            self.tensors[k] = _dev(mw[k], f32, device)
        self.blocks: List[BlockWeights] = list(blocks)
        self._block_array = (_lib.Krea2BlockWeights * max(1, len(self.blocks)))()
        for i, b in enumerate(self.blocks):
            b.fill(self._block_array[i])
        s = _lib.Krea2ModelWeights()
        t = self.tensors
        s.img_in_w, s.img_in_b = _p(t["img_in_w"]), _p(t["img_in_b"])
        s.t1_w, s.t1_b, s.t2_w, s.t2_b = _p(t["t1_w"]), _p(t["t1_b"]), _p(t["t2_w"]), _p(t["t2_b"])
        s.mod_w, s.mod_b = _p(t["mod_w"]), _p(t["mod_b"])
        s.final_norm_w, s.final_table = _p(t["final_norm_w"]), _p(t["final_table"])
        s.final_w, s.final_b = _p(t["final_w"]), _p(t["final_b"])
        s.blocks = ctypes.cast(self._block_array, ctypes.POINTER(_lib.Krea2BlockWeights))
        self.struct = s
