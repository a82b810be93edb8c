/*
 * krea2.h — C ABI of the Krea 2 single-stream MMDiT block / backbone forward for NVIDIA
 * B200 (sm_100a).
 *
 * What is computed (sources, by page title and section):
 *   [API]  "Krea2Transformer2DModel" (diffusers v0.43.0 API docs): constructor defaults,
 *          "Parámetros", and the forward contract (hidden_states (B, image_seq, in_channels),
 *          position_ids (text_seq + image_seq, 3) with zero text rows,
 *          encoder_attention_mask (B, text_seq) bool, timestep (B,) in [0, 1]).
 *   [ARCH] "Diffusers 中的 Krea2Transformer2DModel：Krea 2 单流 MMDiT 流匹配 Transformer 架构全解":
 *          §二 I/O contract, §三 defaults and the head-split check, §四 data flow,
 *          §四.2 block, §四.3 attention, §四.4 RMSNorm, §四.5 time embedding, §四.6 final layer.
 *   [PIPE] "Krea 2" (Krea2Pipeline docs): prepare_position_ids.
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller, row-major, densely packed,
 *     unless a comment says "host". The library never allocates or frees memory and never
 *     synchronises the device; every call is asynchronous on `stream` (a cudaStream_t
 *     passed as void*; NULL = the legacy default stream).
 *   - Tokens are laid out batch-major: row r = b * S + s with S = T + N, text rows (s < T)
 *     first, then image rows in row-major latent-grid order ([API] description: one
 *     [text, image] sequence).
 *   - `dtype` selects the storage/compute type of activations and linear weights:
 *     KREA2_BF16 (bf16 storage, fp32 accumulation, fp32 norms/softmax/epilogues) or
 *     KREA2_F32 (fp32 everywhere; a SIMT reference-precision path for small shapes).
 *     Norm weights, modulation tables, biases, RoPE tables, temb and the residual stream
 *     are fp32 in both modes ([ARCH] §四.4: norm weights are kept in fp32).
 *   - Return value: KREA2_OK (0) or a negative KREA2_ERR_* code; krea2_last_error_string()
 *     then describes the failure (thread-local). Argument errors are detected on the host
 *     before anything is launched. KREA2_ERR_CUDA reports a launch failure.
 *     Kernels that wait on barriers bound every wait; an expired wait sets a device error
 *     word that krea2_check_device_error() reports as KREA2_ERR_TIMEOUT.
 *   - Alignment: the bf16 tensor-core paths move their matrix operands and bf16 outputs with
 *     TMA, which needs 16-byte aligned base addresses (cudaMalloc and torch allocations are
 *     256-byte aligned); the fp32 residual is held to the same rule. A misaligned pointer
 *     there returns KREA2_ERR_ARG before anything is launched.
 *   - text_mask: uint8 (B, T), 1 = valid text token, 0 = padding; NULL means all valid
 *     ([API] encoder_attention_mask). Padding only removes keys: padded text rows are still
 *     computed as queries, and image keys are always valid.
 */
#ifndef KREA2_H
#define KREA2_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
  KREA2_OK = 0,
  KREA2_ERR_ARG = -1,          /* null pointer, bad size, failed [ARCH] §二/§三 check     */
  KREA2_ERR_WORKSPACE = -2,    /* workspace smaller than krea2_workspace_size()          */
  KREA2_ERR_CUDA = -3,         /* a CUDA launch or driver call failed                     */
  KREA2_ERR_TIMEOUT = -4,      /* a bounded device-side wait expired                      */
  KREA2_ERR_UNSUPPORTED = -5   /* valid arguments the library has no kernel for           */
};

enum { KREA2_BF16 = 0, KREA2_F32 = 1 };

/* Model hyper-parameters ([API] constructor; defaults C=6144, H=48, Hkv=12, D=128,
 * F=16384, axes=(32,48,48), theta=1000, eps=1e-5, n_layers=28, in_ch=64, t_dim=256).
 * Checked by every entry point: C == H*D, H % Hkv == 0, axes even and summing to D
 * ([ARCH] §三 ValueError), theta > 0, eps > 0. */
typedef struct {
  int C, H, Hkv, D, F;
  int axes[3];
  float theta, eps;
  int n_layers, in_ch, t_dim;
} Krea2Dims;

/* One block's parameters ([ARCH] §四.2, §四.3). Linear weights are (out, in) row-major in
 * `dtype`. The block linears carry no bias (a reading: the pages list none).
 *   w_qkvg  (H*D + 2*Hkv*D + H*D, C): rows [to_q | to_k | to_v | to_gate], head-major.
 *   w_out   (C, H*D)                   to_out.
 *   w_gu    (2F, C): SwiGLU gate and up rows interleaved in 64-row groups: rows
 *           [128j, 128j+64) are gate rows [64j, 64j+64) and rows [128j+64, 128j+128) are up
 *           rows [64j, 64j+64). (Device layout; F must be a multiple of 64.)
 *   w_down  (C, F).
 *   norm1_w, norm2_w (C) fp32; q_norm_w, k_norm_w (D) fp32, shared by all heads;
 *   the RMSNorm multiplier is (1 + w) ([ARCH] §四.4).
 *   scale_shift_table (6, C) fp32, rows prescale, preshift, pregate, postscale, postshift,
 *   postgate, added to temb ([ARCH] §四.2). */
typedef struct {
  const void* w_qkvg;
  const void* w_out;
  const void* w_gu;
  const void* w_down;
  const float* norm1_w;
  const float* norm2_w;
  const float* q_norm_w;
  const float* k_norm_w;
  const float* scale_shift_table;
} Krea2BlockWeights;

/* Backbone parameters outside the blocks ([ARCH] §四 module list, §四.5, §四.6).
 * Weights in `dtype`, biases and tables fp32.
 *   img_in_w (C, in_ch), img_in_b (C)           img_in = Linear(in_ch, C, bias=True)
 *   t1_w (C, t_dim), t1_b (C); t2_w (C, C), t2_b (C)   time_embed MLP (GELU-tanh between)
 *   mod_w (6C, C), mod_b (6C)                   time_mod_proj
 *   final_norm_w (C), final_table (2, C) rows (scale, shift), final_w (in_ch, C), final_b (in_ch)
 *   blocks: HOST array of n_layers Krea2BlockWeights (its pointers are device pointers). */
typedef struct {
  const void* img_in_w;
  const float* img_in_b;
  const void* t1_w;
  const float* t1_b;
  const void* t2_w;
  const float* t2_b;
  const void* mod_w;
  const float* mod_b;
  const float* final_norm_w;
  const float* final_table;
  const void* final_w;
  const float* final_b;
  const Krea2BlockWeights* blocks;
} Krea2ModelWeights;

/* Message for the last error returned on this thread ("" if none). Host memory owned by
 * the library; valid until the next call on this thread. */
const char* krea2_last_error_string(void);

/* Synchronises `stream`, then reads and clears the device error word set by an expired
 * bounded wait. Returns KREA2_OK, KREA2_ERR_TIMEOUT or KREA2_ERR_CUDA. This is the only
 * entry point that synchronises. */
int krea2_check_device_error(void* stream);

/* Self-test of the failure detection: launches one kernel that waits, with a limit of limit_ms
 * (1..5000), on a barrier that nothing arrives on. The bounded wait expires, the kernel writes 1
 * to *waited (device int) and returns; a following krea2_check_device_error then reports
 * KREA2_ERR_TIMEOUT and clears the error word. The context stays usable. */
int krea2_selftest_wait_timeout(int limit_ms, int* waited, void* stream);

/* Bytes of device workspace that krea2_block_forward / krea2_backbone_forward need for
 * these shapes (0 on invalid arguments). The workspace must be 256-byte aligned. */
size_t krea2_workspace_size(const Krea2Dims* dims, int B, int T, int N, int dtype);

/* 3-axis RoPE tables ([API] axes_dims_rope, rope_theta; [ARCH] §一: adapted from Flux's
 * FluxPosEmbed). position_ids (S, 3) fp32 rows (t, h, w); text rows are zero and image rows
 * (0, h, w) ([PIPE] prepare_position_ids). For axis a with d_a dims, pair j turns by
 * pos_a * theta^(-2j/d_a); pairs are concatenated over the axes in order t, h, w, giving
 * D/2 angles per row. Angles, cos and sin are evaluated in fp64 and stored fp32:
 * cos_out, sin_out (S, D/2). S >= 1. */
int krea2_rope_tables(const Krea2Dims* dims, const float* position_ids, int S,
                      float* cos_out, float* sin_out, void* stream);

/* Grouped-query attention of one block from the raw fused projection ([ARCH] §四.3):
 *   qkvg (B*S, H*D + 2*Hkv*D + H*D) in `dtype`: per row [q | k | v | gate], head-major,
 *        q/k BEFORE their RMSNorm and RoPE.
 *   Per head: q, k <- RMSNorm over D with multiplier (1 + q_norm_w / k_norm_w), eps = dims->eps;
 *   then RoPE with cos/sin (S, D/2) from krea2_rope_tables, rotating adjacent dim pairs
 *   (2p, 2p+1): x0' = x0 c - x1 s, x1' = x1 c + x0 s.
 *   Query head h attends with KV head h / (H/Hkv) (repeat_interleave order) over all S keys of
 *   its batch row except padded text keys; softmax(q.k / sqrt(D)) v; heads are merged and
 *   multiplied elementwise by sigmoid(gate).
 *   out (B*S, H*D) in `dtype`. Requires N >= 1 (every row then has a valid key).
 *   workspace: device scratch of krea2_attention_workspace_size() bytes, 256-byte aligned (the
 *   tensor-core path writes the normalised, rotated q|k there; NULL allowed when that is 0).
 *   Kernels: bf16 with D = 128 and H = 4*Hkv runs on the tensor cores (tcgen05); other shapes
 *   and the fp32 path run a SIMT kernel (D in {64, 128}). */
size_t krea2_attention_workspace_size(const Krea2Dims* dims, int B, int T, int N, int dtype);
int krea2_gqa_attention(const Krea2Dims* dims, int B, int T, int N, int dtype,
                        const void* qkvg, const float* q_norm_w, const float* k_norm_w,
                        const float* cos, const float* sin, const uint8_t* text_mask,
                        void* out, void* workspace, size_t ws_bytes, void* stream);

/* Attention without device allocation. The pages have no counterpart of this entry point:
 * it exists for callers that cannot hand the library a workspace, such as a plugin interface
 * that passes only input and output buffers, or a runtime whose allocator owns all device
 * memory and forbids side allocations while it serves.
 * Arguments, layouts and results are those of krea2_gqa_attention. The q|k scratch that call
 * takes from its workspace lives here in a file-scope device array of
 * KREA2_NOALLOC_SCRATCH_BYTES, resident on every GPU that loads it until the process exits.
 * Shapes needing more scratch than that (B*(T+N)*(H+Hkv)*D*2 bytes on the tensor-core path;
 * 4369 tokens at the default 48/12 heads x 128) are rejected with KREA2_ERR_WORKSPACE before
 * anything runs. The call allocates and frees nothing. The first call on each device looks up
 * the array's device address (cudaGetSymbolAddress) with that device current, so it should
 * come before any stream capture. `stream` must belong to the current device (KREA2_ERR_ARG
 * otherwise). All calls share the array and it keeps the last call's contents (nothing in it
 * needs to start at zero), so calls that overlap on the GPU race. */
#define KREA2_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)
int krea2_gqa_attention_noalloc(const Krea2Dims* dims, int B, int T, int N, int dtype,
                                const void* qkvg, const float* q_norm_w, const float* k_norm_w,
                                const float* cos, const float* sin, const uint8_t* text_mask,
                                void* out, void* stream);

/* Block-causal attention (page "QwenImage21Transformer2DModel": query q reads key k iff
 * q >= k or both lie in the same image block; a variant for models built on this block).
 * That pattern is a per-query key prefix: q reads keys [0, key_end[q]) with key_end[q] = q + 1
 * for a text token and the end of its image block for an image token.
 * krea2_block_causal_key_end computes key_end (HOST arrays, S entries) from image_ids (-1 at text
 * positions, one id per image block, blocks contiguous). Returns KREA2_ERR_ARG if a block is not
 * contiguous. */
int krea2_block_causal_key_end(const int32_t* image_ids, int S, int32_t* key_end);

/* krea2_gqa_attention under the block-causal pattern: key_end (S) int32 DEVICE array from
 * krea2_block_causal_key_end, shared by all batch rows; the text mask still removes padded keys.
 * A query with no readable key outputs zeros. Tensor-core path only (bf16, D = 128,
 * H/Hkv in {1, 2, 4}); other shapes return KREA2_ERR_UNSUPPORTED. Workspace as
 * krea2_gqa_attention. Key tiles beyond every query of a CTA are never loaded. */
int krea2_gqa_attention_block_causal(const Krea2Dims* dims, int B, int T, int N, int dtype,
                                     const void* qkvg, const float* q_norm_w, const float* k_norm_w,
                                     const float* cos, const float* sin, const uint8_t* text_mask,
                                     const int32_t* key_end, void* out, void* workspace,
                                     size_t ws_bytes, void* stream);

/* Key/value cache of the block-causal variant (page "QwenImage21Transformer2DModel": with
 * causal_condition the text and condition-image tokens are modulated from t = 0, so their keys
 * and values do not change between denoising steps and are kept in a kv_cache). The cache holds,
 * per batch row, `capacity` rows of keys and of values: k_cache and v_cache are
 * (B, capacity, Hkv*D) bf16 DEVICE buffers, 16-byte aligned, owned by the caller.
 *
 * krea2_kv_cache_append stores the keys and values of n tokens in rows [row0, row0 + n) of every
 * batch row: k RMS-normalised over head_dim with weight (1 + k_norm_w) and rotated by (cos, sin),
 * v as projected (the same k and v krea2_gqa_attention computes).
 *   qkvg (B*n, H*D + 2*Hkv*D + H*D) raw fused projection of the n tokens; only the k and v
 *   columns are read. cos, sin (n, D/2) fp32: RoPE tables of the n tokens.
 * Returns KREA2_ERR_ARG unless 0 <= row0 and row0 + n <= capacity; tensor-core shapes only
 * (bf16, D = 128, H/Hkv in {1, 2, 4}), else KREA2_ERR_UNSUPPORTED. */
int krea2_kv_cache_append(const Krea2Dims* dims, int B, int n, int row0, int capacity, int dtype,
                          const void* qkvg, const float* k_norm_w, const float* cos, const float* sin,
                          void* k_cache, void* v_cache, void* stream);

/* Attention of Nq new tokens over the first L cached keys, on the tensor-core attention kernel.
 * The new tokens are the keys at positions [L - Nq, L); their keys and values must already be in
 * the cache (krea2_kv_cache_append with row0 = L - Nq). Keys [0, T) are text tokens, and
 * text_mask (B, T) uint8 (NULL: all valid) removes padded ones.
 *   key_end NULL: every new token reads all L keys. That is the last image block of a
 *     block-causal sequence (the image being denoised), which sees every earlier token and its
 *     own block.
 *   key_end (Nq) int32 DEVICE: new token i reads keys [0, key_end[i]) (absolute positions, e.g.
 *     rows L - Nq .. L - 1 of krea2_block_causal_key_end over the whole sequence); a key_end
 *     below the token's own position + 1 is raised to it.
 *   qkvg (B*Nq, H*D + 2*Hkv*D + H*D) raw fused projection of the new tokens: q is RMS-normalised
 *     (1 + q_norm_w) and rotated by cos, sin (Nq, D/2); the gate columns gate the output.
 *   out (B*Nq, H*D) bf16: sigmoid(gate) * attention, heads merged. A token with no readable key
 *     outputs zeros.
 *   workspace: krea2_kv_cache_attention_workspace_size bytes, 256-byte aligned (prepared q).
 * Returns KREA2_ERR_ARG unless 1 <= Nq <= L, 0 <= T <= L and capacity >= L. */
size_t krea2_kv_cache_attention_workspace_size(const Krea2Dims* dims, int B, int Nq, int dtype);
int krea2_gqa_attention_kv_cache(const Krea2Dims* dims, int B, int T, int L, int Nq, int dtype,
                                 const void* qkvg, const float* q_norm_w, const float* cos, const float* sin,
                                 const uint8_t* text_mask, const void* k_cache, const void* v_cache,
                                 int capacity, const int32_t* key_end, void* out, void* workspace,
                                 size_t ws_bytes, void* stream);

/* Shared modulation of one block plus its table, then a modulated RMSNorm ([ARCH] §四.2,
 * §四.4): with mod = temb (B, 6C) viewed as (B, 6, C) plus table (6, C),
 *   out[b, s] = (1 + mod[b, chunk]) * rms(h[b, s]) * (1 + norm_w) + mod[b, chunk + 1].
 * chunk = 0 gives norm1 (prescale, preshift), chunk = 3 gives norm2 (postscale, postshift).
 * h (B*S, C) fp32; out (B*S, C) in `dtype`. */
int krea2_modulated_rmsnorm(const Krea2Dims* dims, int B, int S, int dtype,
                            const float* h, const float* norm_w, const float* temb,
                            const float* table, int chunk, void* out, void* stream);

/* Dense projection out = A · Wᵀ with a fused epilogue (the block's linears, [ARCH] §四.2/§四.3).
 *   A (M, K), W (Nw, K) in `dtype`, fp32 accumulation.
 *   epilogue KREA2_EPI_STORE:  out (M, Nw) in `dtype`.
 *   epilogue KREA2_EPI_SWIGLU: W is gate/up interleaved in 64-row groups (see w_gu);
 *             out (M, Nw/2) in `dtype`, out = silu(gate) * up.
 *   epilogue KREA2_EPI_RESID:  out is the fp32 residual (M, Nw), updated in place:
 *             out[r, c] += gate[(r / rows_per_batch) * gate_stride + c] * (A·Wᵀ)[r, c].
 *             (gate_stride = 6C for a modulation chunk; 0 broadcasts one vector.)
 *   bf16 path: Nw % 128 == 0, K % 64 == 0, M >= 1; gate/rows_per_batch used by RESID only.
 *             A, W and out must be 16-byte aligned: KREA2_ERR_ARG otherwise. Each output
 *             element is written by exactly one thread, so results are deterministic. */
enum { KREA2_EPI_STORE = 0, KREA2_EPI_SWIGLU = 1, KREA2_EPI_RESID = 2 };
int krea2_linear(int dtype, int epilogue, int M, int Nw, int K,
                 const void* A, const void* W, void* out,
                 const float* gate, int rows_per_batch, long long gate_stride, void* stream);

/* Time path ([ARCH] §四 data flow, §四.5): sinusoid of 1000*t, width t_dim, cosine half first,
 * frequencies exp(-ln(10000) i / (t_dim/2)); Linear(t_dim, C) + GELU-tanh + Linear(C, C)
 * (time_embed); e = GELU-tanh(time_embed); temb = time_mod_proj(e) = e · mod_wᵀ + mod_b.
 * timestep (B) fp32 in [0, 1]; temb_out (B, 6C) fp32; e_out (B, C) fp32 (feeds the final
 * layer). Reads w->t1_*, t2_*, mod_*. scratch: device fp32 buffer of >= B*C floats. */
int krea2_time_embed(const Krea2Dims* dims, int B, int dtype, const float* timestep,
                     const Krea2ModelWeights* w, float* temb_out, float* e_out,
                     float* scratch, void* stream);

/* Final layer on image rows ([ARCH] §四.6): (scale, shift) = final_table + e;
 * y = (1 + scale) * rms(x) * (1 + final_norm_w) + shift; velocity = y · final_wᵀ + final_b.
 * h (B*S, C) fp32 full sequence (text rows are skipped, [ARCH] §二); e (B, C) fp32;
 * velocity (B, N, in_ch) in `dtype` (in_ch <= 64). Reads w->final_*.
 * workspace: krea2_final_layer_workspace_size bytes, 256-byte aligned (NULL allowed when that is
 * 0). bf16 with in_ch % 64 == 0: the norm writes y (bf16) there and the projection runs on the
 * tensor cores; otherwise one fused SIMT kernel (no workspace). */
size_t krea2_final_layer_workspace_size(const Krea2Dims* dims, int B, int N, int dtype);
int krea2_final_layer(const Krea2Dims* dims, int B, int T, int N, int dtype,
                      const float* h, const float* e, const Krea2ModelWeights* w,
                      void* velocity, void* workspace, size_t ws_bytes, void* stream);

/* One Krea2TransformerBlock forward ([ARCH] §四.2), in place on the fp32 residual:
 *   mod = temb + table;  xn = (1+prescale)*norm1(h) + preshift;
 *   h += pregate * to_out(attention(xn));  xn2 = (1+postscale)*norm2(h) + postshift;
 *   h += postgate * W_down(silu(W_gate xn2) * W_up xn2).
 * h (B*S, C) fp32 in/out; temb (B, 6C) fp32 (the shared time modulation); cos/sin from
 * krea2_rope_tables; workspace >= krea2_workspace_size(). */
int krea2_block_forward(const Krea2Dims* dims, int B, int T, int N, int dtype,
                        float* h, const float* temb, const Krea2BlockWeights* w,
                        const float* cos, const float* sin, const uint8_t* text_mask,
                        void* workspace, size_t ws_bytes, void* stream);

/* krea2_block_forward that also records caller-created CUDA events (cudaEvent_t passed as
 * void*) on `stream`: events[i] just before launch i and events[8] after the last, for the eight
 * launches 0 modulation, 1 norm1, 2 fused projection (q/k norm + RoPE in its epilogue on the
 * tensor-core path), 3 attention, 4 to_out + gated residual, 5 norm2, 6 gate/up + SwiGLU,
 * 7 down + gated residual. Meant for per-kernel timing; results equal krea2_block_forward. */
int krea2_block_forward_traced(const Krea2Dims* dims, int B, int T, int N, int dtype,
                               float* h, const float* temb, const Krea2BlockWeights* w,
                               const float* cos, const float* sin, const uint8_t* text_mask,
                               void* workspace, size_t ws_bytes, void* const* events, void* stream);

/* Number of kernels this library has launched in this process so far (all entry points). */
unsigned long long krea2_launch_count(void);

/* ---- sampler (the steps either side of the backbone in [PIPE] __call__) ----------------------
 * Resolution-aware shift of the sigma schedule ([PIPE] scheduler: use_dynamic_shifting with
 * base_shift 0.5, max_shift 1.15, base_image_seq_len 256, max_image_seq_len 6400): mu on the
 * straight line through (256, 0.5) and (6400, 1.15) in image_seq_len (a reading; the distilled
 * checkpoint uses the fixed mu = 1.15). Host function. */
double krea2_shift_mu(int image_seq_len);

/* Sigma schedule ([PIPE] __call__: default grid linspace(1, 1/n_steps, n_steps), exponential time
 * shift sigma' = e^mu / (e^mu + (1/sigma - 1)) (a reading), then the terminal 0). Writes n_steps + 1
 * values to sigmas_out (HOST memory), computed in fp64. KREA2_ERR_ARG for n_steps < 1. */
int krea2_sigma_schedule(int n_steps, double mu, float* sigmas_out);

/* One sampler step on the device ([PIPE] guidance_scale, scheduler step; [ARCH] §五):
 *   v = v_cond + guidance * (v_cond - v_uncond)   (v_uncond NULL or guidance <= 0: v = v_cond),
 *   x <- x + (sigma_next - sigma) * v.
 * x (n) fp32 latents, updated in place; v_cond, v_uncond (n) in `dtype`;
 * x_model (copies * n) in `dtype`, optional: receives `copies` back-to-back copies of the new x
 * (the next model input, copies = 2 for a [cond, uncond] batch); timestep_out (copies) fp32,
 * optional: receives sigma_next (the next model timestep, t / num_train_timesteps). */
int krea2_euler_cfg_step(int dtype, long long n, float* x, const void* v_cond, const void* v_uncond,
                         float guidance, float sigma, float sigma_next, void* x_model, int copies,
                         float* timestep_out, void* stream);

/* Bytes of device workspace krea2_sample needs (0 on invalid arguments). */
size_t krea2_sample_workspace_size(const Krea2Dims* dims, int T, int N, int dtype, int cfg);

/* The whole sampling loop on the device, for one image ([PIPE] __call__): for i = 0..n_steps-1 the
 * backbone runs at timestep sigmas[i] on the batch [cond] (guidance <= 0) or [cond, uncond]
 * (guidance > 0, one batch-2 forward), then krea2_euler_cfg_step moves the latents to
 * sigmas[i+1]. latents (N, in_ch) fp32, in/out (initial noise in, sample out); text_cond,
 * text_uncond (T, C) in `dtype` (text_uncond unused when guidance <= 0); mask_cond, mask_uncond
 * (T) uint8 or NULL; position_ids (T+N, 3); sigmas: HOST array of n_steps + 1 values (e.g. from
 * krea2_sigma_schedule); workspace >= krea2_sample_workspace_size(dims, T, N, dtype, guidance > 0).
 * Asynchronous; every launch goes to `stream`, so the call can be captured in a CUDA graph. */
int krea2_sample(const Krea2Dims* dims, int T, int N, int dtype, float* latents,
                 const void* text_cond, const void* text_uncond, const uint8_t* mask_cond,
                 const uint8_t* mask_uncond, const float* position_ids, const float* sigmas,
                 int n_steps, float guidance, const Krea2ModelWeights* w, void* workspace,
                 size_t ws_bytes, void* stream);

/* ---- text conditioning (Krea2TextFusion + txt_in, [ARCH] §四.1 and §四 module list) ----------
 * Text-fusion hyper-parameters ([API] text_hidden_dim Dt = 2560, num_text_layers L = 12,
 * text_num_attention_heads H = 20, text_num_key_value_heads Hkv = 20, text_intermediate_size
 * F = 6912, num_layerwise_text_blocks 2, num_refiner_text_blocks 2; D = Dt / H head dim; C the
 * backbone hidden size that txt_in projects to). */
typedef struct {
  int Dt, L, H, Hkv, D, F, n_layerwise, n_refiner, C;
  float eps;
} Krea2TextDims;

/* Text-fusion parameters. layerwise / refiner: HOST arrays of n_layerwise / n_refiner block
 * weights (Krea2BlockWeights with hidden size Dt; scale_shift_table must be NULL: the fusion
 * blocks have no time modulation); layer_w (L) fp32: Linear(L, 1, bias=False) over the layer
 * axis; txt_in_w (C, Dt) in `dtype`, txt_in_b (C) fp32 (a reading: txt_in is Linear + bias). */
typedef struct {
  const Krea2BlockWeights* layerwise;
  const Krea2BlockWeights* refiner;
  const float* layer_w;
  const void* txt_in_w;
  const float* txt_in_b;
} Krea2TextWeights;

size_t krea2_text_fusion_workspace_size(const Krea2TextDims* td, int B, int T, int dtype);

/* Text conditioning from the stacked encoder states ([ARCH] §四.1): each token's (L, Dt) stack is
 * its own sequence through the layerwise blocks (pre-norm blocks with q/k RMSNorm, sigmoid-gated
 * MHA and SwiGLU, no RoPE, no time modulation: a reading); Linear(L, 1) collapses the layer axis;
 * the token sequence goes through the refiner blocks under the text mask; txt_in projects to C.
 * ehs (B, T, L, Dt) in `dtype`; text_mask (B, T) uint8 or NULL; text_out (B, T, C) in `dtype`,
 * ready for krea2_backbone_forward's text_states. Computed once per prompt (no timestep). */
int krea2_text_fusion(const Krea2TextDims* td, int B, int T, int dtype, const void* ehs,
                      const uint8_t* text_mask, const Krea2TextWeights* w, void* text_out,
                      void* workspace, size_t ws_bytes, void* stream);

/* Backbone forward from post-fusion text features ([API] forward; [ARCH] §四 data flow):
 * RoPE tables; time path; x = cat([text_states, img_in(hidden_states)]); n_layers blocks;
 * drop text rows; final layer.
 *   hidden_states (B, N, in_ch) and text_states (B, T, C) in `dtype` (text_states stands for
 *   the text-fusion + txt_in output); position_ids (T+N, 3) fp32; timestep (B) fp32;
 *   w->blocks host array of n_layers; velocity (B, N, in_ch) in `dtype`. */
int krea2_backbone_forward(const Krea2Dims* dims, int B, int T, int N, int dtype,
                           const void* hidden_states, const void* text_states,
                           const float* position_ids, const uint8_t* text_mask,
                           const float* timestep, const Krea2ModelWeights* w,
                           void* velocity, void* workspace, size_t ws_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* KREA2_H */
