// C ABI entry points (include/krea2.h): argument checks, workspace carving and the launch
// sequence of the block and the backbone. Every step runs in this library's kernels.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <vector>

#include <cuda_bf16.h>

#include "krea2_internal.h"

namespace krea2 {

static thread_local char g_err[512] = "";
static std::atomic<unsigned long long> g_launches{0};

void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

int set_error(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

int num_sms() {
  static int cache[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (!cache[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

namespace {

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// [ARCH] §三: sum(axes_dims_rope) == attention_head_dim, else ValueError; plus the limits of
// this library's kernels.
int check_dims(const Krea2Dims* d, int dtype) {
  if (!d) return set_error(KREA2_ERR_ARG, "dims is NULL");
  if (dtype != KREA2_BF16 && dtype != KREA2_F32) return set_error(KREA2_ERR_ARG, "unknown dtype %d", dtype);
  if (d->H <= 0 || d->Hkv <= 0 || d->D <= 0 || d->C <= 0 || d->F <= 0)
    return set_error(KREA2_ERR_ARG, "non-positive model dimension");
  if ((long long)d->C != (long long)d->H * d->D)
    return set_error(KREA2_ERR_ARG, "hidden size C=%d != heads*head_dim=%lld", d->C, (long long)d->H * d->D);
  if (d->H % d->Hkv) return set_error(KREA2_ERR_ARG, "heads %d not a multiple of kv heads %d", d->H, d->Hkv);
  for (int a = 0; a < 3; ++a)
    if (d->axes[a] < 0 || (d->axes[a] & 1)) return set_error(KREA2_ERR_ARG, "RoPE axis %d has odd size %d", a, d->axes[a]);
  const long long axes_sum = (long long)d->axes[0] + d->axes[1] + d->axes[2];
  if (axes_sum != d->D)
    return set_error(KREA2_ERR_ARG, "sum(axes_dims_rope)=%lld != attention_head_dim=%d", axes_sum, d->D);
  if (!(d->theta > 0.f) || !(d->eps > 0.f)) return set_error(KREA2_ERR_ARG, "theta and eps must be positive");
  if (d->D != 64 && d->D != 128) return set_error(KREA2_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
  if (d->C % 128 || d->C > 8192) return set_error(KREA2_ERR_UNSUPPORTED, "hidden size must be a multiple of 128, <= 8192");
  if (d->F % 64) return set_error(KREA2_ERR_UNSUPPORTED, "intermediate size must be a multiple of 64");
  return KREA2_OK;
}

int check_model_dims(const Krea2Dims* d) {
  if (d->n_layers < 0) return set_error(KREA2_ERR_ARG, "n_layers < 0");
  if (d->in_ch <= 0) return set_error(KREA2_ERR_ARG, "in_ch must be positive");
  if (d->in_ch > 64) return set_error(KREA2_ERR_UNSUPPORTED, "in_ch must be <= 64");
  if (d->t_dim <= 0 || d->t_dim % 8 || d->t_dim > d->C)
    return set_error(KREA2_ERR_UNSUPPORTED, "t_dim must be a positive multiple of 8 and <= C");
  return KREA2_OK;
}

int check_shape(int B, int T, int N) {
  if (B <= 0) return set_error(KREA2_ERR_ARG, "batch must be positive");
  if (T < 0) return set_error(KREA2_ERR_ARG, "text length must be >= 0");
  if (N <= 0) return set_error(KREA2_ERR_ARG, "image_seq_len must be >= 1 (every query then has a valid key)");
  if ((long long)B * ((long long)T + N) > (1LL << 30)) return set_error(KREA2_ERR_ARG, "too many tokens");
  return KREA2_OK;
}

constexpr size_t ALIGN = 256;
inline size_t up(size_t x) { return (x + ALIGN - 1) & ~(ALIGN - 1); }

struct Ws {
  size_t mod, xn, qkvg, attn, u, h, cs, sn, temb, e, tscr, total;
};

Ws ws_layout(const Krea2Dims* d, int B, int T, int N, int dtype) {
  const size_t es = dtype == KREA2_BF16 ? 2 : 4;
  const size_t S = (size_t)T + N, M = (size_t)B * S, C = d->C;
  const size_t QC = 2 * (size_t)d->H * d->D + 2 * (size_t)d->Hkv * d->D;
  Ws w{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off += up(bytes);
    return o;
  };
  w.mod = take((size_t)B * 6 * C * 4);
  w.xn = take(M * C * es);
  w.qkvg = take(M * QC * es);
  w.attn = take(M * (size_t)d->H * d->D * es);
  w.u = take(M * (size_t)d->F * es);
  w.h = take(M * C * 4);
  w.cs = take(S * (size_t)(d->D / 2) * 4);
  w.sn = take(S * (size_t)(d->D / 2) * 4);
  w.temb = take((size_t)B * 6 * C * 4);
  w.e = take((size_t)B * C * 4);
  w.tscr = take((size_t)B * C * 4);
  w.total = off;
  return w;
}

// Standalone attention on raw projection columns ([ARCH] §四.3): the tensor-core path first
// writes normalised, rotated q|k into the workspace, then runs the flash-attention core.
int attention_raw(const AttnParams& p, int dtype, void* ws, cudaStream_t s, const int* key_end = nullptr) {
  if (dtype == KREA2_BF16 && attention_tc_supported(p.D, p.H, p.Hkv)) {
    const long long QC = 2LL * p.H * p.D + 2LL * p.Hkv * p.D;
    int rc = launch_qk_prep(p.qkvg, QC, p.B, p.S, p.H, p.Hkv, p.eps, p.q_norm_w, p.k_norm_w, p.cos, p.sin, ws, s);
    if (rc) return rc;
    AttnTcArgs a{};
    a.B = p.B; a.T = p.T; a.N = p.N; a.H = p.H; a.Hkv = p.Hkv;
    const long long QK = (long long)(p.H + p.Hkv) * p.D;
    const __nv_bfloat16* prep = reinterpret_cast<const __nv_bfloat16*>(ws);
    const __nv_bfloat16* raw = reinterpret_cast<const __nv_bfloat16*>(p.qkvg);
    a.q = prep; a.q_stride = QK;
    a.k = prep + (long long)p.H * p.D; a.k_stride = QK;
    a.v = raw + (long long)(p.H + p.Hkv) * p.D; a.v_stride = QC;
    a.g = raw + (long long)(p.H + 2 * p.Hkv) * p.D; a.g_stride = QC;
    a.text_mask = p.text_mask; a.out = p.out; a.key_end = key_end;
    return attention_tc_core(a, s);
  }
  if (key_end) return set_error(KREA2_ERR_UNSUPPORTED, "block-causal attention needs bf16, D=128, H/Hkv in {1,2,4}");
  return attention_simt(p, dtype == KREA2_BF16, s);
}

size_t attention_ws_bytes(const Krea2Dims* d, int B, int T, int N, int dtype) {
  if (dtype == KREA2_BF16 && attention_tc_supported(d->D, d->H, d->Hkv))
    return (size_t)B * ((size_t)T + N) * (size_t)(d->H + d->Hkv) * d->D * 2;
  return 0;
}

int linear_dispatch(int dtype, int epi, int M, int Nw, int K, const void* A, const void* W, void* out,
                    const float* gate, int rows_per_batch, long long gate_stride, cudaStream_t s) {
  if (dtype == KREA2_BF16) {
    GemmParams p{};
    p.M = M; p.N = Nw; p.K = K; p.out = out;
    p.gate = gate; p.rows_per_batch = rows_per_batch; p.gate_stride = gate_stride;
    return gemm_bf16(epi, p, A, W, s);
  }
  SimtGemmParams p{};
  p.M = M; p.N = Nw; p.K = K; p.out = out;
  p.gate = gate; p.rows_per_batch = rows_per_batch; p.gate_stride = gate_stride;
  const int sepi = epi == EPI_STORE ? SEPI_STORE_F32 : epi == EPI_SWIGLU ? SEPI_SWIGLU_F32 : SEPI_RESID;
  return gemm_simt(sepi, p, A, false, W, false, s);
}

int check_block_weights(const Krea2BlockWeights* w) {
  if (!w || !w->w_qkvg || !w->w_out || !w->w_gu || !w->w_down || !w->norm1_w || !w->norm2_w || !w->q_norm_w ||
      !w->k_norm_w || !w->scale_shift_table)
    return set_error(KREA2_ERR_ARG, "block weights: NULL pointer");
  return KREA2_OK;
}

int check_model_weights(const Krea2ModelWeights* w, int n_layers) {
  if (!w || !w->img_in_w || !w->img_in_b || !w->t1_w || !w->t1_b || !w->t2_w || !w->t2_b || !w->mod_w ||
      !w->mod_b || !w->final_norm_w || !w->final_table || !w->final_w || !w->final_b)
    return set_error(KREA2_ERR_ARG, "model weights: NULL pointer");
  if (n_layers > 0 && !w->blocks) return set_error(KREA2_ERR_ARG, "model weights: blocks is NULL");
  for (int l = 0; l < n_layers; ++l) {
    int rc = check_block_weights(&w->blocks[l]);
    if (rc) return set_error(rc, "block %d weights: NULL pointer", l);
  }
  return KREA2_OK;
}

// Final layer ([ARCH] §四.6). With a bf16 scratch of B*N*C (final_layer_tc_scratch) the modulated
// norm of the image rows goes to the scratch and the projection runs on the tensor cores (W rows
// beyond in_ch read as zeros, only in_ch columns are stored); otherwise one fused SIMT kernel.
int final_layer_impl(const Krea2Dims* d, int B, int T, int N, bool bf, const float* h, const float* e,
                     const Krea2ModelWeights* w, void* velocity, void* scratch, cudaStream_t s) {
  if (!scratch || !final_layer_tc_scratch(d, B, N, bf)) return launch_final_layer(d, B, T, N, bf, h, e, w, velocity, s);
  ModNormArgs a{};
  a.h = h; a.w = w->final_norm_w;
  a.sc = e; a.sh = e; a.mod_stride = d->C;  // (scale, shift) = final_table + e ([ARCH] §四.6, reading c16)
  a.sc_tab = w->final_table; a.sh_tab = w->final_table + d->C;
  a.B = B; a.rows = N; a.S_in = T + N; a.row0 = T; a.C = d->C; a.eps = d->eps;
  a.out = scratch; a.out_bf16 = true;
  int rc = launch_mod_rmsnorm_rows(a, s);
  if (rc) return rc;
  GemmParams gp{};
  gp.M = B * N; gp.N = (d->in_ch + 127) / 128 * 128; gp.K = d->C; gp.out = velocity; gp.bias = w->final_b;
  gp.out_ld = d->in_ch; gp.n_store = d->in_ch; gp.w_rows = d->in_ch;
  return gemm_bf16(EPI_STORE, gp, scratch, w->final_w, s);
}

// img_in = Linear(in_ch, C, bias=True) on the packed latents, written to the image rows of the
// residual (after the T text rows of each batch row) ([ARCH] §四 module list and data flow).
int img_in_impl(const Krea2Dims* d, int B, int T, int N, bool bf, const void* hidden, const Krea2ModelWeights* w,
                float* h, cudaStream_t s) {
  const int S = T + N, C = d->C;
  if (bf && d->in_ch % 64 == 0) {
    GemmParams gp{};
    gp.M = B * N; gp.N = C; gp.K = d->in_ch; gp.out = h; gp.bias = w->img_in_b;
    gp.map_N = N; gp.map_T = T; gp.map_S = S;
    return gemm_bf16(EPI_BIAS_ROWMAP, gp, hidden, w->img_in_w, s);
  }
  SimtGemmParams ip{};
  ip.M = B * N; ip.N = C; ip.K = d->in_ch; ip.out = h; ip.bias = w->img_in_b;
  ip.map_N = N; ip.map_T = T; ip.map_S = S;
  return gemm_simt(SEPI_BIAS_ROWMAP, ip, hidden, bf, w->img_in_w, bf, s);
}

// The block's launch sequence ([ARCH] §四.2) on an already validated configuration.
int block_impl(const Krea2Dims* d, int B, int T, int N, int dtype, float* h, const float* temb,
               const Krea2BlockWeights* w, const float* cs, const float* sn, const uint8_t* mask, uint8_t* ws,
               const Ws& L, cudaStream_t s, void* const* ev = nullptr) {
  auto mark = [&](int i) {
    if (ev) cudaEventRecord(reinterpret_cast<cudaEvent_t>(ev[i]), s);
  };
  const int S = T + N, M = B * S, C = d->C, HD = d->H * d->D;
  const int QC = 2 * HD + 2 * d->Hkv * d->D;
  const bool bf = dtype == KREA2_BF16;
  float* mod = reinterpret_cast<float*>(ws + L.mod);
  void* xn = ws + L.xn;
  void* qkvg = ws + L.qkvg;
  void* attn = ws + L.attn;
  void* u = ws + L.u;
  int rc;
  mark(0);
  // no table: a block without time modulation (text fusion): scale 0, shift 0, gate 1
  if ((rc = w->scale_shift_table ? launch_modulation(temb, w->scale_shift_table, B, C, mod, s)
                                 : launch_unit_modulation(B, C, mod, s)))
    return rc;
  mark(1);
  if ((rc = launch_mod_rmsnorm(h, w->norm1_w, mod, nullptr, 0, B, S, C, d->eps, xn, bf, s))) return rc;
  if (bf && attention_tc_supported(d->D, d->H, d->Hkv)) {
    // fused projection with q/k RMSNorm + RoPE in the epilogue, then the tensor-core attention
    GemmParams gp{};
    gp.M = M; gp.N = QC; gp.K = C; gp.out = qkvg; gp.rows_per_batch = S;
    gp.qw = w->q_norm_w; gp.kw = w->k_norm_w; gp.cos = cs; gp.sin = sn;
    gp.HD = HD; gp.KVD = d->Hkv * d->D; gp.eps = d->eps;
    mark(2);
    if ((rc = gemm_bf16(EPI_QKV, gp, xn, w->w_qkvg, s))) return rc;
    const __nv_bfloat16* base = reinterpret_cast<const __nv_bfloat16*>(qkvg);
    AttnTcArgs a{};
    a.B = B; a.T = T; a.N = N; a.H = d->H; a.Hkv = d->Hkv;
    a.q = base; a.q_stride = QC;
    a.k = base + HD; a.k_stride = QC;
    a.v = base + HD + d->Hkv * d->D; a.v_stride = QC;
    a.g = base + HD + 2 * d->Hkv * d->D; a.g_stride = QC;
    a.text_mask = mask; a.out = attn;
    mark(3);
    if ((rc = attention_tc_core(a, s))) return rc;
  } else {
    mark(2);
    if ((rc = linear_dispatch(dtype, EPI_STORE, M, QC, C, xn, w->w_qkvg, qkvg, nullptr, S, 0, s))) return rc;
    AttnParams ap{};
    ap.B = B; ap.T = T; ap.N = N; ap.S = S; ap.H = d->H; ap.Hkv = d->Hkv; ap.D = d->D; ap.eps = d->eps;
    ap.qkvg = qkvg; ap.q_norm_w = w->q_norm_w; ap.k_norm_w = w->k_norm_w; ap.cos = cs; ap.sin = sn;
    ap.text_mask = mask; ap.out = attn;
    mark(3);
    if ((rc = attention_simt(ap, bf, s))) return rc;
  }
  mark(4);
  if ((rc = linear_dispatch(dtype, EPI_RESID, M, C, HD, attn, w->w_out, h, mod + 2 * C, S, 6LL * C, s))) return rc;
  mark(5);
  if ((rc = launch_mod_rmsnorm(h, w->norm2_w, mod, nullptr, 3, B, S, C, d->eps, xn, bf, s))) return rc;
  mark(6);
  if ((rc = linear_dispatch(dtype, EPI_SWIGLU, M, 2 * d->F, C, xn, w->w_gu, u, nullptr, S, 0, s))) return rc;
  mark(7);
  if ((rc = linear_dispatch(dtype, EPI_RESID, M, C, d->F, u, w->w_down, h, mod + 5 * C, S, 6LL * C, s))) return rc;
  mark(8);
  return KREA2_OK;
}

}  // namespace
}  // namespace krea2

using namespace krea2;

extern "C" {

const char* krea2_last_error_string(void) { return g_err; }

int krea2_check_device_error(void* stream) {
  cudaError_t e = cudaStreamSynchronize(as_stream(stream));
  if (e != cudaSuccess) return set_error(KREA2_ERR_CUDA, "stream error: %s", cudaGetErrorString(e));
  const int ve[2] = {take_device_error_gemm(), take_device_error_attention()};
  const char* names[2] = {"GEMM", "attention"};
  for (int i = 0; i < 2; ++i) {
    if (ve[i] < 0) return set_error(KREA2_ERR_CUDA, "cannot read the device error word");
    if (ve[i] > 0)
      return set_error(KREA2_ERR_TIMEOUT, "a bounded device-side wait expired in the %s kernels (code %d)",
                       names[i], ve[i]);
  }
  return KREA2_OK;
}

int krea2_selftest_wait_timeout(int limit_ms, int* waited, void* stream) {
  if (limit_ms < 1 || limit_ms > 5000 || !waited) return set_error(KREA2_ERR_ARG, "limit_ms must be 1..5000, waited non-NULL");
  return launch_wait_timeout_selftest((unsigned long long)limit_ms * 1000000ull, waited, as_stream(stream));
}

size_t krea2_workspace_size(const Krea2Dims* dims, int B, int T, int N, int dtype) {
  if (check_dims(dims, dtype) || check_shape(B, T, N)) return 0;
  return ws_layout(dims, B, T, N, dtype).total;
}

int krea2_rope_tables(const Krea2Dims* dims, const float* position_ids, int S, float* cos_out, float* sin_out,
                      void* stream) {
  int rc = check_dims(dims, KREA2_F32);
  if (rc) return rc;
  if (!position_ids || !cos_out || !sin_out) return set_error(KREA2_ERR_ARG, "NULL pointer");
  if (S <= 0) return set_error(KREA2_ERR_ARG, "position_ids must have shape (S, 3) with S >= 1");
  return launch_rope_tables(position_ids, S, dims->axes[0], dims->axes[1], dims->axes[2], dims->theta, cos_out,
                            sin_out, as_stream(stream));
}

size_t krea2_attention_workspace_size(const Krea2Dims* dims, int B, int T, int N, int dtype) {
  if (check_dims(dims, dtype) || check_shape(B, T, N)) return 0;
  return attention_ws_bytes(dims, B, T, N, dtype);
}

int krea2_gqa_attention(const Krea2Dims* dims, int B, int T, int N, int dtype, const void* qkvg,
                        const float* q_norm_w, const float* k_norm_w, const float* cos, const float* sin,
                        const uint8_t* text_mask, void* out, void* workspace, size_t ws_bytes, void* stream) {
  int rc = check_dims(dims, dtype);
  if (rc || (rc = check_shape(B, T, N))) return rc;
  if (!qkvg || !q_norm_w || !k_norm_w || !cos || !sin || !out) return set_error(KREA2_ERR_ARG, "NULL pointer");
  const size_t need = attention_ws_bytes(dims, B, T, N, dtype);
  if (need && (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255)))
    return set_error(KREA2_ERR_WORKSPACE, "workspace must be non-NULL and 256-byte aligned");
  if (ws_bytes < need) return set_error(KREA2_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, need);
  AttnParams ap{};
  ap.B = B; ap.T = T; ap.N = N; ap.S = T + N; ap.H = dims->H; ap.Hkv = dims->Hkv; ap.D = dims->D;
  ap.eps = dims->eps; ap.qkvg = qkvg; ap.q_norm_w = q_norm_w; ap.k_norm_w = k_norm_w; ap.cos = cos; ap.sin = sin;
  ap.text_mask = T > 0 ? text_mask : nullptr; ap.out = out;
  return attention_raw(ap, dtype, workspace, as_stream(stream));
}

int krea2_block_causal_key_end(const int32_t* image_ids, int S, int32_t* key_end) {
  if (!image_ids || !key_end || S <= 0) return set_error(KREA2_ERR_ARG, "NULL pointer or S <= 0");
  int end = 0;
  for (int q = S - 1; q >= 0; --q) {  // image ids run contiguously; walk back to know each block's end
    const int id = image_ids[q];
    if (id < 0) {
      key_end[q] = q + 1;
      continue;
    }
    if (q == S - 1 || image_ids[q + 1] != id) end = q + 1;
    key_end[q] = end;
  }
  for (int q = 0; q < S; ++q)  // a block id appearing in two separated runs is not a block
    if (image_ids[q] >= 0 && (q == 0 || image_ids[q - 1] != image_ids[q]))
      for (int k = key_end[q]; k < S; ++k)
        if (image_ids[k] == image_ids[q]) return set_error(KREA2_ERR_ARG, "image block %d is not contiguous", image_ids[q]);
  return KREA2_OK;
}

int krea2_gqa_attention_block_causal(const Krea2Dims* dims, int B, int T, int N, int dtype, const void* qkvg,
                                     const float* q_norm_w, const float* k_norm_w, const float* cos,
                                     const float* sin, const uint8_t* text_mask, const int32_t* key_end, void* out,
                                     void* workspace, size_t ws_bytes, void* stream) {
  int rc = check_dims(dims, dtype);
  if (rc) return rc;
  // every query reads at least its own position, so (unlike the plain entry) no image token is
  // needed; a query whose readable keys are all padded outputs zeros
  if (B <= 0 || T < 0 || N < 0 || (long long)T + N <= 0 || (long long)B * ((long long)T + N) > (1LL << 30))
    return set_error(KREA2_ERR_ARG, "need B >= 1, T + N >= 1 and B * (T + N) <= 2^30");
  if (!qkvg || !q_norm_w || !k_norm_w || !cos || !sin || !out || !key_end)
    return set_error(KREA2_ERR_ARG, "NULL pointer");
  if (dtype != KREA2_BF16 || !attention_tc_supported(dims->D, dims->H, dims->Hkv))
    return set_error(KREA2_ERR_UNSUPPORTED, "block-causal attention needs bf16, D=128, H/Hkv in {1,2,4}");
  const size_t need = attention_ws_bytes(dims, B, T, N, dtype);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return set_error(KREA2_ERR_WORKSPACE, "workspace must be non-NULL and 256-byte aligned");
  if (ws_bytes < need) return set_error(KREA2_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, need);
  AttnParams ap{};
  ap.B = B; ap.T = T; ap.N = N; ap.S = T + N; ap.H = dims->H; ap.Hkv = dims->Hkv; ap.D = dims->D;
  ap.eps = dims->eps; ap.qkvg = qkvg; ap.q_norm_w = q_norm_w; ap.k_norm_w = k_norm_w; ap.cos = cos; ap.sin = sin;
  ap.text_mask = T > 0 ? text_mask : nullptr; ap.out = out;
  return attention_raw(ap, dtype, workspace, as_stream(stream), key_end);
}

size_t krea2_kv_cache_attention_workspace_size(const Krea2Dims* dims, int B, int Nq, int dtype) {
  if (check_dims(dims, dtype) || B <= 0 || Nq <= 0 || dtype != KREA2_BF16 ||
      !attention_tc_supported(dims->D, dims->H, dims->Hkv))
    return 0;
  return (size_t)B * Nq * (size_t)dims->H * dims->D * 2;
}

int krea2_kv_cache_append(const Krea2Dims* dims, int B, int n, int row0, int capacity, int dtype, const void* qkvg,
                          const float* k_norm_w, const float* cos, const float* sin, void* k_cache, void* v_cache,
                          void* stream) {
  int rc = check_dims(dims, dtype);
  if (rc) return rc;
  if (B <= 0 || n <= 0 || row0 < 0 || capacity <= 0 || (long long)row0 + n > capacity)
    return set_error(KREA2_ERR_ARG, "need B >= 1, n >= 1 and 0 <= row0, row0 + n <= capacity (%d + %d > %d)", row0, n,
                     capacity);
  if (!qkvg || !k_norm_w || !cos || !sin || !k_cache || !v_cache) return set_error(KREA2_ERR_ARG, "NULL pointer");
  if (dtype != KREA2_BF16 || !attention_tc_supported(dims->D, dims->H, dims->Hkv))
    return set_error(KREA2_ERR_UNSUPPORTED, "the key/value cache needs bf16, D=128, H/Hkv in {1,2,4}");
  if ((reinterpret_cast<uintptr_t>(k_cache) | reinterpret_cast<uintptr_t>(v_cache)) & 15)
    return set_error(KREA2_ERR_ARG, "k_cache and v_cache must be 16-byte aligned");
  const long long QC = 2LL * dims->H * dims->D + 2LL * dims->Hkv * dims->D;
  return launch_kv_append(qkvg, QC, B, n, dims->H, dims->Hkv, dims->eps, k_norm_w, cos, sin, k_cache, v_cache, row0,
                          capacity, as_stream(stream));
}

int krea2_gqa_attention_kv_cache(const Krea2Dims* dims, int B, int T, int L, int Nq, int dtype, const void* qkvg,
                                 const float* q_norm_w, const float* cos, const float* sin, const uint8_t* text_mask,
                                 const void* k_cache, const void* v_cache, int capacity, const int32_t* key_end,
                                 void* out, void* workspace, size_t ws_bytes, void* stream) {
  int rc = check_dims(dims, dtype);
  if (rc) return rc;
  if (B <= 0 || T < 0 || Nq <= 0 || L < Nq || T > L || capacity < L)
    return set_error(KREA2_ERR_ARG, "need B >= 1, 1 <= Nq <= L, 0 <= T <= L and capacity >= L");
  if (!qkvg || !q_norm_w || !cos || !sin || !k_cache || !v_cache || !out)
    return set_error(KREA2_ERR_ARG, "NULL pointer");
  if (dtype != KREA2_BF16 || !attention_tc_supported(dims->D, dims->H, dims->Hkv))
    return set_error(KREA2_ERR_UNSUPPORTED, "the key/value cache needs bf16, D=128, H/Hkv in {1,2,4}");
  const size_t need = krea2_kv_cache_attention_workspace_size(dims, B, Nq, dtype);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return set_error(KREA2_ERR_WORKSPACE, "workspace must be non-NULL and 256-byte aligned");
  if (ws_bytes < need) return set_error(KREA2_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, need);
  const cudaStream_t s = as_stream(stream);
  const int H = dims->H, Hkv = dims->Hkv, D = dims->D;
  const long long QC = 2LL * H * D + 2LL * Hkv * D;
  // q of the new tokens only (Hkv = 0: no k heads in the prepared rows)
  if ((rc = launch_qk_prep(qkvg, QC, B, Nq, H, 0, dims->eps, q_norm_w, q_norm_w, cos, sin, workspace, s))) return rc;
  AttnTcArgs a{};
  a.B = B; a.T = T; a.N = L - T; a.H = H; a.Hkv = Hkv;
  a.q = workspace; a.q_stride = (long long)H * D;
  a.k = k_cache; a.k_stride = (long long)Hkv * D;
  a.v = v_cache; a.v_stride = (long long)Hkv * D;
  a.g = reinterpret_cast<const __nv_bfloat16*>(qkvg) + (long long)(H + 2 * Hkv) * D; a.g_stride = QC;
  a.text_mask = T > 0 ? text_mask : nullptr; a.out = out; a.key_end = key_end;
  a.Sq = Nq; a.q_off = L - Nq; a.kv_batch_rows = capacity;
  return attention_tc_core(a, s);
}

int krea2_modulated_rmsnorm(const Krea2Dims* dims, int B, int S, int dtype, const float* h, const float* norm_w,
                            const float* temb, const float* table, int chunk, void* out, void* stream) {
  int rc = check_dims(dims, dtype);
  if (rc) return rc;
  if (B <= 0 || S <= 0) return set_error(KREA2_ERR_ARG, "B and S must be positive");
  if (!h || !norm_w || !temb || !table || !out) return set_error(KREA2_ERR_ARG, "NULL pointer");
  if (chunk != 0 && chunk != 3) return set_error(KREA2_ERR_ARG, "chunk must be 0 (norm1) or 3 (norm2)");
  return launch_mod_rmsnorm(h, norm_w, temb, table, chunk, B, S, dims->C, dims->eps, out, dtype == KREA2_BF16,
                            as_stream(stream));
}

int krea2_linear(int dtype, int epilogue, int M, int Nw, int K, const void* A, const void* W, void* out,
                 const float* gate, int rows_per_batch, long long gate_stride, void* stream) {
  if (dtype != KREA2_BF16 && dtype != KREA2_F32) return set_error(KREA2_ERR_ARG, "unknown dtype %d", dtype);
  if (epilogue < EPI_STORE || epilogue > EPI_RESID) return set_error(KREA2_ERR_ARG, "unknown epilogue %d", epilogue);
  if (M <= 0 || Nw <= 0 || K <= 0) return set_error(KREA2_ERR_ARG, "sizes must be positive");
  if (!A || !W || !out) return set_error(KREA2_ERR_ARG, "NULL pointer");
  if (epilogue == EPI_RESID && (!gate || rows_per_batch <= 0 || gate_stride < 0))
    return set_error(KREA2_ERR_ARG, "residual epilogue needs gate, rows_per_batch > 0, gate_stride >= 0");
  if (epilogue == EPI_SWIGLU && Nw % 128) return set_error(KREA2_ERR_ARG, "SwiGLU needs Nw % 128 == 0");
  if (dtype == KREA2_BF16 && (Nw % 128 || K % 64))
    return set_error(KREA2_ERR_UNSUPPORTED, "bf16 linear needs Nw %% 128 == 0 and K %% 64 == 0");
  return linear_dispatch(dtype, epilogue, M, Nw, K, A, W, out, gate, rows_per_batch > 0 ? rows_per_batch : 1,
                         gate_stride, as_stream(stream));
}

int krea2_time_embed(const Krea2Dims* dims, int B, int dtype, const float* timestep, const Krea2ModelWeights* w,
                     float* temb_out, float* e_out, float* scratch, void* stream) {
  int rc = check_dims(dims, dtype);
  if (rc || (rc = check_model_dims(dims))) return rc;
  if (B <= 0) return set_error(KREA2_ERR_ARG, "batch must be positive");
  if (!timestep || !w || !w->t1_w || !w->t1_b || !w->t2_w || !w->t2_b || !w->mod_w || !w->mod_b || !temb_out ||
      !e_out || !scratch)
    return set_error(KREA2_ERR_ARG, "NULL pointer");
  return launch_time_embed(dims, B, dtype == KREA2_BF16, timestep, w, temb_out, e_out, scratch, as_stream(stream));
}

size_t krea2_final_layer_workspace_size(const Krea2Dims* dims, int B, int N, int dtype) {
  if (check_dims(dims, dtype) || check_model_dims(dims) || check_shape(B, 0, N)) return 0;
  return final_layer_tc_scratch(dims, B, N, dtype == KREA2_BF16);
}

int krea2_final_layer(const Krea2Dims* dims, int B, int T, int N, int dtype, const float* h, const float* e,
                      const Krea2ModelWeights* w, void* velocity, void* workspace, size_t ws_bytes, void* stream) {
  int rc = check_dims(dims, dtype);
  if (rc || (rc = check_model_dims(dims)) || (rc = check_shape(B, T, N))) return rc;
  if (!h || !e || !w || !w->final_norm_w || !w->final_table || !w->final_w || !w->final_b || !velocity)
    return set_error(KREA2_ERR_ARG, "NULL pointer");
  const size_t need = final_layer_tc_scratch(dims, B, N, dtype == KREA2_BF16);
  if (need && (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255)))
    return set_error(KREA2_ERR_WORKSPACE, "workspace must be non-NULL and 256-byte aligned");
  if (ws_bytes < need) return set_error(KREA2_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, need);
  return final_layer_impl(dims, B, T, N, dtype == KREA2_BF16, h, e, w, velocity, need ? workspace : nullptr,
                          as_stream(stream));
}

int krea2_block_forward(const Krea2Dims* dims, int B, int T, int N, int dtype, float* h, const float* temb,
                        const Krea2BlockWeights* w, const float* cos, const float* sin, const uint8_t* text_mask,
                        void* workspace, size_t ws_bytes, void* stream) {
  int rc = check_dims(dims, dtype);
  if (rc || (rc = check_shape(B, T, N)) || (rc = check_block_weights(w))) return rc;
  if (!h || !temb || !cos || !sin) return set_error(KREA2_ERR_ARG, "NULL pointer");
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return set_error(KREA2_ERR_WORKSPACE, "workspace must be non-NULL and 256-byte aligned");
  const Ws L = ws_layout(dims, B, T, N, dtype);
  if (ws_bytes < L.total)
    return set_error(KREA2_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, L.total);
  return block_impl(dims, B, T, N, dtype, h, temb, w, cos, sin, T > 0 ? text_mask : nullptr,
                    reinterpret_cast<uint8_t*>(workspace), L, as_stream(stream));
}

int krea2_block_forward_traced(const Krea2Dims* dims, int B, int T, int N, int dtype, float* h, const float* temb,
                               const Krea2BlockWeights* w, const float* cos, const float* sin,
                               const uint8_t* text_mask, void* workspace, size_t ws_bytes, void* const* events,
                               void* stream) {
  int rc = check_dims(dims, dtype);
  if (rc || (rc = check_shape(B, T, N)) || (rc = check_block_weights(w))) return rc;
  if (!h || !temb || !cos || !sin || !events) return set_error(KREA2_ERR_ARG, "NULL pointer");
  for (int i = 0; i < 9; ++i)
    if (!events[i]) return set_error(KREA2_ERR_ARG, "events[%d] is NULL", i);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return set_error(KREA2_ERR_WORKSPACE, "workspace must be non-NULL and 256-byte aligned");
  const Ws L = ws_layout(dims, B, T, N, dtype);
  if (ws_bytes < L.total)
    return set_error(KREA2_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, L.total);
  return block_impl(dims, B, T, N, dtype, h, temb, w, cos, sin, T > 0 ? text_mask : nullptr,
                    reinterpret_cast<uint8_t*>(workspace), L, as_stream(stream), events);
}

unsigned long long krea2_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

namespace {
Krea2Dims text_block_dims(const Krea2TextDims* td) {
  Krea2Dims d{};
  d.C = td->Dt; d.H = td->H; d.Hkv = td->Hkv; d.D = td->D; d.F = td->F;
  d.axes[0] = td->D / 4; d.axes[1] = 3 * td->D / 8; d.axes[2] = td->D - d.axes[0] - d.axes[1];
  d.theta = 1000.f; d.eps = td->eps; d.n_layers = 0; d.in_ch = 1; d.t_dim = 8;
  return d;
}

int check_text_dims(const Krea2TextDims* td, int dtype, int B, int T) {
  if (!td) return set_error(KREA2_ERR_ARG, "text dims is NULL");
  if (td->L <= 0 || td->n_layerwise < 0 || td->n_refiner < 0 || td->C <= 0 || td->C % 128)
    return set_error(KREA2_ERR_ARG, "bad text-fusion dims");
  if (B <= 0 || T <= 0) return set_error(KREA2_ERR_ARG, "need B >= 1 and T >= 1");
  const Krea2Dims d = text_block_dims(td);
  return check_dims(&d, dtype);
}

struct TextWs {
  size_t hl, hr, cs, sn, proj, block, total;
};
TextWs text_layout(const Krea2TextDims* td, int B, int T, int dtype) {
  const Krea2Dims d = text_block_dims(td);
  const size_t es = dtype == KREA2_BF16 ? 2 : 4;
  TextWs w{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off += up(bytes);
    return o;
  };
  const size_t rows_l = (size_t)B * T * td->L;
  w.hl = take(rows_l * td->Dt * 4);
  w.hr = take((size_t)B * T * td->Dt * 4);
  const size_t smax = (size_t)(T > td->L ? T : td->L);
  w.cs = take(smax * (td->D / 2) * 4);
  w.sn = take(smax * (td->D / 2) * 4);
  w.proj = take((size_t)B * T * td->Dt * es);
  const size_t b1 = ws_layout(&d, B * T, 0, td->L, dtype).total, b2 = ws_layout(&d, B, T, 0, dtype).total;
  w.block = take(b1 > b2 ? b1 : b2);
  w.total = off;
  return w;
}
}  // namespace

size_t krea2_text_fusion_workspace_size(const Krea2TextDims* td, int B, int T, int dtype) {
  if (check_text_dims(td, dtype, B, T)) return 0;
  return text_layout(td, B, T, dtype).total;
}

int krea2_text_fusion(const Krea2TextDims* td, int B, int T, int dtype, const void* ehs, const uint8_t* text_mask,
                      const Krea2TextWeights* w, void* text_out, void* workspace, size_t ws_bytes, void* stream) {
  int rc = check_text_dims(td, dtype, B, T);
  if (rc) return rc;
  if (!ehs || !w || !text_out || !w->layer_w || !w->txt_in_w || !w->txt_in_b ||
      (td->n_layerwise && !w->layerwise) || (td->n_refiner && !w->refiner))
    return set_error(KREA2_ERR_ARG, "NULL pointer");
  for (int i = 0; i < td->n_layerwise + td->n_refiner; ++i) {
    const Krea2BlockWeights* b = i < td->n_layerwise ? &w->layerwise[i] : &w->refiner[i - td->n_layerwise];
    if (!b->w_qkvg || !b->w_out || !b->w_gu || !b->w_down || !b->norm1_w || !b->norm2_w || !b->q_norm_w ||
        !b->k_norm_w)
      return set_error(KREA2_ERR_ARG, "text-fusion block %d: NULL pointer", i);
    if (b->scale_shift_table) return set_error(KREA2_ERR_ARG, "text-fusion blocks take no modulation table");
  }
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return set_error(KREA2_ERR_WORKSPACE, "workspace must be non-NULL and 256-byte aligned");
  const TextWs L = text_layout(td, B, T, dtype);
  if (ws_bytes < L.total) return set_error(KREA2_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, L.total);
  const Krea2Dims d = text_block_dims(td);
  const bool bf = dtype == KREA2_BF16;
  cudaStream_t s = as_stream(stream);
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  float* hl = reinterpret_cast<float*>(ws + L.hl);
  float* hr = reinterpret_cast<float*>(ws + L.hr);
  float* cs = reinterpret_cast<float*>(ws + L.cs);
  float* sn = reinterpret_cast<float*>(ws + L.sn);
  const int smax = T > td->L ? T : td->L;
  // no RoPE anywhere in text fusion: the zero-position (identity) rotation
  if ((rc = launch_identity_rope((long)smax * (td->D / 2), cs, sn, s))) return rc;
  // 1. layerwise: B*T sequences of L layer tokens, no mask
  const long rows_l = (long)B * T * td->L;
  if ((rc = launch_to_f32(ehs, bf, rows_l * td->Dt, hl, s))) return rc;
  const Ws bl = ws_layout(&d, B * T, 0, td->L, dtype);
  for (int i = 0; i < td->n_layerwise; ++i)
    if ((rc = block_impl(&d, B * T, 0, td->L, dtype, hl, nullptr, &w->layerwise[i], cs, sn, nullptr, ws + L.block,
                         bl, s)))
      return rc;
  // 2. Linear(L, 1) over the layer axis
  if ((rc = launch_layer_projection(hl, w->layer_w, (long)B * T, td->L, td->Dt, hr, false, s))) return rc;
  // 3. refiner over the token sequence with the text mask (T "text" keys, no image keys)
  const Ws br = ws_layout(&d, B, T, 0, dtype);
  for (int i = 0; i < td->n_refiner; ++i)
    if ((rc = block_impl(&d, B, T, 0, dtype, hr, nullptr, &w->refiner[i], cs, sn, text_mask, ws + L.block, br, s)))
      return rc;
  // 4. txt_in: Linear(Dt, C) + bias
  void* proj = ws + L.proj;
  if ((rc = launch_to_dtype(hr, (long)B * T * td->Dt, proj, bf, s))) return rc;
  if (bf) {
    GemmParams gp{};
    gp.M = B * T; gp.N = td->C; gp.K = td->Dt; gp.out = text_out; gp.bias = w->txt_in_b;
    return gemm_bf16(EPI_STORE, gp, proj, w->txt_in_w, s);
  }
  SimtGemmParams sp{};
  sp.M = B * T; sp.N = td->C; sp.K = td->Dt; sp.out = text_out; sp.bias = w->txt_in_b;
  return gemm_simt(SEPI_BIAS_F32, sp, proj, false, w->txt_in_w, false, s);
}

double krea2_shift_mu(int image_seq_len) {
  const double base_len = 256.0, max_len = 6400.0, base_shift = 0.5, max_shift = 1.15;
  return base_shift + (max_shift - base_shift) / (max_len - base_len) * ((double)image_seq_len - base_len);
}

int krea2_sigma_schedule(int n_steps, double mu, float* sigmas_out) {
  if (n_steps < 1 || !sigmas_out) return set_error(KREA2_ERR_ARG, "need n_steps >= 1 and an output array");
  const double em = exp(mu);
  for (int i = 0; i < n_steps; ++i) {
    // linspace(1, 1/n, n)
    const double s = n_steps == 1 ? 1.0 : 1.0 + (1.0 / n_steps - 1.0) * (double)i / (double)(n_steps - 1);
    sigmas_out[i] = (float)(em / (em + (1.0 / s - 1.0)));
  }
  sigmas_out[n_steps] = 0.f;
  return KREA2_OK;
}

int krea2_euler_cfg_step(int dtype, long long n, float* x, const void* v_cond, const void* v_uncond, float guidance,
                         float sigma, float sigma_next, void* x_model, int copies, float* timestep_out,
                         void* stream) {
  if (dtype != KREA2_BF16 && dtype != KREA2_F32) return set_error(KREA2_ERR_ARG, "unknown dtype %d", dtype);
  if (n < 0 || !x || !v_cond) return set_error(KREA2_ERR_ARG, "NULL pointer or negative size");
  if ((x_model || timestep_out) && (copies < 1 || copies > 32)) return set_error(KREA2_ERR_ARG, "copies must be 1..32");
  return launch_euler_cfg(dtype == KREA2_BF16, n, x, v_cond, guidance > 0.f ? v_uncond : nullptr, guidance, sigma,
                          sigma_next, x_model, copies, timestep_out, as_stream(stream));
}

namespace {
struct SampleWs {
  size_t backbone, backbone_bytes, xin, text, mask, t, vel, total;
};
SampleWs sample_layout(const Krea2Dims* d, int T, int N, int dtype, int cfg) {
  const int B = cfg ? 2 : 1;
  const size_t es = dtype == KREA2_BF16 ? 2 : 4;
  SampleWs w{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off += up(bytes);
    return o;
  };
  w.backbone_bytes = ws_layout(d, B, T, N, dtype).total;
  w.backbone = take(w.backbone_bytes);
  w.xin = take((size_t)B * N * d->in_ch * es);
  w.text = take((size_t)B * T * d->C * es + 16);
  w.mask = take((size_t)B * T + 16);
  w.t = take((size_t)B * 4);
  w.vel = take((size_t)B * N * d->in_ch * es);
  w.total = off;
  return w;
}
}  // namespace

size_t krea2_sample_workspace_size(const Krea2Dims* dims, int T, int N, int dtype, int cfg) {
  if (check_dims(dims, dtype) || check_model_dims(dims) || check_shape(1, T, N)) return 0;
  return sample_layout(dims, T, N, dtype, cfg).total;
}

int krea2_sample(const Krea2Dims* dims, int T, int N, int dtype, float* latents, const void* text_cond,
                 const void* text_uncond, const uint8_t* mask_cond, const uint8_t* mask_uncond,
                 const float* position_ids, const float* sigmas, int n_steps, float guidance,
                 const Krea2ModelWeights* w, void* workspace, size_t ws_bytes, void* stream) {
  int rc = check_dims(dims, dtype);
  if (rc || (rc = check_model_dims(dims)) || (rc = check_shape(1, T, N)) ||
      (rc = check_model_weights(w, dims->n_layers)))
    return rc;
  const bool cfg = guidance > 0.f;
  if (!latents || (T > 0 && !text_cond) || (cfg && T > 0 && !text_uncond) || !position_ids || !sigmas || n_steps < 1)
    return set_error(KREA2_ERR_ARG, "NULL pointer or n_steps < 1");
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return set_error(KREA2_ERR_WORKSPACE, "workspace must be non-NULL and 256-byte aligned");
  const SampleWs L = sample_layout(dims, T, N, dtype, cfg);
  if (ws_bytes < L.total) return set_error(KREA2_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, L.total);
  const int B = cfg ? 2 : 1;
  const bool bf = dtype == KREA2_BF16;
  const size_t es = bf ? 2 : 4;
  cudaStream_t s = as_stream(stream);
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  void* xin = ws + L.xin;
  void* text = ws + L.text;
  uint8_t* mask = ws + L.mask;
  float* tt = reinterpret_cast<float*>(ws + L.t);
  void* vel = ws + L.vel;
  const size_t text_bytes = (size_t)T * dims->C * es;
  // batch rows [cond, uncond]: text, masks (NULL = all valid)
  if (T > 0) {
    cudaError_t e = cudaMemcpyAsync(text, text_cond, text_bytes, cudaMemcpyDeviceToDevice, s);
    if (e == cudaSuccess && cfg)
      e = cudaMemcpyAsync(reinterpret_cast<uint8_t*>(text) + text_bytes, text_uncond, text_bytes,
                          cudaMemcpyDeviceToDevice, s);
    for (int r = 0; r < B && e == cudaSuccess; ++r) {
      const uint8_t* m = r == 0 ? mask_cond : mask_uncond;
      e = m ? cudaMemcpyAsync(mask + (size_t)r * T, m, T, cudaMemcpyDeviceToDevice, s)
            : cudaMemsetAsync(mask + (size_t)r * T, 1, T, s);
    }
    if (e != cudaSuccess) return set_error(KREA2_ERR_CUDA, "staging the text batch failed: %s", cudaGetErrorString(e));
  }
  const long long n = (long long)N * dims->in_ch;
  // first model input: x at sigmas[0]
  if ((rc = launch_euler_cfg(bf, n, latents, nullptr, nullptr, 0.f, sigmas[0], sigmas[0], xin, B, tt, s))) return rc;
  for (int i = 0; i < n_steps; ++i) {
    if ((rc = krea2_backbone_forward(dims, B, T, N, dtype, xin, text, position_ids, T > 0 ? mask : nullptr, tt, w, vel,
                                     ws + L.backbone, L.backbone_bytes, stream)))
      return rc;
    const void* vu = cfg ? reinterpret_cast<uint8_t*>(vel) + (size_t)n * es : nullptr;
    if ((rc = launch_euler_cfg(bf, n, latents, vel, vu, guidance, sigmas[i], sigmas[i + 1], xin, B, tt, s))) return rc;
  }
  return KREA2_OK;
}

int krea2_backbone_forward(const Krea2Dims* dims, int B, int T, int N, int dtype, const void* hidden_states,
                           const void* text_states, const float* position_ids, const uint8_t* text_mask,
                           const float* timestep, const Krea2ModelWeights* w, void* velocity, void* workspace,
                           size_t ws_bytes, void* stream) {
  int rc = check_dims(dims, dtype);
  if (rc || (rc = check_model_dims(dims)) || (rc = check_shape(B, T, N)) ||
      (rc = check_model_weights(w, dims->n_layers)))
    return rc;
  if (!hidden_states || (T > 0 && !text_states) || !position_ids || !timestep || !velocity)
    return set_error(KREA2_ERR_ARG, "NULL pointer");
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return set_error(KREA2_ERR_WORKSPACE, "workspace must be non-NULL and 256-byte aligned");
  const Ws L = ws_layout(dims, B, T, N, dtype);
  if (ws_bytes < L.total)
    return set_error(KREA2_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, L.total);
  cudaStream_t s = as_stream(stream);
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  const bool bf = dtype == KREA2_BF16;
  const int S = T + N, C = dims->C;
  float* h = reinterpret_cast<float*>(ws + L.h);
  float* cs = reinterpret_cast<float*>(ws + L.cs);
  float* sn = reinterpret_cast<float*>(ws + L.sn);
  float* temb = reinterpret_cast<float*>(ws + L.temb);
  float* e = reinterpret_cast<float*>(ws + L.e);
  if ((rc = launch_rope_tables(position_ids, S, dims->axes[0], dims->axes[1], dims->axes[2], dims->theta, cs, sn, s)))
    return rc;
  if ((rc = launch_time_embed(dims, B, bf, timestep, w, temb, e, reinterpret_cast<float*>(ws + L.tscr), s))) return rc;
  if ((rc = launch_copy_text_rows(text_states, bf, B, T, S, C, h, s))) return rc;
  if ((rc = img_in_impl(dims, B, T, N, bf, hidden_states, w, h, s))) return rc;
  const uint8_t* mask = T > 0 ? text_mask : nullptr;
  for (int l = 0; l < dims->n_layers; ++l)
    if ((rc = block_impl(dims, B, T, N, dtype, h, temb, &w->blocks[l], cs, sn, mask, ws, L, s))) return rc;
  // the block activations are dead now: their bf16 xn buffer (B*S*C) holds the final norm's output
  return final_layer_impl(dims, B, T, N, bf, h, e, w, velocity, ws + L.xn, s);
}

}  // extern "C"
