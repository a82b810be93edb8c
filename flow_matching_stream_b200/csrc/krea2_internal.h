// Internal declarations shared by the library's translation units (not part of the ABI).
#pragma once
#include <atomic>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/krea2.h"

namespace krea2 {

// EPI_BIAS_ROWMAP: fp32 out[map(row), col] = acc + bias[col], map(r) = (r / map_N) * map_S + map_T + r % map_N
// (img_in writing the image rows of the residual after the text rows).
enum { EPI_STORE = KREA2_EPI_STORE, EPI_SWIGLU = KREA2_EPI_SWIGLU, EPI_RESID = KREA2_EPI_RESID, EPI_QKV = 3,
       EPI_BIAS_ROWMAP = 4 };

// Records a message for krea2_last_error_string() and returns `code`.
int set_error(int code, const char* fmt, ...);
// Kernel attributes (the dynamic shared-memory opt-in) hold per device. Launchers keep one
// bit per device ordinal to set them once per device; 0 (ordinals >= 64) means set every time.
inline uint64_t device_bit() {
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= 64) return 0;
  return 1ull << d;
}
int num_sms();
// Counts kernel launches (krea2_launch_count); every launcher calls it once per launch.
void count_launch();
// Read and clear the device error word of the GEMM / attention files (0 = none, -1 = read failed).
int take_device_error_gemm();
int take_device_error_attention();

struct GemmParams {
  int M, N, K;              // N = rows of W
  void* out;                // STORE/SWIGLU: bf16 (M, N) / (M, N/2); RESID: fp32 (M, N)
  const float* bias;        // STORE: optional per-column bias (N)
  const float* gate;        // RESID: gate[(row / rows_per_batch) * gate_stride + col]
  int rows_per_batch;       // RESID: batch of a row; QKV: sequence length S (position = row % S)
  long long gate_stride;
  // QKV: columns [q heads (HD) | k heads (KVD) | v | gate]; q/k heads (128 wide) are
  // RMS-normalised with (1 + qw / kw) and rotated with the RoPE tables of the row's position.
  const float* qw;
  const float* kw;
  const float* cos;
  const float* sin;
  int HD, KVD;
  float eps;
  int out_ld;               // STORE: row stride of out in elements (0: N)
  int n_store;              // STORE: columns stored, a multiple of 64 (0: N)
  int w_rows;               // rows of W present (0: N); rows beyond read as zeros
  int map_N, map_T, map_S;  // BIAS_ROWMAP row map
  int tiles_m, tiles_n;     // filled by the launcher
  int group_m;              // row tiles per raster group (filled by the launcher)
};

// tcgen05 bf16 GEMM (gemm_tcgen05.cu). Requires N % 128 == 0, K % 64 == 0.
int gemm_bf16(int epi, const GemmParams& p, const void* A, const void* W, cudaStream_t stream);

// SIMT fp32-accumulate GEMM for the fp32 path and the small projections (simt.cu).
// A (M, K) of type a_bf16 ? bf16 : f32; W (N, K) of type w_bf16 ? bf16 : f32.
enum { SEPI_STORE_F32 = 0, SEPI_STORE_BF16 = 1, SEPI_SWIGLU_F32 = 2, SEPI_RESID = 3, SEPI_BIAS_ROWMAP = 4,
       SEPI_BIAS_F32 = 5, SEPI_BIAS_BF16 = 6 };
struct SimtGemmParams {
  int M, N, K;
  void* out;
  const float* bias;        // BIAS_* : (N)
  const float* gate;        // RESID
  int rows_per_batch;
  long long gate_stride;
  int map_N, map_T, map_S;  // BIAS_ROWMAP: input row r = b*map_N + n -> output row b*map_S + map_T + n
};
int gemm_simt(int epi, const SimtGemmParams& p, const void* A, bool a_bf16, const void* W, bool w_bf16,
              cudaStream_t stream);

// Element-wise / row kernels (simt.cu).
int launch_rope_tables(const float* pos, int S, int a0, int a1, int a2, float theta, float* cos_out, float* sin_out,
                       cudaStream_t stream);
int launch_modulation(const float* temb, const float* table, int B, int C, float* mod, cudaStream_t stream);
// out = (1 + (temb+table)[b, chunk]) * rms(h) * (1 + w) + (temb+table)[b, chunk+1]; table may be null
// (then temb already holds temb+table).
int launch_mod_rmsnorm(const float* h, const float* w, const float* temb, const float* table, int chunk, int B, int S,
                       int C, float eps, void* out, bool out_bf16, cudaStream_t stream);
// General form: output row r (of B * rows) reads h row (r / rows) * S_in + row0 + r % rows;
// scale = sc[b * mod_stride + c] (+ sc_tab[c]), shift = sh[b * mod_stride + c] (+ sh_tab[c]).
struct ModNormArgs {
  const float* h;
  const float* w;
  const float* sc;
  const float* sh;
  long long mod_stride;
  const float* sc_tab;  // nullable
  const float* sh_tab;  // nullable
  int B, rows, S_in, row0, C;
  float eps;
  void* out;
  bool out_bf16;
};
int launch_mod_rmsnorm_rows(const ModNormArgs& a, cudaStream_t stream);
int launch_time_embed(const Krea2Dims* d, int B, bool w_bf16, const float* t, const Krea2ModelWeights* w,
                      float* temb, float* e, float* scratch, cudaStream_t stream);
int launch_final_layer(const Krea2Dims* d, int B, int T, int N, bool bf16, const float* h, const float* e,
                       const Krea2ModelWeights* w, void* velocity, cudaStream_t stream);
// Bytes of bf16 scratch the tensor-core final layer needs (0 when it does not apply).
size_t final_layer_tc_scratch(const Krea2Dims* d, int B, int N, bool bf16);
int launch_euler_cfg(bool bf16, long long n, float* x, const void* vc, const void* vu, float g, float sigma,
                     float sigma_next, void* xm, int copies, float* t_out, cudaStream_t stream);
int launch_unit_modulation(int B, int C, float* mod, cudaStream_t stream);
int launch_identity_rope(long n, float* cs, float* sn, cudaStream_t stream);
int launch_layer_projection(const float* x, const float* w, long rows, int L, int C, void* out, bool out_bf16,
                            cudaStream_t stream);
int launch_to_f32(const void* in, bool in_bf16, long n, float* out, cudaStream_t stream);
int launch_to_dtype(const float* in, long n, void* out, bool out_bf16, cudaStream_t stream);
int launch_copy_text_rows(const void* text, bool bf16, int B, int T, int S, int C, float* h, cudaStream_t stream);

// Attention (attention_*.cu).
struct AttnParams {
  int B, T, N, S, H, Hkv, D;
  float eps;
  const void* qkvg;          // (B*S, 2*H*D + 2*Hkv*D)
  const float* q_norm_w;
  const float* k_norm_w;
  const float* cos;          // (S, D/2)
  const float* sin;
  const uint8_t* text_mask;  // (B, T) or null
  void* out;                 // (B*S, H*D)
};
int attention_simt(const AttnParams& p, bool bf16, cudaStream_t stream);

// tcgen05 flash attention core (attention_tc.cu): q/k already normalised and rotated.
struct AttnTcArgs {
  int B, T, N, H, Hkv;
  const void* q; long long q_stride;   // bf16, row stride in elements
  const void* k; long long k_stride;
  const void* v; long long v_stride;
  const void* g; long long g_stride;
  const uint8_t* text_mask;
  void* out;                           // (B*S, H*128) bf16
  const int* key_end;                  // optional (Sq): query row q reads keys [0, key_end[q]) (block-causal)
  int Sq;                              // query rows per batch row; 0 means S = T + N
  int q_off;                           // key position of query row 0 (queries are keys [q_off, q_off + Sq))
  long long kv_batch_rows;             // rows between batch rows of k and v; 0 means S
};
bool attention_tc_supported(int D, int H, int Hkv);
int launch_wait_timeout_selftest(unsigned long long limit_ns, int* waited, cudaStream_t stream);
int attention_tc_core(const AttnTcArgs& a, cudaStream_t stream);
// raw k and v of n tokens -> rows [row0, row0 + n) of every batch row of a key/value cache
// (k RMS-normalised and rotated, v copied; bf16, (B, capacity, Hkv*128))
int launch_kv_append(const void* qkvg, long long stride, int B, int n, int H, int Hkv, float eps, const float* kw,
                     const float* cs, const float* sn, void* k_cache, void* v_cache, int row0, int capacity,
                     cudaStream_t stream);
// raw [q | k] -> normalised + rotated [q | k] (bf16, row stride (H+Hkv)*128)
int launch_qk_prep(const void* qkvg, long long stride, int B, int S, int H, int Hkv, float eps, const float* qw,
                   const float* kw, const float* cs, const float* sn, void* dst, cudaStream_t stream);

}  // namespace krea2
