// CUDA-core kernels of the Krea 2 path: RoPE tables, modulation, modulated RMSNorm, the time
// path, the final layer, text-row placement, a SIMT GEMM (fp32 path and the small
// projections img_in / final) and a SIMT attention (fp32 reference-precision path).
//
// Sources (page "Diffusers 中的 Krea2Transformer2DModel … 架构全解" = [ARCH],
// page "Krea2Transformer2DModel" API docs = [API]):
//   RoPE          [API] axes_dims_rope / rope_theta; [ARCH] §一 (FluxPosEmbed lineage)
//   RMSNorm       [ARCH] §四.4 (multiplier 1 + w, fp32), eps from [API] norm_eps
//   modulation    [ARCH] §四.2 (temb + scale_shift_table, unbind into six chunks)
//   time path     [ARCH] §四 data flow, §四.5 (cos-first sinusoid of 1000 t, GELU-tanh MLP)
//   final layer   [ARCH] §四.6 ((2, C) scale/shift table, Linear to in_channels)
//   attention     [ARCH] §四.3 (q/k RMSNorm per head, RoPE, GQA, sigmoid output gate)
#include <math.h>

#include "krea2_device.cuh"
#include "krea2_internal.h"

namespace krea2 {

namespace {

// ----------------------------------------------------------------------------- RoPE tables
__global__ void rope_tables_kernel(const float* __restrict__ pos, int S, int a0, int a1, int a2, double theta,
                                   float* __restrict__ cos_out, float* __restrict__ sin_out) {
  const int half = (a0 + a1 + a2) / 2;
  const long idx = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long)S * half) return;
  const int s = (int)(idx / half);
  const int p = (int)(idx % half);
  int axis, j, d;
  if (p < a0 / 2) {
    axis = 0; j = p; d = a0;
  } else if (p < (a0 + a1) / 2) {
    axis = 1; j = p - a0 / 2; d = a1;
  } else {
    axis = 2; j = p - (a0 + a1) / 2; d = a2;
  }
  const double inv_freq = pow(theta, -2.0 * (double)j / (double)d);
  const double ang = (double)pos[(long)s * 3 + axis] * inv_freq;
  double sn, cs;
  sincos(ang, &sn, &cs);
  cos_out[idx] = (float)cs;
  sin_out[idx] = (float)sn;
}

// ----------------------------------------------------------------------------- modulation
__global__ void modulation_kernel(const float* __restrict__ temb, const float* __restrict__ table, int B, int C,
                                  float* __restrict__ mod) {
  const long n = (long)B * 6 * C;
  for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x)
    mod[i] = temb[i] + table[i % (6L * C)];
}

// Unit modulation (scale 0, shift 0, gate 1 for both halves): blocks without time modulation.
__global__ void unit_modulation_kernel(int B, int C, float* __restrict__ mod) {
  const long n = (long)B * 6 * C;
  for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x) {
    const int chunk = (int)((i / C) % 6);
    mod[i] = (chunk == 2 || chunk == 5) ? 1.f : 0.f;
  }
}

// RoPE tables of the zero position: cos 1, sin 0 (the identity rotation).
__global__ void identity_rope_kernel(long n, float* __restrict__ cs, float* __restrict__ sn) {
  for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x) {
    cs[i] = 1.f;
    sn[i] = 0.f;
  }
}

// out[n, c] = sum_l w[l] * x[n*L + l, c]   (Linear(L, 1, bias=False) over the layer axis)
template <bool OUT_BF16>
__global__ void layer_projection_kernel(const float* __restrict__ x, const float* __restrict__ w, long rows, int L,
                                        int C, void* __restrict__ out) {
  const long total = rows * C;
  for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (long)gridDim.x * blockDim.x) {
    const long r = i / C;
    const int c = (int)(i % C);
    float acc = 0.f;
    for (int l = 0; l < L; ++l) acc += w[l] * x[(r * L + l) * C + c];
    if (OUT_BF16) reinterpret_cast<__nv_bfloat16*>(out)[i] = __float2bfloat16_rn(acc);
    else reinterpret_cast<float*>(out)[i] = acc;
  }
}

// fp32 copy of an activation tensor in `dtype`
template <bool IN_BF16>
__global__ void to_f32_kernel(const void* __restrict__ in, long n, float* __restrict__ out) {
  for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x)
    out[i] = IN_BF16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(in)[i])
                     : reinterpret_cast<const float*>(in)[i];
}

template <bool OUT_BF16>
__global__ void from_f32_kernel(const float* __restrict__ in, long n, void* __restrict__ out) {
  for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x) {
    if (OUT_BF16) reinterpret_cast<__nv_bfloat16*>(out)[i] = __float2bfloat16_rn(in[i]);
    else reinterpret_cast<float*>(out)[i] = in[i];
  }
}

// ----------------------------------------------------------------------------- modulated RMSNorm
// One CTA per output row; C % 4 == 0; 256 threads, float4 loads of the fp32 residual. NV float4
// per thread hold the row between the two passes: NV = C / 1024 rounded up (6 for C = 6144), so
// that no registers are reserved for columns the row does not have.
// Output row r reads residual row (r / rows) * S_in + row0 + r % rows (the identity for the block
// norms; the image rows for the final layer) and batch b = r / rows picks the modulation vectors.
// Rows in flight set the bandwidth of this one-pass-over-HBM kernel: the launch bounds keep the
// registers low enough for 6, 5 or 4 resident CTAs per SM as NV grows (NV = 5, 6 spill 16 bytes).
template <bool OUT_BF16, int NV>
__global__ void __launch_bounds__(256, NV <= 4 ? 6 : NV <= 6 ? 5 : 4) mod_rmsnorm_kernel(ModNormArgs a) {
  const long row = blockIdx.x;
  const int C = a.C;
  const int b = (int)(row / a.rows);
  const long in_row = (long)b * a.S_in + a.row0 + row % a.rows;
  const int C4 = C >> 2;
  const float4* x4 = reinterpret_cast<const float4*>(a.h + in_row * C);
  constexpr int MAXV = NV;
  float4 xv[MAXV];
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int c4 = threadIdx.x + i * 256;
    if (c4 < C4) {
      xv[i] = x4[c4];
      ss += xv[i].x * xv[i].x + xv[i].y * xv[i].y + xv[i].z * xv[i].z + xv[i].w * xv[i].w;
    }
  }
  __shared__ float red[8];
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) tot += red[i];
  const float r = rsqrtf(tot / (float)C + a.eps);
  const float* sc_t = a.sc + (long)b * a.mod_stride;
  const float* sh_t = a.sh + (long)b * a.mod_stride;
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int c4 = threadIdx.x + i * 256;
    if (c4 < C4) {
      const int c = c4 * 4;
      float4 ww = __ldg(reinterpret_cast<const float4*>(a.w + c));
      float4 sc = __ldg(reinterpret_cast<const float4*>(sc_t + c));
      float4 sh = __ldg(reinterpret_cast<const float4*>(sh_t + c));
      if (a.sc_tab) {
        const float4 t0 = __ldg(reinterpret_cast<const float4*>(a.sc_tab + c));
        const float4 t1 = __ldg(reinterpret_cast<const float4*>(a.sh_tab + c));
        sc.x += t0.x; sc.y += t0.y; sc.z += t0.z; sc.w += t0.w;
        sh.x += t1.x; sh.y += t1.y; sh.z += t1.z; sh.w += t1.w;
      }
      float y0 = (1.f + sc.x) * (xv[i].x * r * (1.f + ww.x)) + sh.x;
      float y1 = (1.f + sc.y) * (xv[i].y * r * (1.f + ww.y)) + sh.y;
      float y2 = (1.f + sc.z) * (xv[i].z * r * (1.f + ww.z)) + sh.z;
      float y3 = (1.f + sc.w) * (xv[i].w * r * (1.f + ww.w)) + sh.w;
      if (OUT_BF16) {
        uint2 o;
        o.x = pack_bf16x2(y0, y1);
        o.y = pack_bf16x2(y2, y3);
        reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(a.out) + row * C)[c4] = o;
      } else {
        reinterpret_cast<float4*>(reinterpret_cast<float*>(a.out) + row * C)[c4] = make_float4(y0, y1, y2, y3);
      }
    }
  }
}

// ----------------------------------------------------------------------------- time path
__global__ void timestep_sinusoid_kernel(const float* __restrict__ t, int B, int dim, float* __restrict__ out) {
  const int half = dim / 2;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= B * half) return;
  const int b = i / half, k = i % half;
  const double f = exp(-log(10000.0) * (double)k / (double)half);
  const double a = 1000.0 * (double)t[b] * f;
  double sn, cs;
  sincos(a, &sn, &cs);
  out[(long)b * dim + k] = (float)cs;          // cosine half first
  out[(long)b * dim + half + k] = (float)sn;
}

__device__ __forceinline__ float gelu_tanh_f(float x) {
  const float k0 = 0.7978845608028654f;  // sqrt(2/pi)
  return 0.5f * x * (1.f + tanhf(k0 * (x + 0.044715f * x * x * x)));
}

// out[b, n] = act(sum_k x[b, k] W[n, k] + bias[n]); one warp per output feature, all batch rows.
// MAXB accumulators per lane, sized to the batch (1, 2, 4 or 8 at a time), so that with the
// model's batch of one or two the K loop can keep four 16-byte weight loads in flight per lane:
// the weights stream from HBM once and this is a bandwidth-bound GEMV.
template <bool W_BF16, bool GELU, int MAXB>
__global__ void __launch_bounds__(256) small_m_linear_kernel(const float* __restrict__ x, const void* __restrict__ W,
                                                             const float* __restrict__ bias, int B, int N, int K,
                                                             float* __restrict__ out) {
  const int n = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (n >= N) return;
  for (int b0 = 0; b0 < B; b0 += MAXB) {
    float acc[MAXB];
#pragma unroll
    for (int b = 0; b < MAXB; ++b) acc[b] = 0.f;
#pragma unroll 4
    for (int k = lane * 8; k < K; k += 256) {
      float wv[8];
      if (W_BF16) {
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(W) +
                                                             (long)n * K + k));
        wv[0] = bf16_lo(u.x); wv[1] = bf16_hi(u.x); wv[2] = bf16_lo(u.y); wv[3] = bf16_hi(u.y);
        wv[4] = bf16_lo(u.z); wv[5] = bf16_hi(u.z); wv[6] = bf16_lo(u.w); wv[7] = bf16_hi(u.w);
      } else {
        const float4* wp = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(W) + (long)n * K + k);
        const float4 a = __ldg(wp), c = __ldg(wp + 1);
        wv[0] = a.x; wv[1] = a.y; wv[2] = a.z; wv[3] = a.w; wv[4] = c.x; wv[5] = c.y; wv[6] = c.z; wv[7] = c.w;
      }
#pragma unroll
      for (int b = 0; b < MAXB; ++b) {
        if (b0 + b < B) {
          const float4* xp = reinterpret_cast<const float4*>(x + (long)(b0 + b) * K + k);
          const float4 a = __ldg(xp), c = __ldg(xp + 1);
          acc[b] += a.x * wv[0] + a.y * wv[1] + a.z * wv[2] + a.w * wv[3] + c.x * wv[4] + c.y * wv[5] +
                    c.z * wv[6] + c.w * wv[7];
        }
      }
    }
#pragma unroll
    for (int b = 0; b < MAXB; ++b) {
      const float v = warp_sum(acc[b]);
      if (lane == 0 && b0 + b < B) {
        float y = v + (bias ? bias[n] : 0.f);
        out[(long)(b0 + b) * N + n] = GELU ? gelu_tanh_f(y) : y;
      }
    }
  }
}

// ----------------------------------------------------------------------------- final layer
// velocity[b*N + n] = ((1 + table[0] + e[b]) * rms(h[b*S + T + n]) * (1 + w) + table[1] + e[b]) . Wfᵀ + bias
// One CTA per FL_ROWS image rows: the row statistics first, then K-chunks of the modulated rows
// and of Wf staged in shared memory; each thread accumulates FL_ROWS*OUT/256 outputs.
constexpr int FL_ROWS = 16, FL_KC = 128, FL_MAX_OUT = 64;

template <bool BF16>
__global__ void __launch_bounds__(256) final_layer_kernel(const float* __restrict__ h, const float* __restrict__ e,
                                                          const float* __restrict__ w, const float* __restrict__ table,
                                                          const void* __restrict__ Wf, const float* __restrict__ bias,
                                                          int B, int T, int N, int C, int OUT, float eps,
                                                          void* __restrict__ velocity) {
  __shared__ float xs[FL_ROWS][FL_KC + 1];
  __shared__ float ws[FL_MAX_OUT][FL_KC + 1];
  __shared__ float rr[FL_ROWS];
  const int S = T + N;
  const long r0 = (long)blockIdx.x * FL_ROWS;
  const long rows = (long)B * N;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // row statistics: 8 warps x 2 rows
  for (int i = warp; i < FL_ROWS; i += 8) {
    const long r = r0 + i;
    float ss = 0.f;
    if (r < rows) {
      const float* x = h + ((r / N) * S + T + (r % N)) * (long)C;
      for (int c = lane; c < C; c += 32) ss += x[c] * x[c];
    }
    ss = warp_sum(ss);
    if (lane == 0) rr[i] = rsqrtf(ss / (float)C + eps);
  }
  // each thread: row tr, outputs to .. to + OPT-1
  constexpr int THREADS_PER_ROW = 256 / FL_ROWS;  // 16
  const int tr = threadIdx.x / THREADS_PER_ROW;
  const int opt = (OUT + THREADS_PER_ROW - 1) / THREADS_PER_ROW;  // <= 4
  const int to = (threadIdx.x % THREADS_PER_ROW) * opt;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  __syncthreads();
  for (int k0 = 0; k0 < C; k0 += FL_KC) {
    for (int i = threadIdx.x; i < FL_ROWS * FL_KC; i += 256) {
      const int rl = i / FL_KC, k = i % FL_KC;
      const long r = r0 + rl;
      const int c = k0 + k;
      float y = 0.f;
      if (r < rows && c < C) {
        const long b = r / N;
        const float x = h[(b * S + T + (r % N)) * (long)C + c];
        const float sc = table[c] + e[b * C + c], sh = table[C + c] + e[b * C + c];
        y = (1.f + sc) * (x * rr[rl] * (1.f + w[c])) + sh;
      }
      xs[rl][k] = y;
    }
    for (int i = threadIdx.x; i < OUT * FL_KC; i += 256) {
      const int o = i / FL_KC, k = i % FL_KC;
      const int c = k0 + k;
      float v = 0.f;
      if (c < C) {
        v = BF16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(Wf)[(long)o * C + c])
                 : reinterpret_cast<const float*>(Wf)[(long)o * C + c];
      }
      ws[o][k] = v;
    }
    __syncthreads();
#pragma unroll 4
    for (int k = 0; k < FL_KC; ++k) {
      const float a = xs[tr][k];
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (q < opt && to + q < OUT) acc[q] += a * ws[to + q][k];
    }
    __syncthreads();
  }
  const long r = r0 + tr;
  if (r < rows) {
    for (int q = 0; q < opt; ++q) {
      const int o = to + q;
      if (o >= OUT) break;
      const float v = acc[q] + bias[o];
      if (BF16) reinterpret_cast<__nv_bfloat16*>(velocity)[r * OUT + o] = __float2bfloat16_rn(v);
      else reinterpret_cast<float*>(velocity)[r * OUT + o] = v;
    }
  }
}

template <bool IN_BF16>
__global__ void copy_text_rows_kernel(const void* __restrict__ text, int T, int S, int C, long total,
                                      float* __restrict__ h) {
  for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (long)gridDim.x * blockDim.x) {
    const long bt = i / C;
    const int c = (int)(i % C);
    const long b = bt / T, t = bt % T;
    float v = IN_BF16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(text)[i])
                      : reinterpret_cast<const float*>(text)[i];
    h[(b * S + t) * C + c] = v;
  }
}

// ----------------------------------------------------------------------------- SIMT GEMM
// out = A · Wᵀ, 64x128 output tile per CTA, K step 16, 256 threads, 4x(4+4) outputs each.
constexpr int SBM = 64, SBN = 128, SBK = 16;

template <bool A_BF16>
__device__ __forceinline__ float load_elem(const void* p, long i) {
  if (A_BF16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i]);
  return reinterpret_cast<const float*>(p)[i];
}

template <bool A_BF16, bool W_BF16, int EPI>
__global__ void __launch_bounds__(256) simt_gemm_kernel(const void* __restrict__ A, const void* __restrict__ W,
                                                        SimtGemmParams p) {
  __shared__ float As[SBK][SBM + 4];
  __shared__ float Ws[SBK][SBN + 4];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int m0 = blockIdx.y * SBM, n0 = blockIdx.x * SBN;
  float acc[4][8];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

  for (int k0 = 0; k0 < p.K; k0 += SBK) {
    for (int i = threadIdx.x; i < SBM * SBK; i += 256) {
      const int r = i / SBK, k = i % SBK;
      const int gr = m0 + r, gk = k0 + k;
      As[k][r] = (gr < p.M && gk < p.K) ? load_elem<A_BF16>(A, (long)gr * p.K + gk) : 0.f;
    }
    for (int i = threadIdx.x; i < SBN * SBK; i += 256) {
      const int r = i / SBK, k = i % SBK;
      const int gr = n0 + r, gk = k0 + k;
      Ws[k][r] = (gr < p.N && gk < p.K) ? load_elem<W_BF16>(W, (long)gr * p.K + gk) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < SBK; ++k) {
      float a[4], w[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[k][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        w[j] = Ws[k][tx * 4 + j];
        w[4 + j] = Ws[k][64 + tx * 4 + j];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] += a[i] * w[j];
    }
    __syncthreads();
  }

#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = m0 + ty * 4 + i;
    if (r >= p.M) continue;
    if (EPI == SEPI_SWIGLU_F32) {
      // tile = one interleaved 64-row group pair: columns [0,64) gate, [64,128) up
      const int g = blockIdx.x;
      float* o = reinterpret_cast<float*>(p.out) + (long)r * (p.N / 2) + g * 64;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float gv = acc[i][j], uv = acc[i][4 + j];
        o[tx * 4 + j] = gv / (1.f + expf(-gv)) * uv;
      }
      continue;
    }
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) {
      const int c = n0 + (jj < 4 ? tx * 4 + jj : 64 + tx * 4 + (jj - 4));
      if (c >= p.N) continue;
      const float v = acc[i][jj];
      if (EPI == SEPI_STORE_F32) {
        reinterpret_cast<float*>(p.out)[(long)r * p.N + c] = v;
      } else if (EPI == SEPI_STORE_BF16) {
        reinterpret_cast<__nv_bfloat16*>(p.out)[(long)r * p.N + c] = __float2bfloat16_rn(v);
      } else if (EPI == SEPI_RESID) {
        const int b = r / p.rows_per_batch;
        float* hp = reinterpret_cast<float*>(p.out) + (long)r * p.N + c;
        *hp += p.gate[(long)b * p.gate_stride + c] * v;
      } else if (EPI == SEPI_BIAS_ROWMAP) {
        const int b = r / p.map_N, n = r % p.map_N;
        reinterpret_cast<float*>(p.out)[((long)b * p.map_S + p.map_T + n) * p.N + c] = v + p.bias[c];
      } else if (EPI == SEPI_BIAS_F32) {
        reinterpret_cast<float*>(p.out)[(long)r * p.N + c] = v + p.bias[c];
      } else {  // SEPI_BIAS_BF16
        reinterpret_cast<__nv_bfloat16*>(p.out)[(long)r * p.N + c] = __float2bfloat16_rn(v + p.bias[c]);
      }
    }
  }
}

// ----------------------------------------------------------------------------- SIMT attention
// One warp per (row, query head); lane owns DPL = D/32 consecutive dims (whole RoPE pairs).
// Keys are streamed one at a time with an online softmax; k is normalised and rotated on load.
template <typename T>
__device__ __forceinline__ float ld_act(const T* p, long i) {
  if constexpr (sizeof(T) == 2) return __bfloat162float(p[i]);
  else return p[i];
}

template <typename T, int DPL>
__global__ void __launch_bounds__(256) attn_simt_kernel(AttnParams p) {
  const long gw = (long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const long total = (long)p.B * p.S * p.H;
  if (gw >= total) return;
  const int h = (int)(gw % p.H);
  const long row = gw / p.H;
  const int b = (int)(row / p.S);
  const int s = (int)(row % p.S);
  const int D = p.D, HD = p.H * p.D, KVD = p.Hkv * p.D;
  const long QC = 2L * HD + 2L * KVD;
  const int kvh = h / (p.H / p.Hkv);
  const int d0 = lane * DPL;
  const int halfD = D / 2;
  const T* X = reinterpret_cast<const T*>(p.qkvg);

  float q[DPL], o[DPL];
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < DPL; ++i) {
    q[i] = ld_act(X, row * QC + (long)h * D + d0 + i);
    ss += q[i] * q[i];
  }
  float r = rsqrtf(warp_sum(ss) / (float)D + p.eps);
#pragma unroll
  for (int i = 0; i < DPL; ++i) q[i] *= r * (1.f + p.q_norm_w[d0 + i]);
#pragma unroll
  for (int i = 0; i < DPL; i += 2) {
    const int pr = (d0 + i) / 2;
    const float c = p.cos[(long)s * halfD + pr], sn = p.sin[(long)s * halfD + pr];
    const float x0 = q[i], x1 = q[i + 1];
    q[i] = x0 * c - x1 * sn;
    q[i + 1] = x1 * c + x0 * sn;
  }
  const float scale = rsqrtf((float)D);
  float m = -INFINITY, l = 0.f;
#pragma unroll
  for (int i = 0; i < DPL; ++i) o[i] = 0.f;

  for (int t = 0; t < p.S; ++t) {
    if (t < p.T && p.text_mask && !p.text_mask[(long)b * p.T + t]) continue;
    const long krow = ((long)b * p.S + t) * QC;
    float k[DPL], v[DPL];
    float ks = 0.f;
#pragma unroll
    for (int i = 0; i < DPL; ++i) {
      k[i] = ld_act(X, krow + HD + (long)kvh * D + d0 + i);
      v[i] = ld_act(X, krow + HD + KVD + (long)kvh * D + d0 + i);
      ks += k[i] * k[i];
    }
    const float kr = rsqrtf(warp_sum(ks) / (float)D + p.eps);
#pragma unroll
    for (int i = 0; i < DPL; ++i) k[i] *= kr * (1.f + p.k_norm_w[d0 + i]);
    float dot = 0.f;
#pragma unroll
    for (int i = 0; i < DPL; i += 2) {
      const int pr = (d0 + i) / 2;
      const float c = p.cos[(long)t * halfD + pr], sn = p.sin[(long)t * halfD + pr];
      const float x0 = k[i] * c - k[i + 1] * sn;
      const float x1 = k[i + 1] * c + k[i] * sn;
      dot += q[i] * x0 + q[i + 1] * x1;
    }
    const float sc = warp_sum(dot) * scale;
    const float mn = fmaxf(m, sc);
    const float corr = expf(m - mn);
    const float pe = expf(sc - mn);
    l = l * corr + pe;
#pragma unroll
    for (int i = 0; i < DPL; ++i) o[i] = o[i] * corr + pe * v[i];
    m = mn;
  }
  const float inv = l > 0.f ? 1.f / l : 0.f;  // no valid key (text-only sequence, all padded): zeros
  T* out = reinterpret_cast<T*>(p.out);
#pragma unroll
  for (int i = 0; i < DPL; ++i) {
    const float g = ld_act(X, row * QC + HD + 2L * KVD + (long)h * D + d0 + i);
    const float y = o[i] * inv * (1.f / (1.f + expf(-g)));
    if constexpr (sizeof(T) == 2) out[row * HD + (long)h * D + d0 + i] = __float2bfloat16_rn(y);
    else out[row * HD + (long)h * D + d0 + i] = y;
  }
}

// ----------------------------------------------------------------------------- sampler step
// v = v_cond + g (v_cond - v_uncond); x += (sigma_next - sigma) v; then the next model input
// (x repeated `copies` times) and its timestep sigma_next.
template <bool BF16>
__global__ void euler_cfg_kernel(long long n, float* __restrict__ x, const void* __restrict__ vc,
                                 const void* __restrict__ vu, float g, float dsigma, void* __restrict__ xm,
                                 int copies, float* __restrict__ t_out, float sigma_next) {
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    float c = 0.f, u = 0.f;  // no v_cond: v = 0 (only copies x into the model input)
    if (BF16) {
      if (vc) c = __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(vc)[i]);
      if (vu) u = __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(vu)[i]);
    } else {
      if (vc) c = reinterpret_cast<const float*>(vc)[i];
      if (vu) u = reinterpret_cast<const float*>(vu)[i];
    }
    const float v = vu ? c + g * (c - u) : c;
    const float y = x[i] + dsigma * v;
    x[i] = y;
    if (xm) {
      for (int k = 0; k < copies; ++k) {
        if (BF16) reinterpret_cast<__nv_bfloat16*>(xm)[k * n + i] = __float2bfloat16_rn(y);
        else reinterpret_cast<float*>(xm)[k * n + i] = y;
      }
    }
  }
  if (t_out && blockIdx.x == 0 && threadIdx.x < copies) t_out[threadIdx.x] = sigma_next;
}

inline int check_launch(const char* what) {
  count_launch();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(KREA2_ERR_CUDA, "%s launch failed: %s", what, cudaGetErrorString(e));
  return KREA2_OK;
}

inline int grid_for(long n, int threads) {
  long g = (n + threads - 1) / threads;
  long cap = (long)num_sms() * 16;
  return (int)(g < cap ? (g < 1 ? 1 : g) : cap);
}

}  // namespace

int launch_rope_tables(const float* pos, int S, int a0, int a1, int a2, float theta, float* cos_out, float* sin_out,
                       cudaStream_t stream) {
  const long n = (long)S * ((a0 + a1 + a2) / 2);
  rope_tables_kernel<<<(int)((n + 255) / 256), 256, 0, stream>>>(pos, S, a0, a1, a2, (double)theta, cos_out,
                                                                  sin_out);
  return check_launch("rope_tables");
}

int launch_modulation(const float* temb, const float* table, int B, int C, float* mod, cudaStream_t stream) {
  modulation_kernel<<<grid_for((long)B * 6 * C, 256), 256, 0, stream>>>(temb, table, B, C, mod);
  return check_launch("modulation");
}

int launch_unit_modulation(int B, int C, float* mod, cudaStream_t stream) {
  unit_modulation_kernel<<<grid_for((long)B * 6 * C, 256), 256, 0, stream>>>(B, C, mod);
  return check_launch("unit_modulation");
}

int launch_identity_rope(long n, float* cs, float* sn, cudaStream_t stream) {
  if (n <= 0) return KREA2_OK;
  identity_rope_kernel<<<grid_for(n, 256), 256, 0, stream>>>(n, cs, sn);
  return check_launch("identity_rope");
}

int launch_layer_projection(const float* x, const float* w, long rows, int L, int C, void* out, bool out_bf16,
                            cudaStream_t stream) {
  if (rows <= 0) return KREA2_OK;
  if (out_bf16) layer_projection_kernel<true><<<grid_for(rows * C, 256), 256, 0, stream>>>(x, w, rows, L, C, out);
  else layer_projection_kernel<false><<<grid_for(rows * C, 256), 256, 0, stream>>>(x, w, rows, L, C, out);
  return check_launch("layer_projection");
}

int launch_to_f32(const void* in, bool in_bf16, long n, float* out, cudaStream_t stream) {
  if (n <= 0) return KREA2_OK;
  if (in_bf16) to_f32_kernel<true><<<grid_for(n, 256), 256, 0, stream>>>(in, n, out);
  else to_f32_kernel<false><<<grid_for(n, 256), 256, 0, stream>>>(in, n, out);
  return check_launch("to_f32");
}

int launch_to_dtype(const float* in, long n, void* out, bool out_bf16, cudaStream_t stream) {
  if (n <= 0) return KREA2_OK;
  if (out_bf16) from_f32_kernel<true><<<grid_for(n, 256), 256, 0, stream>>>(in, n, out);
  else from_f32_kernel<false><<<grid_for(n, 256), 256, 0, stream>>>(in, n, out);
  return check_launch("to_dtype");
}

int launch_mod_rmsnorm_rows(const ModNormArgs& a, cudaStream_t stream) {
  const long rows = (long)a.B * a.rows;
  if (rows == 0) return KREA2_OK;
  const int nv = (a.C / 4 + 255) / 256;  // C <= 8192 (check_dims)
  switch (nv) {
#define KREA2_NORM_NV(V)                                                                  \
  case V:                                                                                 \
    if (a.out_bf16) mod_rmsnorm_kernel<true, V><<<(unsigned)rows, 256, 0, stream>>>(a);   \
    else mod_rmsnorm_kernel<false, V><<<(unsigned)rows, 256, 0, stream>>>(a);             \
    break;
    KREA2_NORM_NV(1) KREA2_NORM_NV(2) KREA2_NORM_NV(3) KREA2_NORM_NV(4)
    KREA2_NORM_NV(5) KREA2_NORM_NV(6) KREA2_NORM_NV(7) KREA2_NORM_NV(8)
#undef KREA2_NORM_NV
    default: return set_error(KREA2_ERR_ARG, "modulated RMSNorm supports C <= 8192");
  }
  return check_launch("mod_rmsnorm");
}

int launch_mod_rmsnorm(const float* h, const float* w, const float* temb, const float* table, int chunk, int B, int S,
                       int C, float eps, void* out, bool out_bf16, cudaStream_t stream) {
  ModNormArgs a{};
  a.h = h; a.w = w;
  a.sc = temb + (long)chunk * C; a.sh = temb + (long)(chunk + 1) * C; a.mod_stride = 6LL * C;
  a.sc_tab = table ? table + (long)chunk * C : nullptr;
  a.sh_tab = table ? table + (long)(chunk + 1) * C : nullptr;
  a.B = B; a.rows = S; a.S_in = S; a.row0 = 0; a.C = C; a.eps = eps; a.out = out; a.out_bf16 = out_bf16;
  return launch_mod_rmsnorm_rows(a, stream);
}

int launch_time_embed(const Krea2Dims* d, int B, bool w_bf16, const float* t, const Krea2ModelWeights* w,
                      float* temb, float* e, float* scratch, cudaStream_t stream) {
  const int C = d->C, td = d->t_dim;
  // x0 -> e (as scratch), x1 -> scratch, e -> e, temb
  timestep_sinusoid_kernel<<<(B * (td / 2) + 255) / 256, 256, 0, stream>>>(t, B, td, e);
  int rc = check_launch("timestep_sinusoid");
  if (rc) return rc;
  auto lin = [&](const float* x, const void* W, const float* bias, int N, int K, float* out, bool gelu) {
    dim3 grid((N + 7) / 8);
#define KREA2_GEMV(MB)                                                                                   \
  do {                                                                                                   \
    if (w_bf16) {                                                                                        \
      if (gelu) small_m_linear_kernel<true, true, MB><<<grid, 256, 0, stream>>>(x, W, bias, B, N, K, out);   \
      else small_m_linear_kernel<true, false, MB><<<grid, 256, 0, stream>>>(x, W, bias, B, N, K, out);       \
    } else {                                                                                             \
      if (gelu) small_m_linear_kernel<false, true, MB><<<grid, 256, 0, stream>>>(x, W, bias, B, N, K, out);  \
      else small_m_linear_kernel<false, false, MB><<<grid, 256, 0, stream>>>(x, W, bias, B, N, K, out);      \
    }                                                                                                    \
  } while (0)
    if (B <= 1) KREA2_GEMV(1);
    else if (B <= 2) KREA2_GEMV(2);
    else if (B <= 4) KREA2_GEMV(4);
    else KREA2_GEMV(8);
#undef KREA2_GEMV
    return check_launch("time_linear");
  };
  if ((rc = lin(e, w->t1_w, w->t1_b, C, td, scratch, true))) return rc;
  if ((rc = lin(scratch, w->t2_w, w->t2_b, C, C, e, true))) return rc;
  return lin(e, w->mod_w, w->mod_b, 6 * C, C, temb, false);
}

size_t final_layer_tc_scratch(const Krea2Dims* d, int B, int N, bool bf16) {
  if (!bf16 || d->in_ch % 64) return 0;
  return (size_t)B * N * d->C * 2;
}

int launch_final_layer(const Krea2Dims* d, int B, int T, int N, bool bf16, const float* h, const float* e,
                       const Krea2ModelWeights* w, void* velocity, cudaStream_t stream) {
  const long rows = (long)B * N;
  if (rows == 0) return KREA2_OK;
  if (d->in_ch > FL_MAX_OUT) return set_error(KREA2_ERR_UNSUPPORTED, "in_channels must be <= %d", FL_MAX_OUT);
  const unsigned grid = (unsigned)((rows + FL_ROWS - 1) / FL_ROWS);
  if (bf16)
    final_layer_kernel<true><<<grid, 256, 0, stream>>>(h, e, w->final_norm_w, w->final_table, w->final_w, w->final_b,
                                                        B, T, N, d->C, d->in_ch, d->eps, velocity);
  else
    final_layer_kernel<false><<<grid, 256, 0, stream>>>(h, e, w->final_norm_w, w->final_table, w->final_w, w->final_b,
                                                         B, T, N, d->C, d->in_ch, d->eps, velocity);
  return check_launch("final_layer");
}

int launch_euler_cfg(bool bf16, long long n, float* x, const void* vc, const void* vu, float g, float sigma,
                     float sigma_next, void* xm, int copies, float* t_out, cudaStream_t stream) {
  if (n <= 0) return KREA2_OK;
  const float ds = sigma_next - sigma;
  if (bf16) euler_cfg_kernel<true><<<grid_for(n, 256), 256, 0, stream>>>(n, x, vc, vu, g, ds, xm, copies, t_out, sigma_next);
  else euler_cfg_kernel<false><<<grid_for(n, 256), 256, 0, stream>>>(n, x, vc, vu, g, ds, xm, copies, t_out, sigma_next);
  return check_launch("euler_cfg");
}

int launch_copy_text_rows(const void* text, bool bf16, int B, int T, int S, int C, float* h, cudaStream_t stream) {
  const long total = (long)B * T * C;
  if (total == 0) return KREA2_OK;
  if (bf16) copy_text_rows_kernel<true><<<grid_for(total, 256), 256, 0, stream>>>(text, T, S, C, total, h);
  else copy_text_rows_kernel<false><<<grid_for(total, 256), 256, 0, stream>>>(text, T, S, C, total, h);
  return check_launch("copy_text_rows");
}

int gemm_simt(int epi, const SimtGemmParams& p, const void* A, bool a_bf16, const void* W, bool w_bf16,
              cudaStream_t stream) {
  if (p.M == 0) return KREA2_OK;
  dim3 grid((p.N + SBN - 1) / SBN, (p.M + SBM - 1) / SBM);
#define KREA2_SIMT_CASE(AB, WB, E) \
  if (a_bf16 == AB && w_bf16 == WB && epi == E) { simt_gemm_kernel<AB, WB, E><<<grid, 256, 0, stream>>>(A, W, p); return check_launch("simt_gemm"); }
#define KREA2_SIMT_ALL(E) \
  KREA2_SIMT_CASE(false, false, E) KREA2_SIMT_CASE(true, true, E) KREA2_SIMT_CASE(false, true, E) KREA2_SIMT_CASE(true, false, E)
  KREA2_SIMT_ALL(SEPI_STORE_F32)
  KREA2_SIMT_ALL(SEPI_STORE_BF16)
  KREA2_SIMT_ALL(SEPI_SWIGLU_F32)
  KREA2_SIMT_ALL(SEPI_RESID)
  KREA2_SIMT_ALL(SEPI_BIAS_ROWMAP)
  KREA2_SIMT_ALL(SEPI_BIAS_F32)
  KREA2_SIMT_ALL(SEPI_BIAS_BF16)
#undef KREA2_SIMT_ALL
#undef KREA2_SIMT_CASE
  return set_error(KREA2_ERR_ARG, "unknown SIMT epilogue %d", epi);
}

int attention_simt(const AttnParams& p, bool bf16, cudaStream_t stream) {
  const long warps = (long)p.B * p.S * p.H;
  if (warps == 0) return KREA2_OK;
  const unsigned grid = (unsigned)((warps + 7) / 8);
  if (p.D == 64) {
    if (bf16) attn_simt_kernel<__nv_bfloat16, 2><<<grid, 256, 0, stream>>>(p);
    else attn_simt_kernel<float, 2><<<grid, 256, 0, stream>>>(p);
  } else if (p.D == 128) {
    if (bf16) attn_simt_kernel<__nv_bfloat16, 4><<<grid, 256, 0, stream>>>(p);
    else attn_simt_kernel<float, 4><<<grid, 256, 0, stream>>>(p);
  } else {
    return set_error(KREA2_ERR_UNSUPPORTED, "attention needs head_dim 64 or 128, got %d", p.D);
  }
  return check_launch("attention_simt");
}

}  // namespace krea2
