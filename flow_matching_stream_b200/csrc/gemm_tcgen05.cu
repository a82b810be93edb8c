// Dense bf16 projections of the Krea 2 block on the sm_100a tensor cores (tcgen05 + TMEM),
// fed by TMA: out = A · Wᵀ with A (M, K) and W (N, K) both K-major (row-major, K contiguous).
//
// Used for the block's four linears (page "Diffusers 中的 Krea2Transformer2DModel … 架构全解",
// §四.2 block and §四.3 attention): the fused [to_q | to_k | to_v | to_gate] projection, to_out
// with the gated residual, the SwiGLU gate/up projection with silu(gate)*up, and the down
// projection with the second gated residual.
//
// Design (one CTA per SM, persistent over output tiles):
//   warp 0      TMA producer: A tile 128x64 and W tile BNx64 per stage, 128-byte swizzle,
//               STAGES-deep ring guarded by full/empty mbarriers, into this CTA's own shared memory.
//   warp 1      allocates TMEM (2 accumulators x BN fp32 columns) and issues tcgen05.mma
//               (M=128, N=BN, K=16) from one thread; tcgen05.commit frees smem stages and
//               signals a finished accumulator.
//   warps 2..5  epilogue: each thread owns one accumulator row (TMEM lane), reads 32 columns
//               at a time with tcgen05.ld and applies the fused epilogue, while the MMA warp
//               already accumulates the next tile into the other TMEM buffer. The bf16
//               epilogues (plain, SwiGLU, q/k/v/gate) write each warp's 32 rows into swizzled
//               shared-memory boxes that TMA stores; the fp32 residual and the row-mapped
//               output pass through a padded shared tile so that global accesses run in whole
//               128-byte row segments.
// Tiles are visited in raster groups of row tiles, sized so that one wave of tiles reads about
// as many A bytes as W bytes per K step and so that concurrently running CTAs share A and W
// tiles through L2.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstring>

#include "krea2_device.cuh"
#include "krea2_internal.h"

namespace krea2 {

namespace {

constexpr int BM = 128;
constexpr int BK = 64;
// Row tiles per raster group (group_rows below): at least as many as keep the group's A tiles
// (128 x K bf16 each) within about 24 MB of L2, so W streams from HBM once per group pass, and
// at least as many as make one wave of tiles read about as many A bytes as W bytes per K step.
constexpr size_t GROUP_A_BYTES = 24ull << 20;
// Epilogue warps: 8 for the residual (two per TMEM lane quarter, each on half the tile's
// columns), 4 for the others. The residual's read-modify-write of h is bound by the loads in
// flight; with 4 warps it took longer per tile than to_out's mainloop (K = 6144).
template <int EPI>
constexpr int epi_warps() { return EPI == EPI_RESID ? 8 : 4; }
template <int EPI>
constexpr int gemm_threads() { return 64 + 32 * epi_warps<EPI>(); }

template <int BN>
struct GemmCfg {
  static constexpr int A_BYTES = BM * BK * 2;   // 16 KB
  static constexpr int B_BYTES = BN * BK * 2;   // 32 KB (BN=256) or 16 KB (BN=128)
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = (BN == 256) ? 4 : 6;
  // Epilogue staging per warp: two 4 KB swizzled 32x64 bf16 boxes (TMA-store epilogues), or one
  // padded 32x33 fp32 tile (residual and row-mapped epilogues), at 8 KB spacing.
  static constexpr int EPI_WARP_BYTES = 8192;
  static constexpr int EPI_BYTES = 4 * EPI_WARP_BYTES;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + EPI_BYTES + 1024;  // + alignment slack
  static constexpr int TMEM_COLS = 2 * BN;                         // double-buffered fp32
  static constexpr uint32_t IDESC = idesc_bf16_f32(BM, BN);
};

struct TileMap {
  int tiles_m, tiles_n, group_m;
  __device__ __forceinline__ void map(int t, int& mt, int& nt) const {
    int per_group = group_m * tiles_n;
    int g = t / per_group;
    int first_m = g * group_m;
    int gsize = min(tiles_m - first_m, group_m);
    int local = t - g * per_group;
    mt = first_m + local % gsize;
    nt = local / gsize;
  }
};

// The bf16 epilogues hand each warp's 32 rows to the TMA unit through boxes in shared memory:
// 32 rows x 128 bytes (64 bf16 columns), 128-byte swizzle, so 16-byte chunk j of box
// row r sits at position j ^ (r & 7) and a warp's row-wise 16-byte stores spread over all banks.
// Rows and columns outside the output are clipped by the tensor map. Each warp owns two boxes
// and alternates between them; a box is rewritten only once the TMA operation issued from it two
// boxes earlier has finished reading it.
struct EpiBoxes {
  uint8_t* smem;
  int n;
  __device__ __forceinline__ uint8_t* next(int lane) {
    uint8_t* b = smem + (n++ & 1) * 4096;
    if (lane == 0) bulk_wait_group_read<1>();
    __syncwarp();
    return b;
  }
};

__device__ __forceinline__ void box_put16(uint8_t* box, int lane, int j, uint4 v) {
  *reinterpret_cast<uint4*>(box + lane * 128 + ((j ^ (lane & 7)) << 4)) = v;
}

// Thread `lane` holds row `lane` of a 32 x 64 bf16 block as 32 packed pairs; the warp stores the
// block at output column x, row y (issue = false skips a block wholly past the last row).
__device__ __forceinline__ void store_box_bf16(uint8_t* box, const uint32_t* pk, int lane, const CUtensorMap* tm,
                                               int x, int y, bool issue) {
#pragma unroll
  for (int j = 0; j < 8; ++j) box_put16(box, lane, j, make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]));
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0 && issue) {
    tma_store_2d(tm, box, x, y);
    bulk_commit_group();
  }
}

template <int BN, int EPI>
__global__ void __launch_bounds__(gemm_threads<EPI>(), 1)
    gemm_bf16_tcgen05_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                             const __grid_constant__ CUtensorMap tmC, GemmParams p) {
  using Cfg = GemmCfg<BN>;
  constexpr int STAGES = Cfg::STAGES;

  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[STAGES];
  __shared__ __align__(8) uint64_t empty_bar[STAGES];
  __shared__ __align__(8) uint64_t tfull_bar[2];
  __shared__ __align__(8) uint64_t tempty_bar[2];
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t base_u32 = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* base = smem_raw + (base_u32 - smem_u32(smem_raw));

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull_bar[a], 1);
      mbar_init(&tempty_bar[a], 32 * epi_warps<EPI>());
    }
    mbar_init(&drain_bar, 1);
    abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) tmem_alloc(&tmem_slot, Cfg::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_slot;
  volatile int* abort = &abort_flag;

  const TileMap tm{p.tiles_m, p.tiles_n, p.group_m};
  const int total = p.tiles_m * p.tiles_n;
  const int nk = p.K / BK;

  if (warp == 0) {
    if (lane == 0) {
      uint32_t stage = 0, phase = 0;
      IssuedFills fills;
      for (int t = blockIdx.x; t < total; t += gridDim.x) {
        int mt, nt;
        tm.map(t, mt, nt);
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1, abort)) goto producer_done;
          uint8_t* sa = base + stage * Cfg::STAGE_BYTES;
          mbar_arrive_expect_tx(&full_bar[stage], Cfg::STAGE_BYTES);
          tma_load_2d(sa, &tmA, &full_bar[stage], kb * BK, mt * BM);
          tma_load_2d(sa + Cfg::A_BYTES, &tmB, &full_bar[stage], kb * BK, nt * BN);
          fills.note(stage, phase);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
    producer_done:
      // a wait expired somewhere: let the copies this thread issued land before the CTA exits
      if (*abort) fills.drain(full_bar, STAGES);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      uint32_t stage = 0, phase = 0;
      int local = 0;
      bool issued = false;
      // stage s's A tile starts s * STAGE_BYTES into the ring and its W tile A_BYTES later; a
      // K step of 16 is 32 bytes: only the descriptor's start-address field (16-byte units)
      // changes, so each MMA takes a base descriptor plus a constant
      const uint64_t da0 = smem_desc_sw128(smem_u32(base), 16, 1024);
      for (int t = blockIdx.x; t < total; t += gridDim.x, ++local) {
        const int acc = local & 1;
        const uint32_t acc_phase = (local >> 1) & 1;
        if (!mbar_wait(&tempty_bar[acc], acc_phase ^ 1, abort)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&full_bar[stage], phase, abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = da0 + (uint64_t)(stage * (Cfg::STAGE_BYTES >> 4));
          const uint64_t bd = ad + (uint64_t)(Cfg::A_BYTES >> 4);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) tc_mma_bf16(d_tmem, ad + 2 * k, bd + 2 * k, Cfg::IDESC, (kb | k) != 0);
          issued = true;
          tc_commit(&empty_bar[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        tc_commit(&tfull_bar[acc]);
      }
      if (*abort && issued) {
        // let every MMA already issued finish before TMEM is released
        tc_commit(&drain_bar);
        mbar_wait(&drain_bar, 0, &abort_flag /* already set: bounded by the timer below */);
        unsigned long long t0 = globaltimer_ns();
        while (!mbar_try_wait(&drain_bar, 0) && globaltimer_ns() - t0 < WAIT_LIMIT_NS) {
        }
      }
    }
  } else {
    // epilogue warps 2.. -> TMEM lane quarters 2, 3, 0, 1 (2, 3, 0, 1 again for the residual's
    // second four warps, which take the other half of the columns)
    const int quarter = warp & 3;
    const int part = (warp - 2) >> 2;
    EpiBoxes boxes{base + STAGES * Cfg::STAGE_BYTES + (warp - 2) * Cfg::EPI_WARP_BYTES, 0};
    int local = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++local) {
      int mt, nt;
      tm.map(t, mt, nt);
      const int acc = local & 1;
      const uint32_t acc_phase = (local >> 1) & 1;
      if (!mbar_wait(&tfull_bar[acc], acc_phase, abort)) break;
      tc_fence_after();
      const int row = mt * BM + quarter * 32 + lane;
      const bool row_ok = row < p.M;
      const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * BN;

      const int row0 = mt * BM + quarter * 32;
      const int nrows = min(32, p.M - row0);
      uint8_t* epi_smem = base + STAGES * Cfg::STAGE_BYTES + (warp - 2) * Cfg::EPI_WARP_BYTES;
      uint32_t* xpk = reinterpret_cast<uint32_t*>(epi_smem);
      const bool rows_in = row0 < p.M;  // warp-uniform: this 32-row block holds output rows
      if constexpr (EPI == EPI_STORE) {
        const int n_store = p.n_store ? p.n_store : p.N;
#pragma unroll 1
        for (int c = 0; c < BN / 64; ++c) {
          if (nt * BN + c * 64 >= n_store) break;  // warp-uniform: padding columns of W are not stored
          float v[64];
          tmem_ld64(tbase + c * 64, v);
          if (p.bias) {
            const float4* bp = reinterpret_cast<const float4*>(p.bias + (size_t)nt * BN + c * 64);
#pragma unroll
            for (int q = 0; q < 16; ++q) {
              const float4 bv = __ldg(bp + q);
              v[q * 4 + 0] += bv.x;
              v[q * 4 + 1] += bv.y;
              v[q * 4 + 2] += bv.z;
              v[q * 4 + 3] += bv.w;
            }
          }
          uint32_t pk[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) pk[e] = pack_bf16x2(v[2 * e], v[2 * e + 1]);
          store_box_bf16(boxes.next(lane), pk, lane, &tmC, nt * BN + c * 64, row0, rows_in);
        }
      } else if constexpr (EPI == EPI_BIAS_ROWMAP) {
        // fp32 out[map(row), col] = acc + bias[col], rows transposed through shared memory like the
        // residual epilogue below; lane i holds the destination row of tile row row0 + i
        float* xp = reinterpret_cast<float*>(xpk);
        const int rr = min(row0 + lane, p.M - 1);
        const long long my_dst = (long long)(rr / p.map_N) * p.map_S + p.map_T + rr % p.map_N;
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          float v[32];
          tmem_ld32(tbase + c * 32, v);
#pragma unroll
          for (int e = 0; e < 32; ++e) xp[lane * 33 + e] = v[e];
          __syncwarp();
          const int col = nt * BN + c * 32 + lane;
          const float bv = p.bias ? __ldg(p.bias + col) : 0.f;
          float* out = reinterpret_cast<float*>(p.out) + col;
#pragma unroll 8
          for (int i = 0; i < 32; ++i) {
            const long long dst = __shfl_sync(0xffffffffu, my_dst, i);
            if (i < nrows) out[dst * p.N] = xp[i * 33 + lane] + bv;
          }
          __syncwarp();
        }
      } else if constexpr (EPI == EPI_SWIGLU) {
        // interleaved 64-row groups: columns [128g, 128g+64) gate, [128g+64, 128g+128) up; each
        // group gives 64 output columns
#pragma unroll 1
        for (int g = 0; g < BN / 128; ++g) {
          uint32_t pk[32];
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            float gv[32], uv[32];
            tmem_ld32(tbase + g * 128 + half * 32, gv);
            tmem_ld32(tbase + g * 128 + 64 + half * 32, uv);
#pragma unroll
            for (int e = 0; e < 16; ++e)
              pk[half * 16 + e] = pack_bf16x2(silu_f(gv[2 * e]) * uv[2 * e], silu_f(gv[2 * e + 1]) * uv[2 * e + 1]);
          }
          store_box_bf16(boxes.next(lane), pk, lane, &tmC, nt * (BN / 2) + g * 64, row0, rows_in);
        }
      } else if constexpr (EPI == EPI_QKV) {
        // [q | k | v | gate] columns; 128-wide q/k heads get RMSNorm (1 + w) and RoPE here,
        // once per element, on the fp32 accumulator (page §四.3 order: norm, then RoPE)
        const int pos = row_ok ? row % p.rows_per_batch : 0;
        const float* cs = p.cos + (size_t)pos * 64;
        const float* sn = p.sin + (size_t)pos * 64;
#pragma unroll 1
        for (int u = 0; u < BN / 128; ++u) {
          const int c0 = nt * BN + u * 128;
          const bool is_q = c0 < p.HD;
          const bool is_k = !is_q && c0 < p.HD + p.KVD;
          const uint32_t ub = tbase + u * 128;
          float r = 1.f;
          if (is_q || is_k) {  // pass 1: sum of squares over the head's 128 columns
            float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
            for (int h2 = 0; h2 < 2; ++h2) {
              float v[64];
              tmem_ld64(ub + h2 * 64, v);
#pragma unroll
              for (int e = 0; e < 64; ++e) s4[e & 3] += v[e] * v[e];
            }
            r = rsqrtf(((s4[0] + s4[1]) + (s4[2] + s4[3])) * (1.f / 128.f) + p.eps);
          }
          const float4* w4 = reinterpret_cast<const float4*>(is_q ? p.qw : p.kw);
#pragma unroll 1
          for (int h2 = 0; h2 < 2; ++h2) {  // pass 2: normalise, rotate, store 64 columns at a time
            float v[64];
            tmem_ld64(ub + h2 * 64, v);
            if (is_q || is_k) {
              const float4* c4 = reinterpret_cast<const float4*>(cs + h2 * 32);
              const float4* s4p = reinterpret_cast<const float4*>(sn + h2 * 32);
#pragma unroll
              for (int q = 0; q < 8; ++q) {  // 8 dims (4 rotated pairs) per step
                const float4 wa = __ldg(w4 + h2 * 16 + 2 * q), wb = __ldg(w4 + h2 * 16 + 2 * q + 1);
                const float4 co = __ldg(c4 + q), si = __ldg(s4p + q);
                const float wv[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
                const float cv[4] = {co.x, co.y, co.z, co.w}, sv[4] = {si.x, si.y, si.z, si.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const int d = q * 8 + 2 * e;
                  const float x0 = v[d] * r * (1.f + wv[2 * e]);
                  const float x1 = v[d + 1] * r * (1.f + wv[2 * e + 1]);
                  v[d] = x0 * cv[e] - x1 * sv[e];
                  v[d + 1] = x1 * cv[e] + x0 * sv[e];
                }
              }
            }
            uint32_t pk[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) pk[e] = pack_bf16x2(v[2 * e], v[2 * e + 1]);
            store_box_bf16(boxes.next(lane), pk, lane, &tmC, nt * BN + u * 128 + h2 * 64, row0, rows_in);
          }
        }
      } else {  // EPI_RESID: h[row, col] += gate[b, col] * acc
        // A plain read-modify-write of h through L1/L2, not a TMA reduce-add: h is also written
        // by plain stores (img_in, the text rows, the caller), and in one launch sequence a TMA
        // reduce-add of this epilogue returned the value h held before the img_in kernel, several
        // launches earlier in the same stream. After tcgen05.ld each thread holds one row of a
        // 32-column chunk; row-by-row global accesses would touch 32 cache lines per warp access,
        // so the warp transposes its 32x32 block through shared memory (XOR-swizzled: element
        // (row i, column e) at i * 32 + (e ^ i), conflict-free both ways) and walks the rows: each
        // access is one 128-byte line, and 16 rows of loads are in flight before any store. Warp
        // part 0 takes the tile's first BN / 2 columns, part 1 the rest.
        // Lane i knows the batch row of tile row row0 + i (clamped to M - 1, so that rows of the
        // ragged last tile read an in-bounds gate; their results are never stored).
        float* xp = reinterpret_cast<float*>(base + STAGES * Cfg::STAGE_BYTES) + (warp - 2) * (32 * 32);
        const int my_b = min(row0 + lane, p.M - 1) / p.rows_per_batch;
#pragma unroll 1
        for (int c = part * (BN / 64); c < (part + 1) * (BN / 64); ++c) {
          float v[32];
          tmem_ld32(tbase + c * 32, v);
#pragma unroll
          for (int e = 0; e < 32; ++e) xp[lane * 32 + (e ^ lane)] = v[e];
          __syncwarp();
          const int col = nt * BN + c * 32 + lane;
#pragma unroll 1
          for (int i0 = 0; i0 < 32; i0 += 16) {
            float* hp = reinterpret_cast<float*>(p.out) + (size_t)(row0 + i0) * p.N + col;
            float hv[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) hv[i] = i0 + i < nrows ? hp[(size_t)i * p.N] : 0.f;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const int bb = __shfl_sync(0xffffffffu, my_b, i0 + i);
              hv[i] += __ldg(p.gate + (size_t)bb * p.gate_stride + col) * xp[(i0 + i) * 32 + (lane ^ (i0 + i))];
            }
#pragma unroll
            for (int i = 0; i < 16; ++i)
              if (i0 + i < nrows) hp[(size_t)i * p.N] = hv[i];
          }
          __syncwarp();
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty_bar[acc]);
    }
    // the TMA stores must be complete (their boxes read, the output written) before
    // this CTA's shared memory goes away
    if (lane == 0) bulk_wait_all();
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

}  // namespace

// Row-major bf16 matrix (rows, cols) as a 2-D TMA map with a (box_cols x box_rows) box and
// 128-byte swizzle (box_cols * 2 bytes must be 128).
int make_tmap_bf16_2d(CUtensorMap* m, const void* ptr, uint64_t cols, uint64_t rows, uint64_t row_stride_elems,
                      uint32_t box_cols, uint32_t box_rows) {
  auto enc = get_encode_fn();
  if (!enc) return set_error(KREA2_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  if ((reinterpret_cast<uintptr_t>(ptr) & 15) || ((row_stride_elems * 2) & 15))
    return set_error(KREA2_ERR_ARG, "TMA operand must be 16-byte aligned with a 16-byte multiple row stride");
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {row_stride_elems * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t es[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return set_error(KREA2_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return KREA2_OK;
}

// Row-major bf16 matrix viewed as (batches, rows, cols) with `row_stride_elems` between rows and
// rows*row_stride between batches; box (box_cols x box_rows x 1), 128-byte swizzle. Rows past
// `rows` in a batch read as zero.
// (cols, rows, batches) view with batch b starting batch_rows rows after batch b-1 (batch_rows >=
// rows); rows at or beyond `rows` read as zeros, also when the buffer holds more.
int make_tmap_bf16_3d(CUtensorMap* m, const void* ptr, uint64_t cols, uint64_t rows, uint64_t batches,
                      uint64_t row_stride_elems, uint32_t box_cols, uint32_t box_rows, uint64_t batch_rows) {
  auto enc = get_encode_fn();
  if (!enc) return set_error(KREA2_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  if ((reinterpret_cast<uintptr_t>(ptr) & 15) || ((row_stride_elems * 2) & 15))
    return set_error(KREA2_ERR_ARG, "TMA operand must be 16-byte aligned with a 16-byte multiple row stride");
  cuuint64_t dims[3] = {cols, rows, batches};
  if (batch_rows < rows) return set_error(KREA2_ERR_ARG, "batch stride of %llu rows is below the %llu rows read",
                                          (unsigned long long)batch_rows, (unsigned long long)rows);
  cuuint64_t strides[2] = {row_stride_elems * 2, row_stride_elems * 2 * batch_rows};
  cuuint32_t box[3] = {box_cols, box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return set_error(KREA2_ERR_CUDA, "cuTensorMapEncodeTiled (3-D) failed (%d)", (int)r);
  return KREA2_OK;
}

namespace {

// Row tiles per raster group. The persistent CTAs run about `sms` consecutive tiles at once: r
// row tiles by c = sms / r column tiles of one group. Per K step that wave reads r*BM rows of A
// and c*BN rows of W, which is least at r = sqrt(sms * BN / BM) (18 for BN = 256 on 148 SMs);
// with much fewer rows, each wave streams nearly all of W from HBM. The row tiles are then split
// into groups of equal size.
int group_rows(int tiles_m, int K, int BN, int sms) {
  const int by_l2 = (int)(GROUP_A_BYTES / ((size_t)BM * K * 2));
  const int by_wave = (int)std::ceil(std::sqrt((double)sms * BN / BM));
  int g = by_l2 > by_wave ? by_l2 : by_wave;
  if (g >= tiles_m) return tiles_m;
  const int groups = (tiles_m + g - 1) / g;
  return (tiles_m + groups - 1) / groups;
}

template <int BN, int EPI>
int launch_gemm_bn(const GemmParams& p0, const void* A, const void* W, cudaStream_t stream) {
  using Cfg = GemmCfg<BN>;
  static std::atomic<uint64_t> attr_done{0};
  auto kern = gemm_bf16_tcgen05_kernel<BN, EPI>;
  const uint64_t dev_bit = device_bit();
  if (!(attr_done.load(std::memory_order_acquire) & dev_bit) || !dev_bit) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES) != cudaSuccess)
      return set_error(KREA2_ERR_CUDA, "cudaFuncSetAttribute(gemm) failed");
    attr_done.fetch_or(dev_bit, std::memory_order_release);
  }
  CUtensorMap ta, tb, tc;
  int rc = make_tmap_bf16_2d(&ta, A, p0.K, p0.M, p0.K, BK, BM);
  if (rc) return rc;
  rc = make_tmap_bf16_2d(&tb, W, p0.K, p0.w_rows ? p0.w_rows : p0.N, p0.K, BK, BN);
  if (rc) return rc;
  GemmParams p = p0;
  // the bf16 epilogues' TMA target: 32-row boxes of 128 bytes (64 bf16 columns)
  memset(&tc, 0, sizeof(tc));
  if constexpr (EPI == EPI_RESID) {
    // plain loads and stores (see the epilogue); the 16-byte rule keeps the API uniform
    if (reinterpret_cast<uintptr_t>(p.out) & 15)
      return set_error(KREA2_ERR_ARG, "residual output must be 16-byte aligned");
  } else if constexpr (EPI == EPI_STORE) {
    if ((rc = make_tmap_bf16_2d(&tc, p.out, p.n_store ? p.n_store : p.N, p.M, p.out_ld ? p.out_ld : p.N, 64, 32)))
      return rc;
  } else if constexpr (EPI == EPI_SWIGLU) {
    if ((rc = make_tmap_bf16_2d(&tc, p.out, p.N / 2, p.M, p.N / 2, 64, 32))) return rc;
  } else if constexpr (EPI == EPI_QKV) {
    if ((rc = make_tmap_bf16_2d(&tc, p.out, p.N, p.M, p.N, 64, 32))) return rc;
  }
  p.tiles_m = (p.M + BM - 1) / BM;
  p.tiles_n = p.N / BN;
  p.group_m = group_rows(p.tiles_m, p.K, BN, num_sms());
  const int total = p.tiles_m * p.tiles_n;
  const int grid = total < num_sms() ? total : num_sms();
  kern<<<grid, gemm_threads<EPI>(), Cfg::SMEM_BYTES, stream>>>(ta, tb, tc, p);
  count_launch();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(KREA2_ERR_CUDA, "gemm launch failed: %s", cudaGetErrorString(e));
  return KREA2_OK;
}

// Wave efficiency of a tile count on the SMs (1.0 = every wave full).
double wave_eff(long tiles, int sms) {
  long waves = (tiles + sms - 1) / sms;
  return (double)tiles / (double)(waves * sms);
}

}  // namespace

KREA2_DEFINE_ERROR_READER(take_device_error_gemm)

int gemm_bf16(int epi, const GemmParams& p, const void* A, const void* W, cudaStream_t stream) {
  // choose the N tile: 256 unless 128 fills the machine clearly better
  const int sms = num_sms();
  const long tm = (p.M + BM - 1) / BM;
  int bn = 128;
  if (p.N % 256 == 0) {
    const double e256 = wave_eff(tm * (p.N / 256), sms);
    const double e128 = wave_eff(tm * (p.N / 128), sms);
    bn = (e256 >= 0.8 * e128 || tm * (p.N / 256) >= 4L * sms) ? 256 : 128;
  }
  if (bn == 256) {
    switch (epi) {
      case EPI_STORE: return launch_gemm_bn<256, EPI_STORE>(p, A, W, stream);
      case EPI_SWIGLU: return launch_gemm_bn<256, EPI_SWIGLU>(p, A, W, stream);
      case EPI_QKV: return launch_gemm_bn<256, EPI_QKV>(p, A, W, stream);
      case EPI_BIAS_ROWMAP: return launch_gemm_bn<256, EPI_BIAS_ROWMAP>(p, A, W, stream);
      default: return launch_gemm_bn<256, EPI_RESID>(p, A, W, stream);
    }
  }
  switch (epi) {
    case EPI_STORE: return launch_gemm_bn<128, EPI_STORE>(p, A, W, stream);
    case EPI_SWIGLU: return launch_gemm_bn<128, EPI_SWIGLU>(p, A, W, stream);
    case EPI_QKV: return launch_gemm_bn<128, EPI_QKV>(p, A, W, stream);
    case EPI_BIAS_ROWMAP: return launch_gemm_bn<128, EPI_BIAS_ROWMAP>(p, A, W, stream);
    default: return launch_gemm_bn<128, EPI_RESID>(p, A, W, stream);
  }
}

}  // namespace krea2
