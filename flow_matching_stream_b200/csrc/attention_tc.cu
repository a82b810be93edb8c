// Grouped-query flash attention of the Krea 2 block on the sm_100a tensor cores.
//
// Source: page "Diffusers 中的 Krea2Transformer2DModel … 架构全解", §四.3 (Krea2Attention /
// Krea2AttnProcessor): q and k are RMS-normalised per head over head_dim, rotated by the 3-axis
// RoPE, K/V heads are shared by H/Hkv = 4 consecutive query heads (the processor's
// repeat_interleave order), the text padding mask removes keys, and the merged heads are
// multiplied by sigmoid(to_gate(x)).
//
// Kernel layout (one CTA per (128/G query positions, KV head j, batch row b); two CTAs per SM):
//   * The 128-row MMA tile stacks the G query heads of KV head j (G = 4 in the Krea 2 block):
//     row r = QPOS*hl + p holds head G*j+hl at position p0+p, QPOS = 128/G. One K/V tile in
//     shared memory therefore serves all G heads (K/V are never copied per query head).
//   * warp 0: TMA producer (Q once; K and V 64-key tiles, 2-stage ring), into this CTA's own shared memory.
//   * warp 1: MMA issuer. S_i = Q K_iᵀ into one of two TMEM score buffers; P_i (bf16, written
//     back over its own scores) is the TMEM A operand of O += P_i V_i, V being the MN-major B
//     operand in shared memory.
//   * warps 2..9: softmax, two threads per tile row (TMEM lane), each on 32 of the 64 scores:
//     half-row max exchanged in shared memory, exp2 into bf16 P in TMEM, then (after
//     P_{i-1} V_{i-1} has landed) lazy rescaling of its half of O, only when the running max
//     grows by more than 2^8; final 1/l and sigmoid(gate) epilogue.
//   * 96 KB of shared memory and 256 TMEM columns per CTA let two CTAs share an SM, so each
//     SM sub-partition interleaves two independent softmax warps with the MMAs.
//   * Key tiles whose keys are all padded text are skipped entirely; partially padded tiles and
//     the ragged end of the sequence are masked per key, full tiles take a mask-free path.
// q and k arrive already RMS-normalised and rotated (the fused projection's epilogue or the
// prep kernel below does that once per element); v and gate are raw projection columns.
#include <cuda.h>

#include "krea2_device.cuh"
#include "krea2_internal.h"

namespace krea2 {

int make_tmap_bf16_3d(CUtensorMap* m, const void* ptr, uint64_t cols, uint64_t rows, uint64_t batches,
                      uint64_t row_stride_elems, uint32_t box_cols, uint32_t box_rows, uint64_t batch_rows);

namespace {

constexpr int AD = 128;          // head dim
constexpr int KT = 64;           // keys per tile
constexpr int KV_STAGES = 2;
constexpr int ATT_THREADS = 320;  // producer, MMA, 8 softmax warps
constexpr int Q_CHUNK = 128 * 128;                // 128 rows x 64 bf16 (128 B) = 16 KB
constexpr int Q_BYTES = 2 * Q_CHUNK;              // 32 KB
constexpr int KV_CHUNK = KT * 128;                // 64 rows x 128 B = 8 KB
constexpr int KV_TILE_BYTES = 2 * KV_CHUNK;       // 16 KB each for K and V
constexpr int OFF_Q = 0;
constexpr int OFF_K = OFF_Q + Q_BYTES;
constexpr int OFF_V = OFF_K + KV_STAGES * KV_TILE_BYTES;
constexpr int ATT_SMEM = OFF_V + KV_STAGES * KV_TILE_BYTES + 1024;  // + alignment slack
constexpr int MAX_TILES = 1024;  // S <= 65536
constexpr uint32_t TMEM_COLS = 256;  // S0 [0,64), S1 [64,128), O [128,256)
constexpr uint32_t O_COL = 128;
constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, KT, 0, 0);
constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, AD, 0, 1);

struct AttnCore {
  int B, T, N, S, Hkv, HD;
  int Sq;     // query rows per batch row (S, or the new tokens of a key/value cache step)
  int q_off;  // key position of query row 0 (0, or L - Sq for a cache step)
  const uint8_t* text_mask;
  const __nv_bfloat16* gate;  // gate column block base (row stride g_stride)
  long long g_stride;
  __nv_bfloat16* out;         // (B*S, HD)
  float scale_log2;
  const int* key_end;         // PREFIX: query row q reads keys [0, key_end[q]) only (same for all batch rows)
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Paired fp32 ops of sm_100: two lanes of work per instruction.
__device__ __forceinline__ unsigned long long f2u(float lo, float hi) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void u2f(unsigned long long v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ unsigned long long ffma2(unsigned long long a, unsigned long long b, unsigned long long c) {
  unsigned long long r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ unsigned long long fadd2(unsigned long long a, unsigned long long b) {
  unsigned long long r;
  asm("add.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// exp2 of (v * sl2 - m) for NE scores, packed to bf16 pairs; returns the sum of the fp32 values.
template <int NE>
__device__ __forceinline__ float exp_tile(const float* v, float sl2, float m, uint32_t* pk) {
  const unsigned long long s2 = f2u(sl2, sl2), nm2 = f2u(-m, -m);
  unsigned long long acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
  for (int e = 0; e < NE / 2; ++e) {
    float x0, x1;
    u2f(ffma2(f2u(v[2 * e], v[2 * e + 1]), s2, nm2), x0, x1);
    const float a = ex2(x0), c = ex2(x1);
    pk[e] = pack_bf16x2(a, c);
    acc[e & 3] = fadd2(acc[e & 3], f2u(a, c));
  }
  float t[8];
#pragma unroll
  for (int k = 0; k < 4; ++k) u2f(acc[k], t[2 * k], t[2 * k + 1]);
  return ((t[0] + t[1]) + (t[2] + t[3])) + ((t[4] + t[5]) + (t[6] + t[7]));
}

__device__ __forceinline__ bool key_valid(const AttnCore& p, int b, int t) {
  if (t >= p.S) return false;
  if (t < p.T && p.text_mask) return p.text_mask[(long)b * p.T + t] != 0;
  return true;
}

// G query heads share one KV head; the 128-row tile holds G heads x QPOS = 128/G positions.
template <int G, bool PREFIX>
__global__ void __launch_bounds__(ATT_THREADS, 2)
    attn_gqa_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, AttnCore p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t q_full;
  __shared__ __align__(8) uint64_t k_full[KV_STAGES];
  __shared__ __align__(8) uint64_t v_full[KV_STAGES];
  __shared__ __align__(8) uint64_t k_empty[KV_STAGES];  // freed when the S = Q K^T MMA is done
  __shared__ __align__(8) uint64_t v_empty[KV_STAGES];  // freed when the O += P V MMA is done
  __shared__ __align__(8) uint64_t s_full[2];
  // P_i is complete once all 256 softmax threads arrive on p_full[i & 1]. A fast warp may
  // finish tile i+1 before a slow one finishes tile i (nothing else holds them together
  // when no rescale waits on PV), so consecutive tiles count on different barriers; a warp
  // cannot reach tile i+2 before PV_i, and so before every warp's arrival for tile i.
  __shared__ __align__(8) uint64_t p_full[2];
  __shared__ __align__(8) uint64_t pv_done[2];  // PV_i commits on pv_done[i & 1]
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  __shared__ int n_tiles;
  __shared__ int cta_kmin;  // PREFIX: smallest key_end of this CTA's queries (keys below it need no row mask)
  __shared__ uint16_t tiles[MAX_TILES];

  constexpr int QPOS = 128 / G;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int p0 = blockIdx.x * QPOS, j = blockIdx.y, b = blockIdx.z;
  const uint32_t base_u32 = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* base = smem_raw + (base_u32 - smem_u32(smem_raw));

  // ---- key tiles that hold at least one valid key (all-padded text tiles are skipped; with a
  // key prefix, tiles at or beyond the largest key_end of the CTA's queries too)
  if (warp == 0) {
    int kmax = p.S;
    if constexpr (PREFIX) {
      int hi = 0, lo = p.S;
      for (int i = lane; i < QPOS; i += 32) {
        const int q = p0 + i;
        if (q < p.Sq) {
          const int e = min(max(p.key_end[q], p.q_off + q + 1), p.S);
          hi = max(hi, e);
          lo = min(lo, e);
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
        lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
      }
      kmax = hi;
      if (lane == 0) cta_kmin = lo;
    }
    const int total = (min(kmax, p.S) + KT - 1) / KT;
    int count = 0;
    for (int t0 = 0; t0 < total; t0 += 32) {
      const int t = t0 + lane;
      bool valid = false;
      if (t < total) {
        const int k0 = t * KT;
        const int k1 = min(k0 + KT, p.S);
        if (!p.text_mask || k1 > p.T) {
          valid = true;  // every key valid, or the tile holds image keys (always valid)
        } else {
          for (int k = k0; k < k1 && !valid; ++k) valid = p.text_mask[(long)b * p.T + k] != 0;
        }
      }
      const unsigned m = __ballot_sync(0xffffffffu, valid);
      if (valid) tiles[count + __popc(m & ((1u << lane) - 1u))] = (uint16_t)t;
      count += __popc(m);
    }
    if (lane == 0) n_tiles = count;
  }
  if (threadIdx.x == 0) {
    mbar_init(&q_full, 1);
    for (int s = 0; s < KV_STAGES; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    mbar_init(&s_full[0], 1);
    mbar_init(&s_full[1], 1);
    mbar_init(&p_full[0], 256);
    mbar_init(&p_full[1], 256);
    mbar_init(&pv_done[0], 1);
    mbar_init(&pv_done[1], 1);
    mbar_init(&drain_bar, 1);
    abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 1) tmem_alloc(&tmem_slot, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  const int n = n_tiles;
  volatile int* abort = &abort_flag;

  if (warp == 0) {
    if (lane == 0) {
      mbar_arrive_expect_tx(&q_full, Q_BYTES);
#pragma unroll
      for (int hl = 0; hl < G; ++hl)
#pragma unroll
        for (int c = 0; c < 2; ++c)
          tma_load_3d(base + OFF_Q + c * Q_CHUNK + hl * (QPOS * 128), &tmQ, &q_full, (j * G + hl) * AD + c * 64,
                      p0, b);
      IssuedFills k_fills, v_fills;
      // K tile i+1 is issued before V tile i: K stages free up as soon as their S MMA is done,
      // V stages only after P V, so the K loads run a tile further ahead
      auto load_k = [&](int i) -> bool {
        const int st = i % KV_STAGES;
        if (!mbar_wait(&k_empty[st], ((i / KV_STAGES) & 1) ^ 1, abort)) return false;
        uint8_t* kd = base + OFF_K + st * KV_TILE_BYTES;
        const int t0 = tiles[i] * KT;
        mbar_arrive_expect_tx(&k_full[st], KV_TILE_BYTES);
        tma_load_3d(kd, &tmK, &k_full[st], j * AD, t0, b);
        tma_load_3d(kd + KV_CHUNK, &tmK, &k_full[st], j * AD + 64, t0, b);
        k_fills.note(st, (i / KV_STAGES) & 1);
        return true;
      };
      auto load_v = [&](int i) -> bool {
        const int st = i % KV_STAGES;
        if (!mbar_wait(&v_empty[st], ((i / KV_STAGES) & 1) ^ 1, abort)) return false;
        uint8_t* vd = base + OFF_V + st * KV_TILE_BYTES;
        const int t0 = tiles[i] * KT;
        mbar_arrive_expect_tx(&v_full[st], KV_TILE_BYTES);
        tma_load_3d(vd, &tmV, &v_full[st], j * AD, t0, b);
        tma_load_3d(vd + KV_CHUNK, &tmV, &v_full[st], j * AD + 64, t0, b);
        v_fills.note(st, (i / KV_STAGES) & 1);
        return true;
      };
      if (n > 0 && load_k(0)) {
        for (int i = 0; i < n; ++i) {
          if (i + 1 < n && !load_k(i + 1)) break;
          if (!load_v(i)) break;
        }
      }
      if (*abort) {  // a wait expired: let the copies this thread issued land before the CTA exits
        mbar_wait_drain(&q_full, 0);
        k_fills.drain(k_full, KV_STAGES);
        v_fills.drain(v_full, KV_STAGES);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // Shared-memory descriptors differ only in the start-address field (bits 0..13, in
      // 16-byte units), so each is a base descriptor plus a constant offset: the single issuing
      // thread then spends almost no instructions between a barrier and its MMAs.
      const uint64_t dq0 = smem_desc_sw128(smem_u32(base + OFF_Q), 16, 1024);
      const uint64_t dk0 = smem_desc_sw128(smem_u32(base + OFF_K), 16, 1024);
      const uint64_t dv0 = smem_desc_sw128(smem_u32(base + OFF_V), KV_CHUNK, 1024);
      bool issued = false;
      auto issue_pv = [&](int i) -> bool {
        // O += P_i V_i : A = P_i in TMEM (bf16 pairs over its scores), B = V (MN-major)
        const int st = i % KV_STAGES;
        // P_i and V_i: both tests go out together (the V load has usually landed long before)
        if (!mbar_wait2(&p_full[i & 1], (i >> 1) & 1, &v_full[st], (i / KV_STAGES) & 1, abort)) return false;
        tc_fence_after();
        const uint64_t dv = dv0 + (uint64_t)(st * (KV_TILE_BYTES >> 4));
        const uint32_t pt = tmem + (i & 1) * KT;
#pragma unroll
        for (int kk = 0; kk < KT / 16; ++kk)
          tc_mma_bf16_ts(tmem + O_COL, pt + kk * 8, dv + (uint64_t)(kk * 16 * 128 >> 4), IDESC_PV,
                         (i > 0 || kk > 0) ? 1u : 0u);
        tc_commit(&pv_done[i & 1]);
        tc_commit(&v_empty[st]);
        return true;
      };
      if (mbar_wait(&q_full, 0, abort)) {
        for (int i = 0; i < n; ++i) {
          const int st = i % KV_STAGES;
          if (!mbar_wait(&k_full[st], (i / KV_STAGES) & 1, abort)) break;
          tc_fence_after();
          const uint64_t dk = dk0 + (uint64_t)(st * (KV_TILE_BYTES >> 4));
          const uint32_t d_s = tmem + (i & 1) * KT;
#pragma unroll
          for (int kk = 0; kk < AD / 16; ++kk) {
            const uint32_t qo = (kk >> 2) * Q_CHUNK + (kk & 3) * 32;
            const uint32_t ko = (kk >> 2) * KV_CHUNK + (kk & 3) * 32;
            tc_mma_bf16(d_s, dq0 + (uint64_t)(qo >> 4), dk + (uint64_t)(ko >> 4), IDESC_QK, kk > 0 ? 1u : 0u);
          }
          issued = true;
          tc_commit(&s_full[i & 1]);
          tc_commit(&k_empty[st]);
          if (i >= 1 && !issue_pv(i - 1)) break;
        }
        if (!*abort && n > 0) issue_pv(n - 1);
      }
      if (*abort && issued) {
        tc_commit(&drain_bar);
        unsigned long long t0 = globaltimer_ns();
        while (!mbar_try_wait(&drain_bar, 0) && globaltimer_ns() - t0 < WAIT_LIMIT_NS) {
        }
      }
    }
  } else {
    // ---- softmax warps 2..9. Warps w and w + 4 share TMEM lane quarter w & 3; warp w takes its
    // first 16 lanes, w + 4 the last 16. Within a warp, threads t and t + 16 hold the same row
    // (tile row r holds head j*G + r / QPOS at position p0 + r % QPOS) and split its 64 scores:
    // half 0 takes keys [0, 32) of the tile, half 1 keys [32, 64). The two halves meet by warp
    // shuffle: the row max, the rescale decision and the final row sum need no shared memory and
    // no barrier, and each thread keeps its half of the row's output columns.
    const int quarter = warp & 3;
    const int sub = (warp - 2) >> 2;
    const int half = lane >> 4;
    const int r = quarter * 32 + sub * 16 + (lane & 15);
    const uint32_t lane_off = (uint32_t)(quarter * 32 + sub * 16) << 16;
    const float sl2 = p.scale_log2;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    int row_kend = p.S;
    if constexpr (PREFIX) {
      const int q = p0 + r % QPOS;
      row_kend = q < p.Sq ? min(max(p.key_end[q], p.q_off + q + 1), p.S) : p.S;
    }
    constexpr int HK = KT / 2;  // scores per thread and tile
    for (int i = 0; i < n && ok; ++i) {
      const int sb = i & 1;
      // waits are made warp-uniform: the shuffles below need every lane
      if (!__all_sync(0xffffffffu, mbar_wait(&s_full[sb], (i >> 1) & 1, abort))) { ok = false; break; }
      tc_fence_after();
      const int t0 = tiles[i] * KT;
      const int k0 = t0 + half * HK;  // first key of this thread's half
      const uint32_t sbase = tmem + lane_off + sb * KT;
      float v[HK];
      tmem_ld32_pair<HK>(sbase, v);
      if ((t0 < p.T && p.text_mask) || (t0 + KT > p.S)) {  // warp-uniform: only partial tiles mask
        const uint32_t vm0 = __ballot_sync(0xffffffffu, key_valid(p, b, t0 + lane));
        const uint32_t vm1 = __ballot_sync(0xffffffffu, key_valid(p, b, t0 + HK + lane));
        const uint32_t vm = half ? vm1 : vm0;
#pragma unroll
        for (int e = 0; e < HK; ++e)
          if (!((vm >> e) & 1u)) v[e] = -INFINITY;
      }
      if constexpr (PREFIX) {
        if (t0 + KT > cta_kmin) {  // warp-uniform; each row then cuts at its own key_end
          const int lim = row_kend - k0;
#pragma unroll
          for (int e = 0; e < HK; ++e)
            if (e >= lim) v[e] = -INFINITY;
        }
      }
      // half-row max: chain k takes v[k], v[k+4], ..., v[k+28] with three-input maxes; the
      // other half's max comes from lane t ^ 16
      static_assert(HK == 32, "the max chains below cover 32 scores");
      float m4[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        float a = v[k];
#pragma unroll
        for (int t = 1; t < 7; t += 2) a = fmax3(a, v[k + 4 * t], v[k + 4 * t + 4]);
        m4[k] = fmaxf(a, v[k + 28]);
      }
      const float hm = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
      const float mx = fmaxf(hm, __shfl_xor_sync(0xffffffffu, hm, 16));
      const float mnew = fmaxf(m, mx * sl2);
      const bool grow = mnew > m + 8.0f;  // m = -inf on the first tile
      float alpha = 1.f;
      const bool any_grow = __any_sync(0xffffffffu, grow);
      if (grow) {
        alpha = ex2(m - mnew);  // 0 on the first tile
        m = mnew;
      }
      uint32_t pk[HK / 2];
      const float rs = exp_tile<HK>(v, sl2, m == -INFINITY ? 0.f : m, pk);
      l = l * alpha + rs;
      // P_i (bf16 pairs) over the tile's first 32 columns: half 0 writes columns [0, 16), half 1
      // [16, 32). They overlay scores of this warp's own rows only, all read by the load above.
      tmem_st16_pair<HK / 2>(sbase, pk);
      if (i >= 1 && any_grow) {
        // O must hold P_{i-1} V_{i-1} before it is rescaled. PV_{i-1} is the ((i-1)/2)-th
        // commit on pv_done[(i-1) & 1]; s_full_i already implies PV_{i-2} and earlier are
        // done, and PV_{i+1} needs this tile's P, so the parity below names exactly that phase.
        if (!__all_sync(0xffffffffu, mbar_wait(&pv_done[(i - 1) & 1], ((i - 1) >> 1) & 1, abort))) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < AD / 64; ++c) {
          float o[32];
          const uint32_t oa = tmem + lane_off + O_COL + c * 32;  // half 1: 64 columns further on
          tmem_ld32_pair<AD / 2>(oa, o);
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] *= alpha;
          tmem_st32_pair<AD / 2>(oa, o);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&p_full[i & 1]);
    }
    const int pos = p0 + r % QPOS;
    const int h = j * G + r / QPOS;
    if (ok && n == 0) {
      // a batch row without any valid key (possible only without image tokens): zeros
      if (pos < p.Sq) {
        uint4* op = reinterpret_cast<uint4*>(p.out + ((long)b * p.Sq + pos) * p.HD + h * AD + half * (AD / 2));
#pragma unroll
        for (int q = 0; q < AD / 16; ++q) op[q] = make_uint4(0u, 0u, 0u, 0u);
      }
    } else if (ok) {
      // the output needs the last P V in O
      ok = __all_sync(0xffffffffu, mbar_wait(&pv_done[(n - 1) & 1], ((n - 1) >> 1) & 1, abort));
      if (ok) tc_fence_after();
    }
    const float lt = l + __shfl_xor_sync(0xffffffffu, l, 16);  // both halves' row sums
    if (ok && n > 0) {
      const bool row_ok = pos < p.Sq;
      const long grow_idx = (long)b * p.Sq + pos;
      const float inv_l = lt > 0.f ? 1.f / lt : 0.f;  // a row with no readable key: zeros
#pragma unroll 1
      for (int c = 0; c < AD / 64; ++c) {
        const int col = half * (AD / 2) + c * 32;
        float o[32];
        tmem_ld32_pair<AD / 2>(tmem + lane_off + O_COL + c * 32, o);
        if (row_ok) {
          const uint4* gp = reinterpret_cast<const uint4*>(p.gate + grow_idx * p.g_stride + h * AD + col);
          uint4* op = reinterpret_cast<uint4*>(p.out + grow_idx * p.HD + h * AD + col);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint4 gv = __ldg(gp + q);
            const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
            uint32_t ow[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float a = o[q * 8 + 2 * e] * inv_l * sigmoid_f(bf16_lo(gw[e]));
              const float bb = o[q * 8 + 2 * e + 1] * inv_l * sigmoid_f(bf16_hi(gw[e]));
              ow[e] = pack_bf16x2(a, bb);
            }
            op[q] = make_uint4(ow[0], ow[1], ow[2], ow[3]);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// One warp normalises one 128-wide head (RMSNorm over head_dim with weight (1 + w), page §四.3)
// and rotates it by the position's RoPE angles (adjacent pairs); each lane holds 4 columns.
__device__ __forceinline__ uint2 norm_rope_head(const __nv_bfloat16* x, const float* w, const float* cs,
                                               const float* sn, int pos, float eps, int lane) {
  const uint2 raw = *reinterpret_cast<const uint2*>(x + lane * 4);
  float v[4] = {bf16_lo(raw.x), bf16_hi(raw.x), bf16_lo(raw.y), bf16_hi(raw.y)};
  const float ss = warp_sum(v[0] * v[0] + v[1] * v[1] + v[2] * v[2] + v[3] * v[3]);
  const float r = rsqrtf(ss / (float)AD + eps);
#pragma unroll
  for (int e = 0; e < 4; ++e) v[e] *= r * (1.f + w[lane * 4 + e]);
  const float c0 = cs[(long)pos * (AD / 2) + lane * 2], s0 = sn[(long)pos * (AD / 2) + lane * 2];
  const float c1 = cs[(long)pos * (AD / 2) + lane * 2 + 1], s1 = sn[(long)pos * (AD / 2) + lane * 2 + 1];
  uint2 o;
  o.x = pack_bf16x2(v[0] * c0 - v[1] * s0, v[1] * c0 + v[0] * s0);
  o.y = pack_bf16x2(v[2] * c1 - v[3] * s1, v[3] * c1 + v[2] * s1);
  return o;
}

// Raw projection -> RMS-normalised, rotated q and k (bf16), one warp per (row, head).
// dst row layout: [q heads (H*D) | k heads (Hkv*D)]; Hkv = 0 prepares q only.
__global__ void __launch_bounds__(256) qk_prep_kernel(const __nv_bfloat16* __restrict__ src, long long src_stride,
                                                      int S, int H, int Hkv, float eps,
                                                      const float* __restrict__ qw, const float* __restrict__ kw,
                                                      const float* __restrict__ cs, const float* __restrict__ sn,
                                                      long rows, __nv_bfloat16* __restrict__ dst) {
  const long gw = (long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const int heads = H + Hkv;
  if (gw >= rows * heads) return;
  const long row = gw / heads;
  const int hh = (int)(gw % heads);
  const int pos = (int)(row % S);
  const uint2 o = norm_rope_head(src + row * src_stride + (long)hh * AD, hh < H ? qw : kw, cs, sn, pos, eps, lane);
  *reinterpret_cast<uint2*>(dst + row * (long)(heads * AD) + (long)hh * AD + lane * 4) = o;
}

// Keys and values of n new tokens into a key/value cache, one warp per (token, KV head): k is
// normalised and rotated like the attention's keys, v is copied as projected. Token i of batch
// row b lands in cache row b * capacity + row0 + i.
__global__ void __launch_bounds__(256) kv_append_kernel(const __nv_bfloat16* __restrict__ src, long long src_stride,
                                                        int n, int H, int Hkv, float eps,
                                                        const float* __restrict__ kw, const float* __restrict__ cs,
                                                        const float* __restrict__ sn, long rows,
                                                        __nv_bfloat16* __restrict__ kc, __nv_bfloat16* __restrict__ vc,
                                                        int row0, int capacity) {
  const long gw = (long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (gw >= rows * Hkv) return;
  const long row = gw / Hkv;
  const int hh = (int)(gw % Hkv);
  const int i = (int)(row % n);
  const long drow = (row / n) * capacity + row0 + i;
  const __nv_bfloat16* x = src + row * src_stride;
  const uint2 ko = norm_rope_head(x + (long)(H + hh) * AD, kw, cs, sn, i, eps, lane);
  const uint2 vo = *reinterpret_cast<const uint2*>(x + (long)(H + Hkv + hh) * AD + lane * 4);
  const long d = drow * (long)(Hkv * AD) + (long)hh * AD + lane * 4;
  *reinterpret_cast<uint2*>(kc + d) = ko;
  *reinterpret_cast<uint2*>(vc + d) = vo;
}

}  // namespace

KREA2_DEFINE_ERROR_READER(take_device_error_attention)

namespace {
// One thread waits, with the given limit, on an mbarrier that nothing arrives on: the bounded
// wait must expire, record the timeout in the device error word and let the kernel return.
__global__ void wait_timeout_selftest_kernel(unsigned long long limit_ns, int* waited) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
    const bool ok = mbar_wait(&bar, 0, &abort_flag, limit_ns);
    *waited = ok ? 0 : 1;
  }
}
}  // namespace

int launch_wait_timeout_selftest(unsigned long long limit_ns, int* waited, cudaStream_t stream) {
  wait_timeout_selftest_kernel<<<1, 32, 0, stream>>>(limit_ns, waited);
  count_launch();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(KREA2_ERR_CUDA, "self-test launch failed: %s", cudaGetErrorString(e));
  return KREA2_OK;
}

bool attention_tc_supported(int D, int H, int Hkv) {
  if (D != AD || Hkv <= 0 || H % Hkv) return false;
  const int g = H / Hkv;
  return g == 1 || g == 2 || g == 4;
}

namespace {
template <int G, bool PREFIX>
int launch_attention_g(const AttnTcArgs& a, cudaStream_t stream) {
  constexpr int QPOS = 128 / G;
  static std::atomic<uint64_t> attr_done{0};
  const uint64_t dev_bit = device_bit();
  if (!(attr_done.load(std::memory_order_acquire) & dev_bit) || !dev_bit) {
    if (cudaFuncSetAttribute(attn_gqa_tc_kernel<G, PREFIX>, cudaFuncAttributeMaxDynamicSharedMemorySize, ATT_SMEM) !=
            cudaSuccess ||
        cudaFuncSetAttribute(attn_gqa_tc_kernel<G, PREFIX>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared) != cudaSuccess)
      return set_error(KREA2_ERR_CUDA, "cudaFuncSetAttribute(attention) failed");
    attr_done.fetch_or(dev_bit, std::memory_order_release);
  }
  const int S = a.T + a.N;
  const int Sq = a.Sq > 0 ? a.Sq : S;
  const long long kv_rows = a.kv_batch_rows > 0 ? a.kv_batch_rows : S;
  if ((S + KT - 1) / KT > MAX_TILES) return set_error(KREA2_ERR_UNSUPPORTED, "sequence longer than %d", MAX_TILES * KT);
  if (Sq > S || a.q_off < 0 || a.q_off + Sq > S)
    return set_error(KREA2_ERR_ARG, "query rows [%d, %d) lie outside the %d keys", a.q_off, a.q_off + Sq, S);
  CUtensorMap tq, tk, tv;
  int rc;
  if ((rc = make_tmap_bf16_3d(&tq, a.q, (uint64_t)a.H * AD, Sq, a.B, a.q_stride, 64, QPOS, Sq))) return rc;
  if ((rc = make_tmap_bf16_3d(&tk, a.k, (uint64_t)a.Hkv * AD, S, a.B, a.k_stride, 64, KT, kv_rows))) return rc;
  if ((rc = make_tmap_bf16_3d(&tv, a.v, (uint64_t)a.Hkv * AD, S, a.B, a.v_stride, 64, KT, kv_rows))) return rc;
  AttnCore p{};
  p.B = a.B; p.T = a.T; p.N = a.N; p.S = S; p.Hkv = a.Hkv; p.HD = a.H * AD;
  p.Sq = Sq; p.q_off = a.q_off;
  p.text_mask = a.text_mask;
  p.gate = reinterpret_cast<const __nv_bfloat16*>(a.g);
  p.g_stride = a.g_stride;
  p.out = reinterpret_cast<__nv_bfloat16*>(a.out);
  p.scale_log2 = 1.4426950408889634f / sqrtf((float)AD);
  p.key_end = a.key_end;
  dim3 grid((Sq + QPOS - 1) / QPOS, a.Hkv, a.B);
  attn_gqa_tc_kernel<G, PREFIX><<<grid, ATT_THREADS, ATT_SMEM, stream>>>(tq, tk, tv, p);
  count_launch();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(KREA2_ERR_CUDA, "attention launch failed: %s", cudaGetErrorString(e));
  return KREA2_OK;
}
}  // namespace

int attention_tc_core(const AttnTcArgs& a, cudaStream_t stream) {
  if (!attention_tc_supported(AD, a.H, a.Hkv)) return set_error(KREA2_ERR_UNSUPPORTED, "attention group size");
  if (a.key_end) {
    switch (a.H / a.Hkv) {
      case 1: return launch_attention_g<1, true>(a, stream);
      case 2: return launch_attention_g<2, true>(a, stream);
      default: return launch_attention_g<4, true>(a, stream);
    }
  }
  switch (a.H / a.Hkv) {
    case 1: return launch_attention_g<1, false>(a, stream);
    case 2: return launch_attention_g<2, false>(a, stream);
    default: return launch_attention_g<4, false>(a, stream);
  }
}

int launch_kv_append(const void* qkvg, long long stride, int B, int n, int H, int Hkv, float eps, const float* kw,
                     const float* cs, const float* sn, void* k_cache, void* v_cache, int row0, int capacity,
                     cudaStream_t stream) {
  const long rows = (long)B * n;
  const long warps = rows * Hkv;
  kv_append_kernel<<<(unsigned)((warps + 7) / 8), 256, 0, stream>>>(
      reinterpret_cast<const __nv_bfloat16*>(qkvg), stride, n, H, Hkv, eps, kw, cs, sn, rows,
      reinterpret_cast<__nv_bfloat16*>(k_cache), reinterpret_cast<__nv_bfloat16*>(v_cache), row0, capacity);
  count_launch();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(KREA2_ERR_CUDA, "kv_append launch failed: %s", cudaGetErrorString(e));
  return KREA2_OK;
}

int launch_qk_prep(const void* qkvg, long long stride, int B, int S, int H, int Hkv, float eps, const float* qw,
                   const float* kw, const float* cs, const float* sn, void* dst, cudaStream_t stream) {
  const long rows = (long)B * S;
  const long warps = rows * (H + Hkv);
  qk_prep_kernel<<<(unsigned)((warps + 7) / 8), 256, 0, stream>>>(
      reinterpret_cast<const __nv_bfloat16*>(qkvg), stride, S, H, Hkv, eps, qw, kw, cs, sn, rows,
      reinterpret_cast<__nv_bfloat16*>(dst));
  count_launch();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(KREA2_ERR_CUDA, "qk_prep launch failed: %s", cudaGetErrorString(e));
  return KREA2_OK;
}

}  // namespace krea2
