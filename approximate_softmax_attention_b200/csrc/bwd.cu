// bwd.cu -- backward of the fused attention for the exact map and K-interval
// attention ("Pretraining Transformers with Quantized Softmax in Attention",
// abstract: backward rules including calibration derivatives, and a
// straight-through surrogate placed before or after normalization).
//
// Rules (integer decisions of the forward frozen; gw_j = dL/dw_j =
// (dp_j - delta)/Z with dp_j = dO.v_j, delta = dO.O):
//   none  ds_j = gw_j dF/ds_j        (interpolation: slope/Delta; hard: 0)
//   pre   ds_j = gw_j exp(s_j - hi)  (w's own-score derivative taken as exp's)
//   post  ds_j = p*_j (dp_j - delta*), p* = softmax(s), delta* = sum p* dp
//   calibration (unless detached): dhi = sum_j gw_j dF_j/dhi and
//   dlo = sum_j gw_j dF_j/dlo, which belong to ds at the row's argmax /
//   argmin; they are applied as fp32 rank-one updates.
//   dQ = c dS K, dK = c dS^T Q, dV = P^T dO.
//
// Kernels, in launch order on the caller's stream:
//   1. qsm_bwd_delta      delta_r = dO_r . O_r (one warp per row)
//   2. qsm_bwd_rows       one thread per (query row, column quarter) sweeps
//                         S = Q K^T and dP = dO V^T tiles (tcgen05) and
//                         accumulates dhi, dlo and, for the post surrogate,
//                         LSE* and delta* online; the quarters merge at the
//                         end (only run when one of them is needed)
//   3. qsm_bwd_calib      one warp per row: the calibration terms, rank one
//                         per row, in fp32: dQ_r += c (dhi k_argmax + dlo
//                         k_argmin), dKcal[argmax] += c dhi q_r, dKcal[argmin]
//                         += c dlo q_r (kept out of the bf16 dS operand)
//   4. qsm_bwd_main       one CTA per 128-key tile, one thread per key:
//                         S^T = K Q^T and dP^T = V dO^T in TMEM, P^T and dS^T
//                         written back to TMEM (and dS to shared memory),
//                         dV += P^T dO and dK += dS^T Q accumulated in TMEM,
//                         dQ tile = dS K added to an fp32 workspace; dK
//                         gets dKcal added in fp32 before its bf16 store
//   5. qsm_bwd_dq_convert dQ fp32 -> bf16
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "internal.h"
#include "sm100.cuh"
#include "wmap.cuh"

namespace qsm {

namespace {

// rows and main kernels: warp 0 TMA, warp 1 MMA, warps 4-19 four map groups,
// group g owning columns 32g .. 32g+31 of every S / dP (rows) or S^T / dP^T
// (main) tile
constexpr int kMainThreads = 640;
constexpr int kMainMapThreads = 512;
constexpr uint32_t kBwdTmemCols = 512;
constexpr int kRowWs = 8;               // floats per row in the row workspace
enum RowWs { RW_DELTA = 0, RW_DHI = 1, RW_DLO = 2, RW_LSESTAR = 3, RW_DELTASTAR = 4 };

struct BwdParams {
  int S, nqt, nkvt;
  int causal;
  int map;          // 0 exact, 2 K-interval hard, 3 K-interval interp
  int K, fixed_window, flush, surrogate, detach;
  float c, cL2E, window;
  const float *LSE, *hi, *lo;
  const int32_t *amax, *amin;
  float *rowws;
  float *dqacc;
  float *dkcal;     // [rows][D] fp32 calibration part of dK (nullptr: none)
  __nv_bfloat16 *dK, *dV;
  int32_t *status;
  uint32_t tab_off, cst_off, ds_off, bar_off;
};

constexpr int MAPB_EXACT = 0, MAPB_HARD = 2, MAPB_INTERP = 3;

template <int D>
struct BGeo {
  static constexpr int TILE_BYTES = 128 * D * 2;        // bf16 tile of 128 rows
  static constexpr int CHUNKS = (D * 2) / 128;
  static constexpr int EPC = 64;                        // bf16 per 128-byte row
  static constexpr int CHUNK_BYTES = 128 * 128;
  static constexpr int KSTEPS_D = D / 16;               // k-steps over D
  static constexpr int KSTEPS_N = 128 / 16;             // k-steps over a 128 tile
  static constexpr uint32_t IDESC_SS = instr_desc(1, false, 128, 128);
  static constexpr uint32_t IDESC_TS = instr_desc(1, true, 128, D);
  static constexpr uint32_t IDESC_DQ = instr_desc(1, true, 128, D, true);
};

__device__ __forceinline__ bool warp_all_b(bool x) { return __all_sync(0xffffffffu, x); }

// S or dP tile = A B^T over D with both operands K-major in shared memory.
template <int D>
__device__ __forceinline__ void mma_nt(uint32_t d_tmem, uint32_t a_saddr, uint32_t b_saddr) {
  using G = BGeo<D>;
#pragma unroll
  for (int kk = 0; kk < G::KSTEPS_D; ++kk) {
    const int e = kk * 16;
    const uint32_t off = (e / G::EPC) * G::CHUNK_BYTES + (e % G::EPC) * 2;
    mma_ss_f16(d_tmem, smem_desc(a_saddr + off, 16, 1024), smem_desc(b_saddr + off, 16, 1024),
               G::IDESC_SS, kk > 0);
  }
}

// acc (+)= A[tmem, 128 x 128, group layout] B[smem, 128 x D, MN-major]: the
// bf16 values of K-columns 32g .. 32g+31 of A sit in TMEM columns 32g ..
// 32g+15 (each map group writes its P^T / dS^T into the first half of its own
// S^T / dP^T columns), 8 TMEM columns per k-step of 16.
template <int D>
__device__ __forceinline__ void mma_tn_grouped(uint32_t d_tmem, uint32_t a_tmem,
                                               uint32_t b_saddr, bool acc) {
  using G = BGeo<D>;
#pragma unroll
  for (int kk = 0; kk < G::KSTEPS_N; ++kk)
    mma_ts_f16(d_tmem, a_tmem + 32 * (kk >> 1) + 8 * (kk & 1),
               smem_desc(b_saddr + kk * 16 * 128, G::CHUNK_BYTES, 1024), G::IDESC_TS,
               (acc || kk > 0) ? 1u : 0u);
}

// D = A[smem 128 x 128, MN-major] B[smem 128 x D, MN-major]
template <int D>
__device__ __forceinline__ void mma_mn_mn(uint32_t d_tmem, uint32_t a_saddr, uint32_t b_saddr) {
  using G = BGeo<D>;
#pragma unroll
  for (int kk = 0; kk < G::KSTEPS_N; ++kk)
    mma_ss_f16(d_tmem, smem_desc(a_saddr + kk * 16 * 128, G::CHUNK_BYTES, 1024),
               smem_desc(b_saddr + kk * 16 * 128, G::CHUNK_BYTES, 1024), G::IDESC_DQ, kk > 0);
}

// --------------------------------------------------------------- delta
__global__ void __launch_bounds__(256) qsm_bwd_delta(const __nv_bfloat16 *__restrict__ O,
                                                     const __nv_bfloat16 *__restrict__ dO,
                                                     float *__restrict__ rowws, long long rows,
                                                     int D) {
  const long long r = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  float acc = 0.0f;
  for (int d = lane * 2; d < D; d += 64) {
    const __nv_bfloat162 o = *reinterpret_cast<const __nv_bfloat162 *>(O + r * D + d);
    const __nv_bfloat162 g = *reinterpret_cast<const __nv_bfloat162 *>(dO + r * D + d);
    acc = fmaf(__bfloat162float(o.x), __bfloat162float(g.x), acc);
    acc = fmaf(__bfloat162float(o.y), __bfloat162float(g.y), acc);
  }
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) {
    float *w = rowws + r * kRowWs;
    w[RW_DELTA] = acc;
    w[RW_DHI] = 0.0f;
    w[RW_DLO] = 0.0f;
    w[RW_LSESTAR] = 0.0f;
    w[RW_DELTASTAR] = 0.0f;
  }
}

// ----------------------------------------------------------- dQ convert
__global__ void __launch_bounds__(256) qsm_bwd_dq_convert(const float *__restrict__ acc,
                                                          __nv_bfloat16 *__restrict__ dQ,
                                                          long long n) {
  const long long i = (static_cast<long long>(blockIdx.x) * 256 + threadIdx.x) * 4;
  if (i >= n) return;
  const float4 v = *reinterpret_cast<const float4 *>(acc + i);
  __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y);
  __nv_bfloat162 b = __floats2bfloat162_rn(v.z, v.w);
  uint2 out;
  out.x = *reinterpret_cast<uint32_t *>(&a);
  out.y = *reinterpret_cast<uint32_t *>(&b);
  *reinterpret_cast<uint2 *>(dQ + i) = out;
}

// ------------------------------------------------- calibration scatter
__global__ void __launch_bounds__(256) qsm_bwd_calib(const __nv_bfloat16 *__restrict__ Q,
                                                     const __nv_bfloat16 *__restrict__ K,
                                                     const float *__restrict__ rowws,
                                                     const int32_t *__restrict__ amax,
                                                     const int32_t *__restrict__ amin,
                                                     float *__restrict__ dqacc,
                                                     float *__restrict__ dkcal, int S, int D,
                                                     long long rows, float c) {
  const long long r = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  const long long head = r / S;                    // rows of one (b, h) are contiguous
  const float dhi = c * rowws[r * kRowWs + RW_DHI];
  const float dlo = c * rowws[r * kRowWs + RW_DLO];
  const long long ja = head * S + amax[r];
  const long long jb = head * S + amin[r];
  for (int d = lane; d < D; d += 32) {
    const float q = __bfloat162float(Q[r * D + d]);
    dqacc[r * D + d] += dhi * __bfloat162float(K[ja * D + d]) + dlo * __bfloat162float(K[jb * D + d]);
    atomicAdd(dkcal + ja * D + d, dhi * q);
    atomicAdd(dkcal + jb * D + d, dlo * q);
  }
}

struct RowBars {
  uint64_t *kv_full, *kv_empty;   // [ns]
  uint64_t *q_full;
  uint64_t *sd_full, *sd_empty;   // [2]
  uint64_t *drain;
  uint64_t *tab_ready, *part_ready;   // single use: grid table built; partial sums written
  uint32_t *tmem_slot;
  int *abort;
};

// --------------------------------------------------------------- rows
// One CTA per 128 query rows of one (b, h); four map groups, thread = row,
// group g taking columns 32g .. 32g+31 of every S / dP tile.  Computes the
// calibration derivatives dhi, dlo and (post surrogate) LSE*, delta*.
template <int D, int MAP>
__global__ void __launch_bounds__(kMainThreads, 1)
    qsm_bwd_rows(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                 const BwdParams p) {
  using G = BGeo<D>;
  constexpr int NS = 4;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y;
  const int qt = blockIdx.x;
  uint8_t *sQ = smem;
  uint8_t *sdO = smem + G::TILE_BYTES;
  uint8_t *sKV = smem + 2 * G::TILE_BYTES;
  float2 *tab = reinterpret_cast<float2 *>(smem + p.tab_off);
  uint64_t *bp = reinterpret_cast<uint64_t *>(smem + p.bar_off);
  RowBars bars;
  bars.kv_full = bp;
  bars.kv_empty = bp + NS;
  bars.q_full = bp + 2 * NS;
  bars.sd_full = bars.q_full + 1;
  bars.sd_empty = bars.sd_full + 2;
  bars.drain = bars.sd_empty + 2;
  bars.tab_ready = bars.drain + 1;
  bars.part_ready = bars.tab_ready + 1;
  bars.tmem_slot = reinterpret_cast<uint32_t *>(bars.part_ready + 1);
  // per-row partial sums of the four groups: dhi, dlo, m*, l*, a* ([5][4][128])
  float *part = reinterpret_cast<float *>(smem + p.cst_off);
  bars.abort = reinterpret_cast<int *>(bars.tmem_slot + 1);
  volatile int *abort = bars.abort;
  const int nkv = p.causal ? min(p.nkvt, qt + 1) : p.nkvt;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(&bars.kv_full[i], 1);
      mbar_init(&bars.kv_empty[i], 1);
    }
    mbar_init(bars.q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.sd_full[i], 1);
      mbar_init(&bars.sd_empty[i], kMainMapThreads);
    }
    mbar_init(bars.drain, 1);
    mbar_init(bars.tab_ready, kMainMapThreads);
    mbar_init(bars.part_ready, kMainMapThreads);
    *bars.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(bars.tmem_slot, kBwdTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *bars.tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      mbar_expect_tx(bars.q_full, 2 * G::TILE_BYTES);
      for (int ch = 0; ch < G::CHUNKS; ++ch) {
        tma_load_3d(sQ + ch * G::CHUNK_BYTES, &tmQ, bars.q_full, ch * G::EPC, qt * 128, bh);
        tma_load_3d(sdO + ch * G::CHUNK_BYTES, &tmdO, bars.q_full, ch * G::EPC, qt * 128, bh);
      }
      int it = 0;
      bool ok = true;
      for (int j = 0; j < nkv && ok; ++j) {
        for (int w = 0; w < 2 && ok; ++w) {
          const int st = it % NS;
          if (it >= NS) ok = mbar_wait(&bars.kv_empty[st], ((it / NS) & 1) ^ 1, abort);
          if (!ok) break;
          mbar_expect_tx(&bars.kv_full[st], G::TILE_BYTES);
          for (int ch = 0; ch < G::CHUNKS; ++ch)
            tma_load_3d(sKV + st * G::TILE_BYTES + ch * G::CHUNK_BYTES, w ? &tmV : &tmK,
                        &bars.kv_full[st], ch * G::EPC, j * 128, bh);
          ++it;
        }
      }
      mbar_wait(bars.q_full, 0, abort);
      for (int st = 0; st < NS && st < it; ++st)
        mbar_wait(&bars.kv_full[st], (((it - st + NS - 1) / NS) - 1) & 1, abort);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      bool ok = mbar_wait(bars.q_full, 0, abort);
      tc_fence_after();
      int it = 0;
      const uint32_t qa = smem_u32(sQ), da = smem_u32(sdO), kva = smem_u32(sKV);
      for (int j = 0; j < nkv && ok; ++j) {
        const int b = j & 1, use = j >> 1;
        if (use >= 1) {
          ok = mbar_wait(&bars.sd_empty[b], (use - 1) & 1, abort);
          if (!ok) break;
          tc_fence_after();
        }
        const int ks = it % NS;
        ok = mbar_wait(&bars.kv_full[ks], (it / NS) & 1, abort);
        ++it;
        const int vs = it % NS;
        ok = ok && mbar_wait(&bars.kv_full[vs], (it / NS) & 1, abort);
        ++it;
        if (!ok) break;
        tc_fence_after();
        mma_nt<D>(tmem + b * 256, qa, kva + ks * G::TILE_BYTES);
        mma_nt<D>(tmem + b * 256 + 128, da, kva + vs * G::TILE_BYTES);
        mma_commit(&bars.sd_full[b]);
        mma_commit(&bars.kv_empty[ks]);
        mma_commit(&bars.kv_empty[vs]);
      }
      mma_commit(bars.drain);
      mbar_wait(bars.drain, 0, abort);
    }
  } else if (warp >= 4) {
    const int g = (warp - 4) >> 2;                       // map group: columns 32g..32g+31
    const int row = (warp & 3) * 32 + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const int qrow = qt * 128 + row;
    const bool row_ok = qrow < p.S;
    const int L = p.causal ? min(qrow + 1, p.S) : p.S;
    const size_t ri = static_cast<size_t>(bh) * p.S + min(qrow, p.S - 1);
    const float delta = p.rowws[ri * kRowWs + RW_DELTA];
    const float hi = p.hi[ri];
    const float lo_in = p.lo[ri];
    const float Z = expf(p.LSE[ri] - hi);
    const float invZ = 1.0f / Z;
    const RowMap rm = make_rowmap(hi, lo_in, p.K, p.fixed_window != 0, p.window);
    const float a_raw = rm.degenerate ? 0.0f : __fmul_rn(p.c, rm.inv);
    const float b_raw = rm.degenerate ? static_cast<float>(p.K) : rm.b;
    const float Kf = static_cast<float>(p.K);
    const float invK = 1.0f / Kf;
    const float a_s = __fsub_rn(hi, rm.lo);        // hi - lo in score units
    const float inv_a = rm.degenerate ? 0.0f : 1.0f / a_s;
    const float slope_fw = -Kf / p.window;         // fixed window: d(coordinate)/d(hi) per slope
    const bool calib = !p.detach && !rm.degenerate;
    const bool post = p.surrogate == QSM_SURR_POST;
    // this row's grid table column: (g_n, g_{n+1} - g_n), n = 0..K; the four
    // groups build alternate entries
    for (int n = g; n <= p.K; n += 4) {
      const float gk = grid_value(rm, p.K, n);
      const float gk1 = n < p.K ? grid_value(rm, p.K, n + 1) : gk;
      tab[n * 128 + row] = make_float2(gk, __fsub_rn(gk1, gk));
    }
    mbar_arrive(bars.tab_ready);
    bool ok = warp_all_b(mbar_wait(bars.tab_ready, 0, abort));
    float dhi = 0.0f, dlo = 0.0f;
    float mstar = -INFINITY, lstar = 0.0f, astar = 0.0f;
    uint32_t cnt[2] = {0, 0};
    const int c0 = 32 * g;
    for (int j = 0; j < nkv && ok; ++j) {
      const int b = j & 1;
      ok = warp_all_b(mbar_wait(&bars.sd_full[b], cnt[b] & 1, abort));
      ++cnt[b];
      if (!ok) break;
      tc_fence_after();
      const int lim = L - 128 * j - c0;            // valid columns of this group
      uint32_t sv[32], dv[32];
      tmem_ld32(lane_base + b * 256 + c0, sv);
      tmem_ld32(lane_base + b * 256 + 128 + c0, dv);
      tmem_wait_ld();
      reg_fence32(sv);
      reg_fence32(dv);
      // values in registers: hand the buffers back first
      tc_fence_before();
      mbar_arrive(&bars.sd_empty[b]);
      if (post) {
        float cm = -INFINITY;
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (i < lim) cm = fmaxf(cm, __uint_as_float(sv[i]) * p.c);
        if (cm > mstar) {
          const float sc = expf(mstar - cm);
          lstar *= sc;
          astar *= sc;
          mstar = cm;
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          if (i < lim) {
            const float e = expf(__uint_as_float(sv[i]) * p.c - mstar);
            lstar += e;
            astar = fmaf(e, __uint_as_float(dv[i]), astar);
          }
        }
      }
      if (calib && MAP != MAPB_EXACT) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          if (i >= lim) continue;
          const float r = __uint_as_float(sv[i]);
          const float gw = (__uint_as_float(dv[i]) - delta) * invZ;
          const float u = __fmaf_rn(r, a_raw, b_raw);
          const float uc = fminf(fmaxf(u, 0.0f), Kf);
          if (MAP == MAPB_HARD) {
            if (!p.fixed_window) {
              // nearest node from the bits of a magic-number add (no
              // float <-> int conversion on the XU pipe)
              const float tn = __fadd_rn(uc, kMagic);
              const int n = static_cast<int>(__float_as_uint(tn) - kMagicBits);
              const float gv = tab[n * 128 + row].x;
              const float t = gw * (__fsub_rn(tn, kMagic) - Kf) * invK * gv;
              dhi += t;
              dlo -= t;
            }
          } else {
            // floor from a round-down add of 2^23 (exact for 0 <= uc <= K)
            const float tf = __fadd_rd(uc, 8388608.0f);
            const float kf = fminf(__fsub_rn(tf, 8388608.0f), Kf - 1.0f);
            const int k = min(static_cast<int>(__float_as_uint(tf) - 0x4B000000u), p.K - 1);
            const float f = uc - kf;
            const float2 gd = tab[k * 128 + row];
            const float g0 = gd.x, slope = gd.y, g1 = gd.x + gd.y;
            if (!p.fixed_window) {
              const float mix = ((1.0f - f) * (Kf - kf) * g0 + f * (Kf - kf - 1.0f) * g1) * invK;
              dhi += gw * (-slope * uc * inv_a - mix);
              dlo += gw * (-slope * (Kf - uc) * inv_a + mix);
            } else if (u >= 0.0f) {
              dhi += gw * (slope * slope_fw);
            }
          }
        }
      }
    }
    // merge the four groups' partial sums (the online log-sum-exp of the post
    // surrogate rescales each part to the common maximum)
    part[(0 * 4 + g) * 128 + row] = dhi;
    part[(1 * 4 + g) * 128 + row] = dlo;
    part[(2 * 4 + g) * 128 + row] = mstar;
    part[(3 * 4 + g) * 128 + row] = lstar;
    part[(4 * 4 + g) * 128 + row] = astar;
    mbar_arrive(bars.part_ready);
    if (ok) ok = warp_all_b(mbar_wait(bars.part_ready, 0, abort));
    if (ok && row_ok && g == 0) {
      float sdhi = 0.0f, sdlo = 0.0f, M = -INFINITY;
#pragma unroll
      for (int gg = 0; gg < 4; ++gg) {
        sdhi += part[(0 * 4 + gg) * 128 + row];
        sdlo += part[(1 * 4 + gg) * 128 + row];
        M = fmaxf(M, part[(2 * 4 + gg) * 128 + row]);
      }
      float Ls = 0.0f, As = 0.0f;
      if (post) {
#pragma unroll
        for (int gg = 0; gg < 4; ++gg) {
          const float mg = part[(2 * 4 + gg) * 128 + row];
          if (mg == -INFINITY) continue;             // a group with no valid column
          const float sc = expf(mg - M);
          Ls = fmaf(part[(3 * 4 + gg) * 128 + row], sc, Ls);
          As = fmaf(part[(4 * 4 + gg) * 128 + row], sc, As);
        }
      }
      float *w = p.rowws + ri * kRowWs;
      w[RW_DHI] = calib ? sdhi : 0.0f;
      w[RW_DLO] = calib ? sdlo : 0.0f;
      if (post) {
        w[RW_LSESTAR] = M + logf(Ls);
        w[RW_DELTASTAR] = As / Ls;
      }
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kBwdTmemCols);
  if (threadIdx.x == 0 && *bars.abort && p.status != nullptr) atomicExch(p.status, QSM_ERR_TIMEOUT);
}

// --------------------------------------------------------------- main
// Per-query-row record of the main kernel (8 floats, read as two float4):
//   [0] a, [1] b      grid coordinate = fma(r, a, b) (raw accumulator units)
//   [2] 1/Z           K-interval normaliser (exact map: unused)
//   [3] delta         dO . O
//   [4] e             exact: LSE*log2e; pre: hi*log2e; post: LSE* * log2e
//   [5] delta*        post surrogate: sum of softmax(s) dP
//   [6] K / (hi - lo) d(coordinate)/ds
//   [7] unused

struct MainBars {
  uint64_t *kv_full;                // K_j, V_j
  uint64_t *qd_full, *qd_empty;     // [2] Q_i, dO_i stages
  uint64_t *sdp_full, *pds_full;
  uint64_t *dq_full, *dq_empty;
  uint64_t *acc_full, *drain;
  uint64_t *cst_ready;              // map group: this tile's row constants written
  uint32_t *tmem_slot;
  int *abort;
};

// TMEM columns
constexpr uint32_t T_S = 0, T_DP = 128, T_DV = 256;

template <int D, int MAP>
__global__ void __launch_bounds__(kMainThreads, 1)
    qsm_bwd_main(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                 const BwdParams p) {
  using G = BGeo<D>;
  constexpr uint32_t T_DK = T_DV + D, T_DQ = T_DV + 2 * D;
  static_assert(T_DQ + D <= kBwdTmemCols, "TMEM budget");
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y;
  const int kt = blockIdx.x;
  uint8_t *sK = smem;
  uint8_t *sV = smem + G::TILE_BYTES;
  uint8_t *sQD = smem + 2 * G::TILE_BYTES;              // [2 stages][Q, dO]
  uint8_t *sDS = smem + p.ds_off;                        // 128 x 128 bf16, MN-major
  float2 *tab = reinterpret_cast<float2 *>(smem + p.tab_off);   // [row][n]
  float *cst = reinterpret_cast<float *>(smem + p.cst_off);     // [128][8]: one record per row
  uint64_t *bp = reinterpret_cast<uint64_t *>(smem + p.bar_off);
  MainBars bars;
  bars.kv_full = bp;
  bars.qd_full = bp + 1;
  bars.qd_empty = bp + 3;
  bars.sdp_full = bp + 5;
  bars.pds_full = bp + 6;
  bars.dq_full = bp + 7;
  bars.dq_empty = bp + 8;
  bars.acc_full = bp + 9;
  bars.drain = bp + 10;
  bars.cst_ready = bp + 11;
  bars.tmem_slot = reinterpret_cast<uint32_t *>(bp + 12);
  bars.abort = reinterpret_cast<int *>(bars.tmem_slot + 1);
  volatile int *abort = bars.abort;
  const int i0 = p.causal ? kt : 0;                      // first query tile
  const int nq = p.nqt - i0;

  if (threadIdx.x == 0) {
    mbar_init(bars.kv_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.qd_full[i], 1);
      mbar_init(&bars.qd_empty[i], 1);
    }
    mbar_init(bars.sdp_full, 1);
    mbar_init(bars.pds_full, kMainMapThreads);
    mbar_init(bars.dq_full, 1);
    mbar_init(bars.dq_empty, kMainMapThreads);
    mbar_init(bars.acc_full, 1);
    mbar_init(bars.drain, 1);
    mbar_init(bars.cst_ready, kMainMapThreads);
    *bars.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(bars.tmem_slot, kBwdTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *bars.tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      mbar_expect_tx(bars.kv_full, 2 * G::TILE_BYTES);
      for (int ch = 0; ch < G::CHUNKS; ++ch) {
        tma_load_3d(sK + ch * G::CHUNK_BYTES, &tmK, bars.kv_full, ch * G::EPC, kt * 128, bh);
        tma_load_3d(sV + ch * G::CHUNK_BYTES, &tmV, bars.kv_full, ch * G::EPC, kt * 128, bh);
      }
      bool ok = true;
      int issued[2] = {0, 0};
      for (int n = 0; n < nq && ok; ++n) {
        const int st = n & 1;
        if (n >= 2) ok = mbar_wait(&bars.qd_empty[st], ((n >> 1) - 1) & 1, abort);
        if (!ok) break;
        uint8_t *q = sQD + st * 2 * G::TILE_BYTES;
        mbar_expect_tx(&bars.qd_full[st], 2 * G::TILE_BYTES);
        for (int ch = 0; ch < G::CHUNKS; ++ch) {
          tma_load_3d(q + ch * G::CHUNK_BYTES, &tmQ, &bars.qd_full[st], ch * G::EPC,
                      (i0 + n) * 128, bh);
          tma_load_3d(q + G::TILE_BYTES + ch * G::CHUNK_BYTES, &tmdO, &bars.qd_full[st],
                      ch * G::EPC, (i0 + n) * 128, bh);
        }
        ++issued[st];
      }
      mbar_wait(bars.kv_full, 0, abort);
      for (int st = 0; st < 2; ++st)
        if (issued[st] > 0) mbar_wait(&bars.qd_full[st], (issued[st] - 1) & 1, abort);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      bool ok = mbar_wait(bars.kv_full, 0, abort);
      tc_fence_after();
      const uint32_t ka = smem_u32(sK), va = smem_u32(sV), dsa = smem_u32(sDS);
      for (int n = 0; n < nq && ok; ++n) {
        const int st = n & 1;
        ok = mbar_wait(&bars.qd_full[st], (n >> 1) & 1, abort);
        if (!ok) break;
        tc_fence_after();
        const uint32_t qa = smem_u32(sQD + st * 2 * G::TILE_BYTES);
        const uint32_t da = qa + G::TILE_BYTES;
        mma_nt<D>(tmem + T_S, ka, qa);          // S^T  = K Q^T
        mma_nt<D>(tmem + T_DP, va, da);         // dP^T = V dO^T
        mma_commit(bars.sdp_full);
        ok = mbar_wait(bars.pds_full, n & 1, abort);
        if (!ok) break;
        tc_fence_after();
        mma_tn_grouped<D>(tmem + T_DV, tmem + T_S, da, n > 0);    // dV += P^T dO
        mma_tn_grouped<D>(tmem + T_DK, tmem + T_DP, qa, n > 0);   // dK += dS^T Q
        if (n > 0) {
          ok = mbar_wait(bars.dq_empty, (n - 1) & 1, abort);
          if (!ok) break;
          tc_fence_after();
        }
        mma_mn_mn<D>(tmem + T_DQ, dsa, ka);                 // dQ tile = dS K
        mma_commit(bars.dq_full);
        mma_commit(&bars.qd_empty[st]);
      }
      if (ok) mma_commit(bars.acc_full);
      mma_commit(bars.drain);
      mbar_wait(bars.drain, 0, abort);
    }
  } else if (warp >= 4) {
    const int g = (warp - 4) >> 2;                       // map group 0..3
    const int key = (warp & 3) * 32 + (threadIdx.x & 31);  // TMEM lane, key row
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const int kg = kt * 128 + key;
    const bool key_ok = kg < p.S;
    const float Kf = static_cast<float>(p.K);
    const int K1 = p.K + 1;
    const uint32_t ds_base = smem_u32(sDS);
    const int col0 = 32 * g;                             // this group's query columns
    const float4 *cst4 = reinterpret_cast<const float4 *>(cst);
    bool ok = true;
    for (int n = 0; n < nq && ok; ++n) {
      const int qt = i0 + n;
      // ---- per-query-row constants of this tile: thread `key` serves row
      // `key`; group 0 writes the scalars, the groups split the grid table
      {
        const int qg = qt * 128 + key;
        const size_t ri = static_cast<size_t>(bh) * p.S + min(qg, p.S - 1);
        const float *rw = p.rowws + ri * kRowWs;
        const float lse = p.LSE[ri];
        float a = 0.0f, b = 0.0f, invs = 0.0f, e = 0.0f, invz = 0.0f;
        if (MAP == MAPB_EXACT) {
          e = lse * 1.4426950408889634f;
        } else {
          const float hi = p.hi[ri];
          const RowMap rm = make_rowmap(hi, p.lo[ri], p.K, p.fixed_window != 0, p.window);
          a = rm.degenerate ? 0.0f : __fmul_rn(p.c, rm.inv);
          b = rm.degenerate ? Kf : rm.b;
          invs = rm.degenerate ? 0.0f : rm.inv;
          e = (p.surrogate == QSM_SURR_POST) ? rw[RW_LSESTAR] * 1.4426950408889634f
                                             : rm.hiL2E;
          for (int m = g; m <= p.K; m += 4) {
            const float gk = grid_value(rm, p.K, m);
            const float gk1 = m < p.K ? grid_value(rm, p.K, m + 1) : gk;
            tab[key * K1 + m] = make_float2(gk, __fsub_rn(gk1, gk));
          }
          if (g == 0) invz = expf(hi - lse);
        }
        if (g == 0) {
          float4 *c = reinterpret_cast<float4 *>(cst + key * 8);
          c[0] = make_float4(a, b, invz, rw[RW_DELTA]);
          c[1] = make_float4(e, rw[RW_DELTASTAR], invs, 0.0f);
        }
      }
      // every row's constants are in place (a bounded wait, unlike bar.sync)
      mbar_arrive(bars.cst_ready);
      ok = warp_all_b(mbar_wait(bars.cst_ready, n & 1, abort));
      if (!ok) break;
      ok = warp_all_b(mbar_wait(bars.sdp_full, n & 1, abort));
      if (!ok) break;
      tc_fence_after();
      const int qbase = qt * 128;
      const bool full = (qbase + 128 <= p.S) && (kt * 128 + 128 <= p.S) && (!p.causal || qt > kt);
      {
        uint32_t sv[32], dv[32];
        tmem_ld32(lane_base + T_S + col0, sv);
        tmem_ld32(lane_base + T_DP + col0, dv);
        tmem_wait_ld();
        reg_fence32(sv);
        reg_fence32(dv);
        uint32_t pp[16], dd[16];
#pragma unroll
        for (int i2 = 0; i2 < 16; ++i2) {
          float pv2[2], ds2[2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int i = 2 * i2 + h;
            const int col = col0 + i;
            const int qg = qbase + col;
            const bool valid = full || (key_ok && qg < p.S && (!p.causal || kg <= qg));
            const float r = __uint_as_float(sv[i]);
            const float dp = __uint_as_float(dv[i]);
            const float4 c0 = cst4[2 * col], c1 = cst4[2 * col + 1];
            const float delta = c0.w;
            float pw, ds;
            if (MAP == MAPB_EXACT) {
              pw = ex2_approx(__fmaf_rn(r, p.cL2E, -c1.x));
              ds = pw * (dp - delta);
            } else {
              const float invZ = c0.z;
              const float u = __fmaf_rn(r, c0.x, c0.y);
              const float uc = fminf(fmaxf(u, 0.0f), Kf);
              const bool below = p.fixed_window && u < 0.0f;
              float w, slope = 0.0f;
              if (MAP == MAPB_HARD) {
                const int m = static_cast<int>(__float_as_uint(__fadd_rn(uc, kMagic)) - kMagicBits);
                w = tab[col * K1 + m].x;
              } else {
                const float tf = __fadd_rd(uc, 8388608.0f);
                const float kf = fminf(__fsub_rn(tf, 8388608.0f), Kf - 1.0f);
                const int k = min(static_cast<int>(__float_as_uint(tf) - 0x4B000000u), p.K - 1);
                const float2 gd = tab[col * K1 + k];
                w = __fmaf_rn(__fsub_rn(uc, kf), gd.y, gd.x);
                slope = gd.y;
              }
              if (below && p.flush) w = 0.0f;
              pw = w * invZ;
              const float gw = (dp - delta) * invZ;
              if (p.surrogate == QSM_SURR_NONE) {
                ds = (MAP == MAPB_INTERP && !below) ? gw * slope * c1.z : 0.0f;
              } else if (p.surrogate == QSM_SURR_PRE) {
                ds = gw * ex2_approx(__fmaf_rn(r, p.cL2E, -c1.x));
              } else {
                ds = ex2_approx(__fmaf_rn(r, p.cL2E, -c1.x)) * (dp - c1.y);
              }
            }
            pv2[h] = valid ? pw : 0.0f;
            ds2[h] = valid ? ds : 0.0f;
          }
          pp[i2] = pack_bf16x2(pv2[0], pv2[1]);
          dd[i2] = pack_bf16x2(ds2[0], ds2[1]);
        }
        // P^T and dS^T into the first 16 of this group's own TMEM columns
        // (the other groups are still reading theirs)
        tmem_st16(lane_base + T_S + col0, pp);
        tmem_st16(lane_base + T_DP + col0, dd);
        // dS in shared memory as the MN-major A operand of dQ = dS K:
        // K index = key (row of 128 bytes per 64 queries), M = query
        const uint32_t region = ds_base + (g >> 1) * G::CHUNK_BYTES + key * 128;
#pragma unroll
        for (int gi = 0; gi < 4; ++gi) {
          const uint32_t gran = ((g & 1) * 4 + gi) ^ (key & 7);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(region + gran * 16),
                       "r"(dd[4 * gi]), "r"(dd[4 * gi + 1]), "r"(dd[4 * gi + 2]),
                       "r"(dd[4 * gi + 3])
                       : "memory");
        }
      }
      tmem_wait_st();
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(bars.pds_full);
      // ---- dQ tile (lane = query row) into the fp32 workspace: group g adds
      // columns g*D/4 .. (g+1)*D/4 - 1
      ok = warp_all_b(mbar_wait(bars.dq_full, n & 1, abort));
      if (!ok) break;
      tc_fence_after();
      const int qrow = qbase + key;
      float *dst = p.dqacc + (static_cast<size_t>(bh) * p.S + min(qrow, p.S - 1)) * D + g * (D / 4);
      static_assert(D / 4 == 16, "dQ slice of one map group: 16 columns");
      {
        uint32_t v[16];
        tmem_ld16_sync(lane_base + T_DQ + g * (D / 4), v);
        if (qrow < p.S) {
#pragma unroll
          for (int i = 0; i < 4; ++i)
            red_add_v4(dst + 4 * i, __uint_as_float(v[4 * i]) * p.c,
                       __uint_as_float(v[4 * i + 1]) * p.c, __uint_as_float(v[4 * i + 2]) * p.c,
                       __uint_as_float(v[4 * i + 3]) * p.c);
        }
      }
      tc_fence_before();
      mbar_arrive(bars.dq_empty);
    }
    // ---- dK, dV of this key tile: group g stores 32 columns, dK for g < 2
    if (ok && nq > 0) ok = warp_all_b(mbar_wait(bars.acc_full, 0, abort));
    if (ok) {
      tc_fence_after();
      const size_t krow = static_cast<size_t>(bh) * p.S + min(kg, p.S - 1);
      static_assert(D == 64, "dK / dV slices: two groups of 32 columns each");
      const int which = g >> 1, dc = g & 1;
      __nv_bfloat16 *out = (which == 0 ? p.dK : p.dV) + krow * D;
      const float sc = which == 0 ? p.c : 1.0f;
      uint32_t v[32];
      if (nq > 0) {
        tmem_ld32_sync(lane_base + (which == 0 ? T_DK : T_DV) + 32 * dc, v);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0u;
      }
      float x[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) x[i] = __uint_as_float(v[i]) * sc;
      if (which == 0 && p.dkcal != nullptr && key_ok) {
        const float4 *cal = reinterpret_cast<const float4 *>(p.dkcal + krow * D + 32 * dc);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float4 c4 = cal[i];
          x[4 * i] += c4.x;
          x[4 * i + 1] += c4.y;
          x[4 * i + 2] += c4.z;
          x[4 * i + 3] += c4.w;
        }
      }
      uint32_t pk[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(x[2 * i], x[2 * i + 1]);
      if (key_ok) {
        uint4 *d4 = reinterpret_cast<uint4 *>(out + 32 * dc);
#pragma unroll
        for (int i = 0; i < 4; ++i)
          d4[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
      }
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kBwdTmemCols);
  if (threadIdx.x == 0 && *bars.abort && p.status != nullptr) atomicExch(p.status, QSM_ERR_TIMEOUT);
}

template <int D>
qsm_status launch_bwd_d(const BwdArgs &a, BwdParams p, const CUtensorMap &mq,
                        const CUtensorMap &mk, const CUtensorMap &mv, const CUtensorMap &mdo) {
  using G = BGeo<D>;
  const int BH = a.B * a.H;
  const bool need_rows = a.mode == QSM_MODE_KINTERVAL &&
                         (!a.detach || a.surrogate == QSM_SURR_POST);
  const size_t max_smem = 232448;
  if (need_rows) {
    const size_t tab = static_cast<size_t>(128) * (p.K + 1) * sizeof(float2);
    BwdParams r = p;
    r.tab_off = static_cast<uint32_t>(2 * G::TILE_BYTES + 4 * G::TILE_BYTES);
    r.cst_off = static_cast<uint32_t>((r.tab_off + tab + 15) & ~static_cast<size_t>(15));
    r.bar_off = static_cast<uint32_t>(r.cst_off + 5 * 4 * 128 * sizeof(float));
    size_t smem = 1024 + r.bar_off + 256;
    if (smem < 120 * 1024) smem = 120 * 1024;
    if (smem > max_smem) return QSM_ERR_UNSUPPORTED;
    auto kern = (p.map == MAPB_HARD) ? qsm_bwd_rows<D, MAPB_HARD> : qsm_bwd_rows<D, MAPB_INTERP>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return QSM_ERR_CUDA;
    kern<<<dim3(p.nqt, BH), kMainThreads, smem, a.stream>>>(mq, mk, mv, mdo, r);
    if (cudaGetLastError() != cudaSuccess) return QSM_ERR_CUDA;
  }
  if (p.dkcal != nullptr) {
    const long long rows = static_cast<long long>(BH) * p.S;
    qsm_bwd_calib<<<static_cast<unsigned>((rows + 7) / 8), 256, 0, a.stream>>>(
        static_cast<const __nv_bfloat16 *>(a.Q), static_cast<const __nv_bfloat16 *>(a.K),
        p.rowws, p.amax, p.amin, p.dqacc, p.dkcal, p.S, D, rows, p.c);
    if (cudaGetLastError() != cudaSuccess) return QSM_ERR_CUDA;
  }
  {
    const size_t tab = static_cast<size_t>(128) * (p.K + 1) * sizeof(float2);
    p.ds_off = static_cast<uint32_t>(2 * G::TILE_BYTES + 4 * G::TILE_BYTES);
    p.tab_off = p.ds_off + 128 * 128 * 2;
    p.cst_off = static_cast<uint32_t>(p.tab_off + tab);
    p.bar_off = static_cast<uint32_t>((p.cst_off + 128 * 8 * 4 + 15) & ~15u);
    size_t smem = 1024 + p.bar_off + 256;
    if (smem < 120 * 1024) smem = 120 * 1024;
    if (smem > max_smem) return QSM_ERR_UNSUPPORTED;
    auto kern = (p.map == MAPB_EXACT) ? qsm_bwd_main<D, MAPB_EXACT>
                : (p.map == MAPB_HARD) ? qsm_bwd_main<D, MAPB_HARD>
                                       : qsm_bwd_main<D, MAPB_INTERP>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return QSM_ERR_CUDA;
    kern<<<dim3(p.nkvt, BH), kMainThreads, smem, a.stream>>>(mq, mk, mv, mdo, p);
    if (cudaGetLastError() != cudaSuccess) return QSM_ERR_CUDA;
  }
  return QSM_OK;
}

}  // namespace

size_t bwd_workspace_bytes(int B, int H, int S, int D) {
  // dQ fp32 accumulator, dK calibration part (fp32), then kRowWs floats per
  // row; each part 256-byte aligned
  const size_t rows = static_cast<size_t>(B) * H * S;
  const size_t mat = (rows * D * sizeof(float) + 255) & ~static_cast<size_t>(255);
  return 2 * mat + ((rows * kRowWs * sizeof(float) + 255) & ~static_cast<size_t>(255));
}

qsm_status launch_bwd(const BwdArgs &a) {
  if (a.D != 64) return QSM_ERR_UNSUPPORTED;          // TMEM schedule holds D = 64
  if (a.mode == QSM_MODE_KINTERVAL && a.Kint > 32) return QSM_ERR_UNSUPPORTED;
  const size_t rows = static_cast<size_t>(a.B) * a.H * a.S;
  BwdParams p{};
  p.S = a.S;
  p.nqt = (a.S + 127) / 128;
  p.nkvt = p.nqt;
  p.causal = a.causal;
  p.map = a.mode == QSM_MODE_EXACT ? MAPB_EXACT
          : (a.rounding == QSM_ROUND_HARD ? MAPB_HARD : MAPB_INTERP);
  p.K = a.mode == QSM_MODE_KINTERVAL ? a.Kint : 1;
  p.fixed_window = a.calib == QSM_CALIB_FIXED_WINDOW;
  p.flush = a.below_policy == 1;
  p.surrogate = a.surrogate;
  p.detach = a.detach;
  p.c = a.c;
  p.cL2E = a.c * 1.4426950408889634f;
  p.window = a.window;
  p.LSE = a.LSE;
  p.hi = a.row_hi;
  p.lo = a.row_lo;
  p.amax = a.row_argmax;
  p.amin = a.row_argmin;
  const size_t mat = (rows * a.D * sizeof(float) + 255) & ~static_cast<size_t>(255);
  uint8_t *ws = static_cast<uint8_t *>(a.workspace);
  p.dqacc = reinterpret_cast<float *>(ws);
  const bool calib_terms = a.mode == QSM_MODE_KINTERVAL && !a.detach;
  p.dkcal = calib_terms ? reinterpret_cast<float *>(ws + mat) : nullptr;
  p.rowws = reinterpret_cast<float *>(ws + 2 * mat);
  p.dK = static_cast<__nv_bfloat16 *>(a.dK);
  p.dV = static_cast<__nv_bfloat16 *>(a.dV);
  p.status = a.status_dev;

  alignas(64) CUtensorMap mq, mk, mv, mdo;
  const int bh = a.B * a.H;
  if (!make_tmap_3d(&mq, a.Q, false, a.D, a.S, bh, 128) ||
      !make_tmap_3d(&mk, a.K, false, a.D, a.S, bh, 128) ||
      !make_tmap_3d(&mv, a.V, false, a.D, a.S, bh, 128) ||
      !make_tmap_3d(&mdo, a.dO, false, a.D, a.S, bh, 128))
    return QSM_ERR_CUDA;

  if (cudaMemsetAsync(p.dqacc, 0, rows * a.D * sizeof(float), a.stream) != cudaSuccess)
    return QSM_ERR_CUDA;
  if (p.dkcal != nullptr &&
      cudaMemsetAsync(p.dkcal, 0, rows * a.D * sizeof(float), a.stream) != cudaSuccess)
    return QSM_ERR_CUDA;
  const long long nrows = static_cast<long long>(rows);
  qsm_bwd_delta<<<static_cast<unsigned>((nrows + 7) / 8), 256, 0, a.stream>>>(
      static_cast<const __nv_bfloat16 *>(a.O), static_cast<const __nv_bfloat16 *>(a.dO), p.rowws,
      nrows, a.D);
  if (cudaGetLastError() != cudaSuccess) return QSM_ERR_CUDA;
  qsm_status st = launch_bwd_d<64>(a, p, mq, mk, mv, mdo);
  if (st != QSM_OK) return st;
  const long long n = nrows * a.D;
  qsm_bwd_dq_convert<<<static_cast<unsigned>((n / 4 + 255) / 256), 256, 0, a.stream>>>(
      p.dqacc, static_cast<__nv_bfloat16 *>(a.dQ), n);
  return cudaGetLastError() == cudaSuccess ? QSM_OK : QSM_ERR_CUDA;
}

}  // namespace qsm
