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
//   1. qsm_bwd_delta  delta_r = dO_r . O_r (one warp per row)
//   2. qsm_bwd_rows   post surrogate only: LSE* and delta* per query row
//                     (S and dP tiles swept once per query tile)
//   3. qsm_bwd_prep   one thread per query row: the row's map constants and
//                     its grid table (g_n, g_{n+1} - g_n), written once to
//                     the workspace for both passes below
//   4. qsm_bwd_dq     one CTA per 128-row query tile, sweeping the key tiles
//                     in halves of 64 keys: S = Q K^T and dP = dO V^T into a
//                     double-buffered TMEM pair, dS by the rule above into
//                     shared memory, dQ += dS K in TMEM; the calibration sums
//                     dhi, dlo accumulate per row; the epilogue adds the
//                     rank-one terms to dQ (fp32) before its bf16 store and
//                     scatters the dK ones into an fp32 buffer
//   5. qsm_bwd_dkdv   one CTA per 128-key tile, sweeping the query tiles in
//                     halves of 64 rows: S^T = K Q^T, dP^T = V dO^T into a
//                     double-buffered TMEM pair, P^T and dS^T written back to
//                     TMEM, dV += P^T dO and dK += dS^T Q in TMEM; dK gets the
//                     fp32 calibration part before its bf16 store
// Each pass recomputes its products, so no dQ partial sums cross CTAs; the
// double buffers let the map of one half overlap the products of the next.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>

#include "internal.h"
#include "sm100.cuh"
#include "wmap.cuh"

namespace qsm {

namespace {

// rows pass: warp 0 TMA, warp 1 MMA, warps 4-19 four map groups, group g
// owning columns 32g .. 32g+31 of every S / dP tile
constexpr int kMainThreads = 640;
constexpr int kMainMapThreads = 512;
constexpr uint32_t kBwdTmemCols = 512;
constexpr int kRowWs = 8;               // floats per row in the row workspace
enum RowWs { RW_DELTA = 0, RW_DHI = 1, RW_DLO = 2, RW_LSESTAR = 3, RW_DELTASTAR = 4 };
constexpr int kBwdMaxK = 32;            // largest K the backward accepts
constexpr int kCst = 8;                 // floats of one query row's map constants

struct BwdParams {
  int S, nqt, nkvt;
  int causal;
  int map;          // 0 exact, 1 Rowmax-PoT, 2 K-interval hard, 3 K-interval interp
  int pot_floor;
  int K, fixed_window, flush, surrogate, detach;
  int calib;        // calibration terms on (K-interval, not detached)
  int KT;           // float2 entries of one row's table in the workspace (K+1, even)
  float c, cL2E, window;
  const float *LSE, *hi, *lo;
  const int32_t *amax, *amin;
  float *rowws;
  float *cst;       // [rows][kCst] per query row: a, b, 1/Z, delta, e, delta*, inv, 1/(hi-lo)
  float2 *tabg;     // [rows][KT] per query row: (g_n, g_{n+1} - g_n), n = 0..K
  float *dkcal;     // [rows][D] fp32 calibration part of dK (nullptr: none)
  const __nv_bfloat16 *Q, *K_;
  __nv_bfloat16 *dQ, *dK, *dV;
  int32_t *status;
  int num_stages;
  uint32_t tab_off, cst_off, ds_off, bar_off, part_off, stage_bytes;
};

constexpr int MAPB_EXACT = 0, MAPB_POT = 1, MAPB_HARD = 2, MAPB_INTERP = 3;

template <int D>
struct BGeo {
  static constexpr int TILE_BYTES = 128 * D * 2;        // bf16 tile of 128 rows
  static constexpr int CHUNKS = (D * 2) / 128;
  static constexpr int EPC = 64;                        // bf16 per 128-byte row
  static constexpr int CHUNK_BYTES = 128 * 128;
  static constexpr int KSTEPS_D = D / 16;               // k-steps over D
  static constexpr uint32_t IDESC_SS = instr_desc(1, false, 128, 128);
  static constexpr uint32_t IDESC_H = instr_desc(1, false, 128, 64);    // N = 64 half tiles
  static constexpr uint32_t IDESC_MN = instr_desc(1, true, 128, D);     // B MN-major
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

// Half tile: D[128 x 64] = A[128 x D] B[64 x D]^T, both K-major (B: 64 rows
// of a 128-row tile, the start of a 1024-byte swizzle atom).
template <int D>
__device__ __forceinline__ void mma_nt_half(uint32_t d_tmem, uint32_t a_saddr, uint32_t b_saddr) {
  using G = BGeo<D>;
#pragma unroll
  for (int kk = 0; kk < G::KSTEPS_D; ++kk) {
    const int e = kk * 16;
    const uint32_t off = (e / G::EPC) * G::CHUNK_BYTES + (e % G::EPC) * 2;
    mma_ss_f16(d_tmem, smem_desc(a_saddr + off, 16, 1024), smem_desc(b_saddr + off, 16, 1024),
               G::IDESC_H, kk > 0);
  }
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

// ----------------------------------------------------------------- rows
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
    const float lo_in = p.lo != nullptr ? p.lo[ri] : hi;
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

// ------------------------------------------------------------------ prep
// One thread per query row: the constants of the row's map, as the two
// passes read them (cst), and its grid table (g_n, g_{n+1} - g_n).
//   cst = a, b (coordinate = fma(r, a, b) on the raw product r), 1/Z,
//         delta, e (exact: LSE log2e; pre: hi log2e; post: LSE* log2e),
//         delta*, K/(hi-lo) (d coordinate / d score), 1/(hi-lo)
__global__ void __launch_bounds__(256) qsm_bwd_prep(const BwdParams p, long long rows) {
  const long long r = static_cast<long long>(blockIdx.x) * 256 + threadIdx.x;
  if (r >= rows) return;
  const float *rw = p.rowws + r * kRowWs;
  const float lse = p.LSE[r];
  float c[kCst] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
  c[3] = rw[RW_DELTA];
  if (p.map == MAPB_EXACT) {
    c[4] = lse * 1.4426950408889634f;
  } else if (p.map == MAPB_POT) {
    // the forward's exponent coordinate x = fma(r, -c log2e, hi log2e)
    const float hi = p.hi[r];
    const float hiL2E = __fmul_rn(hi, log2e_f());
    c[0] = -p.cL2E;
    c[1] = hiL2E;
    c[2] = expf(hi - lse);
    c[4] = (p.surrogate == QSM_SURR_POST) ? rw[RW_LSESTAR] * 1.4426950408889634f : hiL2E;
    c[5] = rw[RW_DELTASTAR];
  } else {
    const float hi = p.hi[r];
    const RowMap rm = make_rowmap(hi, p.lo[r], p.K, p.fixed_window != 0, p.window);
    c[0] = rm.degenerate ? 0.0f : __fmul_rn(p.c, rm.inv);
    c[1] = rm.degenerate ? static_cast<float>(p.K) : rm.b;
    c[2] = expf(hi - lse);                              // 1/Z, Z = exp(LSE - hi)
    c[4] = (p.surrogate == QSM_SURR_POST) ? rw[RW_LSESTAR] * 1.4426950408889634f : rm.hiL2E;
    c[5] = rw[RW_DELTASTAR];
    c[6] = rm.degenerate ? 0.0f : rm.inv;
    c[7] = rm.degenerate ? 0.0f : 1.0f / __fsub_rn(hi, rm.lo);
    float2 *t = p.tabg + r * p.KT;
    for (int n = 0; n <= p.K; ++n) {
      const float gk = grid_value(rm, p.K, n);
      const float gk1 = n < p.K ? grid_value(rm, p.K, n + 1) : gk;
      t[n] = make_float2(gk, __fsub_rn(gk1, gk));
    }
  }
  float4 *cd = reinterpret_cast<float4 *>(p.cst + r * kCst);
  cd[0] = make_float4(c[0], c[1], c[2], c[3]);
  cd[1] = make_float4(c[4], c[5], c[6], c[7]);
}

// One element of the backward: returns the probability p = w / Z and writes
// ds (the surrogate's dL/ds, before the factor c), the map's intermediate
// values (for the calibration sums) and gw = dL/dw.  c0 = (a, b, 1/Z,
// delta), c1 = (e, delta*, K/(hi-lo), 1/(hi-lo)); tab[n * ts] = (g_n, g_{n+1}
// - g_n) of the element's query row.
template <int MAP>
__device__ __forceinline__ float bwd_elem(float r, float dp, const float4 &c0, const float4 &c1,
                                          const float2 *tab, int ts, const BwdParams &p,
                                          float Kf, float &ds, float &gw, float &u, float &uc,
                                          float &kf, float2 &gd) {
  if (MAP == MAPB_EXACT) {
    const float pw = ex2_approx(__fmaf_rn(r, p.cL2E, -c1.x));
    ds = pw * (dp - c0.w);
    gw = 0.0f;
    return pw;
  }
  if (MAP == MAPB_POT) {
    // the forward's power-of-two weight (exponent frozen: no own-score or
    // anchor derivative; only the surrogate's direct term)
    const float x = __fmaf_rn(r, c0.x, c0.y);
    const float cap = static_cast<float>(p.flush ? p.pot_floor + 1 : p.pot_floor);
    const float t = __fadd_rn(fminf(x, cap), kMagic);
    float w = __uint_as_float(__float_as_uint(t) * 0xFF800000u + 0x3F800000u);
    if (p.flush && t > kMagic + static_cast<float>(p.pot_floor)) w = 0.0f;
    const float pw = w * c0.z;
    gw = (dp - c0.w) * c0.z;
    if (p.surrogate == QSM_SURR_NONE)
      ds = 0.0f;
    else if (p.surrogate == QSM_SURR_PRE)
      ds = gw * ex2_approx(__fmaf_rn(r, p.cL2E, -c1.x));
    else
      ds = ex2_approx(__fmaf_rn(r, p.cL2E, -c1.x)) * (dp - c1.y);
    return pw;
  }
  u = __fmaf_rn(r, c0.x, c0.y);
  uc = fminf(fmaxf(u, 0.0f), Kf);
  const bool below = p.fixed_window && u < 0.0f;
  float w, slope = 0.0f;
  if (MAP == MAPB_HARD) {
    // nearest node from the bits of a magic-number add
    const float tn = __fadd_rn(uc, kMagic);
    gd = tab[static_cast<int>(__float_as_uint(tn) - kMagicBits) * ts];
    w = gd.x;
    kf = __fsub_rn(tn, kMagic);
  } else {
    // floor from a round-down add of 2^23 (exact for 0 <= uc <= K)
    const float tf = __fadd_rd(uc, 8388608.0f);
    kf = fminf(__fsub_rn(tf, 8388608.0f), Kf - 1.0f);
    gd = tab[min(static_cast<int>(__float_as_uint(tf) - 0x4B000000u), p.K - 1) * ts];
    w = __fmaf_rn(__fsub_rn(uc, kf), gd.y, gd.x);
    slope = gd.y;
  }
  if (below && p.flush) w = 0.0f;
  const float pw = w * c0.z;
  gw = (dp - c0.w) * c0.z;
  if (p.surrogate == QSM_SURR_NONE)
    ds = (MAP == MAPB_INTERP && !below) ? gw * slope * c1.z : 0.0f;
  else if (p.surrogate == QSM_SURR_PRE)
    ds = gw * ex2_approx(__fmaf_rn(r, p.cL2E, -c1.x));
  else
    ds = ex2_approx(__fmaf_rn(r, p.cL2E, -c1.x)) * (dp - c1.y);
  return pw;
}

// Calibration sums of one element: dhi += gw dF/dhi, dlo += gw dF/dlo with s
// and the decision held fixed (min-max hard: dF/dhi = -(K-n)/K w = -dF/dlo;
// interpolation: the slope and mixing terms; fixed window: only hi moves).
template <int MAP>
__device__ __forceinline__ void calib_elem(const BwdParams &p, float Kf, float invK, float gw,
                                           float u, float uc, float kf, float2 gd, float inv_a,
                                           float &dhi, float &dlo) {
  if (MAP == MAPB_HARD) {
    if (!p.fixed_window) {
      const float t = gw * (kf - Kf) * invK * gd.x;
      dhi += t;
      dlo -= t;
    }
  } else if (MAP == MAPB_INTERP) {
    const float f = uc - kf;
    const float slope = gd.y;
    if (!p.fixed_window) {
      // ((1-f)(K-k) g_k + f (K-k-1) g_{k+1}) / K = ((K-k) w - f g_{k+1}) / K
      // with w = g_k + f (g_{k+1} - g_k) the interpolated weight
      const float w = gd.x + f * slope;
      const float mix = ((Kf - kf) * w - f * (gd.x + slope)) * invK;
      const float ts = gw * slope * inv_a;
      const float gm = gw * mix;
      dhi += -ts * uc - gm;
      dlo += -ts * (Kf - uc) + gm;
    } else if (u >= 0.0f) {
      dhi += gw * (slope * (-Kf / p.window));
    }
  }
}

// ----------------------------------------------------------------- dQ pass
// One CTA per 128-row query tile of one (b, h); thread = query row (TMEM
// lane); the key tiles are taken in halves of 64 keys, half h in TMEM pair
// x = h & 1 (S at 128x, dP at 128x + 64) and shared dS buffer x; map group g
// owns keys 16g .. 16g+15 of each half.  dQ accumulates at TMEM column 256.
struct DqBars {
  uint64_t *kv_full, *kv_empty;       // [ns]: K_j, V_j
  uint64_t *q_full;                   // Q, dO
  uint64_t *sdp_full, *sdp_free;      // [2]
  uint64_t *ds_full, *ds_free;        // [2]
  uint64_t *dq_full, *tab_ready, *part_ready, *drain;
  uint32_t *tmem_slot;
  int *abort;
};
constexpr uint32_t T_DQ = 256;

template <int D, int MAP>
__global__ void __launch_bounds__(kMainThreads, 1)
    qsm_bwd_dq(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
               const BwdParams p) {
  using G = BGeo<D>;
  static_assert(D == 64, "dQ slices of the four map groups: 16 columns each");
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y, qt = blockIdx.x;
  const int ns = p.num_stages;
  uint8_t *sQ = smem;
  uint8_t *sdO = smem + G::TILE_BYTES;
  uint8_t *sKV = smem + 2 * G::TILE_BYTES;              // ns stages of (K_j, V_j)
  uint8_t *sDS = smem + p.ds_off;                        // 2 x 128 rows x 128 bytes
  float2 *tab = reinterpret_cast<float2 *>(smem + p.tab_off);   // [n][128]
  float *part = reinterpret_cast<float *>(smem + p.part_off);   // [2][4][128]
  uint64_t *bp = reinterpret_cast<uint64_t *>(smem + p.bar_off);
  DqBars bars;
  bars.kv_full = bp;
  bars.kv_empty = bp + ns;
  bars.q_full = bp + 2 * ns;
  bars.sdp_full = bars.q_full + 1;
  bars.sdp_free = bars.sdp_full + 2;
  bars.ds_full = bars.sdp_free + 2;
  bars.ds_free = bars.ds_full + 2;
  bars.dq_full = bars.ds_free + 2;
  bars.tab_ready = bars.dq_full + 1;
  bars.part_ready = bars.tab_ready + 1;
  bars.drain = bars.part_ready + 1;
  bars.tmem_slot = reinterpret_cast<uint32_t *>(bars.drain + 1);
  bars.abort = reinterpret_cast<int *>(bars.tmem_slot + 1);
  volatile int *abort = bars.abort;
  const int nkv = p.causal ? min(p.nkvt, qt + 1) : p.nkvt;
  const int nh = 2 * nkv;

  if (threadIdx.x == 0) {
    for (int i = 0; i < ns; ++i) {
      mbar_init(&bars.kv_full[i], 1);
      mbar_init(&bars.kv_empty[i], 1);
    }
    mbar_init(bars.q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.sdp_full[i], 1);
      mbar_init(&bars.sdp_free[i], kMainMapThreads);
      mbar_init(&bars.ds_full[i], kMainMapThreads);
      mbar_init(&bars.ds_free[i], 1);
    }
    mbar_init(bars.dq_full, 1);
    mbar_init(bars.tab_ready, kMainMapThreads);
    mbar_init(bars.part_ready, kMainMapThreads);
    mbar_init(bars.drain, 2);
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
      bool ok = true;
      for (int j = 0; j < nkv && ok; ++j) {
        const int st = j % ns;
        if (j >= ns) ok = mbar_wait(&bars.kv_empty[st], ((j / ns) - 1) & 1, abort);
        if (!ok) break;
        uint8_t *kdst = sKV + st * 2 * G::TILE_BYTES;
        mbar_expect_tx(&bars.kv_full[st], 2 * G::TILE_BYTES);
        for (int ch = 0; ch < G::CHUNKS; ++ch) {
          tma_load_3d(kdst + ch * G::CHUNK_BYTES, &tmK, &bars.kv_full[st], ch * G::EPC, j * 128, bh);
          tma_load_3d(kdst + G::TILE_BYTES + ch * G::CHUNK_BYTES, &tmV, &bars.kv_full[st],
                      ch * G::EPC, j * 128, bh);
        }
      }
      // every load issued must land before the CTA may exit
      mbar_wait(bars.q_full, 0, abort);
      for (int st = 0; st < ns && st < nkv; ++st)
        mbar_wait(&bars.kv_full[st], (((nkv - st + ns - 1) / ns) - 1) & 1, abort);
    }
  } else if (warp == 1) {
    // S = Q K_h^T and dP = dO V_h^T of half h into TMEM pair h & 1
    if (lane == 0) {
      bool ok = mbar_wait(bars.q_full, 0, abort);
      tc_fence_after();
      const uint32_t qa = smem_u32(sQ), da = smem_u32(sdO), kva = smem_u32(sKV);
      for (int h = 0; h < nh && ok; ++h) {
        const int j = h >> 1, e = h & 1, x = h & 1;
        if (e == 0) {
          ok = mbar_wait(&bars.kv_full[j % ns], (j / ns) & 1, abort);
          if (!ok) break;
          tc_fence_after();
        }
        if (h >= 2) {
          ok = mbar_wait(&bars.sdp_free[x], ((h >> 1) - 1) & 1, abort);
          if (!ok) break;
          tc_fence_after();
        }
        const uint32_t kb = kva + (j % ns) * 2 * G::TILE_BYTES + e * 64 * 128;
        mma_nt_half<D>(tmem + 128 * x, qa, kb);
        mma_nt_half<D>(tmem + 128 * x + 64, da, kb + G::TILE_BYTES);
        mma_commit(&bars.sdp_full[x]);
      }
      mma_commit(bars.drain);
      mbar_wait(bars.drain, 0, abort);
    }
  } else if (warp == 2) {
    // dQ += dS_h K_h (dS K-major in shared memory, K as an MN-major operand)
    if (lane == 0) {
      bool ok = true;
      const uint32_t kva = smem_u32(sKV), dsa = smem_u32(sDS);
      for (int h = 0; h < nh && ok; ++h) {
        const int j = h >> 1, e = h & 1, x = h & 1;
        if (e == 0) {
          // K_j has landed (this warp reads it too; the stage cannot refill
          // before this warp's own release below)
          ok = mbar_wait(&bars.kv_full[j % ns], (j / ns) & 1, abort);
          if (!ok) break;
        }
        ok = mbar_wait(&bars.ds_full[x], (h >> 1) & 1, abort);
        if (!ok) break;
        tc_fence_after();
        const uint32_t kb = kva + (j % ns) * 2 * G::TILE_BYTES + e * 64 * 128;
        const uint32_t ab = dsa + x * 128 * 128;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ss_f16(tmem + T_DQ, smem_desc(ab + kk * 32, 16, 1024),
                     smem_desc(kb + kk * 16 * 128, G::CHUNK_BYTES, 1024), G::IDESC_MN,
                     (h > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&bars.ds_free[x]);
        if (e == 1) mma_commit(&bars.kv_empty[j % ns]);
      }
      if (ok) mma_commit(bars.dq_full);
      mma_commit(bars.drain);
      mbar_wait(bars.drain, 0, abort);
    }
  } else if (warp >= 4) {
    const int g = (warp - 4) >> 2;
    const int row = (warp & 3) * 32 + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const int qrow = qt * 128 + row;
    const bool row_ok = qrow < p.S;
    const int L = p.causal ? min(qrow + 1, p.S) : p.S;
    const size_t ri = static_cast<size_t>(bh) * p.S + min(qrow, p.S - 1);
    const float4 *cg = reinterpret_cast<const float4 *>(p.cst + ri * kCst);
    const float4 c0 = cg[0], c1 = cg[1];
    const float Kf = static_cast<float>(p.K), invK = 1.0f / Kf;
    const bool calib = p.calib && c1.w != 0.0f;          // 1/(hi-lo) = 0: degenerate row
    if (MAP == MAPB_HARD || MAP == MAPB_INTERP)
      for (int n = g; n <= p.K; n += 4) tab[n * 128 + row] = p.tabg[ri * p.KT + n];
    mbar_arrive(bars.tab_ready);
    bool ok = warp_all_b(mbar_wait(bars.tab_ready, 0, abort));
    float dhi = 0.0f, dlo = 0.0f;
    const uint32_t dsb = smem_u32(sDS);
    for (int h = 0; h < nh && ok; ++h) {
      const int j = h >> 1, e = h & 1, x = h & 1;
      ok = warp_all_b(mbar_wait(&bars.sdp_full[x], (h >> 1) & 1, abort));
      if (!ok) break;
      tc_fence_after();
      uint32_t sv[16], dv[16];
      tmem_ld16(lane_base + 128 * x + 16 * g, sv);
      tmem_ld16(lane_base + 128 * x + 64 + 16 * g, dv);
      tmem_wait_ld();
      reg_fence16(sv);
      reg_fence16(dv);
      tc_fence_before();
      mbar_arrive(&bars.sdp_free[x]);                  // the pair can take half h + 2
      const int lim = L - (128 * j + 64 * e + 16 * g);  // valid keys of this slice
      uint32_t dd[8];
#pragma unroll
      for (int i2 = 0; i2 < 8; ++i2) {
        float d2[2];
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          const int i = 2 * i2 + t;
          float ds, gw, u = 0.0f, uc = 0.0f, kf = 0.0f;
          float2 gd = make_float2(0.0f, 0.0f);
          (void)bwd_elem<MAP>(__uint_as_float(sv[i]), __uint_as_float(dv[i]), c0, c1,
                              tab + row, 128, p, Kf, ds, gw, u, uc, kf, gd);
          const bool valid = i < lim;
          if ((MAP == MAPB_HARD || MAP == MAPB_INTERP) && calib && valid)
            calib_elem<MAP>(p, Kf, invK, gw, u, uc, kf, gd, c1.w, dhi, dlo);
          d2[t] = valid ? ds : 0.0f;
        }
        dd[i2] = pack_bf16x2(d2[0], d2[1]);
      }
      if (h >= 2) {
        ok = warp_all_b(mbar_wait(&bars.ds_free[x], ((h >> 1) - 1) & 1, abort));
        if (!ok) break;
      }
      // dS row-major (K-major operand), 128-byte swizzle: this group's 16
      // keys are granules 2g, 2g + 1 of the row
      const uint32_t rowa = dsb + x * 128 * 128 + row * 128;
#pragma unroll
      for (int gi = 0; gi < 2; ++gi) {
        const uint32_t gran = static_cast<uint32_t>((2 * g + gi) ^ (row & 7));
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(rowa + gran * 16),
                     "r"(dd[4 * gi]), "r"(dd[4 * gi + 1]), "r"(dd[4 * gi + 2]), "r"(dd[4 * gi + 3])
                     : "memory");
      }
      fence_async_smem();
      mbar_arrive(&bars.ds_full[x]);
    }
    // ---- epilogue: the row's calibration sums, dQ
    part[(0 * 4 + g) * 128 + row] = dhi;
    part[(1 * 4 + g) * 128 + row] = dlo;
    mbar_arrive(bars.part_ready);
    if (ok) ok = warp_all_b(mbar_wait(bars.part_ready, 0, abort));
    if (ok) ok = warp_all_b(mbar_wait(bars.dq_full, 0, abort));
    if (ok) {
      tc_fence_after();
      const float tdhi = (part[row] + part[128 + row]) + (part[256 + row] + part[384 + row]);
      const float tdlo = (part[512 + row] + part[640 + row]) + (part[768 + row] + part[896 + row]);
      uint32_t v[16];
      tmem_ld16_sync(lane_base + T_DQ + 16 * g, v);
      float xq[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) xq[i] = __uint_as_float(v[i]) * p.c;
      if (calib && row_ok) {
        // rank-one calibration terms in fp32: dQ_r += c (dhi k_argmax + dlo k_argmin)
        const size_t head = static_cast<size_t>(bh) * p.S;
        const __nv_bfloat16 *ka = p.K_ + (head + p.amax[ri]) * D + 16 * g;
        const __nv_bfloat16 *kb = p.K_ + (head + p.amin[ri]) * D + 16 * g;
        const float sh = p.c * tdhi, sl = p.c * tdlo;
#pragma unroll
        for (int i = 0; i < 16; ++i)
          xq[i] += sh * __bfloat162float(ka[i]) + sl * __bfloat162float(kb[i]);
        // and dK_argmax += c dhi q_r, dK_argmin += c dlo q_r, into the fp32
        // calibration part of dK (many rows can share one key: atomics)
        const __nv_bfloat16 *qr = p.Q + ri * D + 16 * g;
        float *da = p.dkcal + (head + p.amax[ri]) * D + 16 * g;
        float *db = p.dkcal + (head + p.amin[ri]) * D + 16 * g;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float qv = __bfloat162float(qr[i]);
          atomicAdd(da + i, sh * qv);
          atomicAdd(db + i, sl * qv);
        }
        if (g == 0) {
          p.rowws[ri * kRowWs + RW_DHI] = tdhi;
          p.rowws[ri * kRowWs + RW_DLO] = tdlo;
        }
      }
      uint32_t pk[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) pk[i] = pack_bf16x2(xq[2 * i], xq[2 * i + 1]);
      if (row_ok) {
        uint4 *d4 = reinterpret_cast<uint4 *>(p.dQ + ri * D + 16 * g);
        d4[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        d4[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
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

// --------------------------------------------------------------- dK/dV pass
// One CTA per 128-key tile of one (b, h); thread = key (TMEM lane); the
// query tiles are taken in halves of 64 rows, half h in TMEM pair x = h & 1
// (S^T at 128x, dP^T at 128x + 64); map group g owns queries 16g .. 16g+15 of
// each half and writes its P^T and dS^T (bf16) into the first 8 of its own 16
// columns, which the dV / dK products read as their TMEM A operand.  A ring
// stage holds Q_i, dO_i and the tile's per-row constants and grid tables.
struct KvBars {
  uint64_t *qd_full, *qd_empty;       // [ns]
  uint64_t *kv_full;                  // K, V once
  uint64_t *sdp_full, *pds_full, *s_free;   // [2]
  uint64_t *acc_full, *drain;
  uint32_t *tmem_slot;
  int *abort;
};
constexpr uint32_t T_DV = 256, T_DK = 320;

template <int D, int MAP>
__global__ void __launch_bounds__(kMainThreads, 1)
    qsm_bwd_dkdv(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                 const BwdParams p) {
  using G = BGeo<D>;
  static_assert(D == 64, "dK / dV slices of the four map groups: 16 columns each");
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y, kt = blockIdx.x;
  const int ns = p.num_stages;
  uint8_t *sK = smem;
  uint8_t *sV = smem + G::TILE_BYTES;
  uint8_t *sSt = smem + 2 * G::TILE_BYTES;              // ns stages: Q, dO, cst, tab
  const uint32_t SB = p.stage_bytes;
  const uint32_t CST_OFF = 2 * G::TILE_BYTES;
  const uint32_t TAB_OFF = CST_OFF + 128 * kCst * 4;
  uint64_t *bp = reinterpret_cast<uint64_t *>(smem + p.bar_off);
  KvBars bars;
  bars.qd_full = bp;
  bars.qd_empty = bp + ns;
  bars.kv_full = bp + 2 * ns;
  bars.sdp_full = bars.kv_full + 1;
  bars.pds_full = bars.sdp_full + 2;
  bars.s_free = bars.pds_full + 2;
  bars.acc_full = bars.s_free + 2;
  bars.drain = bars.acc_full + 1;
  bars.tmem_slot = reinterpret_cast<uint32_t *>(bars.drain + 1);
  bars.abort = reinterpret_cast<int *>(bars.tmem_slot + 1);
  volatile int *abort = bars.abort;
  const int i0 = p.causal ? kt : 0;                      // first query tile
  const int nq = p.nqt - i0;
  const int nh = 2 * nq;

  if (threadIdx.x == 0) {
    for (int i = 0; i < ns; ++i) {
      mbar_init(&bars.qd_full[i], 1);
      mbar_init(&bars.qd_empty[i], 1);
    }
    mbar_init(bars.kv_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.sdp_full[i], 1);
      mbar_init(&bars.pds_full[i], kMainMapThreads);
      mbar_init(&bars.s_free[i], 1);
    }
    mbar_init(bars.acc_full, 1);
    mbar_init(bars.drain, 2);
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
      for (int n = 0; n < nq && ok; ++n) {
        const int st = n % ns, it = i0 + n;
        if (n >= ns) ok = mbar_wait(&bars.qd_empty[st], ((n / ns) - 1) & 1, abort);
        if (!ok) break;
        uint8_t *s = sSt + st * SB;
        // the constants and tables of the tile's rows that exist (a ragged last
        // tile copies fewer; its missing rows are never valid)
        const int nrow = min(128, p.S - it * 128);
        const size_t r0 = static_cast<size_t>(bh) * p.S + static_cast<size_t>(it) * 128;
        const uint32_t cbytes = static_cast<uint32_t>(nrow) * kCst * 4;
        const uint32_t tbytes =
            (MAP == MAPB_EXACT || MAP == MAPB_POT) ? 0u : static_cast<uint32_t>(nrow) * p.KT * 8;
        mbar_expect_tx(&bars.qd_full[st], 2 * G::TILE_BYTES + cbytes + tbytes);
        for (int ch = 0; ch < G::CHUNKS; ++ch) {
          tma_load_3d(s + ch * G::CHUNK_BYTES, &tmQ, &bars.qd_full[st], ch * G::EPC, it * 128, bh);
          tma_load_3d(s + G::TILE_BYTES + ch * G::CHUNK_BYTES, &tmdO, &bars.qd_full[st],
                      ch * G::EPC, it * 128, bh);
        }
        bulk_load(s + CST_OFF, p.cst + r0 * kCst, cbytes, &bars.qd_full[st]);
        if (tbytes) bulk_load(s + TAB_OFF, p.tabg + r0 * p.KT, tbytes, &bars.qd_full[st]);
      }
      mbar_wait(bars.kv_full, 0, abort);
      for (int st = 0; st < ns && st < nq; ++st)
        mbar_wait(&bars.qd_full[st], (((nq - st + ns - 1) / ns) - 1) & 1, abort);
    }
  } else if (warp == 1) {
    // S^T = K Q_h^T and dP^T = V dO_h^T of half h into TMEM pair h & 1, once
    // the dV / dK products of half h - 2 have read it
    if (lane == 0) {
      bool ok = mbar_wait(bars.kv_full, 0, abort);
      tc_fence_after();
      const uint32_t ka = smem_u32(sK), va = smem_u32(sV), sa = smem_u32(sSt);
      for (int h = 0; h < nh && ok; ++h) {
        const int n = h >> 1, e = h & 1, x = h & 1;
        if (e == 0) {
          ok = mbar_wait(&bars.qd_full[n % ns], (n / ns) & 1, abort);
          if (!ok) break;
          tc_fence_after();
        }
        if (h >= 2) {
          ok = mbar_wait(&bars.s_free[x], ((h >> 1) - 1) & 1, abort);
          if (!ok) break;
          tc_fence_after();
        }
        const uint32_t qb = sa + (n % ns) * SB + e * 64 * 128;
        mma_nt_half<D>(tmem + 128 * x, ka, qb);
        mma_nt_half<D>(tmem + 128 * x + 64, va, qb + G::TILE_BYTES);
        mma_commit(&bars.sdp_full[x]);
      }
      mma_commit(bars.drain);
      mbar_wait(bars.drain, 0, abort);
    }
  } else if (warp == 2) {
    // dV += P^T_h dO_h and dK += dS^T_h Q_h (A from TMEM, B MN-major)
    if (lane == 0) {
      bool ok = true;
      const uint32_t sa = smem_u32(sSt);
      for (int h = 0; h < nh && ok; ++h) {
        const int n = h >> 1, e = h & 1, x = h & 1;
        if (e == 0) {
          ok = mbar_wait(&bars.qd_full[n % ns], (n / ns) & 1, abort);
          if (!ok) break;
        }
        ok = mbar_wait(&bars.pds_full[x], (h >> 1) & 1, abort);
        if (!ok) break;
        tc_fence_after();
        const uint32_t qb = sa + (n % ns) * SB + e * 64 * 128;
        const uint32_t db = qb + G::TILE_BYTES;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint32_t acc = (h > 0 || kk > 0) ? 1u : 0u;
          mma_ts_f16(tmem + T_DV, tmem + 128 * x + 16 * kk,
                     smem_desc(db + kk * 16 * 128, G::CHUNK_BYTES, 1024), G::IDESC_MN, acc);
          mma_ts_f16(tmem + T_DK, tmem + 128 * x + 64 + 16 * kk,
                     smem_desc(qb + kk * 16 * 128, G::CHUNK_BYTES, 1024), G::IDESC_MN, acc);
        }
        mma_commit(&bars.s_free[x]);
        if (e == 1) mma_commit(&bars.qd_empty[n % ns]);
      }
      if (ok) mma_commit(bars.acc_full);
      mma_commit(bars.drain);
      mbar_wait(bars.drain, 0, abort);
    }
  } else if (warp >= 4) {
    const int g = (warp - 4) >> 2;
    const int key = (warp & 3) * 32 + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const int kg = kt * 128 + key;
    const bool key_ok = kg < p.S;
    const float Kf = static_cast<float>(p.K);
    bool ok = true;
    for (int h = 0; h < nh && ok; ++h) {
      const int n = h >> 1, e = h & 1, x = h & 1;
      if (e == 0) {
        // the stage's constants and tables have landed (the stage cannot
        // refill before this tile's products, which wait for these threads)
        ok = warp_all_b(mbar_wait(&bars.qd_full[n % ns], (n / ns) & 1, abort));
        if (!ok) break;
      }
      ok = warp_all_b(mbar_wait(&bars.sdp_full[x], (h >> 1) & 1, abort));
      if (!ok) break;
      tc_fence_after();
      const uint8_t *s = sSt + (n % ns) * SB;
      const float4 *cst4 = reinterpret_cast<const float4 *>(s + CST_OFF);
      const float2 *tabs = reinterpret_cast<const float2 *>(s + TAB_OFF);
      uint32_t sv[16], dv[16];
      tmem_ld16(lane_base + 128 * x + 16 * g, sv);
      tmem_ld16(lane_base + 128 * x + 64 + 16 * g, dv);
      tmem_wait_ld();
      reg_fence16(sv);
      reg_fence16(dv);
      const int qbase = (i0 + n) * 128 + 64 * e + 16 * g;   // first query row of the slice
      uint32_t pp[8], dd[8];
#pragma unroll
      for (int i2 = 0; i2 < 8; ++i2) {
        float p2[2], d2[2];
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          const int i = 2 * i2 + t;
          const int ql = 64 * e + 16 * g + i;              // query row within the tile
          const int qg = qbase + i;
          const bool valid = key_ok && qg < p.S && (!p.causal || kg <= qg);
          const float4 c0 = cst4[2 * ql], c1 = cst4[2 * ql + 1];
          float ds, gw, u, uc, kf;
          float2 gd;
          const float pw = bwd_elem<MAP>(__uint_as_float(sv[i]), __uint_as_float(dv[i]), c0, c1,
                                         tabs + ql * p.KT, 1, p, Kf, ds, gw, u, uc, kf, gd);
          p2[t] = valid ? pw : 0.0f;
          d2[t] = valid ? ds : 0.0f;
        }
        pp[i2] = pack_bf16x2(p2[0], p2[1]);
        dd[i2] = pack_bf16x2(d2[0], d2[1]);
      }
      tmem_st8(lane_base + 128 * x + 16 * g, pp);
      tmem_st8(lane_base + 128 * x + 64 + 16 * g, dd);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars.pds_full[x]);
    }
    if (ok) ok = warp_all_b(mbar_wait(bars.acc_full, 0, abort));
    if (ok) {
      tc_fence_after();
      const size_t krow = static_cast<size_t>(bh) * p.S + min(kg, p.S - 1);
      uint32_t v[16];
      tmem_ld16_sync(lane_base + T_DV + 16 * g, v);
      uint32_t pk[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) pk[i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
      if (key_ok) {
        uint4 *d4 = reinterpret_cast<uint4 *>(p.dV + krow * D + 16 * g);
        d4[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        d4[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
      }
      tmem_ld16_sync(lane_base + T_DK + 16 * g, v);
      float xk[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) xk[i] = __uint_as_float(v[i]) * p.c;
      if (p.dkcal != nullptr && key_ok) {
        const float4 *cal = reinterpret_cast<const float4 *>(p.dkcal + krow * D + 16 * g);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float4 c4 = cal[i];
          xk[4 * i] += c4.x;
          xk[4 * i + 1] += c4.y;
          xk[4 * i + 2] += c4.z;
          xk[4 * i + 3] += c4.w;
        }
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) pk[i] = pack_bf16x2(xk[2 * i], xk[2 * i + 1]);
      if (key_ok) {
        uint4 *d4 = reinterpret_cast<uint4 *>(p.dK + krow * D + 16 * g);
        d4[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        d4[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
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

// Raise a kernel's dynamic shared-memory limit once per device (a driver
// round trip otherwise paid on every call).
constexpr int kMaxDevices = 64;
template <typename F>
bool set_smem_once(F kern, int bytes, std::atomic<int> (&cache)[kMaxDevices]) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (dev >= 0 && dev < kMaxDevices && cache[dev].load(std::memory_order_acquire) >= bytes)
    return true;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
      cudaSuccess)
    return false;
  if (dev >= 0 && dev < kMaxDevices) {
    int prev = cache[dev].load(std::memory_order_relaxed);
    while (prev < bytes &&
           !cache[dev].compare_exchange_weak(prev, bytes, std::memory_order_acq_rel)) {
    }
  }
  return true;
}

constexpr size_t kMaxSmem = 232448;                      // 227 KB opt-in per CTA

template <int D, int MAP>
qsm_status launch_passes(const BwdArgs &a, BwdParams p, const CUtensorMap &mq,
                         const CUtensorMap &mk, const CUtensorMap &mv, const CUtensorMap &mdo) {
  using G = BGeo<D>;
  const int BH = a.B * a.H;
  const size_t bar_bytes = ((2 * 8 + 16) * 8 + 8 + 15) & ~static_cast<size_t>(15);
  {
    // dQ pass: Q, dO, ns x (K, V), 2 dS buffers, table, partial sums, barriers
    const size_t tab = static_cast<size_t>(p.K + 1) * 128 * sizeof(float2);
    const size_t fixed = 1024 + 2 * G::TILE_BYTES + 2 * 128 * 128 + tab + 2 * 4 * 128 * 4 + bar_bytes;
    int ns = static_cast<int>((kMaxSmem - fixed) / (2 * G::TILE_BYTES));
    if (ns > 4) ns = 4;
    if (ns < 2) return QSM_ERR_UNSUPPORTED;
    BwdParams q = p;
    q.num_stages = ns;
    q.ds_off = static_cast<uint32_t>(2 * G::TILE_BYTES + ns * 2 * G::TILE_BYTES);
    q.tab_off = q.ds_off + 2 * 128 * 128;
    q.part_off = static_cast<uint32_t>(q.tab_off + tab);
    q.bar_off = q.part_off + 2 * 4 * 128 * 4;
    size_t smem = 1024 + q.bar_off + bar_bytes;
    if (smem < 120 * 1024) smem = 120 * 1024;            // one CTA per SM (all of TMEM)
    if (smem > kMaxSmem) return QSM_ERR_UNSUPPORTED;
    auto kern = qsm_bwd_dq<D, MAP>;
    static std::atomic<int> cache[kMaxDevices];
    if (!set_smem_once(kern, static_cast<int>(smem), cache)) return QSM_ERR_CUDA;
    kern<<<dim3(p.nqt, BH), kMainThreads, smem, a.stream>>>(mq, mk, mv, mdo, q);
    if (cudaGetLastError() != cudaSuccess) return QSM_ERR_CUDA;
  }
  {
    // dK/dV pass: K, V, ns x (Q, dO, constants, tables), barriers
    const size_t tabb = (MAP == MAPB_EXACT || MAP == MAPB_POT) ? 0 : static_cast<size_t>(128) * p.KT * 8;
    const size_t stage = (2 * G::TILE_BYTES + 128 * kCst * 4 + tabb + 1023) & ~static_cast<size_t>(1023);
    const size_t fixed = 1024 + 2 * G::TILE_BYTES + bar_bytes;
    int ns = static_cast<int>((kMaxSmem - fixed) / stage);
    if (ns > 4) ns = 4;
    if (ns < 2) return QSM_ERR_UNSUPPORTED;
    BwdParams k = p;
    k.num_stages = ns;
    k.stage_bytes = static_cast<uint32_t>(stage);
    k.bar_off = static_cast<uint32_t>(2 * G::TILE_BYTES + ns * stage);
    size_t smem = 1024 + k.bar_off + bar_bytes;
    if (smem < 120 * 1024) smem = 120 * 1024;
    if (smem > kMaxSmem) return QSM_ERR_UNSUPPORTED;
    auto kern = qsm_bwd_dkdv<D, MAP>;
    static std::atomic<int> cache[kMaxDevices];
    if (!set_smem_once(kern, static_cast<int>(smem), cache)) return QSM_ERR_CUDA;
    kern<<<dim3(p.nkvt, BH), kMainThreads, smem, a.stream>>>(mq, mk, mv, mdo, k);
    if (cudaGetLastError() != cudaSuccess) return QSM_ERR_CUDA;
  }
  return QSM_OK;
}

template <int D>
qsm_status launch_rows(const BwdArgs &a, BwdParams p, const CUtensorMap &mq,
                       const CUtensorMap &mk, const CUtensorMap &mv, const CUtensorMap &mdo) {
  using G = BGeo<D>;
  const size_t tab = static_cast<size_t>(128) * (p.K + 1) * sizeof(float2);
  BwdParams r = p;
  r.tab_off = static_cast<uint32_t>(2 * G::TILE_BYTES + 4 * G::TILE_BYTES);
  r.cst_off = static_cast<uint32_t>((r.tab_off + tab + 15) & ~static_cast<size_t>(15));
  r.bar_off = static_cast<uint32_t>(r.cst_off + 5 * 4 * 128 * sizeof(float));
  size_t smem = 1024 + r.bar_off + 256;
  if (smem < 120 * 1024) smem = 120 * 1024;
  if (smem > kMaxSmem) return QSM_ERR_UNSUPPORTED;
  auto kern = (p.map == MAPB_HARD) ? qsm_bwd_rows<D, MAPB_HARD> : qsm_bwd_rows<D, MAPB_INTERP>;
  static std::atomic<int> cache_h[kMaxDevices], cache_i[kMaxDevices];
  if (!set_smem_once(kern, static_cast<int>(smem), p.map == MAPB_HARD ? cache_h : cache_i))
    return QSM_ERR_CUDA;
  kern<<<dim3(p.nqt, a.B * a.H), kMainThreads, smem, a.stream>>>(mq, mk, mv, mdo, r);
  return cudaGetLastError() == cudaSuccess ? QSM_OK : QSM_ERR_CUDA;
}

constexpr int kTabKT = (kBwdMaxK + 2) & ~1;              // table row stride in the workspace

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

}  // namespace

size_t bwd_workspace_bytes(int B, int H, int S, int D) {
  // fp32 calibration part of dK, then per query row: the row workspace, the
  // map constants and the grid table; each part 256-byte aligned
  const size_t rows = static_cast<size_t>(B) * H * S;
  return align256(rows * D * sizeof(float)) + align256(rows * kRowWs * sizeof(float)) +
         align256(rows * kCst * sizeof(float)) + align256(rows * kTabKT * sizeof(float2));
}

qsm_status launch_bwd(const BwdArgs &a) {
  if (a.D != 64) return QSM_ERR_UNSUPPORTED;          // TMEM schedule holds D = 64
  if (a.mode == QSM_MODE_KINTERVAL && a.Kint > kBwdMaxK) return QSM_ERR_UNSUPPORTED;
  const size_t rows = static_cast<size_t>(a.B) * a.H * a.S;
  BwdParams p{};
  p.S = a.S;
  p.nqt = (a.S + 127) / 128;
  p.nkvt = p.nqt;
  p.causal = a.causal;
  p.map = a.mode == QSM_MODE_EXACT       ? MAPB_EXACT
          : a.mode == QSM_MODE_ROWMAX_POT ? MAPB_POT
          : (a.rounding == QSM_ROUND_HARD ? MAPB_HARD : MAPB_INTERP);
  p.pot_floor = a.pot_floor;
  p.K = a.mode == QSM_MODE_KINTERVAL ? a.Kint : 1;
  p.fixed_window = a.calib == QSM_CALIB_FIXED_WINDOW;
  p.flush = a.below_policy == 1;
  p.surrogate = a.surrogate;
  p.detach = a.detach;
  p.calib = a.mode == QSM_MODE_KINTERVAL && !a.detach;
  p.KT = (p.K + 2) & ~1;
  p.c = a.c;
  p.cL2E = a.c * 1.4426950408889634f;
  p.window = a.window;
  p.LSE = a.LSE;
  p.hi = a.row_hi;
  p.lo = a.row_lo;
  p.amax = a.row_argmax;
  p.amin = a.row_argmin;
  uint8_t *ws = static_cast<uint8_t *>(a.workspace);
  const size_t o_dk = 0;
  const size_t o_rw = o_dk + align256(rows * a.D * sizeof(float));
  const size_t o_cst = o_rw + align256(rows * kRowWs * sizeof(float));
  const size_t o_tab = o_cst + align256(rows * kCst * sizeof(float));
  p.dkcal = p.calib ? reinterpret_cast<float *>(ws + o_dk) : nullptr;
  p.rowws = reinterpret_cast<float *>(ws + o_rw);
  p.cst = reinterpret_cast<float *>(ws + o_cst);
  p.tabg = reinterpret_cast<float2 *>(ws + o_tab);
  p.Q = static_cast<const __nv_bfloat16 *>(a.Q);
  p.K_ = static_cast<const __nv_bfloat16 *>(a.K);
  p.dQ = static_cast<__nv_bfloat16 *>(a.dQ);
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

  if (p.dkcal != nullptr &&
      cudaMemsetAsync(p.dkcal, 0, rows * a.D * sizeof(float), a.stream) != cudaSuccess)
    return QSM_ERR_CUDA;
  const long long nrows = static_cast<long long>(rows);
  qsm_bwd_delta<<<static_cast<unsigned>((nrows + 7) / 8), 256, 0, a.stream>>>(
      static_cast<const __nv_bfloat16 *>(a.O), static_cast<const __nv_bfloat16 *>(a.dO), p.rowws,
      nrows, a.D);
  if (cudaGetLastError() != cudaSuccess) return QSM_ERR_CUDA;
  if (a.mode != QSM_MODE_EXACT && a.surrogate == QSM_SURR_POST) {
    // LSE* and delta* of the post surrogate (for Rowmax-PoT without the
    // calibration sums, which it does not have)
    BwdParams r = p;
    if (p.map == MAPB_POT) {
      r.map = MAPB_HARD;
      r.detach = 1;
    }
    qsm_status st = launch_rows<64>(a, r, mq, mk, mv, mdo);
    if (st != QSM_OK) return st;
  }
  qsm_bwd_prep<<<static_cast<unsigned>((nrows + 255) / 256), 256, 0, a.stream>>>(p, nrows);
  if (cudaGetLastError() != cudaSuccess) return QSM_ERR_CUDA;
  if (p.map == MAPB_EXACT) return launch_passes<64, MAPB_EXACT>(a, p, mq, mk, mv, mdo);
  if (p.map == MAPB_POT) return launch_passes<64, MAPB_POT>(a, p, mq, mk, mv, mdo);
  if (p.map == MAPB_HARD) return launch_passes<64, MAPB_HARD>(a, p, mq, mk, mv, mdo);
  return launch_passes<64, MAPB_INTERP>(a, p, mq, mk, mv, mdo);
}

}  // namespace qsm
