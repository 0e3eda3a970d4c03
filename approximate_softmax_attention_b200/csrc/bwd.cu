// bwd.cu -- backward of the fused attention for the exact map, K-interval
// attention and Rowmax-PoT ("Pretraining Transformers with Quantized Softmax
// in Attention", abstract: backward rules including calibration derivatives,
// and a straight-through surrogate placed before or after normalization).
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
// Within one grid interval both calibration derivatives are affine in the
// coordinate u: interpolation dF/dhi = A_k + B_k u and dF/dhi + dF/dlo =
// -d_k K/(hi - lo); hard rounding dF/dhi = -dF/dlo = (n - K)/K g_n; fixed
// window dF/dhi = -d_k K/W.  Each element therefore costs one table read and
// at most three FMAs for them (the per-node coefficients are built once per
// row).
//
// Kernels, in launch order on the caller's stream:
//   1. qsm_bwd_rows   post surrogate only: LSE* and delta* per query row, sums
//                     of 2^((s - hi) log2 e) at the forward's row maximum over
//                     whole S and dP tiles (persistent)
//   2. qsm_bwd_prep   one CTA per query tile, two or four threads a row: delta =
//                     dO . O, the map constants and grid tables of both
//                     passes, into the workspace; zeroes the tile's rows of
//                     the fp32 calibration part of dK
//   3. qsm_bwd_dq     persistent, one CTA per SM over the query tiles: a tile's
//                     constants and table copied in, then the key tiles in
//                     halves of 64 keys: S = Q K^T and dP = dO V^T into one of
//                     three TMEM pairs, dS by the rule above into shared
//                     memory, dQ += dS K in TMEM (two accumulators, by tile
//                     parity); the calibration sums accumulate per row.  A
//                     tile's dQ is read out after the next tile's halves: the
//                     rank-one terms are added to dQ (fp32) before its bf16
//                     store and the dK ones are scattered into an fp32 buffer
//   4. qsm_bwd_dkdv   persistent over the key tiles, sweeping the query tiles
//                     in halves of 64 rows: S^T = K Q^T, dP^T = V dO^T into one
//                     of three TMEM pairs, P^T and dS^T written back to TMEM,
//                     dV += P^T dO and dK += dS^T Q in TMEM; dK gets the fp32
//                     calibration part before its bf16 store
// Each pass recomputes its products, so no dQ partial sums cross CTAs; the
// buffered halves let the map of one half overlap the products of the next.
// The element code is specialised per map, surrogate and calibration form,
// so no per-element branch remains.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>

#include "internal.h"
#include "sm100.cuh"
#include "wmap.cuh"

namespace qsm {

namespace {

// warp 0 TMA, warps 1-2 MMA, warps 4-19 four map groups of 128 threads
constexpr int kMainThreads = 640;
constexpr int kMainMapThreads = 512;
// The dQ and dK/dV passes keep three halves in flight (TMEM buffers, and dS
// tiles in the dQ pass): a buffer's round trip through the products that
// read it and refill it overlaps the map of the two halves in between.
constexpr int kHalfBufs = 3;
constexpr uint32_t kBwdTmemCols = 512;
constexpr int kRowWs = 8;               // floats per row in the row workspace
enum RowWs { RW_LSESTAR = 0, RW_DELTASTAR = 1 };
constexpr int kBwdMaxK = 32;            // largest K the backward accepts
constexpr int kCst = 8;                 // floats of one query row's map constants
constexpr float kL2E = 1.4426950408889634f;

constexpr int MAPB_EXACT = 0, MAPB_POT = 1, MAPB_HARD = 2, MAPB_INTERP = 3;
constexpr int SURR_NONE = QSM_SURR_NONE, SURR_PRE = QSM_SURR_PRE, SURR_POST = QSM_SURR_POST;
// calibration form of the dQ pass: none (detached, or fixed-window hard
// rounding, whose weights do not move with hi), min-max, fixed window
constexpr int CAL_OFF = 0, CAL_MINMAX = 1, CAL_FIXED = 2;

struct BwdParams {
  int S, nqt, nkvt, BH;
  int causal;
  int hgroup;       // causal query-tile order: heads per group (see q_tile_of)
  int K, fixed_window, flush, pot_floor;
  int TS;           // floats of one query row's dK / dV pass table (a multiple of 4)
  float c, cL2E, window;
  float gq, gk;     // gradient scales: dQ = gq dS K, dK = gk dS^T Q (c, or for
                    // e4m3 the score scale with one descale each: see launch_bwd)
  const float *LSE, *hi, *lo;
  const int32_t *amax, *amin;
  float *rowws;     // [rows][kRowWs]: LSE*, delta* (post surrogate)
  float *cst;       // [tile rows / 2][16]: row pairs' constants, interleaved (cst_index)
  float *tabk;      // [tile rows][TS]: the dK / dV pass's grid table of each row
  uint8_t *tabq;    // [query tiles][tabq_tile bytes]: the dQ pass's table of each tile
  float *dkcal;     // [rows][D] fp32 calibration part of dK (nullptr: none)
  const __nv_bfloat16 *Q, *K_, *O, *dO;
  __nv_bfloat16 *dQ, *dK, *dV;
  int32_t *status;
  int num_stages;
  uint32_t tabq_tile;   // bytes of one tile's dQ-pass table (0: none)
  uint32_t tab_off, ds_off, bar_off, part_off, stage_bytes, cst_off;
};

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
// at the start of a 1024-byte swizzle atom).  A is a whole 128-row tile
// (64-column chunks 16 KB apart); B's chunks sit BCH bytes apart (16 KB
// within a whole tile, 8 KB in a 64-row stage).
template <int D, int BCH = 128 * 128>
__device__ __forceinline__ void mma_nt_half(uint32_t d_tmem, uint32_t a_saddr, uint32_t b_saddr) {
  using G = BGeo<D>;
#pragma unroll
  for (int kk = 0; kk < G::KSTEPS_D; ++kk) {
    const int e = kk * 16;
    const uint32_t offa = (e / G::EPC) * G::CHUNK_BYTES + (e % G::EPC) * 2;
    const uint32_t offb = (e / G::EPC) * BCH + (e % G::EPC) * 2;
    mma_ss_f16(d_tmem, smem_desc(a_saddr + offa, 16, 1024), smem_desc(b_saddr + offb, 16, 1024),
               G::IDESC_H, kk > 0);
  }
}

// The (head, query tile) of query tile number b of nqt * BH: non-causal
// head after head; causal in groups of hgroup heads (their K / V share L2),
// heaviest tiles first within a group.
__device__ __forceinline__ void q_tile_of(const BwdParams &p, int b, int &bh, int &qt) {
  if (p.causal) {
    const int per = p.hgroup * p.nqt;
    const int grp = b / per;
    const int within = b - grp * per;
    const int h0 = grp * p.hgroup;
    const int gh = min(p.hgroup, p.BH - h0);
    const int rank = within / gh;
    bh = h0 + (within - rank * gh);
    qt = p.nqt - 1 - rank;
  } else {
    qt = b % p.nqt;
    bh = b / p.nqt;
  }
}

// The (head, key tile) of key tile number b of nkvt * BH: non-causal head
// after head; causal in groups of hgroup heads, heaviest (lowest) key tiles
// first within a group.
__device__ __forceinline__ void kv_tile_of(const BwdParams &p, int b, int &bh, int &kt) {
  if (p.causal) {
    const int per = p.hgroup * p.nkvt;
    const int grp = b / per;
    const int within = b - grp * per;
    const int h0 = grp * p.hgroup;
    const int gh = min(p.hgroup, p.BH - h0);
    kt = within / gh;
    bh = h0 + (within - kt * gh);
  } else {
    kt = b % p.nkvt;
    bh = b / p.nkvt;
  }
}

// Tile number of this CTA's round k in a persistent pass: the heaviest-first
// tile list is dealt out in rounds of gridDim.x tiles, in block order in the
// even rounds and in reverse block order in the odd ones, so that the CTA
// that takes a round's heaviest tile takes the lightest of the next (dealing
// in block order every round leaves the low blocks the heaviest tile of each
// round).  Strictly increasing in k: the first number >= the tile count ends
// the CTA's sequence.
__device__ __forceinline__ int cta_tile(int k) {
  const int g = static_cast<int>(gridDim.x), b = static_cast<int>(blockIdx.x);
  return k * g + ((k & 1) ? g - 1 - b : b);
}

// bf16 bit patterns to fp32 (exact).
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ float dot_bf16x8(uint4 a, uint4 b, float acc) {
  const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    acc = __fmaf_rn(bf_lo(aw[k]), bf_lo(bw[k]), acc);
    acc = __fmaf_rn(bf_hi(aw[k]), bf_hi(bw[k]), acc);
  }
  return acc;
}

// Sixteen bf16 (two uint4, already loaded) to fp32.
__device__ __forceinline__ void bf16x16_to_f32(const uint4 (&src)[2], float (&x)[16]) {
  const uint4 a = src[0], b = src[1];
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    x[2 * k] = bf_lo(w[k]);
    x[2 * k + 1] = bf_hi(w[k]);
  }
}

__device__ __forceinline__ float2 ex2_pair(float2 x) {
  return make_float2(ex2_approx(x.x), ex2_approx(x.y));
}

// ----------------------------------------------------------------- rows
struct RowBars {
  uint64_t *kv_full, *kv_empty;       // [ns]: K_j, V_j
  uint64_t *q_full, *q_free;          // Q, dO of the current tile
  uint64_t *sdp_full, *sdp_free;      // [2]: S, dP of a key tile
  uint64_t *part_ready, *part_free;   // [2]: a tile's partial sums written / read
  uint64_t *drain;
  uint32_t *tmem_slot;
  int *abort;
};

// The post surrogate's row statistics: LSE* = log sum_j exp(s_j) and delta*
// = sum_j p*_j dp_j.  The forward's row maximum hi bounds every score, so the
// sums are taken at the fixed offset hi (no running maximum, no rescaling):
// L = sum_j 2^(x_j), A = sum_j 2^(x_j) dp_j with x_j = (s_j - hi) log2 e, and
// LSE* = hi + ln L, delta* = A / L.
// Persistent like the dQ pass: one CTA per SM takes the query tiles
// cta_tile(0), cta_tile(1), ...; S = Q K^T and dP = dO V^T of whole
// 128-key tiles (products of N = 128: the map here is light, so the products
// set the pace) in TMEM pair n mod 2 (n counting key tiles across query
// tiles; S at 256 (n mod 2), dP 128 columns on); thread = query row, map
// group g owning keys 32g .. 32g+31 of each tile.  A query tile's sums go
// through shared memory (buffer k mod 2), and the group-0 threads combine
// them after the next tile's key tiles.
template <int D>
__global__ void __launch_bounds__(kMainThreads, 1)
    qsm_bwd_rows(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                 const BwdParams p) {
  using G = BGeo<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = smem_align1024(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntiles = p.nqt * p.BH;
  const int ns = p.num_stages;
  uint8_t *sQ = smem;
  uint8_t *sdO = smem + G::TILE_BYTES;
  uint8_t *sKV = smem + 2 * G::TILE_BYTES;              // ns stages of (K_j, V_j)
  float *part = reinterpret_cast<float *>(smem + p.part_off);   // [2][2][4][128]
  uint64_t *bp = reinterpret_cast<uint64_t *>(smem + p.bar_off);
  RowBars bars;
  bars.kv_full = bp;
  bars.kv_empty = bp + ns;
  bars.q_full = bp + 2 * ns;
  bars.q_free = bars.q_full + 1;
  bars.sdp_full = bars.q_free + 1;
  bars.sdp_free = bars.sdp_full + 2;
  bars.part_ready = bars.sdp_free + 2;
  bars.part_free = bars.part_ready + 2;
  bars.drain = bars.part_free + 2;
  bars.tmem_slot = reinterpret_cast<uint32_t *>(bars.drain + 1);
  bars.abort = reinterpret_cast<int *>(bars.tmem_slot + 1);
  volatile int *abort = bars.abort;

  if (threadIdx.x == 0) {
    for (int i = 0; i < ns; ++i) {
      mbar_init(&bars.kv_full[i], 1);
      mbar_init(&bars.kv_empty[i], 1);
    }
    mbar_init(bars.q_full, 1);
    mbar_init(bars.q_free, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.sdp_full[i], 1);
      mbar_init(&bars.sdp_free[i], kMainMapThreads);
      mbar_init(&bars.part_ready[i], kMainMapThreads);
      mbar_init(&bars.part_free[i], kMainMapThreads);
    }
    mbar_init(bars.drain, 1);
    *bars.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(bars.tmem_slot, kBwdTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *bars.tmem_slot;
  // the prep kernel (launched as a dependent at D = 64) may start on the SMs
  // this grid frees; it waits for this grid before reading LSE* and delta*
  grid_dep_launch();

  if (warp == 0) {
    if (lane == 0) {
      bool ok = true;
      int it = 0, k = 0;
      for (int t = cta_tile(k); t < ntiles && ok; t = cta_tile(++k)) {
        int bh, qt;
        q_tile_of(p, t, bh, qt);
        const int nkv = p.causal ? min(p.nkvt, qt + 1) : p.nkvt;
        // Q, dO of the previous tile are no longer read
        if (k >= 1) ok = mbar_wait(bars.q_free, (k - 1) & 1, abort);
        if (!ok) break;
        mbar_expect_tx(bars.q_full, 2 * G::TILE_BYTES);
        for (int ch = 0; ch < G::CHUNKS; ++ch) {
          tma_load_3d(sQ + ch * G::CHUNK_BYTES, &tmQ, bars.q_full, ch * G::EPC, qt * 128, bh);
          tma_load_3d(sdO + ch * G::CHUNK_BYTES, &tmdO, bars.q_full, ch * G::EPC, qt * 128, bh);
        }
        for (int j = 0; j < nkv && ok; ++j, ++it) {
          const int st = it % ns;
          if (it >= ns) ok = mbar_wait(&bars.kv_empty[st], ((it / ns) - 1) & 1, abort);
          if (!ok) break;
          uint8_t *kdst = sKV + st * 2 * G::TILE_BYTES;
          mbar_expect_tx(&bars.kv_full[st], 2 * G::TILE_BYTES);
          for (int ch = 0; ch < G::CHUNKS; ++ch) {
            tma_load_3d(kdst + ch * G::CHUNK_BYTES, &tmK, &bars.kv_full[st], ch * G::EPC,
                        j * 128, bh);
            tma_load_3d(kdst + G::TILE_BYTES + ch * G::CHUNK_BYTES, &tmV, &bars.kv_full[st],
                        ch * G::EPC, j * 128, bh);
          }
        }
      }
      // every load issued must land before the CTA may exit
      if (k >= 1) mbar_wait(bars.q_full, (k - 1) & 1, abort);
      for (int st = 0; st < ns && st < it; ++st)
        mbar_wait(&bars.kv_full[st], (((it - st + ns - 1) / ns) - 1) & 1, abort);
    }
  } else if (warp == 1) {
    // S = Q K_j^T and dP = dO V_j^T of key tile j into TMEM pair n mod 2,
    // once the map threads have read the pair's previous use
    if (lane == 0) {
      bool ok = true;
      int it0 = 0, k = 0;
      const uint32_t qa = smem_u32(sQ), da = smem_u32(sdO), kva = smem_u32(sKV);
      for (int t = cta_tile(k); t < ntiles && ok; t = cta_tile(++k)) {
        int bh, qt;
        q_tile_of(p, t, bh, qt);
        const int nkv = p.causal ? min(p.nkvt, qt + 1) : p.nkvt;
        ok = mbar_wait(bars.q_full, k & 1, abort);
        tc_fence_after();
        for (int j = 0; j < nkv && ok; ++j) {
          const int n = it0 + j, x = n & 1, u = n >> 1;
          ok = mbar_wait(&bars.kv_full[n % ns], (n / ns) & 1, abort);
          if (ok && u >= 1) ok = mbar_wait(&bars.sdp_free[x], (u - 1) & 1, abort);
          if (!ok) break;
          tc_fence_after();
          const uint32_t kb = kva + (n % ns) * 2 * G::TILE_BYTES;
          mma_nt<D>(tmem + 256 * x, qa, kb);
          mma_nt<D>(tmem + 256 * x + 128, da, kb + G::TILE_BYTES);
          mma_commit(&bars.sdp_full[x]);
          mma_commit(&bars.kv_empty[n % ns]);
        }
        if (ok) mma_commit(bars.q_free);                // the tile's Q, dO are read
        it0 += nkv;
      }
      mma_commit(bars.drain);
      mbar_wait(bars.drain, 0, abort);
    }
  } else if (warp >= 4) {
    const int g = (warp - 4) >> 2;
    const int row = (warp & 3) * 32 + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const float2 cl2 = make_float2(p.cL2E, p.cL2E);
    // A finished tile (position kp, tile t): the group-0 thread of each row
    // combines the four groups' sums; every map thread then releases the
    // buffer.
    auto finish = [&](int t, int kp, float hi) -> bool {
      const int x = kp & 1;
      bool rok = true;
      if (g == 0) {
        rok = warp_all_b(mbar_wait(&bars.part_ready[x], static_cast<uint32_t>(kp >> 1) & 1u, abort));
        if (rok) {
          int bh, qt;
          q_tile_of(p, t, bh, qt);
          const int qrow = qt * 128 + row;
          const float *pp = part + x * 1024;
          const float Ls = (pp[row] + pp[128 + row]) + (pp[256 + row] + pp[384 + row]);
          const float As = (pp[512 + row] + pp[640 + row]) + (pp[768 + row] + pp[896 + row]);
          // the loaded sums are consumed before the release
          asm volatile("" ::"f"(Ls), "f"(As) : "memory");
          if (qrow < p.S) {
            float *w = p.rowws + (static_cast<size_t>(bh) * p.S + qrow) * kRowWs;
            w[RW_LSESTAR] = hi + logf(Ls);
            w[RW_DELTASTAR] = As / Ls;
          }
        }
      }
      mbar_arrive(&bars.part_free[x]);
      return rok;
    };
    auto row_hi = [&](int t) -> float {
      int bh, qt;
      q_tile_of(p, t, bh, qt);
      return p.hi[static_cast<size_t>(bh) * p.S + min(qt * 128 + row, p.S - 1)];
    };
    bool ok = true;
    int n = 0, k = 0;
    float pv_hi = 0.0f;
    float hi_next = cta_tile(0) < ntiles ? row_hi(cta_tile(0)) : 0.0f;
    for (int t = cta_tile(k); t < ntiles && ok; t = cta_tile(++k)) {
      int bh, qt;
      q_tile_of(p, t, bh, qt);
      const int nkv = p.causal ? min(p.nkvt, qt + 1) : p.nkvt;
      const int qrow = qt * 128 + row;
      const int L = p.causal ? min(qrow + 1, p.S) : p.S;
      const float hi = hi_next;
      const int t_next = cta_tile(k + 1);
      if (t_next < ntiles) hi_next = row_hi(t_next);          // consumed a tile later
      const float hl = __fmul_rn(hi, log2e_f());
      const float2 nh = make_float2(-hl, -hl);
      float2 l2 = make_float2(0.0f, 0.0f), a2 = make_float2(0.0f, 0.0f);
      for (int j = 0; j < nkv && ok; ++j, ++n) {
        const int x = n & 1, u = n >> 1;
        ok = warp_all_b(mbar_wait(&bars.sdp_full[x], u & 1, abort));
        if (!ok) break;
        tc_fence_after();
        uint32_t sv[32], dv[32];
        tmem_ld32(lane_base + 256 * x + 32 * g, sv);
        tmem_ld32(lane_base + 256 * x + 128 + 32 * g, dv);
        tmem_wait_ld();
        reg_fence32(sv);
        reg_fence32(dv);
        tc_fence_before();
        mbar_arrive(&bars.sdp_free[x]);                // the pair can take key tile n + 2
        const int lim = L - (128 * j + 32 * g);        // valid keys of this slice
#pragma unroll
        for (int i2 = 0; i2 < 16; ++i2) {
          const float2 r = make_float2(__uint_as_float(sv[2 * i2]), __uint_as_float(sv[2 * i2 + 1]));
          const float2 dp =
              make_float2(__uint_as_float(dv[2 * i2]), __uint_as_float(dv[2 * i2 + 1]));
          float2 ev = ex2_pair(fma2_rn(r, cl2, nh));
          if (2 * i2 >= lim) ev.x = 0.0f;
          if (2 * i2 + 1 >= lim) ev.y = 0.0f;
          l2 = add2_rn(l2, ev);
          a2 = fma2_rn(ev, dp, a2);
        }
      }
      if (!ok) break;
      // this tile's sums, once the buffer's previous tile (k - 2) is combined
      if (k >= 2) {
        ok = warp_all_b(mbar_wait(&bars.part_free[k & 1], ((k >> 1) - 1) & 1, abort));
        if (!ok) break;
      }
      float *pp = part + (k & 1) * 1024;
      pp[g * 128 + row] = l2.x + l2.y;
      pp[512 + g * 128 + row] = a2.x + a2.y;
      mbar_arrive(&bars.part_ready[k & 1]);
      if (k >= 1 && !finish(cta_tile(k - 1), k - 1, pv_hi)) {
        ok = false;
        break;
      }
      pv_hi = hi;
    }
    if (ok && k >= 1) finish(cta_tile(k - 1), k - 1, pv_hi);
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kBwdTmemCols);
  if (threadIdx.x == 0 && *bars.abort && p.status != nullptr) atomicExch(p.status, QSM_ERR_TIMEOUT);
}

// The dK / dV pass evaluates the coordinate in the saturating form
// (fma_sat on the coordinate divided by K) when K = 2^m, unless the
// below-window flush or the no-surrogate rule needs what the saturation
// hides (the coordinate's sign, the below-window entry's zero derivative).
// The prep kernel lays the pass's table out for the same choice.
template <int SURR>
__device__ __forceinline__ bool kv_sat(const BwdParams &p) {
  return SURR != SURR_NONE && k_pow2(p.K) && p.flush == 0;
}

// ------------------------------------------------------------ row constants
// The constants of one query row, as both passes use them (registers in the
// dQ pass, the workspace copy cst in the dK / dV pass):
//   a, b   coordinate u = fma(r, a, b) on the raw product r (PoT: the
//          exponent coordinate, a = -c log2e, b = hi log2e); K-interval
//          with K = 2^m: a / K and b / K (exact), for the saturating form
//   invZ   1/Z, Z = exp(LSE - hi)
//   nDZ    -delta/Z, so that gw = fma(dp, invZ, nDZ)
//   e0     the surrogate's exponent offset in log2 units: exact LSE log2e,
//          pre hi log2e, post LSE* log2e (w* = 2^(r c log2e - e0))
//   ds_    delta (exact, no surrogate) or delta* (post)
//   kinv   K / (hi - lo): d coordinate / d score (0 for a degenerate row)
struct RowC {
  float a, b, invZ, nDZ, e0, ds_, kinv;
  bool calib;       // the row takes calibration terms
};

// Workspace rows are tile rows: (bh * nqt + qt) * 128 + row, so that every
// query tile starts a row pair.  The constants of rows 2m and 2m + 1 sit
// together, each field as a pair, so that one 16-byte load gives the packed
// operands of two rows: [a a' b b' | invZ invZ' nDZ nDZ' | -e0 -e0' -ds_ -ds_'
// | kinv kinv' cal cal'] (16 floats; cal = 1 when the row takes calibration
// terms, else 0).
__device__ __forceinline__ size_t tile_row(const BwdParams &p, int bh, int qt, int row) {
  return (static_cast<size_t>(bh) * p.nqt + qt) * 128 + row;
}
__device__ __forceinline__ void store_row_constants(const BwdParams &p, size_t trow, const RowC &k) {
  float *c = p.cst + (trow >> 1) * 16 + (trow & 1);
  c[0] = k.a;
  c[2] = k.b;
  c[4] = k.invZ;
  c[6] = k.nDZ;
  c[8] = -k.e0;
  c[10] = -k.ds_;
  c[12] = k.kinv;
  c[14] = k.calib ? 1.0f : 0.0f;
}

// Table layouts (K-interval).  Entry i of a row, interpolation, i = 0..K+1:
// i = 0 the below-window entry (fixed window: weight g_0, or 0 when flushed,
// no derivative; min-max: a copy of interval 0), i = k + 1 interval k =
// 0..K-1, i = K + 1 a copy of interval K - 1 (u = K).  The index is
// floor(clamp(u, -1, K)) + 1 from a round-down add of 1.5 * 2^23.  Hard
// rounding: entry n = 0..K at rne(clamp(u, 0, K)).
//   dQ pass (shared memory, [entry][128 rows]): interpolation with min-max
//   calibration (A, B, d, 0); interpolation otherwise d; hard rounding with
//   min-max calibration (n - K)/K g_n.
//   dK / dV pass (workspace, [row][TS]), times 1/Z (so that the lookup is P
//   itself): interpolation (e, d) pairs with P = fma(u, d, e), on the
//   saturating path (kv_sat) (e, K d) with P = fma(u / K, K d, e); hard
//   rounding g_n.
template <int MAP, int SURR, int CAL>
struct DqTab {
  static constexpr bool KI = MAP == MAPB_HARD || MAP == MAPB_INTERP;
  static constexpr bool ANY = KI && (CAL != CAL_OFF || (MAP == MAPB_INTERP && SURR == SURR_NONE));
  static constexpr int ESZ = (MAP == MAPB_INTERP && CAL == CAL_MINMAX) ? 16 : 4;
  static constexpr int STRIDE = ESZ * 128;
  static constexpr int entries(int K) { return MAP == MAPB_INTERP ? K + 2 : K + 1; }
  static constexpr size_t bytes(int K) {
    return ANY ? static_cast<size_t>(entries(K)) * STRIDE : 0;
  }
};

// The constants of one query row before delta is known, and (K-interval) its
// grid map.
template <int MAP, int SURR, int CAL>
__device__ __forceinline__ RowC row_constants(const BwdParams &p, size_t ri, RowMap &rm) {
  RowC k;
  k.a = k.b = k.invZ = k.nDZ = k.e0 = k.ds_ = k.kinv = 0.0f;
  k.calib = false;
  const float lse = p.LSE[ri];
  if (MAP == MAPB_EXACT) {
    k.e0 = __fmul_rn(lse, kL2E);
    return k;
  }
  const float hi = p.hi[ri];
  k.invZ = expf(__fsub_rn(hi, lse));
  if (MAP == MAPB_POT) {
    k.a = -p.cL2E;
    k.b = __fmul_rn(hi, log2e_f());
    k.e0 = k.b;
  } else {
    rm = make_rowmap(hi, p.lo != nullptr ? p.lo[ri] : hi, p.K, p.fixed_window != 0, p.window);
    k.a = rm.degenerate ? 0.0f : __fmul_rn(p.c, rm.inv);
    k.b = rm.degenerate ? static_cast<float>(p.K) : rm.b;
    if (k_pow2(p.K)) {
      // K = 2^m: kept divided by K (exact), the coordinate of the saturating
      // form fma_sat(r, a, b) = clamp(u, 0, K) / K
      const float invK = 1.0f / static_cast<float>(p.K);
      k.a = __fmul_rn(k.a, invK);
      k.b = __fmul_rn(k.b, invK);
    }
    k.e0 = rm.hiL2E;
    k.kinv = rm.inv;
    k.calib = CAL != CAL_OFF && !rm.degenerate;
  }
  if (SURR == SURR_POST) {
    const float *w = p.rowws + ri * kRowWs;
    k.e0 = __fmul_rn(w[RW_LSESTAR], kL2E);
    k.ds_ = w[RW_DELTASTAR];
  }
  return k;
}

// The grid tables of one row (K-interval), the part of thread q = 0..NQ-1
// of the row's NQ: the dK / dV pass's row tk (TS floats) and the dQ pass's
// entries, entry i at byte tq + i * STRIDE.  Thread q takes the intervals
// (interpolation) or grid values (hard rounding) k = q, q + NQ, ... and
// forms the grid values it needs itself; x/K is a product with 1/K when K
// is a power of two (exact, so the same value).
template <int MAP, int SURR, int CAL, int NQ>
__device__ __forceinline__ void row_tables(const BwdParams &p, const RowMap &rm, float invZ, int q,
                                           float *tk, uint8_t *tq) {
  using T = DqTab<MAP, SURR, CAL>;
  const int K = p.K;
  const float Kf = static_cast<float>(K);
  const bool sat = kv_sat<SURR>(p);
  const bool p2 = (K & (K - 1)) == 0;
  const float rK = 1.0f / Kf;
  auto divK = [&](float x) { return p2 ? __fmul_rn(x, rK) : __fdiv_rn(x, Kf); };
  if (MAP == MAPB_INTERP) {
    const float inv_a = rm.degenerate ? 0.0f : __fdiv_rn(1.0f, __fsub_rn(rm.hi, rm.lo));
    auto put = [&](int i, float e, float d, float A, float B) {
      *reinterpret_cast<float2 *>(tk + 2 * i) =
          make_float2(__fmul_rn(e, invZ), __fmul_rn(sat ? __fmul_rn(d, Kf) : d, invZ));
      if (CAL == CAL_MINMAX)
        *reinterpret_cast<float4 *>(tq + i * T::STRIDE) = make_float4(A, B, d, 0.0f);
      else if (T::ANY)
        *reinterpret_cast<float *>(tq + i * T::STRIDE) = d;
    };
    for (int kk = q; kk < K; kk += NQ) {
      const float gk = grid_value(rm, K, kk), gk1 = grid_value(rm, K, kk + 1);
      const float kf = static_cast<float>(kk), kmk = static_cast<float>(K - kk);
      const float d = __fsub_rn(gk1, gk);
      const float e = __fmaf_rn(-kf, d, gk);
      float A = 0.0f, B = 0.0f;
      if (CAL == CAL_MINMAX) {
        A = -divK(__fmaf_rn(kmk, e, __fmul_rn(kf, gk1)));
        B = __fsub_rn(-__fmul_rn(d, inv_a), divK(__fsub_rn(__fmul_rn(kmk, d), gk1)));
      }
      put(kk + 1, e, d, A, B);
      if (kk == 0) {
        // below the window: fixed window g_0 (0 when flushed), no
        // derivative; min-max: interval 0
        if (p.fixed_window)
          put(0, p.flush ? 0.0f : gk, 0.0f, 0.0f, 0.0f);
        else
          put(0, e, d, A, B);
      }
      if (kk == K - 1) put(K + 1, e, d, A, B);            // u = K: interval K - 1
    }
  } else {
    for (int n = q; n <= K; n += NQ) {
      const float g = grid_value(rm, K, n);
      tk[n] = __fmul_rn(g, invZ);
      if (T::ANY)
        *reinterpret_cast<float *>(tq + n * T::STRIDE) = __fmul_rn(divK(static_cast<float>(n - K)), g);
    }
  }
}

// ------------------------------------------------------------- e4m3 inputs
// The backward of an e4m3 forward runs on bf16 copies: the Q and K codes as
// they are (every e4m3 value is a bf16 value, so the recomputed scores are the
// forward's), the V codes times v_descale (rounded to bf16; dP = dO V~^T
// needs V~ itself).  Eight elements a thread step, as 8-byte loads and
// 16-byte stores.
__device__ __forceinline__ uint4 e4m3x8_to_bf16(uint2 w, float scale) {
  __nv_fp8x4_e4m3 lo, hi;
  lo.__x = w.x;
  hi.__x = w.y;
  const float4 a = static_cast<float4>(lo), b = static_cast<float4>(hi);
  return make_uint4(pack_bf16x2(__fmul_rn(a.x, scale), __fmul_rn(a.y, scale)),
                    pack_bf16x2(__fmul_rn(a.z, scale), __fmul_rn(a.w, scale)),
                    pack_bf16x2(__fmul_rn(b.x, scale), __fmul_rn(b.y, scale)),
                    pack_bf16x2(__fmul_rn(b.z, scale), __fmul_rn(b.w, scale)));
}

__global__ void __launch_bounds__(256)
    qsm_bwd_dequant(const uint2 *__restrict__ q8, const uint2 *__restrict__ k8,
                    const uint2 *__restrict__ v8, uint4 *qb, uint4 *kb, uint4 *vb, size_t n8,
                    float v_descale) {
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    qb[i] = e4m3x8_to_bf16(q8[i], 1.0f);
    kb[i] = e4m3x8_to_bf16(k8[i], 1.0f);
    vb[i] = e4m3x8_to_bf16(v8[i], v_descale);
  }
}

// ----------------------------------------------------------- row prep
// One CTA of 128 NQ threads per query tile, NQ threads a row (thread q of
// row r is thread 128 q + r; NQ = 4 for interpolation, whose tables are the
// longest, else 2): each row's delta = dO_r . O_r (four D/4-column parts,
// 4/NQ of them a thread), map constants and grid tables (thread q every
// NQ-th entry), written to the workspace -- the constants (both
// passes), the dK / dV pass's table per row (staged in shared memory, then
// copied out as one contiguous run per tile) and the dQ pass's table per
// tile in its shared-memory layout (entry-major, so the rows of a warp store
// one contiguous run), which the dQ pass copies in with one bulk load per
// tile.  The tile's rows of the fp32 calibration part of dK are zeroed here,
// ahead of the dQ pass's reductions into them.  Rows past S in a ragged last
// tile take the last row's values, so every workspace entry of a tile is
// defined.
constexpr int kTabKRow = 2 * ((kBwdMaxK + 2) & ~1);     // floats: the widest table row (TS)
template <int MAP>
constexpr int prep_split() { return MAP == MAPB_INTERP ? 4 : 2; }

template <int D, int MAP, int SURR, int CAL>
__global__ void __launch_bounds__(128 * prep_split<MAP>())
    qsm_bwd_prep(const BwdParams p) {
  using T = DqTab<MAP, SURR, CAL>;
  constexpr int NQ = prep_split<MAP>(), NT = 128 * NQ;
  static_assert(D == 64 || D == 128, "delta in four D/4-column parts");
  constexpr bool KI = MAP == MAPB_HARD || MAP == MAPB_INTERP;
  __shared__ float dpart[4][128];
  __shared__ __align__(16) float tks[KI ? 128 * kTabKRow : 4];
  // the dQ pass may start its prologue once every CTA of this grid runs
  grid_dep_launch();
  const int row = threadIdx.x & 127, q = threadIdx.x >> 7;
  const int tix = static_cast<int>(blockIdx.x);         // bh * nqt + qt
  const int bh = tix / p.nqt, qt = tix - bh * p.nqt;
  const int qrow = qt * 128 + row;
  const bool row_ok = qrow < p.S;
  const size_t ri = static_cast<size_t>(bh) * p.S + min(qrow, p.S - 1);
  {
    // this thread's parts of delta (parts q, q + NQ, ...), each a running
    // sum over its 8-column chunks
    constexpr int CPP = D / 32;                           // 8-column chunks per part
    constexpr int PPT = 4 / NQ;                           // parts per thread
    const uint4 *o4 = reinterpret_cast<const uint4 *>(p.O + ri * D);
    const uint4 *d4 = reinterpret_cast<const uint4 *>(p.dO + ri * D);
    uint4 ov[PPT][CPP], dv[PPT][CPP];
#pragma unroll
    for (int j = 0; j < PPT; ++j)
#pragma unroll
      for (int c = 0; c < CPP; ++c) {
        ov[j][c] = o4[CPP * (q + NQ * j) + c];
        dv[j][c] = d4[CPP * (q + NQ * j) + c];
      }
#pragma unroll
    for (int j = 0; j < PPT; ++j) {
      float acc = 0.0f;
#pragma unroll
      for (int c = 0; c < CPP; ++c) acc = dot_bf16x8(ov[j][c], dv[j][c], acc);
      dpart[q + NQ * j][row] = acc;
    }
  }
  if (p.dkcal != nullptr) {
    const int nrow = min(128, p.S - qt * 128);
    float4 *z = reinterpret_cast<float4 *>(p.dkcal + (static_cast<size_t>(bh) * p.S + qt * 128) * D);
    for (int i = static_cast<int>(threadIdx.x); i < nrow * (D / 4); i += NT)
      z[i] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  }
  RowMap rm{};
  // post surrogate at D = 64: launched as a dependent of the row pass, whose
  // LSE* and delta* the constants read (a no-op for a plain launch)
  if (SURR == SURR_POST) grid_dep_wait();
  RowC kc = row_constants<MAP, SURR, CAL>(p, ri, rm);
  if (KI)
    row_tables<MAP, SURR, CAL, NQ>(p, rm, kc.invZ, q, tks + row * p.TS,
                               p.tabq + static_cast<size_t>(tix) * p.tabq_tile + row * T::ESZ);
  __syncthreads();
  if (q == 0) {
    const float delta = (dpart[0][row] + dpart[1][row]) + (dpart[2][row] + dpart[3][row]);
    if (MAP == MAPB_EXACT || SURR == SURR_NONE) kc.ds_ = delta;
    if (MAP != MAPB_EXACT) kc.nDZ = -__fmul_rn(delta, kc.invZ);
    if (!row_ok) kc.calib = false;
    store_row_constants(p, tile_row(p, bh, qt, row), kc);
  }
  if (KI) {
    // the tile's table rows are contiguous in the workspace (TS a multiple
    // of four floats): 16-byte copies
    const int n4 = 32 * p.TS;
    const float4 *src = reinterpret_cast<const float4 *>(tks);
    float4 *dst = reinterpret_cast<float4 *>(p.tabk + static_cast<size_t>(tix) * 128 * p.TS);
    for (int i = static_cast<int>(threadIdx.x); i < n4; i += NT) dst[i] = src[i];
  }
}

// The dQ pass's per-row values for the element loop.
struct DqK {
  float a, b, invZ, nDZ, ne0, nds, kinv, cL2E, Kf;
  float mk;          // hard rounding, K = 2^m: 1.5 * 2^23 / K
  uint32_t tq_row;   // biased shared address of this row's dQ-pass table
};

// dS of one 16-key slice of a row (bf16 pairs into dd) and the calibration
// sums, two elements per packed fp32 operation.  FULL: every key valid.  SAT
// (hard rounding, K = 2^m): the node from the saturating coordinate, rne of
// fma_sat(r, a/K, b/K) at a unit of 1/K -- rne(clamp(u, 0, K)), the same node.
template <int MAP, int SURR, int CAL, bool FULL, bool SAT = false>
__device__ __forceinline__ void dq_slice(const uint32_t (&sv)[16], const uint32_t (&dv)[16],
                                         const DqK &k, int lim, uint32_t (&dd)[8], float2 &s1,
                                         float2 &s2) {
  using T = DqTab<MAP, SURR, CAL>;
  const float2 cl2 = make_float2(k.cL2E, k.cL2E), ne0 = make_float2(k.ne0, k.ne0);
  const float2 nds = make_float2(k.nds, k.nds);
  const float2 mg = make_float2(kMagic, kMagic);
#pragma unroll
  for (int i2 = 0; i2 < 8; ++i2) {
    const float2 r = make_float2(__uint_as_float(sv[2 * i2]), __uint_as_float(sv[2 * i2 + 1]));
    const float2 dp = make_float2(__uint_as_float(dv[2 * i2]), __uint_as_float(dv[2 * i2 + 1]));
    const bool v0 = FULL || 2 * i2 < lim, v1 = FULL || 2 * i2 + 1 < lim;
    float2 ds = make_float2(0.0f, 0.0f);
    if (MAP == MAPB_EXACT) {
      ds = mul2_rn(ex2_pair(fma2_rn(r, cl2, ne0)), add2_rn(dp, nds));
    } else {
      float2 gw = fma2_rn(dp, make_float2(k.invZ, k.invZ), make_float2(k.nDZ, k.nDZ));
      if (!v0) gw.x = 0.0f;
      if (!v1) gw.y = 0.0f;
      if (SURR == SURR_PRE)
        ds = mul2_rn(gw, ex2_pair(fma2_rn(r, cl2, ne0)));
      else if (SURR == SURR_POST)
        ds = mul2_rn(ex2_pair(fma2_rn(r, cl2, ne0)), add2_rn(dp, nds));
      if (T::ANY) {
        const float2 u = fma2_rn(r, make_float2(k.a, k.a), make_float2(k.b, k.b));
        if (MAP == MAPB_INTERP) {
          const float2 uc = make_float2(fminf(fmaxf(u.x, -1.0f), k.Kf), fminf(fmaxf(u.y, -1.0f), k.Kf));
          const float2 t = add2_rd(uc, mg);
          const uint32_t ad0 = __float_as_uint(t.x) * T::STRIDE + k.tq_row;
          const uint32_t ad1 = __float_as_uint(t.y) * T::STRIDE + k.tq_row;
          float2 d;
          if (CAL == CAL_MINMAX) {
            const float4 e0 = lds_f32x4(ad0), e1 = lds_f32x4(ad1);     // A, B, d
            s1 = fma2_rn(gw, make_float2(__fmaf_rn(e0.y, uc.x, e0.x), __fmaf_rn(e1.y, uc.y, e1.x)),
                         s1);
            d = make_float2(e0.z, e1.z);
            s2 = fma2_rn(gw, d, s2);
          } else {
            d = make_float2(lds_f32(ad0), lds_f32(ad1));
            if (CAL == CAL_FIXED) s2 = fma2_rn(gw, d, s2);
          }
          if (SURR == SURR_NONE) ds = mul2_rn(mul2_rn(gw, d), make_float2(k.kinv, k.kinv));
        } else {
          float2 t;
          if (SAT) {
            t = add2_rn(make_float2(fma_sat(r.x, k.a, k.b), fma_sat(r.y, k.a, k.b)),
                        make_float2(k.mk, k.mk));
          } else {
            const float2 uc =
                make_float2(fminf(fmaxf(u.x, 0.0f), k.Kf), fminf(fmaxf(u.y, 0.0f), k.Kf));
            t = add2_rn(uc, mg);
          }
          s1 = fma2_rn(gw,
                       make_float2(lds_f32(__float_as_uint(t.x) * T::STRIDE + k.tq_row),
                                   lds_f32(__float_as_uint(t.y) * T::STRIDE + k.tq_row)),
                       s1);
        }
      }
    }
    if (!v0) ds.x = 0.0f;
    if (!v1) ds.y = 0.0f;
    dd[i2] = pack_bf16x2(ds.x, ds.y);
  }
}

// ----------------------------------------------------------------- dQ pass
// Persistent: one CTA per SM takes the 128-row query tiles cta_tile(0),
// cta_tile(1), ... of the heaviest-first order; thread = query row
// (TMEM lane); the key tiles are taken in halves of 64 keys, half number hc
// (counted across tiles) in TMEM pair x = hc mod 3 (S at 128x, dP at 128x +
// 64) and shared dS buffer x; map group g owns keys 16g .. 16g+15 of each
// half.  The row constants and the table of a tile come from the prep kernel
// (warp 3 copies them in).  dQ of tile k accumulates in TMEM buffer k mod 2
// (columns 384 + 64 (k mod 2)), and the map threads read it out after the
// halves of tile k + 1: by then every map thread has finished tile k, so
// the read-out waits for no straggler and the products of tile k + 1 run
// meanwhile.
struct DqBars {
  uint64_t *kv_full, *kv_empty;       // [ns]: K_j, V_j
  uint64_t *q_full, *q_free;          // Q, dO of the current tile
  uint64_t *sdp_full, *sdp_free;      // [HB]
  uint64_t *ds_full, *ds_free;        // [HB]
  uint64_t *dq_full, *dq_free;        // [2]: a tile's dQ complete / read out of TMEM
  uint64_t *tab_full, *tab_free;      // the tile's constants and table
  uint64_t *part_ready, *part_free;   // [2]: a tile's calibration sums written / read
  uint64_t *drain;
  uint32_t *tmem_slot;
  int *abort;
};
// Geometry of the dQ pass: D = 64 keeps three TMEM pairs and whole key
// tiles per ring stage; D = 128 (accumulators of 128 columns) two pairs and
// half key tiles (64 keys) per stage.
template <int D>
struct DqGeo {
  static constexpr int HB = D > 64 ? 2 : 3;          // TMEM S / dP pairs, dS buffers
  static constexpr int KROWS = D > 64 ? 64 : 128;    // key rows per ring stage
  static constexpr int HPU = KROWS / 64;             // halves per stage
  static constexpr int KBYTES = KROWS * D * 2;       // the K (or V) rows of a stage
  static constexpr int KCHUNK = KROWS * 128;         // bytes between their 64-column chunks
  static constexpr uint32_t T_DQ = HB * 128;         // dQ accumulators: T_DQ + D (k mod 2)
  static constexpr int DG = D / 4;                   // dQ columns per map group
};

// The calibration state of a finished tile that its read-out needs: the
// tile, the row's argmax / argmin key (amx < 0: no calibration terms) and
// K/(hi - lo).
struct DqPrev {
  int t, amx, amn;
  float kinv;
};

template <int D, int MAP, int SURR, int CAL>
__global__ void __launch_bounds__(kMainThreads, 1)
    qsm_bwd_dq(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
               const BwdParams p) {
  using G = BGeo<D>;
  using T = DqTab<MAP, SURR, CAL>;
  using QG = DqGeo<D>;
  static_assert(D == 64 || D == 128, "dQ slices of the four map groups: D / 4 columns");
  constexpr int HB = QG::HB;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = smem_align1024(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntiles = p.nqt * p.BH;
  const int ns = p.num_stages;
  uint8_t *sQ = smem;
  uint8_t *sdO = smem + G::TILE_BYTES;
  uint8_t *sKV = smem + 2 * G::TILE_BYTES;              // ns stages of (K_j, V_j)
  uint8_t *sDS = smem + p.ds_off;                        // 3 x 128 rows x 128 bytes
  uint8_t *sCst = smem + p.cst_off;                      // 64 row pairs x 16 floats
  float *part = reinterpret_cast<float *>(smem + p.part_off);   // [2][2][4][128]
  uint64_t *bp = reinterpret_cast<uint64_t *>(smem + p.bar_off);
  DqBars bars;
  bars.kv_full = bp;
  bars.kv_empty = bp + ns;
  bars.q_full = bp + 2 * ns;
  bars.q_free = bars.q_full + 1;
  bars.sdp_full = bars.q_free + 1;
  bars.sdp_free = bars.sdp_full + HB;
  bars.ds_full = bars.sdp_free + HB;
  bars.ds_free = bars.ds_full + HB;
  bars.dq_full = bars.ds_free + HB;
  bars.dq_free = bars.dq_full + 2;
  bars.tab_full = bars.dq_free + 2;
  bars.tab_free = bars.tab_full + 1;
  bars.part_ready = bars.tab_free + 1;
  bars.part_free = bars.part_ready + 2;
  bars.drain = bars.part_free + 2;
  bars.tmem_slot = reinterpret_cast<uint32_t *>(bars.drain + 1);
  bars.abort = reinterpret_cast<int *>(bars.tmem_slot + 1);
  volatile int *abort = bars.abort;

  if (threadIdx.x == 0) {
    for (int i = 0; i < ns; ++i) {
      mbar_init(&bars.kv_full[i], 1);
      mbar_init(&bars.kv_empty[i], 1);
    }
    mbar_init(bars.q_full, 1);
    mbar_init(bars.q_free, 1);
    for (int i = 0; i < HB; ++i) {
      mbar_init(&bars.sdp_full[i], 1);
      mbar_init(&bars.sdp_free[i], kMainMapThreads);
      mbar_init(&bars.ds_full[i], kMainMapThreads);
      mbar_init(&bars.ds_free[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.dq_full[i], 1);
      mbar_init(&bars.dq_free[i], kMainMapThreads);
      mbar_init(&bars.part_ready[i], kMainMapThreads);
      mbar_init(&bars.part_free[i], kMainMapThreads);
    }
    mbar_init(bars.tab_full, 1);
    mbar_init(bars.tab_free, kMainMapThreads);
    mbar_init(bars.drain, 2);
    *bars.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(bars.tmem_slot, kBwdTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *bars.tmem_slot;
  // The prologue above may overlap the prep kernel's last CTAs; its
  // constants and tables (and the e4m3 path's bf16 copies) are complete from
  // here on.  Then the dK/dV pass may start on the SMs this grid frees.
  grid_dep_wait();
  grid_dep_launch();

  // Tiles of this CTA: cta_tile(0), cta_tile(1), ... of the heaviest-first
  // order (persistent: the next tile's loads and first
  // products overlap this tile's last halves).  Every role walks the same
  // sequence; the ring position `it` and the half counter `hc` run on across
  // tiles, and per-tile barriers take the tile's own parity.
  if (warp == 0) {
    if (lane == 0) {
      bool ok = true;
      int it = 0, k = 0;
      for (int t = cta_tile(k); t < ntiles && ok; t = cta_tile(++k)) {
        int bh, qt;
        q_tile_of(p, t, bh, qt);
        const int nkv = p.causal ? min(p.nkvt, qt + 1) : p.nkvt;
        // Q, dO of the previous tile are no longer read
        if (k >= 1) ok = mbar_wait(bars.q_free, (k - 1) & 1, abort);
        if (!ok) break;
        mbar_expect_tx(bars.q_full, 2 * G::TILE_BYTES);
        for (int ch = 0; ch < G::CHUNKS; ++ch) {
          tma_load_3d(sQ + ch * G::CHUNK_BYTES, &tmQ, bars.q_full, ch * G::EPC, qt * 128, bh);
          tma_load_3d(sdO + ch * G::CHUNK_BYTES, &tmdO, bars.q_full, ch * G::EPC, qt * 128, bh);
        }
        // one stage per KROWS keys (K / V tensor maps of KROWS-row boxes)
        for (int j = 0; j < nkv * (128 / QG::KROWS) && ok; ++j, ++it) {
          const int st = it % ns;
          if (it >= ns) ok = mbar_wait(&bars.kv_empty[st], ((it / ns) - 1) & 1, abort);
          if (!ok) break;
          uint8_t *kdst = sKV + st * 2 * QG::KBYTES;
          mbar_expect_tx(&bars.kv_full[st], 2 * QG::KBYTES);
          for (int ch = 0; ch < G::CHUNKS; ++ch) {
            tma_load_3d(kdst + ch * QG::KCHUNK, &tmK, &bars.kv_full[st], ch * G::EPC,
                        j * QG::KROWS, bh);
            tma_load_3d(kdst + QG::KBYTES + ch * QG::KCHUNK, &tmV, &bars.kv_full[st],
                        ch * G::EPC, j * QG::KROWS, bh);
          }
        }
      }
      // every load issued must land before the CTA may exit: the last Q / dO
      // load and the latest fill of each ring stage
      if (k >= 1) mbar_wait(bars.q_full, (k - 1) & 1, abort);
      for (int st = 0; st < ns && st < it; ++st)
        mbar_wait(&bars.kv_full[st], (((it - st + ns - 1) / ns) - 1) & 1, abort);
    }
  } else if (warp == 1) {
    // S = Q K_h^T and dP = dO V_h^T of half h into TMEM pair hc mod HB
    if (lane == 0) {
      bool ok = true;
      int it0 = 0, hc = 0, k = 0;
      const uint32_t qa = smem_u32(sQ), da = smem_u32(sdO), kva = smem_u32(sKV);
      for (int t = cta_tile(k); t < ntiles && ok; t = cta_tile(++k)) {
        int bh, qt;
        q_tile_of(p, t, bh, qt);
        const int nkv = p.causal ? min(p.nkvt, qt + 1) : p.nkvt;
        ok = mbar_wait(bars.q_full, k & 1, abort);
        tc_fence_after();
        for (int h = 0; h < 2 * nkv && ok; ++h, ++hc) {
          const int e = h % QG::HPU, x = hc % HB, u = hc / HB;
          const int itj = it0 + h / QG::HPU;                // the half's stage
          if (e == 0) {
            ok = mbar_wait(&bars.kv_full[itj % ns], (itj / ns) & 1, abort);
            if (!ok) break;
            tc_fence_after();
          }
          if (u >= 1) {
            ok = mbar_wait(&bars.sdp_free[x], (u - 1) & 1, abort);
            if (!ok) break;
            tc_fence_after();
          }
          const uint32_t kb = kva + (itj % ns) * 2 * QG::KBYTES + e * 64 * 128;
          mma_nt_half<D, QG::KCHUNK>(tmem + 128 * x, qa, kb);
          mma_nt_half<D, QG::KCHUNK>(tmem + 128 * x + 64, da, kb + QG::KBYTES);
          mma_commit(&bars.sdp_full[x]);
        }
        if (ok) mma_commit(bars.q_free);                // the tile's Q, dO are read
        it0 += 2 * nkv / QG::HPU;
      }
      mma_commit(bars.drain);
      mbar_wait(bars.drain, 0, abort);
    }
  } else if (warp == 2) {
    // dQ += dS_h K_h (dS K-major in shared memory, K as an MN-major operand)
    // into TMEM buffer k mod 2
    if (lane == 0) {
      bool ok = true;
      int it0 = 0, hc = 0, k = 0;
      const uint32_t kva = smem_u32(sKV), dsa = smem_u32(sDS);
      for (int t = cta_tile(k); t < ntiles && ok; t = cta_tile(++k)) {
        int bh, qt;
        q_tile_of(p, t, bh, qt);
        const int nkv = p.causal ? min(p.nkvt, qt + 1) : p.nkvt;
        const uint32_t dq = tmem + QG::T_DQ + D * (k & 1);
        for (int h = 0; h < 2 * nkv && ok; ++h, ++hc) {
          const int e = h % QG::HPU, x = hc % HB, u = hc / HB;
          const int itj = it0 + h / QG::HPU;                // the half's stage
          if (e == 0) {
            // K_j has landed (this warp reads it too; the stage cannot refill
            // before this warp's own release below)
            ok = mbar_wait(&bars.kv_full[itj % ns], (itj / ns) & 1, abort);
            if (!ok) break;
          }
          ok = mbar_wait(&bars.ds_full[x], u & 1, abort);
          // the buffer's previous tile (k - 2) has been read out of TMEM
          if (ok && h == 0 && k >= 2) ok = mbar_wait(&bars.dq_free[k & 1], ((k >> 1) - 1) & 1, abort);
          if (!ok) break;
          tc_fence_after();
          const uint32_t kb = kva + (itj % ns) * 2 * QG::KBYTES + e * 64 * 128;
          const uint32_t ab = dsa + x * 128 * 128;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ss_f16(dq, smem_desc(ab + kk * 32, 16, 1024),
                       smem_desc(kb + kk * 16 * 128, QG::KCHUNK, 1024), G::IDESC_MN,
                       (h > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&bars.ds_free[x]);
          if (e == QG::HPU - 1) mma_commit(&bars.kv_empty[itj % ns]);
        }
        if (ok) mma_commit(&bars.dq_full[k & 1]);
        it0 += 2 * nkv / QG::HPU;
      }
      mma_commit(bars.drain);
      mbar_wait(bars.drain, 0, abort);
    }
  } else if (warp == 3) {
    // the tile's row constants and dQ-pass table (prep kernel output), once
    // every map thread is done with the previous tile's
    if (lane == 0) {
      bool ok = true;
      int k = 0;
      const uint32_t cbytes = 128u * kCst * 4;
      for (int t = cta_tile(k); t < ntiles && ok; t = cta_tile(++k)) {
        int bh, qt;
        q_tile_of(p, t, bh, qt);
        if (k >= 1) ok = mbar_wait(bars.tab_free, (k - 1) & 1, abort);
        if (!ok) break;
        const size_t tix = static_cast<size_t>(bh) * p.nqt + qt;
        mbar_expect_tx(bars.tab_full, cbytes + p.tabq_tile);
        bulk_load(sCst, p.cst + tix * 128 * kCst, cbytes, bars.tab_full);
        if (p.tabq_tile)
          bulk_load(smem + p.tab_off, p.tabq + tix * p.tabq_tile, p.tabq_tile, bars.tab_full);
      }
      // every load issued must land before the CTA may exit
      if (k >= 1) mbar_wait(bars.tab_full, (k - 1) & 1, abort);
    }
  } else if (warp >= 4) {
    const int g = (warp - 4) >> 2;
    const int row = (warp & 3) * 32 + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const uint32_t tq_base = smem_u32(smem + p.tab_off);
    // this row's constants: field f at ca + 8 f (row pairs interleaved)
    const uint32_t ca = smem_u32(sCst) + (row >> 1) * 64 + (row & 1) * 4;
    const float *cstf = reinterpret_cast<const float *>(sCst) + (row >> 1) * 16 + (row & 1);
    const uint32_t dsb = smem_u32(sDS);
    const float Kf = static_cast<float>(p.K);
    // Read-out of a finished tile (position kp in this CTA's sequence, tile
    // t): dQ out of TMEM buffer kp mod 2, the rank-one calibration terms in
    // fp32 -- dQ_r += c (dhi k_argmax + dlo k_argmin), and dK_argmax += c dhi
    // q_r, dK_argmin += c dlo q_r into the fp32 calibration part of dK (rows
    // can share a key: vector reductions) -- and the bf16 store.  amx < 0:
    // the row takes no calibration terms.
    auto read_out = [&](int t, int kp, int amx, int amn, float kinv) -> bool {
      constexpr int NP = D / 64;                         // 16-column pieces of the slice
      const int x = kp & 1;
      const uint32_t ph = static_cast<uint32_t>(kp >> 1) & 1u;
      int bh, qt;
      q_tile_of(p, t, bh, qt);
      const int qrow = qt * 128 + row;
      const size_t head = static_cast<size_t>(bh) * p.S;
      const size_t ri = head + min(qrow, p.S - 1);
      const bool cal_row = CAL != CAL_OFF && amx >= 0;
      // the key rows and the query row of a piece (the first one before the
      // waits)
      uint4 kaw[2] = {}, kbw[2] = {}, qw[2] = {};
      auto gather = [&](int c0) {
        if (cal_row) {
          const uint4 *ka = reinterpret_cast<const uint4 *>(p.K_ + (head + amx) * D + c0);
          const uint4 *qr = reinterpret_cast<const uint4 *>(p.Q + ri * D + c0);
          kaw[0] = ka[0];
          kaw[1] = ka[1];
          qw[0] = qr[0];
          qw[1] = qr[1];
          if (CAL == CAL_MINMAX) {
            const uint4 *kb = reinterpret_cast<const uint4 *>(p.K_ + (head + amn) * D + c0);
            kbw[0] = kb[0];
            kbw[1] = kb[1];
          }
        }
      };
      gather(QG::DG * g);
      bool rok = warp_all_b(mbar_wait(&bars.part_ready[x], ph, abort));
      if (rok) rok = warp_all_b(mbar_wait(&bars.dq_full[x], ph, abort));
      if (!rok) return false;
      tc_fence_after();
      uint32_t v[NP][16];
#pragma unroll
      for (int pc = 0; pc < NP; ++pc)
        tmem_ld16(lane_base + QG::T_DQ + D * x + QG::DG * g + 16 * pc, v[pc]);
      tmem_wait_ld();
#pragma unroll
      for (int pc = 0; pc < NP; ++pc) reg_fence16(v[pc]);
      // the accumulator is in registers: tile kp + 2 may take the buffer
      tc_fence_before();
      mbar_arrive(&bars.dq_free[x]);
      // the row's calibration derivatives from the four groups' sums; they
      // are computed (the loaded sums consumed) before the buffer's release
      float sh = 0.0f, sl = 0.0f, shk = 0.0f, slk = 0.0f;   // dQ side, dK side
      if (cal_row) {
        const float *pp = part + x * 1024;
        const float S1 = (pp[row] + pp[128 + row]) + (pp[256 + row] + pp[384 + row]);
        const float S2 = (pp[512 + row] + pp[640 + row]) + (pp[768 + row] + pp[896 + row]);
        float dhi, dlo;
        if (CAL == CAL_FIXED) {
          dhi = -(Kf / p.window) * S2;
          dlo = 0.0f;
        } else if (MAP == MAPB_HARD) {
          dhi = S1;
          dlo = -S1;
        } else {
          dhi = S1;
          dlo = -S1 - kinv * S2;
        }
        sh = p.gq * dhi;
        sl = p.gq * dlo;
        shk = p.gk * dhi;
        slk = p.gk * dlo;
      }
      asm volatile("" ::"f"(sh), "f"(sl), "f"(shk), "f"(slk) : "memory");
      mbar_arrive(&bars.part_free[x]);
#pragma unroll
      for (int pc = 0; pc < NP; ++pc) {
        const int c0 = QG::DG * g + 16 * pc;
        if (pc > 0) gather(c0);
        float xq[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) xq[i] = __uint_as_float(v[pc][i]) * p.gq;
        if (cal_row) {
          float kx[16], qx[16];
          bf16x16_to_f32(kaw, kx);
          bf16x16_to_f32(qw, qx);
#pragma unroll
          for (int i = 0; i < 16; ++i) xq[i] = __fmaf_rn(sh, kx[i], xq[i]);
          float *da = p.dkcal + (head + amx) * D + c0;
#pragma unroll
          for (int i = 0; i < 4; ++i)
            red_add_f32x4(da + 4 * i, make_float4(shk * qx[4 * i], shk * qx[4 * i + 1],
                                                  shk * qx[4 * i + 2], shk * qx[4 * i + 3]));
          if (CAL == CAL_MINMAX) {
            bf16x16_to_f32(kbw, kx);
#pragma unroll
            for (int i = 0; i < 16; ++i) xq[i] = __fmaf_rn(sl, kx[i], xq[i]);
            float *db = p.dkcal + (head + amn) * D + c0;
#pragma unroll
            for (int i = 0; i < 4; ++i)
              red_add_f32x4(db + 4 * i, make_float4(slk * qx[4 * i], slk * qx[4 * i + 1],
                                                    slk * qx[4 * i + 2], slk * qx[4 * i + 3]));
          }
        }
        uint32_t pk[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) pk[i] = pack_bf16x2(xq[2 * i], xq[2 * i + 1]);
        if (qrow < p.S) {
          uint4 *d4 = reinterpret_cast<uint4 *>(p.dQ + ri * D + c0);
          d4[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          d4[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        }
      }
      return true;
    };

    bool ok = true;
    int hc = 0, k = 0;
    int pv_amx = -1, pv_amn = 0;        // the previous tile's read-out state
    float pv_kinv = 0.0f;
    for (int t = cta_tile(k); t < ntiles && ok; t = cta_tile(++k)) {
      int bh, qt;
      q_tile_of(p, t, bh, qt);
      const int nkv = p.causal ? min(p.nkvt, qt + 1) : p.nkvt;
      const int qrow = qt * 128 + row;
      const bool row_ok = qrow < p.S;
      const int L = p.causal ? min(qrow + 1, p.S) : p.S;
      const size_t ri = static_cast<size_t>(bh) * p.S + min(qrow, p.S - 1);
      ok = warp_all_b(mbar_wait(bars.tab_full, k & 1, abort));
      if (!ok) break;
      // table addresses: the entry is bits(M + floor(clamp(u, -1, K))) -
      // bits(M) + 1 (interpolation) or bits(M + rne(clamp(u, 0, K))) - bits(M)
      // (hard), M = 1.5 * 2^23 -- on the saturating path bits(M/K + v) -
      // bits(M/K); the address arithmetic wraps mod 2^32.  The stored a, b
      // are divided by K when K = 2^m: interpolation takes them back (exact).
      DqK dk;
      const bool kp2 = k_pow2(p.K);
      const bool hsat = MAP == MAPB_HARD && kp2;        // hard rounding: saturating form
      dk.a = lds_f32(ca);
      dk.b = lds_f32(ca + 8);
      if (MAP == MAPB_INTERP && kp2) {
        dk.a = __fmul_rn(dk.a, Kf);
        dk.b = __fmul_rn(dk.b, Kf);
      }
      dk.invZ = lds_f32(ca + 16);
      dk.nDZ = lds_f32(ca + 24);
      dk.ne0 = lds_f32(ca + 32);
      dk.nds = lds_f32(ca + 40);
      dk.kinv = lds_f32(ca + 48);
      dk.cL2E = p.cL2E;
      dk.Kf = Kf;
      dk.mk = hsat ? __fmul_rn(kMagic, 1.0f / Kf) : kMagic;
      dk.tq_row = (MAP == MAPB_INTERP)
                      ? tq_base + row * T::ESZ - kMagicBits * T::STRIDE + T::STRIDE
                      : tq_base + row * T::ESZ - __float_as_uint(dk.mk) * T::STRIDE;
      float2 s1 = make_float2(0.0f, 0.0f), s2 = make_float2(0.0f, 0.0f);   // calibration sums
      for (int h = 0; h < 2 * nkv && ok; ++h, ++hc) {
        const int j = h >> 1, e = h & 1, x = hc % HB, u = hc / HB;
        ok = warp_all_b(mbar_wait(&bars.sdp_full[x], u & 1, abort));
        if (!ok) break;
        tc_fence_after();
        uint32_t sv[16], dv[16];
        tmem_ld16(lane_base + 128 * x + 16 * g, sv);
        tmem_ld16(lane_base + 128 * x + 64 + 16 * g, dv);
        tmem_wait_ld();
        reg_fence16(sv);
        reg_fence16(dv);
        tc_fence_before();
        mbar_arrive(&bars.sdp_free[x]);                // the pair can take half hc + 3
        const int lim = L - (128 * j + 64 * e + 16 * g);  // valid keys of this slice
        uint32_t dd[8];
        const bool full = warp_all_b(lim >= 16);
        if constexpr (MAP == MAPB_HARD) {
          if (hsat) {
            if (full)
              dq_slice<MAP, SURR, CAL, true, true>(sv, dv, dk, lim, dd, s1, s2);
            else
              dq_slice<MAP, SURR, CAL, false, true>(sv, dv, dk, lim, dd, s1, s2);
          } else if (full) {
            dq_slice<MAP, SURR, CAL, true>(sv, dv, dk, lim, dd, s1, s2);
          } else {
            dq_slice<MAP, SURR, CAL, false>(sv, dv, dk, lim, dd, s1, s2);
          }
        } else if (full) {
          dq_slice<MAP, SURR, CAL, true>(sv, dv, dk, lim, dd, s1, s2);
        } else {
          dq_slice<MAP, SURR, CAL, false>(sv, dv, dk, lim, dd, s1, s2);
        }
        if (u >= 1) {
          // the dQ product of half hc - 3 has read dS buffer x
          ok = warp_all_b(mbar_wait(&bars.ds_free[x], (u - 1) & 1, abort));
          if (!ok) break;
        }
        // dS row-major (K-major operand), 128-byte swizzle: this group's 16
        // keys are granules 2g, 2g + 1 of the row
        const uint32_t rowa = dsb + x * 128 * 128 + row * 128;
#pragma unroll
        for (int gi = 0; gi < 2; ++gi) {
          const uint32_t gran = static_cast<uint32_t>((2 * g + gi) ^ (row & 7));
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(rowa + gran * 16),
                       "r"(dd[4 * gi]), "r"(dd[4 * gi + 1]), "r"(dd[4 * gi + 2]),
                       "r"(dd[4 * gi + 3])
                       : "memory");
        }
        fence_async_smem();
        mbar_arrive(&bars.ds_full[x]);
      }
      if (!ok) break;
      // The tile's constants and table are no longer read.  The next bulk copy
      // (async proxy) overwrites them, so every value read from them is
      // consumed by an instruction ahead of the release -- the sums the last
      // table reads feed, the calibration flag (a load whose result is still
      // in flight is not ordered by the arrive) -- and a proxy fence orders
      // those reads before the copy.
      const bool calib = CAL != CAL_OFF && row_ok && cstf[14] != 0.0f;
      asm volatile("" ::"f"(s1.x), "f"(s1.y), "f"(s2.x), "f"(s2.y), "r"(calib ? 1 : 0)
                   : "memory");
      fence_async_smem();
      mbar_arrive(bars.tab_free);
      // this row's argmax / argmin key, needed at the tile's read-out (after
      // the next tile's halves)
      int amx = -1, amn = 0;
      if (calib) {
        amx = p.amax[ri];
        if (CAL == CAL_MINMAX) amn = p.amin[ri];
      }
      // the calibration sums, once the buffer's previous tile (k - 2) has been
      // read out
      if (k >= 2) {
        ok = warp_all_b(mbar_wait(&bars.part_free[k & 1], ((k >> 1) - 1) & 1, abort));
        if (!ok) break;
      }
      float *pp = part + (k & 1) * 1024;
      pp[g * 128 + row] = s1.x + s1.y;
      pp[512 + g * 128 + row] = s2.x + s2.y;
      mbar_arrive(&bars.part_ready[k & 1]);
      if (k >= 1 && !read_out(cta_tile(k - 1), k - 1, pv_amx, pv_amn, pv_kinv)) {
        ok = false;
        break;
      }
      pv_amx = amx;
      pv_amn = amn;
      pv_kinv = dk.kinv;
    }
    if (ok && k >= 1) read_out(cta_tile(k - 1), k - 1, pv_amx,
                               pv_amn, pv_kinv);
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kBwdTmemCols);
  if (threadIdx.x == 0 && *bars.abort && p.status != nullptr) atomicExch(p.status, QSM_ERR_TIMEOUT);
}

// --------------------------------------------------------------- dK/dV pass
// Persistent: one CTA per SM takes the 128-key tiles in the heaviest-first
// order; thread = key (TMEM lane); the query tiles are taken in halves of 64
// rows, half number hc (counted across tiles) in TMEM pair x = hc mod HB
// (S^T at 128x, dP^T at 128x + 64); map group g owns rows 16g .. 16g+15 of
// each half and writes its P^T and dS^T (bf16) into the first 8 of its own 16
// columns, which the dV / dK products (dV at TMEM column T_DV, dK at T_DK)
// read as their TMEM A operand.  A ring stage holds Q, dO rows and their
// per-row constants and grid tables: a whole query tile at D = 64 (three
// pairs), a half tile at D = 128, whose accumulators take twice the TMEM
// columns (two pairs) and whose tiles twice the shared memory.
struct KvBars {
  uint64_t *qd_full, *qd_empty;       // [ns]
  uint64_t *kv_full, *kv_free;        // K, V of the current tile
  uint64_t *sdp_full, *pds_full, *s_free;   // [HB]
  uint64_t *acc_full, *acc_free;      // the tile's dV, dK complete / read out of TMEM
  uint64_t *drain;
  uint32_t *tmem_slot;
  int *abort;
};
template <int D>
struct KvGeo {
  static constexpr int HB = D > 64 ? 2 : 3;          // TMEM S^T / dP^T pairs
  static constexpr int SROWS = D > 64 ? 64 : 128;    // query rows per ring stage
  static constexpr int HPU = SROWS / 64;             // halves per stage
  static constexpr int QBYTES = SROWS * D * 2;       // the Q (or dO) rows of a stage
  static constexpr int QCHUNK = SROWS * 128;         // bytes between their 64-column chunks
  static constexpr uint32_t T_DV = HB * 128, T_DK = T_DV + D;
  static constexpr int DG = D / 4;                   // dV / dK columns per map group
};

// Sixteen fp32 TMEM values, times scale, to bf16 at d4 (two 16-byte stores);
// with cal, its sixteen fp32 values are added first.
__device__ __forceinline__ void store_bf16x16(uint4 *d4, const uint32_t (&v)[16], float scale) {
  uint32_t pk[8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
    pk[i] = pack_bf16x2(__uint_as_float(v[2 * i]) * scale, __uint_as_float(v[2 * i + 1]) * scale);
  d4[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  d4[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
}
__device__ __forceinline__ void store_bf16x16_cal(uint4 *d4, const uint32_t (&v)[16], float scale,
                                                  const float *cal) {
  float x[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) x[i] = __uint_as_float(v[i]) * scale;
  if (cal != nullptr) {
    const float4 *c4 = reinterpret_cast<const float4 *>(cal);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 c = c4[i];
      x[4 * i] += c.x;
      x[4 * i + 1] += c.y;
      x[4 * i + 2] += c.z;
      x[4 * i + 3] += c.w;
    }
  }
  uint32_t pk[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) pk[i] = pack_bf16x2(x[2 * i], x[2 * i + 1]);
  d4[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  d4[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
}

// The dK / dV pass's per-thread values for the element loop.
struct KvK {
  float cL2E, Kf, cap, flush_t;
  float Ksc;         // K when K = 2^m (the stored a, b are divided by it), else 1
  float mk;          // saturating form: 1.5 * 2^23 / K
  bool flush, flush_below;
};

// P^T and dS^T of one key against a 16-row query slice (bf16 pairs into pp,
// dd), two rows per packed fp32 operation.  cb: shared address of the
// slice's first row pair of constants (64 bytes a pair, see
// store_row_constants); tr: biased shared address of the slice's first row
// table, ts its row stride in bytes; vmask: valid rows (bit i) unless FULL.
// The K-interval tables hold the weights times 1/Z, so a lookup gives P.
// SAT (kv_sat): the coordinate divided by K in one saturating FMA, v =
// clamp(u, 0, K) / K; the node or interval from v + 1.5 * 2^23 / K, whose
// unit is 1 / K (the same node or interval as from u), and interpolation's
// P = fma(v, K d, e) with K d in the table.
template <int MAP, int SURR, bool FULL, bool SAT>
__device__ __forceinline__ void kv_slice(const uint32_t (&sv)[16], const uint32_t (&dv)[16],
                                         uint32_t cb, uint32_t tr, uint32_t ts, const KvK &k,
                                         uint32_t vmask, uint32_t (&pp)[8], uint32_t (&dd)[8]) {
  const float2 cl2 = make_float2(k.cL2E, k.cL2E);
  const float2 mg = make_float2(kMagic, kMagic);
#pragma unroll
  for (int i2 = 0; i2 < 8; ++i2) {
    const float2 r = make_float2(__uint_as_float(sv[2 * i2]), __uint_as_float(sv[2 * i2 + 1]));
    const float2 dp = make_float2(__uint_as_float(dv[2 * i2]), __uint_as_float(dv[2 * i2 + 1]));
    const uint32_t c = cb + i2 * 64;
    const uint32_t t0 = tr + (2 * i2) * ts, t1 = t0 + ts;
    float2 pw, ds = make_float2(0.0f, 0.0f);
    if (MAP == MAPB_EXACT) {
      const float4 c2 = lds_f32x4(c + 32);                 // -e0 pair, -delta pair
      pw = ex2_pair(fma2_rn(r, cl2, make_float2(c2.x, c2.y)));
      ds = mul2_rn(pw, add2_rn(dp, make_float2(c2.z, c2.w)));
    } else {
      const float4 c0 = lds_f32x4(c);                      // a pair, b pair
      float4 c1 = make_float4(0.0f, 0.0f, 0.0f, 0.0f);    // 1/Z pair, -delta/Z pair
      if (MAP == MAPB_POT || SURR == SURR_PRE) c1 = lds_f32x4(c + 16);
      float2 dn = make_float2(0.0f, 0.0f);
      if (MAP == MAPB_POT) {
        // the forward's power-of-two weight (exponent frozen: no own-score or
        // anchor derivative; only the surrogate's direct term)
        const float2 u = fma2_rn(r, make_float2(c0.x, c0.y), make_float2(c0.z, c0.w));
        const float2 t = add2_rn(make_float2(fminf(u.x, k.cap), fminf(u.y, k.cap)), mg);
        float2 w = make_float2(__uint_as_float(__float_as_uint(t.x) * 0xFF800000u + 0x3F800000u),
                               __uint_as_float(__float_as_uint(t.y) * 0xFF800000u + 0x3F800000u));
        if (k.flush && t.x > k.flush_t) w.x = 0.0f;
        if (k.flush && t.y > k.flush_t) w.y = 0.0f;
        pw = mul2_rn(w, make_float2(c1.x, c1.y));
      } else if (SAT) {
        const float2 v = make_float2(fma_sat(r.x, c0.x, c0.z), fma_sat(r.y, c0.y, c0.w));
        const float2 mk = make_float2(k.mk, k.mk);
        if (MAP == MAPB_HARD) {
          const float2 t = add2_rn(v, mk);
          pw = make_float2(lds_f32(__float_as_uint(t.x) * 4u + t0),
                           lds_f32(__float_as_uint(t.y) * 4u + t1));
        } else {
          const float2 t = add2_rd(v, mk);
          const float2 e0 = lds_f32x2(__float_as_uint(t.x) * 8u + t0);
          const float2 e1 = lds_f32x2(__float_as_uint(t.y) * 8u + t1);
          pw = make_float2(__fmaf_rn(v.x, e0.y, e0.x), __fmaf_rn(v.y, e1.y, e1.x));
        }
      } else {
        // u itself: the stored a, b times Ksc (exact)
        const float2 ks = make_float2(k.Ksc, k.Ksc);
        const float2 u = fma2_rn(r, mul2_rn(make_float2(c0.x, c0.y), ks),
                                 mul2_rn(make_float2(c0.z, c0.w), ks));
        if (MAP == MAPB_HARD) {
          const float2 uc =
              make_float2(fminf(fmaxf(u.x, 0.0f), k.Kf), fminf(fmaxf(u.y, 0.0f), k.Kf));
          const float2 t = add2_rn(uc, mg);
          pw = make_float2(lds_f32(__float_as_uint(t.x) * 4u + t0),
                           lds_f32(__float_as_uint(t.y) * 4u + t1));
          if (k.flush_below && u.x < 0.0f) pw.x = 0.0f;
          if (k.flush_below && u.y < 0.0f) pw.y = 0.0f;
        } else {
          const float2 uc =
              make_float2(fminf(fmaxf(u.x, -1.0f), k.Kf), fminf(fmaxf(u.y, -1.0f), k.Kf));
          const float2 t = add2_rd(uc, mg);
          const float2 e0 = lds_f32x2(__float_as_uint(t.x) * 8u + t0);
          const float2 e1 = lds_f32x2(__float_as_uint(t.y) * 8u + t1);
          pw = make_float2(__fmaf_rn(uc.x, e0.y, e0.x), __fmaf_rn(uc.y, e1.y, e1.x));
          dn = make_float2(e0.y, e1.y);                    // d / Z
        }
      }
      if (SURR == SURR_PRE) {
        const float2 gw =
            fma2_rn(dp, make_float2(c1.x, c1.y), make_float2(c1.z, c1.w));
        ds = mul2_rn(gw, ex2_pair(fma2_rn(r, cl2, lds_f32x2(c + 32))));
      } else if (SURR == SURR_POST) {
        const float4 c2 = lds_f32x4(c + 32);               // -e0 pair, -delta* pair
        ds = mul2_rn(ex2_pair(fma2_rn(r, cl2, make_float2(c2.x, c2.y))),
                     add2_rn(dp, make_float2(c2.z, c2.w)));
      } else if (MAP == MAPB_INTERP) {
        // (dp - delta) d / Z K / (hi - lo)
        const float4 c2 = lds_f32x4(c + 32);               // -delta pair at z, w
        ds = mul2_rn(mul2_rn(add2_rn(dp, make_float2(c2.z, c2.w)), dn), lds_f32x2(c + 48));
      }
    }
    if (!FULL) {
      if (!((vmask >> (2 * i2)) & 1u)) pw.x = ds.x = 0.0f;
      if (!((vmask >> (2 * i2 + 1)) & 1u)) pw.y = ds.y = 0.0f;
    }
    pp[i2] = pack_bf16x2(pw.x, pw.y);
    dd[i2] = pack_bf16x2(ds.x, ds.y);
  }
}

template <int D, int MAP, int SURR>
__global__ void __launch_bounds__(kMainThreads, 1)
    qsm_bwd_dkdv(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                 const BwdParams p) {
  using G = BGeo<D>;
  using KG = KvGeo<D>;
  static_assert(D == 64 || D == 128, "dK / dV slices of the four map groups: D / 4 columns");
  constexpr int HB = KG::HB;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = smem_align1024(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntiles = p.nkvt * p.BH;
  const int ns = p.num_stages;
  uint8_t *sK = smem;
  uint8_t *sV = smem + G::TILE_BYTES;
  uint8_t *sSt = smem + 2 * G::TILE_BYTES;              // ns stages: Q, dO, cst, tab
  const uint32_t SB = p.stage_bytes;
  const uint32_t CST_OFF = 2 * KG::QBYTES;
  const uint32_t TAB_OFF = CST_OFF + KG::SROWS * kCst * 4;
  uint64_t *bp = reinterpret_cast<uint64_t *>(smem + p.bar_off);
  KvBars bars;
  bars.qd_full = bp;
  bars.qd_empty = bp + ns;
  bars.kv_full = bp + 2 * ns;
  bars.kv_free = bars.kv_full + 1;
  bars.sdp_full = bars.kv_free + 1;
  bars.pds_full = bars.sdp_full + HB;
  bars.s_free = bars.pds_full + HB;
  bars.acc_full = bars.s_free + HB;
  bars.acc_free = bars.acc_full + 1;
  bars.drain = bars.acc_free + 1;
  bars.tmem_slot = reinterpret_cast<uint32_t *>(bars.drain + 1);
  bars.abort = reinterpret_cast<int *>(bars.tmem_slot + 1);
  volatile int *abort = bars.abort;

  if (threadIdx.x == 0) {
    for (int i = 0; i < ns; ++i) {
      mbar_init(&bars.qd_full[i], 1);
      mbar_init(&bars.qd_empty[i], 1);
    }
    mbar_init(bars.kv_full, 1);
    mbar_init(bars.kv_free, 1);
    for (int i = 0; i < HB; ++i) {
      mbar_init(&bars.sdp_full[i], 1);
      mbar_init(&bars.pds_full[i], kMainMapThreads);
      mbar_init(&bars.s_free[i], 1);
    }
    mbar_init(bars.acc_full, 1);
    mbar_init(bars.acc_free, kMainMapThreads);
    mbar_init(bars.drain, 2);
    *bars.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(bars.tmem_slot, kBwdTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *bars.tmem_slot;

  // Tiles of this CTA: cta_tile(0), cta_tile(1), ... of the heaviest-first
  // key-tile order (persistent, as the dQ pass); the ring
  // position and the half counter run on across tiles.
  if (warp == 0) {
    if (lane == 0) {
      bool ok = true;
      int rc = 0, k = 0;
      for (int t = cta_tile(k); t < ntiles && ok; t = cta_tile(++k)) {
        int bh, kt;
        kv_tile_of(p, t, bh, kt);
        const int i0 = p.causal ? kt : 0;                // first query tile
        const int nq = p.nqt - i0;
        // K, V of the previous tile are no longer read
        if (k >= 1) ok = mbar_wait(bars.kv_free, (k - 1) & 1, abort);
        if (!ok) break;
        mbar_expect_tx(bars.kv_full, 2 * G::TILE_BYTES);
        for (int ch = 0; ch < G::CHUNKS; ++ch) {
          tma_load_3d(sK + ch * G::CHUNK_BYTES, &tmK, bars.kv_full, ch * G::EPC, kt * 128, bh);
          tma_load_3d(sV + ch * G::CHUNK_BYTES, &tmV, bars.kv_full, ch * G::EPC, kt * 128, bh);
        }
        // one stage per SROWS query rows (Q / dO tensor maps of SROWS-row boxes)
        for (int n = 0; n < nq * (128 / KG::SROWS) && ok; ++n, ++rc) {
          const int st = rc % ns;
          const int row0 = (i0 * 128) + n * KG::SROWS;     // first query row of the stage
          if (rc >= ns) ok = mbar_wait(&bars.qd_empty[st], ((rc / ns) - 1) & 1, abort);
          if (!ok) break;
          uint8_t *s = sSt + st * SB;
          // the constants and tables of the stage's tile rows (rows past S in
          // a ragged last tile are never valid)
          const size_t r0 = static_cast<size_t>(bh) * p.nqt * 128 + row0;
          const uint32_t cbytes = KG::SROWS * kCst * 4;
          const uint32_t tbytes = KG::SROWS * static_cast<uint32_t>(p.TS) * 4;
          mbar_expect_tx(&bars.qd_full[st], 2 * KG::QBYTES + cbytes + tbytes);
          for (int ch = 0; ch < G::CHUNKS; ++ch) {
            tma_load_3d(s + ch * KG::QCHUNK, &tmQ, &bars.qd_full[st], ch * G::EPC, row0, bh);
            tma_load_3d(s + KG::QBYTES + ch * KG::QCHUNK, &tmdO, &bars.qd_full[st], ch * G::EPC,
                        row0, bh);
          }
          bulk_load(s + CST_OFF, p.cst + r0 * kCst, cbytes, &bars.qd_full[st]);
          if (tbytes) bulk_load(s + TAB_OFF, p.tabk + r0 * p.TS, tbytes, &bars.qd_full[st]);
        }
      }
      // every load issued must land before the CTA may exit
      if (k >= 1) mbar_wait(bars.kv_full, (k - 1) & 1, abort);
      for (int st = 0; st < ns && st < rc; ++st)
        mbar_wait(&bars.qd_full[st], (((rc - st + ns - 1) / ns) - 1) & 1, abort);
    }
  } else if (warp == 1) {
    // S^T = K Q_h^T and dP^T = V dO_h^T of half h into TMEM pair hc mod HB,
    // once the dV / dK products of half hc - HB have read it
    if (lane == 0) {
      bool ok = true;
      int rc0 = 0, hc = 0, k = 0;
      const uint32_t ka = smem_u32(sK), va = smem_u32(sV), sa = smem_u32(sSt);
      for (int t = cta_tile(k); t < ntiles && ok; t = cta_tile(++k)) {
        int bh, kt;
        kv_tile_of(p, t, bh, kt);
        const int nq = p.nqt - (p.causal ? kt : 0);
        ok = mbar_wait(bars.kv_full, k & 1, abort);
        tc_fence_after();
        for (int h = 0; h < 2 * nq && ok; ++h, ++hc) {
          const int e = h % KG::HPU, x = hc % HB, u = hc / HB;
          const int rn = rc0 + h / KG::HPU;                 // the half's stage
          if (e == 0) {
            ok = mbar_wait(&bars.qd_full[rn % ns], (rn / ns) & 1, abort);
            if (!ok) break;
            tc_fence_after();
          }
          if (u >= 1) {
            ok = mbar_wait(&bars.s_free[x], (u - 1) & 1, abort);
            if (!ok) break;
            tc_fence_after();
          }
          const uint32_t qb = sa + (rn % ns) * SB + e * 64 * 128;
          mma_nt_half<D, KG::QCHUNK>(tmem + 128 * x, ka, qb);
          mma_nt_half<D, KG::QCHUNK>(tmem + 128 * x + 64, va, qb + KG::QBYTES);
          mma_commit(&bars.sdp_full[x]);
        }
        if (ok) mma_commit(bars.kv_free);               // the tile's K, V are read
        rc0 += 2 * nq / KG::HPU;
      }
      mma_commit(bars.drain);
      mbar_wait(bars.drain, 0, abort);
    }
  } else if (warp == 2) {
    // dV += P^T_h dO_h and dK += dS^T_h Q_h (A from TMEM, B MN-major)
    if (lane == 0) {
      bool ok = true;
      int rc0 = 0, hc = 0, k = 0;
      const uint32_t sa = smem_u32(sSt);
      for (int t = cta_tile(k); t < ntiles && ok; t = cta_tile(++k)) {
        int bh, kt;
        kv_tile_of(p, t, bh, kt);
        const int nq = p.nqt - (p.causal ? kt : 0);
        for (int h = 0; h < 2 * nq && ok; ++h, ++hc) {
          const int e = h % KG::HPU, x = hc % HB, u = hc / HB;
          const int rn = rc0 + h / KG::HPU;                 // the half's stage
          if (e == 0) {
            ok = mbar_wait(&bars.qd_full[rn % ns], (rn / ns) & 1, abort);
            if (!ok) break;
          }
          ok = mbar_wait(&bars.pds_full[x], u & 1, abort);
          // the previous tile's dV, dK have been read out of TMEM
          if (ok && h == 0 && k >= 1) ok = mbar_wait(bars.acc_free, (k - 1) & 1, abort);
          if (!ok) break;
          tc_fence_after();
          const uint32_t qb = sa + (rn % ns) * SB + e * 64 * 128;
          const uint32_t db = qb + KG::QBYTES;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t acc = (h > 0 || kk > 0) ? 1u : 0u;
            mma_ts_f16(tmem + KG::T_DV, tmem + 128 * x + 16 * kk,
                       smem_desc(db + kk * 16 * 128, KG::QCHUNK, 1024), G::IDESC_MN, acc);
            mma_ts_f16(tmem + KG::T_DK, tmem + 128 * x + 64 + 16 * kk,
                       smem_desc(qb + kk * 16 * 128, KG::QCHUNK, 1024), G::IDESC_MN, acc);
          }
          mma_commit(&bars.s_free[x]);
          if (e == KG::HPU - 1) mma_commit(&bars.qd_empty[rn % ns]);
        }
        if (ok) mma_commit(bars.acc_full);
        rc0 += 2 * nq / KG::HPU;
      }
      mma_commit(bars.drain);
      mbar_wait(bars.drain, 0, abort);
    }
  } else if (warp >= 4) {
    const int g = (warp - 4) >> 2;
    const int key = (warp & 3) * 32 + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    KvK kk;
    kk.cL2E = p.cL2E;
    kk.Kf = static_cast<float>(p.K);
    kk.cap = static_cast<float>(p.flush ? p.pot_floor + 1 : p.pot_floor);
    kk.flush_t = kMagic + static_cast<float>(p.pot_floor);
    kk.flush = p.flush != 0;
    kk.flush_below = MAP == MAPB_HARD && p.flush && p.fixed_window;
    kk.Ksc = k_pow2(p.K) ? kk.Kf : 1.0f;
    kk.mk = __fmul_rn(kMagic, 1.0f / kk.Ksc);
    const bool sat = (MAP == MAPB_HARD || MAP == MAPB_INTERP) && kv_sat<SURR>(p);
    // table entry bias: bits(M + floor(clamp(u, -1, K))) - bits(M) + 1 (interp)
    // or bits(M + rne(clamp(u, 0, K))) - bits(M) (hard), M = 1.5 * 2^23; on
    // the saturating path M / K and v in place of M and u; mod 2^32
    const uint32_t mbits = sat ? __float_as_uint(kk.mk) : kMagicBits;
    const uint32_t tbias = (MAP == MAPB_INTERP) ? 8u - mbits * 8u : 0u - mbits * 4u;
    const uint32_t tsb = static_cast<uint32_t>(p.TS) * 4u;
    bool ok = true;
    int rc0 = 0, hc = 0, k = 0;
    for (int t = cta_tile(k); t < ntiles && ok; t = cta_tile(++k)) {
      int bh, kt;
      kv_tile_of(p, t, bh, kt);
      const int i0 = p.causal ? kt : 0;                  // first query tile
      const int nq = p.nqt - i0;
      const int kg = kt * 128 + key;
      const bool key_ok = kg < p.S;
      for (int h = 0; h < 2 * nq && ok; ++h, ++hc) {
        const int n = h >> 1, e = h & 1, x = hc % HB, u = hc / HB;
        const int rn = rc0 + h / KG::HPU;                   // the half's stage
        if (h % KG::HPU == 0) {
          // the stage's constants and tables have landed (the stage cannot
          // refill before this tile's products, which wait for these threads)
          ok = warp_all_b(mbar_wait(&bars.qd_full[rn % ns], (rn / ns) & 1, abort));
          if (!ok) break;
        }
        ok = warp_all_b(mbar_wait(&bars.sdp_full[x], u & 1, abort));
        if (!ok) break;
        tc_fence_after();
        const uint32_t st = smem_u32(sSt + (rn % ns) * SB);
        uint32_t sv[16], dv[16];
        tmem_ld16(lane_base + 128 * x + 16 * g, sv);
        tmem_ld16(lane_base + 128 * x + 64 + 16 * g, dv);
        tmem_wait_ld();
        reg_fence16(sv);
        reg_fence16(dv);
        const int qbase = (i0 + n) * 128 + 64 * e + 16 * g;   // first query row of the slice
        const int ql0 = 64 * (h % KG::HPU) + 16 * g;          // its row within the stage
        // every element valid: the key exists, the slice's rows exist and
        // (causal) lie at or below this key
        const bool full = warp_all_b(key_ok && qbase + 15 < p.S && (!p.causal || kg <= qbase));
        const uint32_t cb = st + CST_OFF + ql0 * (kCst * 4);
        const uint32_t tr = st + TAB_OFF + ql0 * tsb + tbias;
        uint32_t pp[8], dd[8];
        constexpr bool KI = MAP == MAPB_HARD || MAP == MAPB_INTERP;
        if (full) {
          if (KI && sat)
            kv_slice<MAP, SURR, true, KI>(sv, dv, cb, tr, tsb, kk, 0u, pp, dd);
          else
            kv_slice<MAP, SURR, true, false>(sv, dv, cb, tr, tsb, kk, 0u, pp, dd);
        } else {
          uint32_t vmask = 0;
#pragma unroll
          for (int i = 0; i < 16; ++i)
            vmask |= (key_ok && qbase + i < p.S && (!p.causal || kg <= qbase + i)) ? (1u << i) : 0u;
          if (KI && sat)
            kv_slice<MAP, SURR, false, KI>(sv, dv, cb, tr, tsb, kk, vmask, pp, dd);
          else
            kv_slice<MAP, SURR, false, false>(sv, dv, cb, tr, tsb, kk, vmask, pp, dd);
        }
        tmem_st8(lane_base + 128 * x + 16 * g, pp);
        tmem_st8(lane_base + 128 * x + 64 + 16 * g, dd);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars.pds_full[x]);
      }
      if (!ok) break;
      rc0 += 2 * nq / KG::HPU;
      // the dQ pass (whose fp32 calibration part of dK the read-out adds)
      // has completed: this pass may have started on the SMs it freed
      if (k == 0) grid_dep_wait();
      if constexpr (D > 64) {
        // D = 128: 32 columns a group, dV read out first, then dK
        if (!warp_all_b(mbar_wait(bars.acc_full, k & 1, abort))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const size_t krow = static_cast<size_t>(bh) * p.S + min(kg, p.S - 1);
        uint32_t v0[16], v1[16];
        tmem_ld16(lane_base + KG::T_DV + KG::DG * g, v0);
        tmem_ld16(lane_base + KG::T_DV + KG::DG * g + 16, v1);
        tmem_wait_ld();
        reg_fence16(v0);
        reg_fence16(v1);
        if (key_ok) {
          uint4 *d4 = reinterpret_cast<uint4 *>(p.dV + krow * D + KG::DG * g);
          store_bf16x16(d4, v0, 1.0f);
          store_bf16x16(d4 + 2, v1, 1.0f);
        }
        tmem_ld16(lane_base + KG::T_DK + KG::DG * g, v0);
        tmem_ld16(lane_base + KG::T_DK + KG::DG * g + 16, v1);
        tmem_wait_ld();
        reg_fence16(v0);
        reg_fence16(v1);
        // dV, dK are in registers: the next tile's products may start
        tc_fence_before();
        mbar_arrive(bars.acc_free);
        if (key_ok) {
          const float *cal = p.dkcal != nullptr ? p.dkcal + krow * D + KG::DG * g : nullptr;
          uint4 *d4 = reinterpret_cast<uint4 *>(p.dK + krow * D + KG::DG * g);
          store_bf16x16_cal(d4, v0, p.gk, cal);
          store_bf16x16_cal(d4 + 2, v1, p.gk, cal != nullptr ? cal + 16 : nullptr);
        }
        continue;
      }
      // the key's fp32 calibration part of dK (written by the dQ pass) is
      // fetched before the wait for the tile's last products
      const size_t krow = static_cast<size_t>(bh) * p.S + min(kg, p.S - 1);
      float4 cal[4] = {};
      if (p.dkcal != nullptr && key_ok) {
        const float4 *c4 = reinterpret_cast<const float4 *>(p.dkcal + krow * D + 16 * g);
#pragma unroll
        for (int i = 0; i < 4; ++i) cal[i] = c4[i];
      }
      ok = warp_all_b(mbar_wait(bars.acc_full, k & 1, abort));
      if (!ok) break;
      tc_fence_after();
      uint32_t v[16], w[16];
      tmem_ld16(lane_base + KG::T_DV + 16 * g, v);
      tmem_ld16(lane_base + KG::T_DK + 16 * g, w);
      tmem_wait_ld();
      reg_fence16(v);
      reg_fence16(w);
      // dV, dK are in registers: the next tile's products may start
      tc_fence_before();
      mbar_arrive(bars.acc_free);
      uint32_t pk[8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        pk[i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
      if (key_ok) {
        uint4 *d4 = reinterpret_cast<uint4 *>(p.dV + krow * D + 16 * g);
        d4[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        d4[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
      }
      float xk[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) xk[i] = __uint_as_float(w[i]) * p.gk;
      if (p.dkcal != nullptr && key_ok) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          xk[4 * i] += cal[i].x;
          xk[4 * i + 1] += cal[i].y;
          xk[4 * i + 2] += cal[i].z;
          xk[4 * i + 3] += cal[i].w;
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
  grid_dep_wait();                                    // no-op once waited
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

// Streaming multiprocessors of the current device (cached per device).
int sm_count() {
  static std::atomic<int> cache[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  const bool in = dev >= 0 && dev < kMaxDevices;
  if (in) {
    const int v = cache[dev].load(std::memory_order_relaxed);
    if (v > 0) return v;
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    n = 148;
  if (in) cache[dev].store(n, std::memory_order_relaxed);
  return n;
}
constexpr size_t kBarBytes = ((2 * 8 + 26) * 8 + 8 + 15) & ~static_cast<size_t>(15);

// The backward's tensor maps: whole 128-row tiles, and the row boxes the
// passes stage by (the same at D = 64; 64 rows at D = 128).
struct alignas(64) BwdMaps {
  CUtensorMap q, k, v, dO;
  CUtensorMap q_stage, k_stage, v_stage, dO_stage;
};

// A kernel launched with programmatic stream serialization: its CTAs may
// start (prologue, then grid_dep_wait) while the previous kernel on the
// stream finishes, once every CTA of that kernel has issued grid_dep_launch
// or exited.
template <typename... Args>
cudaError_t launch_dependent_block(void (*kern)(Args...), int grid, int block, size_t smem,
                                   cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}
// The persistent passes (640 threads).
template <typename... Args>
cudaError_t launch_dependent(void (*kern)(Args...), int grid, size_t smem, cudaStream_t stream,
                             Args... args) {
  return launch_dependent_block(kern, grid, kMainThreads, smem, stream, args...);
}

template <int D, int MAP, int SURR, int CAL>
qsm_status launch_dq(const BwdArgs &a, BwdParams p, const CUtensorMap &mq, const CUtensorMap &mk,
                     const CUtensorMap &mv, const CUtensorMap &mdo) {
  using G = BGeo<D>;
  using QG = DqGeo<D>;
  // Q, dO, ns x (K, V rows), HB dS buffers, constants, table, two tiles'
  // calibration sums, barriers
  const size_t tab = (static_cast<size_t>(p.tabq_tile) + 15) & ~static_cast<size_t>(15);
  const size_t cst = 128 * kCst * sizeof(float);
  const size_t part = 2 * 2 * 4 * 128 * sizeof(float);
  const size_t fixed =
      1024 + 2 * G::TILE_BYTES + QG::HB * 128 * 128 + cst + tab + part + kBarBytes;
  int ns = static_cast<int>((kMaxSmem - fixed) / (2 * QG::KBYTES));
  if (ns > 4) ns = 4;
  if (ns < (D > 64 ? 1 : 2)) return QSM_ERR_UNSUPPORTED;
  p.num_stages = ns;
  p.ds_off = static_cast<uint32_t>(2 * G::TILE_BYTES + ns * 2 * QG::KBYTES);
  p.cst_off = p.ds_off + QG::HB * 128 * 128;
  p.tab_off = static_cast<uint32_t>(p.cst_off + cst);
  p.part_off = static_cast<uint32_t>(p.tab_off + tab);
  p.bar_off = static_cast<uint32_t>(p.part_off + part);
  size_t smem = 1024 + p.bar_off + kBarBytes;
  if (smem < 120 * 1024) smem = 120 * 1024;            // one CTA per SM (all of TMEM)
  if (smem > kMaxSmem) return QSM_ERR_UNSUPPORTED;
  auto kern = qsm_bwd_dq<D, MAP, SURR, CAL>;
  static std::atomic<int> cache[kMaxDevices];
  if (!set_smem_once(kern, static_cast<int>(smem), cache)) return QSM_ERR_CUDA;
  // persistent: one CTA per SM walks the query tiles
  const int ntiles = p.nqt * a.B * a.H;
  const int grid = ntiles < sm_count() ? ntiles : sm_count();
  return launch_dependent(kern, grid, smem, a.stream, mq, mk, mv, mdo, p) == cudaSuccess ? QSM_OK
                                                                           : QSM_ERR_CUDA;
}

template <int D, int MAP, int SURR>
qsm_status launch_dkdv(const BwdArgs &a, BwdParams p, const CUtensorMap &mq,
                       const CUtensorMap &mk, const CUtensorMap &mv, const CUtensorMap &mdo) {
  using G = BGeo<D>;
  using KG = KvGeo<D>;
  // K, V, ns x (Q, dO rows, their constants and tables), barriers
  const size_t stage = (2 * KG::QBYTES + KG::SROWS * kCst * 4 +
                        static_cast<size_t>(KG::SROWS) * p.TS * 4 + 1023) &
                       ~static_cast<size_t>(1023);
  const size_t fixed = 1024 + 2 * G::TILE_BYTES + kBarBytes;
  int ns = static_cast<int>((kMaxSmem - fixed) / stage);
  if (ns > 4) ns = 4;
  if (ns < 2) return QSM_ERR_UNSUPPORTED;
  p.num_stages = ns;
  p.stage_bytes = static_cast<uint32_t>(stage);
  p.bar_off = static_cast<uint32_t>(2 * G::TILE_BYTES + ns * stage);
  size_t smem = 1024 + p.bar_off + kBarBytes;
  if (smem < 120 * 1024) smem = 120 * 1024;
  if (smem > kMaxSmem) return QSM_ERR_UNSUPPORTED;
  auto kern = qsm_bwd_dkdv<D, MAP, SURR>;
  static std::atomic<int> cache[kMaxDevices];
  if (!set_smem_once(kern, static_cast<int>(smem), cache)) return QSM_ERR_CUDA;
  // persistent: one CTA per SM walks the key tiles
  const int ntiles = p.nkvt * a.B * a.H;
  const int grid = ntiles < sm_count() ? ntiles : sm_count();
  return launch_dependent(kern, grid, smem, a.stream, mq, mk, mv, mdo, p) == cudaSuccess ? QSM_OK
                                                                           : QSM_ERR_CUDA;
}

template <int D, int MAP, int SURR, int CAL>
qsm_status launch_prep(const BwdArgs &a, const BwdParams &p) {
  const int grid = p.nqt * a.B * a.H, block = 128 * prep_split<MAP>();
  if (SURR == SURR_POST && D == 64) {
    // behind the row pass, as its dependent (it waits before the row
    // constants).  Measured against the plain launch on one box: +0.3-2.5 %
    // for the D = 64 post-surrogate calls, but -5 to -7 % at D = 128 with
    // min-max calibration, so D = 128 keeps the plain launch.
    return launch_dependent_block(qsm_bwd_prep<D, MAP, SURR, CAL>, grid, block, 0, a.stream, p) ==
                   cudaSuccess
               ? QSM_OK
               : QSM_ERR_CUDA;
  }
  qsm_bwd_prep<D, MAP, SURR, CAL><<<dim3(grid), block, 0, a.stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? QSM_OK : QSM_ERR_CUDA;
}

template <int D, int MAP, int SURR, int CAL>
qsm_status launch_passes(const BwdArgs &a, const BwdParams &p0, const BwdMaps &m) {
  BwdParams p = p0;
  p.tabq_tile = static_cast<uint32_t>(DqTab<MAP, SURR, CAL>::bytes(p.K));
  qsm_status st = launch_prep<D, MAP, SURR, CAL>(a, p);
  if (st != QSM_OK) return st;
  // the dQ pass stages K, V by KROWS-row boxes, the dK / dV pass Q, dO by
  // SROWS-row boxes
  st = launch_dq<D, MAP, SURR, CAL>(a, p, m.q, m.k_stage, m.v_stage, m.dO);
  if (st != QSM_OK) return st;
  return launch_dkdv<D, MAP, SURR>(a, p, m.q_stage, m.k, m.v, m.dO_stage);
}

template <int D, int MAP, int CAL>
qsm_status launch_by_surr(int surr, const BwdArgs &a, const BwdParams &p, const BwdMaps &m) {
  if (surr == SURR_PRE) return launch_passes<D, MAP, SURR_PRE, CAL>(a, p, m);
  if (surr == SURR_POST) return launch_passes<D, MAP, SURR_POST, CAL>(a, p, m);
  return launch_passes<D, MAP, SURR_NONE, CAL>(a, p, m);
}

template <int D>
qsm_status launch_rows(const BwdArgs &a, BwdParams p, const CUtensorMap &mq,
                       const CUtensorMap &mk, const CUtensorMap &mv, const CUtensorMap &mdo) {
  using G = BGeo<D>;
  // Q, dO, ns x (K, V), two tiles' partial sums, barriers
  const size_t part = 2 * 2 * 4 * 128 * sizeof(float);
  const size_t fixed = 1024 + 2 * G::TILE_BYTES + part + kBarBytes;
  int ns = static_cast<int>((kMaxSmem - fixed) / (2 * G::TILE_BYTES));
  if (ns > 4) ns = 4;
  if (ns < 2) return QSM_ERR_UNSUPPORTED;
  p.num_stages = ns;
  p.part_off = static_cast<uint32_t>(2 * G::TILE_BYTES + ns * 2 * G::TILE_BYTES);
  p.bar_off = static_cast<uint32_t>(p.part_off + part);
  size_t smem = 1024 + p.bar_off + kBarBytes;
  if (smem < 120 * 1024) smem = 120 * 1024;            // one CTA per SM (all of TMEM)
  if (smem > kMaxSmem) return QSM_ERR_UNSUPPORTED;
  auto kern = qsm_bwd_rows<D>;
  static std::atomic<int> cache[kMaxDevices];
  if (!set_smem_once(kern, static_cast<int>(smem), cache)) return QSM_ERR_CUDA;
  // persistent: one CTA per SM walks the query tiles
  const int ntiles = p.nqt * a.B * a.H;
  const int grid = ntiles < sm_count() ? ntiles : sm_count();
  kern<<<dim3(grid), kMainThreads, smem, a.stream>>>(mq, mk, mv, mdo, p);
  return cudaGetLastError() == cudaSuccess ? QSM_OK : QSM_ERR_CUDA;
}

constexpr int kTabKT = (kBwdMaxK + 2) & ~1;              // float2 entries per row, workspace
// bytes of one query tile's dQ-pass table at the largest K (interpolation
// with min-max calibration: K + 2 entries of 16 bytes per row)
constexpr size_t kTabQTile = static_cast<size_t>(kBwdMaxK + 2) * 16 * 128;

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// The post surrogate's row pass, then the passes of the map, surrogate and
// calibration form.
template <int D>
qsm_status launch_maps(const BwdArgs &a, const BwdParams &p, int map, int cal, const BwdMaps &m) {
  if (map != MAPB_EXACT && a.surrogate == QSM_SURR_POST) {
    const qsm_status st = launch_rows<D>(a, p, m.q, m.k, m.v, m.dO);
    if (st != QSM_OK) return st;
  }
  const int surr = a.surrogate;
  if (map == MAPB_EXACT) return launch_passes<D, MAPB_EXACT, SURR_NONE, CAL_OFF>(a, p, m);
  if (map == MAPB_POT) return launch_by_surr<D, MAPB_POT, CAL_OFF>(surr, a, p, m);
  if (map == MAPB_HARD) {
    if (cal == CAL_MINMAX) return launch_by_surr<D, MAPB_HARD, CAL_MINMAX>(surr, a, p, m);
    return launch_by_surr<D, MAPB_HARD, CAL_OFF>(surr, a, p, m);
  }
  if (cal == CAL_MINMAX) return launch_by_surr<D, MAPB_INTERP, CAL_MINMAX>(surr, a, p, m);
  if (cal == CAL_FIXED) return launch_by_surr<D, MAPB_INTERP, CAL_FIXED>(surr, a, p, m);
  return launch_by_surr<D, MAPB_INTERP, CAL_OFF>(surr, a, p, m);
}

}  // namespace

size_t bwd_workspace_bytes(int B, int H, int S, int D) {
  // fp32 calibration part of dK and the row workspace per query row, then
  // per tile row (each head's rows padded to whole 128-row tiles) the map
  // constants and the dK / dV pass's grid table, and per query tile the dQ
  // pass's table; each part 256-byte aligned
  const size_t rows = static_cast<size_t>(B) * H * S;
  const size_t tiles = static_cast<size_t>(B) * H * ((S + 127) / 128);
  const size_t trows = tiles * 128;
  // (D = 128: bf16 copies of e4m3 Q, K, V)
  const size_t deq = D == 128 ? 3 * align256(rows * D * 2) : 0;
  return align256(rows * D * sizeof(float)) + align256(rows * kRowWs * sizeof(float)) +
         align256(trows * kCst * sizeof(float)) + align256(trows * kTabKT * sizeof(float2)) +
         align256(tiles * kTabQTile) + deq;
}

qsm_status launch_bwd(const BwdArgs &a) {
  if (a.D != 64 && a.D != 128) return QSM_ERR_UNSUPPORTED;
  if (a.mode == QSM_MODE_KINTERVAL && a.Kint > kBwdMaxK) return QSM_ERR_UNSUPPORTED;
  const size_t rows = static_cast<size_t>(a.B) * a.H * a.S;
  const int map = a.mode == QSM_MODE_EXACT       ? MAPB_EXACT
                  : a.mode == QSM_MODE_ROWMAX_POT ? MAPB_POT
                  : (a.rounding == QSM_ROUND_HARD ? MAPB_HARD : MAPB_INTERP);
  BwdParams p{};
  p.S = a.S;
  p.nqt = (a.S + 127) / 128;
  p.nkvt = p.nqt;
  p.BH = a.B * a.H;
  p.causal = a.causal;
  p.hgroup = causal_head_group(a.S, a.D, false, p.BH);
  p.pot_floor = a.pot_floor;
  p.K = a.mode == QSM_MODE_KINTERVAL ? a.Kint : 1;
  p.fixed_window = a.calib == QSM_CALIB_FIXED_WINDOW;
  p.flush = a.below_policy == 1;
  // the dK / dV pass's table row: interpolation K + 2 (e, d) pairs, hard
  // rounding K + 1 grid values; a multiple of 4 floats (16-byte copies)
  p.TS = map == MAPB_INTERP ? ((2 * (p.K + 2) + 3) & ~3)
         : map == MAPB_HARD ? ((p.K + 1 + 3) & ~3)
                            : 0;
  p.c = a.c;
  p.cL2E = a.c * 1.4426950408889634f;
  // gradients with respect to the tensors the scores are formed from: Q, K
  // (bf16), or q_descale Q, k_descale K (e4m3), whose bf16 copies hold the
  // codes, so dQ = scale k_descale dS K and dK = scale q_descale dS^T Q
  p.gq = a.fp8 ? a.scale * a.k_descale : a.c;
  p.gk = a.fp8 ? a.scale * a.q_descale : a.c;
  p.window = a.window;
  p.LSE = a.LSE;
  p.hi = a.row_hi;
  p.lo = a.row_lo;
  p.amax = a.row_argmax;
  p.amin = a.row_argmin;
  // calibration form: none when detached, and for fixed-window hard rounding,
  // whose grid does not move with hi
  const bool calib = a.mode == QSM_MODE_KINTERVAL && !a.detach &&
                     !(map == MAPB_HARD && p.fixed_window);
  const int cal = !calib ? CAL_OFF : (p.fixed_window ? CAL_FIXED : CAL_MINMAX);
  uint8_t *ws = static_cast<uint8_t *>(a.workspace);
  const size_t o_dk = 0;
  const size_t o_rw = o_dk + align256(rows * a.D * sizeof(float));
  const size_t o_cst = o_rw + align256(rows * kRowWs * sizeof(float));
  const size_t trows = static_cast<size_t>(p.BH) * p.nqt * 128;
  const size_t o_tab = o_cst + align256(trows * kCst * sizeof(float));
  const size_t o_tabq = o_tab + align256(trows * kTabKT * sizeof(float2));
  const size_t o_deq = o_tabq + align256(static_cast<size_t>(p.BH) * p.nqt * kTabQTile);
  p.dkcal = calib ? reinterpret_cast<float *>(ws + o_dk) : nullptr;
  p.rowws = reinterpret_cast<float *>(ws + o_rw);
  p.cst = reinterpret_cast<float *>(ws + o_cst);
  p.tabk = reinterpret_cast<float *>(ws + o_tab);
  p.tabq = ws + o_tabq;
  const void *Qp = a.Q, *Kp = a.K, *Vp = a.V;
  if (a.fp8) {
    if (a.D != 128) return QSM_ERR_UNSUPPORTED;
    const size_t part = align256(rows * a.D * 2);
    uint4 *qb = reinterpret_cast<uint4 *>(ws + o_deq);
    uint4 *kb = reinterpret_cast<uint4 *>(ws + o_deq + part);
    uint4 *vb = reinterpret_cast<uint4 *>(ws + o_deq + 2 * part);
    const size_t n8 = rows * a.D / 8;
    const size_t want = (n8 + 255) / 256;
    const int grid = static_cast<int>(want < 8 * 148 ? want : 8 * 148);
    qsm_bwd_dequant<<<grid, 256, 0, a.stream>>>(static_cast<const uint2 *>(a.Q),
                                                 static_cast<const uint2 *>(a.K),
                                                 static_cast<const uint2 *>(a.V), qb, kb, vb, n8,
                                                 a.v_descale);
    if (cudaGetLastError() != cudaSuccess) return QSM_ERR_CUDA;
    Qp = qb;
    Kp = kb;
    Vp = vb;
  }
  p.Q = static_cast<const __nv_bfloat16 *>(Qp);
  p.K_ = static_cast<const __nv_bfloat16 *>(Kp);
  p.O = static_cast<const __nv_bfloat16 *>(a.O);
  p.dO = static_cast<const __nv_bfloat16 *>(a.dO);
  p.dQ = static_cast<__nv_bfloat16 *>(a.dQ);
  p.dK = static_cast<__nv_bfloat16 *>(a.dK);
  p.dV = static_cast<__nv_bfloat16 *>(a.dV);
  p.status = a.status_dev;

  BwdMaps m;
  const int bh = a.B * a.H;
  const int srows = a.D > 64 ? 64 : 128;               // the passes' stage boxes
  if (!make_tmap_3d(&m.q, Qp, false, a.D, a.S, bh, 128) ||
      !make_tmap_3d(&m.k, Kp, false, a.D, a.S, bh, 128) ||
      !make_tmap_3d(&m.v, Vp, false, a.D, a.S, bh, 128) ||
      !make_tmap_3d(&m.dO, a.dO, false, a.D, a.S, bh, 128) ||
      !make_tmap_3d(&m.q_stage, Qp, false, a.D, a.S, bh, srows) ||
      !make_tmap_3d(&m.k_stage, Kp, false, a.D, a.S, bh, srows) ||
      !make_tmap_3d(&m.v_stage, Vp, false, a.D, a.S, bh, srows) ||
      !make_tmap_3d(&m.dO_stage, a.dO, false, a.D, a.S, bh, srows))
    return QSM_ERR_CUDA;

  // (the prep kernel zeroes the calibration part of dK, p.dkcal)
  return a.D == 64 ? launch_maps<64>(a, p, map, cal, m) : launch_maps<128>(a, p, map, cal, m);
}

}  // namespace qsm
