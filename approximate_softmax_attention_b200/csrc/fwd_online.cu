// fwd_online.cu -- one-sweep attention forward for sm_100a: the online
// softmax (exact map) and the online-anchor approximate maps.
//
// The pages' kernel is a one-sweep FlashAttention-4 patch ("Rowmax-H15 in
// FlashAttention-4 on B200", wiki flowchart: QK tile -> row max (anchor) ->
// power-of-two weights -> PV matmul -> output).  A one-sweep kernel knows only
// the maximum of the keys it has visited, so here each key tile is anchored
// at the row's running maximum after that tile, tiles in increasing key
// order, and the accumulators carry over by the factor the anchor's move
// implies:
//   exact       w = exp(s - a_t), carried by exp(a_{t-1} - a_t): softmax;
//   Rowmax-PoT  w = 2^-min(rne((a_t - s) log2 e), N), carried by
//               2^-rne((a_t - a_{t-1}) log2 e): every weight a power of two;
//   K-interval  (fixed window) the grid [a_t - W, a_t], carried by
//               exp(a_{t-1} - a_t).
//
// One CTA per 128-row query tile (same grid and order as the two-sweep
// kernel), 640 threads:
//   warp 0      TMA producer: Q once, then K and V tiles through a ring (K
//               three tiles ahead of V).
//   warp 1      QK issuer: S_j = Q K_j^T into TMEM buffer j % 3.
//   warp 2      PV issuer: O += P_j V_j, P read from TMEM.
//   warps 4-7   the anchor warpgroup: one thread per query row sweeps every
//               tile in key order, folds the tile's row maximum into the
//               running maximum (in its own registers), decides the frame,
//               publishes both for the tile, and rescales O when the frame
//               moves (after PV(j-1) has landed, before PV(j)).
//   warps 8-19  three map warpgroups; group g maps the key tiles j = g mod 3
//               (buffer g), one thread per query row covering all 128 key
//               columns, against the anchor published for the tile.
// TMEM: S / P buffers at columns 0, 128, 256; O at 384.
//
// Frames.  The accumulators are kept in a per-row frame `base` (log2 units)
// that follows the anchor lazily: the weights written to P are w * 2^(F -
// base) with F the anchor's own frame value, and O (and the groups' row sums)
// are rescaled only when F - base would exceed what the P format holds (exact
// and K-interval: 2^8 in bf16; e4m3: 2^8 exact, 2^4 K-interval with a 16x P
// scale; PoT, whose frame value is the integer sum of its rounded anchor
// moves: 2^64 in bf16, 2^2 in e4m3 with its 64x P scale).  The result is the same up to rounding (PoT: exactly,
// every factor being a power of two).
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

struct OnParams {
  int S, nqt, BH;
  int causal;
  int hgroup;       // causal work order: heads per group (their K/V shares L2)
  int K;
  int flush;        // below_policy == 1
  int pot_floor;
  float c;          // score scale
  float cL2E;       // c * log2(e)
  float window;
  float v_descale;
  float pscale;     // P is stored as w * pscale (e4m3 approximate maps: 64)
  float tau;        // frame slack in log2 units (see the file comment)
  int num_stages;
  uint32_t table_off, bar_off, row_off;
  __nv_bfloat16 *O;
  float *LSE, *hi, *lo;
  int8_t *dbg;
  int32_t *status;
  int debug_flags;
};

template <int D, bool FP8>
struct OGeo {
  static constexpr int ELEM = FP8 ? 1 : 2;
  static constexpr int EPC = 128 / ELEM;                // elements per 128-byte swizzle row
  static constexpr int CHUNKS = (D * ELEM) / 128;       // swizzle columns per tile
  static constexpr int CHUNK_BYTES = 128 * 128;
  static constexpr int TILE_BYTES = 128 * D * ELEM;
  static constexpr int MMA_K = FP8 ? 32 : 16;
  static constexpr int KSTEPS_QK = D / MMA_K;
  static constexpr int KSTEPS_PV = 128 / MMA_K;
  static constexpr uint32_t FMT = FP8 ? 0u : 1u;
  static constexpr uint32_t IDESC_QK = instr_desc(FMT, false, 128, 128);
  static constexpr uint32_t IDESC_PV = instr_desc(FMT, true, 128, D);
};

constexpr int kOnThreads = 640;     // control, anchor and three map warpgroups
constexpr int kOnGroups = 3;
constexpr int kOnMapThreads = 128 * kOnGroups;
constexpr int kOnBufs = 3;
constexpr uint32_t kOnOCol = 384;
constexpr uint32_t kOnTmemCols = 512;
constexpr int kOnMaxStages = 8;
constexpr int kOnLead = 3;          // K tiles enter the ring this far ahead of V

__device__ __forceinline__ int on_pos_k(int j) { return j < kOnLead ? j : 2 * j - kOnLead + 1; }
__device__ __forceinline__ int on_pos_v(int j, int n) {
  return j < n - kOnLead ? kOnLead + 2 * j : n + j;
}

struct OnBars {
  uint64_t *kv_full, *kv_empty;          // [stages]
  uint64_t *q_full;
  uint64_t *s_full, *p_full, *s_free;    // [kOnBufs]
  uint64_t *anc_ready;                   // [kOnBufs]: tile j's anchor and frame published
  uint64_t *tab_ready;                   // the grid table is built
  uint64_t *o_full, *drain, *fin_ready, *zx;
  uint32_t *tmem_slot;
  int *abort;
};
constexpr int kOnFixedBars = 1 + 4 * kOnBufs + 1 + 4;

__host__ __device__ constexpr size_t on_bar_bytes(int ns) {
  return ((2 * static_cast<size_t>(ns) + kOnFixedBars) * 8 + 8 + 15) & ~static_cast<size_t>(15);
}

__device__ __forceinline__ OnBars on_carve(uint8_t *base, int ns) {
  OnBars b;
  uint64_t *p = reinterpret_cast<uint64_t *>(base);
  b.kv_full = p;
  b.kv_empty = p + ns;
  b.q_full = p + 2 * ns;
  b.s_full = b.q_full + 1;
  b.p_full = b.s_full + kOnBufs;
  b.s_free = b.p_full + kOnBufs;
  b.anc_ready = b.s_free + kOnBufs;
  b.tab_ready = b.anc_ready + kOnBufs;
  b.o_full = b.tab_ready + 1;
  b.drain = b.o_full + 1;
  b.fin_ready = b.drain + 1;
  b.zx = b.fin_ready + 1;
  b.tmem_slot = reinterpret_cast<uint32_t *>(b.zx + 1);
  b.abort = reinterpret_cast<int *>(b.tmem_slot + 1);
  return b;
}

// Per-row state in shared memory: the anchor published for each buffer's
// tile, the final values, and the map groups' row sums at the end.
struct OnRows {
  float *a, *base, *C;     // [kOnBufs][128]: running max of r, frame, PoT move sum
  float *fa, *fbase, *fC, *fmn;   // [128]: after the last tile (and the running min)
  float *zx;               // [kOnGroups][128]
};
constexpr size_t kOnRowBytes = (3 * kOnBufs + 4 + kOnGroups) * 128 * 4;

__device__ __forceinline__ bool on_all(bool x) { return __all_sync(0xffffffffu, x); }
__device__ __forceinline__ bool on_any(bool x) { return __any_sync(0xffffffffu, x); }

__device__ __forceinline__ bool on_full_tile(const OnParams &p, int qi, int j) {
  return 128 * (j + 1) <= p.S && (!p.causal || j < qi);
}

// 2^(from - to), the factor that carries a value from one frame to another:
// for Rowmax-PoT the frames are whole numbers and the factor is built from
// the exponent field (exact); otherwise exp2 of the difference.
template <int MAP>
__device__ __forceinline__ float frame_factor(float from, float to) {
  const float d = __fsub_rn(from, to);
  if (MAP == MAP_POT) {
    const int e = static_cast<int>(d);
    if (e < -126) return 0.0f;
    return __int_as_float((127 + min(e, 127)) << 23);
  }
  return exp2f(d);
}

// Weights of one 32-column chunk (masked), packed for the PV product and
// stored into the buffer's columns c*16 (bf16) or c*8 (e4m3) -- columns this
// thread has already read -- with the row sum accumulated.
template <int MAP, bool FULL, bool FLUSH, bool FP8, bool SAT = false>
__device__ __forceinline__ void on_chunk(const uint32_t (&v)[32], const MapRow &mr, float cL2E,
                                         float fr, bool flush_below, int c0, int lim,
                                         float2 (&z)[4], uint32_t taddr) {
  auto wt = [&](int i) {
    const float2 r = make_float2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
    float2 x;
    if (MAP == MAP_EXACT) {
      x = exact_pair(r, cL2E, mr.mL2E);
    } else if (MAP == MAP_POT) {
      x = map_pair<MAP_POT, FLUSH>(r, mr);
    } else {
      x = pair_weights<MAP, false, SAT>(r, mr, flush_below);
      x = mul2_rn(x, make_float2(fr, fr));           // into the group's frame
    }
    if (!FULL) {
      x.x = (c0 + 2 * i < lim) ? x.x : 0.0f;
      x.y = (c0 + 2 * i + 1 < lim) ? x.y : 0.0f;
    }
    z[i & 3] = add2_rn(z[i & 3], x);
    return x;
  };
  if (FP8) {
    uint32_t pk[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float2 a = wt(2 * i), b = wt(2 * i + 1);
      pk[i] = pack_e4m3x4(a.x, a.y, b.x, b.y);
    }
    tmem_st8(taddr, pk);
  } else {
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float2 a = wt(i);
      pk[i] = pack_bf16x2(a.x, a.y);
    }
    tmem_st16(taddr, pk);
  }
}

// The frame value F of a tile with running maximum a (raw units): the
// anchor in log2 units (exact, K-interval); PoT keeps the integer sum of its
// rounded moves, tracked by the caller.
template <int MAP>
__device__ __forceinline__ float anchor_l2e(const OnParams &p, float a) {
  if (MAP == MAP_EXACT) return __fmul_rn(a, p.cL2E);
  return __fmul_rn(__fmul_rn(p.c, a), log2e_f());
}

// The anchor warpgroup.  Thread `row` owns query row qi*128 + row and visits
// every key tile in order: the tile's row maximum (and minimum) from TMEM, the
// running maximum, the frame, the published slot for the tile's map group, and
// the O rescale when the frame moves.
template <int D, int MAP>
__device__ __forceinline__ void on_anchor(const OnParams &p, const OnBars &bars, const OnRows &rs,
                                          int row, uint32_t lane_base, int qi, int n,
                                          volatile int *abort) {
  const int qrow = qi * 128 + row;
  const int L = p.causal ? min(qrow + 1, p.S) : p.S;
  const bool want_min = p.lo != nullptr && MAP != MAP_KI_HARD && MAP != MAP_KI_INTERP;
  float a = -INFINITY, mn = INFINITY, base = 0.0f, C = 0.0f, prev_l2e = 0.0f;
  bool ok = true;
  for (int j = 0; j < n && ok; ++j) {
    const int b = j % kOnBufs;
    ok = on_all(mbar_wait(&bars.s_full[b], (j / kOnBufs) & 1, abort));
    if (!ok) break;
    tc_fence_after();
    const int lim = L - 128 * j;
    const bool full = on_full_tile(p, qi, j);
    const uint32_t sb = lane_base + b * 128;
    float tmax = -INFINITY, tmin = INFINITY;
#pragma unroll 1
    for (int h = 0; h < 2; ++h) {
      uint32_t v0[32], v1[32];
      tmem_ld32(sb + 64 * h, v0);
      tmem_ld32(sb + 64 * h + 32, v1);
      tmem_wait_ld();
      reg_fence32(v0);
      reg_fence32(v1);
      if (full) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          tmax = max3n(tmax, __uint_as_float(v0[2 * i]), __uint_as_float(v0[2 * i + 1]));
          tmax = max3n(tmax, __uint_as_float(v1[2 * i]), __uint_as_float(v1[2 * i + 1]));
          if (want_min) {
            tmin = min3n(tmin, __uint_as_float(v0[2 * i]), __uint_as_float(v0[2 * i + 1]));
            tmin = min3n(tmin, __uint_as_float(v1[2 * i]), __uint_as_float(v1[2 * i + 1]));
          }
        }
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const bool o0 = 64 * h + i < lim, o1 = 64 * h + 32 + i < lim;
          const float x0 = __uint_as_float(v0[i]), x1 = __uint_as_float(v1[i]);
          tmax = max3n(tmax, o0 ? x0 : -INFINITY, o1 ? x1 : -INFINITY);
          if (want_min) tmin = min3n(tmin, o0 ? x0 : INFINITY, o1 ? x1 : INFINITY);
        }
      }
    }
    // every row has a valid key in every tile it visits (key 0 in tile 0; a
    // later tile below the diagonal is full); the NaN-propagating max keeps a
    // NaN anchor NaN
    const float an = (lim > 0) ? max3n(a, tmax, tmax) : a;
    mn = min3n(mn, tmin, tmin);
    const float l2e = anchor_l2e<MAP>(p, an);
    if (MAP == MAP_POT && j > 0) C = __fadd_rn(C, rne_f(__fsub_rn(l2e, prev_l2e)));
    const float F = (MAP == MAP_POT) ? C : l2e;
    // move the frame to the anchor when the slack runs out (or on a NaN)
    const float nb = (j == 0 || !(__fsub_rn(F, base) <= p.tau)) ? F : base;
    const float resc = (j == 0 || nb == base) ? 1.0f : frame_factor<MAP>(base, nb);
    rs.a[b * 128 + row] = an;
    rs.base[b * 128 + row] = nb;
    rs.C[b * 128 + row] = C;
    mbar_arrive(&bars.anc_ready[b]);
    if (j > 0 && on_any(resc != 1.0f)) {
      // O to the new frame, after PV(j-1) has landed (PV(j) waits for this
      // group's arrival below)
      const int pj = j - 1;
      ok = on_all(mbar_wait(&bars.s_free[pj % kOnBufs], (pj / kOnBufs) & 1, abort));
      if (!ok) break;
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t v[32];
        tmem_ld32_sync(lane_base + kOnOCol + 32 * c, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * resc);
        tmem_st32(lane_base + kOnOCol + 32 * c, v);
      }
      tmem_wait_st();
    }
    tc_fence_before();
    mbar_arrive(&bars.p_full[b]);
    a = an;
    base = nb;
    prev_l2e = l2e;
  }
  rs.fa[row] = a;
  rs.fbase[row] = base;
  rs.fC[row] = C;
  rs.fmn[row] = mn;
  mbar_arrive(bars.fin_ready);
}

// One map warpgroup.  Thread `row` owns query row qi*128 + row (TMEM lane
// `row`) and maps key tiles j = g, g + 3, ... in S buffer g against the
// anchor and frame the anchor group published for the tile.  DBG: the
// kernel writes the decision dump (a separate instantiation, so that the
// dump's code takes no registers from the ordinary one).
template <int D, bool FP8, int MAP, bool KSAT, bool DBG>
__device__ __forceinline__ void on_map(const OnParams &p, const OnBars &bars, const OnRows &rs,
                                       int g, int row, uint32_t lane_base, int qi, int n, int bh,
                                       float *tab, volatile int *abort) {
  constexpr int PCOLS = FP8 ? 8 : 16;                   // TMEM columns per 32 P values
  const int qrow = qi * 128 + row;
  const bool row_ok = qrow < p.S;
  const int L = p.causal ? min(qrow + 1, p.S) : p.S;
  const bool flush_below = (MAP == MAP_KI_HARD || MAP == MAP_KI_INTERP) && p.flush;
  const bool pot_flush = MAP == MAP_POT && p.flush;

  bool ok = true;

  MapCall mc;
  mc.K = p.K;
  mc.fixed_window = 1;
  mc.flush = p.flush;
  mc.pot_floor = p.pot_floor;
  mc.c = p.c;
  mc.cL2E = p.cL2E;
  mc.window = p.window;
  mc.pscale = p.pscale;
  mc.thr = 0.0f;
  if (MAP == MAP_KI_HARD || MAP == MAP_KI_INTERP) {
    // the fixed-window grid values do not depend on the anchor: one table,
    // built once (the three groups take interleaved entries of each row)
    float hi_d, lo_d;
    (void)row_setup<MAP>(mc, 0.0f, 0.0f, tab, row, g, kOnGroups, hi_d, lo_d);
    mbar_arrive(bars.tab_ready);
    ok = on_all(mbar_wait(bars.tab_ready, 0, abort));
  }

  float2 z[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) z[i] = make_float2(0.0f, 0.0f);
  float zbase = 0.0f;                  // frame of this group's row sums
  bool zset = false;
  int8_t *dbg_row = (DBG && p.dbg != nullptr && row_ok)
                        ? p.dbg + (static_cast<size_t>(bh) * p.S + qrow) * p.S
                        : nullptr;

  for (int j = g; j < n && ok; j += kOnGroups) {
    const int b = g;                                    // j % 3
    const uint32_t par = (j / kOnBufs) & 1;
    ok = on_all(mbar_wait(&bars.s_full[b], par, abort));
    if (ok) ok = on_all(mbar_wait(&bars.anc_ready[b], par, abort));
    if (!ok) break;
    tc_fence_after();
    const int lim = L - 128 * j;
    const bool full = on_full_tile(p, qi, j);
    const uint32_t sb = lane_base + b * 128;
    const float a = rs.a[b * 128 + row];
    const float base = rs.base[b * 128 + row];
    MapRow mr;
    float fr = 1.0f;                                    // K-interval frame factor
    if (MAP == MAP_EXACT) {
      mr.mL2E = base;
    } else if (MAP == MAP_POT) {
      float hi_t, lo_t;
      mr = row_setup<MAP_POT>(mc, a, a, tab, row, 0, 1, hi_t, lo_t);
      mr.pow_bias = __float_as_uint(p.pscale) +
                    (static_cast<uint32_t>(static_cast<int>(__fsub_rn(rs.C[b * 128 + row], base)))
                     << 23);
    } else {
      // n0 = K + 1: no table entry is written (the table is shared and
      // constant); this only forms the tile's coordinate map
      float hi_t, lo_t;
      mr = row_setup<MAP>(mc, a, a, tab, row, p.K + 1, 1, hi_t, lo_t);
      fr = exp2f(__fsub_rn(anchor_l2e<MAP>(p, a), base));
    }
    // this group's row sums into the tile's frame
    if (zset && zbase != base) {
      const float f = frame_factor<MAP>(zbase, base);
#pragma unroll
      for (int i = 0; i < 4; ++i) z[i] = make_float2(z[i].x * f, z[i].y * f);
    }
    zbase = base;
    zset = true;
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      uint32_t v[32];
      tmem_ld32_sync(sb + 32 * c, v);
      const uint32_t pc = sb + c * PCOLS;
      if (pot_flush) {
        if (full)
          on_chunk<MAP, true, true, FP8>(v, mr, p.cL2E, fr, flush_below, 32 * c, lim, z, pc);
        else
          on_chunk<MAP, false, true, FP8>(v, mr, p.cL2E, fr, flush_below, 32 * c, lim, z, pc);
      } else if (KSAT) {
        if (full)
          on_chunk<MAP, true, false, FP8, true>(v, mr, p.cL2E, fr, flush_below, 32 * c, lim, z, pc);
        else
          on_chunk<MAP, false, false, FP8, true>(v, mr, p.cL2E, fr, flush_below, 32 * c, lim, z, pc);
      } else if (full) {
        on_chunk<MAP, true, false, FP8>(v, mr, p.cL2E, fr, flush_below, 32 * c, lim, z, pc);
      } else {
        on_chunk<MAP, false, false, FP8>(v, mr, p.cL2E, fr, flush_below, 32 * c, lim, z, pc);
      }
      if (dbg_row != nullptr) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int kv = 128 * j + 32 * c + i;
          if (kv < p.S) {
            const float r = __uint_as_float(v[i]);
            int d = map_raw_index<MAP, KSAT>(r, mr, p.flush != 0, p.pot_floor);
            if (flush_below && __fmaf_rn(r, mr.a, mr.b) < 0.0f) d = -2;
            dbg_row[kv] = static_cast<int8_t>((32 * c + i < lim) ? d : -1);
          }
        }
      }
    }
    tmem_wait_st();
    tc_fence_before();
    mbar_arrive(&bars.p_full[b]);
  }

  // ---------------------------------------------------------- epilogue
  if (ok) ok = on_all(mbar_wait(bars.o_full, 0, abort));
  if (ok) ok = on_all(mbar_wait(bars.fin_ready, 0, abort));
  if (!ok) return;
  tc_fence_after();
  const float a = rs.fa[row], base = rs.fbase[row], Cf = rs.fC[row];
  const float zg = ((z[0].x + z[0].y) + (z[1].x + z[1].y)) + ((z[2].x + z[2].y) + (z[3].x + z[3].y));
  rs.zx[g * 128 + row] =
      (zset && zg != 0.0f) ? (zbase == base ? zg : zg * frame_factor<MAP>(zbase, base)) : 0.0f;
  mbar_arrive(bars.zx);
  if (!on_all(mbar_wait(bars.zx, 0, abort))) return;
  const float Z = (rs.zx[row] + rs.zx[128 + row]) + rs.zx[256 + row];
  const float hi = __fmul_rn(p.c, a);
  // the final weights' frame: the last anchor (exact, K-interval) or the
  // sum of the anchor moves (PoT)
  const float ref = (MAP == MAP_POT) ? Cf : anchor_l2e<MAP>(p, a);
  const bool bad = !(fabsf(hi) <= 3.402823466e38f);
  const float qnan = __int_as_float(0x7FFFFFFF);
  const float oscale = bad ? qnan : p.v_descale / Z;   // pscale and the frame cancel
#pragma unroll 1
  for (int ch = g; ch < D / 32; ch += kOnGroups) {
    uint32_t v[32];
    tmem_ld32_sync(lane_base + kOnOCol + 32 * ch, v);
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 16; ++i)
      pk[i] = pack_bf16x2(__uint_as_float(v[2 * i]) * oscale, __uint_as_float(v[2 * i + 1]) * oscale);
    if (row_ok) {
      uint4 *d4 = reinterpret_cast<uint4 *>(p.O + (static_cast<size_t>(bh) * p.S + qrow) * D + 32 * ch);
#pragma unroll
      for (int i = 0; i < 4; ++i) d4[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
    }
  }
  if (row_ok && g == 0) {
    const size_t ri = static_cast<size_t>(bh) * p.S + qrow;
    p.LSE[ri] = bad ? qnan : hi + (logf(Z / p.pscale) + __fsub_rn(base, ref) * 0.6931471805599453f);
    if (p.hi) p.hi[ri] = hi;
    if (p.lo) p.lo[ri] = (MAP == MAP_KI_HARD || MAP == MAP_KI_INTERP)
                             ? __fsub_rn(hi, p.window) : __fmul_rn(p.c, rs.fmn[row]);
  }
}

template <int D, bool FP8, int MAP, bool KSAT, bool DBG>
__global__ void __launch_bounds__(kOnThreads, 1)
    qsm_fwd_online_kernel(const __grid_constant__ CUtensorMap tmQ,
                          const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV, const OnParams p) {
  using G = OGeo<D, FP8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = smem_align1024(smem_raw);
  const int warp = threadIdx.x >> 5;
  int bh, qi;
  if (p.causal) {
    const int per = p.hgroup * p.nqt;
    const int grp = static_cast<int>(blockIdx.x) / per;
    const int within = static_cast<int>(blockIdx.x) - grp * per;
    const int h0 = grp * p.hgroup;
    const int gh = min(p.hgroup, p.BH - h0);
    const int rank = within / gh;
    bh = h0 + (within - rank * gh);
    qi = p.nqt - 1 - rank;
  } else {
    qi = static_cast<int>(blockIdx.x) % p.nqt;
    bh = static_cast<int>(blockIdx.x) / p.nqt;
  }
  const int ns = p.num_stages;
  uint8_t *sQ = smem;
  uint8_t *sKV = smem + G::TILE_BYTES;
  float *sTab = reinterpret_cast<float *>(smem + p.table_off);
  OnBars bars = on_carve(smem + p.bar_off, ns);
  OnRows rs;
  float *rowp = reinterpret_cast<float *>(smem + p.row_off);
  rs.a = rowp;
  rs.base = rowp + kOnBufs * 128;
  rs.C = rowp + 2 * kOnBufs * 128;
  rs.fa = rowp + 3 * kOnBufs * 128;
  rs.fbase = rs.fa + 128;
  rs.fC = rs.fa + 256;
  rs.fmn = rs.fa + 384;
  rs.zx = rs.fa + 512;
  volatile int *abort = bars.abort;
  const int nkvt = (p.S + 127) / 128;
  const int n = p.causal ? min(nkvt, qi + 1) : nkvt;

  if (threadIdx.x == 0) {
    for (int i = 0; i < ns; ++i) {
      mbar_init(&bars.kv_full[i], 1);
      mbar_init(&bars.kv_empty[i], 1);
    }
    mbar_init(bars.q_full, 1);
    for (int i = 0; i < kOnBufs; ++i) {
      mbar_init(&bars.s_full[i], 1);
      mbar_init(&bars.p_full[i], 256);           // the tile's map group + the anchor group
      mbar_init(&bars.s_free[i], 1);
      mbar_init(&bars.anc_ready[i], 128);
    }
    mbar_init(bars.tab_ready, kOnMapThreads);
    mbar_init(bars.o_full, 1);
    mbar_init(bars.drain, 2);
    mbar_init(bars.fin_ready, 128);
    mbar_init(bars.zx, kOnMapThreads);
    *bars.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(bars.tmem_slot, kOnTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *bars.tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (!(p.debug_flags & 1)) {
      const bool leader = elect_one();
      if (leader) {
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
        mbar_expect_tx(bars.q_full, G::TILE_BYTES);
        for (int ch = 0; ch < G::CHUNKS; ++ch)
          tma_load_3d(sQ + ch * G::CHUNK_BYTES, &tmQ, bars.q_full, ch * G::EPC, qi * 128, bh);
      }
      __syncwarp();
      int it = 0, st = 0;
      uint32_t ph = 0;
      bool ok = true;
      auto load = [&](const CUtensorMap *m, int kvt) {
        if (it >= ns) ok = ok && on_all(mbar_wait(&bars.kv_empty[st], ph ^ 1, abort));
        if (!ok) return;
        if (leader) {
          mbar_expect_tx(&bars.kv_full[st], G::TILE_BYTES);
          for (int ch = 0; ch < G::CHUNKS; ++ch)
            tma_load_3d(sKV + st * G::TILE_BYTES + ch * G::CHUNK_BYTES, m, &bars.kv_full[st],
                        ch * G::EPC, kvt * 128, bh);
        }
        __syncwarp();
        ++it;
        if (++st == ns) {
          st = 0;
          ph ^= 1;
        }
      };
      for (int j = 0; j < kOnLead && j < n && ok; ++j) load(&tmK, j);
      for (int j = 0; j < n && ok; ++j) {
        load(&tmV, j);
        if (j + kOnLead < n) load(&tmK, j + kOnLead);
      }
      // let every load issued so far land before the CTA may exit
      mbar_wait(bars.q_full, 0, abort);
      for (int s = 0; s < ns && s < it; ++s) {
        const int fills = (it - s + ns - 1) / ns;
        mbar_wait(&bars.kv_full[s], (fills - 1) & 1, abort);
      }
    }
  } else if (warp == 1 || warp == 2) {
    // ---------------------------------------------------------------- MMA
    const bool leader = elect_one();
    const uint32_t qaddr = smem_u32(sQ);
    const uint32_t kvaddr0 = smem_u32(sKV);
    int pos = 0, pst = 0;
    uint32_t pph = 0;
    bool ok = on_all(mbar_wait(bars.q_full, 0, abort));
    tc_fence_after();
    auto acquire = [&](int target) -> int {
      while (pos < target) {
        ++pos;
        if (++pst == ns) {
          pst = 0;
          pph ^= 1;
        }
      }
      ok = ok && on_all(mbar_wait(&bars.kv_full[pst], pph, abort));
      tc_fence_after();
      return pst;
    };
    auto commit = [&](uint64_t *bar) {
      if (leader) mma_commit(bar);
      __syncwarp();
    };
    const uint64_t qdesc = smem_desc(qaddr, 16, 1024);
    const uint64_t kdesc = smem_desc(kvaddr0, 16, 1024);
    const uint64_t vdesc = smem_desc(kvaddr0, G::CHUNK_BYTES, 1024);
    if (warp == 1) {
      // S_j = Q K_j^T into buffer j % 3, once PV(j - 3) has read its P
      int b = 0;
      uint32_t ph = 0;
      for (int j = 0; j < n && ok; ++j) {
        const int st = acquire(on_pos_k(j));
        if (!ok) break;
        if (j >= kOnBufs) {
          ok = on_all(mbar_wait(&bars.s_free[b], ph ^ 1, abort));
          tc_fence_after();
          if (!ok) break;
        }
        const uint64_t kd = kdesc + ((st * G::TILE_BYTES) >> 4);
#pragma unroll
        for (int kk = 0; kk < G::KSTEPS_QK; ++kk) {
          const int e = kk * G::MMA_K;
          const uint32_t off = (e / G::EPC) * G::CHUNK_BYTES + (e % G::EPC) * G::ELEM;
          if (leader) {
            if (FP8)
              mma_ss_f8(tmem + b * 128, qdesc + (off >> 4), kd + (off >> 4), G::IDESC_QK, kk > 0);
            else
              mma_ss_f16(tmem + b * 128, qdesc + (off >> 4), kd + (off >> 4), G::IDESC_QK, kk > 0);
          }
        }
        __syncwarp();
        commit(&bars.s_full[b]);
        commit(&bars.kv_empty[st]);
        if (++b == kOnBufs) { b = 0; ph ^= 1; }
      }
    } else {
      // O += P_j V_j, P_j in the first columns of buffer j % 3 (8 columns per
      // k-step)
      int b = 0;
      uint32_t ph = 0;
      for (int j = 0; j < n && ok; ++j) {
        const int st = acquire(on_pos_v(j, n));
        if (!ok) break;
        ok = on_all(mbar_wait(&bars.p_full[b], ph, abort));
        tc_fence_after();
        if (!ok) break;
        const uint64_t vd = vdesc + ((st * G::TILE_BYTES) >> 4);
#pragma unroll
        for (int kk = 0; kk < G::KSTEPS_PV; ++kk) {
          const uint64_t bd = vd + ((kk * G::MMA_K * 128) >> 4);
          const uint32_t at = tmem + b * 128 + kk * 8;
          if (leader) {
            if (FP8)
              mma_ts_f8(tmem + kOnOCol, at, bd, G::IDESC_PV, (j > 0 || kk > 0) ? 1u : 0u);
            else
              mma_ts_f16(tmem + kOnOCol, at, bd, G::IDESC_PV, (j > 0 || kk > 0) ? 1u : 0u);
          }
        }
        __syncwarp();
        commit(&bars.s_free[b]);
        commit(&bars.kv_empty[st]);
        if (++b == kOnBufs) { b = 0; ph ^= 1; }
      }
      if (ok) commit(bars.o_full);
    }
    commit(bars.drain);
    mbar_wait(bars.drain, 0, abort);
  } else if (warp >= 4 && warp < 8) {
    on_anchor<D, MAP>(p, bars, rs, threadIdx.x - 128,
                      tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16), qi, n, abort);
  } else if (warp >= 8) {
    const int g = (warp - 8) >> 2;
    on_map<D, FP8, MAP, KSAT, DBG>(p, bars, rs, g, threadIdx.x - 256 - g * 128,
                        tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16), qi, n, bh, sTab,
                        abort);
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kOnTmemCols);
  if (threadIdx.x == 0 && *bars.abort && p.status != nullptr) atomicExch(p.status, QSM_ERR_TIMEOUT);
}

constexpr int kMaxDevices = 64;

template <int D, bool FP8, int MAP, bool KSAT>
qsm_status launch_on_t(const FwdArgs &a, const CUtensorMap &mq, const CUtensorMap &mk,
                       const CUtensorMap &mv) {
  using G = OGeo<D, FP8>;
  OnParams p{};
  p.S = a.S;
  p.nqt = (a.S + 127) / 128;
  p.BH = a.B * a.H;
  p.causal = a.causal;
  p.hgroup = causal_head_group(a.S, a.D, a.fp8, a.B * a.H);
  p.K = (MAP == MAP_KI_HARD || MAP == MAP_KI_INTERP) ? a.Kint : 1;
  p.flush = a.below_policy == 1;
  p.pot_floor = a.pot_floor;
  p.c = a.c;
  p.cL2E = a.c * 1.4426950408889634f;
  p.window = a.window;
  p.v_descale = a.v_descale;
  // P scale and frame slack (log2 units): P = w * pscale * 2^(F - base) must
  // stay finite in the P format -- bf16 has fp32's range; e4m3 tops out at
  // 448.  e4m3 Rowmax-PoT keeps 64 (every weight down to 2^-15 exact) and so
  // only 2^2 of slack; e4m3 K-interval takes 16 and 2^4 (its smallest
  // fixed-window weight, e^-8 * 16, is an e4m3 subnormal with the ~6 %
  // rounding e4m3 gives every weight)
  if (MAP == MAP_POT) {
    p.pscale = FP8 ? 64.0f : 1.0f;
    p.tau = FP8 ? 2.0f : 64.0f;
  } else if (MAP == MAP_EXACT) {
    p.pscale = 1.0f;
    p.tau = 8.0f;
  } else {
    p.pscale = FP8 ? 16.0f : 1.0f;
    p.tau = FP8 ? 4.0f : 8.0f;
  }
  p.O = static_cast<__nv_bfloat16 *>(a.O);
  p.LSE = a.LSE;
  p.hi = a.row_hi;
  p.lo = a.row_lo;
  p.dbg = a.debug_idx;
  p.status = a.status_dev;
  p.debug_flags = a.debug_flags;

  const size_t table_bytes = static_cast<size_t>(table_bytes_for(MAP, p.K));
  const size_t bar_bytes = on_bar_bytes(kOnMaxStages);
  const size_t max_smem = 232448;                        // 227 KB opt-in per CTA
  const size_t fixed = 1024 + G::TILE_BYTES + table_bytes + 16 + bar_bytes + kOnRowBytes;
  int ns = static_cast<int>((max_smem - fixed) / G::TILE_BYTES);
  if (ns > kOnMaxStages) ns = kOnMaxStages;
  if (ns < 2) return QSM_ERR_UNSUPPORTED;
  p.num_stages = ns;
  p.table_off = static_cast<uint32_t>(G::TILE_BYTES + ns * G::TILE_BYTES);
  p.bar_off = static_cast<uint32_t>((p.table_off + table_bytes + 15) & ~static_cast<size_t>(15));
  p.row_off = p.bar_off + static_cast<uint32_t>(bar_bytes);
  size_t smem = 1024 + p.row_off + kOnRowBytes;
  if (smem < 120 * 1024) smem = 120 * 1024;            // one CTA per SM (all of TMEM)
  if (smem > max_smem) return QSM_ERR_UNSUPPORTED;

  // the decision dump, when asked for, runs in its own instantiation
  const int dbg = p.dbg != nullptr ? 1 : 0;
  auto kern = dbg ? qsm_fwd_online_kernel<D, FP8, MAP, KSAT, true>
                  : qsm_fwd_online_kernel<D, FP8, MAP, KSAT, false>;
  static std::atomic<int> smem_set[2][kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return QSM_ERR_CUDA;
  const bool cached = dev >= 0 && dev < kMaxDevices &&
                      smem_set[dbg][dev].load(std::memory_order_acquire) >= static_cast<int>(smem);
  if (!cached) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return QSM_ERR_CUDA;
    if (dev >= 0 && dev < kMaxDevices) {
      int prev = smem_set[dbg][dev].load(std::memory_order_relaxed);
      while (prev < static_cast<int>(smem) &&
             !smem_set[dbg][dev].compare_exchange_weak(prev, static_cast<int>(smem),
                                                       std::memory_order_acq_rel)) {
      }
    }
  }
  kern<<<dim3(p.nqt * a.B * a.H), kOnThreads, smem, a.stream>>>(mq, mk, mv, p);
  return cudaGetLastError() == cudaSuccess ? QSM_OK : QSM_ERR_CUDA;
}

template <int D, bool FP8>
qsm_status launch_on_d(const FwdArgs &a, const CUtensorMap &mq, const CUtensorMap &mk,
                       const CUtensorMap &mv) {
  if (a.mode == QSM_MODE_EXACT) return launch_on_t<D, FP8, MAP_EXACT, false>(a, mq, mk, mv);
  if (a.mode == QSM_MODE_ROWMAX_POT) return launch_on_t<D, FP8, MAP_POT, false>(a, mq, mk, mv);
  // K-interval: K a power of two takes the saturating coordinate (map_pair)
  const bool p2 = k_pow2(a.Kint);
  if (a.rounding == QSM_ROUND_HARD)
    return p2 ? launch_on_t<D, FP8, MAP_KI_HARD, true>(a, mq, mk, mv)
              : launch_on_t<D, FP8, MAP_KI_HARD, false>(a, mq, mk, mv);
  return p2 ? launch_on_t<D, FP8, MAP_KI_INTERP, true>(a, mq, mk, mv)
            : launch_on_t<D, FP8, MAP_KI_INTERP, false>(a, mq, mk, mv);
}

}  // namespace

qsm_status launch_fwd_online(const FwdArgs &a) {
  alignas(64) CUtensorMap mq, mk, mv;
  const int bh = a.B * a.H;
  if (!make_tmap_3d(&mq, a.Q, a.fp8, a.D, a.S, bh, 128) ||
      !make_tmap_3d(&mk, a.K, a.fp8, a.D, a.S, bh, 128) ||
      !make_tmap_3d(&mv, a.V, a.fp8, a.D, a.S, bh, 128))
    return QSM_ERR_CUDA;
  if (a.fp8) {
    if (a.D == 128) return launch_on_d<128, true>(a, mq, mk, mv);
    return QSM_ERR_UNSUPPORTED;
  }
  if (a.D == 128) return launch_on_d<128, false>(a, mq, mk, mv);
  if (a.D == 64) return launch_on_d<64, false>(a, mq, mk, mv);
  return QSM_ERR_UNSUPPORTED;
}

}  // namespace qsm
