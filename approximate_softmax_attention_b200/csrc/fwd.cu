// fwd.cu -- fused approximate-softmax attention forward for sm_100a.
//
// One CTA owns two 128-row query tiles of one (b, h) and sweeps the key/value
// tiles of 128 rows ("QK tile -> row max -> power-of-two weights -> PV matmul
// -> output", the tile loop of "Approximating Softmax in Pretrained LLMs",
// wiki flowchart).  Roles (12 warps):
//   warp 0      TMA producer: Q tiles once, then K (statistics sweep) and
//               K, V (main sweep) through a ring of shared-memory stages.
//   warp 1      MMA issuer (one thread): S = Q K^T into TMEM (tcgen05, both
//               operands in shared memory) and O += P V with P read from TMEM.
//   warps 4-7   map group for query tile 0, one thread per row (TMEM lane).
//   warps 8-11  map group for query tile 1.
// TMEM (512 columns): S0 at 0, S1 at 128, O0 at 256, O1 at 384.  P (bf16 or
// e4m3, packed) overwrites the S columns it was computed from.  During the
// statistics sweep the O columns double as second S buffers.
//
// Approximate maps are defined against the row's final maximum (and minimum),
// so they run a statistics sweep first (S tiles, max/min/argmax/argmin only,
// no PV), then the main sweep with the row constants fixed.  The exact map
// needs no such sweep: it rescales online, and rescales O only when the
// running maximum grew by more than 2^8 in weight.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "internal.h"
#include "sm100.cuh"
#include "wmap.cuh"

namespace qsm {

enum MapKind { MAP_EXACT = 0, MAP_POT = 1, MAP_KI_HARD = 2, MAP_KI_INTERP = 3 };

struct FwdParams {
  int S, nqt, nqb, BH;
  int causal;
  int K;
  int fixed_window;
  int flush;        // below_policy == 1
  int pot_floor;
  float c;          // score scale
  float cL2E;       // c * log2(e), exact map
  float window;
  float v_descale;
  float pscale;     // P is stored as w * pscale (FP8 approximate maps: 64)
  int tab_stride;   // floats of grid table per query tile
  int num_stages;
  uint32_t table_off, bar_off, xch_off;
  __nv_bfloat16 *O;
  float *LSE, *hi, *lo;
  int32_t *amax, *amin;
  int8_t *dbg;
  int32_t *status;
  int debug_flags;
};

template <int D, bool FP8>
struct Geo {
  static constexpr int BM = 128, BN = 128;
  static constexpr int ELEM = FP8 ? 1 : 2;
  static constexpr int EPC = 128 / ELEM;                // elements per 128-byte swizzle row
  static constexpr int CHUNKS = (D * ELEM) / 128;       // swizzle columns per tile
  static constexpr int CHUNK_BYTES = 128 * 128;         // 128 rows x 128 bytes
  static constexpr int TILE_BYTES = BM * D * ELEM;
  static constexpr int MMA_K = FP8 ? 32 : 16;           // K of one MMA instruction
  static constexpr int KSTEPS_QK = D / MMA_K;
  static constexpr int KSTEPS_PV = BN / MMA_K;
  static constexpr uint32_t FMT = FP8 ? 0u : 1u;        // e4m3 / bf16 format code
  static constexpr uint32_t IDESC_QK = instr_desc(FMT, false, 128, BN);
  static constexpr uint32_t IDESC_PV = instr_desc(FMT, true, 128, D);
  static constexpr int P_COLS_PER_CHUNK = FP8 ? 8 : 16; // TMEM columns per 32 P values
};

constexpr int kThreads = 640;      // 4 control warps + 4 map warp groups
constexpr int kLaunchRegs = 96;    // 65536 / 640 rounded down to a multiple of 8
// Register split (see the kernel): with sixteen map warps every warp keeps
// the launch allocation of 96 (no reallocation).
template <int MAP>
struct RegSplit {
  static constexpr int ctrl = 96;
  static constexpr int map = 96;
};
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleLog2 = 8.0f;

// barrier slots (uint64 each) after the stage barriers
struct Bars {
  uint64_t *kv_full, *kv_empty;   // [stages]
  uint64_t *q_full;               // 1
  uint64_t *s_full;               // [2 tiles][2 buffers]
  uint64_t *s_empty;              // [2][2]
  uint64_t *p_full;               // [2]
  uint64_t *o_full;               // [2]
  uint64_t *drain;                // 1
  uint64_t *xstat, *xtile, *xz;   // [2 tiles] each: the halves' exchanges
  uint32_t *tmem_slot;
  int *abort;
};

__device__ __forceinline__ Bars carve_bars(uint8_t *base, int ns) {
  Bars b;
  uint64_t *p = reinterpret_cast<uint64_t *>(base);
  b.kv_full = p;
  b.kv_empty = p + ns;
  b.q_full = p + 2 * ns;
  b.s_full = b.q_full + 1;
  b.s_empty = b.s_full + 4;
  b.p_full = b.s_empty + 4;
  b.o_full = b.p_full + 2;
  b.drain = b.o_full + 2;
  b.xstat = b.drain + 1;
  b.xtile = b.xstat + 2;
  b.xz = b.xtile + 2;
  b.tmem_slot = reinterpret_cast<uint32_t *>(b.xz + 2);
  b.abort = reinterpret_cast<int *>(b.tmem_slot + 1);
  return b;
}

// Per-row constants of the fused map, with the score scale folded in: the
// map consumes the raw fp32 accumulator r = q.k of the MMA.
//   PoT:        x = fma(r, -c*log2e, hi*log2e), w = 2^-rne(min(x, cap)) * pscale
//   K-interval: u = fma(r, c*K/(hi-lo), -lo*K/(hi-lo)); hard: g[rne(u)];
//               interpolation: u d_k + c_k at k = floor(u) (grid values
//               pre-multiplied by pscale).  Same decisions as the library's
//               fp32 map up to the rounding of the folded scale.
struct MapRow {
  float a, b;        // coordinate = fma(r, a, b)
  float cap, Kf, Km1;
  uint32_t tab;      // shared address bias of this row's table column
  uint32_t pow_bias; // bits of pscale (PoT)
};

template <int MAP>
__device__ __forceinline__ float map_raw(float r, const MapRow &m) {
  if (MAP == MAP_POT) {
    const float x = __fmaf_rn(r, m.a, m.b);
    const float t = __fadd_rn(fminf(x, m.cap), kMagic);
    // 2^-n * pscale from the exponent field: bits(t) = kMagicBits + n and
    // kMagicBits << 23 == 0 (mod 2^32), so -(bits(t) << 23) == -(n << 23)
    return __uint_as_float(__float_as_uint(t) * 0xFF800000u + m.pow_bias);
  } else if (MAP == MAP_KI_HARD) {
    // the clamp to [0, K] bounds the table index for every input (masked
    // keys, ragged rows, near-degenerate rows, inf and NaN included)
    const float u = fminf(fmaxf(__fmaf_rn(r, m.a, m.b), 0.0f), m.Kf);
    const uint32_t tb = __float_as_uint(__fadd_rn(u, kMagic));
    return lds_f32(tb * 512u + m.tab);
  } else {
    // interpolation as one FMA: w = g_k + (u - k) d_k = u d_k + c_k with
    // c_k = g_k - k d_k; k = floor(u) in [0, K] (the clamp bounds the index)
    // through a round-down add of 2^23; the table entry at k = K repeats
    // k = K - 1, which is the interpolation's value at u = K
    const float u = fminf(fmaxf(__fmaf_rn(r, m.a, m.b), 0.0f), m.Kf);
    const uint32_t tb = __float_as_uint(__fadd_rd(u, 8388608.0f));
    const float2 cd = lds_f32x2(tb * 1024u + m.tab);
    return __fmaf_rn(u, cd.y, cd.x);
  }
}

// Decision index of one element (debug dump only; same arithmetic).
template <int MAP>
__device__ __forceinline__ int map_raw_index(float r, const MapRow &m, bool flush, int N) {
  if (MAP == MAP_EXACT) return 0;
  const float x = __fmaf_rn(r, m.a, m.b);
  if (MAP == MAP_POT) {
    const int n = static_cast<int>(__float_as_uint(__fadd_rn(fminf(x, m.cap), kMagic)) -
                                   kMagicBits);
    return (flush && n > N) ? -2 : n;
  }
  const float uc = fminf(fmaxf(x, 0.0f), m.Kf);
  if (MAP == MAP_KI_HARD)
    return static_cast<int>(__float_as_uint(__fadd_rn(uc, kMagic)) - kMagicBits);
  const float kf = fminf(__fsub_rn(__fadd_rd(uc, 8388608.0f), 8388608.0f), m.Km1);
  return static_cast<int>(kf);
}

// Weights of one 32-column chunk, packed for the PV MMA and stored to TMEM;
// FULL: every column valid.
template <int MAP, bool FULL, bool FP8>
__device__ __forceinline__ void map_chunk(const uint32_t (&v)[32], const MapRow &m, int c0,
                                          int lim, bool flush_below, float (&z)[8],
                                          uint32_t taddr_pc) {
  auto wt = [&](int i) {
    const float r = __uint_as_float(v[i]);
    float wi = map_raw<MAP>(r, m);
    if (MAP == MAP_KI_HARD || MAP == MAP_KI_INTERP) {
      // fixed-window flush: coordinate below the window
      if (flush_below && __fmaf_rn(r, m.a, m.b) < 0.0f) wi = 0.0f;
    }
    if (!FULL) wi = (c0 + i < lim) ? wi : 0.0f;
    z[i & 7] += wi;
    return wi;
  };
  if (FP8) {
    uint32_t pk[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float a = wt(4 * i), b = wt(4 * i + 1), c = wt(4 * i + 2), d = wt(4 * i + 3);
      pk[i] = pack_e4m3x4(a, b, c, d);
    }
    tmem_st8(taddr_pc, pk);
  } else {
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float a = wt(2 * i), b = wt(2 * i + 1);
      pk[i] = pack_bf16x2(a, b);
    }
    tmem_st16(taddr_pc, pk);
  }
}

// Decision dump of one chunk (debug option).
template <int MAP>
__device__ __forceinline__ void debug_chunk(int8_t *dbg_row, const uint32_t (&v)[32],
                                            const MapRow &m, int kv0, int c0, int lim,
                                            const FwdParams &p, bool flush_below) {
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    if (dbg_row != nullptr && kv0 + i < p.S) {
      const float r = __uint_as_float(v[i]);
      int n = map_raw_index<MAP>(r, m, p.flush != 0, p.pot_floor);
      if (flush_below && __fmaf_rn(r, m.a, m.b) < 0.0f) n = -2;
      dbg_row[kv0 + i] = static_cast<int8_t>((c0 + i < lim) ? n : -1);
    }
  }
}

// Every tcgen05.ld / tcgen05.st below is .sync.aligned: the 32 lanes of a
// warp must reach it together.  Branches around them therefore depend only on
// warp-uniform values (tile-level flags, votes), never on a row's own data.
// Key tile j is valid in every column for every row of query tile qi (a
// tile-level fact, so the same for all 128 threads of the group).
__device__ __forceinline__ bool full_tile(const FwdParams &p, int qi, int j) {
  return 128 * (j + 1) <= p.S && (!p.causal || j < qi);
}

__device__ __forceinline__ bool warp_all(bool x) { return __all_sync(0xffffffffu, x); }
__device__ __forceinline__ bool warp_any(bool x) { return __any_sync(0xffffffffu, x); }

// Per-row values the two halves of a query tile exchange through shared
// memory (see map_half).
struct Xch {
  float4 *stats;      // [2 tiles][2 halves][128]: max, min, argmax, argmin
  float *tilemax;     // [2 tiles][2 slots][2 halves][128]  (exact map)
  float *zsum;        // [2 tiles][2 halves][128]
};

// One map warp group: 128 threads own half h (64 of the 128 key columns) of
// every S tile of query tile t; thread `row` owns query row qi*128+row (TMEM
// lane `row`).  The group that owns the other half shares the row: the two
// combine row statistics, the exact map's tile maxima and the row sums
// through shared memory behind bounded-wait barriers.  P of half h goes to
// TMEM columns 64h.. of the tile's S buffer, which only this group reads.
template <int D, bool FP8, int MAP>
__device__ __forceinline__ void map_half(const FwdParams &p, const Bars &bars, int t, int h,
                                         int row, uint32_t lane_base, int qi, int n_t, int bh,
                                         float *tab, const Xch &xc, volatile int *abort) {
  constexpr bool kTwoPass = MAP != MAP_EXACT;
  constexpr int PCOLS = FP8 ? 8 : 16;                  // TMEM columns per 32 P values
  const int qrow = qi * 128 + row;
  const bool row_ok = qrow < p.S;
  const int L = p.causal ? min(qrow + 1, p.S) : p.S;   // valid keys of the row
  if (n_t <= 0) return;
  const int c_off = 64 * h;                            // first key column of this half
  uint32_t sf_cnt0 = 0, sf_cnt1 = 0;
  bool ok = true;
  float rmax = -INFINITY, rmin = INFINITY;
  int amax = 0, amin = 0;
  const bool want_arg = p.amax != nullptr || p.amin != nullptr;
  const bool want_min =
      ((MAP == MAP_KI_HARD || MAP == MAP_KI_INTERP) && !p.fixed_window) || p.lo != nullptr;

  // -------------------------------------------------- statistics sweep
  if (kTwoPass) {
    float mx[8], mn[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) { mx[i] = -INFINITY; mn[i] = INFINITY; }
    for (int j = 0; j < n_t && ok; ++j) {
      const int b = j & 1;
      ok = warp_all(mbar_wait(&bars.s_full[t * 2 + b], (b ? sf_cnt1 : sf_cnt0) & 1, abort));
      if (b) ++sf_cnt1; else ++sf_cnt0;
      if (!ok) break;
      tc_fence_after();
      const int lim = L - 128 * j - c_off;             // valid columns of this half
      const bool full = full_tile(p, qi, j);
      const uint32_t base = lane_base + t * 128 + b * 256 + c_off;
      if (want_arg) {
        auto scan = [&](const uint32_t(&cur)[32], int c0) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float x = __uint_as_float(cur[i]);
            const bool valid = c0 + i < lim;
            const int col = 128 * j + c_off + c0 + i;
            if (valid && x > rmax) { rmax = x; amax = col; }
            if (valid && x < rmin) { rmin = x; amin = col; }
          }
        };
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
          uint32_t v[32];
          tmem_ld32_sync(base + 32 * c, v);
          scan(v, 32 * c);
        }
      } else {
        auto reduce = [&](const uint32_t(&cur)[32], int c0) {
          if (full) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const float x = __uint_as_float(cur[i]);
              mx[i & 7] = fmaxf(mx[i & 7], x);
              if (want_min) mn[i & 7] = fminf(mn[i & 7], x);
            }
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const float x = __uint_as_float(cur[i]);
              const bool valid = c0 + i < lim;
              mx[i & 7] = fmaxf(mx[i & 7], valid ? x : -INFINITY);
              if (want_min) mn[i & 7] = fminf(mn[i & 7], valid ? x : INFINITY);
            }
          }
        };
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
          uint32_t v[32];
          tmem_ld32_sync(base + 32 * c, v);
          reduce(v, 32 * c);
        }
      }
      tc_fence_before();
      mbar_arrive(&bars.s_empty[t * 2 + b]);
    }
    if (!want_arg) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        rmax = fmaxf(rmax, mx[i]);
        rmin = fminf(rmin, mn[i]);
      }
    }
    // combine the two halves (ties: the lower key index)
    if (ok) {
      xc.stats[(t * 2 + h) * 128 + row] =
          make_float4(rmax, rmin, __int_as_float(amax), __int_as_float(amin));
      mbar_arrive(&bars.xstat[t]);
      ok = warp_all(mbar_wait(&bars.xstat[t], 0, abort));
    }
    if (ok) {
      const float4 o = xc.stats[(t * 2 + (h ^ 1)) * 128 + row];
      const int oamax = __float_as_int(o.z), oamin = __float_as_int(o.w);
      if (o.x > rmax || (o.x == rmax && oamax < amax)) { rmax = o.x; amax = oamax; }
      if (o.y < rmin || (o.y == rmin && oamin < amin)) { rmin = o.y; amin = oamin; }
    }
  }

  // ------------------------------------------------------ main sweep
  float z[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) z[i] = 0.0f;
  float hi = 0.0f, lo = 0.0f;
  float m_used = -INFINITY, m_run = -INFINITY;      // exact map, raw units
  MapRow mr;
  mr.a = mr.b = 0.0f;
  mr.cap = static_cast<float>(p.flush ? p.pot_floor + 1 : p.pot_floor);
  mr.Kf = static_cast<float>(p.K);
  mr.Km1 = static_cast<float>(p.K - 1);
  mr.tab = 0;
  mr.pow_bias = __float_as_uint(p.pscale);
  const bool flush_below = (MAP == MAP_KI_HARD || MAP == MAP_KI_INTERP) && p.flush &&
                           p.fixed_window;
  if (kTwoPass && ok) {
    hi = __fmul_rn(p.c, rmax);
    lo = __fmul_rn(p.c, rmin);
    RowMap rm = make_rowmap(hi, lo, p.K, p.fixed_window != 0, p.window);
    if (MAP == MAP_POT) {
      mr.a = -p.cL2E;
      mr.b = rm.hiL2E;
    } else {
      mr.a = __fmul_rn(p.c, rm.inv);
      mr.b = rm.b;
      if (rm.degenerate) {           // every key sits at the top node
        mr.a = 0.0f;
        mr.b = mr.Kf;
      }
      lo = rm.lo;
      const uint32_t tb = smem_u32(tab);
      // the two halves build alternate entries of this row's grid table
      if (MAP == MAP_KI_HARD) {
        for (int n = h; n <= p.K; n += 2) tab[n * 128 + row] = grid_value(rm, p.K, n) * p.pscale;
        mr.tab = tb + row * 4 - kMagicBits * 512u;
      } else {
        // entries k = 0 .. K: (c_k, d_k) with d_k = g_{k+1} - g_k and
        // c_k = g_k - k d_k; entry K repeats entry K - 1
        for (int n = h; n <= p.K; n += 2) {
          const int k = n < p.K ? n : p.K - 1;
          const float gk = grid_value(rm, p.K, k);
          const float gk1 = grid_value(rm, p.K, k + 1);
          const float d = __fsub_rn(gk1, gk) * p.pscale;
          tab[(n * 128 + row) * 2 + 0] = __fmaf_rn(-static_cast<float>(k), d, gk * p.pscale);
          tab[(n * 128 + row) * 2 + 1] = d;
        }
        // floor bits: bits(2^23 + k) = 0x4B000000 + k  ->  table row k
        mr.tab = tb + row * 8 - 0x4B000000u * 1024u;
      }
      // the table is complete before either half reads it
      mbar_arrive(&bars.xstat[t]);
      ok = warp_all(mbar_wait(&bars.xstat[t], 1, abort));
    }
  }
  int8_t *dbg_row = (p.dbg != nullptr && row_ok)
                        ? p.dbg + (static_cast<size_t>(bh) * p.S + qrow) * p.S
                        : nullptr;
  const uint32_t pbase = lane_base + t * 128 + c_off;       // P columns of this half

  for (int j = 0; j < n_t && ok; ++j) {
    ok = warp_all(mbar_wait(&bars.s_full[t * 2 + 0], sf_cnt0 & 1, abort));
    ++sf_cnt0;
    if (!ok) break;
    tc_fence_after();
    const int lim = L - 128 * j - c_off;
    const bool full = full_tile(p, qi, j);
    const uint32_t sbase = lane_base + t * 128 + c_off;
    if (MAP == MAP_EXACT) {
      float mx[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mx[i] = -INFINITY;
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        uint32_t v[32];
        tmem_ld32_sync(sbase + 32 * c, v);
#pragma unroll
        for (int i = 0; i < 32; ++i)
          mx[i & 7] = fmaxf(mx[i & 7], (full || 32 * c + i < lim) ? __uint_as_float(v[i]) : -INFINITY);
      }
      float mt = mx[0];
#pragma unroll
      for (int i = 1; i < 8; ++i) mt = fmaxf(mt, mx[i]);
      // the tile maximum of the whole row
      float *slot = xc.tilemax + ((t * 2 + (j & 1)) * 2) * 128;
      slot[h * 128 + row] = mt;
      mbar_arrive(&bars.xtile[t]);
      ok = warp_all(mbar_wait(&bars.xtile[t], j & 1, abort));
      if (!ok) break;
      mt = fmaxf(mt, slot[(h ^ 1) * 128 + row]);
      m_run = fmaxf(m_run, mt);
      // move this row's anchor on its first tile, or when the running max grew
      // by more than 2^8 in weight; O is rescaled in TMEM when any row of the
      // warp moved (rows that did not move use alpha = 1).  Both halves take
      // the same decisions (same rows, same combined maxima).
      const bool first = m_used == -INFINITY;
      const bool move = first || (m_run - m_used) * p.cL2E > kRescaleLog2;
      const float alpha = (move && !first) ? ex2_approx((m_used - m_run) * p.cL2E) : 1.0f;
      if (move) m_used = m_run;
#pragma unroll
      for (int i = 0; i < 8; ++i) z[i] *= alpha;
      if (j > 0 && warp_any(move)) {
        const uint32_t obase = lane_base + 256 + t * 128 + h * (D / 2);
#pragma unroll 1
        for (int dc = 0; dc < D / 64; ++dc) {
          uint32_t v[32];
          tmem_ld32_sync(obase + 32 * dc, v);
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * alpha);
          tmem_st32(obase + 32 * dc, v);
        }
      }
      const float mb = m_used * p.cL2E;
      auto ex = [&](const uint32_t(&cur)[32], int c0, uint32_t taddr) {
        auto e = [&](int i) {
          const float w = ex2_approx(__fmaf_rn(__uint_as_float(cur[i]), p.cL2E, -mb));
          const float wi = (full || c0 + i < lim) ? w : 0.0f;
          z[i & 7] += wi;
          return wi;
        };
        if (FP8) {
          uint32_t pk[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float a = e(4 * i), b = e(4 * i + 1), c = e(4 * i + 2), d = e(4 * i + 3);
            pk[i] = pack_e4m3x4(a, b, c, d);
          }
          tmem_st8(taddr, pk);
        } else {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float a = e(2 * i), b = e(2 * i + 1);
            pk[i] = pack_bf16x2(a, b);
          }
          tmem_st16(taddr, pk);
        }
      };
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        uint32_t v[32];
        tmem_ld32_sync(sbase + 32 * c, v);
        ex(v, 32 * c, pbase + c * PCOLS);
      }
      if (dbg_row != nullptr) {
        for (int i = 0; i < 64; ++i) {
          const int kv = 128 * j + c_off + i;
          if (kv < p.S) dbg_row[kv] = (i < lim) ? 0 : -1;
        }
      }
    } else {
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        uint32_t v[32];
        tmem_ld32_sync(sbase + 32 * c, v);
        if (full)
          map_chunk<MAP, true, FP8>(v, mr, 32 * c, lim, flush_below, z, pbase + c * PCOLS);
        else
          map_chunk<MAP, false, FP8>(v, mr, 32 * c, lim, flush_below, z, pbase + c * PCOLS);
        if (p.dbg != nullptr)
          debug_chunk<MAP>(dbg_row, v, mr, 128 * j + c_off + 32 * c, 32 * c, lim, p,
                           flush_below);
      }
    }
    tmem_wait_st();
    tc_fence_before();
    mbar_arrive(&bars.p_full[t]);
  }

  // ---------------------------------------------------------- epilogue
  if (ok) ok = warp_all(mbar_wait(&bars.o_full[t], 0, abort));
  if (!ok) return;
  tc_fence_after();
  float Z = ((z[0] + z[1]) + (z[2] + z[3])) + ((z[4] + z[5]) + (z[6] + z[7]));
  xc.zsum[(t * 2 + h) * 128 + row] = Z;
  mbar_arrive(&bars.xz[t]);
  if (!warp_all(mbar_wait(&bars.xz[t], 0, abort))) return;
  Z += xc.zsum[(t * 2 + (h ^ 1)) * 128 + row];
  if (MAP == MAP_EXACT) hi = p.c * m_run;
  const float oscale = p.v_descale / Z;          // pscale cancels: P and Z both carry it
  const uint32_t obase = lane_base + 256 + t * 128 + h * (D / 2);
  __nv_bfloat16 *orow = p.O + (static_cast<size_t>(bh) * p.S + qrow) * D + h * (D / 2);
#pragma unroll 1
  for (int dc = 0; dc < D / 64; ++dc) {
    uint32_t v[32];
    tmem_ld32_sync(obase + 32 * dc, v);
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 16; ++i)
      pk[i] = pack_bf16x2(__uint_as_float(v[2 * i]) * oscale,
                          __uint_as_float(v[2 * i + 1]) * oscale);
    if (row_ok) {
      uint4 *dst = reinterpret_cast<uint4 *>(orow + 32 * dc);
#pragma unroll
      for (int i = 0; i < 4; ++i)
        dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
    }
  }
  if (row_ok && h == 0) {
    const size_t ri = static_cast<size_t>(bh) * p.S + qrow;
    const float anchor = (MAP == MAP_EXACT) ? p.c * m_used : hi;
    p.LSE[ri] = anchor + logf(Z / p.pscale);
    if (p.hi) p.hi[ri] = hi;
    if (MAP != MAP_EXACT) {          // the exact map runs no statistics sweep
      if (p.lo) p.lo[ri] = lo;
      if (p.amax) p.amax[ri] = amax;
      if (p.amin) p.amin[ri] = amin;
    }
  }
}

template <int D, bool FP8, int MAP>
__global__ void __launch_bounds__(kThreads, 1)
    qsm_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  using G = Geo<D, FP8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Work order: non-causal CTAs sweep one head's query blocks after another
  // (the running CTAs share few heads' K/V in L2); causal CTAs go heaviest
  // first over all heads (longest-processing-time order, so the lightest
  // blocks form the tail).
  int bh, qb;
  if (p.causal) {
    const int rank = static_cast<int>(blockIdx.x) / p.BH;
    bh = static_cast<int>(blockIdx.x) - rank * p.BH;
    qb = p.nqb - 1 - rank;
  } else {
    qb = static_cast<int>(blockIdx.x) % p.nqb;
    bh = static_cast<int>(blockIdx.x) / p.nqb;
  }
  const int ns = p.num_stages;

  uint8_t *sQ = smem;                                   // 2 tiles
  uint8_t *sKV = smem + 2 * G::TILE_BYTES;              // ns stages
  float *sTab = reinterpret_cast<float *>(smem + p.table_off);
  Bars bars = carve_bars(smem + p.bar_off, ns);
  Xch xc;
  xc.stats = reinterpret_cast<float4 *>(smem + p.xch_off);
  xc.tilemax = reinterpret_cast<float *>(smem + p.xch_off + 4 * 128 * 16);
  xc.zsum = xc.tilemax + 8 * 128;
  volatile int *abort = bars.abort;

  const int nkvt = (p.S + 127) / 128;
  // per query tile: index and number of key tiles (scalars, so the control
  // loops never index a local array)
  const int qi0 = 2 * qb, qi1 = 2 * qb + 1;
  const int nt0 = p.causal ? min(nkvt, qi0 + 1) : nkvt;
  const int nt1 = qi1 < p.nqt ? (p.causal ? min(nkvt, qi1 + 1) : nkvt) : 0;
  auto NT = [&](int t) { return t ? nt1 : nt0; };
  auto QI = [&](int t) { return t ? qi1 : qi0; };
  const int nkv = max(nt0, nt1);
  constexpr bool kTwoPass = MAP != MAP_EXACT;

  if (threadIdx.x == 0) {
    for (int i = 0; i < ns; ++i) {
      mbar_init(&bars.kv_full[i], 1);
      mbar_init(&bars.kv_empty[i], 1);
    }
    mbar_init(bars.q_full, 1);
    for (int i = 0; i < 4; ++i) {
      mbar_init(&bars.s_full[i], 1);
      mbar_init(&bars.s_empty[i], 256);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.p_full[i], 256);
      mbar_init(&bars.o_full[i], 1);
      mbar_init(&bars.xstat[i], 256);
      mbar_init(&bars.xtile[i], 256);
      mbar_init(&bars.xz[i], 256);
    }
    mbar_init(bars.drain, 1);
    *bars.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(bars.tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *bars.tmem_slot;

  // The CTA launches with kThreads x kLaunchRegs registers; the control warp
  // group (producer, MMA issuer, two idle warps) gives most of its share to
  // the four map groups: 128 x kCtrlRegs + 512 x kMapRegs <= 640 x kLaunchRegs
  // (an increase beyond what the decrease freed would wait forever).
  constexpr int kCtrlRegs = RegSplit<MAP>::ctrl;
  constexpr int kMapRegs = RegSplit<MAP>::map;
  static_assert(128 * kCtrlRegs + 512 * kMapRegs <= kThreads * kLaunchRegs,
                "register split must equal the launch allocation");
  if (warp < 4) {
    if (kCtrlRegs < kLaunchRegs) regs_dec<kCtrlRegs>();
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && !(p.debug_flags & 1)) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      const int nq = (nt0 > 0) + (nt1 > 0);
      mbar_expect_tx(bars.q_full, nq * G::TILE_BYTES);
      for (int t = 0; t < 2; ++t)
        if (NT(t) > 0)
          for (int ch = 0; ch < G::CHUNKS; ++ch)
            tma_load_3d(sQ + t * G::TILE_BYTES + ch * G::CHUNK_BYTES, &tmQ, bars.q_full,
                        ch * G::EPC, QI(t) * 128, bh);
      int it = 0, st = 0;
      uint32_t ph = 0;                  // completed passes over the ring
      bool ok = true;
      auto load = [&](const CUtensorMap *m, int kvt) {
        if (it >= ns) ok = ok && mbar_wait(&bars.kv_empty[st], ph ^ 1, abort);
        if (!ok) return;
        mbar_expect_tx(&bars.kv_full[st], G::TILE_BYTES);
        for (int ch = 0; ch < G::CHUNKS; ++ch)
          tma_load_3d(sKV + st * G::TILE_BYTES + ch * G::CHUNK_BYTES, m, &bars.kv_full[st],
                      ch * G::EPC, kvt * 128, bh);
        ++it;
        if (++st == ns) {
          st = 0;
          ph ^= 1;
        }
      };
      if (kTwoPass)
        for (int j = 0; j < nkv && ok; ++j) load(&tmK, j);
      for (int j = 0; j < nkv && ok; ++j) {
        load(&tmK, j);
        load(&tmV, j);
      }
      // let every load issued so far land before the CTA may exit
      mbar_wait(bars.q_full, 0, abort);
      for (int s = 0; s < ns && s < it; ++s) {
        const int fills = (it - s + ns - 1) / ns;  // loads issued into stage s
        mbar_wait(&bars.kv_full[s], (fills - 1) & 1, abort);
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    if (lane == 0) {
      const uint32_t qaddr0 = smem_u32(sQ);
      const uint32_t kvaddr0 = smem_u32(sKV);
      int cst = 0;                      // next ring stage to consume
      uint32_t cph = 0;                 // its phase parity
      bool ok = mbar_wait(bars.q_full, 0, abort);
      tc_fence_after();
      auto acquire = [&]() -> int {
        const int st = cst;
        ok = ok && mbar_wait(&bars.kv_full[st], cph, abort);
        if (++cst == ns) {
          cst = 0;
          cph ^= 1;
        }
        tc_fence_after();
        return st;
      };
      auto issue_qk = [&](int t, int st, uint32_t scol) {
        const uint32_t qa = qaddr0 + t * G::TILE_BYTES;
        const uint32_t ka = kvaddr0 + st * G::TILE_BYTES;
#pragma unroll
        for (int kk = 0; kk < G::KSTEPS_QK; ++kk) {
          const int e = kk * G::MMA_K;
          const uint32_t off = (e / G::EPC) * G::CHUNK_BYTES + (e % G::EPC) * G::ELEM;
          const uint64_t ad = smem_desc(qa + off, 16, 1024);
          const uint64_t bd = smem_desc(ka + off, 16, 1024);
          if (FP8)
            mma_ss_f8(tmem + scol, ad, bd, G::IDESC_QK, kk > 0);
          else
            mma_ss_f16(tmem + scol, ad, bd, G::IDESC_QK, kk > 0);
        }
      };
      auto issue_pv = [&](int t, int st, bool acc) {
        const uint32_t va = kvaddr0 + st * G::TILE_BYTES;
        const uint32_t pcol = t * 128;
        const uint32_t ocol = 256 + t * 128;
#pragma unroll
        for (int kk = 0; kk < G::KSTEPS_PV; ++kk) {
          const uint64_t bd = smem_desc(va + kk * G::MMA_K * 128, G::CHUNK_BYTES, 1024);
          // keys 64h.. of the tile sit at TMEM columns 64h.. (each map half
          // writes its P into its own S columns), 8 columns per k-step
          const int key0 = kk * G::MMA_K;
          const uint32_t at = tmem + pcol + 64 * (key0 / 64) + ((key0 % 64) / G::MMA_K) * 8;
          if (FP8)
            mma_ts_f8(tmem + ocol, at, bd, G::IDESC_PV, (acc || kk > 0) ? 1u : 0u);
          else
            mma_ts_f16(tmem + ocol, at, bd, G::IDESC_PV, (acc || kk > 0) ? 1u : 0u);
        }
      };

      if (kTwoPass) {
        for (int j = 0; j < nkv && ok; ++j) {
          const int st = acquire();
          if (!ok) break;
          for (int t = 0; t < 2 && ok; ++t) {
            if (j >= NT(t)) continue;
            const int b = j & 1, use = j >> 1;
            if (use >= 1) {
              ok = mbar_wait(&bars.s_empty[t * 2 + b], (use - 1) & 1, abort);
              tc_fence_after();
              if (!ok) break;
            }
            issue_qk(t, st, t * 128 + b * 256);
            mma_commit(&bars.s_full[t * 2 + b]);
          }
          mma_commit(&bars.kv_empty[st]);
        }
        // both S buffers of each tile must be read out before the main sweep
        for (int t = 0; t < 2 && ok; ++t) {
          const int u0 = (NT(t) + 1) / 2, u1 = NT(t) / 2;
          if (u0 >= 1) ok = ok && mbar_wait(&bars.s_empty[t * 2 + 0], (u0 - 1) & 1, abort);
          if (u1 >= 1) ok = ok && mbar_wait(&bars.s_empty[t * 2 + 1], (u1 - 1) & 1, abort);
        }
        tc_fence_after();
      }
      if (ok && nkv > 0) {
        const int k0 = acquire();
        if (ok) {
          for (int t = 0; t < 2; ++t)
            if (NT(t) > 0) {
              issue_qk(t, k0, t * 128);
              mma_commit(&bars.s_full[t * 2 + 0]);
            }
          mma_commit(&bars.kv_empty[k0]);
        }
        for (int j = 0; j < nkv && ok; ++j) {
          const int vst = acquire();
          const bool has_next = j + 1 < nkv;
          const int knext = has_next ? acquire() : -1;
          if (!ok) break;
          for (int t = 0; t < 2 && ok; ++t) {
            if (j < NT(t)) {
              ok = mbar_wait(&bars.p_full[t], j & 1, abort);
              tc_fence_after();
              if (!ok) break;
              issue_pv(t, vst, j > 0);
            }
            if (has_next && j + 1 < NT(t)) {
              issue_qk(t, knext, t * 128);
              mma_commit(&bars.s_full[t * 2 + 0]);
            }
          }
          mma_commit(&bars.kv_empty[vst]);
          if (has_next) mma_commit(&bars.kv_empty[knext]);
        }
        for (int t = 0; t < 2; ++t)
          if (NT(t) > 0) mma_commit(&bars.o_full[t]);
      }
      // every MMA issued must finish before TMEM is released
      mma_commit(bars.drain);
      mbar_wait(bars.drain, 0, abort);
    }
  }
  } else {
    if (kMapRegs > kLaunchRegs) regs_inc<kMapRegs>();
    const int g = (warp - 4) >> 2;                 // map group 0..3
    const int t = g >> 1, h = g & 1;               // query tile, key-column half
    map_half<D, FP8, MAP>(p, bars, t, h, threadIdx.x - 128 - g * 128,
                          tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16), QI(t), NT(t),
                          bh, sTab + t * p.tab_stride, xc, abort);
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
  if (threadIdx.x == 0 && *bars.abort && p.status != nullptr) atomicExch(p.status, QSM_ERR_TIMEOUT);
}

// ------------------------------------------------------------------- host

template <int D, bool FP8, int MAP>
static qsm_status launch_t(const FwdArgs &a, const CUtensorMap &mq, const CUtensorMap &mk,
                           const CUtensorMap &mv) {
  using G = Geo<D, FP8>;
  FwdParams p{};
  p.S = a.S;
  p.nqt = (a.S + 127) / 128;
  p.nqb = (p.nqt + 1) / 2;
  p.BH = a.B * a.H;
  p.causal = a.causal;
  p.K = (MAP == MAP_KI_HARD || MAP == MAP_KI_INTERP) ? a.Kint : 1;
  p.fixed_window = a.calib == QSM_CALIB_FIXED_WINDOW;
  p.flush = a.below_policy == 1;
  p.pot_floor = a.pot_floor;
  p.c = a.c;
  p.cL2E = a.c * 1.4426950408889634f;
  p.window = a.window;
  p.pscale = (FP8 && MAP != MAP_EXACT) ? 64.0f : 1.0f;
  p.v_descale = a.v_descale;
  p.O = static_cast<__nv_bfloat16 *>(a.O);
  p.LSE = a.LSE;
  p.hi = a.row_hi;
  p.lo = a.row_lo;
  p.amax = a.row_argmax;
  p.amin = a.row_argmin;
  p.dbg = a.debug_idx;
  p.status = a.status_dev;
  p.debug_flags = a.debug_flags;

  // grid table per query tile: [K+1][128] values (hard) or [K+1][128]
  // (c_k, d_k) pairs (interpolation)
  p.tab_stride = (MAP == MAP_KI_INTERP) ? (p.K + 1) * 128 * 2 : (p.K + 1) * 128;
  const size_t table_bytes = static_cast<size_t>(2) * p.tab_stride * sizeof(float);
  // Bars: 2 per ring stage + 20 fixed mbarriers, then tmem_slot and abort;
  // sized for the deepest ring allowed below
  constexpr int kMaxStages = 8;
  const size_t bar_bytes = ((2 * kMaxStages + 20) * 8 + 8 + 15) & ~static_cast<size_t>(15);
  const size_t max_smem = 232448;                        // 227 KB opt-in per CTA
  const size_t fixed = 1024 + 2 * G::TILE_BYTES + table_bytes + bar_bytes +
                       (4 * 128 * 16 + 8 * 128 * 4 + 4 * 128 * 4);
  int ns = static_cast<int>((max_smem - fixed) / G::TILE_BYTES);
  if (ns > kMaxStages) ns = kMaxStages;
  if (ns < 2) return QSM_ERR_UNSUPPORTED;
  p.num_stages = ns;
  p.table_off = static_cast<uint32_t>(2 * G::TILE_BYTES + ns * G::TILE_BYTES);
  p.bar_off = static_cast<uint32_t>((p.table_off + table_bytes + 15) & ~static_cast<size_t>(15));
  p.xch_off = p.bar_off + static_cast<uint32_t>(bar_bytes);
  const size_t xch_bytes = 4 * 128 * 16 + 8 * 128 * 4 + 4 * 128 * 4;
  size_t smem = 1024 + p.xch_off + xch_bytes;
  // one CTA per SM: the kernel allocates all 512 TMEM columns
  if (smem < 120 * 1024) smem = 120 * 1024;

  auto kern = qsm_fwd_kernel<D, FP8, MAP>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return QSM_ERR_CUDA;
  dim3 grid(p.nqb * a.B * a.H);
  kern<<<grid, kThreads, smem, a.stream>>>(mq, mk, mv, p);
  return cudaGetLastError() == cudaSuccess ? QSM_OK : QSM_ERR_CUDA;
}

template <int D, bool FP8>
static qsm_status launch_d(const FwdArgs &a, const CUtensorMap &mq, const CUtensorMap &mk,
                           const CUtensorMap &mv) {
  if (a.mode == QSM_MODE_EXACT) return launch_t<D, FP8, MAP_EXACT>(a, mq, mk, mv);
  if (a.mode == QSM_MODE_ROWMAX_POT) return launch_t<D, FP8, MAP_POT>(a, mq, mk, mv);
  if (a.rounding == QSM_ROUND_HARD) return launch_t<D, FP8, MAP_KI_HARD>(a, mq, mk, mv);
  return launch_t<D, FP8, MAP_KI_INTERP>(a, mq, mk, mv);
}

qsm_status launch_fwd(const FwdArgs &a) {
  alignas(64) CUtensorMap mq, mk, mv;
  const int bh = a.B * a.H;
  if (!make_tmap_3d(&mq, a.Q, a.fp8, a.D, a.S, bh, 128) ||
      !make_tmap_3d(&mk, a.K, a.fp8, a.D, a.S, bh, 128) ||
      !make_tmap_3d(&mv, a.V, a.fp8, a.D, a.S, bh, 128))
    return QSM_ERR_CUDA;
  if (a.fp8) {
    if (a.D == 128) return launch_d<128, true>(a, mq, mk, mv);
    return QSM_ERR_UNSUPPORTED;
  }
  if (a.D == 128) return launch_d<128, false>(a, mq, mk, mv);
  if (a.D == 64) return launch_d<64, false>(a, mq, mk, mv);
  return QSM_ERR_UNSUPPORTED;
}

}  // namespace qsm
