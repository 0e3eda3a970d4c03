// fwd.cu -- fused approximate-softmax attention forward for sm_100a.
//
// One CTA owns one 128-row query tile of one (b, h) and sweeps the key/value
// tiles of 128 rows ("QK tile -> row max -> power-of-two weights -> PV matmul
// -> output", the tile loop of "Approximating Softmax in Pretrained LLMs",
// wiki flowchart).  Roles (20 warps):
//   warp 0      TMA producer: the Q tile once, then K (statistics sweep) and
//               K, V (main sweep) through a ring of shared-memory stages.
//   warp 1      QK issuer (one thread): S = Q K^T into TMEM (tcgen05, both
//               operands in shared memory).
//   warp 2      PV issuer (one thread): O += P V with P read from TMEM.
//   warps 4-19  four map groups of four warps (one thread per query row, the
//               row's TMEM lane), paired: pair 0 (warps 4-11) maps the even
//               key tiles, pair 1 (warps 12-19) the odd ones, so the two
//               pairs work on consecutive tiles at once; within a pair each
//               group owns 64 of the tile's 128 key columns.
// TMEM (512 columns): three S buffers at 0, 128, 256 and O at 384.  P (bf16
// or e4m3, packed) overwrites the S columns it was computed from, so the QK
// issuer runs up to two key tiles ahead of the map.  During the statistics
// sweep the O columns serve as a fourth S buffer.  Splitting the MMA stream
// over two issuers on different SM sub-partitions halves the instructions
// each must issue per key tile; the statistics sweep alternates key tiles
// between them.
//
// The approximate maps are defined against the row's final maximum (and
// minimum), so every map runs a statistics sweep first (S tiles, max / min /
// argmax / argmin only, no PV), then the main sweep with the row constants
// fixed.  The exact map uses the same two sweeps: softmax against the true
// row maximum, so O is never rescaled and the maps differ only in the weight
// arithmetic.
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

struct FwdParams {
  int S, nqt, BH;
  int causal;
  int hgroup;       // causal work order: heads per group (their K/V shares L2)
  int K;
  int fixed_window;
  int flush;        // below_policy == 1
  int pot_floor;
  float c;          // score scale
  float cL2E;       // c * log2(e), exact map
  float window;
  float v_descale;
  float pscale;     // P is stored as w * pscale (FP8 approximate maps: 64)
  float thr;        // probes: -(support width * log2e)
  int tab_stride;   // floats of grid table
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
};

constexpr int kThreads = 640;      // 4 control warps + 4 map warp groups
// Every warp keeps the launch allocation of 96 registers (65536 / 640).
constexpr int kGroups = 4;         // map warp groups
constexpr int kHalfCols = 64;     // key columns per map group and tile
constexpr int kMapThreads = 128 * kGroups;
constexpr int kPairThreads = 256;  // two groups map one key tile
constexpr int kSBufs = 3;          // S / P buffers of the main sweep
constexpr int kStatBufs = 4;       // S buffers of the statistics sweep
constexpr uint32_t kOCol = 384;    // first TMEM column of O
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxStages = 8;
// Statistics-sweep issuers: warps 1 and 2 take alternate key tiles, so each
// S buffer (tile j % 4) is always fed by the same issuer; a buffer shared by
// two issuers could see a later tile's wait pass on an older phase of the
// same parity.
constexpr int kStatIssuers = 2;
static_assert(kStatBufs % kStatIssuers == 0, "each statistics buffer needs a single issuer");
constexpr int kLead = 3;           // K tiles enter the ring this far ahead of V

// Main-sweep ring order: K_0 .. K_{kLead-1}, then V_0, K_kLead, V_1,
// K_kLead+1, ..., and the V tiles left over at the end.  K runs ahead because
// S = Q K^T is issued up to two tiles before the PV product that needs V.
__device__ __forceinline__ int ring_pos_k(int j) { return j < kLead ? j : 2 * j - kLead + 1; }
__device__ __forceinline__ int ring_pos_v(int j, int n) {
  return j < n - kLead ? kLead + 2 * j : n + j;
}

// mbarriers: two per ring stage, then the fixed ones
struct Bars {
  uint64_t *kv_full, *kv_empty;          // [stages]
  uint64_t *q_full;                      // 1
  uint64_t *st_full, *st_empty;          // [kStatBufs] statistics sweep
  uint64_t *st_done;                     // 1: every map thread finished the statistics sweep
  uint64_t *s_full, *p_full, *s_free;    // [kSBufs] main sweep
  uint64_t *o_full;                      // 1
  uint64_t *drain;                       // 1
  uint64_t *xstat, *xz;                  // 1 each: the map groups' exchanges
  uint32_t *tmem_slot;
  int *abort;
};
constexpr int kFixedBars = 1 + 2 * kStatBufs + 1 + 3 * kSBufs + 2 + 2;

__host__ __device__ constexpr size_t bar_bytes_for(int ns) {
  return ((2 * static_cast<size_t>(ns) + kFixedBars) * 8 + 8 + 15) & ~static_cast<size_t>(15);
}

__device__ __forceinline__ Bars carve_bars(uint8_t *base, int ns) {
  Bars b;
  uint64_t *p = reinterpret_cast<uint64_t *>(base);
  b.kv_full = p;
  b.kv_empty = p + ns;
  b.q_full = p + 2 * ns;
  b.st_full = b.q_full + 1;
  b.st_empty = b.st_full + kStatBufs;
  b.st_done = b.st_empty + kStatBufs;
  b.s_full = b.st_done + 1;
  b.p_full = b.s_full + kSBufs;
  b.s_free = b.p_full + kSBufs;
  b.o_full = b.s_free + kSBufs;
  b.drain = b.o_full + 1;
  b.xstat = b.drain + 1;
  b.xz = b.xstat + 1;
  b.tmem_slot = reinterpret_cast<uint32_t *>(b.xz + 1);
  b.abort = reinterpret_cast<int *>(b.tmem_slot + 1);
  return b;
}

// Weights of one 32-column chunk, packed for the PV MMA and stored to TMEM;
// FULL: every column valid.  z holds eight partial row sums as four pairs.
template <int MAP, bool FULL, bool FP8, bool FLUSH, bool SAT>
__device__ __forceinline__ void map_chunk(const uint32_t (&v)[32], const MapRow &m, int c0,
                                          int lim, bool flush_below, float2 (&z)[4],
                                          uint32_t taddr_pc) {
  auto wt = [&](int i) {          // weights of columns 2i, 2i+1
    const float2 r = make_float2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
    float2 w = pair_weights<MAP, FLUSH, SAT>(r, m, flush_below);
    if (!FULL) {
      w.x = (c0 + 2 * i < lim) ? w.x : 0.0f;
      w.y = (c0 + 2 * i + 1 < lim) ? w.y : 0.0f;
    }
    z[i & 3] = add2_rn(z[i & 3], w);
    return w;
  };
  if (FP8) {
    uint32_t pk[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float2 a = wt(2 * i), b = wt(2 * i + 1);
      pk[i] = pack_e4m3x4(a.x, a.y, b.x, b.y);
    }
    tmem_st8(taddr_pc, pk);
  } else {
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float2 a = wt(i);
      pk[i] = pack_bf16x2(a.x, a.y);
    }
    tmem_st16(taddr_pc, pk);
  }
}

// Decision dump of one chunk (debug option).
template <int MAP, bool SAT>
__device__ __forceinline__ void debug_chunk(int8_t *dbg_row, const uint32_t (&v)[32],
                                            const MapRow &m, int kv0, int c0, int lim,
                                            const FwdParams &p, bool flush_below) {
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    if (dbg_row != nullptr && kv0 + i < p.S) {
      const float r = __uint_as_float(v[i]);
      int n = map_raw_index<MAP, SAT>(r, m, p.flush != 0, p.pot_floor);
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

// Per-row values the map groups exchange through shared memory (see
// map_half).
struct Xch {
  float4 *stats;      // [kGroups][128]: max, min, argmax, argmin
  float *zsum;        // [kGroups][128]
};
constexpr size_t kXchBytes = kGroups * 128 * 16 + kGroups * 128 * 4;

// Scale this group's O columns, pack to bf16 and store the row's slice.
template <int OC>
__device__ __forceinline__ void o_store(uint32_t taddr, float oscale, __nv_bfloat16 *dst,
                                        bool row_ok) {
  uint32_t v[OC];
  if constexpr (OC == 32)
    tmem_ld32_sync(taddr, v);
  else
    tmem_ld16_sync(taddr, v);
  uint32_t pk[OC / 2];
#pragma unroll
  for (int i = 0; i < OC / 2; ++i)
    pk[i] = pack_bf16x2(__uint_as_float(v[2 * i]) * oscale, __uint_as_float(v[2 * i + 1]) * oscale);
  if (row_ok) {
    uint4 *d4 = reinterpret_cast<uint4 *>(dst);
#pragma unroll
    for (int i = 0; i < OC / 8; ++i)
      d4[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
  }
}

// Exact weights of one 32-column chunk against the row maximum, packed and
// stored to TMEM like map_chunk.
template <bool FULL, bool FP8>
__device__ __forceinline__ void exp_chunk(const uint32_t (&v)[32], float cL2E, float mL2E, int c0,
                                          int lim, float2 (&z)[4], uint32_t taddr_pc) {
  auto e = [&](int i) {           // weights of columns 2i, 2i+1
    float2 w = exact_pair(make_float2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1])),
                          cL2E, mL2E);
    if (!FULL) {
      w.x = (c0 + 2 * i < lim) ? w.x : 0.0f;
      w.y = (c0 + 2 * i + 1 < lim) ? w.y : 0.0f;
    }
    z[i & 3] = add2_rn(z[i & 3], w);
    return w;
  };
  if (FP8) {
    uint32_t pk[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float2 a = e(2 * i), b = e(2 * i + 1);
      pk[i] = pack_e4m3x4(a.x, a.y, b.x, b.y);
    }
    tmem_st8(taddr_pc, pk);
  } else {
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float2 a = e(i);
      pk[i] = pack_bf16x2(a.x, a.y);
    }
    tmem_st16(taddr_pc, pk);
  }
}

// One map warp group: group g = 2 * pair + half.  The pair takes key tiles
// j = pair, pair + 2, ... (the two pairs work on consecutive tiles at once);
// the half owns key columns 64 * half .. 64 * half + 63 of each of them.
// Thread `row` owns query row qi*128+row (TMEM lane `row`).  The four groups
// share each row: they combine the row statistics and the row sums through
// shared memory behind bounded-wait barriers, and build the row's grid table
// together.  P of the group's columns goes to the first 16 (e4m3) or 32
// (bf16) of its own S columns.
//
// Every map runs two sweeps: the statistics sweep finds the row's maximum
// (and minimum, arguments) over all keys, then the main sweep maps each score
// against those final values.  For the exact map this is softmax against the
// true row maximum, with no online rescaling of O.  DBG: the kernel writes
// the decision dump (a separate instantiation, so that the dump's code takes
// no registers from the ordinary one).
template <int D, bool FP8, int MAP, bool KSAT, bool DBG>
__device__ __forceinline__ void map_half(const FwdParams &p, const Bars &bars, int g, int row,
                                         uint32_t lane_base, int qi, int n, int bh, float *tab,
                                         const Xch &xc, volatile int *abort) {
  constexpr int OC = D / kGroups;                      // O columns of this group
  constexpr int PCOLS = FP8 ? 8 : 16;                  // TMEM columns per 32 P values
  const int pair = g >> 1, h = g & 1;
  const int qrow = qi * 128 + row;
  const bool row_ok = qrow < p.S;
  const int L = p.causal ? min(qrow + 1, p.S) : p.S;   // valid keys of the row
  const int c_off = kHalfCols * h;                     // first key column of this group
  bool ok = true;
  float rmax = -INFINITY, rmin = INFINITY;
  int amax = 0, amin = 0;
  bool nan_seen = false;             // argument scan: a NaN score (comparisons skip it)
  const bool want_arg = p.amax != nullptr || p.amin != nullptr;
  const bool want_min =
      ((MAP == MAP_KI_HARD || MAP == MAP_KI_INTERP) && !p.fixed_window) || p.lo != nullptr;

  // -------------------------------------------------- statistics sweep
  {
    float mx[4], mn[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) { mx[i] = -INFINITY; mn[i] = INFINITY; }
    for (int j = pair; j < n && ok; j += 2) {
      const int b = j & 3;                             // S buffer of tile j
      ok = warp_all(mbar_wait(&bars.st_full[b], (j >> 2) & 1, abort));
      if (!ok) break;
      tc_fence_after();
      const int lim = L - 128 * j - c_off;             // valid columns of this group
      const bool full = full_tile(p, qi, j);
      uint32_t v0[32], v1[32];
      tmem_ld32(lane_base + b * 128 + c_off, v0);
      tmem_ld32(lane_base + b * 128 + c_off + 32, v1);
      tmem_wait_ld();
      reg_fence32(v0);
      reg_fence32(v1);
      // the values are in registers: hand the buffer back before the reduction
      tc_fence_before();
      mbar_arrive(&bars.st_empty[b]);
      if (want_arg) {
        auto scan = [&](const uint32_t(&v)[32], int c0) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float x = __uint_as_float(v[i]);
            const bool valid = c0 + i < lim;
            const int col = 128 * j + c_off + c0 + i;
            if (valid && x > rmax) { rmax = x; amax = col; }
            if (valid && x < rmin) { rmin = x; amin = col; }
            nan_seen = nan_seen || (valid && x != x);
          }
        };
        scan(v0, 0);
        scan(v1, 32);
      } else if (full) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float a0 = __uint_as_float(v0[2 * i]), a1 = __uint_as_float(v0[2 * i + 1]);
          const float b0 = __uint_as_float(v1[2 * i]), b1 = __uint_as_float(v1[2 * i + 1]);
          mx[i & 1] = max3n(mx[i & 1], a0, a1);
          mx[2 + (i & 1)] = max3n(mx[2 + (i & 1)], b0, b1);
          if (want_min) {
            mn[i & 1] = min3n(mn[i & 1], a0, a1);
            mn[2 + (i & 1)] = min3n(mn[2 + (i & 1)], b0, b1);
          }
        }
      } else {
        auto red = [&](const uint32_t(&v)[32], int c0, int k) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float a0 = __uint_as_float(v[2 * i]), a1 = __uint_as_float(v[2 * i + 1]);
            const bool va = c0 + 2 * i < lim, vb = c0 + 2 * i + 1 < lim;
            mx[k + (i & 1)] = max3n(mx[k + (i & 1)], va ? a0 : -INFINITY, vb ? a1 : -INFINITY);
            if (want_min)
              mn[k + (i & 1)] = min3n(mn[k + (i & 1)], va ? a0 : INFINITY, vb ? a1 : INFINITY);
          }
        };
        red(v0, 0, 0);
        red(v1, 32, 2);
      }
    }
    // this thread has read every statistics tile it owns (a single-use
    // barrier: an issuer must not wait on another issuer's buffers by
    // parity, whose phases may still be two or more behind)
    mbar_arrive(bars.st_done);
    if (!want_arg) {
      rmax = max3n(mx[0], mx[1], max3n(mx[2], mx[3], mx[3]));
      rmin = min3n(mn[0], mn[1], min3n(mn[2], mn[3], mn[3]));
    } else if (nan_seen) {
      rmax = rmin = __int_as_float(0x7FFFFFFF);
    }
    // combine the four groups in a fixed order (ties: the lower key index), so
    // every group ends with the same row statistics
    if (ok) {
      xc.stats[g * 128 + row] = make_float4(rmax, rmin, __int_as_float(amax), __int_as_float(amin));
      mbar_arrive(bars.xstat);
      ok = warp_all(mbar_wait(bars.xstat, 0, abort));
    }
    if (ok) {
      rmax = -INFINITY;
      rmin = INFINITY;
      amax = amin = 0;
      bool nan_max = false, nan_min = false;
#pragma unroll
      for (int gg = 0; gg < kGroups; ++gg) {
        const float4 o = xc.stats[gg * 128 + row];
        const int oamax = __float_as_int(o.z), oamin = __float_as_int(o.w);
        if (o.x > rmax || (o.x == rmax && oamax < amax)) { rmax = o.x; amax = oamax; }
        if (o.y < rmin || (o.y == rmin && oamin < amin)) { rmin = o.y; amin = oamin; }
        nan_max = nan_max || o.x != o.x;
        nan_min = nan_min || o.y != o.y;
      }
      // a NaN score makes the row's statistics NaN (and its output NaN)
      if (nan_max) rmax = __int_as_float(0x7FFFFFFF);
      if (nan_min) rmin = __int_as_float(0x7FFFFFFF);
    }
  }

  // ------------------------------------------------------ main sweep
  float2 z[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) z[i] = make_float2(0.0f, 0.0f);
  float hi = 0.0f, lo = 0.0f;
  MapCall mc;
  mc.K = p.K;
  mc.fixed_window = p.fixed_window;
  mc.flush = p.flush;
  mc.pot_floor = p.pot_floor;
  mc.c = p.c;
  mc.cL2E = p.cL2E;
  mc.window = p.window;
  mc.pscale = p.pscale;
  mc.thr = p.thr;
  const bool pot_flush = MAP == MAP_POT && p.flush;

  const bool flush_below = (MAP == MAP_KI_HARD || MAP == MAP_KI_INTERP) && p.flush &&
                           p.fixed_window;
  // the four groups build interleaved entries of this row's grid table
  const MapRow mr = row_setup<MAP>(mc, rmax, rmin, tab, row, g, kGroups, hi, lo);
  const float mL2E = mr.mL2E;                       // exact map: the anchor in log2 units
  if ((MAP == MAP_KI_HARD || MAP == MAP_KI_INTERP) && ok) {
    // the table is complete before any group reads it
    mbar_arrive(bars.xstat);
    ok = warp_all(mbar_wait(bars.xstat, 1, abort));
  }
  int8_t *dbg_row = (DBG && p.dbg != nullptr && row_ok)
                        ? p.dbg + (static_cast<size_t>(bh) * p.S + qrow) * p.S
                        : nullptr;

  for (int j = pair; j < n && ok; j += 2) {
    const int b = j % kSBufs;                        // S / P buffer of tile j
    ok = warp_all(mbar_wait(&bars.s_full[b], (j / kSBufs) & 1, abort));
    if (!ok) break;
    tc_fence_after();
    const int lim = L - 128 * j - c_off;
    const bool full = full_tile(p, qi, j);
    const uint32_t sb = lane_base + b * 128 + c_off;
#pragma unroll 1
    for (int c = 0; c < 2; ++c) {
      uint32_t v[32];
      tmem_ld32_sync(sb + 32 * c, v);
      // P of chunk c lands in columns this group has already read
      const uint32_t pc = sb + c * PCOLS;
      if (MAP == MAP_EXACT) {
        if (full)
          exp_chunk<true, FP8>(v, p.cL2E, mL2E, 32 * c, lim, z, pc);
        else
          exp_chunk<false, FP8>(v, p.cL2E, mL2E, 32 * c, lim, z, pc);
        if (dbg_row != nullptr) {
          for (int i = 0; i < 32; ++i) {
            const int kv = 128 * j + c_off + 32 * c + i;
            if (kv < p.S) dbg_row[kv] = (32 * c + i < lim) ? 0 : -1;
          }
        }
      } else {
        if (pot_flush) {
          if (full)
            map_chunk<MAP, true, FP8, true, false>(v, mr, 32 * c, lim, false, z, pc);
          else
            map_chunk<MAP, false, FP8, true, false>(v, mr, 32 * c, lim, false, z, pc);
        } else if (KSAT) {
          if (full)
            map_chunk<MAP, true, FP8, false, true>(v, mr, 32 * c, lim, flush_below, z, pc);
          else
            map_chunk<MAP, false, FP8, false, true>(v, mr, 32 * c, lim, flush_below, z, pc);
        } else if (full) {
          map_chunk<MAP, true, FP8, false, false>(v, mr, 32 * c, lim, flush_below, z, pc);
        } else {
          map_chunk<MAP, false, FP8, false, false>(v, mr, 32 * c, lim, flush_below, z, pc);
        }
        if (DBG && p.dbg != nullptr)
          debug_chunk<MAP, KSAT>(dbg_row, v, mr, 128 * j + c_off + 32 * c, 32 * c, lim, p,
                           flush_below);
      }
    }
    tmem_wait_st();
    tc_fence_before();
    mbar_arrive(&bars.p_full[b]);
  }

  // ---------------------------------------------------------- epilogue
  if (ok) ok = warp_all(mbar_wait(bars.o_full, 0, abort));
  if (!ok) return;
  tc_fence_after();
  const float Zg = ((z[0].x + z[0].y) + (z[1].x + z[1].y)) + ((z[2].x + z[2].y) + (z[3].x + z[3].y));
  xc.zsum[g * 128 + row] = Zg;
  mbar_arrive(bars.xz);
  if (!warp_all(mbar_wait(bars.xz, 0, abort))) return;
  const float Z = (xc.zsum[row] + xc.zsum[128 + row]) + (xc.zsum[256 + row] + xc.zsum[384 + row]);
  // a row whose maximum is NaN or +inf (or, for min-max calibration, whose
  // minimum is -inf) has no defined weights: its O and LSE are NaN
  const bool bad = !(fabsf(hi) <= 3.402823466e38f) ||
                   ((MAP == MAP_KI_HARD || MAP == MAP_KI_INTERP) && !p.fixed_window &&
                    !(fabsf(lo) <= 3.402823466e38f));
  const float qnan = __int_as_float(0x7FFFFFFF);
  const float oscale = bad ? qnan : p.v_descale / Z;  // pscale cancels: P and Z both carry it
  o_store<OC>(lane_base + kOCol + g * OC, oscale,
              p.O + (static_cast<size_t>(bh) * p.S + qrow) * D + g * OC, row_ok);
  if (row_ok && g == 0) {
    const size_t ri = static_cast<size_t>(bh) * p.S + qrow;
    p.LSE[ri] = bad ? qnan : hi + logf(Z / p.pscale);
    if (p.hi) p.hi[ri] = hi;
    if (p.lo) p.lo[ri] = lo;
    if (p.amax) p.amax[ri] = amax;
    if (p.amin) p.amin[ri] = amin;
  }
}

template <int D, bool FP8, int MAP, bool KSAT, bool DBG>
__global__ void __launch_bounds__(kThreads, 1)
    qsm_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  using G = Geo<D, FP8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = smem_align1024(smem_raw);
  const int warp = threadIdx.x >> 5;
  // Work order: non-causal CTAs sweep one head's query tiles after another
  // (the running CTAs share few heads' K/V in L2); causal CTAs take groups of
  // hgroup heads, whose K/V fit in L2 together, and within a group go
  // heaviest first (longest-processing-time order, so the lightest tiles
  // form each group's tail).
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

  uint8_t *sQ = smem;                                   // the query tile
  uint8_t *sKV = smem + G::TILE_BYTES;                  // ns stages
  float *sTab = reinterpret_cast<float *>(smem + p.table_off);
  Bars bars = carve_bars(smem + p.bar_off, ns);
  Xch xc;
  xc.stats = reinterpret_cast<float4 *>(smem + p.xch_off);
  xc.zsum = reinterpret_cast<float *>(smem + p.xch_off + kGroups * 128 * 16);
  volatile int *abort = bars.abort;

  const int nkvt = (p.S + 127) / 128;
  const int n = p.causal ? min(nkvt, qi + 1) : nkvt;    // key tiles of this query tile

  if (threadIdx.x == 0) {
    for (int i = 0; i < ns; ++i) {
      mbar_init(&bars.kv_full[i], 1);
      mbar_init(&bars.kv_empty[i], 1);
    }
    mbar_init(bars.q_full, 1);
    for (int i = 0; i < kStatBufs; ++i) {
      mbar_init(&bars.st_full[i], 1);
      mbar_init(&bars.st_empty[i], kPairThreads);
    }
    mbar_init(bars.st_done, kMapThreads);
    for (int i = 0; i < kSBufs; ++i) {
      mbar_init(&bars.s_full[i], 1);
      mbar_init(&bars.p_full[i], kPairThreads);
      mbar_init(&bars.s_free[i], 1);
    }
    mbar_init(bars.o_full, 1);
    mbar_init(bars.drain, kStatIssuers);       // one commit per issuer
    mbar_init(bars.xstat, kMapThreads);
    mbar_init(bars.xz, kMapThreads);
    *bars.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(bars.tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *bars.tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // ring positions: statistics sweep K_0 .. K_{n-1}, then the main sweep in
    // the order of ring_pos_k / ring_pos_v
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
      uint32_t ph = 0;                  // completed passes over the ring
      bool ok = true;
      auto load = [&](const CUtensorMap *m, int kvt) {
        if (it >= ns) ok = ok && warp_all(mbar_wait(&bars.kv_empty[st], ph ^ 1, abort));
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
      for (int j = 0; j < n && ok; ++j) load(&tmK, j);
      for (int j = 0; j < kLead && j < n && ok; ++j) load(&tmK, j);
      for (int j = 0; j < n && ok; ++j) {
        load(&tmV, j);
        if (j + kLead < n) load(&tmK, j + kLead);
      }
      // let every load issued so far land before the CTA may exit
      mbar_wait(bars.q_full, 0, abort);
      for (int s = 0; s < ns && s < it; ++s) {
        const int fills = (it - s + ns - 1) / ns;  // loads issued into stage s
        mbar_wait(&bars.kv_full[s], (fills - 1) & 1, abort);
      }
    }
  } else if (warp <= kStatIssuers) {
    // ---------------------------------------------------------------- MMA
    // Warp 1 issues S = Q K^T, warp 2 issues O += P V (main sweep); in the
    // statistics sweep they take alternate key tiles.  Each ring position is
    // consumed, and released by an MMA commit, by exactly one of them.  The
    // whole warp runs the loop; the elected lane issues every MMA and every
    // commit (a commit tracks the MMAs of the thread that issues it).
    const bool leader = elect_one();
    const bool qk_role = warp == 1;
    const bool pv_role = warp == 2;
    const uint32_t qaddr = smem_u32(sQ);
    const uint32_t kvaddr0 = smem_u32(sKV);
    int pos = 0, pst = 0;               // ring position, its stage
    uint32_t pph = 0;                   // and the parity of its fill
    bool ok = warp_all(mbar_wait(bars.q_full, 0, abort));
    tc_fence_after();
    auto acquire = [&](int target) -> int {
      while (pos < target) {
        ++pos;
        if (++pst == ns) {
          pst = 0;
          pph ^= 1;
        }
      }
      ok = ok && warp_all(mbar_wait(&bars.kv_full[pst], pph, abort));
      tc_fence_after();
      return pst;
    };
    auto commit = [&](uint64_t *bar) {
      if (leader) mma_commit(bar);
      __syncwarp();
    };
    // Descriptors: the start-address field is the low 14 bits (address >> 4)
    // and every operand lies below 256 KB, so an operand offset is added to a
    // base descriptor instead of building each descriptor again.
    const uint64_t qdesc = smem_desc(qaddr, 16, 1024);
    const uint64_t kdesc = smem_desc(kvaddr0, 16, 1024);
    const uint64_t vdesc = smem_desc(kvaddr0, G::CHUNK_BYTES, 1024);
    auto issue_qk = [&](int st, uint32_t col) {
      const uint64_t kd = kdesc + ((st * G::TILE_BYTES) >> 4);
#pragma unroll
      for (int kk = 0; kk < G::KSTEPS_QK; ++kk) {
        const int e = kk * G::MMA_K;
        const uint32_t off = (e / G::EPC) * G::CHUNK_BYTES + (e % G::EPC) * G::ELEM;
        const uint64_t ad = qdesc + (off >> 4);
        const uint64_t bd = kd + (off >> 4);
        if (leader) {
          if (FP8)
            mma_ss_f8(tmem + col, ad, bd, G::IDESC_QK, kk > 0);
          else
            mma_ss_f16(tmem + col, ad, bd, G::IDESC_QK, kk > 0);
        }
      }
      __syncwarp();
    };
    auto issue_pv = [&](int st, uint32_t pcol, bool acc) {
      const uint64_t vd = vdesc + ((st * G::TILE_BYTES) >> 4);
#pragma unroll
      for (int kk = 0; kk < G::KSTEPS_PV; ++kk) {
        const uint64_t bd = vd + ((kk * G::MMA_K * 128) >> 4);
        // keys 64h .. 64h+63 of the tile sit, packed, from TMEM column 64h
        // (the map group owning that half writes its P into the first of
        // its own S columns): 8 columns per k-step
        const int key0 = kk * G::MMA_K;
        const uint32_t at = tmem + pcol + kHalfCols * (key0 / kHalfCols) +
                            ((key0 % kHalfCols) / G::MMA_K) * 8;
        if (leader) {
          if (FP8)
            mma_ts_f8(tmem + kOCol, at, bd, G::IDESC_PV, (acc || kk > 0) ? 1u : 0u);
          else
            mma_ts_f16(tmem + kOCol, at, bd, G::IDESC_PV, (acc || kk > 0) ? 1u : 0u);
        }
      }
      __syncwarp();
    };

    {
      // statistics sweep: key tile j goes to issuer warp 1 + j % 2, S buffer j % 4
      for (int j = warp - 1; j < n && ok; j += kStatIssuers) {
        const int st = acquire(j);
        if (!ok) break;
        const int b = j & 3, u = j >> 2;
        if (u >= 1) {
          ok = warp_all(mbar_wait(&bars.st_empty[b], (u - 1) & 1, abort));
          tc_fence_after();
          if (!ok) break;
        }
        issue_qk(st, b * 128);
        commit(&bars.st_full[b]);
        commit(&bars.kv_empty[st]);
      }
      // the main sweep writes S into buffers 0-2 (QK issuer) and O into
      // buffer 3 (PV issuer): wait until every statistics tile is read (the
      // map threads report that once, on a single-use barrier)
      if (qk_role || pv_role) {
        ok = ok && warp_all(mbar_wait(bars.st_done, 0, abort));
        tc_fence_after();
      }
    }
    const int base = n;                              // first main-sweep position
    int b = 0;
    uint32_t ph = 0;                                 // buffer j % 3, parity of its use
    if (qk_role) {
      for (int j = 0; j < n && ok; ++j) {
        const int st = acquire(base + ring_pos_k(j));
        if (!ok) break;
        if (j >= kSBufs) {
          // tile j-3's P has gone through its PV product
          ok = warp_all(mbar_wait(&bars.s_free[b], ph ^ 1, abort));
          tc_fence_after();
          if (!ok) break;
        }
        issue_qk(st, b * 128);
        commit(&bars.s_full[b]);
        commit(&bars.kv_empty[st]);
        if (++b == kSBufs) { b = 0; ph ^= 1; }
      }
    } else if (pv_role) {
      for (int j = 0; j < n && ok; ++j) {
        const int st = acquire(base + ring_pos_v(j, n));
        if (!ok) break;
        ok = warp_all(mbar_wait(&bars.p_full[b], ph, abort));
        tc_fence_after();
        if (!ok) break;
        issue_pv(st, b * 128, j > 0);
        commit(&bars.s_free[b]);
        commit(&bars.kv_empty[st]);
        if (++b == kSBufs) { b = 0; ph ^= 1; }
      }
      if (ok) commit(bars.o_full);
    }
    // every MMA issued must finish before TMEM is released
    commit(bars.drain);
    mbar_wait(bars.drain, 0, abort);
  } else if (warp >= 4) {
    const int g = (warp - 4) >> 2;                 // map group 0..3
    map_half<D, FP8, MAP, KSAT, DBG>(p, bars, g, threadIdx.x - 128 - g * 128,
                           tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16), qi, n, bh,
                           sTab, xc, abort);
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
  if (threadIdx.x == 0 && *bars.abort && p.status != nullptr) atomicExch(p.status, QSM_ERR_TIMEOUT);
}

// ------------------------------------------------------------------- host

constexpr int kMaxDevices = 64;

template <int D, bool FP8, int MAP, bool KSAT>
static qsm_status launch_t(const FwdArgs &a, const CUtensorMap &mq, const CUtensorMap &mk,
                           const CUtensorMap &mv) {
  using G = Geo<D, FP8>;
  FwdParams p{};
  p.S = a.S;
  p.nqt = (a.S + 127) / 128;
  p.BH = a.B * a.H;
  p.causal = a.causal;
  p.hgroup = causal_head_group(a.S, a.D, a.fp8, a.B * a.H);
  p.K = (MAP == MAP_KI_HARD || MAP == MAP_KI_INTERP) ? a.Kint : 1;
  p.fixed_window = a.calib == QSM_CALIB_FIXED_WINDOW;
  p.flush = a.below_policy == 1;
  p.pot_floor = a.pot_floor;
  p.c = a.c;
  p.cL2E = a.c * 1.4426950408889634f;
  p.window = a.window;
  // P carries 64 w in e4m3 for the maps whose weights reach 2^-15 exactly
  // (the exact and truncated maps keep w: ex2 values are not e4m3-exact anyway)
  p.pscale = (FP8 && MAP != MAP_EXACT && MAP != MAP_TRUNC) ? 64.0f : 1.0f;
  p.thr = -a.support * 1.4426950408889634f;
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

  // grid table: [K+1][128] values (hard) or [K+1][128] (c_k, d_k) pairs
  // (interpolation)
  p.tab_stride = (MAP == MAP_KI_INTERP) ? (p.K + 1) * 128 * 2 : (p.K + 1) * 128;
  const size_t table_bytes = static_cast<size_t>(p.tab_stride) * sizeof(float);
  const size_t bar_bytes = bar_bytes_for(kMaxStages);
  const size_t max_smem = 232448;                        // 227 KB opt-in per CTA
  const size_t fixed = 1024 + G::TILE_BYTES + table_bytes + 16 + bar_bytes + kXchBytes;
  int ns = static_cast<int>((max_smem - fixed) / G::TILE_BYTES);
  if (ns > kMaxStages) ns = kMaxStages;
  if (ns < 2) return QSM_ERR_UNSUPPORTED;
  p.num_stages = ns;
  p.table_off = static_cast<uint32_t>(G::TILE_BYTES + ns * G::TILE_BYTES);
  p.bar_off = static_cast<uint32_t>((p.table_off + table_bytes + 15) & ~static_cast<size_t>(15));
  p.xch_off = p.bar_off + static_cast<uint32_t>(bar_bytes);
  size_t smem = 1024 + p.xch_off + kXchBytes;
  // one CTA per SM: the kernel allocates all 512 TMEM columns
  if (smem < 120 * 1024) smem = 120 * 1024;
  if (smem > max_smem) return QSM_ERR_UNSUPPORTED;

  // the decision dump, when asked for, runs in its own instantiation
  const int dbg = p.dbg != nullptr ? 1 : 0;
  auto kern = dbg ? qsm_fwd_kernel<D, FP8, MAP, KSAT, true> : qsm_fwd_kernel<D, FP8, MAP, KSAT, false>;
  // Raising the kernel's dynamic shared memory limit is a driver round trip;
  // this instantiation remembers, per device, the largest limit already set.
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
  dim3 grid(p.nqt * a.B * a.H);
  kern<<<grid, kThreads, smem, a.stream>>>(mq, mk, mv, p);
  return cudaGetLastError() == cudaSuccess ? QSM_OK : QSM_ERR_CUDA;
}

template <int D, bool FP8>
static qsm_status launch_d(const FwdArgs &a, const CUtensorMap &mq, const CUtensorMap &mk,
                           const CUtensorMap &mv) {
  if (a.mode == QSM_MODE_EXACT) return launch_t<D, FP8, MAP_EXACT, false>(a, mq, mk, mv);
  if (a.mode == QSM_MODE_ROWMAX_POT) return launch_t<D, FP8, MAP_POT, false>(a, mq, mk, mv);
  if (a.mode == QSM_MODE_TRUNCATED) return launch_t<D, FP8, MAP_TRUNC, false>(a, mq, mk, mv);
  if (a.mode == QSM_MODE_UNIFORM) return launch_t<D, FP8, MAP_UNIFORM, false>(a, mq, mk, mv);
  // K-interval: K a power of two takes the saturating coordinate (map_pair)
  const bool p2 = k_pow2(a.Kint);
  if (a.rounding == QSM_ROUND_HARD)
    return p2 ? launch_t<D, FP8, MAP_KI_HARD, true>(a, mq, mk, mv)
              : launch_t<D, FP8, MAP_KI_HARD, false>(a, mq, mk, mv);
  return p2 ? launch_t<D, FP8, MAP_KI_INTERP, true>(a, mq, mk, mv)
            : launch_t<D, FP8, MAP_KI_INTERP, false>(a, mq, mk, mv);
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
