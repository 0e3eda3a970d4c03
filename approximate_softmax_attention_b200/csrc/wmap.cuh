// wmap.cuh -- the per-row weight maps, as the fused kernels evaluate them.
//
// K-interval attention ("Pretraining Transformers with Quantized Softmax in
// Attention", abstract: exp approximated from K+1 grid values, per-row grid
// calibration, interpolation versus hard rounding) and Rowmax-PoT
// ("Approximating Softmax in Pretrained LLMs", abstract: power-of-two weights
// anchored at each row maximum), plus the exact map.  The fused forward and
// the standalone map (qsm_weight_map) both call the functions below, so the
// standalone map is a bit-exact window onto the forward's arithmetic.
//
// Inputs are raw fp32 products r = q.k (the MMA accumulator); the score is
// s = c r with c = scale * q_descale * k_descale, folded into one FMA:
//
//   row statistics  rmax, rmin over the valid r (NaN-propagating max / min);
//                   hi = c*rmax, lo = c*rmin
//   exact       x = fma(r, c*log2e, -(rmax * c*log2e));   w = ex2.approx(x)
//   PoT         x = fma(r, -(c*log2e), hi*log2e); t = min(x, cap) + 1.5*2^23;
//               n = bits(t) - bits(1.5*2^23); w = 2^-n from the exponent field
//   K-interval  lc = lo (min-max) or hi - W; a = hi - lc; inv = K/a;
//               x = fma(r, c*inv, -(lc*inv))  (x = K on a degenerate row);
//               uc = min(max(x, 0), K)
//               hard:   n = bits(uc + 1.5*2^23) - bits(1.5*2^23); w = g[n]
//               interp: k = floor(uc) (a round-down add of 2^23), entry k of
//                       (c_k, d_k) = (g_k - k d_k, g_{k+1} - g_k), entry K
//                       repeating entry K-1; w = fma(uc, d_k, c_k)
//   grid        g[k] = own_exp(-(K-k) * step), step = a/K or W/K
//   probes      x as for the exact map; kept when x >= thr = -(T*log2e):
//               truncated w = 2^x (ex2.approx), uniform w = 1; 0 when cut
//
// Every operation is an explicit round-to-nearest (or round-down) intrinsic,
// so the compiler can neither contract nor reorder it, and an IEEE fp32
// restatement of the same sequence reproduces it bit for bit (the exact map's
// ex2.approx excepted, which is the hardware's own approximation).
#pragma once

#include <cstdint>

#include "sm100.cuh"

namespace qsm {

enum MapKind {
  MAP_EXACT = 0, MAP_POT = 1, MAP_KI_HARD = 2, MAP_KI_INTERP = 3,
  // the sensitivity probes: keys within the support width of the row
  // maximum keep their exact weight (TRUNC) or weight 1 (UNIFORM), the rest 0
  MAP_TRUNC = 4, MAP_UNIFORM = 5
};

constexpr float kMagic = 12582912.0f;                  // 1.5 * 2^23
constexpr uint32_t kMagicBits = 0x4B400000u;

__device__ __forceinline__ float f_of(uint32_t u) { return __uint_as_float(u); }

// log2(e) rounded to fp32
__device__ __forceinline__ float log2e_f() { return f_of(0x3FB8AA3Bu); }

__device__ __forceinline__ float rne_f(float x) {
  return __fsub_rn(__fadd_rn(x, kMagic), kMagic);
}

// exp(x) for x <= 0 without the special-function unit: Cody-Waite reduction
// x = n ln2 + r with ln2 split in a 16-bit head and a tail, then the degree-7
// Taylor polynomial of e^r (coefficients 1/k! rounded to fp32) in Horner
// form, scaled by 2^n through the exponent field.  Returns 0 below 2^-125.
// Faithfully rounded (< 1 ulp) on the range the grids use.
__device__ __forceinline__ float own_exp(float x) {
  const float n = rne_f(__fmul_rn(x, log2e_f()));
  if (n < -125.0f) return 0.0f;
  float r = __fmaf_rn(n, -f_of(0x3F317200u), x);       // ln2 head
  r = __fmaf_rn(n, -f_of(0x35BFBE8Eu), r);             // ln2 tail
  float p = f_of(0x39500D01u);                          // 1/7!
  p = __fmaf_rn(p, r, f_of(0x3AB60B61u));               // 1/6!
  p = __fmaf_rn(p, r, f_of(0x3C088889u));               // 1/5!
  p = __fmaf_rn(p, r, f_of(0x3D2AAAABu));               // 1/4!
  p = __fmaf_rn(p, r, f_of(0x3E2AAAABu));               // 1/3!
  p = __fmaf_rn(p, r, 0.5f);
  p = __fmaf_rn(p, r, 1.0f);
  p = __fmaf_rn(p, r, 1.0f);
  const int e = __float2int_rn(n);
  return __fmul_rn(p, __int_as_float((e + 127) << 23));
}

// Per-row constants of a K-interval grid, computed once per row from its
// statistics (score units).
struct RowMap {
  float hi;       // row max of s
  float lo;       // calibrated lower end (K-interval) / row min
  float inv;      // K / (hi - lo)          (K-interval; 0 when degenerate)
  float b;        // -(lo * inv)
  float hiL2E;    // hi * log2e              (PoT)
  float step;     // grid step               (K-interval)
  bool degenerate;
};

// hi, lo_obs: fp32 row max / min of s.
__device__ __forceinline__ RowMap make_rowmap(float hi, float lo_obs, int K, bool fixed_window,
                                              float window) {
  RowMap m;
  m.hi = hi;
  const float lc = fixed_window ? __fsub_rn(hi, window) : lo_obs;
  const float a = __fsub_rn(hi, lc);
  m.degenerate = !(a > 0.0f);
  const float Kf = static_cast<float>(K);
  m.step = fixed_window ? __fdiv_rn(window, Kf) : __fdiv_rn(a, Kf);
  m.inv = m.degenerate ? 0.0f : __fdiv_rn(Kf, a);
  m.b = -__fmul_rn(lc, m.inv);
  m.lo = lc;
  m.hiL2E = __fmul_rn(hi, log2e_f());
  return m;
}

// Grid value g[k] of a row, k = 0..K.
__device__ __forceinline__ float grid_value(const RowMap &m, int K, int k) {
  return own_exp(__fmul_rn(-static_cast<float>(K - k), m.step));
}

// ------------------------------------------------ packed fp32 pair arithmetic
// sm_100 f32x2 instructions: two IEEE round-to-nearest (or round-down)
// operations per instruction, the same results as the scalar forms.
__device__ __forceinline__ uint64_t f2_bits(float2 a) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a.x), "f"(a.y));
  return r;
}
__device__ __forceinline__ float2 f2_from(uint64_t r) {
  float2 a;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a.x), "=f"(a.y) : "l"(r));
  return a;
}
__device__ __forceinline__ float2 fma2_rn(float2 a, float2 b, float2 c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(f2_bits(a)), "l"(f2_bits(b)), "l"(f2_bits(c)));
  return f2_from(r);
}
__device__ __forceinline__ float2 add2_rn(float2 a, float2 b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(f2_bits(a)), "l"(f2_bits(b)));
  return f2_from(r);
}
__device__ __forceinline__ float2 mul2_rn(float2 a, float2 b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(f2_bits(a)), "l"(f2_bits(b)));
  return f2_from(r);
}
__device__ __forceinline__ float2 add2_rd(float2 a, float2 b) {
  uint64_t r;
  asm("add.rm.f32x2 %0, %1, %2;" : "=l"(r) : "l"(f2_bits(a)), "l"(f2_bits(b)));
  return f2_from(r);
}

// NaN-propagating fp32 maximum / minimum of three (one instruction on
// sm_100): a row with a NaN score gets NaN statistics.
__device__ __forceinline__ float max3n(float a, float b, float c) {
  float r;
  asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ float min3n(float a, float b, float c) {
  float r;
  asm("min.NaN.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// ------------------------------------------------------------ fused map
// Per-row constants of the fused map, with the score scale folded in: the
// map consumes the raw fp32 accumulator r of the QK product.
//   PoT:        x = fma(r, -c*log2e, hi*log2e), w = 2^-rne(min(x, cap)) * pscale
//   K-interval: x = fma(r, c*K/(hi-lo), -lo*K/(hi-lo)); hard: g[rne(x)];
//               interpolation: u d_k + c_k at k = floor(u) (grid values
//               pre-multiplied by pscale)
//   exact:      x = fma(r, c*log2e, -mL2E), w = 2^x
struct MapRow {
  float a, b;        // coordinate = fma(r, a, b) (K-interval, K = 2^m: both / K)
  float mk;          // K-interval, K = 2^m: 1.5 * 2^23 / K
  float cap, Kf, Km1;
  float flush_t;     // PoT flush: kMagic + floor (t above it: exponent past the floor)
  float mL2E;        // exact map: the anchor rmax * c * log2e
  uint32_t tab;      // shared address bias of this row's table column
  uint32_t pow_bias; // bits of pscale (PoT)
};

// Constants of one call of a map.
struct MapCall {
  int K;
  int fixed_window;
  int flush;        // below_policy == 1
  int pot_floor;
  float c;          // score scale
  float cL2E;       // c * log2(e)
  float window;
  float pscale;     // weights are produced as w * pscale (FP8 P: 64)
  float thr;        // probes: the support threshold -(T * log2e)
};

// K a power of two: the K-interval coordinate can be formed already divided
// by K and clamped by one saturating FMA (see map_pair).
__host__ __device__ constexpr bool k_pow2(int K) { return K > 0 && (K & (K - 1)) == 0; }

// Grid table layout: node n of the row in table column `row` (0..127) sits at
// float offset n*128 + row (hard rounding: g_n * pscale) or float2 offset
// n*128 + row (interpolation: (c_n, d_n) * pscale, d_n further times K when
// K is a power of two), n = 0..K.  Bytes needed: (K+1) * 128 * 4 (hard) or
// * 8 (interpolation).
__host__ __device__ constexpr int table_bytes_for(int map, int K) {
  return map == MAP_KI_HARD ? (K + 1) * 128 * 4 : (map == MAP_KI_INTERP ? (K + 1) * 128 * 8 : 0);
}

// Set up the map constants of one row from its raw statistics and write
// table entries n = n0, n0 + nstep, ... (<= K) of its grid column.  The
// caller makes the whole column visible before any map_pair on it.  Writes
// the row's hi (c*rmax) and calibrated lower end (K-interval) or row min.
template <int MAP>
__device__ __forceinline__ MapRow row_setup(const MapCall &mc, float rmax, float rmin, float *tab,
                                            int row, int n0, int nstep, float &hi, float &lo) {
  MapRow mr;
  mr.a = mr.b = 0.0f;
  mr.mk = kMagic;
  mr.cap = static_cast<float>(mc.flush ? mc.pot_floor + 1 : mc.pot_floor);
  mr.Kf = static_cast<float>(mc.K);
  mr.Km1 = static_cast<float>(mc.K - 1);
  mr.tab = 0;
  mr.pow_bias = __float_as_uint(mc.pscale);
  mr.flush_t = kMagic + static_cast<float>(mc.pot_floor);
  mr.mL2E = __fmul_rn(rmax, mc.cL2E);
  hi = __fmul_rn(mc.c, rmax);
  lo = __fmul_rn(mc.c, rmin);
  if (MAP == MAP_EXACT) return mr;
  if (MAP == MAP_TRUNC || MAP == MAP_UNIFORM) {
    mr.a = mc.cL2E;
    mr.b = -mr.mL2E;
    mr.cap = mc.thr;
    return mr;
  }
  const RowMap rm = make_rowmap(hi, lo, mc.K, mc.fixed_window != 0, mc.window);
  if (MAP == MAP_POT) {
    mr.a = -mc.cL2E;
    mr.b = rm.hiL2E;
    return mr;
  }
  mr.a = __fmul_rn(mc.c, rm.inv);
  mr.b = rm.b;
  if (rm.degenerate) {           // every key sits at the top node
    mr.a = 0.0f;
    mr.b = mr.Kf;
  }
  lo = rm.lo;
  // K = 2^m: the coordinate is kept divided by K (a / K and b / K are exact;
  // its sign, which the below-window flush tests, is unchanged), and 1.5 *
  // 2^23 / K has a unit in the last place of exactly 1 / K over [M/K, M/K + 1]
  const bool sat = k_pow2(mc.K);
  const float invK = sat ? 1.0f / mr.Kf : 1.0f;
  mr.a = __fmul_rn(mr.a, invK);
  mr.b = __fmul_rn(mr.b, invK);
  mr.mk = __fmul_rn(kMagic, invK);
  const uint32_t mkbits = __float_as_uint(mr.mk);
  const uint32_t tb = smem_u32(tab);
  if (MAP == MAP_KI_HARD) {
    for (int nn = n0; nn <= mc.K; nn += nstep)
      tab[nn * 128 + row] = __fmul_rn(grid_value(rm, mc.K, nn), mc.pscale);
    // bits(rne(u) + kMagic) = kMagicBits + n  ->  table row n (scaled:
    // bits(rne(u)/K + M/K) = bits(M/K) + n)
    mr.tab = tb + row * 4 - (sat ? mkbits : kMagicBits) * 512u;
  } else {
    // entries k = 0 .. K: (c_k, d_k) with d_k = g_{k+1} - g_k and
    // c_k = g_k - k d_k; entry K repeats entry K - 1.  K a power of two:
    // d_k is stored times K (exact), for w = (u/K) (K d_k) + c_k
    for (int nn = n0; nn <= mc.K; nn += nstep) {
      const int k = nn < mc.K ? nn : mc.K - 1;
      const float gk = grid_value(rm, mc.K, k);
      const float gk1 = grid_value(rm, mc.K, k + 1);
      const float d = __fmul_rn(__fsub_rn(gk1, gk), mc.pscale);
      tab[(nn * 128 + row) * 2 + 0] = __fmaf_rn(-static_cast<float>(k), d, __fmul_rn(gk, mc.pscale));
      tab[(nn * 128 + row) * 2 + 1] = sat ? __fmul_rn(d, mr.Kf) : d;
    }
    // floor bits: bits(2^23 + k) = 0x4B000000 + k  ->  table row k (scaled:
    // bits(floor_K(u/K) + M/K) = bits(M/K) + k)
    mr.tab = tb + row * 8 - (sat ? mkbits : 0x4B000000u) * 1024u;
  }
  return mr;
}

// fma with the result clamped to [0, 1] (NaN gives 0), one instruction.
__device__ __forceinline__ float fma_sat(float a, float b, float c) {
  return __saturatef(__fmaf_rn(a, b, c));
}

// Weights of two scores (the map's arithmetic on a pair; FLUSH: Rowmax-PoT
// with the below-floor policy "flush", exponents above the floor give 0).
// SAT (K-interval, K = 2^m, the row set up for it): the clamped coordinate
// is formed as v = sat(fma(r, a/K, b/K)) = clamp(u, 0, K) / K, exactly
// (scaling by a power of two commutes with rounding), so the node index,
// the rounding and the interpolated weight are bit-identical to the unscaled
// form's, for one instruction instead of an FMA and two clamps.  Callers
// take SAT exactly when k_pow2(K), as row_setup does.
template <int MAP, bool FLUSH, bool SAT = false>
__device__ __forceinline__ float2 map_pair(float2 r, const MapRow &m) {
  if ((MAP == MAP_KI_HARD || MAP == MAP_KI_INTERP) && SAT) {
    const float2 v = make_float2(fma_sat(r.x, m.a, m.b), fma_sat(r.y, m.a, m.b));
    if (MAP == MAP_KI_HARD) {
      const float2 t = add2_rn(v, make_float2(m.mk, m.mk));
      return make_float2(lds_f32(__float_as_uint(t.x) * 512u + m.tab),
                         lds_f32(__float_as_uint(t.y) * 512u + m.tab));
    }
    const float2 t = add2_rd(v, make_float2(m.mk, m.mk));
    const float2 c0 = lds_f32x2(__float_as_uint(t.x) * 1024u + m.tab);
    const float2 c1 = lds_f32x2(__float_as_uint(t.y) * 1024u + m.tab);
    return make_float2(__fmaf_rn(v.x, c0.y, c0.x), __fmaf_rn(v.y, c1.y, c1.x));
  }
  const float2 x = fma2_rn(r, make_float2(m.a, m.a), make_float2(m.b, m.b));
  if (MAP == MAP_TRUNC || MAP == MAP_UNIFORM) {
    float2 w = (MAP == MAP_TRUNC) ? make_float2(ex2_approx(x.x), ex2_approx(x.y))
                                  : make_float2(__uint_as_float(m.pow_bias),
                                                __uint_as_float(m.pow_bias));
    if (!(x.x >= m.cap)) w.x = 0.0f;
    if (!(x.y >= m.cap)) w.y = 0.0f;
    return w;
  } else if (MAP == MAP_POT) {
    const float2 t =
        add2_rn(make_float2(fminf(x.x, m.cap), fminf(x.y, m.cap)), make_float2(kMagic, kMagic));
    // 2^-n * pscale from the exponent field: bits(t) = kMagicBits + n and
    // kMagicBits << 23 == 0 (mod 2^32), so -(bits(t) << 23) == -(n << 23)
    float2 w = make_float2(__uint_as_float(__float_as_uint(t.x) * 0xFF800000u + m.pow_bias),
                           __uint_as_float(__float_as_uint(t.y) * 0xFF800000u + m.pow_bias));
    if (FLUSH) {
      // t is kMagic + n exactly: n > floor  <=>  t > kMagic + floor
      if (t.x > m.flush_t) w.x = 0.0f;
      if (t.y > m.flush_t) w.y = 0.0f;
    }
    return w;
  } else if (MAP == MAP_KI_HARD) {
    // the clamp to [0, K] bounds the table index for every input (masked
    // keys, ragged rows, near-degenerate rows, inf and NaN included)
    const float2 u = make_float2(fminf(fmaxf(x.x, 0.0f), m.Kf), fminf(fmaxf(x.y, 0.0f), m.Kf));
    const float2 t = add2_rn(u, make_float2(kMagic, kMagic));
    return make_float2(lds_f32(__float_as_uint(t.x) * 512u + m.tab),
                       lds_f32(__float_as_uint(t.y) * 512u + m.tab));
  } else {
    // interpolation as one FMA: w = g_k + (u - k) d_k = u d_k + c_k with
    // c_k = g_k - k d_k; k = floor(u) in [0, K] (the clamp bounds the index)
    // through a round-down add of 2^23; the table entry at k = K repeats
    // k = K - 1, which is the interpolation's value at u = K
    const float2 u = make_float2(fminf(fmaxf(x.x, 0.0f), m.Kf), fminf(fmaxf(x.y, 0.0f), m.Kf));
    const float2 t = add2_rd(u, make_float2(8388608.0f, 8388608.0f));
    const float2 c0 = lds_f32x2(__float_as_uint(t.x) * 1024u + m.tab);
    const float2 c1 = lds_f32x2(__float_as_uint(t.y) * 1024u + m.tab);
    return make_float2(__fmaf_rn(u.x, c0.y, c0.x), __fmaf_rn(u.y, c1.y, c1.x));
  }
}

// Weights of a pair with the K-interval fixed-window flush (coordinate below
// the window -> 0) applied when flush_below.
template <int MAP, bool FLUSH, bool SAT = false>
__device__ __forceinline__ float2 pair_weights(float2 r, const MapRow &m, bool flush_below) {
  float2 w = map_pair<MAP, FLUSH, SAT>(r, m);
  if (MAP == MAP_KI_HARD || MAP == MAP_KI_INTERP) {
    if (flush_below) {
      if (__fmaf_rn(r.x, m.a, m.b) < 0.0f) w.x = 0.0f;
      if (__fmaf_rn(r.y, m.a, m.b) < 0.0f) w.y = 0.0f;
    }
  }
  return w;
}

// Exact weights of a pair against the anchor mL2E (log2 units).
__device__ __forceinline__ float2 exact_pair(float2 r, float cL2E, float mL2E) {
  const float2 x = fma2_rn(r, make_float2(cL2E, cL2E), make_float2(-mL2E, -mL2E));
  return make_float2(ex2_approx(x.x), ex2_approx(x.y));
}

// Decision index of one element (debug dump and the standalone map; the same
// arithmetic as map_pair): PoT exponent (-2 flushed), hard node, lower node of
// the interpolation, 0 for the exact map.
template <int MAP, bool SAT = false>
__device__ __forceinline__ int map_raw_index(float r, const MapRow &m, bool flush, int N) {
  if (MAP == MAP_EXACT) return 0;
  const float x = __fmaf_rn(r, m.a, m.b);
  if (MAP == MAP_TRUNC || MAP == MAP_UNIFORM) return x >= m.cap ? 0 : -2;
  if (MAP == MAP_POT) {
    const int n = static_cast<int>(__float_as_uint(__fadd_rn(fminf(x, m.cap), kMagic)) -
                                   kMagicBits);
    return (flush && n > N) ? -2 : n;
  }
  if (SAT) {
    // the row was set up with the coordinate divided by K (map_pair's SAT)
    const float v = fma_sat(r, m.a, m.b);
    const uint32_t mb = __float_as_uint(m.mk);
    if (MAP == MAP_KI_HARD) return static_cast<int>(__float_as_uint(__fadd_rn(v, m.mk)) - mb);
    return min(static_cast<int>(__float_as_uint(__fadd_rd(v, m.mk)) - mb),
               static_cast<int>(m.Km1));
  }
  const float uc = fminf(fmaxf(x, 0.0f), m.Kf);
  if (MAP == MAP_KI_HARD)
    return static_cast<int>(__float_as_uint(__fadd_rn(uc, kMagic)) - kMagicBits);
  const float kf = fminf(__fsub_rn(__fadd_rd(uc, 8388608.0f), 8388608.0f), m.Km1);
  return static_cast<int>(kf);
}

}  // namespace qsm
