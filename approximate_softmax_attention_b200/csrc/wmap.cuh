// wmap.cuh -- the per-row weight maps on fp32 scores.
//
// K-interval attention ("Pretraining Transformers with Quantized Softmax in
// Attention", abstract: exp approximated from K+1 grid values, per-row grid
// calibration, interpolation versus hard rounding) and Rowmax-PoT
// ("Approximating Softmax in Pretrained LLMs", abstract: power-of-two weights
// anchored at each row maximum), in the library's fp32 operation order:
//
//   PoT        x = fma(s, -log2e, hi*log2e); n = rne(min(x, cap)); w = 2^-n
//   K-interval u = fma(s, inv, b) with inv = K/(hi-lo), b = -(lo*inv);
//              uc = clamp(u, 0, K); hard: n = rne(uc), w = g[n];
//              interp: k = min(floor(uc), K-1), f = uc - k,
//                      w = fma(f, g[k+1] - g[k], g[k])
//   grid       g[k] = own_exp(-(K-k) * step), step = (hi-lo)/K or W/K
//
// rne(x) = (x + 1.5*2^23) - 1.5*2^23.  Every operation is written with an
// explicit round-to-nearest intrinsic, so the compiler cannot contract or
// reorder it; the result is therefore reproducible bit for bit by any IEEE
// fp32 implementation of the same sequence.
#pragma once

#include <cstdint>

namespace qsm {

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

// Per-row constants of a map, computed once per row from its statistics.
struct RowMap {
  float hi;       // row max of s
  float lo;       // calibrated lower end (K-interval) / row min
  float inv;      // K / (hi - lo)          (K-interval; 0 when degenerate)
  float b;        // -(lo * inv)
  float hiL2E;    // hi * log2e              (PoT)
  float step;     // grid step               (K-interval)
  bool degenerate;
};

// hi, lo_obs: exact fp32 row max / min of s.
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

// Rowmax-PoT: returns w and writes the exponent n (or -2 when flushed).
// cap = N (clamp) or N + 1 (flush).
__device__ __forceinline__ float pot_weight(float s, float hiL2E, float cap, int N, bool flush,
                                            int &n_out) {
  const float x = __fmaf_rn(s, -log2e_f(), hiL2E);
  const float t = __fadd_rn(fminf(x, cap), kMagic);
  const int n = static_cast<int>(__float_as_uint(t) - kMagicBits);
  if (flush && n > N) {
    n_out = -2;
    return 0.0f;
  }
  n_out = n;
  return __uint_as_float(0x3F800000u - (static_cast<uint32_t>(n) << 23));
}

// K-interval grid coordinate before clamping.
__device__ __forceinline__ float kint_u(float s, const RowMap &m, float Kf) {
  return m.degenerate ? Kf : __fmaf_rn(s, m.inv, m.b);
}

// Hard rounding: nearest node of the clamped coordinate.
__device__ __forceinline__ int kint_hard_node(float u, float Kf) {
  const float uc = fminf(fmaxf(u, 0.0f), Kf);
  return static_cast<int>(__float_as_uint(__fadd_rn(uc, kMagic)) - kMagicBits);
}

// Interpolation: lower node k and fraction f of the clamped coordinate.
__device__ __forceinline__ int kint_interp_node(float u, float Kf, float &f) {
  const float uc = fminf(fmaxf(u, 0.0f), Kf);
  const float kf = fminf(floorf(uc), __fsub_rn(Kf, 1.0f));
  f = __fsub_rn(uc, kf);
  return static_cast<int>(__float_as_uint(__fadd_rn(kf, kMagic)) - kMagicBits);
}

__device__ __forceinline__ float kint_interp_weight(float f, float g0, float g1) {
  return __fmaf_rn(f, __fsub_rn(g1, g0), g0);
}

}  // namespace qsm
