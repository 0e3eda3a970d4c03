// wmap_kernel.cu -- the weight map alone on given fp32 raw products (the
// maps' bit-exact test surface).
//
// It runs the fused forward's own device functions (wmap.cuh): row_setup
// for the per-row constants and grid table, pair_weights / exact_pair for the
// weights and map_raw_index for the decision index, on raw products r with
// the score scale c folded in exactly as the forward folds it.  One thread
// per row (the table layout keeps one column per row of a 128-row block),
// columns taken in pairs as the forward takes them; the row statistics come
// from a sequential NaN-propagating max / min, exact in fp32 whatever the
// order.
#include <cuda_runtime.h>

#include <cstdint>

#include "internal.h"
#include "wmap.cuh"

namespace qsm {

namespace {

constexpr int kRowsPerBlock = 128;

template <int MAP, bool FLUSH>
__global__ void __launch_bounds__(kRowsPerBlock)
    qsm_weight_map_kernel(const float *__restrict__ r_in, const int32_t *__restrict__ vlen,
                          int rows, int cols, MapCall mc, int below_flush,
                          float *__restrict__ w, int32_t *__restrict__ idx,
                          float *__restrict__ hi_out, float *__restrict__ lo_out) {
  extern __shared__ float tab[];                       // [K+1][128] entries
  const int row = threadIdx.x;
  const int r = blockIdx.x * kRowsPerBlock + row;
  if (r >= rows) return;                               // no block-wide barrier below
  const float *rr = r_in + static_cast<size_t>(r) * cols;
  float *wr = w + static_cast<size_t>(r) * cols;
  int32_t *ir = idx ? idx + static_cast<size_t>(r) * cols : nullptr;
  int L = vlen[r];
  L = L < 1 ? 1 : (L > cols ? cols : L);
  float rmax = -INFINITY, rmin = INFINITY;
  for (int j = 0; j < L; ++j) {
    rmax = max3n(rmax, rr[j], rr[j]);
    rmin = min3n(rmin, rr[j], rr[j]);
  }
  float hi, lo;
  // this thread owns table column `row` and writes all of it
  const MapRow mr = row_setup<MAP>(mc, rmax, rmin, tab, row, 0, 1, hi, lo);
  const bool flush_below = (MAP == MAP_KI_HARD || MAP == MAP_KI_INTERP) && below_flush != 0;
  for (int j = 0; j < cols; j += 2) {
    const bool v0 = j < L, v1 = j + 1 < L;
    const float2 x = make_float2(rr[j], j + 1 < cols ? rr[j + 1] : 0.0f);
    float2 wt;
    if (MAP == MAP_EXACT)
      wt = exact_pair(x, mc.cL2E, mr.mL2E);
    else if ((MAP == MAP_KI_HARD || MAP == MAP_KI_INTERP) && k_pow2(mc.K))
      wt = pair_weights<MAP, FLUSH, true>(x, mr, flush_below);   // as the fused forward
    else
      wt = pair_weights<MAP, FLUSH>(x, mr, flush_below);
    wr[j] = v0 ? wt.x : 0.0f;
    if (j + 1 < cols) wr[j + 1] = v1 ? wt.y : 0.0f;
    if (ir) {
      for (int e = 0; e < 2 && j + e < cols; ++e) {
        const float xe = e ? x.y : x.x;
        int n = ((MAP == MAP_KI_HARD || MAP == MAP_KI_INTERP) && k_pow2(mc.K))
                    ? map_raw_index<MAP, true>(xe, mr, mc.flush != 0, mc.pot_floor)
                    : map_raw_index<MAP, false>(xe, mr, mc.flush != 0, mc.pot_floor);
        if (flush_below && __fmaf_rn(xe, mr.a, mr.b) < 0.0f) n = -2;
        ir[j + e] = (j + e < L) ? n : -1;
      }
    }
  }
  if (hi_out) hi_out[r] = hi;
  if (lo_out) lo_out[r] = lo;
}

template <int MAP, bool FLUSH>
qsm_status launch_map_t(const MapArgs &a, const MapCall &mc) {
  const size_t smem = static_cast<size_t>(table_bytes_for(MAP, mc.K));
  auto kern = qsm_weight_map_kernel<MAP, FLUSH>;
  // the largest table (interpolation, K = 64) needs 66.5 KB
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return QSM_ERR_CUDA;
  const dim3 grid((a.rows + kRowsPerBlock - 1) / kRowsPerBlock);
  kern<<<grid, kRowsPerBlock, smem, a.stream>>>(
      a.scores, a.valid_len, a.rows, a.cols, mc,
      a.below_policy == 1 && a.calib == QSM_CALIB_FIXED_WINDOW, a.w, a.idx, a.hi, a.lo);
  return cudaGetLastError() == cudaSuccess ? QSM_OK : QSM_ERR_CUDA;
}

}  // namespace

qsm_status launch_weight_map(const MapArgs &a) {
  MapCall mc;
  mc.K = a.mode == QSM_MODE_KINTERVAL ? a.Kint : 1;
  mc.fixed_window = a.calib == QSM_CALIB_FIXED_WINDOW;
  mc.flush = a.below_policy == 1;
  mc.pot_floor = a.pot_floor;
  mc.c = a.c;
  mc.cL2E = a.c * 1.4426950408889634f;
  mc.window = a.window;
  mc.pscale = 1.0f;
  mc.thr = -a.support * 1.4426950408889634f;
  if (a.mode == QSM_MODE_EXACT) return launch_map_t<MAP_EXACT, false>(a, mc);
  if (a.mode == QSM_MODE_TRUNCATED) return launch_map_t<MAP_TRUNC, false>(a, mc);
  if (a.mode == QSM_MODE_UNIFORM) return launch_map_t<MAP_UNIFORM, false>(a, mc);
  if (a.mode == QSM_MODE_ROWMAX_POT)
    return mc.flush ? launch_map_t<MAP_POT, true>(a, mc) : launch_map_t<MAP_POT, false>(a, mc);
  if (a.rounding == QSM_ROUND_HARD) return launch_map_t<MAP_KI_HARD, false>(a, mc);
  return launch_map_t<MAP_KI_INTERP, false>(a, mc);
}

}  // namespace qsm
