// wmap_kernel.cu -- the weight map alone on given fp32 scores (the maps'
// bit-exact test surface).  One warp per row: the row's max / min come from a
// warp reduction (exact in fp32 whatever the order), the grid values from the
// library's own exp, and every element goes through the same device functions
// the fused forward uses (wmap.cuh).
#include <cuda_runtime.h>

#include <cstdint>

#include "internal.h"
#include "wmap.cuh"

namespace qsm {

__global__ void __launch_bounds__(256)
    qsm_weight_map_kernel(const float *__restrict__ s, const int32_t *__restrict__ vlen, int rows,
                          int cols, int mode, int K, int fixed_window, int hard, float window,
                          int pot_floor, int flush, float *__restrict__ w,
                          int32_t *__restrict__ idx, float *__restrict__ hi_out,
                          float *__restrict__ lo_out) {
  extern __shared__ float tab[];                       // [warps][K+1]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.x * (blockDim.x >> 5) + warp;
  if (r >= rows) return;
  const float *sr = s + static_cast<size_t>(r) * cols;
  float *wr = w + static_cast<size_t>(r) * cols;
  int32_t *ir = idx ? idx + static_cast<size_t>(r) * cols : nullptr;
  int L = vlen[r];
  L = L < 1 ? 1 : (L > cols ? cols : L);
  float hi = -INFINITY, lo = INFINITY;
  for (int j = lane; j < L; j += 32) {
    hi = fmaxf(hi, sr[j]);
    lo = fminf(lo, sr[j]);
  }
  for (int o = 16; o > 0; o >>= 1) {
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
  }
  float *g = tab + warp * (K + 1);
  RowMap m = make_rowmap(hi, lo, K, fixed_window != 0, window);
  if (mode == QSM_MODE_KINTERVAL) {
    for (int k = lane; k <= K; k += 32) g[k] = grid_value(m, K, k);
    __syncwarp();
  }
  const float Kf = static_cast<float>(K);
  const float cap = static_cast<float>(flush ? pot_floor + 1 : pot_floor);
  for (int j = lane; j < cols; j += 32) {
    float wj = 0.0f;
    int n = -1;
    if (j < L) {
      const float x = sr[j];
      if (mode == QSM_MODE_EXACT) {
        wj = own_exp(__fsub_rn(x, hi));
        n = 0;
      } else if (mode == QSM_MODE_ROWMAX_POT) {
        wj = pot_weight(x, m.hiL2E, cap, pot_floor, flush != 0, n);
      } else {
        const float u = kint_u(x, m, Kf);
        if (flush && fixed_window && u < 0.0f) {
          wj = 0.0f;
          n = -2;
        } else if (hard) {
          n = kint_hard_node(u, Kf);
          wj = g[n];
        } else {
          float f;
          n = kint_interp_node(u, Kf, f);
          wj = kint_interp_weight(f, g[n], g[n + 1]);
        }
      }
    }
    wr[j] = wj;
    if (ir) ir[j] = n;
  }
  if (lane == 0) {
    if (hi_out) hi_out[r] = hi;
    if (lo_out) lo_out[r] = (mode == QSM_MODE_KINTERVAL) ? m.lo : lo;
  }
}

qsm_status launch_weight_map(const MapArgs &a) {
  const int K = a.mode == QSM_MODE_KINTERVAL ? a.Kint : 1;
  const int warps = 8;
  const dim3 grid((a.rows + warps - 1) / warps);
  const size_t smem = static_cast<size_t>(warps) * (K + 1) * sizeof(float);
  qsm_weight_map_kernel<<<grid, warps * 32, smem, a.stream>>>(
      a.scores, a.valid_len, a.rows, a.cols, a.mode, K, a.calib == QSM_CALIB_FIXED_WINDOW,
      a.rounding == QSM_ROUND_HARD, a.window, a.pot_floor, a.below_policy == 1, a.w, a.idx, a.hi,
      a.lo);
  return cudaGetLastError() == cudaSuccess ? QSM_OK : QSM_ERR_CUDA;
}

}  // namespace qsm
