// internal.h -- host-side declarations shared by the library's .cu files.
#pragma once

#include <cstddef>
#include <cstdint>

#include "../../include/qsm.h"

namespace qsm {

// Everything a forward launch needs, validated by the C entry point.
struct FwdArgs {
  const void *Q, *K, *V;
  void *O;
  float *LSE;
  int B, H, S, D;
  int causal;
  int mode, Kint, calib, rounding;
  int fp8;
  float c;          // scale * q_descale * k_descale
  float v_descale;
  float window;
  int pot_floor, below_policy;
  float support;    // probes: support width T (natural-log units of s)
  float *row_hi, *row_lo;
  int32_t *row_argmax, *row_argmin;
  int8_t *debug_idx;
  int32_t *status_dev;
  int debug_flags;
  int anchor;
  cudaStream_t stream;
};

qsm_status launch_fwd(const FwdArgs &a);         // two sweeps (anchor 0)
qsm_status launch_fwd_online(const FwdArgs &a);  // one sweep (anchor 1)

struct MapArgs {
  const float *scores;     // raw products r; the score is c * r
  float c;
  const int32_t *valid_len;
  int rows, cols;
  int mode, Kint, calib, rounding;
  float window;
  int pot_floor, below_policy;
  float support;
  float *w;
  int32_t *idx;
  float *hi, *lo;
  cudaStream_t stream;
};

qsm_status launch_weight_map(const MapArgs &a);

struct BwdArgs {
  const void *Q, *K, *V, *O, *dO;
  const float *LSE;
  void *dQ, *dK, *dV;
  int B, H, S, D, causal;
  int mode, Kint, calib, rounding, surrogate, detach;
  float c, window;
  // e4m3 inputs (D = 128): Q, K, V hold codes that stand for q_descale Q,
  // k_descale K, v_descale V; scale is the score scale before the descales
  int fp8;
  float scale, q_descale, k_descale, v_descale;
  int below_policy, pot_floor;
  const float *row_hi, *row_lo;
  const int32_t *row_argmax, *row_argmin;
  void *workspace;
  size_t workspace_bytes;
  int32_t *status_dev;
  cudaStream_t stream;
};

qsm_status launch_bwd(const BwdArgs &a);

// Causal forward work order: heads per group, so that the K and V of one
// group (2 S D bytes per element each head) stay within about 48 MB of the
// 126 MB L2 while the running CTAs sweep them.
inline int causal_head_group(int S, int D, bool fp8, int BH) {
  const double kv = 2.0 * S * D * (fp8 ? 1 : 2);
  int g = static_cast<int>((48.0 * 1024 * 1024) / kv);
  if (g < 1) g = 1;
  if (g > BH) g = BH;
  return g;
}
size_t bwd_workspace_bytes(int B, int H, int S, int D);

// cuTensorMapEncodeTiled through the runtime's driver entry point (no
// link-time dependency on libcuda).
bool make_tmap_3d(void *map_out, const void *base, bool fp8, int D, int S, int BH, int box_rows);

}  // namespace qsm
