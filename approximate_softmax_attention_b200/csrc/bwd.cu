// bwd.cu -- backward of the fused attention (K-interval and exact maps).
#include <cuda_runtime.h>

#include "internal.h"

namespace qsm {

size_t bwd_workspace_bytes(int B, int H, int S, int D) {
  // dQ fp32 accumulator + per-row fp32 terms, 256-byte aligned
  const size_t rows = static_cast<size_t>(B) * H * S;
  size_t bytes = rows * D * sizeof(float);
  bytes = (bytes + 255) & ~static_cast<size_t>(255);
  bytes += ((rows * 4 * sizeof(float)) + 255) & ~static_cast<size_t>(255);
  return bytes;
}

qsm_status launch_bwd(const BwdArgs &) { return QSM_ERR_UNSUPPORTED; }

}  // namespace qsm
