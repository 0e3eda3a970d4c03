// bwd_noalloc.cu -- qsm_attn_bwd_noalloc: the backward without a caller
// workspace.
//
// Some callers cannot allocate device memory when they call the backward:
// for example a plugin inside a host framework that owns every device byte
// through its own pool and forbids driver allocations, or a latency-critical
// loop that cannot afford cudaMalloc's implicit device synchronisation.  For
// them the backward's scratch (the fp32 dQ accumulator, the fp32 dK
// calibration part and eight floats per query row) lives in one fixed
// array of this file, kScratchBytes long, which every GPU that loads the
// library holds until the process exits.
//
// In host code `g_bwd_scratch` names a host-side stand-in, not the device
// array, so the device address is looked up with cudaGetSymbolAddress, with
// the device current, the first time the entry point runs there, and cached
// for the driver context that is current then; a call under another context
// (after cudaDeviceReset, or with a non-primary context current) looks it up
// again.  Every call shares the array and the array keeps what the last call
// left in it: the launch clears the parts that must start at zero, and calls
// whose kernels overlap on the GPU (two streams, two host threads) race on it.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>
#include <mutex>

#include "internal.h"

namespace qsm {
namespace {

constexpr size_t kScratchBytes = QSM_NOALLOC_SCRATCH_BYTES;
static_assert(kScratchBytes % 256 == 0, "scratch size must keep 256-byte alignment");

__device__ __align__(256) unsigned char g_bwd_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
struct Cached {
  CUcontext ctx;
  void *ptr;
};
Cached g_scratch[kMaxDevices] = {};

using CtxGetCurrentFn = CUresult (*)(CUcontext *);

// The calling thread's current driver context (nullptr if none is bound yet
// or the driver entry point is unavailable).
CUcontext current_context() {
  static CtxGetCurrentFn fn = [] {
    void *f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<CtxGetCurrentFn>(nullptr);
    return reinterpret_cast<CtxGetCurrentFn>(f);
  }();
  CUcontext c = nullptr;
  if (fn == nullptr || fn(&c) != CUDA_SUCCESS) return nullptr;
  return c;
}

// Device address of the scratch array in the current context (nullptr on a
// CUDA error).
void *scratch_on_current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  const CUcontext ctx = current_context();
  if (g_scratch[dev].ptr != nullptr && ctx != nullptr && g_scratch[dev].ctx == ctx)
    return g_scratch[dev].ptr;
  void *p = nullptr;
  if (cudaGetSymbolAddress(&p, g_bwd_scratch) != cudaSuccess) return nullptr;
  // the lookup made the runtime's context current if none was
  g_scratch[dev].ctx = current_context();
  g_scratch[dev].ptr = p;
  return p;
}

}  // namespace
}  // namespace qsm

using namespace qsm;

extern "C" qsm_status qsm_attn_bwd_noalloc(const void *Q, const void *K, const void *V,
                                           const void *O, const void *dO, const float *LSE,
                                           void *dQ, void *dK, void *dV, int B, int H, int S,
                                           int D, int causal, qsm_mode mode, int Kint,
                                           qsm_calib calibration, qsm_rounding rounding,
                                           qsm_surrogate surrogate, const qsm_opts *opts,
                                           qsm_stream_t stream) {
  if (B < 1 || H < 1 || S < 1) return QSM_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return QSM_ERR_UNSUPPORTED;     // as qsm_attn_bwd
  if (qsm_attn_bwd_workspace_size(B, H, S, D) > kScratchBytes) return QSM_ERR_INVALID_ARG;
  void *scratch = scratch_on_current_device();
  if (scratch == nullptr) return QSM_ERR_CUDA;
  qsm_opts o;
  if (opts != nullptr)
    o = *opts;
  else
    qsm_opts_default(&o);
  o.workspace = scratch;
  o.workspace_bytes = kScratchBytes;
  return qsm_attn_bwd(Q, K, V, O, dO, LSE, dQ, dK, dV, B, H, S, D, causal, mode, Kint,
                      calibration, rounding, surrogate, &o, stream);
}
