// api.cu -- the library's C entry points: argument validation (every error is
// returned before any launch, and nothing is written), option defaults and
// dispatch to the launchers.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>

#include "internal.h"

namespace qsm {

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void *f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  }
  return fn;
}

qsm_opts defaults() {
  qsm_opts o;
  std::memset(&o, 0, sizeof(o));
  o.dtype = QSM_BF16;
  o.scale = 0.0f;
  o.q_descale = o.k_descale = o.v_descale = 1.0f;
  o.window = 8.0f;
  o.pot_floor = 15;
  o.below_policy = 0;
  o.support = 4.0f;
  return o;
}

bool finite_pos(float x) { return std::isfinite(x) && x > 0.0f; }

// Checks shared by forward and backward; fills *c with the score scale.
qsm_status check_common(int B, int H, int S, int D, int causal, int mode, int Kint, int calib,
                        int rounding, int surrogate, const qsm_opts &o, float *c) {
  if (B < 1 || H < 1 || S < 1 || S > 65536) return QSM_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * H > 65535) return QSM_ERR_UNSUPPORTED;
  if (causal != 0 && causal != 1) return QSM_ERR_INVALID_ARG;
  if (mode < QSM_MODE_EXACT || mode > QSM_MODE_UNIFORM) return QSM_ERR_INVALID_ARG;
  if (calib != QSM_CALIB_MINMAX && calib != QSM_CALIB_FIXED_WINDOW) return QSM_ERR_INVALID_ARG;
  if (rounding != QSM_ROUND_INTERP && rounding != QSM_ROUND_HARD) return QSM_ERR_INVALID_ARG;
  if (surrogate < QSM_SURR_NONE || surrogate > QSM_SURR_POST) return QSM_ERR_INVALID_ARG;
  if (mode == QSM_MODE_KINTERVAL && (Kint < 1 || Kint > 64)) return QSM_ERR_INVALID_ARG;
  if (o.dtype != QSM_BF16 && o.dtype != QSM_FP8_E4M3) return QSM_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return QSM_ERR_UNSUPPORTED;
  if (o.dtype == QSM_FP8_E4M3 && D != 128) return QSM_ERR_UNSUPPORTED;
  if (!(o.scale == 0.0f || finite_pos(o.scale))) return QSM_ERR_INVALID_ARG;
  if (!finite_pos(o.q_descale) || !finite_pos(o.k_descale) || !finite_pos(o.v_descale))
    return QSM_ERR_INVALID_ARG;
  if (!finite_pos(o.window)) return QSM_ERR_INVALID_ARG;
  if (o.pot_floor < 0 || o.pot_floor > 126) return QSM_ERR_INVALID_ARG;
  if (o.below_policy != 0 && o.below_policy != 1) return QSM_ERR_INVALID_ARG;
  if (o.detach_extrema != 0 && o.detach_extrema != 1) return QSM_ERR_INVALID_ARG;
  if (o.anchor != 0 && o.anchor != 1) return QSM_ERR_INVALID_ARG;
  if (!(o.support >= 0.0f) || !std::isfinite(o.support)) return QSM_ERR_INVALID_ARG;
  // the probes are defined against the final row maximum only
  if (o.anchor == 1 && (mode == QSM_MODE_TRUNCATED || mode == QSM_MODE_UNIFORM))
    return QSM_ERR_UNSUPPORTED;
  // the running anchor has no min-max form (the grid would follow the
  // running minimum too)
  if (o.anchor == 1 && mode == QSM_MODE_KINTERVAL && calib == QSM_CALIB_MINMAX)
    return QSM_ERR_UNSUPPORTED;
  const float scale = o.scale > 0.0f ? o.scale : 1.0f / std::sqrt(static_cast<float>(D));
  *c = scale * o.q_descale * o.k_descale;
  if (!finite_pos(*c)) return QSM_ERR_INVALID_ARG;
  return QSM_OK;
}

}  // namespace

bool make_tmap_3d(void *map_out, const void *base, bool fp8, int D, int S, int BH,
                  int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  const cuuint64_t es = fp8 ? 1 : 2;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(S),
                        static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {D * es, static_cast<cuuint64_t>(S) * D * es};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / es), static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(static_cast<CUtensorMap *>(map_out),
                   fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                   const_cast<void *>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace qsm

using namespace qsm;

extern "C" {

void qsm_opts_default(qsm_opts *opts) {
  if (opts) *opts = defaults();
}

const char *qsm_version(void) { return "0.1.0"; }

const char *qsm_status_string(qsm_status s) {
  switch (s) {
    case QSM_OK: return "QSM_OK";
    case QSM_ERR_INVALID_ARG: return "QSM_ERR_INVALID_ARG: invalid argument";
    case QSM_ERR_UNSUPPORTED: return "QSM_ERR_UNSUPPORTED: configuration not implemented";
    case QSM_ERR_CUDA: return "QSM_ERR_CUDA: CUDA call failed";
    case QSM_ERR_TIMEOUT: return "QSM_ERR_TIMEOUT: a device-side wait ran out";
  }
  return "QSM unknown status";
}

qsm_status qsm_attn_fwd(const void *Q, const void *K, const void *V, void *O, float *LSE, int B,
                        int H, int S, int D, int causal, qsm_mode mode, int Kint,
                        qsm_calib calibration, qsm_rounding rounding, qsm_surrogate surrogate,
                        const qsm_opts *opts, qsm_stream_t stream) {
  const qsm_opts o = opts ? *opts : defaults();
  float c = 0.0f;
  qsm_status st = check_common(B, H, S, D, causal, mode, Kint, calibration, rounding, surrogate,
                               o, &c);
  if (st != QSM_OK) return st;
  if (!Q || !K || !V || !O || !LSE) return QSM_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) ||
      (reinterpret_cast<uintptr_t>(LSE) & 3u))
    return QSM_ERR_INVALID_ARG;
  FwdArgs a{};
  a.Q = Q; a.K = K; a.V = V; a.O = O; a.LSE = LSE;
  a.B = B; a.H = H; a.S = S; a.D = D; a.causal = causal;
  a.mode = mode; a.Kint = Kint; a.calib = calibration; a.rounding = rounding;
  a.fp8 = o.dtype == QSM_FP8_E4M3;
  a.c = c;
  a.v_descale = o.v_descale;
  a.window = o.window;
  a.pot_floor = o.pot_floor;
  a.below_policy = o.below_policy;
  a.support = o.support;
  a.row_hi = o.row_hi; a.row_lo = o.row_lo;
  a.row_argmax = o.row_argmax; a.row_argmin = o.row_argmin;
  a.debug_idx = o.debug_idx;
  a.status_dev = o.status_dev;
  a.debug_flags = o.debug_flags;
  a.anchor = o.anchor;
  a.stream = reinterpret_cast<cudaStream_t>(stream);
  if (o.anchor == 1) {
    if (o.row_argmax || o.row_argmin) return QSM_ERR_UNSUPPORTED;
    return launch_fwd_online(a);
  }
  return launch_fwd(a);
}

qsm_status qsm_attn_bwd(const void *Q, const void *K, const void *V, const void *O,
                        const void *dO, const float *LSE, void *dQ, void *dK, void *dV, int B,
                        int H, int S, int D, int causal, qsm_mode mode, int Kint,
                        qsm_calib calibration, qsm_rounding rounding, qsm_surrogate surrogate,
                        const qsm_opts *opts, qsm_stream_t stream) {
  const qsm_opts o = opts ? *opts : defaults();
  float c = 0.0f;
  qsm_status st = check_common(B, H, S, D, causal, mode, Kint, calibration, rounding, surrogate,
                               o, &c);
  if (st != QSM_OK) return st;
  if (!Q || !K || !V || !O || !dO || !LSE || !dQ || !dK || !dV) return QSM_ERR_INVALID_ARG;
  // rows are read and written as 16-byte vectors
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(dO) ||
      !aligned16(dQ) || !aligned16(dK) || !aligned16(dV) ||
      (reinterpret_cast<uintptr_t>(LSE) & 3u))
    return QSM_ERR_INVALID_ARG;
  // the probes are forward-only sensitivity studies
  if (mode == QSM_MODE_TRUNCATED || mode == QSM_MODE_UNIFORM) return QSM_ERR_UNSUPPORTED;
  // the rules are derived for maps anchored at the final row statistics; the
  // exact map is softmax under either anchor
  if (o.anchor == 1 && mode != QSM_MODE_EXACT) return QSM_ERR_UNSUPPORTED;
  if (mode == QSM_MODE_KINTERVAL &&
      (!o.row_hi || !o.row_lo || !o.row_argmax || !o.row_argmin))
    return QSM_ERR_INVALID_ARG;
  if (mode == QSM_MODE_ROWMAX_POT && !o.row_hi) return QSM_ERR_INVALID_ARG;
  const size_t need = bwd_workspace_bytes(B, H, S, D);
  if (!o.workspace || o.workspace_bytes < need ||
      (reinterpret_cast<uintptr_t>(o.workspace) & 255u))
    return QSM_ERR_INVALID_ARG;
  BwdArgs a{};
  a.Q = Q; a.K = K; a.V = V; a.O = O; a.dO = dO; a.LSE = LSE;
  a.dQ = dQ; a.dK = dK; a.dV = dV;
  a.B = B; a.H = H; a.S = S; a.D = D; a.causal = causal;
  a.mode = mode; a.Kint = Kint; a.calib = calibration; a.rounding = rounding;
  a.surrogate = surrogate; a.detach = o.detach_extrema;
  a.c = c; a.window = o.window; a.below_policy = o.below_policy; a.pot_floor = o.pot_floor;
  a.fp8 = o.dtype == QSM_FP8_E4M3;
  a.scale = o.scale > 0.0f ? o.scale : 1.0f / std::sqrt(static_cast<float>(D));
  a.q_descale = o.q_descale; a.k_descale = o.k_descale; a.v_descale = o.v_descale;
  a.row_hi = o.row_hi; a.row_lo = o.row_lo;
  a.row_argmax = o.row_argmax; a.row_argmin = o.row_argmin;
  a.workspace = o.workspace; a.workspace_bytes = o.workspace_bytes;
  a.status_dev = o.status_dev;
  a.stream = reinterpret_cast<cudaStream_t>(stream);
  return launch_bwd(a);
}

size_t qsm_attn_bwd_workspace_size(int B, int H, int S, int D) {
  if (B < 1 || H < 1 || S < 1 || (D != 64 && D != 128)) return 0;
  return bwd_workspace_bytes(B, H, S, D);
}

qsm_status qsm_weight_map(const float *scores, const int32_t *valid_len, int rows, int cols,
                          qsm_mode mode, int Kint, qsm_calib calibration, qsm_rounding rounding,
                          const qsm_opts *opts, float *w, int32_t *idx, float *hi, float *lo,
                          qsm_stream_t stream) {
  const qsm_opts o = opts ? *opts : defaults();
  if (!scores || !valid_len || !w) return QSM_ERR_INVALID_ARG;
  if (rows < 1 || cols < 1) return QSM_ERR_INVALID_ARG;
  if (mode < QSM_MODE_EXACT || mode > QSM_MODE_UNIFORM) return QSM_ERR_INVALID_ARG;
  if (calibration != QSM_CALIB_MINMAX && calibration != QSM_CALIB_FIXED_WINDOW)
    return QSM_ERR_INVALID_ARG;
  if (!(o.support >= 0.0f) || !std::isfinite(o.support)) return QSM_ERR_INVALID_ARG;
  if (rounding != QSM_ROUND_INTERP && rounding != QSM_ROUND_HARD) return QSM_ERR_INVALID_ARG;
  if (mode == QSM_MODE_KINTERVAL && (Kint < 1 || Kint > 64)) return QSM_ERR_INVALID_ARG;
  if (!finite_pos(o.window) || o.pot_floor < 0 || o.pot_floor > 126) return QSM_ERR_INVALID_ARG;
  if (o.below_policy != 0 && o.below_policy != 1) return QSM_ERR_INVALID_ARG;
  if (!(o.scale == 0.0f || finite_pos(o.scale))) return QSM_ERR_INVALID_ARG;
  if (!finite_pos(o.q_descale) || !finite_pos(o.k_descale)) return QSM_ERR_INVALID_ARG;
  // the score scale folded into the map, formed as the forward forms it
  const float c = (o.scale > 0.0f ? o.scale : 1.0f) * o.q_descale * o.k_descale;
  if (!finite_pos(c)) return QSM_ERR_INVALID_ARG;
  MapArgs a{};
  a.scores = scores; a.c = c; a.valid_len = valid_len; a.rows = rows; a.cols = cols;
  a.mode = mode; a.Kint = Kint; a.calib = calibration; a.rounding = rounding;
  a.window = o.window; a.pot_floor = o.pot_floor; a.below_policy = o.below_policy;
  a.support = o.support;
  a.w = w; a.idx = idx; a.hi = hi; a.lo = lo;
  a.stream = reinterpret_cast<cudaStream_t>(stream);
  return launch_weight_map(a);
}

}  // extern "C"
