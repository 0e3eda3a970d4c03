/*
 * qsm.h -- C ABI of the approximate-softmax fused attention library for
 * NVIDIA B200 (sm_100a).  Library: libqsm.so.
 *
 * The operation ("Approximating Softmax in Pretrained LLMs: Model Sensitivity
 * and Kernel Acceleration", arXiv 2609.33586, abstract and the wiki page's
 * tile-loop flowchart; "Pretraining Transformers with Quantized Softmax in
 * Attention", arXiv 2609.33591, abstract):
 *
 *   for each (b, h) and query row r, over the valid keys j (all j, or j <= r
 *   when causal):  s_j = c * (q_r . k_j),  c = scale * q_descale * k_descale
 *   w_j = F_mode(s_j; row statistics)         -- the per-row weight map
 *   O_r = (sum_j w_j v_j) / (sum_j w_j) * v_descale,   LSE_r = hi + ln sum_j w_j
 *
 * where F is exact softmax (exp(s - hi)), K-interval attention (exp read off
 * K+1 grid values calibrated per row, by interpolation or hard rounding) or
 * Rowmax-PoT (power-of-two weights anchored at the row maximum).  The precise
 * readings of the maps are stated at qsm_mode / qsm_calib / qsm_rounding.
 *
 * Conventions shared by every entry point
 *   - Pointers named as device pointers are caller-owned device memory; the
 *     library never frees them and keeps no reference after the call returns.
 *   - Tensors are contiguous, row-major [B, H, S, D] (Q, K, V, O, dO, dQ, dK,
 *     dV) or [B, H, S] (LSE and row statistics).  Device pointers must be
 *     16-byte aligned.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream).  Argument errors are detected on the host before any
 *     launch, and then nothing is written.  No C++ exception crosses the ABI.
 *   - A CUDA launch error returns QSM_ERR_CUDA.  Device-side waits are
 *     bounded (about one second); a wait that runs out writes QSM_ERR_TIMEOUT
 *     into opts->status_dev (if given) and the kernel returns without
 *     trapping, leaving the CUDA context usable.
 */
#ifndef QSM_H_
#define QSM_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
typedef struct CUstream_st *qsm_stream_t;   /* same type as cudaStream_t */

typedef enum {
  QSM_OK = 0,
  QSM_ERR_INVALID_ARG = 1,   /* bad pointer, size, enum or option value      */
  QSM_ERR_UNSUPPORTED = 2,   /* valid request this build does not implement  */
  QSM_ERR_CUDA = 3,          /* a CUDA runtime / driver call failed          */
  QSM_ERR_TIMEOUT = 4        /* a bounded device-side wait ran out           */
} qsm_status;

/* The weight map.
 *  EXACT:      w = exp(s - hi), i.e. softmax (the pages' reference path, the
 *              "old path" through the special-function unit in the wiki
 *              flowchart).  Evaluated in two sweeps like the other maps: a
 *              statistics sweep finds the row maximum, then the weights are
 *              taken against it (no rescaling of O).
 *  KINTERVAL:  "approximates the exponential using K+1 grid values" (arXiv
 *              2609.33591, abstract).  Grid over [lo, hi] of the row's scores,
 *              step Delta = (hi - lo)/K, grid values g_k = exp(-(K-k) Delta);
 *              coordinate u = clamp((s - lo)/Delta, 0, K).
 *  ROWMAX_POT: "coarse logarithmic weight representation anchored at each row
 *              maximum" (arXiv 2609.33586, abstract): n = round((hi-s) log2 e),
 *              clamped to pot_floor, w = 2^-n; w = 1 exactly at the row max. */
typedef enum {
  QSM_MODE_EXACT = 0,
  QSM_MODE_KINTERVAL = 1,
  QSM_MODE_ROWMAX_POT = 2,
  /* The sensitivity probes of "Approximating Softmax in Pretrained LLMs"
   * (abstract: the number of positions can be cut substantially, yet uniform
   * weighting of them is damaging), read as maps on the same kernel: the kept
   * positions are the valid keys within opts->support of the row maximum
   * (s >= hi - support).  TRUNCATED: exp(s - hi) on them; UNIFORM: 1 on
   * them; 0 on every other key.  Forward only, anchored at the final row
   * maximum (two sweeps). */
  QSM_MODE_TRUNCATED = 3,
  QSM_MODE_UNIFORM = 4
} qsm_mode;

/* K-interval grid calibration ("per-row grid calibration", arXiv 2609.33591):
 *  MINMAX: lo = the row's minimum score.  FIXED_WINDOW: lo = hi - window. */
typedef enum { QSM_CALIB_MINMAX = 0, QSM_CALIB_FIXED_WINDOW = 1 } qsm_calib;

/* K-interval read-out ("interpolation versus hard rounding"):
 *  INTERP: linear interpolation between the two neighbouring grid values.
 *  HARD:   the grid value at the nearest node (round half to even). */
typedef enum { QSM_ROUND_INTERP = 0, QSM_ROUND_HARD = 1 } qsm_rounding;

/* Backward surrogate ("the placement of a straight-through surrogate relative
 * to normalization", arXiv 2609.33591):
 *  NONE: the exact gradient of the map with its rounding decisions frozen.
 *  PRE:  before normalization: the map's own-score derivative is replaced by
 *        that of exp(s - hi).
 *  POST: after normalization: the probabilities' own-score derivative is
 *        replaced by that of softmax(s).
 * Ignored by the forward (accepted so both calls share one argument list). */
typedef enum { QSM_SURR_NONE = 0, QSM_SURR_PRE = 1, QSM_SURR_POST = 2 } qsm_surrogate;

/* Element type of Q, K, V.  O, dO, dQ, dK, dV are always bf16. */
typedef enum { QSM_BF16 = 0, QSM_FP8_E4M3 = 1 } qsm_dtype;

/* Options; pass NULL for all defaults (qsm_opts_default fills them in). */
typedef struct {
  qsm_dtype dtype;        /* default QSM_BF16 */
  float scale;            /* score scale; <= 0 selects 1/sqrt(D) (default 0) */
  float q_descale, k_descale, v_descale;  /* FP8 per-tensor factors (default 1) */
  float window;           /* fixed-window width W in units of s (default 8) */
  int pot_floor;          /* PoT exponent floor N, 0..126 (default 15) */
  int below_policy;       /* 0: clamp to the lowest grid value / 2^-N (default);
                             1: flush such weights to 0 */
  int detach_extrema;     /* backward: 1 drops the calibration derivatives */
  /* Row statistics [B,H,S], optional in the forward (written when non-NULL)
   * and required by the K-interval backward.  hi = row max of s.  lo = hi -
   * window for fixed-window K-interval, else the row min of s.  argmax /
   * argmin = lowest key index of the row max / min.  Device pointers.  Every
   * map, the exact one included, runs the statistics sweep and writes each
   * of the four that is non-NULL. */
  float *row_hi, *row_lo;
  int32_t *row_argmax, *row_argmin;
  /* Backward scratch, at least qsm_attn_bwd_workspace_size() bytes, device,
   * 256-byte aligned; required by qsm_attn_bwd. */
  void *workspace;
  size_t workspace_bytes;
  int32_t *status_dev;    /* optional device word; a timeout writes QSM_ERR_TIMEOUT */
  int8_t *debug_idx;      /* optional [B,H,S,S] dump of the per-element decision:
                             grid node (hard), lower node (interp), PoT
                             exponent, 0 (exact); -1 masked, -2 flushed.
                             Key tiles wholly above the causal diagonal are
                             never visited and their entries are left as they
                             were. */
  int debug_flags;        /* test hooks, 0 in normal use; bit 0: the forward's
                             load warp issues no loads, so every consumer wait
                             runs out (exercises the timeout path) */
  int anchor;             /* where the maps are anchored (default 0):
                             0: at the row's final maximum (and minimum): a
                                statistics sweep, then the weights -- the maps
                                exactly as defined above;
                             1: at the row's running maximum after each key
                                tile of 128 keys, tiles in increasing key
                                order, in one sweep (the form a one-sweep
                                kernel such as the pages' FlashAttention-4
                                patch can take; "Rowmax-H15 in FlashAttention-4
                                on B200", wiki flowchart).  Earlier tiles are
                                carried over by 2^-rne((a_t - a_{t-1}) log2 e)
                                (Rowmax-PoT: every weight stays a power of two)
                                or exp(a_{t-1} - a_t) (exact: softmax, the
                                online softmax; K-interval: fixed-window
                                calibration only, QSM_ERR_UNSUPPORTED for
                                min-max).  Only row_hi / row_lo are written
                                (row_argmax / row_argmin must be NULL), and the
                                backward accepts it for the exact map only. */
  float support;          /* probes (TRUNCATED, UNIFORM): the support width T
                             in units of s, >= 0 (default 4) */
} qsm_opts;

/* Fill *opts with the defaults listed above. */
void qsm_opts_default(qsm_opts *opts);

/* Fused attention forward.
 *  Q, K, V: device [B,H,S,D], bf16 or e4m3 per opts->dtype.
 *  O:       device [B,H,S,D] bf16 (written).
 *  LSE:     device [B,H,S] fp32 (written), natural log, hi + ln(sum of w).
 *  B, H >= 1; 1 <= S <= 65536 (any S; ragged tails are masked); D in {64,128}
 *  (e4m3: D = 128).  causal: key j valid for row r iff j <= r.
 *  Kint: K of K-interval attention, 1..64 (checked for KINTERVAL only).
 *  Returns QSM_OK after enqueuing the kernel on `stream`. */
qsm_status qsm_attn_fwd(const void *Q, const void *K, const void *V, void *O, float *LSE,
                        int B, int H, int S, int D, int causal, qsm_mode mode, int Kint,
                        qsm_calib calibration, qsm_rounding rounding,
                        qsm_surrogate surrogate, const qsm_opts *opts, qsm_stream_t stream);

/* Backward of qsm_attn_fwd (D = 64 or 128): the exact map, K-interval
 * attention (K <= 32) and Rowmax-PoT.
 *  Q, K, V: device [B,H,S,D] as given to the forward: bf16, or (D = 128)
 *        e4m3 with the forward's opts->q_descale/k_descale/v_descale.
 *  O, dO: device [B,H,S,D] bf16 (O = the forward's output).
 *  LSE:  device [B,H,S] fp32 from the forward.
 *  dQ, dK, dV: device [B,H,S,D] bf16 (written): the gradients with respect
 *        to the tensors the forward's scores and output are formed from --
 *        Q, K, V for bf16; q_descale Q, k_descale K, v_descale V for e4m3,
 *        whose codes are copied to bf16 in the workspace (Q and K exactly, so
 *        the recomputed scores are the forward's; V times v_descale, rounded
 *        to bf16) before the bf16 passes run.
 *  The rules are the exact gradients of the surrogate graphs with the
 *  forward's rounding decisions frozen (see qsm_surrogate).  Rowmax-PoT's
 *  backward is not derived on the pages; the same surrogates apply to it,
 *  and with its exponents frozen a power-of-two weight has no derivative of
 *  its own, nor a calibration term (QSM_SURR_NONE gives dQ = dK = 0).
 *  K-interval needs opts->row_hi/row_lo/row_argmax/row_argmin from the
 *  forward, Rowmax-PoT opts->row_hi; all need opts->workspace.  e4m3 at
 *  D = 64 and K > 32 return QSM_ERR_UNSUPPORTED. */
qsm_status qsm_attn_bwd(const void *Q, const void *K, const void *V, const void *O,
                        const void *dO, const float *LSE, void *dQ, void *dK, void *dV,
                        int B, int H, int S, int D, int causal, qsm_mode mode, int Kint,
                        qsm_calib calibration, qsm_rounding rounding,
                        qsm_surrogate surrogate, const qsm_opts *opts, qsm_stream_t stream);

/* Bytes of opts->workspace that qsm_attn_bwd needs for this shape (at
 * D = 128 including room for bf16 copies of e4m3 Q, K, V). */
size_t qsm_attn_bwd_workspace_size(int B, int H, int S, int D);

/* Size of the library's own backward scratch array (16 MiB). */
#define QSM_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)

/* qsm_attn_bwd without a caller-provided workspace.  (The papers have no
 * counterpart: this is a convenience of the library.)
 *
 * For callers that cannot allocate device memory at the time of the call,
 * such as a plugin whose host framework owns every device allocation through
 * its own pool, or a latency-critical loop that cannot take cudaMalloc's
 * implicit synchronisation.  The backward's scratch comes instead from one
 * static device array of QSM_NOALLOC_SCRATCH_BYTES bytes inside the library,
 * which every GPU that loads the library holds until the process exits.  This
 * call allocates and frees nothing.
 *
 * Arguments and results are those of qsm_attn_bwd; opts->workspace and
 * opts->workspace_bytes are ignored.  Returns QSM_ERR_INVALID_ARG when
 * qsm_attn_bwd_workspace_size(B, H, S, D) exceeds QSM_NOALLOC_SCRATCH_BYTES
 * (for D = 64, about 14 700 query rows B*H*S), before any launch.
 *
 * The first call on each device looks up the array's device address (with
 * that device current); make that first call before any stream capture.  The
 * address is kept for the driver context current at that first call; a call
 * under another context (after cudaDeviceReset, or with a non-primary
 * context current) looks it up again, so make such a call before any capture
 * as well.  Every call uses the same array, so calls whose work overlaps on a
 * GPU (different streams or host threads) race; serialise them.  D outside
 * {64, 128} returns QSM_ERR_UNSUPPORTED, as qsm_attn_bwd does. */
qsm_status qsm_attn_bwd_noalloc(const void *Q, const void *K, const void *V, const void *O,
                                const void *dO, const float *LSE, void *dQ, void *dK, void *dV,
                                int B, int H, int S, int D, int causal, qsm_mode mode, int Kint,
                                qsm_calib calibration, qsm_rounding rounding,
                                qsm_surrogate surrogate, const qsm_opts *opts,
                                qsm_stream_t stream);

/* The weight map alone, on given fp32 raw products, through the fused
 * forward's own per-element map code (row set-up, grid table, pair
 * arithmetic, decision index): the bit-exact window onto the forward's
 * weights.  The score of a product r is s = c * r with
 * c = (opts->scale, or 1 when opts->scale is 0) * q_descale * k_descale,
 * folded into one fused multiply-add exactly as the forward folds it.
 * The exact map's 2^x is the hardware's approximate instruction (not
 * bit-reproducible elsewhere); the other maps are.
 *  scores:    device [rows, cols] fp32 raw products r.
 *  valid_len: device [rows] int32; keys 0..valid_len[r]-1 of row r are valid
 *             (1 <= valid_len[r] <= cols).
 *  w:         device [rows, cols] fp32 (written; 0 where masked).
 *  idx:       device [rows, cols] int32 (written; decision index as in
 *             opts->debug_idx), may be NULL.
 *  hi, lo:    device [rows] fp32 (written: c * row max of r; calibrated lower
 *             end for K-interval, c * row min otherwise), may be NULL.  A NaN
 *             among a row's valid products makes both NaN.
 *  Uses opts->scale, q_descale, k_descale, window, pot_floor, below_policy. */
qsm_status qsm_weight_map(const float *scores, const int32_t *valid_len, int rows, int cols,
                          qsm_mode mode, int Kint, qsm_calib calibration,
                          qsm_rounding rounding, const qsm_opts *opts, float *w,
                          int32_t *idx, float *hi, float *lo, qsm_stream_t stream);

/* Static description of a status code (never NULL). */
const char *qsm_status_string(qsm_status status);

/* Library version, e.g. "0.1.0". */
const char *qsm_version(void);

#ifdef __cplusplus
}
#endif

#endif /* QSM_H_ */
