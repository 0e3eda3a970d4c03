/*
 * fp32 weight-map specification, restated in plain C.
 *
 * TEST INFRASTRUCTURE ONLY: only tests/ (through oracle/spec.py) load this.
 * It shares no code with the CUDA path; the GPU map (the fused forward's own
 * per-element arithmetic, exposed as qsm_weight_map) must reproduce its
 * output bit for bit on the same fp32 inputs.
 *
 * Compile with -O2 -ffp-contract=off and without -ffast-math: every a*b+c
 * below is two correctly rounded operations unless written as fmaf().
 *
 * The maps are the ones named on the pages ("Pretraining Transformers with
 * Quantized Softmax in Attention", abstract: K-interval attention with K+1 grid
 * values, per-row calibration, interpolation vs hard rounding; "Approximating
 * Softmax in Pretrained LLMs", abstract: Rowmax-PoT, power-of-two weights
 * anchored at the row maximum).  The fp32 operation order is this library's
 * own specification (the pages fix none).  Inputs are raw products r = q.k;
 * the score is s = c*r with the scale c folded into one fused multiply-add:
 *
 *   rmax, rmin = max / min of r over the valid keys (a NaN propagates)
 *   hi = c*rmax, lo_obs = c*rmin, cl2e = c*L2E
 *   EXACT      x = fmaf(r, cl2e, -(rmax*cl2e)); w = 2^x  (the GPU evaluates
 *              2^x with its approximate hardware instruction, so for EXACT
 *              this file returns x, not w)
 *   ROWMAX_POT x = fmaf(r, -cl2e, hi*L2E); n = rne(min(x, cap)) with
 *              cap = N (clamp) or N+1 (flush, n > N gives w = 0);
 *              w = 2^-n built from exponent bits
 *   KINTERVAL  lc = lo_obs (min-max) or hi - W (fixed-window); a = hi - lc;
 *              degenerate when !(a > 0): coordinate x = K for every key;
 *              else inv = K/a, b = -(lc*inv), x = fmaf(r, c*inv, b);
 *              flushed when below_policy == 1, fixed-window and x < 0;
 *              uc = min(max(x, 0), K);
 *              step = a/K (min-max) or W/K (fixed-window),
 *              g[k] = spec_exp(-(K-k) * step);
 *              hard   n = rne(uc), w = g[n]
 *              interp k = floor(uc) (0..K); the table entry of node k holds
 *                     d = g[k'+1] - g[k'] and e = fmaf(-k', d, g[k']) with
 *                     k' = min(k, K-1); w = fmaf(uc, d, e); the decision
 *                     index reported is k'
 *   TRUNCATED  x as for EXACT; kept when x >= thr, thr = -(T*L2E) (T the
 *              support width); returns x for a kept key and -inf otherwise
 *   UNIFORM    the same kept test; w = 1 kept, 0 otherwise
 *   rne(x) = (x + 1.5*2^23) - 1.5*2^23  (round half to even, |x| < 2^22)
 *
 *   spec_exp(x): Cody-Waite reduction x = n*ln2 + r with n = rne(x*log2 e),
 *   ln2 split into a 16-bit head and a tail; e^r by the degree-7 Taylor
 *   polynomial (coefficients 1/k! rounded to fp32) in Horner form with fmaf;
 *   scaled by 2^n through the exponent bits; 0 when n < -125.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define MODE_EXACT 0
#define MODE_KINTERVAL 1
#define MODE_POT 2
#define MODE_TRUNC 3
#define MODE_UNIFORM 4
#define CAL_MINMAX 0
#define CAL_FIXED 1
#define RND_INTERP 0
#define RND_HARD 1

static const float MAGIC = 12582912.0f;          /* 1.5 * 2^23 */
static const float L2E = 1.44269502162933349609375f;   /* fp32(log2 e) */
static const float LN2_HEAD = 0.693145751953125f;      /* ln 2, 16 bits */
static const float LN2_TAIL = 1.428606765330187e-06f;  /* ln 2 - head   */

static float bits2f(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t f2bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

static float rne(float x) { float t = x + MAGIC; return t - MAGIC; }

float spec_exp(float x) {
    float n = rne(x * L2E);
    if (n < -125.0f) return 0.0f;
    float r = fmaf(n, -LN2_HEAD, x);
    r = fmaf(n, -LN2_TAIL, r);
    float p = 1.98412701138295233249664306640625e-4f;  /* 1/7! */
    p = fmaf(p, r, 1.38888892251998186111450195312500e-3f); /* 1/6! */
    p = fmaf(p, r, 8.33333376795053482055664062500000e-3f); /* 1/5! */
    p = fmaf(p, r, 4.16666679084300994873046875000000e-2f); /* 1/4! */
    p = fmaf(p, r, 1.66666671633720397949218750000000e-1f); /* 1/3! */
    p = fmaf(p, r, 0.5f);
    p = fmaf(p, r, 1.0f);
    p = fmaf(p, r, 1.0f);
    int32_t e = (int32_t)n;                  /* exact: n is integral */
    return p * bits2f((uint32_t)(e + 127) << 23);
}

/* NaN-propagating maximum / minimum (a NaN operand gives NaN). */
static float nmax(float a, float b) { return (a != a || b != b) ? NAN : (b > a ? b : a); }
static float nmin(float a, float b) { return (a != a || b != b) ? NAN : (b < a ? b : a); }

/*
 * Map `rows` rows of `cols` raw products with score scale c.  valid_len[r]
 * keys (a prefix) are valid in row r.  Outputs w [rows*cols] (0 where masked;
 * for EXACT the exponent x of 2^x, see above) and idx [rows*cols] (node /
 * lower node / exponent; -1 masked, -2 flushed), and the per-row hi = c*rmax
 * and lo (the calibrated lower end for K-interval, c*rmin otherwise).
 */
void spec_map_rows(const float *rin, int rows, int cols, const int *valid_len, float c,
                   int mode, int K, int calib, int rounding, float window,
                   int pot_floor, int below_policy, float support, float *w, int *idx,
                   float *hi_out, float *lo_out) {
    float g[130];
    float cl2e = c * L2E;
    for (int r = 0; r < rows; ++r) {
        const float *rr = rin + (size_t)r * cols;
        float *wr = w + (size_t)r * cols;
        int *ir = idx + (size_t)r * cols;
        int L = valid_len[r];
        float rmax = -INFINITY, rmin = INFINITY;
        for (int j = 0; j < L; ++j) { rmax = nmax(rmax, rr[j]); rmin = nmin(rmin, rr[j]); }
        float hi = c * rmax, lo = c * rmin;
        for (int j = L; j < cols; ++j) { wr[j] = 0.0f; ir[j] = -1; }
        if (mode == MODE_EXACT) {
            float m = rmax * cl2e;
            for (int j = 0; j < L; ++j) { wr[j] = fmaf(rr[j], cl2e, -m); ir[j] = 0; }
        } else if (mode == MODE_TRUNC || mode == MODE_UNIFORM) {
            float m = rmax * cl2e;
            float thr = -(support * L2E);
            for (int j = 0; j < L; ++j) {
                float x = fmaf(rr[j], cl2e, -m);
                int kept = x >= thr;
                if (mode == MODE_TRUNC) wr[j] = kept ? x : -INFINITY;
                else wr[j] = kept ? 1.0f : 0.0f;
                ir[j] = kept ? 0 : -2;
            }
        } else if (mode == MODE_POT) {
            float b = hi * L2E;
            float cap = below_policy ? (float)(pot_floor + 1) : (float)pot_floor;
            for (int j = 0; j < L; ++j) {
                float x = fmaf(rr[j], -cl2e, b);
                float t = fminf(x, cap) + MAGIC;
                int32_t n = (int32_t)f2bits(t) - (int32_t)f2bits(MAGIC);
                if (below_policy && n > pot_floor) { wr[j] = 0.0f; ir[j] = -2; continue; }
                wr[j] = bits2f((uint32_t)(127 - n) << 23);
                ir[j] = n;
            }
        } else {
            float lc = (calib == CAL_MINMAX) ? lo : hi - window;
            float a = hi - lc;
            int degenerate = !(a > 0.0f);
            float Kf = (float)K;
            float step = (calib == CAL_MINMAX) ? a / Kf : window / Kf;
            for (int k = 0; k <= K; ++k) g[k] = spec_exp(-(float)(K - k) * step);
            float inv = degenerate ? 0.0f : Kf / a;
            float b = -(lc * inv);
            float ca = c * inv;
            if (degenerate) { ca = 0.0f; b = Kf; }
            lo = lc;
            for (int j = 0; j < L; ++j) {
                float x = fmaf(rr[j], ca, b);
                if (below_policy == 1 && calib == CAL_FIXED && x < 0.0f) {
                    wr[j] = 0.0f; ir[j] = -2; continue;
                }
                float uc = fminf(fmaxf(x, 0.0f), Kf);
                if (rounding == RND_HARD) {
                    int32_t n = (int32_t)f2bits(uc + MAGIC) - (int32_t)f2bits(MAGIC);
                    wr[j] = g[n];
                    ir[j] = n;
                } else {
                    int k = (int)floorf(uc);
                    if (k > K - 1) k = K - 1;
                    float d = g[k + 1] - g[k];
                    float e = fmaf(-(float)k, d, g[k]);
                    wr[j] = fmaf(uc, d, e);
                    ir[j] = k;
                }
            }
        }
        hi_out[r] = hi;
        lo_out[r] = lo;
    }
}

/* Vector form of spec_exp, for the accuracy pins. */
void spec_exp_vec(const float *x, float *y, int n) {
    for (int i = 0; i < n; ++i) y[i] = spec_exp(x[i]);
}
