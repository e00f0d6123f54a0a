/*
 * fp4q_oracle.c -- plain, slow, single-threaded CPU oracle for block-scaled FP4
 * quantization (NVFP4 AbsMax / 4-over-6 / ScaleSweep MSE and WMSE, IF4, MXFP4 with an
 * optional block Hadamard, and dequantization), and its element codec.  Parity unpinned
 * against the pages for end-to-end MSE values (they print no worked numbers); every function
 * is pinned by the tests to exact rationals, brute force, closed forms or hand-worked blocks.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test-suite, the smoke check and the benchmark's
 * CPU-baseline leg may load this library.  It shares no code with the CUDA path: it has
 * its own codec, its own scale rules and its own error arithmetic, written from the
 * method descriptions:
 *   [SS]  ScaleSweep (gist.science/ko/paper/2606.07618), "Methodology: ScaleSweep":
 *         global scale S = max|x|/(256*6); per-block base scale = the FP8 (E4M3) rounding
 *         of the block maximum over 6 in units of S; candidate scales at FP8 bit-pattern
 *         offsets [-3,+7] (MSE) or [-8,+7] (WMSE); 126 positive finite E4M3 values;
 *         objectives MSE and importance-weighted MSE.
 *   [IF4] Adaptive Block-Scaled Data Types (gist.science/ko/paper/2603.28765),
 *         "Methodology", IF4 structure: one E4M3 scale per 16 values, per-group choice
 *         between FP4 and scaled INT4 by lower MSE, indicator in the scale's unused sign
 *         bit (0 = FP4, 1 = INT4), INT4 pre-scaled by 7/6 and dequantized by 6/7.
 *   [46]  same page, "Problem": Four-over-Six picks per block between max->6 and max->4.
 *   [MR]  Bridging the Gap ... Microscaling FP4 (gist.science/ko/paper/2509.23202),
 *         "Methodology": MXFP4 = 32-element blocks with power-of-two (E8M0) scales;
 *         block-wise Hadamard rotation before quantization.
 *   [TQ]  TORQ (gist.science/ko/paper/2605.19561), "Method", S-step: the block scale maps
 *         the block maximum onto the largest codeword.
 * The E2M1 value set {0,.5,1,1.5,2,3,4,6}, round-to-nearest-even with saturation, and the
 * "lowest offset wins a tie" rule are fixed by the workload specification that
 * accompanies the pages.
 *
 * Arithmetic (the readings where the pages are silent).  RN is one IEEE-754 binary32
 * operation rounded to nearest even; no contraction, no flush-to-zero.
 *   S      = RN(amax / 1536)                      (amax = max |x| over the tensor)
 *   p0     = E4M3(RN(a_b / RN(6*S)))               (a_b = max |x| over the block)
 *   p4     = E4M3(RN(a_b / RN(4*S)))               (4/6 only)
 *   sv(p)  = RN(e(p) * S), inv(p) = RN(1 / sv(p)); sv(0) = inv(0) = 0   (the block scale the
 *            quantizer holds in binary32, and its reciprocal)
 *   codes  : FP4  q = E2M1(RN(x * inv));  INT4 n = clamp(rint(RN(RN(x * inv) * RN(7/6))), -7, 7);
 *            MXFP4 q = E2M1(RN(x * 2^-e))
 *   reconstruction (exact real products): FP4 xhat = q * sv; INT4 xhat = n * g with
 *            g = RN(RN(6/7) * sv), the INT4 block's scale (the 6/7 dequantization folded into the
 *            block scale, held in binary32 like every scale); MXFP4 xhat = q * 2^e
 *   MSE objective (AbsMax has none; 4/6, the MSE sweep, IF4, the IF4 sweep, the MX sweep):
 *            the block's squared reconstruction error E = sum_i (x_i - xhat_i)^2, compared
 *            EXACTLY (no rounding anywhere in the comparison; see exact_F below).  Ties go to
 *            the lowest offset (4/6: the max->6 scale; IF4: FP4; the IF4 sweep: lowest offset,
 *            then FP4; the MX sweep: the lowest exponent).
 *   WMSE objective (importance-weighted; exact sums are out of reach with arbitrary weights, so
 *            binary32 with one accumulator per candidate, in element order):
 *            xhat = RN(q * sv), d = RN(x - xhat), acc = fma(RN(w * d), d, acc) for i = 0..15;
 *            argmin (acc, offset) lexicographic; NaN never wins; if every acc is +inf the first
 *            candidate is kept.
 *   MXFP4  = e = smallest integer with a_b <= 6*2^e (clamped to [-127,127]), byte e+127.
 *   MX sweep = e among e_c - 2 .. e_c (e_c the rule above, none below -127), exact MSE.
 *   Hadamard(32) = Sylvester fast Walsh-Hadamard butterflies for h = 1,2,4,8,16
 *            (v_j, v_j+h) <- (RN(v_j + v_j+h), RN(v_j - v_j+h)), then RN(v * RN(1/sqrt(32))).
 *   dequant NVFP4 x^ = RN(q * sv); IF4-INT4 x^ = RN(n * RN(RN(6/7) * sv)); MXFP4 x^ = RN(q*2^e)
 *            (the binary32 output is the rounding of the objective's exact reconstruction).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#include <float.h>
#include <stdlib.h>

#define ST_OK 0
#define ST_NONFINITE 1
#define ST_RANGE 2

/* ------------------------------------------------------------------------------------
 * Codec
 * ---------------------------------------------------------------------------------- */

/* E4M3FN value of bit pattern p (sign bit ignored): 4 exponent bits (bias 7), 3 mantissa
 * bits, subnormals below 2^-6, no infinities, 0x7F = NaN.  [SS]: 126 positive finite
 * values, i.e. patterns 0x01..0x7E. */
double fp4q_o_e4m3_value(int p)
{
    p &= 0x7F;
    int E = p >> 3, M = p & 7;
    if (p == 0x7F) return NAN;
    if (E == 0) return ldexp((double)M, -9);
    return ldexp(1.0 + M / 8.0, E - 7);
}

/* Round a finite v >= 0 to the nearest E4M3FN pattern; ties go to the even pattern;
 * values beyond the largest finite value (448) saturate to 0x7E. */
int fp4q_o_e4m3_encode(float v)
{
    double dv = (double)v;  /* exact */
    if (dv >= 448.0) return 0x7E;
    int best = 0;
    double bestd = dv;  /* distance to pattern 0 (value 0) */
    for (int p = 1; p <= 0x7E; ++p) {
        double d = fabs(dv - fp4q_o_e4m3_value(p)); /* exact: both have <= 24 bits, close */
        if (d < bestd || (d == bestd && (p & 1) == 0 && (best & 1) == 1)) { best = p; bestd = d; }
    }
    return best;
}

static const float E2M1_MAG[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};

/* E2M1 value of a 4-bit code: bit 3 = sign, bits 0..2 = index into the magnitude set. */
float fp4q_o_e2m1_value(int code)
{
    float m = E2M1_MAG[code & 7];
    return (code & 8) ? -m : m;
}

/* Round-to-nearest-even onto the E2M1 grid with saturation at 6, keeping the sign
 * (so -0 and small negatives give 0x8).  Ties go to the even code index. */
int fp4q_o_e2m1_encode(float y)
{
    int s = signbit(y) ? 8 : 0;
    float a = fabsf(y);
    int k;
    if (a <= 0.25f) k = 0;        /* tie at 0.25 -> 0 (index 0 even)   */
    else if (a < 0.75f) k = 1;    /* tie at 0.75 -> 1.0 (index 2)       */
    else if (a <= 1.25f) k = 2;   /* tie at 1.25 -> 1.0 (index 2)       */
    else if (a < 1.75f) k = 3;    /* tie at 1.75 -> 2.0 (index 4)       */
    else if (a <= 2.5f) k = 4;    /* tie at 2.5  -> 2.0 (index 4)       */
    else if (a < 3.5f) k = 5;     /* tie at 3.5  -> 4.0 (index 6)       */
    else if (a <= 5.0f) k = 6;    /* tie at 5    -> 4.0 (index 6)       */
    else k = 7;                   /* above 5 -> 6, saturating            */
    return s | k;
}

/* Batch codec over n values (the reference the hardware conversions are checked against).
 * kind 0: fp4q_o_e2m1_encode of each value.  kind 1: E4M3FN byte, sign in bit 7, magnitude
 * rounded to the nearest of the 127 values 0 .. 448 with ties to the even pattern and
 * saturation at 448 (infinities included); NaN gives 0x7F.  The magnitude's pattern is found by
 * bisection over the increasing value table (the values of fp4q_o_e4m3_value), then the nearer
 * of the two bracketing patterns is taken; this equals fp4q_o_e4m3_encode, which scans all
 * patterns (a pin checks the two against each other). */
int fp4q_o_encode(const float* x, int64_t n, int kind, uint8_t* out)
{
    if (kind == 0) {
        for (int64_t i = 0; i < n; ++i) out[i] = (uint8_t)fp4q_o_e2m1_encode(x[i]);
        return ST_OK;
    }
    if (kind != 1) return -1;
    double tab[127];
    for (int p = 0; p <= 0x7E; ++p) tab[p] = fp4q_o_e4m3_value(p);
    for (int64_t i = 0; i < n; ++i) {
        const float v = x[i];
        const int s = signbit(v) ? 0x80 : 0;
        if (isnan(v)) { out[i] = (uint8_t)(s | 0x7F); continue; }
        const double a = fabs((double)v);
        if (a >= 448.0) { out[i] = (uint8_t)(s | 0x7E); continue; }
        int lo = 0, hi = 0x7E;          /* tab[lo] <= a < tab[hi] */
        while (hi - lo > 1) {
            const int mid = (lo + hi) / 2;
            if (tab[mid] <= a) lo = mid; else hi = mid;
        }
        const double dl = a - tab[lo], dh = tab[hi] - a;
        const int p = dl < dh ? lo : (dh < dl ? hi : ((lo & 1) == 0 ? lo : hi));
        out[i] = (uint8_t)(s | p);
    }
    return ST_OK;
}

/* ------------------------------------------------------------------------------------
 * Global scale  [SS] S = max|x|/(256*6)
 * ---------------------------------------------------------------------------------- */

/* Max |x| over rows x cols (row stride ld); returns ST_NONFINITE if any element is NaN/Inf. */
static int tensor_amax(const float* x, int64_t rows, int64_t cols, int64_t ld, float* amax)
{
    float m = 0.0f;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c) {
            float v = x[r * ld + c];
            if (!isfinite(v)) { *amax = NAN; return ST_NONFINITE; }
            float a = fabsf(v);
            if (a > m) m = a;
        }
    *amax = m;
    return ST_OK;
}

float fp4q_o_global_scale(float amax) { return amax / 1536.0f; }

/* S must keep every candidate scale normal and every reciprocal finite. */
static int scale_range_ok(float S)
{
    if (S == 0.0f) return 1;
    return S >= ldexpf(1.0f, -117) && S <= ldexpf(1.0f, 125) / 1536.0f;
}

/* S of a whole tensor (status ST_NONFINITE if any element is not finite). */
int fp4q_o_tensor_scale(const float* x, int64_t rows, int64_t cols, int64_t ld, float* S)
{
    float amax;
    int st = tensor_amax(x, rows, cols, ld, &amax);
    *S = st == ST_OK ? fp4q_o_global_scale(amax) : NAN;
    if (st == ST_OK && !scale_range_ok(*S)) st = ST_RANGE;
    return st;
}


/* ------------------------------------------------------------------------------------
 * Exact block errors
 * ---------------------------------------------------------------------------------- */

/* long double carries at least 64 significand bits on the hosts this runs on (x86-64 extended
 * precision, or binary128); every exactness bound below relies on it. */
_Static_assert(LDBL_MANT_DIG >= 64, "the exact block errors need a 64-bit long double significand");

/* The block error of one candidate relative to the block energy, held exactly:
 *   E = sum_i (|x_i| - m_i g)^2 = sum_i x_i^2 + F,   F = g (g Q - 2 X),
 * with m_i >= 0 the magnitude of element i's code (FP4: E2M1 value; INT4: |n|; MX: E2M1 value),
 * g the grid step (FP4: sv; INT4: RN(RN(6/7) * sv); MX: 2^e), Q = sum m_i^2, X = sum |x_i| m_i.
 * sum x_i^2 is the same for every candidate of a block, so candidates are ordered by F.
 * Why no step rounds (x_i binary32, so |x_i| = M 2^E with M < 2^24):
 *  - an element with m_i > 0 has |x_i| >= g/4 (its quotient reached the first rounding
 *    threshold: 0.25 for E2M1, 0.5 for INT4 before the 7/6 pre-scale), so every term |x_i| m_i
 *    (exact: 24 + 3 bits) is a multiple of 2^(floor(log2 g) - 27); within the windows the block
 *    maximum is at most 27 g (the worst case is p0 = 4 with offset -3 to pattern 1), so X < 2^13 g
 *    and spans at most 41 bit positions: an exact long double sum (the brute-force modes reach
 *    max|x| <= 2^20 g, still under 64 positions for FP4); Q is a multiple of 1/4 below 2^10;
 *  - g Q is exact (g is a binary32 value, Q has at most 12 bits), and u = g Q - 2 X spans at
 *    most 44 bit positions in the windows (58 in the FP4 brute force), so it is exact too;
 *  - F = g u is kept as hi + lo with hi = RN(g u) and lo = fma(g, u, -hi), the exact remainder.
 * Comparing (hi, lo) lexicographically therefore compares the exact block errors. */
typedef struct { long double hi, lo; int exact; } exact_F;

/* Candidates compared with an inexact F (possible only in the brute-force window checks, for
 * scales far below the block's, where X outgrows the span bound) are decided on hi alone; if
 * two such values come within 2^-56 of each other the oracle cannot decide and counts it here
 * (the bindings raise).  Every window mode is exact by the bounds above, which this also checks. */
static long g_undecided = 0, g_inexact = 0;
long fp4q_o_undecided(void) { long n = g_undecided; g_undecided = 0; return n; }
long fp4q_o_inexact(void) { long n = g_inexact; g_inexact = 0; return n; }

/* s = RN(a + b) is exactly a + b (Knuth's TwoSum remainder is zero). */
static int sum_is_exact(long double a, long double b, long double s)
{
    const long double bb = s - a;
    return ((a - (s - bb)) + (b - bb)) == 0.0L;
}

static exact_F block_F(const float* x, int B, const float* m, long double g)
{
    long double Q = 0.0L, X = 0.0L;
    int exact = 1;
    for (int i = 0; i < B; ++i) {
        if (m[i] == 0.0f) continue;
        Q += (long double)m[i] * (long double)m[i];
        const long double t = fabsl((long double)x[i]) * (long double)m[i], s = X + t;
        exact &= sum_is_exact(X, t, s);
        X = s;
    }
    const long double p = g * Q;
    exact &= fmal(g, Q, -p) == 0.0L;
    const long double u = p - 2.0L * X;
    exact &= sum_is_exact(p, -2.0L * X, u);
    exact_F f;
    f.hi = g * u;
    f.lo = fmal(g, u, -f.hi);
    f.exact = exact;
    if (!exact) ++g_inexact;
    return f;
}

static int F_less(exact_F a, exact_F b)
{
    if (a.exact && b.exact) return a.hi < b.hi || (a.hi == b.hi && a.lo < b.lo);
    const long double m = fmaxl(fabsl(a.hi), fabsl(b.hi));
    if (fabsl(a.hi - b.hi) <= ldexpl(m, -56)) ++g_undecided;
    return a.hi < b.hi;
}
static int F_equal(exact_F a, exact_F b) { return a.exact && b.exact && a.hi == b.hi && a.lo == b.lo; }
/* (b - a) as a long double (accurate to the last bits; used only for reporting). */
static long double F_diff(exact_F a, exact_F b) { return (b.hi - a.hi) + (b.lo - a.lo); }

/* The block error E itself, for reporting: the sum of the squared differences, each difference
 * exact in long double (it spans fewer than 64 bit positions), the squares rounded to 64 bits.
 * E is exactly 0 for a block the candidate reproduces. */
static double block_E(const float* x, int B, const float* m, long double g)
{
    long double e = 0.0L;
    for (int i = 0; i < B; ++i) {
        const long double d = fabsl((long double)x[i]) - (long double)m[i] * g;
        e += d * d;
    }
    return (double)e;
}

/* Relative gap of the runner-up to the best, (E2 - E1) / max(E1, FLT_MIN), the near-tie
 * statistic; +inf when there is no runner-up. */
static double rel_gap(double E1, long double diff)
{
    const double den = E1 > FLT_MIN ? E1 : FLT_MIN;
    return (double)(diff / den);
}

/* ------------------------------------------------------------------------------------
 * NVFP4
 * ---------------------------------------------------------------------------------- */

static void scale_pair(int p, float S, float* sv, float* inv)
{
    if (p == 0) { *sv = 0.0f; *inv = 0.0f; return; }
    *sv = (float)fp4q_o_e4m3_value(p) * S;   /* e(p) is exact in float; one RN product */
    *inv = 1.0f / *sv;
}

/* E2M1 magnitudes of a block's codes at reciprocal scale inv (the quantizer: RN(x * inv), then
 * round to nearest even on the E2M1 grid). */
static void fp4_mags(const float* x, int B, float inv, float* m)
{
    for (int i = 0; i < B; ++i) m[i] = E2M1_MAG[fp4q_o_e2m1_encode(x[i] * inv) & 7];
}

/* WMSE error of one candidate: binary32, one accumulator, element order.  The zero scale
 * (sv = inv = 0) needs no special case: every code is +-0, xhat = 0, d = x. */
static float wmse_error(const float* x, const float* w, int B, float sv, float inv)
{
    float acc = 0.0f;
    for (int i = 0; i < B; ++i) {
        const float q = fp4q_o_e2m1_value(fp4q_o_e2m1_encode(x[i] * inv));
        const float xh = q * sv;
        const float d = x[i] - xh;
        acc = fmaf(w[i] * d, d, acc);
    }
    return acc;
}

static void pack_codes_for(const float* x, int B, float inv, uint8_t* codes_row, int64_t c0)
{
    for (int i = 0; i < B; i += 2) {
        int lo = fp4q_o_e2m1_encode(x[i] * inv);
        int hi = fp4q_o_e2m1_encode(x[i + 1] * inv);
        codes_row[(c0 + i) / 2] = (uint8_t)(lo | (hi << 4));
    }
}

/* objective: 0 AbsMax, 1 4/6, 2 sweep MSE [-3,7], 3 sweep WMSE [-8,7],
 *            4 brute-force MSE over all patterns 0..126, 5 brute-force WMSE.
 * Per block outputs (optional, may be NULL): chosen pattern; its error (MSE kinds: the exact
 * block error E rounded to double; WMSE: the binary32 accumulator); the relative gap of the
 * runner-up, (E2 - E1) / max(E1, FLT_MIN) (+inf with one candidate); whether the runner-up
 * ties the best exactly; the runner-up's pattern (-1 with one candidate); the number of valid
 * candidates. */
int fp4q_o_nvfp4_quantize(const float* x, int64_t rows, int64_t cols, int64_t ld,
                          int objective, const float* importance, int scale_given,
                          float* S_io, uint8_t* codes, uint8_t* scales,
                          int* blk_p, double* blk_err, double* blk_gap, int* blk_tie, int* blk_p2, int* blk_nvalid)
{
    const int B = 16;
    if (cols % B) return -1;
    int status = ST_OK;
    float S;
    if (scale_given) {
        S = *S_io;
        if (!isfinite(S)) status = ST_NONFINITE;
    } else {
        float amax;
        status = tensor_amax(x, rows, cols, ld, &amax);
        S = status == ST_OK ? fp4q_o_global_scale(amax) : NAN;
        *S_io = S;
    }
    if (status == ST_OK && !scale_range_ok(S)) status = ST_RANGE;
    const int64_t nb = cols / B;
    if (status != ST_OK) {  /* outputs are zero-filled when the data is out of contract */
        memset(codes, 0, (size_t)(rows * cols / 2));
        memset(scales, 0, (size_t)(rows * nb));
        return status;
    }
    int lo = 0, hi = 0;
    if (objective == 2) { lo = -3; hi = 7; }
    if (objective == 3) { lo = -8; hi = 7; }
    const int weighted = (objective == 3 || objective == 5);
    const float d6 = 6.0f * S, d4 = 4.0f * S;

    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < nb; ++b) {
            const float* xb = x + r * ld + b * B;
            const float* wb = weighted ? importance + b * B : NULL;
            float ab = 0.0f;
            for (int i = 0; i < B; ++i) ab = fmaxf(ab, fabsf(xb[i]));
            int p0 = 0, p4 = 0;
            if (S > 0.0f) {
                p0 = fp4q_o_e4m3_encode(ab / d6);
                p4 = fp4q_o_e4m3_encode(ab / d4);
            }
            /* candidate list in increasing offset order */
            int cand[128], nc = 0;
            if (objective == 0) cand[nc++] = p0;
            else if (objective == 1) { cand[nc++] = p0; if (p4 != p0) cand[nc++] = p4; }
            else if (objective == 4 || objective == 5) { for (int p = 0; p <= 0x7E; ++p) cand[nc++] = p; }
            else { for (int k = lo; k <= hi; ++k) { int p = p0 + k; if (p >= 0 && p <= 0x7E) cand[nc++] = p; } }
            if (S == 0.0f) { nc = 1; cand[0] = 0; }

            int bestp = cand[0], secp = -1, tie = 0;
            double err = 0.0, gap = INFINITY;
            if (weighted) {
                float best = INFINITY, second = INFINITY;
                for (int c = 0; c < nc; ++c) {
                    float sv, inv;
                    scale_pair(cand[c], S, &sv, &inv);
                    const float e = wmse_error(xb, wb, B, sv, inv);
                    if (c == 0 || e < best) { if (c) { second = best; secp = bestp; } best = e; bestp = cand[c]; }
                    else if (c == 1 || e < second) { second = e; secp = cand[c]; }
                }
                err = best;
                if (nc > 1) { gap = rel_gap(best, (long double)second - (long double)best); tie = second == best; }
            } else {
                exact_F best = {0.0L, 0.0L, 1}, second = {INFINITY, 0.0L, 1};
                float m[16];
                for (int c = 0; c < nc; ++c) {
                    float sv, inv;
                    scale_pair(cand[c], S, &sv, &inv);
                    fp4_mags(xb, B, inv, m);
                    const exact_F f = block_F(xb, B, m, (long double)sv);
                    if (c == 0 || F_less(f, best)) { if (c) { second = best; secp = bestp; } best = f; bestp = cand[c]; }
                    else if (c == 1 || F_less(f, second)) { second = f; secp = cand[c]; }
                }
                float sv, inv;
                scale_pair(bestp, S, &sv, &inv);
                fp4_mags(xb, B, inv, m);
                err = block_E(xb, B, m, (long double)sv);
                if (nc > 1) { gap = rel_gap(err, F_diff(best, second)); tie = F_equal(best, second); }
            }
            float sv, inv;
            scale_pair(bestp, S, &sv, &inv);
            pack_codes_for(xb, B, inv, codes + r * (cols / 2), b * B);
            scales[r * nb + b] = (uint8_t)bestp;
            if (blk_p) blk_p[r * nb + b] = bestp;
            if (blk_err) blk_err[r * nb + b] = err;
            if (blk_gap) blk_gap[r * nb + b] = gap;
            if (blk_tie) blk_tie[r * nb + b] = tie;
            if (blk_p2) blk_p2[r * nb + b] = secp;
            if (blk_nvalid) blk_nvalid[r * nb + b] = nc;
        }
    }
    return ST_OK;
}

/* ------------------------------------------------------------------------------------
 * IF4  [IF4]
 * ---------------------------------------------------------------------------------- */

static float rint_even(float z) { return nearbyintf(z); } /* default rounding mode: to nearest even */

/* The scaled-INT4 code of x at reciprocal scale inv: n = clamp(rint(RN(RN(x*inv) * RN(7/6))), -7, 7). */
static int int4_code(float x, float inv)
{
    const float K76 = 7.0f / 6.0f;   /* RN(7/6) */
    const float y = x * inv;
    float n = rint_even(y * K76);
    if (n > 7.0f) n = 7.0f;
    if (n < -7.0f) n = -7.0f;
    return (int)n;
}

/* Both types of one candidate pattern: their exact F values and their magnitudes. */
static void if4_candidate(const float* xb, float S, int p, exact_F* ffp, exact_F* fint, float* mfp, float* mint,
                          long double* gfp, long double* gint)
{
    float sv, inv;
    scale_pair(p, S, &sv, &inv);
    const float K67 = 6.0f / 7.0f;   /* RN(6/7) */
    fp4_mags(xb, 16, inv, mfp);
    for (int i = 0; i < 16; ++i) mint[i] = (float)abs(int4_code(xb[i], inv));
    *gfp = (long double)sv;
    *gint = (long double)(K67 * sv);   /* the INT4 block scale RN(RN(6/7) * sv) */
    *ffp = block_F(xb, 16, mfp, *gfp);
    *fint = block_F(xb, 16, mint, *gint);
}

/* sweep: 0 = IF4 at the AbsMax scale p0 (INT4 iff E_int < E_fp, exactly);
 *        1 = IF4 x ScaleSweep: every candidate p0 + k, k = -3..+7 (patterns 0..126), under
 *            both element types, exact errors, lexicographic (error, offset, type) with FP4 before
 *            INT4, so the lowest offset and then FP4 win ties;
 *        2 = the same over all patterns 0..126 (window check).
 * blk_err_fp / blk_err_int receive both types' exact errors E at the chosen pattern (rounded to
 * double); blk_gap / blk_tie the runner-up's relative gap and exact-tie flag over all (pattern,
 * type) candidates. */
int fp4q_o_if4_quantize(const float* x, int64_t rows, int64_t cols, int64_t ld, int sweep,
                        int scale_given, float* S_io, uint8_t* codes, uint8_t* scales,
                        double* blk_err_fp, double* blk_err_int, double* blk_gap, int* blk_tie)
{
    const int B = 16;
    if (cols % B) return -1;
    int status = ST_OK;
    float S;
    if (scale_given) {
        S = *S_io;
        if (!isfinite(S)) status = ST_NONFINITE;
    } else {
        float amax;
        status = tensor_amax(x, rows, cols, ld, &amax);
        S = status == ST_OK ? fp4q_o_global_scale(amax) : NAN;
        *S_io = S;
    }
    if (status == ST_OK && !scale_range_ok(S)) status = ST_RANGE;
    const int64_t nb = cols / B;
    if (status != ST_OK) {
        memset(codes, 0, (size_t)(rows * cols / 2));
        memset(scales, 0, (size_t)(rows * nb));
        return status;
    }
    const float d6 = 6.0f * S;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < nb; ++b) {
            const float* xb = x + r * ld + b * B;
            float ab = 0.0f;
            for (int i = 0; i < B; ++i) ab = fmaxf(ab, fabsf(xb[i]));
            const int p0 = S > 0.0f ? fp4q_o_e4m3_encode(ab / d6) : 0;
            int plo = p0, phi = p0;
            if (sweep == 1) { plo = p0 - 3; phi = p0 + 7; }
            if (sweep == 2) { plo = 0; phi = 0x7E; }
            if (plo < 0) plo = 0;
            if (phi > 0x7E) phi = 0x7E;
            int bp = plo, use_int = 0, first = 1, tie = 0;
            exact_F best = {0.0L, 0.0L, 1}, second = {INFINITY, 0.0L, 1};
            for (int p = plo; p <= phi; ++p) {
                exact_F f[2];
                float mf[16], mi[16];
                long double gf, gi;
                if4_candidate(xb, S, p, &f[0], &f[1], mf, mi, &gf, &gi);
                for (int t = 0; t < 2; ++t) {
                    if (first || F_less(f[t], best)) {
                        if (!first) second = best;
                        best = f[t]; bp = p; use_int = t; first = 0;
                    } else if (F_less(f[t], second)) {
                        second = f[t];
                    }
                }
            }
            exact_F ff, fi;
            float mf[16], mi[16];
            long double gf, gi;
            if4_candidate(xb, S, bp, &ff, &fi, mf, mi, &gf, &gi);
            const double ef = block_E(xb, B, mf, gf), ei = block_E(xb, B, mi, gi);
            float sv, inv;
            scale_pair(bp, S, &sv, &inv);
            uint8_t* crow = codes + r * (cols / 2) + b * B / 2;
            for (int i = 0; i < B; i += 2) {
                int lo = use_int ? (int4_code(xb[i], inv) & 0xF) : fp4q_o_e2m1_encode(xb[i] * inv);
                int hi = use_int ? (int4_code(xb[i + 1], inv) & 0xF) : fp4q_o_e2m1_encode(xb[i + 1] * inv);
                crow[i / 2] = (uint8_t)(lo | (hi << 4));
            }
            tie = F_equal(best, second);
            scales[r * nb + b] = (uint8_t)(bp | (use_int ? 0x80 : 0));
            if (blk_err_fp) blk_err_fp[r * nb + b] = ef;
            if (blk_err_int) blk_err_int[r * nb + b] = ei;
            if (blk_gap) blk_gap[r * nb + b] = rel_gap(use_int ? ei : ef, F_diff(best, second));
            if (blk_tie) blk_tie[r * nb + b] = tie;
        }
    }
    return ST_OK;
}

/* ------------------------------------------------------------------------------------
 * MXFP4 (+ block Hadamard)  [MR], [TQ]
 * ---------------------------------------------------------------------------------- */

void fp4q_o_hadamard32(float* v)
{
    for (int h = 1; h < 32; h <<= 1)
        for (int j = 0; j < 32; ++j)
            if ((j & h) == 0) {
                float a = v[j], b = v[j + h];
                v[j] = a + b;
                v[j + h] = a - b;
            }
    const float KH = (float)(1.0 / sqrt(32.0));
    for (int j = 0; j < 32; ++j) v[j] = v[j] * KH;
}

/* Normalized 16-point block Hadamard for NVFP4/IF4 (the rotation the MR-GPTQ page applies to
 * both formats, with the block size of NVFP4): butterflies h = 1, 2, 4, 8 in binary32, then a
 * multiplication by 1/sqrt(16) = 1/4, an exact power of two. */
void fp4q_o_hadamard16(float* v)
{
    for (int h = 1; h < 16; h <<= 1)
        for (int j = 0; j < 16; ++j)
            if ((j & h) == 0) {
                float a = v[j], b = v[j + h];
                v[j] = a + b;
                v[j + h] = a - b;
            }
    for (int j = 0; j < 16; ++j) v[j] = v[j] * 0.25f;
}

/* out[r][c] = the 16-point rotation of each 16-element block of row r of x (row stride ld). */
int fp4q_o_rotate16(const float* x, int64_t rows, int64_t cols, int64_t ld, float* out)
{
    if (cols % 16) return -1;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; c += 16) {
            float v[16];
            memcpy(v, x + r * ld + c, sizeof v);
            fp4q_o_hadamard16(v);
            memcpy(out + r * cols + c, v, sizeof v);
        }
    return 0;
}

/* Smallest e with a <= 6*2^e (ocp_floor = 0), or floor(log2 a) - 2 (ocp_floor = 1). */
int fp4q_o_mx_exponent(float a, int ocp_floor)
{
    if (a == 0.0f) return -127;
    int E;
    double f = frexp((double)a, &E);   /* a = f * 2^E, f in [0.5, 1) */
    int e = ocp_floor ? (E - 1) - 2 : (f <= 0.75 ? E - 3 : E - 2);
    if (e < -127) e = -127;
    if (e > 127) e = 127;
    return e;
}

/* E2M1 magnitudes of a 32-element block at scale 2^e: y = RN(v * 2^-e), exact for normal
 * results. */
static void mx_mags(const float* v, int e, float* m)
{
    const float s = ldexpf(1.0f, -e);
    for (int i = 0; i < 32; ++i) m[i] = E2M1_MAG[fp4q_o_e2m1_encode(v[i] * s) & 7];
}

/* MX scale sweep [MR] ("Scale Fitting" for MXFP4: the page fits the power-of-two scale grid
 * to the data to cut the error that E8M0's coarse, over-wide grid causes, without giving the
 * rule; the plainest reading is ScaleSweep's search carried over to E8M0).  Exponent of one
 * block under mode: 0 the max rule (ceil, or OCP floor with ocp_floor); 1 the sweep over
 * e_c + k, k = -2..0, e_c = the ceil rule, exponents below -127 skipped, the exact block error
 * sum (v - q 2^e)^2 compared exactly, the lowest exponent winning a tie; 2 the same over every
 * e in [-127, 127] (checks that the window of mode 1 holds the optimum).  gap / tie: the
 * runner-up's relative gap and exact-tie flag (modes 1 and 2). */
static int mx_block_exponent(const float* v, float ab, int ocp_floor, int mode, double* gap, int* tie)
{
    const int ec = fp4q_o_mx_exponent(ab, 0);
    *gap = INFINITY;
    *tie = 0;
    if (mode == 0) return ocp_floor ? fp4q_o_mx_exponent(ab, 1) : ec;
    const int lo = mode == 1 ? (ec - 2 < -127 ? -127 : ec - 2) : -127, hi = mode == 1 ? ec : 127;
    int be = lo, n = 0;
    exact_F best = {0.0L, 0.0L, 1}, second = {INFINITY, 0.0L, 1};
    float m[32];
    for (int e = lo; e <= hi; ++e) {
        mx_mags(v, e, m);
        const exact_F f = block_F(v, 32, m, ldexpl(1.0L, e));
        if (n == 0 || F_less(f, best)) { if (n) second = best; best = f; be = e; }
        else if (F_less(f, second)) second = f;
        ++n;
    }
    if (n > 1) {
        mx_mags(v, be, m);
        *gap = rel_gap(block_E(v, 32, m, ldexpl(1.0L, be)), F_diff(best, second));
        *tie = F_equal(best, second);
    }
    return be;
}

/* sweep: 0 the max rule, 1 the MX scale sweep (window [-2, 0]), 2 brute force over all
 * exponents; ocp_floor applies to sweep = 0 only.  blk_gap / blk_tie (optional): the near-tie
 * statistic of the sweep modes. */
int fp4q_o_mxfp4_quantize(const float* x, int64_t rows, int64_t cols, int64_t ld,
                          int hadamard, int ocp_floor, int sweep, uint8_t* codes, uint8_t* scales,
                          double* blk_gap, int* blk_tie)
{
    const int B = 32;
    if (cols % B) return -1;
    int status = ST_OK;
    const int64_t nb = cols / B;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < nb; ++b) {
            float v[32];
            memcpy(v, x + r * ld + b * B, sizeof v);
            int bad = 0;
            for (int i = 0; i < B; ++i) if (!isfinite(v[i])) bad = 1;
            uint8_t* crow = codes + r * (cols / 2) + b * B / 2;
            double gap = INFINITY;
            int tie = 0;
            if (bad) {
                status |= ST_NONFINITE;
                memset(crow, 0, B / 2);
                scales[r * nb + b] = 0xFF;   /* E8M0 NaN */
            } else {
                if (hadamard) fp4q_o_hadamard32(v);
                float ab = 0.0f;
                for (int i = 0; i < B; ++i) ab = fmaxf(ab, fabsf(v[i]));
                int e = mx_block_exponent(v, ab, ocp_floor, sweep, &gap, &tie);
                float m = ldexpf(1.0f, -e);   /* exact power of two (subnormal for e = 127) */
                for (int i = 0; i < B; i += 2) {
                    int lo = fp4q_o_e2m1_encode(v[i] * m), hi = fp4q_o_e2m1_encode(v[i + 1] * m);
                    crow[i / 2] = (uint8_t)(lo | (hi << 4));
                }
                scales[r * nb + b] = (uint8_t)(e + 127);
            }
            if (blk_gap) blk_gap[r * nb + b] = gap;
            if (blk_tie) blk_tie[r * nb + b] = tie;
        }
    }
    return status;
}

/* Exact block errors sum (v - q 2^e)^2 (rounded to double) of MXFP4 blocks (after the optional
 * rotation) at the exponents given by the scale bytes.  Returns -1 on a bad shape. */
int fp4q_o_mx_block_errors(const float* x, int64_t rows, int64_t cols, int64_t ld, int hadamard,
                           const uint8_t* scales, double* err)
{
    if (cols % 32) return -1;
    const int64_t nb = cols / 32;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t b = 0; b < nb; ++b) {
            float v[32], m[32];
            memcpy(v, x + r * ld + b * 32, sizeof v);
            if (hadamard) fp4q_o_hadamard32(v);
            const int e = (int)scales[r * nb + b] - 127;
            mx_mags(v, e, m);
            err[r * nb + b] = block_E(v, 32, m, ldexpl(1.0L, e));
        }
    return 0;
}

/* ------------------------------------------------------------------------------------
 * IF6  [IF4] "Methodology", extensibility: the same per-block type choice for 6-bit elements
 * ---------------------------------------------------------------------------------- */

/* FP6 E2M3 magnitude of a 6-bit code (bit 5 = sign, ignored here): 2 exponent bits (bias 1),
 * 3 mantissa bits; exponent 0 holds the subnormals k/8, k = 0..7; the largest value is 7.5. */
double fp4q_o_e2m3_value(int code)
{
    const int e = (code >> 3) & 3, f = code & 7;
    return e == 0 ? f / 8.0 : (1.0 + f / 8.0) * ldexp(1.0, e - 1);
}

/* Round y to the nearest E2M3 value with ties to the even code, saturating at 7.5, sign kept in
 * bit 5: a scan over the 32 magnitudes. */
int fp4q_o_e2m3_encode(float y)
{
    const int s = signbit(y) ? 0x20 : 0;
    const double a = fabs((double)y);
    int best = 0;
    double bestd = a;
    for (int c = 1; c < 32; ++c) {
        const double d = fabs(a - fp4q_o_e2m3_value(c));
        if (d < bestd || (d == bestd && (c & 1) == 0 && (best & 1) == 1)) { best = c; bestd = d; }
    }
    return s | best;
}

/* The scaled-INT6 code of x at reciprocal scale inv: n = clamp(rint(RN(RN(x*inv) * RN(62/15))), -31, 31). */
static int int6_code(float x, float inv)
{
    const float K = 62.0f / 15.0f;   /* RN(31 / 7.5): the INT6 maximum 31 onto the FP6 maximum 7.5 */
    const float y = x * inv;
    float n = rint_even(y * K);
    if (n > 31.0f) n = 31.0f;
    if (n < -31.0f) n = -31.0f;
    return (int)n;
}

/* Pack the 6-bit fields of one 16-element block into 12 bytes: element i in bits 6i .. 6i+5 of
 * the block's little-endian 96-bit field. */
static void pack6(const int* f, uint8_t* dst)
{
    memset(dst, 0, 12);
    for (int i = 0; i < 16; ++i)
        for (int b = 0; b < 6; ++b)
            if ((f[i] >> b) & 1) dst[(6 * i + b) >> 3] |= (uint8_t)(1u << ((6 * i + b) & 7));
}

static int unpack6(const uint8_t* src, int i)
{
    int v = 0;
    for (int b = 0; b < 6; ++b) v |= ((src[(6 * i + b) >> 3] >> ((6 * i + b) & 7)) & 1) << b;
    return v;
}

/* S of an IF6 tensor: RN(amax / (256 * 7.5)), the FP6 maximum in place of FP4's 6. */
float fp4q_o_global_scale_if6(float amax) { return amax / 1920.0f; }

/* IF6 quantization: per 16-element block one E4M3 scale p0 = E4M3(RN(a_b / RN(7.5 S))) shared by
 * both element types; FP6 codes E2M3(RN(x * inv)) with reconstruction q * sv, INT6 codes n with
 * reconstruction n * RN(RN(15/62) * sv); INT6 (indicator 0x80 in the scale byte) iff its exact
 * block error is lower.  codes: [rows][cols * 3 / 4] bytes (12 per block, pack6); FP6 fields are
 * the E2M3 bits (sign in bit 5), INT6 fields 6-bit two's complement.  err_fp / err_int: both exact
 * errors (double); gap / tie: the runner-up's relative gap and exact-tie flag. */
int fp4q_o_if6_quantize(const float* x, int64_t rows, int64_t cols, int64_t ld, int scale_given, float* S_io,
                        uint8_t* codes, uint8_t* scales, double* blk_err_fp, double* blk_err_int,
                        double* blk_gap, int* blk_tie)
{
    const int B = 16;
    if (cols % B) return -1;
    int status = ST_OK;
    float S;
    if (scale_given) {
        S = *S_io;
        if (!isfinite(S)) status = ST_NONFINITE;
    } else {
        float amax;
        status = tensor_amax(x, rows, cols, ld, &amax);
        S = status == ST_OK ? fp4q_o_global_scale_if6(amax) : NAN;
        *S_io = S;
    }
    if (status == ST_OK && !scale_range_ok(S)) status = ST_RANGE;
    const int64_t nb = cols / B;
    if (status != ST_OK) {
        memset(codes, 0, (size_t)(rows * cols * 3 / 4));
        memset(scales, 0, (size_t)(rows * nb));
        return status;
    }
    const float d75 = 7.5f * S, K = 15.0f / 62.0f;   /* RN(7.5 S), RN(15/62) */
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < nb; ++b) {
            const float* xb = x + r * ld + b * B;
            float ab = 0.0f;
            for (int i = 0; i < B; ++i) ab = fmaxf(ab, fabsf(xb[i]));
            const int p0 = S > 0.0f ? fp4q_o_e4m3_encode(ab / d75) : 0;
            float sv, inv;
            scale_pair(p0, S, &sv, &inv);
            float mf[16], mi[16];
            int cf[16], ci[16];
            for (int i = 0; i < B; ++i) {
                cf[i] = fp4q_o_e2m3_encode(xb[i] * inv);
                mf[i] = (float)fp4q_o_e2m3_value(cf[i]);
                const int n = int6_code(xb[i], inv);
                mi[i] = (float)abs(n);
                ci[i] = n & 0x3F;
            }
            const long double gf = (long double)sv, gi = (long double)(K * sv);
            const exact_F ff = block_F(xb, B, mf, gf), fi = block_F(xb, B, mi, gi);
            const int use_int = F_less(fi, ff);
            const double ef = block_E(xb, B, mf, gf), ei = block_E(xb, B, mi, gi);
            pack6(use_int ? ci : cf, codes + r * (cols * 3 / 4) + b * 12);
            scales[r * nb + b] = (uint8_t)(p0 | (use_int ? 0x80 : 0));
            if (blk_err_fp) blk_err_fp[r * nb + b] = ef;
            if (blk_err_int) blk_err_int[r * nb + b] = ei;
            if (blk_gap) blk_gap[r * nb + b] = rel_gap(use_int ? ei : ef, use_int ? F_diff(fi, ff) : F_diff(ff, fi));
            if (blk_tie) blk_tie[r * nb + b] = F_equal(ff, fi);
        }
    }
    return ST_OK;
}

/* ------------------------------------------------------------------------------------
 * Dequantize
 * ---------------------------------------------------------------------------------- */

/* Own bf16 rounding (nearest even) for the bf16 output option. */
static uint16_t f32_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x7FFFFFu)) return (uint16_t)((u >> 16) | 0x40);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

int fp4q_o_if6_dequantize(const uint8_t* codes, const uint8_t* scales, float S, int64_t rows, int64_t cols,
                          void* out, int out_bf16)
{
    if (cols % 16) return -1;
    const int64_t nb = cols / 16;
    const float K = 15.0f / 62.0f;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t b = 0; b < nb; ++b) {
            const uint8_t sb = scales[r * nb + b];
            float sv, inv;
            scale_pair(sb & 0x7F, S, &sv, &inv);
            const uint8_t* src = codes + r * (cols * 3 / 4) + b * 12;
            for (int i = 0; i < 16; ++i) {
                const int f = unpack6(src, i);
                float v;
                if (sb & 0x80) {
                    const int n = f >= 32 ? f - 64 : f;
                    v = (float)n * (K * sv);
                } else {
                    const float m = (float)fp4q_o_e2m3_value(f);
                    v = ((f & 0x20) ? -m : m) * sv;
                }
                const int64_t idx = r * cols + b * 16 + i;
                if (out_bf16) ((uint16_t*)out)[idx] = f32_to_bf16(v);
                else ((float*)out)[idx] = v;
            }
        }
    return ST_OK;
}

/* Batch form of the bf16 rounding (for its pin). */
void fp4q_o_f32_to_bf16(const float* x, int64_t n, uint16_t* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = f32_to_bf16(x[i]);
}

/* fmt: 0 NVFP4, 1 IF4, 2 MXFP4.  out is float32 [rows][cols] (out_bf16 = 0) or uint16
 * bf16 bit patterns (out_bf16 = 1).  inverse_hadamard applies the 32-point transform to
 * every dequantized MXFP4 block, the 16-point one to NVFP4/IF4 blocks (each normalized
 * transform is its own inverse). */
int fp4q_o_dequantize(const uint8_t* codes, const uint8_t* scales, float S,
                      int64_t rows, int64_t cols, int fmt, int inverse_hadamard,
                      void* out, int out_bf16)
{
    const int B = fmt == 2 ? 32 : 16;
    if (cols % B) return -1;
    const int64_t nb = cols / B;
    const float K67 = 6.0f / 7.0f;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < nb; ++b) {
            float v[32];
            uint8_t sb = scales[r * nb + b];
            const uint8_t* crow = codes + r * (cols / 2) + b * B / 2;
            for (int i = 0; i < B; ++i) {
                int code = (crow[i / 2] >> ((i & 1) * 4)) & 0xF;
                if (fmt == 2) {
                    if (sb == 0xFF) { v[i] = NAN; continue; }
                    float m = ldexpf(1.0f, (int)sb - 127);
                    v[i] = fp4q_o_e2m1_value(code) * m;
                } else {
                    float sv, inv;
                    scale_pair(sb & 0x7F, S, &sv, &inv);
                    if (fmt == 1 && (sb & 0x80)) {
                        int n = code >= 8 ? code - 16 : code;
                        v[i] = (float)n * (K67 * sv);
                    } else {
                        v[i] = fp4q_o_e2m1_value(code) * sv;
                    }
                }
            }
            if (fmt == 2 && inverse_hadamard) fp4q_o_hadamard32(v);
            if (fmt != 2 && inverse_hadamard) fp4q_o_hadamard16(v);
            for (int i = 0; i < B; ++i) {
                int64_t idx = r * cols + b * B + i;
                if (out_bf16) ((uint16_t*)out)[idx] = f32_to_bf16(v[i]);
                else ((float*)out)[idx] = v[i];
            }
        }
    }
    return ST_OK;
}
