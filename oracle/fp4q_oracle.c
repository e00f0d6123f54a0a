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
 * Arithmetic contract (the readings where the pages are silent; every floating point
 * step is one IEEE-754 binary32 operation rounded to nearest even, written RN below;
 * no contraction, no flush-to-zero):
 *   S      = RN(amax / 1536)                      (amax = max |x| over the tensor)
 *   p0     = E4M3(RN(a_b / RN(6*S)))               (a_b = max |x| over the block)
 *   p4     = E4M3(RN(a_b / RN(4*S)))               (4/6 only)
 *   sv(p)  = RN(e(p) * S), inv(p) = RN(1 / sv(p)); sv(0) = inv(0) = 0
 *   y      = RN(x * inv),  q = E2M1(y),  r = RN(q - y)   (the quantizer's own rounding
 *            error, in units of the scale)
 *   error  = RN(RN(sv*sv) * E) with E = RN(acc_even + acc_odd); acc_even / acc_odd are fp32
 *            accumulators over the even / odd element positions, each acc = fma(r, r, acc)
 *            (WMSE: acc = fma(RN(w*r), r, acc)) in element order.  For the zero scale
 *            (p = 0) every code is 0 and the error is the same fma sum over x itself.
 *            This is the block MSE sum (x - q*s)^2 = s^2 sum (x/s - q)^2 evaluated on the
 *            binary32 quotient y the quantizer rounds.
 *   argmin = lexicographic (error, offset): the lowest offset wins a tie.
 *   IF4    = AbsMax scale p0; INT4 path z = RN(y*RN(7/6)), n = clamp(rint(z), -7, 7),
 *            v = RN(n*RN(6/7)), r = RN(v - y); both paths share s, so INT4 iff
 *            E_int < E_fp.
 *   IF4 sweep = every MSE-window candidate p0-3 .. p0+7 under both types, error
 *            RN(RN(sv*sv) * E) as for the NVFP4 sweep; (error, offset, FP4-before-INT4)
 *            lexicographic.
 *   MXFP4  = e = smallest integer with a_b <= 6*2^e (clamped to [-127,127]), byte e+127,
 *            y = RN(x * 2^-e), q = E2M1(y), dequant q*2^e.
 *   MX sweep = e among e_c - 2 .. e_c (e_c the rule above) minimizing RN(E * 4^(e - e_c)),
 *            E = RN(acc_even + acc_odd) of fma(r, r, acc), r = RN(q - y) at that e; lowest e
 *            wins a tie.
 *   Hadamard(32) = Sylvester fast Walsh-Hadamard butterflies for h = 1,2,4,8,16
 *            (v_j, v_j+h) <- (RN(v_j + v_j+h), RN(v_j - v_j+h)), then RN(v * RN(1/sqrt(32))).
 *   dequant NVFP4 x^ = RN(q * sv); IF4-INT4 x^ = RN(RN(n*RN(6/7)) * sv); MXFP4 x^ = RN(q*2^e).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#include <float.h>

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
 * NVFP4 candidate evaluation
 * ---------------------------------------------------------------------------------- */

static void scale_pair(int p, float S, float* sv, float* inv)
{
    if (p == 0) { *sv = 0.0f; *inv = 0.0f; return; }
    *sv = (float)fp4q_o_e4m3_value(p) * S;   /* e(p) is exact in float; one RN product */
    *inv = 1.0f / *sv;
}

/* Error of one candidate scale for a block of B values.  p = 0 (sv = 0): every code is
 * zero and the error is the sum of x^2 (WMSE: w x^2).  Otherwise: residuals of the
 * quantizer in units of the scale, r = RN(q - y), squares summed by fma into two
 * accumulators by element parity, combined once, then scaled by RN(sv^2). */
static float block_error(const float* x, const float* w, int B, float sv, float inv)
{
    float acc[2] = {0.0f, 0.0f};
    if (sv == 0.0f) {
        for (int i = 0; i < B; ++i) {
            if (w) acc[i & 1] = fmaf(w[i] * x[i], x[i], acc[i & 1]);
            else acc[i & 1] = fmaf(x[i], x[i], acc[i & 1]);
        }
        return acc[0] + acc[1];
    }
    for (int i = 0; i < B; ++i) {
        float y = x[i] * inv;
        float q = fp4q_o_e2m1_value(fp4q_o_e2m1_encode(y));
        float r = q - y;
        if (w) acc[i & 1] = fmaf(w[i] * r, r, acc[i & 1]);
        else acc[i & 1] = fmaf(r, r, acc[i & 1]);
    }
    float E = acc[0] + acc[1];
    return (sv * sv) * E;
}

static uint8_t pack_codes_for(const float* x, int B, float inv, uint8_t* codes_row, int64_t c0)
{
    for (int i = 0; i < B; i += 2) {
        int lo = fp4q_o_e2m1_encode(x[i] * inv);
        int hi = fp4q_o_e2m1_encode(x[i + 1] * inv);
        codes_row[(c0 + i) / 2] = (uint8_t)(lo | (hi << 4));
    }
    return 0;
}

/* objective: 0 AbsMax, 1 4/6, 2 sweep MSE [-3,7], 3 sweep WMSE [-8,7],
 *            4 brute-force MSE over all patterns 0..126, 5 brute-force WMSE.
 * Per block outputs (optional, may be NULL): chosen pattern, its error, runner-up error
 * (+inf when only one candidate), number of valid candidates. */
int fp4q_o_nvfp4_quantize(const float* x, int64_t rows, int64_t cols, int64_t ld,
                          int objective, const float* importance, int scale_given,
                          float* S_io, uint8_t* codes, uint8_t* scales,
                          int* blk_p, float* blk_err, float* blk_err2, int* blk_nvalid)
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

            int bestp = cand[0];
            float best = INFINITY, second = INFINITY;
            for (int c = 0; c < nc; ++c) {
                float sv, inv;
                scale_pair(cand[c], S, &sv, &inv);
                float e = block_error(xb, wb, B, sv, inv);
                if (e < best) { second = best; best = e; bestp = cand[c]; }
                else if (e < second) second = e;
            }
            float sv, inv;
            scale_pair(bestp, S, &sv, &inv);
            pack_codes_for(xb, B, inv, codes + r * (cols / 2), b * B);
            scales[r * nb + b] = (uint8_t)bestp;
            if (blk_p) blk_p[r * nb + b] = bestp;
            if (blk_err) blk_err[r * nb + b] = best;
            if (blk_err2) blk_err2[r * nb + b] = second;
            if (blk_nvalid) blk_nvalid[r * nb + b] = nc;
        }
    }
    return ST_OK;
}

/* ------------------------------------------------------------------------------------
 * IF4  [IF4]
 * ---------------------------------------------------------------------------------- */

static float rint_even(float z) { return nearbyintf(z); } /* default rounding mode: to nearest even */

/* FP4 and scaled-INT4 residual sums of one block at reciprocal scale inv, in units of the
 * scale (E = RN(acc_even + acc_odd), fma accumulation in element order), and the codes of both
 * paths.  [IF4]: INT4 z = RN(y*RN(7/6)), n = clamp(rint(z), -7, 7), v = RN(n*RN(6/7)). */
static void if4_block_sums(const float* xb, float inv, float* ef, float* ei, int* cf, int* ci)
{
    const float K76 = 7.0f / 6.0f, K67 = 6.0f / 7.0f;   /* RN of each ratio */
    float accf[2] = {0, 0}, acci[2] = {0, 0};
    for (int i = 0; i < 16; ++i) {
        float y = xb[i] * inv;
        cf[i] = fp4q_o_e2m1_encode(y);
        float q = fp4q_o_e2m1_value(cf[i]);
        float rf = q - y;
        accf[i & 1] = fmaf(rf, rf, accf[i & 1]);
        float z = y * K76;
        float n = rint_even(z);
        if (n > 7.0f) n = 7.0f;
        if (n < -7.0f) n = -7.0f;
        float v = n * K67;
        float ri = v - y;
        acci[i & 1] = fmaf(ri, ri, acci[i & 1]);
        ci[i] = ((int)n) & 0xF;   /* two's complement nibble */
    }
    *ef = accf[0] + accf[1];
    *ei = acci[0] + acci[1];
}

/* sweep: 0 = IF4 at the AbsMax scale p0 (INT4 iff E_int < E_fp);
 *        1 = IF4 x ScaleSweep: every candidate p0 + k, k = -3..+7 (patterns 0..126), under
 *            both element types; error = RN(RN(sv^2) * E) (the zero scale: the fma sum of x^2,
 *            both types alike); lexicographic (error, offset, type) with FP4 before INT4, so
 *            the lowest offset and then FP4 win ties;
 *        2 = the same over all patterns 0..126 (window check).
 * blk_err_fp / blk_err_int receive both types' errors at the chosen pattern (mode 0: the
 * unscaled E; modes 1-2: the scaled errors). */
int fp4q_o_if4_quantize(const float* x, int64_t rows, int64_t cols, int64_t ld, int sweep,
                        int scale_given, float* S_io, uint8_t* codes, uint8_t* scales,
                        float* blk_err_fp, float* blk_err_int)
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
            int p0 = S > 0.0f ? fp4q_o_e4m3_encode(ab / d6) : 0;
            int bp = p0, use_int = 0;
            float ef, ei;
            int cf[16], ci[16];
            if (sweep == 0) {
                float sv, inv;
                scale_pair(p0, S, &sv, &inv);
                if4_block_sums(xb, inv, &ef, &ei, cf, ci);
                use_int = ei < ef;
            } else {
                int lo = sweep == 1 ? p0 - 3 : 0, hi = sweep == 1 ? p0 + 7 : 0x7E;
                if (lo < 0) lo = 0;
                if (hi > 0x7E) hi = 0x7E;
                if (S == 0.0f) lo = hi = 0;
                float best = INFINITY, bf = 0.0f, bi = 0.0f;
                bp = lo;
                for (int p = lo; p <= hi; ++p) {
                    float e_fp, e_int;
                    if (p == 0) {
                        float acc[2] = {0, 0};
                        for (int i = 0; i < B; ++i) acc[i & 1] = fmaf(xb[i], xb[i], acc[i & 1]);
                        e_fp = e_int = acc[0] + acc[1];
                    } else {
                        float sv, inv, E_f, E_i;
                        scale_pair(p, S, &sv, &inv);
                        if4_block_sums(xb, inv, &E_f, &E_i, cf, ci);
                        const float s2 = sv * sv;
                        e_fp = s2 * E_f;
                        e_int = s2 * E_i;
                    }
                    if (e_fp < best) { best = e_fp; bp = p; use_int = 0; bf = e_fp; bi = e_int; }
                    if (e_int < best) { best = e_int; bp = p; use_int = 1; bf = e_fp; bi = e_int; }
                }
                float sv, inv;
                scale_pair(bp, S, &sv, &inv);
                if4_block_sums(xb, inv, &ef, &ei, cf, ci);   /* codes of the chosen scale */
                ef = bf;
                ei = bi;
            }
            uint8_t* crow = codes + r * (cols / 2) + b * B / 2;
            for (int i = 0; i < B; i += 2) {
                int lo = use_int ? ci[i] : cf[i], hi = use_int ? ci[i + 1] : cf[i + 1];
                crow[i / 2] = (uint8_t)(lo | (hi << 4));
            }
            scales[r * nb + b] = (uint8_t)(bp | (use_int ? 0x80 : 0));
            if (blk_err_fp) blk_err_fp[r * nb + b] = ef;
            if (blk_err_int) blk_err_int[r * nb + b] = ei;
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

/* MX scale sweep [MR] ("Scale Fitting" for MXFP4: the page fits the power-of-two scale grid
 * to the data to cut the error that E8M0's coarse, over-wide grid causes, without giving the
 * rule; the plainest reading is ScaleSweep's search carried over to E8M0).  Error of one
 * 32-element block at scale 2^e, in units of 4^e: y = RN(x*2^-e), q = E2M1(y), r = RN(q - y),
 * E = RN(acc_even + acc_odd) with acc = fma(r, r, acc) over the even / odd positions in order,
 * as for NVFP4.  Multiplying by 2^-e is exact for normal results, so r is the rounding error
 * of the block in units of the scale. */
static float mx_block_error(const float* v, int e)
{
    const float m = ldexpf(1.0f, -e);
    float acc[2] = {0.0f, 0.0f};
    for (int i = 0; i < 32; ++i) {
        float y = v[i] * m;
        float q = fp4q_o_e2m1_value(fp4q_o_e2m1_encode(y));
        float r = q - y;
        acc[i & 1] = fmaf(r, r, acc[i & 1]);
    }
    return acc[0] + acc[1];
}

/* Exponent of one block under mode: 0 the max rule (ceil, or OCP floor with ocp_floor);
 * 1 the sweep over e_c + k, k = -2..0, e_c = the ceil rule, patterns below -127 skipped,
 * comparing RN(E_k * 4^k) (the block error in units of 4^e_c; the power-of-two factor is
 * exact) lexicographically with the lowest k winning a tie;
 * 2 brute force over every e in [-127, 127] on the reconstruction error itself,
 * sum (x - q * 2^e)^2 accumulated in double (each term exact), lowest e winning a tie (checks
 * that the window of mode 1 holds the optimum; away from the window the scaled error of
 * mode 1 would underflow, the absolute one does not). */
static double mx_block_abs_error(const float* v, int e)
{
    const float m = ldexpf(1.0f, -e);
    double err = 0.0;
    for (int i = 0; i < 32; ++i) {
        double d = (double)v[i] - ldexp((double)fp4q_o_e2m1_value(fp4q_o_e2m1_encode(v[i] * m)), e);
        err += d * d;
    }
    return err;
}

static int mx_block_exponent(const float* v, float ab, int ocp_floor, int mode)
{
    const int ec = fp4q_o_mx_exponent(ab, 0);
    if (mode == 0) return ocp_floor ? fp4q_o_mx_exponent(ab, 1) : ec;
    if (mode == 1) {
        int be = ec + (ec - 2 < -127 ? -127 - ec : -2);   /* the first candidate */
        float best = INFINITY;
        for (int k = -2; k <= 0; ++k) {
            if (ec + k < -127) continue;
            float err = mx_block_error(v, ec + k) * ldexpf(1.0f, 2 * k);
            if (err < best) { best = err; be = ec + k; }
        }
        return be;
    }
    int be = -127;
    double best = INFINITY;
    for (int e = -127; e <= 127; ++e) {
        double err = mx_block_abs_error(v, e);
        if (err < best) { best = err; be = e; }
    }
    return be;
}

/* sweep: 0 the max rule, 1 the MX scale sweep (window [-2, 0]), 2 brute force over all
 * exponents; ocp_floor applies to sweep = 0 only. */
int fp4q_o_mxfp4_quantize(const float* x, int64_t rows, int64_t cols, int64_t ld,
                          int hadamard, int ocp_floor, int sweep, uint8_t* codes, uint8_t* scales)
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
            if (bad) {
                status |= ST_NONFINITE;
                memset(crow, 0, B / 2);
                scales[r * nb + b] = 0xFF;   /* E8M0 NaN */
                continue;
            }
            if (hadamard) fp4q_o_hadamard32(v);
            float ab = 0.0f;
            for (int i = 0; i < B; ++i) ab = fmaxf(ab, fabsf(v[i]));
            int e = mx_block_exponent(v, ab, ocp_floor, sweep);
            float m = ldexpf(1.0f, -e);   /* exact power of two (subnormal for e = 127) */
            for (int i = 0; i < B; i += 2) {
                int lo = fp4q_o_e2m1_encode(v[i] * m), hi = fp4q_o_e2m1_encode(v[i + 1] * m);
                crow[i / 2] = (uint8_t)(lo | (hi << 4));
            }
            scales[r * nb + b] = (uint8_t)(e + 127);
        }
    }
    return status;
}

/* Block errors of MXFP4 blocks (after the optional rotation) at the exponents given by the
 * scale bytes, in units of 4^e: the E of mx_block_error.  Returns -1 on a bad shape. */
int fp4q_o_mx_block_errors(const float* x, int64_t rows, int64_t cols, int64_t ld, int hadamard,
                           const uint8_t* scales, float* err)
{
    if (cols % 32) return -1;
    const int64_t nb = cols / 32;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t b = 0; b < nb; ++b) {
            float v[32];
            memcpy(v, x + r * ld + b * 32, sizeof v);
            if (hadamard) fp4q_o_hadamard32(v);
            err[r * nb + b] = mx_block_error(v, (int)scales[r * nb + b] - 127);
        }
    return 0;
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
                        v[i] = ((float)n * K67) * sv;
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
