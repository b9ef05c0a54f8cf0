/*
 * qamw_oracle.c -- plain, slow, fp64 CPU statement of the QAM-W weight codec.
 *
 * TEST INFRASTRUCTURE.  This file is the oracle that the CUDA path is checked
 * against.  Only the test suite, the smoke check and the CPU-baseline leg of the
 * benchmark may load it; the library path never calls it and shares no code,
 * header, table or constant with it.
 *
 * Source: "QAM-W: Joint 2D Codebook Quantization for LLM Weights via Hadamard
 * Rotation and Activation-Aware Scaling" (Sharma & Dobek), section 3 "The QAM-W
 * codec pipeline":
 *   3.1 encoder steps 1-6, 3.2 decoder, 3.3 choice of rotation (block rule),
 *   3.4 pair calibration (eq. 1), 3.6 joint 2D QAM (eq. 2, nearest codeword),
 *   3.7 bitrate (eq. 3), 3.8 QAM-W-3.5;
 * and the gist.science explainer of the same paper, "Methodology" list item
 * "activation-aware scaling" (s_j proportional to r_j^alpha, applied before
 * quantisation).
 *
 * Every function is the definition written out: dense Hadamard products, brute
 * force over the whole codebook in ascending index with a strict '<', fp64
 * accumulation, and rounding to binary16 only where the codec stores a value.
 * Readings of points the paper leaves open are listed at each function.
 *
 * Pins (tests/test_oracle_*.py): H H^T = bI and scipy's Sylvester matrix; the
 * binary16 rounding against numpy; a published splitmix64 output; isometry of
 * the rotation; the Rayleigh-mean statistic of eq. (1) on Gaussian rows; brute
 * force argmin on tiny codebooks; lossless round trip on codeword-synthesised
 * rows; Lloyd centroid / nearest-neighbour conditions and the K=2, K=4 closed
 * forms and high-rate distortion on the unit circular Gaussian of eq. (2); the
 * bitrate of eq. (3) and the block rule examples of section 3.3; the trace
 * identity and the AWQ direction on outlier activations.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* binary16 <-> double, from the IEEE 754 binary16 layout (1 sign bit,       */
/* 5 exponent bits with bias 15, 10 fraction bits), round to nearest even.   */
/* ------------------------------------------------------------------------ */

double ref_half_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int m = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24); /* subnormal: m * 2^-24 */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(m + 1024), e - 25); /* (1 + m/1024) * 2^(e-15) */
    return sign ? -v : v;
}

uint16_t ref_double_to_half(double x)
{
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    if (isnan(x))
        return 0x7e00;
    double a = fabs(x);
    if (a < ldexp(1.0, -14)) {
        /* subnormal range: quantum 2^-24; 1024 quanta rounds up into 0x0400 */
        double q = nearbyint(ldexp(a, 24));
        return (uint16_t)(sign | (uint16_t)q);
    }
    int e;
    frexp(a, &e);                       /* a in [2^(e-1), 2^e) */
    double q = nearbyint(ldexp(a, 11 - e)); /* 11 significant bits, in [1024, 2048] */
    int biased = e - 1 + 15;
    if (q == 2048.0) {
        q = 1024.0;
        biased += 1;
    }
    if (biased >= 31)
        return (uint16_t)(sign | 0x7c00);
    return (uint16_t)(sign | (uint16_t)(biased << 10) | (uint16_t)((int)q - 1024));
}

/* ------------------------------------------------------------------------ */
/* Deterministic sign mask (section 3.1 step 2: "deterministic sign-masked   */
/* block Hadamard rotation").  The paper does not give the mask; the reading */
/* used here is D_j = -1 when bit 63 of splitmix64 at counter               */
/* (mask_seed * 2^32 + j) is set, else +1.  splitmix64 is the published      */
/* generator of Steele, Lea and Flood (2014) in Vigna's formulation: add the */
/* golden-ratio increment, then two xor-shift-multiply rounds.              */
/* ------------------------------------------------------------------------ */

uint64_t ref_splitmix64(uint64_t counter)
{
    uint64_t z = counter + 0x9e3779b97f4a7c15ULL;
    z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ULL;
    z = (z ^ (z >> 27)) * 0x94d049bb133111ebULL;
    return z ^ (z >> 31);
}

int ref_sign(uint64_t mask_seed, int64_t j)
{
    uint64_t h = ref_splitmix64((mask_seed << 32) + (uint64_t)j);
    return (h >> 63) ? -1 : 1;
}

/* ------------------------------------------------------------------------ */
/* Section 3.3: block size = largest power of two dividing d_in, at most     */
/* 1024 (d_in = 2048 -> 1024, d_in = 5632 -> 512).                           */
/* ------------------------------------------------------------------------ */

int ref_default_block(int d_in)
{
    if (d_in <= 0)
        return 0;
    int b = 1;
    while (b < 1024 && (d_in % (2 * b)) == 0)
        b *= 2;
    return b;
}

/* Section 3.7 eq. (3): bpw = B/2 + 16/d_in (B bits per pair, one 16-bit row
 * norm per row), before byte alignment. */
double ref_bits_per_weight(int d_in, int bits)
{
    return bits / 2.0 + 16.0 / (double)d_in;
}

/* Row stride of the bit-packed index stream: P*bits bits rounded up to a
 * multiple of 16 bytes (the "row-level packing and alignment" of 3.7). */
int64_t ref_row_bytes(int d_in, int bits)
{
    int64_t nbits = (int64_t)(d_in / 2) * bits;
    return ((nbits + 127) / 128) * 16;
}

/* ------------------------------------------------------------------------ */
/* Sylvester Hadamard matrix in natural order: H[m][n] = (-1)^popcount(m&n). */
/* ------------------------------------------------------------------------ */

static int parity(unsigned v)
{
    int p = 0;
    while (v) {
        p ^= 1;
        v &= v - 1;
    }
    return p;
}

void ref_hadamard(int b, int8_t *H)
{
    for (int m = 0; m < b; ++m)
        for (int n = 0; n < b; ++n)
            H[(int64_t)m * b + n] = parity((unsigned)(m & n)) ? -1 : 1;
}

/* R_fwd = blockdiag(H_b) * diag(D) / sqrt(b): the sign mask is applied
 * first, then the Hadamard of each block, then the 1/sqrt(b) that makes the
 * map an isometry (Lemma 1).  Written as a dense product per block. */
void ref_rotate_fwd(const double *u, int d, int b, uint64_t mask_seed, double *y)
{
    double inv = 1.0 / sqrt((double)b);
    for (int base = 0; base < d; base += b)
        for (int m = 0; m < b; ++m) {
            double acc = 0.0;
            for (int n = 0; n < b; ++n) {
                int h = parity((unsigned)(m & n)) ? -1 : 1;
                acc += h * ref_sign(mask_seed, base + n) * u[base + n];
            }
            y[base + m] = acc * inv;
        }
}

/* R_inv = R_fwd^T = diag(D) * blockdiag(H_b) / sqrt(b) (H_b is symmetric). */
void ref_rotate_inv(const double *y, int d, int b, uint64_t mask_seed, double *u)
{
    double inv = 1.0 / sqrt((double)b);
    for (int base = 0; base < d; base += b)
        for (int n = 0; n < b; ++n) {
            double acc = 0.0;
            for (int m = 0; m < b; ++m) {
                int h = parity((unsigned)(m & n)) ? -1 : 1;
                acc += h * y[base + m];
            }
            u[base + n] = ref_sign(mask_seed, base + n) * acc * inv;
        }
}

/* ------------------------------------------------------------------------ */
/* Activation-aware per-input-channel scale (explainer, "activation-aware    */
/* scaling": s_j proportional to r_j^alpha, r_j the input-channel activation */
/* statistic).  Reading: the proportionality constant is 1/mean(a)^alpha,    */
/* i.e. s_j = (a_j / mean_j a_j)^alpha, stored as binary16; with no          */
/* statistic or alpha == 0, s_j = 1.  Returns -1 on a non-positive or        */
/* non-finite statistic.                                                     */
/* ------------------------------------------------------------------------ */

int ref_channel_scales(const double *a, int d_in, double alpha, uint16_t *s_half)
{
    if (a == NULL || alpha == 0.0) {
        for (int j = 0; j < d_in; ++j)
            s_half[j] = ref_double_to_half(1.0);
        return 0;
    }
    double sum = 0.0;
    for (int j = 0; j < d_in; ++j) {
        if (!(a[j] > 0.0) || !isfinite(a[j]))
            return -1;
        sum += a[j];
    }
    double mean = sum / d_in;
    for (int j = 0; j < d_in; ++j)
        s_half[j] = ref_double_to_half(pow(a[j] / mean, alpha));
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Encoder steps 1-2 for one row: w' = w * s, r = ||w'||_2, u = w'/r,        */
/* y = R_fwd u.  Returns r (0 for a zero row, in which case y is zeroed).    */
/* ------------------------------------------------------------------------ */

static double row_to_rotated(const double *w, int d_in, int b, uint64_t mask_seed,
                             const uint16_t *s_half, double *scratch, double *y)
{
    double ss = 0.0;
    for (int j = 0; j < d_in; ++j) {
        scratch[j] = w[j] * ref_half_to_double(s_half[j]);
        ss += scratch[j] * scratch[j];
    }
    double r = sqrt(ss);
    if (r == 0.0) {
        memset(y, 0, sizeof(double) * (size_t)d_in);
        return 0.0;
    }
    for (int j = 0; j < d_in; ++j)
        scratch[j] /= r;
    ref_rotate_fwd(scratch, d_in, b, mask_seed, y);
    return r;
}

/* ------------------------------------------------------------------------ */
/* Section 3.4 eq. (1): sigma_k = mean(|z_k|) / sqrt(pi/2), the mean taken   */
/* over at most 1024 unit-normalised rows of the matrix.  Readings: the      */
/* first min(1024, #non-zero rows) non-zero rows in row order, after the     */
/* channel scaling; stored as binary16; a pair whose estimate rounds to 0    */
/* (or a matrix with no non-zero row) gets sigma = 1.                        */
/* ------------------------------------------------------------------------ */

void ref_calibrate_sigma(const double *W, int d_out, int d_in, int b, uint64_t mask_seed,
                         const uint16_t *s_half, uint16_t *sigma_half)
{
    int P = d_in / 2;
    double *sum = calloc((size_t)P, sizeof(double));
    double *scratch = malloc(sizeof(double) * (size_t)d_in);
    double *y = malloc(sizeof(double) * (size_t)d_in);
    int n_cal = 0;
    for (int i = 0; i < d_out && n_cal < 1024; ++i) {
        double r = row_to_rotated(W + (int64_t)i * d_in, d_in, b, mask_seed, s_half, scratch, y);
        if (r == 0.0)
            continue;
        for (int k = 0; k < P; ++k)
            sum[k] += hypot(y[2 * k], y[2 * k + 1]);
        ++n_cal;
    }
    double rayleigh = sqrt(M_PI / 2.0);
    for (int k = 0; k < P; ++k) {
        uint16_t h = n_cal ? ref_double_to_half(sum[k] / n_cal / rayleigh) : 0;
        if ((h & 0x7fff) == 0)
            h = ref_double_to_half(1.0);
        sigma_half[k] = h;
    }
    free(sum);
    free(scratch);
    free(y);
}

/* ------------------------------------------------------------------------ */
/* Section 3.6: nearest codebook entry in Euclidean distance.  Brute force   */
/* over j = 0..K-1 with a strict '<', so ties go to the lowest index.        */
/* codebook is K interleaved (x, y) pairs.                                   */
/* ------------------------------------------------------------------------ */

int ref_nearest(double px, double py, const double *codebook, int K)
{
    int best = 0;
    double bd = INFINITY;
    for (int j = 0; j < K; ++j) {
        double dx = px - codebook[2 * j];
        double dy = py - codebook[2 * j + 1];
        double d = dx * dx + dy * dy;
        if (d < bd) {
            bd = d;
            best = j;
        }
    }
    return best;
}

void ref_nearest_batch(const double *points, int64_t n, const double *codebook, int K,
                       int32_t *idx_out)
{
    for (int64_t t = 0; t < n; ++t)
        idx_out[t] = ref_nearest(points[2 * t], points[2 * t + 1], codebook, K);
}

/* ------------------------------------------------------------------------ */
/* Section 3.1 steps 1-5 for rows [row_begin, row_end): row norm, rotation,  */
/* pairing z_k = y_2k + i y_2k+1, division by sigma_k, nearest codeword.     */
/* A zero row is encoded as a zero row: all indices 0 and r = 0 (step 1).    */
/* Also returns the normalised points p (nullable) for near-tie checks.      */
/* ------------------------------------------------------------------------ */

void ref_encode_rows(const double *W, int d_out, int d_in, int b, uint64_t mask_seed,
                     const uint16_t *s_half, const uint16_t *sigma_half,
                     const double *codebook, int K, int row_begin, int row_end,
                     uint16_t *rnorm_half, int32_t *idx, double *points_out)
{
    (void)d_out;
    int P = d_in / 2;
    double *scratch = malloc(sizeof(double) * (size_t)d_in);
    double *y = malloc(sizeof(double) * (size_t)d_in);
    for (int i = row_begin; i < row_end; ++i) {
        double r = row_to_rotated(W + (int64_t)i * d_in, d_in, b, mask_seed, s_half, scratch, y);
        rnorm_half[i] = ref_double_to_half(r);
        for (int k = 0; k < P; ++k) {
            double sg = ref_half_to_double(sigma_half[k]);
            double px = y[2 * k] / sg;
            double py = y[2 * k + 1] / sg;
            int64_t o = (int64_t)i * P + k;
            idx[o] = (r == 0.0) ? 0 : ref_nearest(px, py, codebook, K);
            if (points_out) {
                points_out[2 * o] = px;
                points_out[2 * o + 1] = py;
            }
        }
    }
    free(scratch);
    free(y);
}

/* ------------------------------------------------------------------------ */
/* Section 3.1 step 6: bit-packed byte stream.  Reading: per row, index k    */
/* occupies stream bits [k*bits, (k+1)*bits), least significant bit first;  */
/* stream bit t is bit (t mod 8) of byte t/8; rows padded with zero bits to  */
/* a multiple of 16 bytes.                                                   */
/* ------------------------------------------------------------------------ */

void ref_pack_rows(const int32_t *idx, int n_rows, int P, int bits, int64_t row_bytes,
                   uint8_t *packed)
{
    memset(packed, 0, (size_t)(n_rows * row_bytes));
    for (int i = 0; i < n_rows; ++i)
        for (int k = 0; k < P; ++k) {
            uint32_t v = (uint32_t)idx[(int64_t)i * P + k];
            for (int t = 0; t < bits; ++t) {
                int64_t bit = (int64_t)k * bits + t;
                if ((v >> t) & 1u)
                    packed[i * row_bytes + bit / 8] |= (uint8_t)(1u << (bit % 8));
            }
        }
}

void ref_unpack_rows(const uint8_t *packed, int n_rows, int P, int bits, int64_t row_bytes,
                     int32_t *idx)
{
    for (int i = 0; i < n_rows; ++i)
        for (int k = 0; k < P; ++k) {
            uint32_t v = 0;
            for (int t = 0; t < bits; ++t) {
                int64_t bit = (int64_t)k * bits + t;
                if ((packed[i * row_bytes + bit / 8] >> (bit % 8)) & 1u)
                    v |= 1u << t;
            }
            idx[(int64_t)i * P + k] = (int32_t)v;
        }
}

/* ------------------------------------------------------------------------ */
/* Section 3.2 decoder for rows [row_begin, row_end): unpack, look up the    */
/* centroid, rescale pair k by sigma_k, reassemble, apply R_inv, multiply by */
/* the stored row norm; then undo the channel scaling (divide by s_j).       */
/* Output in fp64.                                                           */
/* ------------------------------------------------------------------------ */

void ref_decode_rows(const uint8_t *packed, int64_t row_bytes, int d_in, int b, int bits,
                     uint64_t mask_seed, const uint16_t *rnorm_half, const uint16_t *sigma_half,
                     const uint16_t *s_half, const double *codebook, int row_begin, int row_end,
                     double *W_out)
{
    int P = d_in / 2;
    int32_t *idx = malloc(sizeof(int32_t) * (size_t)P);
    double *yhat = malloc(sizeof(double) * (size_t)d_in);
    double *v = malloc(sizeof(double) * (size_t)d_in);
    for (int i = row_begin; i < row_end; ++i) {
        ref_unpack_rows(packed + (int64_t)i * row_bytes, 1, P, bits, row_bytes, idx);
        for (int k = 0; k < P; ++k) {
            double sg = ref_half_to_double(sigma_half[k]);
            yhat[2 * k] = sg * codebook[2 * idx[k]];
            yhat[2 * k + 1] = sg * codebook[2 * idx[k] + 1];
        }
        ref_rotate_inv(yhat, d_in, b, mask_seed, v);
        double r = ref_half_to_double(rnorm_half[i]);
        for (int j = 0; j < d_in; ++j)
            W_out[(int64_t)i * d_in + j] = r * v[j] / ref_half_to_double(s_half[j]);
    }
    free(idx);
    free(yhat);
    free(v);
}

/* ------------------------------------------------------------------------ */
/* The product the decoded weights feed: y[t][i] = sum_j x[t][j] W[i][j],    */
/* the plain dense definition (no rotation identity).                        */
/* ------------------------------------------------------------------------ */

void ref_gemv(const double *W, int d_out, int d_in, const double *x, int batch,
              int row_begin, int row_end, double *y)
{
    (void)d_out;
    for (int t = 0; t < batch; ++t)
        for (int i = row_begin; i < row_end; ++i) {
            double acc = 0.0;
            for (int j = 0; j < d_in; ++j)
                acc += x[(int64_t)t * d_in + j] * W[(int64_t)i * d_in + j];
            y[(int64_t)t * d_out + i] = acc;
        }
}

/* ------------------------------------------------------------------------ */
/* Section 3.6 eq. (2): Lloyd iterations for a K-entry 2D codebook on        */
/* samples of the unit circular Gaussian (the samples are an input; drawing  */
/* them is not part of the codec).  Readings: start from the first K         */
/* samples; each iteration assigns every sample to its nearest codeword      */
/* (ref_nearest), records the mean squared distance of that assignment, and  */
/* moves each codeword to the mean of its cell; an empty cell keeps its      */
/* codeword.  Runs exactly `iters` iterations.                               */
/* ------------------------------------------------------------------------ */

void ref_lloyd(const double *samples, int64_t n, int K, int iters, double *codebook,
               double *distortion)
{
    for (int j = 0; j < 2 * K; ++j)
        codebook[j] = samples[j];
    double *sx = malloc(sizeof(double) * (size_t)K);
    double *sy = malloc(sizeof(double) * (size_t)K);
    int64_t *cnt = malloc(sizeof(int64_t) * (size_t)K);
    for (int it = 0; it < iters; ++it) {
        memset(sx, 0, sizeof(double) * (size_t)K);
        memset(sy, 0, sizeof(double) * (size_t)K);
        memset(cnt, 0, sizeof(int64_t) * (size_t)K);
        double dsum = 0.0;
        for (int64_t t = 0; t < n; ++t) {
            double px = samples[2 * t], py = samples[2 * t + 1];
            int j = ref_nearest(px, py, codebook, K);
            double dx = px - codebook[2 * j], dy = py - codebook[2 * j + 1];
            dsum += dx * dx + dy * dy;
            sx[j] += px;
            sy[j] += py;
            cnt[j] += 1;
        }
        if (distortion)
            distortion[it] = dsum / (double)n;
        for (int j = 0; j < K; ++j)
            if (cnt[j] > 0) {
                codebook[2 * j] = sx[j] / (double)cnt[j];
                codebook[2 * j + 1] = sy[j] / (double)cnt[j];
            }
    }
    free(sx);
    free(sy);
    free(cnt);
}

/* ------------------------------------------------------------------------ */
/* Section 3.5, polar baseline: the amplitude |z_k|/sigma_k is quantised     */
/* with an N_a-level Lloyd-Max codebook of the unit Rayleigh density          */
/* f(r) = r exp(-r^2/2), the phase arg(z_k) is rounded to one of N_p uniform  */
/* bins, B = B_a + B_p bits per pair.  Readings: B_a = floor(B/2),            */
/* B_p = B - B_a (5 + 6 for B = 11, as the paper pairs them; 3 + 4 for        */
/* B = 7); the phase bins are centred on 2 pi i / N_p and a phase is rounded  */
/* to the nearest centre; index = i_a * N_p + i_p, so that the polar code is  */
/* an ordinary K-entry table a_i (cos phi, sin phi) for the decoder.          */
/* ------------------------------------------------------------------------ */

/* Probability mass and first moment of the unit Rayleigh density on [t0, t1)
 * (t1 = INFINITY allowed):  mass = e^{-t0^2/2} - e^{-t1^2/2};
 * int r * r e^{-r^2/2} dr = t0 e^{-t0^2/2} - t1 e^{-t1^2/2}
 *                           + sqrt(pi/2) (erf(t1/sqrt2) - erf(t0/sqrt2)). */
static void rayleigh_cell(double t0, double t1, double *mass, double *moment)
{
    double e0 = exp(-0.5 * t0 * t0);
    double e1 = isinf(t1) ? 0.0 : exp(-0.5 * t1 * t1);
    double te1 = isinf(t1) ? 0.0 : t1 * e1;
    double erf1 = isinf(t1) ? 1.0 : erf(t1 / sqrt(2.0));
    *mass = e0 - e1;
    *moment = t0 * e0 - te1 + sqrt(M_PI / 2.0) * (erf1 - erf(t0 / sqrt(2.0)));
}

/* Lloyd-Max on the continuous density: start from the equal-probability
 * thresholds t_i = sqrt(-2 ln(1 - i/N)); alternate centroids (conditional
 * means) and midpoint thresholds for `iters` iterations (20000 reach a fixed
 * point to 1e-13 for every N <= 32 the codec uses; the paper gives no count). */
void ref_rayleigh_lloyd_max(int N, int iters, double *levels)
{
    double *t = malloc(sizeof(double) * (size_t)(N + 1));
    for (int i = 0; i <= N; ++i)
        t[i] = (i == N) ? INFINITY : sqrt(-2.0 * log(1.0 - (double)i / N));
    for (int it = 0; it < iters; ++it) {
        for (int i = 0; i < N; ++i) {
            double m, mom;
            rayleigh_cell(t[i], t[i + 1], &m, &mom);
            levels[i] = mom / m;
        }
        for (int i = 1; i < N; ++i)
            t[i] = 0.5 * (levels[i - 1] + levels[i]);
    }
    for (int i = 0; i < N; ++i) {
        double m, mom;
        rayleigh_cell(t[i], t[i + 1], &m, &mom);
        levels[i] = mom / m;
    }
    free(t);
}

void ref_polar_codebook(int bits, const double *levels, double *codebook)
{
    int ba = bits / 2, Na = 1 << ba, Np = 1 << (bits - ba);
    for (int ia = 0; ia < Na; ++ia)
        for (int ip = 0; ip < Np; ++ip) {
            double phi = 2.0 * M_PI * ip / Np;
            codebook[2 * (ia * Np + ip)] = levels[ia] * cos(phi);
            codebook[2 * (ia * Np + ip) + 1] = levels[ia] * sin(phi);
        }
}

/* Amplitude: nearest level (ascending, strict '<'); phase: nearest bin centre. */
int ref_polar_index(double px, double py, const double *levels, int bits)
{
    int ba = bits / 2, Na = 1 << ba, Np = 1 << (bits - ba);
    double r = hypot(px, py);
    int ia = 0;
    double bd = INFINITY;
    for (int i = 0; i < Na; ++i) {
        double d = fabs(r - levels[i]);
        if (d < bd) {
            bd = d;
            ia = i;
        }
    }
    double u = atan2(py, px) * Np / (2.0 * M_PI);
    long ip = (long)floor(u + 0.5);
    ip = ((ip % Np) + Np) % Np;
    return ia * Np + (int)ip;
}

/* Encoder rows with the polar quantiser in place of the joint 2D one. */
void ref_encode_rows_polar(const double *W, int d_out, int d_in, int b, uint64_t mask_seed,
                           const uint16_t *s_half, const uint16_t *sigma_half,
                           const double *levels, int bits, int row_begin, int row_end,
                           uint16_t *rnorm_half, int32_t *idx, double *points_out)
{
    (void)d_out;
    int P = d_in / 2;
    double *scratch = malloc(sizeof(double) * (size_t)d_in);
    double *y = malloc(sizeof(double) * (size_t)d_in);
    for (int i = row_begin; i < row_end; ++i) {
        double r = row_to_rotated(W + (int64_t)i * d_in, d_in, b, mask_seed, s_half, scratch, y);
        rnorm_half[i] = ref_double_to_half(r);
        for (int k = 0; k < P; ++k) {
            double sg = ref_half_to_double(sigma_half[k]);
            double px = y[2 * k] / sg, py = y[2 * k + 1] / sg;
            int64_t o = (int64_t)i * P + k;
            idx[o] = (r == 0.0) ? 0 : ref_polar_index(px, py, levels, bits);
            if (points_out) {
                points_out[2 * o] = px;
                points_out[2 * o + 1] = py;
            }
        }
    }
    free(scratch);
    free(y);
}

/* ------------------------------------------------------------------------ */
/* Section 2 ("parallel work"), the d = 1 ablation the paper names as its    */
/* first follow-up: the same pipeline with a one-dimensional codebook.       */
/* Readings: each normalised coordinate of pair k (p = z_k / sigma_k; under   */
/* eq. (1)'s model each coordinate is ~ N(0, 1)) is quantised on its own to   */
/* the nearest of L = 2^(B/2) levels (ascending, strict '<', lowest index on */
/* ties); the levels are the L-level Lloyd-Max quantiser of N(0, 1); B is     */
/* even, so the scalar code spends B/2 bits per weight like the joint code    */
/* with K = 2^B; index = i_x * L + i_y, so that it is an ordinary K-entry     */
/* product table (l_ix, l_iy) for the decoder.                                */
/* ------------------------------------------------------------------------ */

/* Probability mass and first moment of N(0, 1) on [t0, t1) (infinite ends
 * allowed): mass = (erf(t1/sqrt2) - erf(t0/sqrt2)) / 2,
 * int x phi(x) dx = phi(t0) - phi(t1). */
static void gauss_cell(double t0, double t1, double *mass, double *moment)
{
    double e0 = isinf(t0) ? -1.0 : erf(t0 / sqrt(2.0));
    double e1 = isinf(t1) ? 1.0 : erf(t1 / sqrt(2.0));
    double p0 = isinf(t0) ? 0.0 : exp(-0.5 * t0 * t0) / sqrt(2.0 * M_PI);
    double p1 = isinf(t1) ? 0.0 : exp(-0.5 * t1 * t1) / sqrt(2.0 * M_PI);
    *mass = 0.5 * (e1 - e0);
    *moment = p0 - p1;
}

/* Lloyd-Max on N(0, 1): thresholds start evenly spaced on [-3, 3] (the paper
 * gives no start; N(0, 1) is log-concave, so the fixed point is unique);
 * alternate conditional means and midpoint thresholds for `iters` iterations. */
void ref_gauss_lloyd_max(int L, int iters, double *levels)
{
    double *t = malloc(sizeof(double) * (size_t)(L + 1));
    t[0] = -INFINITY;
    t[L] = INFINITY;
    for (int i = 1; i < L; ++i)
        t[i] = -3.0 + 6.0 * i / L;
    for (int it = 0; it <= iters; ++it) {
        for (int i = 0; i < L; ++i) {
            double m, mom;
            gauss_cell(t[i], t[i + 1], &m, &mom);
            levels[i] = mom / m;
        }
        if (it == iters)
            break;
        for (int i = 1; i < L; ++i)
            t[i] = 0.5 * (levels[i - 1] + levels[i]);
    }
    free(t);
}

/* Mean squared error of the quantiser with these levels (midpoint cells) on
 * N(0, 1): sum over cells of int (x - l)^2 phi = second moment - 2 l m1 + l^2 m0,
 * with int x^2 phi on [a, b) = m0 + a phi(a) - b phi(b). */
double ref_gauss_mse(int L, const double *levels)
{
    double mse = 0.0;
    for (int i = 0; i < L; ++i) {
        double a = i == 0 ? -INFINITY : 0.5 * (levels[i - 1] + levels[i]);
        double b = i == L - 1 ? INFINITY : 0.5 * (levels[i] + levels[i + 1]);
        double m0, m1;
        gauss_cell(a, b, &m0, &m1);
        double pa = isinf(a) ? 0.0 : a * exp(-0.5 * a * a) / sqrt(2.0 * M_PI);
        double pb = isinf(b) ? 0.0 : b * exp(-0.5 * b * b) / sqrt(2.0 * M_PI);
        double m2 = m0 + pa - pb;
        mse += m2 - 2.0 * levels[i] * m1 + levels[i] * levels[i] * m0;
    }
    return mse;
}

void ref_scalar_codebook(int bits, const double *levels, double *codebook)
{
    int L = 1 << (bits / 2);
    for (int ix = 0; ix < L; ++ix)
        for (int iy = 0; iy < L; ++iy) {
            codebook[2 * (ix * L + iy)] = levels[ix];
            codebook[2 * (ix * L + iy) + 1] = levels[iy];
        }
}

static int nearest_level(double v, const double *levels, int L)
{
    int best = 0;
    double bd = INFINITY;
    for (int i = 0; i < L; ++i) {
        double d = fabs(v - levels[i]);
        if (d < bd) {
            bd = d;
            best = i;
        }
    }
    return best;
}

int ref_scalar_index(double px, double py, const double *levels, int bits)
{
    int L = 1 << (bits / 2);
    return nearest_level(px, levels, L) * L + nearest_level(py, levels, L);
}

/* Encoder rows with the scalar quantiser in place of the joint 2D one. */
void ref_encode_rows_scalar(const double *W, int d_out, int d_in, int b, uint64_t mask_seed,
                            const uint16_t *s_half, const uint16_t *sigma_half,
                            const double *levels, int bits, int row_begin, int row_end,
                            uint16_t *rnorm_half, int32_t *idx, double *points_out)
{
    (void)d_out;
    int P = d_in / 2;
    double *scratch = malloc(sizeof(double) * (size_t)d_in);
    double *y = malloc(sizeof(double) * (size_t)d_in);
    for (int i = row_begin; i < row_end; ++i) {
        double r = row_to_rotated(W + (int64_t)i * d_in, d_in, b, mask_seed, s_half, scratch, y);
        rnorm_half[i] = ref_double_to_half(r);
        for (int k = 0; k < P; ++k) {
            double sg = ref_half_to_double(sigma_half[k]);
            double px = y[2 * k] / sg, py = y[2 * k + 1] / sg;
            int64_t o = (int64_t)i * P + k;
            idx[o] = (r == 0.0) ? 0 : ref_scalar_index(px, py, levels, bits);
            if (points_out) {
                points_out[2 * o] = px;
                points_out[2 * o + 1] = py;
            }
        }
    }
    free(scratch);
    free(y);
}
