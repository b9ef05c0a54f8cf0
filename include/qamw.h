/*
 * qamw.h -- C ABI of the QAM-W weight codec on NVIDIA B200 (sm_100a).
 *
 * QAM-W ("QAM-W: Joint 2D Codebook Quantization for LLM Weights via Hadamard
 * Rotation and Activation-Aware Scaling", Sharma & Dobek) stores each row w of
 * a weight matrix W (d_out x d_in) as
 *   - its L2 norm r as binary16 (section 3.1 step 1, section 3.2),
 *   - d_in/2 codebook indices of `bits` bits each, one per pair of coordinates
 *     of the rotated, pair-normalised unit row (section 3.1 steps 2-6),
 * plus, per matrix, one binary16 pair scale sigma_k per pair position
 * (section 3.4 eq. 1) and one binary16 scale s_j per input channel
 * (activation-aware scaling, s_j proportional to the channel's activation
 * statistic to the power alpha).  One codebook of K = 2^bits points in the
 * plane, trained by Lloyd iterations on the unit circular Gaussian
 * (section 3.6 eq. 2), serves every matrix.
 *
 * Conventions for every entry point:
 *   - Pointers named d_* are DEVICE pointers (current CUDA device); h_* are
 *     host pointers.  The caller allocates and owns every buffer; no entry
 *     point allocates device memory or keeps a pointer after it returns.
 *     Scratch memory comes from the caller's d_workspace, sized by
 *     qamw_workspace_bytes().
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every
 *     call only enqueues work on that stream and returns; results are ready
 *     when the stream reaches them.  Calls on different streams may run
 *     concurrently as long as they do not share output or workspace buffers.
 *   - The return value is QAMW_OK or a negative QAMW_ERR_* code, detected on
 *     the host before anything is enqueued (QAMW_ERR_CUDA: a launch failed).
 *     Nothing is enqueued when an error is returned.
 *   - Errors that depend on the data (non-finite inputs, binary16 overflow)
 *     are OR-ed into *d_status (an int32 in device memory, nullable) as
 *     QAMW_STATUS_* flags; read it after synchronising.  The outputs are still
 *     written.
 *   - Matrices are row-major and dense.  bf16 / binary16 values are passed as
 *     their 16-bit patterns (uint16_t) so that this header needs no CUDA
 *     headers.
 *   - Shape limits: d_in is a positive multiple of 64 and at most 32768; the
 *     Hadamard block is a power of two in [1, 1024] that divides d_in;
 *     1 <= bits <= 11; d_out >= 0 (0 is a no-op).
 */
#ifndef QAMW_H
#define QAMW_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define QAMW_API __attribute__((visibility("default")))
#else
#define QAMW_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ------------------------------------------------------------ return codes */
#define QAMW_OK 0
#define QAMW_ERR_INVALID (-1)   /* null pointer, bad enum or parameter          */
#define QAMW_ERR_SHAPE (-2)     /* d_in / d_out / block outside the limits      */
#define QAMW_ERR_ALIGN (-3)     /* a buffer is not 16-byte aligned              */
#define QAMW_ERR_WORKSPACE (-4) /* d_workspace missing or smaller than needed   */
#define QAMW_ERR_CUDA (-5)      /* a CUDA call or kernel launch failed          */

/* -------------------------------------------- device status flags (OR-ed) */
#define QAMW_STATUS_NONFINITE 0x1 /* NaN/Inf in W, x, or the training samples  */
#define QAMW_STATUS_RANGE 0x2     /* binary16 overflow of r, s or sigma; s_j    */
                                  /* underflowing to 0; |sample| >= 2^10        */
#define QAMW_STATUS_BAD_STAT 0x4  /* activation statistic <= 0 or non-finite;  */
                                  /* the scale of that channel is set to 1      */
#define QAMW_STATUS_TIMEOUT 0x8   /* a bounded wait for an asynchronous copy    */
                                  /* gave up; the outputs of that call are not  */
                                  /* valid                                       */

/* ------------------------------------------------------------------ enums */
#define QAMW_DTYPE_F32 0  /* W as IEEE binary32                              */
#define QAMW_DTYPE_BF16 1 /* W as bfloat16                                   */

#define QAMW_SIGMA_GIVEN 0x1  /* encode: use m->sigma as given, skip eq. (1)  */
#define QAMW_SCALES_GIVEN 0x2 /* encode: use m->chan_scale as given           */
#define QAMW_POLAR 0x4        /* encode: polar baseline quantiser (section    */
                              /* 3.5) against a qamw_polar_codebook table     */
#define QAMW_SCALAR 0x8       /* encode: d = 1 scalar quantiser (section 2)   */
                              /* against a qamw_scalar_codebook table; even   */
                              /* bits only                                    */

#define QAMW_OP_TRAIN 0
#define QAMW_OP_ENCODE 1
#define QAMW_OP_GEMV 2
#define QAMW_OP_CALIBRATE 3
#define QAMW_OP_GEMM 4

/* --------------------------------------------------------- encoded matrix */
/* All pointers are device pointers owned by the caller.  The caller fills
 * every field before qamw_encode(); qamw_encode() writes the arrays. */
typedef struct qamw_matrix {
    int32_t d_out;          /* rows of W                                     */
    int32_t d_in;           /* columns of W (input channels)                 */
    int32_t block;          /* Hadamard block size b (section 3.3)           */
    int32_t bits;           /* bits per pair B; K = 2^bits codewords         */
    uint64_t mask_seed;     /* seed of the deterministic sign mask           */
    int64_t row_bytes;      /* must equal qamw_row_bytes(d_in, bits)         */
    uint8_t *packed;        /* [d_out][row_bytes] bit-packed indices, 16B-aligned */
    uint16_t *row_norm;     /* [d_out] binary16 row norms r                   */
    uint16_t *sigma;        /* [d_in/2] binary16 pair scales sigma_k, 16B-aligned */
    uint16_t *chan_scale;   /* [d_in] binary16 channel scales s_j, 16B-aligned */
    const float *codebook;  /* [K][2] fp32 codewords (x, y), 16B-aligned      */
    const void *prefilter;  /* table from qamw_build_prefilter() for this
                               codebook, or NULL (then qamw_encode builds one
                               in its workspace on every call)                */
} qamw_matrix;

/* Packed index stream (section 3.1 step 6, 3.7): index k of a row occupies
 * stream bits [k*bits, (k+1)*bits), least significant bit first; stream bit t
 * is bit t%8 of byte t/8; rows are zero-padded to a multiple of 16 bytes. */
QAMW_API int64_t qamw_row_bytes(int d_in, int bits);

/* Section 3.3: the largest power of two dividing d_in, capped at 1024
 * (2048 -> 1024, 5632 -> 512).  Returns 0 for d_in <= 0. */
QAMW_API int qamw_default_block(int d_in);

/* Section 3.7 eq. (3): bits per weight bits/2 + 16/d_in before byte alignment. */
QAMW_API double qamw_bits_per_weight(int d_in, int bits);

/* Bytes of d_workspace needed by op (QAMW_OP_*).  TRAIN: d_out is ignored,
 * d_in is ignored, `bits` fixes K; ENCODE: includes room for a prefilter table
 * (needed when m->prefilter is NULL); CALIBRATE: row norms and partial sums of
 * qamw_calibrate_sigma; GEMV: batch columns of the rotated activation; GEMM:
 * the rotated activation of `batch` tokens and the fp32 partial sums of
 * qamw_decode_gemm (batch = tokens).
 * Returns 0 on invalid arguments. */
QAMW_API size_t qamw_workspace_bytes(int op, int d_out, int d_in, int bits, int batch);

/* Bytes of the nearest-codeword prefilter table for a 2^bits codebook. */
QAMW_API size_t qamw_prefilter_bytes(int bits);

/* Human-readable text for a QAMW_OK / QAMW_ERR_* code or a status flag word. */
QAMW_API const char *qamw_status_string(int code);

/* qamw_selftest_wait_timeout: a check of the failure path of the bounded waits
 *   (no counterpart in the paper).  One CTA waits, with the wait the kernels
 *   use on their bulk-copy rings, on an mbarrier that nothing arrives on, for
 *   `tries` polls (1 .. the kernels' own limit, 2^18: about 1 s), then ORs
 *   QAMW_STATUS_TIMEOUT into *d_status and stores the wait's clock cycles in
 *   *d_cycles (nullable, device).  The kernels give up after 2^18 polls in the
 *   same way: they flag TIMEOUT, let their copies in flight land and return,
 *   and the CUDA context stays usable.  Errors: QAMW_ERR_INVALID for tries out
 *   of range or a null status. */
QAMW_API int qamw_selftest_wait_timeout(unsigned tries, int32_t *d_status, long long *d_cycles,
                                        void *stream);

/* ------------------------------------------------------------------ calls */

/* Section 3.6 eq. (2): Lloyd iterations for the joint 2D codebook.
 *   d_samples   [n][2] fp32 draws of the unit circular Gaussian (the caller
 *               draws them; n >= 2^bits), 8-byte aligned.
 *   bits        K = 2^bits codewords, 1..11.
 *   iters       number of Lloyd iterations (>= 0).
 *   d_codebook  [K][2] fp32 output (16-byte aligned); initialised to the first
 *               K samples, then
 *               each iteration assigns every sample to its nearest codeword
 *               (lowest index on ties) and moves each codeword to the mean of
 *               its cell; an empty cell keeps its codeword.  Cell sums are
 *               accumulated in 2^-28 fixed point, so the result is bitwise
 *               reproducible.
 *   d_distortion [iters] fp64 mean squared distance of each iteration's
 *               assignment (nullable).
 *   d_workspace qamw_workspace_bytes(QAMW_OP_TRAIN, 0, 0, bits, 0) bytes,
 *               16-byte aligned (cell sums and the per-iteration prefilter
 *               table that makes the assignment exact at a few codewords per
 *               sample).
 * Samples are skipped (and flagged) when non-finite (NONFINITE) or when a
 * coordinate has |x| >= 2^10 (RANGE); n <= 2^25 keeps the fixed-point sums exact. */
QAMW_API int qamw_train_codebook(const float *d_samples, int64_t n, int bits, int iters,
                        float *d_codebook, double *d_distortion, void *d_workspace,
                        size_t ws_bytes, int32_t *d_status, void *stream);

/* Builds the exact nearest-codeword prefilter for a codebook into d_table
 * (qamw_prefilter_bytes(bits) bytes, 16B-aligned).  The table lists, for each
 * cell of a square grid over the codebook, every codeword that can be the
 * fp32 nearest codeword of a point in that cell; points off the grid are
 * searched exhaustively.  Rebuild it whenever the codebook changes. */
QAMW_API int qamw_build_prefilter(const float *d_codebook, int bits, void *d_table, size_t table_bytes,
                         void *stream);

/* Section 3.1 (encoder steps 1-6) with activation-aware per-channel scaling.
 *   d_W        [m->d_out][m->d_in] weights, dtype QAMW_DTYPE_F32 or _BF16,
 *              16B-aligned.
 *   d_act_stat [d_in] fp32 positive per-channel activation statistic (e.g.
 *              activation RMS), nullable.  s_j = binary16((a_j/mean a)^alpha);
 *              NULL or alpha == 0 gives s_j = 1.  Ignored with
 *              QAMW_SCALES_GIVEN (then m->chan_scale is read).
 *   flags      QAMW_SIGMA_GIVEN | QAMW_SCALES_GIVEN | QAMW_POLAR or QAMW_SCALAR.
 *   m          shape, block, bits, mask_seed, row_bytes and buffers (in);
 *              packed, row_norm, sigma (unless given), chan_scale (unless
 *              given) (out).
 * Per row: w' = w * s; r = ||w'||_2 (row_norm = binary16(r)); a row with
 * r = 0 is stored as r = 0 and all indices 0; else u = w'/r,
 * y = blockdiag(H_b) diag(D) u / sqrt(b) with D_j = -1 when bit 63 of
 * splitmix64((mask_seed << 32) + j) is set; z_k = (y_2k, y_2k+1) / sigma_k;
 * index_k = nearest codeword (lowest index on ties, fp32 distances).
 * sigma_k = binary16(mean |z_k| / sqrt(pi/2)) over the first min(1024,
 * #non-zero rows) non-zero rows of W*s (a pair whose sigma rounds to 0 gets 1).
 * Flags: NONFINITE, RANGE, BAD_STAT. */
QAMW_API int qamw_encode(const void *d_W, int dtype, const float *d_act_stat, float alpha, int flags,
                const qamw_matrix *m, void *d_workspace, size_t ws_bytes, int32_t *d_status,
                void *stream);

/* The three stages qamw_encode runs, for callers that reuse side values (e.g.
 * re-encoding with a fixed sigma, or encoding row shards of one matrix on
 * several GPUs with the sigma of the whole matrix).  Same arguments and
 * semantics as qamw_encode.
 *
 * qamw_channel_scales: d_scale[j] = binary16((a_j / mean a)^alpha) for
 *   j < d_in (d_in a multiple of 64); NULL d_act_stat or alpha == 0 gives 1.
 *   Flags: BAD_STAT (that channel gets 1), RANGE. */
QAMW_API int qamw_channel_scales(const float *d_act_stat, int d_in, float alpha, uint16_t *d_scale,
                                 int32_t *d_status, void *stream);

/* qamw_calibrate_sigma: section 3.4 eq. (1) over the first min(1024,
 *   #non-zero) non-zero rows of W*s; reads m->chan_scale, writes m->sigma.
 *   d_workspace: qamw_workspace_bytes(QAMW_OP_CALIBRATE, d_out, d_in, bits, 0).
 *   Flags: NONFINITE, RANGE. */
QAMW_API int qamw_calibrate_sigma(const void *d_W, int dtype, const qamw_matrix *m,
                                  void *d_workspace, size_t ws_bytes, int32_t *d_status,
                                  void *stream);

/* qamw_calibrate_many: qamw_channel_scales followed by qamw_calibrate_sigma
 *   for each of n matrices, in four kernel launches per 64 matrices instead of
 *   four per matrix (the results are bitwise those of the single calls).
 *   d_W[i]: matrix i's weights (dtype as for qamw_encode, 16B-aligned);
 *   d_act_stat: NULL, or n statistic pointers (each nullable: s = 1); alpha
 *   applies to all; ms[i]: shape, block, mask_seed and the chan_scale and
 *   sigma arrays written (packed and row_norm are not touched).  d_W,
 *   d_act_stat and ms are host arrays of n entries.  Shapes may differ;
 *   every d_out must be positive.
 *   d_workspace: qamw_calibrate_many_workspace_bytes(ms, n) bytes (16B-aligned).
 *   Errors: those of qamw_calibrate_sigma for any matrix (nothing is enqueued
 *   then).  Flags: BAD_STAT, RANGE, NONFINITE. */
QAMW_API int qamw_calibrate_many(const void *const *d_W, int dtype, const float *const *d_act_stat,
                                 float alpha, const qamw_matrix *ms, int n, void *d_workspace,
                                 size_t ws_bytes, int32_t *d_status, void *stream);

/* Bytes of d_workspace qamw_calibrate_many needs for these n matrices (0 for
 * invalid arguments). */
QAMW_API size_t qamw_calibrate_many_workspace_bytes(const qamw_matrix *ms, int n);

/* qamw_encode_rows: section 3.1 steps 1-6 for every row with the given
 *   m->chan_scale and m->sigma; writes m->packed and m->row_norm.  One kernel,
 *   no workspace.  m->prefilter may be NULL (exhaustive search; same result,
 *   slower for large K).  d_candidates (nullable, 8-byte aligned): the number
 *   of distinct list candidates the search scored is added to it (work
 *   accounting for the roofline; costs one reduction per CTA).  A row whose
 *   norm is zero, or not finite (NaN/Inf in the row; flagged NONFINITE), is
 *   stored with all indices 0.  Flags: NONFINITE, RANGE. */
QAMW_API int qamw_encode_rows(const void *d_W, int dtype, const qamw_matrix *m,
                              uint64_t *d_candidates, int32_t *d_status, void *stream);

/* qamw_normalised_pairs: the normalised points p_k = z_k / sigma_k (section
 *   3.1 steps 1-4 with the given m->chan_scale and m->sigma: the points the
 *   encoder searches, bitwise) of rows [row0, row0 + nrows), written to
 *   d_points as float pairs, row-major [nrows][d_in / 2][2] (caller-owned,
 *   16-byte aligned, nrows * d_in * 4 bytes).  Rows whose norm is zero or not
 *   finite give NaN points (qamw_train_codebook skips and flags them).  This is
 *   the input of a per-checkpoint codebook: the explainer page's "Significance
 *   and Claims" names training on the empirical normalised pairs instead of
 *   the unit circular Gaussian as a possible gain; qamw_train_codebook on
 *   these points does that.  m->packed and m->row_norm are not touched.
 *   Errors: QAMW_ERR_SHAPE for a row range outside [0, d_out).  Flags:
 *   NONFINITE. */
QAMW_API int qamw_normalised_pairs(const void *d_W, int dtype, const qamw_matrix *m, int64_t row0,
                                   int64_t nrows, float *d_points, int32_t *d_status,
                                   void *stream);

/* Section 3.5, the polar baseline: the amplitude |z_k|/sigma_k is quantised
 * with an N_a-level Lloyd-Max codebook of the unit Rayleigh density
 * r exp(-r^2/2) and the phase arg z_k is rounded to one of N_p uniform bins;
 * B = B_a + B_p bits per pair with B_a = floor(B/2) (5 + 6 for B = 11, 3 + 4 for
 * B = 7).  qamw_polar_codebook computes the levels (continuous Lloyd-Max in
 * fp64, 20000 iterations from the equal-probability partition) and writes the
 * expanded table d_codebook[ia * N_p + ip] = a_ia (cos 2 pi ip/N_p,
 * sin 2 pi ip/N_p), [2^bits][2] fp32, 16-byte aligned.  That table is an
 * ordinary codebook for qamw_decode and qamw_decode_gemv. */
QAMW_API int qamw_polar_codebook(int bits, float *d_codebook, void *stream);

/* qamw_encode_rows with the polar quantiser: amplitude to the nearest level
 * (lowest index on ties), phase to the nearest bin centre 2 pi ip/N_p; the
 * levels are read from m->codebook (a qamw_polar_codebook table); m->prefilter
 * is ignored.  Same as qamw_encode with QAMW_POLAR. */
QAMW_API int qamw_encode_rows_polar(const void *d_W, int dtype, const qamw_matrix *m,
                                    int32_t *d_status, void *stream);

/* The d = 1 ablation that section 2 ("parallel work") names as the first
 * follow-up: the same pipeline with a one-dimensional codebook.  Each
 * normalised coordinate of pair k (p = z_k / sigma_k, ~ N(0, 1) under eq. 1's
 * model) is quantised on its own to the nearest of L = 2^(bits/2) levels (lowest
 * index on ties); the levels are the L-level Lloyd-Max quantiser of N(0, 1);
 * index = i_x * L + i_y, so the scalar code spends bits/2 bits per weight like
 * the joint code with K = 2^bits.  bits must be even (2..10).
 * qamw_scalar_codebook computes the levels (fp64 Lloyd-Max iteration, 20000
 * steps from thresholds evenly spaced on [-3, 3]) and writes the product table
 * d_codebook[ix * L + iy] = (l_ix, l_iy), [2^bits][2] fp32, 16-byte aligned: an
 * ordinary codebook for qamw_decode and qamw_decode_gemv. */
QAMW_API int qamw_scalar_codebook(int bits, float *d_codebook, void *stream);

/* qamw_encode_rows with the d = 1 scalar quantiser; the levels are read from
 * m->codebook (a qamw_scalar_codebook table); m->prefilter is ignored.  Same as
 * qamw_encode with QAMW_SCALAR.  Errors: QAMW_ERR_INVALID for odd bits. */
QAMW_API int qamw_encode_rows_scalar(const void *d_W, int dtype, const qamw_matrix *m,
                                     int32_t *d_status, void *stream);

/* Section 3.2 decoder: unpack, look up the codeword, rescale pair k by
 * sigma_k, reassemble, apply R_inv = diag(D) blockdiag(H_b) / sqrt(b),
 * multiply by the row norm and divide by the channel scale.
 *   d_W_out [d_out][d_in] bf16 (round to nearest even), 16B-aligned.
 * Needs no workspace. */
QAMW_API int qamw_decode(const qamw_matrix *m, uint16_t *d_W_out, int32_t *d_status, void *stream);

/* qamw_decode for n matrices in one call: matrix i is decoded into
 * d_W_out[i] (a host array of n device pointers, each [ms[i].d_out][ms[i].d_in]
 * bf16, 16B-aligned; ms is a host array of n descriptors).  The result equals n
 * qamw_decode calls.  Matrices that share bits, codebook and the class of the
 * Hadamard block (1, or >= 2) -- consecutive in ms -- go through one kernel
 * launch (up to 64 at a time), so the per-launch set-up (the codeword table)
 * is paid once for the run and the tail of one matrix overlaps the next.
 * Shapes, blocks and seeds may differ.  Errors: those of qamw_decode for any
 * matrix (nothing is enqueued then); QAMW_ERR_INVALID for n < 0 or null
 * arrays.  Needs no workspace. */
QAMW_API int qamw_decode_many(const qamw_matrix *ms, int n, uint16_t *const *d_W_out,
                              int32_t *d_status, void *stream);

/* y = x * W_hat^T without forming W_hat: since R_inv = R_fwd^T,
 * y[t][i] = r_i * sum_k < xbar_t[k], c[index_ik] > with
 * xbar_t = sigma (.) R_fwd(x_t / s) (pair k = coordinates 2k, 2k+1).
 *   d_x [batch][d_in] bf16, 16B-aligned; 1 <= batch <= 16.
 *   d_y [batch][d_out] bf16 output (fp32 accumulation).
 *   d_workspace qamw_workspace_bytes(QAMW_OP_GEMV, d_out, d_in, bits, batch).
 * Flags: NONFINITE (non-finite x). */
QAMW_API int qamw_decode_gemv(const qamw_matrix *m, const uint16_t *d_x, int batch, uint16_t *d_y,
                     void *d_workspace, size_t ws_bytes, int32_t *d_status, void *stream);

/* qamw_decode_gemv at batch 1 for n matrices in one call: y_i = x_i * W_hat_i^T
 * (ms: host array of n descriptors; d_x, d_y: host arrays of n device
 * pointers, d_x[i] [d_in_i] bf16 16B-aligned, d_y[i] [d_out_i] bf16).  The
 * rotated activations x_bar_i are formed once each, into the workspace, and the
 * products of consecutive matrices with the same d_in, block, bits and codebook
 * share one launch (up to 64 at a time): the per-launch set-up (the replicated
 * codeword table) is paid once for the run.  Each y_i equals the
 * qamw_decode_gemv result for (ms[i], d_x[i]) bit for bit.
 *   d_workspace qamw_decode_gemv_many_workspace_bytes(ms, n) bytes, 16B-aligned.
 * Errors: those of qamw_decode_gemv for any matrix (nothing is enqueued then);
 * QAMW_ERR_INVALID for n < 0 or null arrays.  Flags: NONFINITE (non-finite x). */
QAMW_API size_t qamw_decode_gemv_many_workspace_bytes(const qamw_matrix *ms, int n);
QAMW_API int qamw_decode_gemv_many(const qamw_matrix *ms, int n, const uint16_t *const *d_x,
                                   uint16_t *const *d_y, void *d_workspace, size_t ws_bytes,
                                   int32_t *d_status, void *stream);

/* Prefill-size product Y = X * W_hat^T for many tokens, on the tensor cores,
 * without forming W_hat (the form the paper's section 1 leaves to future work:
 * fused kernels for latency).  The same identity as qamw_decode_gemv:
 * Y[t][i] = r_i * sum_k < xbar_t[k], c[index_ik] >, xbar_t = sigma (.)
 * R_fwd(x_t / s), as a dense contraction of gathered codewords with xbar
 * (binary16 high and low parts of both, fp32 accumulation).
 *   d_x [ntok][d_in] bf16, 16B-aligned; 1 <= ntok <= 65536.
 *   d_y [ntok][d_out] bf16 output.
 *   d_workspace qamw_workspace_bytes(QAMW_OP_GEMM, d_out, d_in, bits, ntok),
 *     queried with the same device current (the work is shared out over its
 *     SMs, and the partial sums of that split live in the workspace).
 * The result is deterministic for a given device (fixed split, fixed order of
 * the partial sums).
 * Flags: NONFINITE (non-finite x), RANGE (|xbar| beyond binary16), TIMEOUT (a
 * bounded wait inside the kernel ran out; the output is then not valid). */
QAMW_API int qamw_decode_gemm(const qamw_matrix *m, const uint16_t *d_x, int ntok, uint16_t *d_y,
                              void *d_workspace, size_t ws_bytes, int32_t *d_status, void *stream);

/* Allocation-free variant of qamw_decode_gemv.  The paper has no counterpart:
 * this entry point exists for callers that cannot allocate device memory,
 * neither a workspace nor anything else -- plugins whose interface hands over
 * only input and output pointers, engines that reserve all free device memory
 * for their own pools up front, and latency-critical loops that must not call
 * cudaMalloc/cudaFree because those synchronise the device.
 *   Same arguments and result as qamw_decode_gemv minus the workspace: the
 *   rotated activation lives in a fixed 1 MiB array in device memory that the
 *   library reserves on every GPU that loads it, held until the process exits.
 *   Limit: padded_batch * d_in/2 <= 131072, where padded_batch is batch rounded
 *   up to 1, 4, 8 or 16 (e.g. batch 16 with d_in <= 16384, or batch 1 with any
 *   d_in the library accepts); larger problems return QAMW_ERR_SHAPE and
 *   enqueue nothing.
 *   The first call on each device looks up that array's device address (with
 *   the device current) and caches it with the device's CUDA context, looking
 *   it up again if that context is ever recreated (e.g. after
 *   cudaDeviceReset); make that first call before any stream capture.  With
 *   lazy module loading (the CUDA default) the array is reserved on a device
 *   only when the library's device code first loads there, so a caller that
 *   reserves all free device memory for itself should make one library call
 *   on each device before doing so.  The call allocates nothing and calls no
 *   allocating routine.
 *   Every call on a device uses the same array, which keeps the previous
 *   call's contents (each call overwrites everything it reads): calls whose
 *   work overlaps on the GPU -- e.g. on two streams at once -- race on it, so
 *   serialise them. */
QAMW_API int qamw_decode_gemv_noalloc(const qamw_matrix *m, const uint16_t *d_x, int batch,
                                      uint16_t *d_y, int32_t *d_status, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* QAMW_H */
