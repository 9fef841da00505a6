/*
 * gptq.h -- C ABI of the B200 (sm_100a) GPTQ per-layer quantization library.
 *
 * The library implements GPTQ's one-shot quantization of ONE linear layer:
 *
 *   1. gptq_hessian_accum   H += alpha * X^T X over chunks of calibration
 *                           tokens (GPTQ knowledge note, "How It Works": the
 *                           layer-output reconstruction loss has Hessian
 *                           H = 2 X X^T; alpha = 2/N reproduces it).
 *   2. gptq_prepare_hinv    dead columns, relative damping, the optional
 *                           act-order permutation and the upper factor U with
 *                           U^T U = (H + lambda I)^-1 (knowledge note, "How It
 *                           Works": a damped Cholesky formulation supplies the
 *                           correction rows; anthology record SOTA-185: the
 *                           reordering trick).
 *   3. gptq_quantize_layer  the column loop: every row follows one column
 *                           order, each column is rounded to the low-bit grid
 *                           and its scaled error is pushed into the columns not
 *                           yet quantized; 128-column blocks batch the
 *                           corrections before one global update of the rest
 *                           (knowledge note, "How It Works"; "Daily Papers"
 *                           GPTQ-2D abstract: fixed order, triangular feedback).
 *   4. gptq_pack            codes to a packed low-bit stream (knowledge note,
 *                           "Tradeoffs": deployment reads packed weights).
 *
 * plus gptq_quantize_rtn, the round-to-nearest baseline on the same grid
 * (knowledge note, "Common Confusions"), gptq_dequant_matvec (inference with
 * the packed weights) and gptq2d_round (GPTQ-2D, the two-sided task of the
 * GPTQ-2D abstract on the "Daily Papers" page).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Every array pointer is a DEVICE pointer on the current CUDA device, owned
 *   by the caller.  The library allocates no device memory: scratch comes from
 *   the caller's workspace `ws` (size from the matching *_workspace_size call;
 *   ws may be NULL when that size is 0).  Workspaces must be 256-byte aligned.
 * - Matrices are row-major with contiguous rows.
 * - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *   stream).  All calls are asynchronous on `stream` except
 *   gptq_prepare_hinv, which synchronizes `stream` once to report a failed
 *   factorization.
 * - Arguments are validated before anything is launched; an invalid call
 *   returns GPTQ_ERR_INVALID_ARG (or GPTQ_ERR_UNSUPPORTED for a valid but
 *   unimplemented combination) and touches no memory.  A launch failure
 *   returns GPTQ_ERR_CUDA.  No C++ exception crosses this boundary.
 * - Kernels that wait on other threads (pipeline barriers) bound every wait;
 *   a wait that runs out sets GPTQ_ERR_TIMEOUT in the library's device status
 *   word, which gptq_get_device_status() reads and clears.
 *
 * Grid (a reading; the pages fix only "a fixed low-bit grid" with one scale per
 * group, encyclopedia "GPTQ", "Technical Approach"): asymmetric min-max over
 * the group, widened to include 0 (an all-zero group uses [0, 1]);
 *   scale = (xmax - xmin) / maxq,  zero = rint(-xmin / scale),
 *   code  = clamp(rint(w / scale) + zero, 0, maxq),  maxq = 2^bits - 1,
 * every step an IEEE float32 operation with round-half-to-even rint.
 */
#ifndef GPTQ_B200_GPTQ_H
#define GPTQ_B200_GPTQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  GPTQ_OK = 0,
  GPTQ_ERR_INVALID_ARG = 1,  /* bad pointer, size, alignment or option        */
  GPTQ_ERR_NOT_PD = 2,       /* damped Hessian has a Cholesky pivot <= 0      */
  GPTQ_ERR_NONFINITE = 3,    /* NaN/Inf met in H (or in a pivot)              */
  GPTQ_ERR_CUDA = 4,         /* a CUDA runtime/driver call failed             */
  GPTQ_ERR_UNSUPPORTED = 5,  /* valid request this build does not implement   */
  GPTQ_ERR_TIMEOUT = 6       /* a bounded in-kernel wait ran out              */
} gptq_status;

typedef enum { GPTQ_F32 = 0, GPTQ_BF16 = 1 } gptq_dtype;

/* Human-readable name of a status code (static string, never NULL). */
const char* gptq_status_string(gptq_status status);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int32_t gptq_version(void);

/* Number of CUDA kernels this library has launched in the process so far
 * (all devices).  Lets a caller count the kernels inside a timed region. */
uint64_t gptq_kernel_launches(void);

/* Reads and clears the device status word that asynchronous kernels set when
 * a bounded wait runs out (GPTQ_ERR_TIMEOUT); synchronizes `stream`.  The
 * first failure since the last read is kept. */
gptq_status gptq_get_device_status(void* stream);

/* Tracing: per-kernel device time.
 *
 * The pages have no counterpart to this; it is the measurement hook that
 * reports where a layer pass spends its time.  While enabled, every kernel
 * this library launches (from any host thread) is bracketed by two CUDA
 * events recorded on its stream; the events cost a few microseconds of host
 * time per launch, so leave tracing off in timed work.
 * gptq_trace_read waits for the recorded launches to finish and writes, per
 * kernel (name without namespaces and parameters, e.g.
 * "gptq_block_kernel<16>"), the launches and the summed device milliseconds
 * since the previous read into out[0 .. max_entries), largest time first.  It
 * returns the number of entries written (at most max_entries), or -1 if an
 * event could not be read (the records are dropped either way). */
typedef struct {
  char name[64];
  uint64_t launches;
  double ms;
} gptq_trace_entry;
void gptq_trace_enable(int32_t on);
int32_t gptq_trace_read(gptq_trace_entry* out, int32_t max_entries);

/* Bound, in nanoseconds, on every in-kernel pipeline wait of later launches
 * (default 2 s; UINT64_MAX restores the default).  A wait that runs out
 * records GPTQ_ERR_TIMEOUT in the device status word; the kernel then lets its
 * own in-flight copies and tensor-core work finish (separately bounded),
 * releases its tensor memory and returns, so the context stays usable.  Meant
 * for tests of that failure path: 0 makes the first wait that is not already
 * satisfied give up. */
void gptq_set_wait_limit_ns(uint64_t ns);

/* Column loop of gptq_quantize_layer (process-wide, read at each call, safe
 * to set from any thread; GPTQ knowledge note, "How It Works": 128-column
 * blocks whose corrections accumulate before one global update).
 *   0 (default): per block, one quantize-and-propagate kernel over all rows
 *      and one tensor-core update of the rest of its 1024-column super-block,
 *      chained by programmatic dependent launch; one update per super-block
 *      for the rest of the matrix.
 *   1: the fused single pass per row slab: one launch per super-block in
 *      which each CTA takes its rows through all of the super-block's blocks,
 *      applying the earlier blocks' corrections left-looking (fp32, CUDA
 *      cores) before each block's chain; the same outer updates.  Used where
 *      it applies (n >= 2048, block 128, groups that divide 128 or one group
 *      per row, at most 32 rows per SM), the default loop elsewhere.  Same
 *      sums in another order: codes agree with mode 0 to fp32 rounding.
 * Other values select 0. */
void gptq_set_column_loop(int32_t mode);
int32_t gptq_get_column_loop(void);

/* ------------------------------------------------------------------------ */
/* 1. Hessian accumulation                                                   */
/* ------------------------------------------------------------------------ */

/* Bytes of workspace gptq_hessian_accum needs for n features, n_tok tokens. */
size_t gptq_hessian_workspace_size(int32_t n, int64_t n_tok);

/* H += alpha * X^T X  (and hdiag += alpha * sum_t X[t,i]^2 in fp64).
 *
 * Source: GPTQ knowledge note, "How It Works" (H = 2 X X^T from recorded layer
 * inputs).  The pages store X as features x tokens; here X is token-major,
 * X[t, i] = input feature i of calibration token t, so X^T X is the same
 * matrix.  Call once per chunk of tokens with alpha = 2 / N_total.
 *
 *   H      fp32 [n, n], accumulated in place; both triangles are written, so H
 *          stays exactly symmetric.  Products are bf16 x bf16 (exact in fp32)
 *          accumulated in fp32 on the tensor cores.
 *   hdiag  fp64 [n] or NULL.  When given, also accumulates the diagonal
 *          alpha * sum_t X[t,i]^2 in fp64 with a fixed summation order; it is
 *          the key gptq_prepare_hinv uses for act-order and dead columns.
 *   X      bf16 [n_tok, ldx] (first n columns used), 16-byte aligned,
 *          ldx >= n and ldx % 8 == 0 (TMA row pitch is a multiple of 16 bytes).
 *   n      1 <= n <= 65535.   0 <= n_tok < 2^31 - 128 (n_tok == 0 is a no-op).
 *   ws     workspace of at least gptq_hessian_workspace_size(n, n_tok) bytes.
 * Deterministic: the same inputs give bit-identical H and hdiag.
 */
gptq_status gptq_hessian_accum(float* H, double* hdiag, const void* X,
                               int64_t n_tok, int32_t n, int64_t ldx, float alpha,
                               void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------ */
/* 2. Damping, act-order and the upper inverse factor                        */
/* ------------------------------------------------------------------------ */

/* Bytes of workspace gptq_prepare_hinv needs for an n x n Hessian. */
size_t gptq_prepare_workspace_size(int32_t n);

/* Builds U (upper, U^T U = (P^T H' P)^-1) from the accumulated Hessian.
 *
 * Source: GPTQ knowledge note, "How It Works" (damped Cholesky formulation of
 * the inverse Hessian); anthology record SOTA-185 (the reordering trick).
 * Steps: a column i with key_i == 0 is dead (H_ii := 1; the quantize call
 * zeroes its weights); lambda = damp * mean(diag H) after that fix;
 * H' = H + lambda I; with act_order, perm = stable argsort of -key (ties keep
 * the lower column first), else the identity; U is computed as
 * J * inv(chol(J P^T H' P J)) * J with J the order reversal (one Cholesky and
 * one triangular inverse), which equals the upper Cholesky factor of the
 * inverse.
 *
 *   H        fp32 [n, n] symmetric, read only (entries of either triangle are
 *            read, so both must hold the same values, as gptq_hessian_accum
 *            writes them).
 *   hdiag    fp64 [n] or NULL: the key for dead columns and act-order
 *            (NULL: the fp32 diagonal of H).
 *   damp     relative damping, >= 0 and finite.
 *   perm     int32 [n] out: processing position -> original column.  May be
 *            NULL only when act_order == 0.
 *   dead     uint8 [n] out (1 = dead column, original order) or NULL.
 *   U        fp32 [n, n] out, processing order; the strict lower triangle is
 *            written as 0.
 *   ws       workspace of at least gptq_prepare_workspace_size(n) bytes.
 * Returns GPTQ_ERR_NOT_PD when a pivot is <= 0 and GPTQ_ERR_NONFINITE when H
 * holds NaN/Inf; U is then unspecified.  Synchronizes `stream`.
 */
gptq_status gptq_prepare_hinv(const float* H, const double* hdiag, int32_t n,
                              float damp, int32_t act_order, int32_t* perm,
                              uint8_t* dead, float* U, void* ws, size_t ws_bytes,
                              void* stream);

/* ------------------------------------------------------------------------ */
/* 3. The column loop                                                        */
/* ------------------------------------------------------------------------ */

/* Bytes of workspace gptq_quantize_layer needs. */
size_t gptq_quantize_workspace_size(int64_t rows, int32_t n, int32_t block);

/* Number of groups per row: ceil(n / group), or 1 when group == 0. */
int32_t gptq_num_groups(int32_t n, int32_t group);

/* GPTQ column loop over one layer.
 *
 * Source: GPTQ knowledge note, "How It Works" and "Common Confusions";
 * "Daily Papers" GPTQ-2D abstract (fixed order, triangular feedback);
 * encyclopedia "GPTQ", "Technical Approach" (bit widths, per-group scales).
 * For every block [i1, i2) of `block` processing positions and every j in it:
 * when a group starts at j its (scale, zero) are fixed from the current
 * weights of the group's columns; column j is rounded; its scaled error
 * e_j = (w_j - deq_j) / U_jj is subtracted as e_j * U[j, k] from the later
 * columns k of the block.  After the block, W[:, i2:] -= E[:, i1:i2] U[i1:i2, i2:].
 *
 *   W        [rows, n] weights (wdt = GPTQ_F32 or GPTQ_BF16), original column
 *            order, read only.
 *   U, perm, dead   from gptq_prepare_hinv (perm/dead may be NULL: identity /
 *            no dead columns).
 *   bits     2, 3, 4 or 8.
 *   group    0 (one group per row, fixed from the row before any update) or
 *            1..n; groups are contiguous in processing order and the last one
 *            may be short.  group and block must nest: block % group == 0 or
 *            group % block == 0.
 *   block    lazy-batch width, a multiple of 32 in [32, 128] (128 in GPTQ).
 * Outputs (all required unless marked optional):
 *   codes    uint8 [rows, n], original column order.
 *   scales   fp32  [rows, n_groups], group index in processing order.
 *   zeros    uint8 [rows, n_groups].
 *   g_idx    int32 [n] optional: original column -> group index.
 *   Wq_out   fp32 [rows, n] optional: scale * (code - zero), original order.
 *   row_loss fp32 [rows] optional: sum_j e_j^2, which equals
 *            (w - q)^T H' (w - q) for the row.
 *   ws       workspace of at least gptq_quantize_workspace_size(rows, n, block).
 */
gptq_status gptq_quantize_layer(const void* W, gptq_dtype wdt, int64_t rows,
                                int32_t n, const float* U, const int32_t* perm,
                                const uint8_t* dead, int32_t bits, int32_t group,
                                int32_t block, uint8_t* codes, float* scales,
                                uint8_t* zeros, int32_t* g_idx, float* Wq_out,
                                float* row_loss, void* ws, size_t ws_bytes,
                                void* stream);

/* Allocation-free variant of gptq_quantize_layer.
 *
 * The pages have no counterpart to this call; it exists for callers that
 * cannot provide a workspace: code that must not call cudaMalloc or cudaFree
 * (cudaFree synchronizes the whole device), plugins inside a host application
 * that owns all device memory through its own pool, and callers not allowed
 * to allocate at all.  Same arguments, outputs and kernels as
 * gptq_quantize_layer, minus ws / ws_bytes: the scratch is a fixed device array
 * of GPTQ_NOALLOC_SCRATCH_BYTES compiled into the library, which every GPU that
 * loads the library holds until the process exits.
 *   - Layers whose gptq_quantize_workspace_size(rows, n, block) exceeds
 *     GPTQ_NOALLOC_SCRATCH_BYTES are rejected with GPTQ_ERR_INVALID_ARG
 *     (e.g. 1024 x 1024 fits, 1024 x 2048 does not).
 *   - The first call on a device looks up the array's device address (with
 *     that device current); make that first call before any stream capture.
 *     The address is kept for the life of the process: after cudaDeviceReset
 *     (or in another context on the same device) it is stale, so do not call
 *     this entry point again in that process after a reset.
 *   - All calls share the array: calls whose kernels overlap on the GPU race
 *     and give wrong results.  The array keeps the last call's contents; the
 *     column loop writes every scratch byte before reading it.
 *   - It allocates nothing (no cudaMalloc, cudaFree or allocating routine). */
#define GPTQ_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
gptq_status gptq_quantize_layer_noalloc(const void* W, gptq_dtype wdt, int64_t rows,
                                        int32_t n, const float* U, const int32_t* perm,
                                        const uint8_t* dead, int32_t bits, int32_t group,
                                        int32_t block, uint8_t* codes, float* scales,
                                        uint8_t* zeros, int32_t* g_idx, float* Wq_out,
                                        float* row_loss, void* stream);

/* Round-to-nearest on the same grid (groups of `group` original columns, 0 =
 * per row); the baseline GPTQ improves on (knowledge note, "Why It Exists").
 * Outputs as in gptq_quantize_layer.  Needs no workspace. */
gptq_status gptq_quantize_rtn(const void* W, gptq_dtype wdt, int64_t rows,
                              int32_t n, int32_t bits, int32_t group,
                              uint8_t* codes, float* scales, uint8_t* zeros,
                              void* stream);

/* ------------------------------------------------------------------------ */
/* 4. Packing                                                                */
/* ------------------------------------------------------------------------ */

/* 32-bit words per packed row: bits * ceil(n / 32). */
int32_t gptq_packed_words_per_row(int32_t n, int32_t bits);

/* Packs codes [rows, n] (each < 2^bits) into uint32 [rows, words_per_row].
 *
 * Source: GPTQ knowledge note, "Tradeoffs" (packed-weight kernels); the format
 * is a reading, as the pages give none: each row is a little-endian bitstream,
 * code j at bits [j*bits, (j+1)*bits); a row is padded with zero codes to a
 * multiple of 32 codes, so each run of 32 codes fills exactly `bits` words.
 * Works for the zero points too (pass zeros as codes with n = n_groups).
 * Codes >= 2^bits are masked to their low `bits` bits.
 */
gptq_status gptq_pack(const uint8_t* codes, int64_t rows, int32_t n, int32_t bits,
                      uint32_t* packed, void* stream);

/* ------------------------------------------------------------------------ */
/* 5. Inference with the packed weights                                      */
/* ------------------------------------------------------------------------ */

/* Bytes of workspace gptq_dequant_matvec needs: 0 in this version (x is read
 * in place in either dtype); kept so that callers size it the usual way. */
size_t gptq_matvec_workspace_size(int32_t n, int32_t batch, gptq_dtype xdt);

/* y[b, r] = sum_c Q[r, c] * x[b, c] for b < batch, r < rows, where
 * Q[r, c] = scales[r, g(c)] * (code[r, c] - zeros[r, g(c)]) is read straight
 * from the packed rows; g(c) = g_idx[c] when g_idx is given (act-order), else
 * c / group (group 0: one group per row).
 *
 * Source: the GPTQ abstract on the "Daily Papers" page (the packed 3/4-bit
 * weights run generative inference faster than FP16) and the GPTQ knowledge
 * note, "Tradeoffs" (deployment reads packed weights).  The arithmetic is the
 * grid's dequantization (scale * (code - zero)) applied to the packed format
 * of gptq_pack.
 *
 *   packed   uint32 [rows, gptq_packed_words_per_row(n, bits)], codes in
 *            ORIGINAL column order (as gptq_quantize_layer returns them, then
 *            gptq_pack), 4-byte aligned
 *   scales   fp32 [rows, n_groups]; zeros uint8 [rows, n_groups]
 *   g_idx    int32 [n] group of each original column, or NULL
 *   x        [batch, n] (xdt = GPTQ_F32 or GPTQ_BF16), 1 <= batch <= 8
 *   y        fp32 [batch, rows], written
 *   ws       gptq_matvec_workspace_size(n, batch, xdt) bytes (256-byte aligned;
 *            may be NULL when that is 0, as it is in this version)
 * Accumulates in fp32.  4-bit codes with bf16 x, n a multiple of 128, groups
 * of a multiple of 128 columns (or one group per row), no g_idx, and packed
 * and x 16-byte aligned run on the tensor cores (mma.sync, bf16 operands
 * 128 + code and x, which are exact; fp32 sums of s (128 + code) x per
 * 128-column block, the 128 offsets subtracted once per output); every other
 * case runs the general kernel.  Asynchronous on `stream`.
 * Errors: GPTQ_ERR_INVALID_ARG (sizes, bits not in {2,3,4,8}, group > n,
 * batch outside 1..8, NULL or misaligned pointers, small workspace), before any
 * launch; GPTQ_ERR_CUDA. */
gptq_status gptq_dequant_matvec(const uint32_t* packed, const float* scales, const uint8_t* zeros,
                                const int32_t* g_idx, int64_t rows, int32_t n, int32_t bits, int32_t group,
                                const void* x, gptq_dtype xdt, int32_t batch, float* y, void* ws,
                                size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------ */
/* 6. GPTQ-2D: two-sided rounding                                            */
/* ------------------------------------------------------------------------ */

/* Bytes of workspace gptq2d_round needs for an m x n matrix (0 for sizes it
 * rejects). */
size_t gptq2d_workspace_size(int64_t m, int64_t n);

/* Rounds W [m, n] to scale * integers under ||A (W - Q) B||_F^2, where only
 * the Grams HL = A^T A and HR = B B^T enter, through their upper inverse
 * factors:
 *   UL  fp32 [m, m], UL^T UL = HL^-1, upper (entries below the diagonal are
 *       never read), e.g. gptq_prepare_hinv(HL, NULL, m, 0, 0, ...);
 *   UR  fp32 [n, n], UR^T UR = HR^-1, upper, likewise.
 *
 * Source: the GPTQ-2D abstract on the "Daily Papers" page.  The
 * one-dimensional algorithm (fixed order, each rounding error fed forward
 * through a triangular matrix) applied to vec(W) under the Kronecker Gram
 * HL kron HR, computed anti-diagonal by anti-diagonal in cubic time: entry
 * (i, j) is rounded at
 *     v = W[i, j] - sum_{i' <= i} UL[i', i] * (E UR)[i', j]
 * (E: the scaled errors of the entries already rounded, all of which lie
 * above and to the left), q = rint(v / scale) (IEEE fp32 division, round half
 * to even), clamped to [qmin, qmax] when clamp == 1, and its scaled error is
 * e = (v - scale * q) / (UL[i, i] * UR[j, j]).  With HL = I this is the
 * one-sided GPTQ column loop on every row with Hessian HR.
 *
 *   W       [m, n] fp32 or bf16 (wdt), row-major
 *   scale   grid step, finite and > 0
 *   clamp   0 (unbounded integers) or 1 (clamp to [qmin, qmax],
 *           -2^24 <= qmin <= qmax <= 2^24)
 *   codes   int32 [m, n] out: the integers q (Q = scale * codes)
 *   E       fp32 [m, n] out, the scaled errors e, or NULL.  They satisfy
 *           W - Q = UL^T E UR and tr(HL (W - Q) HR (W - Q)^T) = sum e^2.
 *   ws      gptq2d_workspace_size(m, n) bytes, 256-byte aligned
 * Accumulates in fp32 on the CUDA cores; about 2 * (m + n) / 64 kernel
 * launches, on two streams the library keeps per device (the tile rounds on a
 * high-priority one, the pushes to tiles two or more wavefronts ahead on a
 * low-priority one), joined to `stream` by events: asynchronous on `stream`;
 * calls from several host threads on one device share those streams and run
 * one after another.  Codes for non-finite inputs are unspecified.
 * Errors: GPTQ_ERR_INVALID_ARG (negative sizes or sizes above 4,194,304, a bad
 * dtype, scale or clamp range, NULL or misaligned pointers, small workspace),
 * before any launch; GPTQ_ERR_CUDA. */
gptq_status gptq2d_round(const void* W, gptq_dtype wdt, int64_t m, int64_t n,
                         const float* UL, const float* UR, float scale, int32_t clamp,
                         int32_t qmin, int32_t qmax, int32_t* codes, float* E,
                         void* ws, size_t ws_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* GPTQ_B200_GPTQ_H */
