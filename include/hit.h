/*
 * hit.h -- C ABI of libhit.so: batched randomized Walsh-Hadamard transforms,
 * mixed-radix butterfly rotations, fused group quantization and the sparse
 * Walsh-Hadamard adapter expansion, as CUDA kernels for sm_100a (B200).
 *
 * Sources (page title, section):
 *  [HARP]  "HARP: Hadamard-Preconditioned Adaptive Rotation Processor for
 *          Extreme LLM Quantization", technical summary: §1 problem statement
 *          (randomized Hadamard transform, O(d log d), exactly orthogonal);
 *          §2.1 core architecture (mixed-radix schedule, stride stages of
 *          block-diagonal orthogonal matrices); §2.2 Hadamard preconditioning
 *          (normalized Sylvester mixer, zero init recovers the RHT); §2.4
 *          deployment (fused stride-stage kernel); §5 (two-sided processor,
 *          exact change of basis).
 *  [QWHA]  "QWHA: Quantization-Aware Walsh-Hadamard Adaptation for
 *          Parameter-Efficient Fine-Tuning on Large Language Models",
 *          technical summary: §2.1 adapter design (dW = F H^-1, F sparse from a
 *          value vector c and an index list E; +-1 kernel, add/subtract only);
 *          §4 results (scatter operations).
 *
 * Conventions shared by every entry point
 *  - Every tensor pointer is a DEVICE pointer owned by the caller.  The
 *    library never allocates; ops that need an fp32 intermediate take a
 *    caller-supplied workspace whose size hit_workspace_bytes() reports.
 *  - Matrices are row-major [rows, n] with a leading dimension `ld` counted in
 *    elements (ld >= n).  axis = 1 transforms every row (length n); axis = 0
 *    transforms every column (length rows).
 *  - H_n is the Sylvester Hadamard matrix (H[i][j] = (-1)^popcount(i & j)).
 *    The forward transform of a length-n vector is y = H_n diag(s) x / sqrt(n)
 *    and the inverse is x = diag(s) H_n y / sqrt(n).  A NULL sign pointer means
 *    s = +1 everywhere.  Signs are int8 values +1 or -1 (any negative byte is
 *    read as -1, anything else as +1).
 *  - dtype codes: HIT_F32 (IEEE binary32) and HIT_BF16 (bfloat16).  All
 *    arithmetic is fp32; bf16 outputs are rounded to nearest-even once.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Calls are asynchronous and stream-ordered; no call synchronizes.
 *  - Return value: HIT_OK (0) or a negative status.  All argument checks run on
 *    the host before any launch, so a rejected call launches nothing and
 *    touches no memory.  hit_last_error() gives a message for the last failed
 *    call on the calling thread.  There is no CPU fallback.
 *  - Alignment: device base pointers must be 16-byte aligned and every row
 *    start must be aligned to the vector width the kernel uses (16 bytes for
 *    fp32 / 8 bytes for bf16 when the transform length is >= 4); violations
 *    return HIT_EALIGN.
 *  - Sizes: power-of-two transform lengths 1 .. 32768 along rows; any
 *    power-of-two length up to 2^24 along columns.
 */
#ifndef HIT_H_
#define HIT_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define HIT_API __attribute__((visibility("default")))
#else
#define HIT_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define HIT_OK 0
#define HIT_EINVAL (-1)       /* bad shape, size, pointer or parameter */
#define HIT_EUNSUPPORTED (-2) /* dtype / size combination not provided */
#define HIT_EALIGN (-3)       /* pointer or leading dimension misaligned */
#define HIT_ECUDA (-4)        /* a CUDA launch or attribute call failed */
#define HIT_EWORKSPACE (-5)   /* workspace missing or too small */
#define HIT_ETIMEOUT (-6)     /* a bounded device-side wait gave up (see hit_wait_timeouts) */

#define HIT_F32 0
#define HIT_BF16 1

/* operation codes for hit_workspace_bytes */
#define HIT_OP_RHT 0        /* rht_forward / rht_inverse: flags = axis */
#define HIT_OP_QUANT 1      /* rht_quantize_pack: flags = 1 if two-sided */
#define HIT_OP_DEQUANT 2    /* dequant_inverse: flags = 1 if two-sided */
#define HIT_OP_BUTTERFLY 3  /* butterfly_apply: flags = number of stages */

/* Library version as 10000*major + 100*minor + patch. */
HIT_API int hit_version(void);

/* Static text for a status code. */
HIT_API const char* hit_status_string(int status);

/* Message describing the last failed call made by this host thread ("" if none). */
HIT_API const char* hit_last_error(void);

/* Bytes of workspace the op needs for a [rows, n] problem with output dtype
 * `dtype_out` (0 means the op needs none).  Workspace must be 16-byte aligned. */
HIT_API size_t hit_workspace_bytes(int op, int64_t rows, int64_t n, int dtype_out, int flags);

/*
 * Bounded device-side waits (not an operation of the pages; failure reporting).
 * The persistent row kernels (row lengths 4096 and 5120) wait on shared-memory barriers
 * for their row copies.  Every such wait is bounded (2 s): one that gives up
 * stops its warp, leaves that launch's outputs undefined, and increments a
 * per-device counter instead of hanging the GPU.  Launches cannot report this
 * through their return value (they are asynchronous), so:
 *
 * hit_wait_timeouts: synchronizes the current device (cudaDeviceSynchronize),
 *   adds the number of waits that gave up on it since the library was loaded
 *   (or since the last reset) to *count, and clears the counter when `reset`
 *   is nonzero.  Returns HIT_OK when the count is zero, HIT_ETIMEOUT when it is
 *   not (every output written since the last check is then suspect), and
 *   HIT_ECUDA if the device could not be read.  count may be NULL.
 *
 * hit_wait_selftest: launches on `stream` one warp that waits, through the
 *   same bounded-wait routine and counter, on a barrier that nothing ever
 *   completes, giving up after limit_ns nanoseconds (1000 <= limit_ns <=
 *   1000000000); a following hit_wait_timeouts then reports it.  Nothing is
 *   left in flight, so the context stays usable.
 */
HIT_API int hit_wait_timeouts(unsigned long long* count, int reset);
HIT_API int hit_wait_selftest(int64_t limit_ns, void* stream);

/*
 * Randomized Hadamard transform [HARP §1, §2.2; QWHA §2.1].
 * x: [rows, n] (dtype_in, leading dim ldx), y: [rows, n] (dtype_out, ldy).
 * axis = 1: every row y_r = H_n diag(signs) x_r / sqrt(n), signs length n.
 * axis = 0: every column, transform length rows, signs length rows.
 * x == y (same ld and dtype) is allowed.  Along rows n must be a power of two
 * <= 32768; along columns rows must be a power of two <= 2^24.  A column
 * transform longer than 128 runs in several passes over y: when dtype_out is
 * bf16 those passes need hit_workspace_bytes(HIT_OP_RHT, rows, n, dtype_out, 0)
 * bytes of fp32 workspace; otherwise workspace may be NULL.
 */
HIT_API int rht_forward(const void* x, void* y, int64_t rows, int64_t n, int64_t ldx, int64_t ldy,
                int dtype_in, int dtype_out, const int8_t* signs, int axis,
                void* workspace, size_t workspace_bytes, void* stream);

/* Inverse transform x = diag(signs) H y / sqrt(n); same arguments as rht_forward. */
HIT_API int rht_inverse(const void* x, void* y, int64_t rows, int64_t n, int64_t ldx, int64_t ldy,
                int dtype_in, int dtype_out, const int8_t* signs, int axis,
                void* workspace, size_t workspace_bytes, void* stream);

/*
 * Mixed-radix stride butterfly rotation y = R x [HARP §2.1, §2.2, §2.4].
 * The transform length L (= n for axis 1, = rows for axis 0) is written
 * L = b_0 * ... * b_{m-1} (radices[t] = b_t >= 1, host array of n_stages).
 * An index i has row-major digits i = sum_t i_t S_t, S_t = prod_{u>t} b_u.
 * Stage t replaces x[i] by sum_k B_{t,c}[i_t][k] x[i with digit t := k], where
 * the group id c numbers the other digits in row-major order (digit t
 * removed).  Stages run t = 0 first, so R = B_{m-1} ... B_0.
 * blocks: host array of n_stages device pointers; blocks[t] is fp32
 *         [G_t, b_t, b_t] row-major with G_t = n_groups[t] (host array), which
 *         must be L / b_t (one block per group) or 1 (one shared block).
 * transpose = 1 applies R^T (transposed blocks, stages in reverse order).
 * With n_stages > 1 and a bf16 y the fp32 intermediate needs
 * hit_workspace_bytes(HIT_OP_BUTTERFLY, rows, n, dtype_out, n_stages) bytes.
 * Limits: b_t <= 64, n_stages <= 16.
 */
HIT_API int butterfly_apply(const void* x, void* y, int64_t rows, int64_t n, int64_t ldx, int64_t ldy,
                    int dtype_in, int dtype_out, int n_stages, const int32_t* radices,
                    const float* const* blocks, const int64_t* n_groups, int transpose, int axis,
                    void* workspace, size_t workspace_bytes, void* stream);

/*
 * The same rotation y = R x as butterfly_apply [HARP §2.1, §2.4: the stride
 * stages as fused passes], on the tensor cores.  A run of consecutive stages
 * whose digits vary inside a window of at most 256 positions is, restricted
 * to each window, one dense matrix (the product of its blocks); the library
 * composes these window matrices on the device (fp32, rounded once to bf16)
 * and applies each pass as bf16 x bf16 products with fp32 accumulation
 * (tcgen05 MMAs, operands staged by TMA).  Passes run on the tensor cores
 * when the window is:
 *   along rows (axis 1): the last digits with a product P dividing 128
 *     (windows of 128 contiguous positions holding 128 / P groups);
 *   along columns (axis 0): digits with P in {128, 256} (positions at the
 *     stride of the run's last digit), or the last digits with P dividing 128;
 * two adjacent digits along rows at a stride that is a multiple of 8, with
 * radices (7, 16), (4, 16), (8, 8) or (16, 4), run as one register-resident
 * pass with their blocks rounded to bf16: on mma.sync tensor-core tiles
 * (block-diagonal products, bf16 between the two stages) for (7, 16) and
 * (4, 16) with a bf16 result, else in fp32 SIMT arithmetic;
 * other runs use the SIMT passes of butterfly_apply.  Data between passes is
 * bf16, so results carry bf16 rounding per pass (use butterfly_apply for an
 * fp32-accurate rotation).
 * Arguments as butterfly_apply, with: dtype_in must be HIT_BF16; x and y must
 * not alias; x, y 16-byte aligned, row pitches multiples of 16 bytes, n a
 * multiple of 8; workspace (256-byte aligned) of at least
 * butterfly_tc_workspace_bytes(rows, n, axis, n_stages, radices, transpose)
 * bytes (the window matrices and the bf16 intermediates).
 */
HIT_API int butterfly_apply_tc(const void* x, void* y, int64_t rows, int64_t n, int64_t ldx, int64_t ldy,
                               int dtype_in, int dtype_out, int n_stages, const int32_t* radices,
                               const float* const* blocks, const int64_t* n_groups, int transpose, int axis,
                               void* workspace, size_t workspace_bytes, void* stream);
/* Workspace bound of butterfly_apply_tc (0 for invalid arguments); host arithmetic only. */
HIT_API size_t butterfly_tc_workspace_bytes(int64_t rows, int64_t n, int axis, int n_stages, const int32_t* radices,
                                            int transpose);

/*
 * Fused RHT + group-wise symmetric absmax round-to-nearest quantization + code
 * packing [HARP §1, §5: incoherence processing before a blockwise quantizer].
 * x: [rows, n] (dtype_in, ldx).  One-sided (col_signs == NULL):
 *   Y = rows of x transformed with row_signs (length n).
 * Two-sided (col_signs != NULL, length rows, rows a power of two):
 *   Y = (H_rows D_col / sqrt(rows)) x (H_n D_row / sqrt(n))^T, computed with an
 *   fp32 intermediate in `workspace` (hit_workspace_bytes(HIT_OP_QUANT, rows,
 *   n, HIT_F32, 1) bytes).
 * Then, per row, groups of `group` consecutive elements (power of two,
 * 32 <= group <= min(n, 4096)):
 *   yf = fp32(Y); a = max|yf|; s = a / qmax (qmax = 2^(bits-1) - 1, IEEE
 *   division); q = clamp(rint(yf / s), -qmax, qmax) (ties to even); a = 0
 *   gives s = 0 and q = 0.
 * codes: uint8 [rows, n*bits/8], stored code u = q + 2^(bits-1) packed LSB
 *   first in a per-row bit stream (code j at stream bits [bits*j, bits*j+bits),
 *   stream bit k = bit k%8 of byte k/8): 4-bit two per byte low nibble first,
 *   2-bit four per byte, 3-bit eight codes per three bytes.
 * scales: fp32 [rows, n/group].
 * bits in {2, 3, 4}; n a power of two with 32 <= n <= 32768.
 */
HIT_API int rht_quantize_pack(const void* x, int64_t rows, int64_t n, int64_t ldx, int dtype_in,
                      const int8_t* row_signs, const int8_t* col_signs, int bits, int group,
                      uint8_t* codes, float* scales, void* workspace, size_t workspace_bytes,
                      void* stream);

/*
 * Fused randomized transform of the non-power-of-two length n = 5120 + group
 * quantization [HARP §2.1: mixed-radix schedules such as (8, 8, 8, 5, 2) for
 * d = 5120, with an orthogonal mixer (QR of a Gaussian) for the radix that is
 * not a power of two; §2.2: the mixers of power-of-two radices are the
 * normalized Sylvester Hadamard blocks].
 * Each row is transformed by y = R diag(signs) x with R the stage product of
 * the schedule (8, 8, 8, 5, 2) (the butterfly_apply digit convention) whose
 * radix-8 and radix-2 blocks are H_b / sqrt(b) and whose radix-5 blocks are
 * all the given mixer G_5; equivalently R = (H_512 / sqrt 512) (x) G_5 (x)
 * (H_2 / sqrt 2).  Then 4-bit symmetric absmax RTN in groups of 128 exactly as
 * rht_quantize_pack: codes uint8 [rows, 2560], scales fp32 [rows, 40].
 * x: fp32 [rows, ldx], 16-byte aligned rows.  signs: int8 [5120] or NULL.
 * mixer: HOST pointer to the 25 fp32 entries of G_5 (row-major, orthogonal).
 * n must be 5120, bits 4 and group 128 (HIT_EUNSUPPORTED otherwise).
 */
HIT_API int rht_mixed_quantize_pack(const float* x, int64_t rows, int64_t n, int64_t ldx, const int8_t* signs,
                                    const float* mixer, int bits, int group, uint8_t* codes, float* scales,
                                    void* stream);

/*
 * Dequantize then inverse-transform [HARP §5: exact change of basis, so the
 * reconstruction is the inverse rotation of the dequantized codes].
 * codes / scales as written by rht_quantize_pack; yhat = fp32(u - 2^(bits-1)) * s.
 * One-sided: y_r = diag(row_signs) H_n yhat_r / sqrt(n).
 * Two-sided (col_signs != NULL): additionally the inverse column transform.
 *   With dtype_out = HIT_F32 it runs in place in y; with bf16 it needs
 *   hit_workspace_bytes(HIT_OP_DEQUANT, rows, n, HIT_BF16, 1) bytes.
 * y: [rows, n] (dtype_out, ldy).
 */
HIT_API int dequant_inverse(const uint8_t* codes, const float* scales, int64_t rows, int64_t n, int bits,
                    int group, const int8_t* row_signs, const int8_t* col_signs, void* y,
                    int64_t ldy, int dtype_out, void* workspace, size_t workspace_bytes,
                    void* stream);

/*
 * Walsh-Hadamard expansion of sparse coefficients [QWHA §2.1, §4].
 * values, cols: [batch, rows, nnz] (fp32, int32); dense: fp32 [batch, rows, n].
 * mode 0 (forward): dense[b, r, :] = scatter(values, cols)[b, r, :] H_n * scale;
 *   duplicate columns within a row add up.
 * mode 1 (backward): values[b, r, k] = (dense[b, r, :] H_n * scale)[cols[b, r, k]]
 *   -- the gradient of mode 0 with respect to the values.
 * n a power of two with 32 <= n <= 32768; 1 <= nnz <= n.  Column indices
 * outside [0, n) are ignored in mode 0 and give 0 in mode 1 (the kernel never
 * accesses memory out of bounds).
 */
HIT_API int wht_expand_sparse(float* values, const int32_t* cols, int64_t batch, int64_t rows, int64_t n,
                      int32_t nnz, float scale, float* dense, int mode, void* stream);

/*
 * Two-transform Walsh-Hadamard expansion of sparse coefficients [QWHA §2.1:
 * the form dW = H'^-1 F H^-1 of other Fourier-type adapters, here with
 * Walsh-Hadamard transforms on both sides].
 * values, cols: [batch, m, nnz] (fp32, int32); dense: fp32 [batch, m, n].
 * mode 0: dense[b] = (H_m / sqrt m) scatter(values, cols)[b] H_n * scale
 *   (duplicate columns add up);
 * mode 1: values[b, r, k] = ((H_m / sqrt m) dense[b] H_n * scale)[r, cols[b, r, k]]
 *   -- the gradient of mode 0 with respect to the values; dense is not
 *   modified and the column transforms go to `workspace` (fp32, batch * m * n
 *   elements, 16-byte aligned).
 * m a power of two <= 2^24; n a power of two in [32, 32768]; 1 <= nnz <= n.
 * Columns outside [0, n) are ignored (mode 0) / give 0 (mode 1).
 */
HIT_API int wht_expand_sparse_2d(float* values, const int32_t* cols, int64_t batch, int64_t m, int64_t n, int32_t nnz,
                                 float scale, float* dense, int mode, void* workspace, size_t workspace_bytes,
                                 void* stream);

/*
 * AdaAlloc around the sparse expansion [QWHA §2.2: a budget of coefficients
 * is spread over the output channels (rows) in proportion to each channel's
 * error with a minimum per channel; inside a channel the coefficients of
 * largest magnitude are kept].
 *
 * row_norms: norms[r] = ||x[r, :n]||_2 (fp64 accumulation of the fp32
 *   squares), x fp32 [rows, ldx] with n and ldx multiples of 4 and 16-byte
 *   aligned rows; norms fp64 [rows] (device).  The channel error without
 *   activations (the norm of a row of dW, equal to that of its coefficients).
 *
 * qwha_allocate (HOST pointers, no device work): counts[r] in [k_min, n] with
 *   sum = budget (rows * k_min <= budget <= rows * n).  Every row gets k_min;
 *   the remaining R units are split in proportion to err[r]: the share of an
 *   uncapped row is (R' * err[r]) / S in float64, R' the units left for the
 *   uncapped rows and S the left-to-right float64 sum of their errors; rows
 *   whose share passes n - k_min are capped there and the rest re-split until
 *   none passes; shares are rounded down and the leftover units go one each
 *   to the largest fractional parts (ties to the lower row).  All-zero errors
 *   split equally.  err must be finite and >= 0.
 *
 * qwha_select: per row r, the counts[r] = offsets[r+1] - offsets[r] entries of
 *   largest |f[r, j]| (ties to the lower j), written in ascending j:
 *   cols[offsets[r] + i] = j, values[...] = f[r, j].  f fp32 [rows, ldf]
 *   (ldf >= n, multiple of 4, 16-byte aligned); offsets int64 [rows + 1],
 *   cols int32 and values fp32 [offsets[rows]] (device).  n must be 1024,
 *   2048, 4096 or 8192; counts must not exceed n.
 */
HIT_API int row_norms(const float* x, int64_t rows, int64_t n, int64_t ldx, double* norms, void* stream);
HIT_API int qwha_allocate(const double* err, int64_t rows, int64_t budget, int64_t k_min, int64_t n, int64_t* counts);
HIT_API int qwha_select(const float* f, int64_t rows, int64_t n, int64_t ldf, const int64_t* offsets, int32_t* cols,
                        float* values, void* stream);

/*
 * HARP stage blocks from learnable parameters [HARP §2.2: each block is a
 * learnable orthogonal factor times a fixed base mixer, B_c = Q(theta_c) G_b,
 * Givens for b = 2, Cayley map (I - A)^-1 (I + A) for b > 2, all parameters
 * zero = the fixed RHT; §2.4: int8 parameter storage].
 * Builds every block of ONE stage of radix b (1 <= b <= 16) for `groups`
 * groups, in the layout butterfly_apply reads: blocks [groups, b, b] fp32
 * row-major (groups = L / b for the stage of a length-L transform).
 *  - Parameters per block P = 0 (b = 1), 1 (b = 2: the angle phi of
 *    Q = [[cos phi, -sin phi], [sin phi, cos phi]]), b (b - 1) / 2 (b > 2: A is
 *    skew-symmetric with A[i][j] = theta_k, A[j][i] = -theta_k for i < j, pairs
 *    k numbered row by row (0,1), (0,2), ..., (1,2), ...).
 *  - Give exactly one of theta (fp32 [groups, P]) and theta_q (int8
 *    [groups, P], standing for fp32(q) * theta_scale); both may be NULL for b = 1.
 *  - mixer: fp32 [b, b] row-major orthogonal G_b; NULL means the normalized
 *    Sylvester Hadamard H_b / sqrt(b), and is only allowed for powers of two.
 *  - signs: NULL, or int8 [b * groups]: column k of block c is multiplied by
 *    signs[k * groups + c], the sign of the input position that column reads
 *    in the FIRST stage (t = 0) of a transform.  Folding the RHT's sign vector
 *    into stage 0 this way makes butterfly_apply compute R(theta) diag(s) x,
 *    and with transpose = 1 its inverse diag(s) R(theta)^T y.
 * All pointers are device pointers.  Arithmetic in fp32 (Gauss-Jordan solve
 * without pivoting: the symmetric part of I - A is the identity).
 */
HIT_API int harp_blocks(const float* theta, const int8_t* theta_q, float theta_scale, int64_t groups, int b,
                        const float* mixer, const int8_t* signs, float* blocks, void* stream);

/*
 * Fused RHT + group quantization without any allocation (no counterpart in
 * the pages; a deployment convenience).
 *
 * Same arguments and results as rht_quantize_pack, minus the workspace.  Some
 * callers cannot call cudaMalloc at all -- for example plug-ins whose host
 * application owns every byte of device memory, or latency-critical paths that
 * must never block on the allocator -- and so cannot hand the two-sided
 * quantizer its fp32 intermediate.  This entry point places that intermediate
 * in a scratch array the library carries as a static device variable of
 * HIT_NOALLOC_MAX_ELEMS fp32 elements (16 MiB); every GPU that loads
 * libhit.so holds it until the process exits.
 *  - Two-sided calls need rows * n <= HIT_NOALLOC_MAX_ELEMS; larger problems
 *    return HIT_EWORKSPACE.  One-sided calls (col_signs == NULL) use no
 *    scratch and have no extra limit.
 *  - The first two-sided call on a device resolves the array's device address
 *    (cudaGetSymbolAddress, with that device current) and keeps it for the
 *    life of the process; make that first call before any stream capture.  The
 *    address belongs to the device's primary context: after cudaDeviceReset
 *    (or anything else that destroys that context) do not call this entry
 *    point on that device again.
 *  - Arguments are checked exactly as rht_quantize_pack checks them (same
 *    statuses) before the size limit below.
 *  - Every call on a device shares the one array and it keeps the last call's
 *    contents (each call overwrites all of the part it reads, so nothing needs
 *    clearing).  Calls whose executions overlap on the GPU -- on different
 *    streams, or from several host threads -- race on the array.
 *  - The call allocates nothing: no cudaMalloc, cudaFree or allocating library
 *    routine.
 */
#define HIT_NOALLOC_MAX_ELEMS 4194304
HIT_API int rht_quantize_pack_noalloc(const void* x, int64_t rows, int64_t n, int64_t ldx, int dtype_in,
                                      const int8_t* row_signs, const int8_t* col_signs, int bits, int group,
                                      uint8_t* codes, float* scales, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* HIT_H_ */
