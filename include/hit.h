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
 * The persistent row kernels (row length 4096) wait on shared-memory barriers
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
