/*
 * halo.h -- C ABI of the B200 (sm_100a) Hadamard-rotated quantized linear layer.
 *
 * The operation: "HALO: Hadamard-Assisted Lower-Precision Optimization for
 * LLMs" (arXiv 2501.02625, abstract) places Hadamard rotations in the forward
 * and backward passes of a transformer's linear layers so that every large
 * matrix multiplication runs in low precision (INT8 or FP8: same page, "key
 * design").  For nn.Linear shapes X[M,K], W[N,K]:
 *     Y  = X  W^T   contraction over K      (forward)
 *     dX = dY W     contraction over N      (backward, input gradient)
 *     dW = dY^T X   contraction over M      (backward, weight gradient)
 * each GEMM rotates both operands along its contraction dimension with a
 * block-local Walsh-Hadamard transform (blocks of 128 or 256 consecutive
 * elements, natural Sylvester order, normalised by 1/sqrt(blk): QWHA page,
 * sec. 2.1-2.2 for the transform, HALO blog page sec. 5 for block locality),
 * quantises each operand symmetrically with one fp32 scale per
 * non-contraction index (scale = max|v| / qmax, q = round-half-even(v /
 * scale), INT8 qmax 127 clamped to +-127, E4M3 qmax 448 saturating: QWHA page
 * sec. 2.2 "quantize"), multiplies the codes on the tensor cores with int32 /
 * fp32 accumulation, and dequantises with the product of the two scales.
 *
 * Conventions for every entry point:
 *   - All data pointers are DEVICE pointers owned by the caller.  The library
 *     never allocates device memory; scratch comes from the caller's
 *     workspace (see halo_workspace_size).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Every call is asynchronous on that stream; nothing is
 *     synchronised by the library.
 *   - Arguments are validated on the host before anything is launched; an
 *     invalid argument returns an error status and launches nothing.
 *   - Matrices are row-major with an explicit leading dimension `ld_*` counted
 *     in ELEMENTS.  bf16 = 2 bytes, INT8 / E4M3 codes = 1 byte.
 *   - Alignment: every pointer must be 16-byte aligned and every row stride
 *     must be a multiple of 16 bytes (the tensor-memory-accelerator copy
 *     rule); otherwise HALO_ERR_ALIGN.
 *   - A device that is not compute capability 10.0 (B200 / sm_100a) gives
 *     HALO_ERR_UNSUPPORTED.  There is no fallback path.
 *   - Kernels bound every wait they make; a wait that runs out records a
 *     device-side error that halo_device_error() reports (HALO_ERR_TIMEOUT).
 */
#ifndef HALO_H_
#define HALO_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  HALO_OK = 0,
  HALO_ERR_NULL = 1,        /* a required pointer is NULL                      */
  HALO_ERR_SHAPE = 2,       /* a size <= 0, a stride shorter than its row, or  */
                            /* a size beyond a documented limit                */
  HALO_ERR_BLOCK = 3,       /* blk not supported for this call                 */
  HALO_ERR_ALIGN = 4,       /* pointer not 16-byte aligned / stride rule       */
  HALO_ERR_DTYPE = 5,       /* unknown qtype / otype / axis / major            */
  HALO_ERR_WORKSPACE = 6,   /* workspace NULL or smaller than required         */
  HALO_ERR_CUDA = 7,        /* a CUDA runtime / driver call failed             */
  HALO_ERR_TIMEOUT = 8,     /* a kernel's bounded wait ran out                 */
  HALO_ERR_UNSUPPORTED = 9  /* device is not sm_100 (B200)                     */
} halo_status_t;

typedef enum { HALO_Q_INT8 = 0, HALO_Q_E4M3 = 1 } halo_qtype_t;
typedef enum { HALO_OUT_FP32 = 0, HALO_OUT_BF16 = 1 } halo_otype_t;

/* Rotation axis of halo_hadamard_quantize. */
typedef enum {
  HALO_AXIS_COLS = 0, /* rotate along the contiguous dimension (blocks of blk
                         consecutive elements of a row); one scale per ROW    */
  HALO_AXIS_ROWS = 1  /* rotate along dimension 0 (blocks of blk consecutive
                         rows of a column); one scale per COLUMN              */
} halo_axis_t;

/* Storage order of a GEMM operand of halo_qgemm. */
typedef enum {
  HALO_MAJOR_K = 0,  /* A stored [M, K] (B stored [N, K]): contraction dim contiguous */
  HALO_MAJOR_MN = 1  /* A stored [K, M] (B stored [K, N]): the other dim contiguous   */
} halo_major_t;

/*
 * Rotate + quantise one bf16 matrix X[rows, cols] (row stride ld_x elements,
 * ld_x * 2 a multiple of 16 bytes).
 *   axis = HALO_AXIS_COLS: blk in {128, 256}; cols_p = cols rounded up to a
 *       multiple of blk, cols_p <= 32768.  Codes q_out[rows, cols_p], ld_q >=
 *       cols_p.  scales_out[rows]: s_r = max_c |Xrot[r, c]| / qmax.
 *   axis = HALO_AXIS_ROWS: blk == 128, cols % 8 == 0; rows_p = rows rounded
 *       up to a multiple of 128.  Codes q_out[rows_p, cols] (the buffer must
 *       hold rows_p rows of ld_q bytes).  scales_out[cols]: s_c = max_r
 *       |Xrot[r, c]| / qmax.
 * A rotated length that is not a multiple of the block is zero-padded to
 * whole blocks (QWHA page, sec. 3.1 and 5: zero-fill to the transform
 * length); the codes cover the padded length.  Xrot is the (padded) X with
 * every block transformed by H_blk / sqrt(blk).  q_out (row stride ld_q bytes,
 * a multiple of 16) receives q = round-half-even(Xrot / s) clamped to +-127 as
 * two's-complement int8 (qtype INT8), or Xrot / s rounded to nearest-even and
 * saturated to +-448 as OCP E4M3 bytes (qtype E4M3).  A group whose max is 0
 * gets scale 0 and all-zero codes.  The codes keep the input's layout in both
 * axes (nothing is transposed); halo_qgemm reads the dimension-0-rotated codes
 * as an MN-major operand.
 * Defined by: HALO paper page (abstract; "key design": INT8 or FP8); QWHA page
 * sec. 2.1-2.2 (Walsh-Hadamard transform, symmetric quantiser).
 */
halo_status_t halo_hadamard_quantize(const void* x_bf16, int64_t rows, int64_t cols, int64_t ld_x,
                                     int axis, int blk, int qtype, void* q_out, int64_t ld_q,
                                     float* scales_out, void* stream);

/*
 * halo_hadamard_quantize with the two variants of the rotation and rounding:
 *   signs      NULL, or int8 +1 / -1 (only the sign bit is read) for every
 *              position along the rotated dimension, padded length (cols_p
 *              entries for HALO_AXIS_COLS, rows_p for HALO_AXIS_ROWS; the
 *              entries past the input meet zeros), 16-byte aligned:
 *              random-sign rotation, each block becomes H_blk D x / sqrt(blk)
 *              with D = diag(signs).  Both operands of a GEMM must use the
 *              same signs along the contraction dimension; the product is
 *              then unchanged, since (H D)^T (H D) = I.  Seeded random signs
 *              shared by all workers: HALO blog page, sec. 4.2.
 *   rand_bits  NULL (round half to even), or 16 random bits per element of
 *              the codes, layout [rows, cols_p] (HALO_AXIS_COLS) or [rows_p,
 *              cols] (HALO_AXIS_ROWS) with row stride ld_rand elements
 *              (16-byte aligned base, ld_rand * 2 a multiple of 16): stochastic
 *              rounding.  With u = rand_bits / 65536, t = Xrot / s rounds to
 *              its upper grid neighbour when u < (t - lo) / (hi - lo), else
 *              to its lower one (INT8 grid clamped to +-127; E4M3 grid
 *              saturating at 448).  QWHA page, sec. 5 (random rounding).
 * The scales are those of halo_hadamard_quantize.  Everything else as there.
 */
halo_status_t halo_hadamard_quantize_ex(const void* x_bf16, int64_t rows, int64_t cols, int64_t ld_x,
                                        int axis, int blk, int qtype, const int8_t* signs,
                                        const uint16_t* rand_bits, int64_t ld_rand, void* q_out,
                                        int64_t ld_q, float* scales_out, void* stream);

/*
 * Both 8-bit encodings of one rotation from a single read of X: the block
 * rotation along the contiguous dimension (HALO_AXIS_COLS) of
 * halo_hadamard_quantize, quantised per row to INT8 (codes q_int8 [rows, cols_p],
 * row stride ld_q8 bytes, scales_int8 [rows] = amax / (127 sqrt(blk))) and to
 * E4M3 (q_e4m3, ld_qf8, scales_e4m3 [rows] = amax / (448 sqrt(blk))).  Each
 * output equals what halo_hadamard_quantize writes for its qtype, byte for
 * byte; the input is read once instead of twice.  The two outputs must not
 * overlap.  Arguments, alignment rules and errors as for
 * halo_hadamard_quantize (axis HALO_AXIS_COLS, blk 128 or 256).
 * Defined by: HALO paper page ("key design": INT8 or FP8 for every matmul);
 * QWHA page sec. 2.1-2.2 (Walsh-Hadamard transform, symmetric quantiser).
 */
halo_status_t halo_hadamard_quantize_dual(const void* x_bf16, int64_t rows, int64_t cols, int64_t ld_x,
                                          int blk, void* q_int8, int64_t ld_q8, float* scales_int8,
                                          void* q_e4m3, int64_t ld_qf8, float* scales_e4m3, void* stream);

/*
 * Both code sets of one matrix that feeds two GEMMs of the backward pass
 * (dY: dX = dY W contracts its columns, dW = dY^T X its rows): rotated along
 * the contiguous dimension (blocks of blk, one scale per row) into q_rows /
 * scales_rows, exactly as halo_hadamard_quantize(axis HALO_AXIS_COLS), and
 * along dimension 0 (blocks of 128, one scale per column) into q_cols /
 * scales_cols, exactly as halo_hadamard_quantize(axis HALO_AXIS_ROWS).  The
 * two rotations run back to back on the stream, so that the second reads X
 * from L2 when X fits there (up to about 64 MB): one read of X from memory
 * for both code sets.  Arguments, layouts and errors as the two calls; both
 * are checked before either is launched.  Defined by: HALO paper page,
 * abstract (rotations in the backward pass: dY is rotated along N for dX and
 * along the tokens for dW).
 */
halo_status_t halo_hadamard_quantize_both(const void* x_bf16, int64_t rows, int64_t cols, int64_t ld_x,
                                          int blk, int qtype, void* q_rows, int64_t ld_qr,
                                          float* scales_rows, void* q_cols, int64_t ld_qc,
                                          float* scales_cols, void* stream);

/*
 * The dimension-0 rotation split at its column maxima, for a matrix whose
 * rows are spread over several devices, each holding whole 128-row blocks
 * (fully sharded data parallelism with low-precision communication: HALO
 * paper page, "technical framework").  The devices exchange one fp32 vector
 * of column maxima instead of the bf16 rows.
 *
 * halo_hadamard_colmax: amax_out[c] = the largest |u| over this device's rows
 *   of column c, u = H_128 x the unnormalised block transform along dimension 0
 *   (rows zero-padded to whole blocks as in halo_hadamard_quantize).  The
 *   caller merges the devices' vectors by element-wise maximum (an all-reduce).
 *   amax_out: [cols] fp32, device memory, 16-byte aligned, overwritten (the
 *   call clears it on the stream, then accumulates).
 * halo_hadamard_quantize_colmax: codes and scales of X[rows, cols] rotated
 *   along dimension 0 with given column maxima amax[c] (those of every
 *   device's rows): q = round_half_even(u * qmax / amax[c]) clamped to +-127
 *   (INT8), or the E4M3 encoding of u * qmax / amax[c] (satfinite);
 *   scales_out[c] = amax[c] / (qmax sqrt(128)); amax[c] = 0 gives code 0 and
 *   scale 0.  Given the maxima of the whole matrix, each device's codes and
 *   scales are byte for byte those halo_hadamard_quantize (axis
 *   HALO_AXIS_ROWS) writes for its rows of the whole matrix.
 * blk must be 128 and cols % 8 == 0; x, q_out, ld_q, scales_out, layouts and
 * errors as halo_hadamard_quantize with axis HALO_AXIS_ROWS; amax: [cols]
 * fp32, device, 16-byte aligned, not written.
 */
halo_status_t halo_hadamard_colmax(const void* x_bf16, int64_t rows, int64_t cols, int64_t ld_x, int blk,
                                   float* amax_out, void* stream);
halo_status_t halo_hadamard_quantize_colmax(const void* x_bf16, int64_t rows, int64_t cols,
                                            int64_t ld_x, int blk, int qtype, const float* amax,
                                            void* q_out, int64_t ld_q, float* scales_out, void* stream);

/*
 * Low-precision GEMM on codes with a dequantising epilogue:
 *     C[i, j] = (sum_k A[i, k] B[j, k]) * s_a[i] * s_b[j]
 * A is M x K and B is N x K (logically).  a_major / b_major give their
 * storage: HALO_MAJOR_K means A stored [M, K] with row stride ld_a (B: [N, K],
 * ld_b); HALO_MAJOR_MN means A stored [K, M] (B: [K, N]) with that row stride.
 * INT8 codes accumulate exactly in int32 (requires K * 127^2 < 2^31, i.e.
 * K <= 133144); E4M3 codes accumulate in fp32.  C is [M, N] with row stride
 * ld_c elements, fp32 or bf16 (round-to-nearest-even of the fp32 value).
 * Strides: ld_a, ld_b multiples of 16; ld_c * sizeof(C element) multiple of 16.
 * Defined by: HALO paper page, abstract ("all large matrix multiplications
 * ... executed in lower precision") and "key design" (INT8 or FP8).
 */
halo_status_t halo_qgemm(const void* a_q, const float* s_a, int a_major, int64_t ld_a,
                         const void* b_q, const float* s_b, int b_major, int64_t ld_b, int64_t m,
                         int64_t n, int64_t k, int qtype, void* c, int otype, int64_t ld_c,
                         void* stream);

/*
 * Scratch bytes halo_linear_fwd (which = 0) or halo_linear_bwd (which = 1)
 * needs for these sizes: the operands' codes (contraction dimension
 * zero-padded to whole blocks; the forward size covers either block size) and
 * scales.
 */
size_t halo_workspace_size(int64_t m, int64_t n, int64_t k, int which);

/*
 * Forward linear layer Y[M, N] = X[M, K] W[N, K]^T with both operands
 * rotated along K (blocks of blk; K % 8 == 0; a K that is not a multiple of
 * blk is zero-padded to whole blocks, at most 32768), quantised per row
 * (qtype), multiplied on codes and dequantised.  x, w, y dense row-major.  ws
 * must hold halo_workspace_size(m, n, k, 0) bytes and be 16-byte aligned.
 * Defined by: HALO paper page, abstract (rotations in the forward pass).
 */
halo_status_t halo_linear_fwd(const void* x_bf16, const void* w_bf16, int64_t m, int64_t n,
                              int64_t k, int blk, int qtype, void* y, int otype, void* ws,
                              size_t ws_bytes, void* stream);

/*
 * Backward linear layer for Y = X W^T, given dY[M, N], X[M, K], W[N, K]:
 *   dX[M, K] = dY W:    dY rotated along N per row, W rotated along N
 *                       (dimension 0) per column; K % 16 == 0.
 *   dW[N, K] = dY^T X:  dY and X both rotated along M (dimension 0), one
 *                       scale per column; N % 16 == 0, K % 16 == 0.
 * N % 8 == 0.  An N (dX) or M (dW) that is not a multiple of blk is
 * zero-padded to whole blocks (N padded at most 32768).
 * blk must be 128.  dx or dw may be NULL to skip that product (the inputs it
 * alone needs may then be NULL too).  All matrices dense row-major.  ws must
 * hold halo_workspace_size(m, n, k, 1) bytes.
 * Defined by: HALO paper page, abstract (rotations in the backward pass so that
 * both backward matmuls run in low precision).
 */
halo_status_t halo_linear_bwd(const void* dy_bf16, const void* x_bf16, const void* w_bf16,
                              int64_t m, int64_t n, int64_t k, int blk, int qtype, void* dx,
                              int otype_dx, void* dw, int otype_dw, void* ws, size_t ws_bytes,
                              void* stream);

/*
 * Group-wise scales (QWHA page sec. 3.1, the quantiser's group_quantize: one
 * scale max|x| / qmax per group of group_size consecutive values; sec. 3.2
 * recommends 64, sec. 6 32-128): the variant of the calls above in which each
 * operand carries one scale per `group` (64 or 128) consecutive positions of
 * the GEMM's contraction dimension instead of one per row.
 *
 * halo_hadamard_quantize_grouped: as halo_hadamard_quantize (zero padding
 * included), with scales
 *   HALO_AXIS_COLS: scales_out[rows][cols_p / group] (dense), the scale of
 *                   elements g*group .. g*group + group - 1 of a row;
 *   HALO_AXIS_ROWS: scales_out[rows_p / group][cols] (dense), the scale of
 *                   rows g*group .. of a column.
 * group in {64, 128}, else HALO_ERR_BLOCK.
 */
halo_status_t halo_hadamard_quantize_grouped(const void* x_bf16, int64_t rows, int64_t cols,
                                             int64_t ld_x, int axis, int blk, int group, int qtype,
                                             void* q_out, int64_t ld_q, float* scales_out, void* stream);

/*
 * halo_qgemm_grouped: C[i, j] = sum_G s_a[i, G] s_b[j, G] sum_{k in group G}
 * A[i, k] B[j, k], K a multiple of 128.  Scale layouts follow the codes: a
 * K-major operand ([M, K] codes) has scales [M][K / group]; an MN-major one
 * ([K, M] codes, rotated along dimension 0) has scales [K / group][M] -- the
 * layouts halo_hadamard_quantize_grouped writes.  Everything else as
 * halo_qgemm.  Each group's partial product is accumulated exactly (int32 /
 * fp32 on the tensor cores) and scaled into an fp32 running sum.
 */
halo_status_t halo_qgemm_grouped(const void* a_q, const float* s_a, int a_major, int64_t ld_a,
                                 const void* b_q, const float* s_b, int b_major, int64_t ld_b,
                                 int64_t m, int64_t n, int64_t k, int group, int qtype, void* c,
                                 int otype, int64_t ld_c, void* stream);

/* Scratch bytes of halo_linear_fwd_grouped (which = 0) / halo_linear_bwd_grouped (which = 1). */
size_t halo_workspace_size_grouped(int64_t m, int64_t n, int64_t k, int group, int which);

/* halo_linear_fwd / halo_linear_bwd with group-wise scales along each GEMM's
 * contraction dimension (group 64 or 128); ws as halo_workspace_size_grouped. */
halo_status_t halo_linear_fwd_grouped(const void* x_bf16, const void* w_bf16, int64_t m, int64_t n,
                                      int64_t k, int blk, int group, int qtype, void* y, int otype,
                                      void* ws, size_t ws_bytes, void* stream);
halo_status_t halo_linear_bwd_grouped(const void* dy_bf16, const void* x_bf16, const void* w_bf16,
                                      int64_t m, int64_t n, int64_t k, int blk, int group, int qtype,
                                      void* dx, int otype_dx, void* dw, int otype_dw, void* ws,
                                      size_t ws_bytes, void* stream);

/*
 * Size of the library-owned scratch array used by halo_linear_fwd_noalloc.
 */
#define HALO_NOALLOC_SCRATCH_BYTES (64ull << 20) /* 64 MiB */

/*
 * Forward linear layer computed exactly as halo_linear_fwd, but for callers
 * that cannot allocate device memory.  There is no counterpart in the paper:
 * this is an interface variant, not part of the method.
 *
 * Who needs it: code that only ever receives input and output pointers and has
 * no way to obtain scratch -- for example a plugin inside an inference server
 * or framework whose interface hands over no workspace, or a latency-critical
 * loop that must not call cudaMalloc, because cudaMalloc can synchronise the
 * device and stall every other stream.  Such a caller passes X, W and Y only.
 *
 * Where the scratch comes from: a file-scope __device__ array of
 * HALO_NOALLOC_SCRATCH_BYTES inside the library.  Every GPU that loads the
 * library holds that array until the process exits.  The call allocates
 * nothing: no cudaMalloc, no cudaFree, no allocating library routine.
 *
 * Limits and behaviour:
 *   - Arguments and layout as for halo_linear_fwd.  Sizes whose codes and
 *     scales do not fit (more than HALO_NOALLOC_SCRATCH_BYTES; at most
 *     halo_workspace_size(m, n, k, 0) are needed) return HALO_ERR_WORKSPACE and
 *     launch nothing; halo_last_error_detail() then gives the bytes needed.
 *   - The first call on a device looks up the array's device address with
 *     that device current; make that first call before any stream capture.
 *   - All calls share the one array, which keeps the last call's contents.
 *     Nothing in it has to start at zero: a call reads only bytes it wrote
 *     earlier in the same call.  Calls that can overlap on the GPU (on
 *     unordered streams, or from several host threads) race on the array;
 *     order them on one stream or with events.
 */
halo_status_t halo_linear_fwd_noalloc(const void* x_bf16, const void* w_bf16, int64_t m, int64_t n,
                                      int64_t k, int blk, int qtype, void* y, int otype, void* stream);

/* Human-readable name of a status code (static string, never NULL). */
const char* halo_status_string(int status);

/*
 * Synchronises the current device, then reports and clears the device-side
 * error word that kernels set when a bounded wait runs out.  Returns HALO_OK
 * when no kernel recorded an error, HALO_ERR_TIMEOUT when one did (the kernel
 * site is written to *where if where != NULL), HALO_ERR_CUDA when the
 * synchronisation itself failed.
 */
halo_status_t halo_device_error(int* where);

/*
 * Diagnostic of the failure path (no counterpart in the paper): launches one
 * kernel that waits, bounded by limit_ns (0 < limit_ns <= 2e9, else
 * HALO_ERR_SHAPE), on an mbarrier that nothing ever completes.  The wait runs
 * out, records site 0xF01 in the device error word and returns, exactly as any
 * other bounded wait in the library does; halo_device_error() then reports
 * HALO_ERR_TIMEOUT with that site and clears it, and the context stays usable.
 * Nothing faults, traps or hangs.
 */
halo_status_t halo_selftest_wait_timeout(int64_t limit_ns, void* stream);

/* The last CUDA error code seen by the library on this thread (0 if none).
 * A failed tensor-map encoding is reported as 10000 + its CUresult. */
int halo_last_cuda_error(void);

/* Text naming the last failing CUDA call on this thread ("" if none).  The
 * string is owned by the library and stays valid until the next failure. */
const char* halo_last_error_detail(void);

#ifdef __cplusplus
}
#endif

#endif /* HALO_H_ */
