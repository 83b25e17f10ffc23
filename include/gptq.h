/*
 * gptq.h -- C ABI of libgptq_b200: GPTQ layer quantization on NVIDIA B200 (sm_100a).
 *
 * The problem: for a linear layer with weights W (rows x cols) and calibration inputs X, find a
 * k-bit W_hat that keeps ||W X - W_hat X||^2 small ("GPTQ second-order quantization" blog, section
 * "The objective is layer output, not weight distance"), by rounding columns in a fixed order and
 * moving the not-yet-rounded columns to absorb each rounding error, with the inverse-Hessian
 * information read from a Cholesky factor ("Part 3: Adaptive Rounding: GPTQ", "Algorithm GPTQ").
 *
 * Three calls make the path, in this order:
 *   1. gptq_hessian_accumulate  S += X^T X over chunks of calibration tokens        (step S1)
 *   2. gptq_prepare_hinv        H = 2S/N; damping; upper factor R of (H+lambda I)^-1 (S2-S5)
 *   3. gptq_quantize_layer      blocked column loop with lazy trailing updates       (S6-S8)
 *
 * Conventions for every call:
 *   - Pointers named *_dev, and every matrix argument, are DEVICE pointers to caller-owned
 *     memory (e.g. torch CUDA tensors). The library never allocates, frees or keeps them.
 *   - Matrices are row-major. "ld" arguments are leading dimensions in elements.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream). Every call only enqueues work
 *     on that stream and returns; it never synchronizes.
 *   - The return value reports argument and launch errors found on the host, before or while
 *     enqueueing; on any error other than GPTQ_OK nothing further was enqueued.
 *   - Conditions found on the device are written to the caller's int32 status word `info_dev`
 *     (see GPTQ_INFO_*). The caller sets it to 0 once; kernels only ever replace 0 by the first
 *     error they detect, and the library never clears it. Read it after synchronizing.
 *   - Calls on distinct buffers may run concurrently on different streams.
 */
#ifndef GPTQ_B200_H
#define GPTQ_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum gptq_status {
  GPTQ_OK = 0,
  GPTQ_EINVAL = 1,         /* an argument is out of range, misaligned or inconsistent */
  GPTQ_ENOTPD = 2,         /* (from gptq_info_status) a factorization met a non-positive pivot */
  GPTQ_ECUDA = 3,          /* a CUDA runtime call failed (launch, attribute, driver entry point) */
  GPTQ_EUNSUPPORTED = 4,   /* a valid request the library does not implement (e.g. dtype/size) */
  GPTQ_ETIMEOUT = 5,       /* (from gptq_info_status) a bounded device-side wait expired */
  GPTQ_EWORKSPACE = 6      /* workspace missing or smaller than gptq_workspace_size() */
} gptq_status;

typedef enum gptq_dtype { GPTQ_BF16 = 0, GPTQ_FP32 = 1 } gptq_dtype;

/* How gptq_prepare_hinv_route() reaches R (both give the same R up to rounding: the upper factor
 * with positive diagonal of (H + lambda I)^-1 is unique). */
typedef enum gptq_route {
  GPTQ_ROUTE_DEFAULT = 0,     /* the library's choice: GPTQ_ROUTE_REVERSED */
  GPTQ_ROUTE_THREE_STEP = 1,  /* Cholesky, triangular inverse, L^-T L^-1, Cholesky of the inverse */
  GPTQ_ROUTE_REVERSED = 2     /* one Cholesky of the order-reversed matrix, one triangular inverse */
} gptq_route;

/* Values the kernels write into *info_dev (the first one detected wins). */
#define GPTQ_INFO_OK 0
/* 1 .. cols:        H + lambda I is not positive definite; value = 1-based column index of the
 *                   pivot that failed (S3; for the reversed route the factorization runs from the
 *                   last column to the first, and the index still names the original column). */
/* cols+1 .. 2*cols: the formed inverse is not positive definite; value - cols = pivot (S5, three-
 *                   step route only). */
#define GPTQ_INFO_TIMEOUT (-1)        /* a bounded wait inside a kernel expired */
#define GPTQ_INFO_BAD_HESSIAN (-2)    /* mean(diag H) <= 0 or not finite: nothing to damp */
#define GPTQ_INFO_BAD_CODE (-3)       /* a pack call met a code too wide for its format */

/* Which workspace gptq_workspace_size() reports. */
#define GPTQ_WS_PREPARE 1
#define GPTQ_WS_QUANTIZE 2

/*
 * S1 -- proxy Hessian accumulation: S += X^T X.
 *
 * Source: "Part 2: Adaptive Rounding: Optimal Brain Quantizer (OBQ)", section "Goal" (the input
 * covariance E[x x^T] is the proxy Hessian); "Part 3: Adaptive Rounding: GPTQ", "Algorithm GPTQ"
 * (H = X X^T + lambda I, X stored there as cols x tokens).
 *
 *   S_dev      float32 [cols x cols], ld = cols. Only the lower triangle (i >= j) is accumulated
 *              and meaningful; the strict upper triangle is scratch (it may receive partial sums).
 *              The caller zeroes S once before the first chunk.
 *   X_dev      calibration inputs, TOKEN-major: [n_tokens x ldx], columns 0..cols-1 used.
 *              GPTQ_BF16: tensor-core path (tcgen05, bf16 products, fp32 accumulation);
 *                requires cols % 8 == 0, ldx % 8 == 0 and a 16-byte aligned X_dev.
 *              GPTQ_FP32: fp32 CUDA-core path (exact fp32 products and sums), any cols.
 *   n_tokens   tokens in this chunk (0 = nothing to do). Call repeatedly to stream chunks; the
 *              total over all calls is the N given to gptq_prepare_hinv.
 *   info_dev   status word (GPTQ_INFO_TIMEOUT if a pipeline wait expires).
 * Errors: GPTQ_EINVAL for null pointers, cols <= 0, ldx < cols, n_tokens < 0 or alignment.
 */
gptq_status gptq_hessian_accumulate(float* S_dev, int64_t cols, const void* X_dev,
                                    gptq_dtype x_dtype, int64_t n_tokens, int64_t ldx,
                                    int32_t* info_dev, void* stream);

/*
 * S2-S5 -- damped inverse-Hessian factor.
 *
 * Source: "GPTQ second-order quantization" blog, sections "The objective is layer output"
 * (H = 2 X X^T) and "3. Cholesky reformulation" (damping of about 1 % of the mean Hessian
 * diagonal; Cholesky factor computed once); "Part 3: Adaptive Rounding: GPTQ", "Observation 3:
 * The Cholesky Reformulation" and "Algorithm GPTQ" (Cholesky of H^-1, one factor row read per
 * column). The pages' route: H_d = H + lambda I = L L^T (blocked Cholesky), L^-1 (triangular
 * inverse), H_d^-1 = L^-T L^-1, H_d^-1 = R^T R with R upper (Cholesky of the inverse). This call
 * takes GPTQ_ROUTE_DEFAULT, i.e. the reversed route of gptq_prepare_hinv_route(), which reaches
 * the same R with half the arithmetic.
 *
 *   S_H_dev    in:  S from gptq_hessian_accumulate (lower triangle read).
 *              out: H = (2 / n_total) S, both triangles, undamped (kept for the layer metric).
 *   R_dev      out: float32 [cols x cols], ld = cols: R upper triangular with positive diagonal,
 *              (H + lambda I)^-1 = R^T R, strictly lower part set to 0.
 *   n_total    total number of calibration tokens accumulated into S (> 0).
 *   damp_rel   lambda = damp_rel * mean(diag H) (the pages use 0.01); must be >= 0.
 *   ws_dev     device workspace of at least gptq_workspace_size(GPTQ_WS_PREPARE, 0, cols, 0)
 *              bytes, 256-byte aligned; contents on entry do not matter.
 *   info_dev   status word: pivot codes (see GPTQ_INFO_*), GPTQ_INFO_BAD_HESSIAN.
 * Requirements: cols % 4 == 0; S_H_dev and R_dev 16-byte aligned (the matrix products run on
 * the tensor cores through TMA, whose rows must start on 16-byte boundaries).
 * Errors: GPTQ_EINVAL (null pointers, cols <= 0 or not a multiple of 4, misaligned buffers,
 * n_total <= 0, damp_rel < 0), GPTQ_EWORKSPACE.
 */
gptq_status gptq_prepare_hinv(float* S_H_dev, float* R_dev, int64_t cols, int64_t n_total,
                              float damp_rel, void* ws_dev, size_t ws_bytes, int32_t* info_dev,
                              void* stream);

/*
 * gptq_prepare_hinv with an explicit route (a gptq_route value; anything else is GPTQ_EINVAL).
 *
 * GPTQ_ROUTE_THREE_STEP follows the pages step by step (two Cholesky factorizations, a
 * triangular inverse and a triangular product: 4/3 cols^3 flops). GPTQ_ROUTE_REVERSED uses that
 * the upper factor is unique: with J the permutation that reverses the column order,
 * J H_d J = M M^T (lower M) gives H_d = U U^T with U = J M J upper, so H_d^-1 = U^-T U^-1 and
 * R = U^-1 = J M^-1 J -- one Cholesky and one triangular inverse (2/3 cols^3 flops). Arguments,
 * outputs, workspace and errors are those of gptq_prepare_hinv.
 */
gptq_status gptq_prepare_hinv_route(float* S_H_dev, float* R_dev, int64_t cols, int64_t n_total,
                                    float damp_rel, int route, void* ws_dev, size_t ws_bytes,
                                    int32_t* info_dev, void* stream);

/*
 * S6-S8 -- the GPTQ column loop with lazy batch updates.
 *
 * Source: "Part 3: Adaptive Rounding: GPTQ", "Observation 1" (one fixed left-to-right column
 * order shared by all rows), "Observation 2: Lazy Batch Updates" (B columns processed on chip,
 * later columns updated by one matrix product per block) and "Algorithm GPTQ"; the update
 * W[:, B:] -= E R[B, B:] as the Vietnamese edition of the GPTQ blog writes it ("2. Lazy batch
 * update"); the design table (asymmetric uniform, 3-4 bit, per row or group 128) and the blog's
 * "Group-wise quantization". For each block of B columns [b0, b1) and each column j in order:
 *     q_j   = clamp(rint(w_j / s) + z, 0, 2^bits - 1)           (float32, round half to even)
 *     what_j = s * (q_j - z)
 *     e_j   = (w_j - what_j) / R[j][j];   E[:, j - b0] = e_j
 *     W[:, j+1 : b1] -= e_j * R[j, j+1 : b1]                    (in-block, on chip)
 *   then W[:, b1:] -= E * R[b0:b1, b1:]                           (lazy trailing update)
 * Grid of a row or group: lo = min(0, min v), hi = max(0, max v) (an all-zero v uses [-1, 1]),
 * s = (hi - lo) / (2^bits - 1), z = clamp(rint(-lo / s), 0, 2^bits - 1), each step rounded once
 * in float32. Per-row grids come from the ORIGINAL weights; group grids from the current
 * (already compensated) weights when the group's first column is reached.
 *
 *   W_dev      original weights [rows x ldw] (GPTQ_BF16 or GPTQ_FP32); not modified.
 *   R_dev      float32 [cols x cols] from gptq_prepare_hinv (upper triangle read).
 *   bits       2..8.
 *   group      -1 (one grid per row) or a group size g >= 1 with cols % g == 0 and either
 *              g % block == 0 or block % g == 0.
 *   block      B, one of 32, 64, 128.
 *   W_hat_dev  out: float32 [rows x cols], ld = cols: the dequantized weights s * (q - z).
 *              Also the working buffer of the loop.
 *   codes_dev  out: uint8 [rows x cols], ld = cols, values 0 .. 2^bits - 1 (unpacked).
 *   scales_dev out: float32 [rows x G]; zeros_dev out: uint8 [rows x G]; G = 1 (per-row) or
 *              cols / group.
 *   err_sq_dev out (may be NULL): float32 [rows], sum over j of e_j^2 (the damped proxy loss of
 *              the row, since W_hat - W = -e R and (H + lambda I) = R^-1 R^-T).
 *   ws_dev     device workspace of gptq_workspace_size(GPTQ_WS_QUANTIZE, rows, cols, block)
 *              bytes, 256-byte aligned.
 *   info_dev   status word.
 * Requirements: cols % 4 == 0; R_dev and W_hat_dev 16-byte aligned.
 * Errors: GPTQ_EINVAL (shapes, bits, group/block rules, alignment, null pointers),
 * GPTQ_EWORKSPACE.
 */
gptq_status gptq_quantize_layer(const void* W_dev, gptq_dtype w_dtype, int64_t rows, int64_t cols,
                                int64_t ldw, const float* R_dev, int bits, int group, int block,
                                float* W_hat_dev, uint8_t* codes_dev, float* scales_dev,
                                uint8_t* zeros_dev, float* err_sq_dev, void* ws_dev,
                                size_t ws_bytes, int32_t* info_dev, void* stream);

/*
 * gptq_quantize_layer without a workspace argument, for callers that cannot allocate device
 * memory (no counterpart on the pages: it packages the same S6-S8 computation differently).
 *
 * Who needs it: code whose host framework owns all device memory through its own pool, where a
 * cudaMalloc of its own would fail or break the pool's accounting, and code that may not pay
 * cudaMalloc's implicit device-wide synchronization. It computes exactly what gptq_quantize_layer
 * computes, with the same arguments and outputs (the caller still passes all inputs and outputs),
 * but keeps the error buffer E in a scratch array compiled into the library:
 *   - size GPTQ_NOALLOC_SCRATCH_BYTES (16 MiB); every GPU that loads the library holds it
 *     until exit;
 *   - a call needing more than that, i.e. gptq_workspace_size(GPTQ_WS_QUANTIZE, rows, cols,
 *     block) bytes (2 * rows * block * 4 + 2 * block * cols * 4, each part rounded up to 256),
 *     returns GPTQ_EWORKSPACE without enqueueing anything; at block 128 a layer of up to
 *     8192 x 8192 fits;
 *   - the first call on each device looks up the array's device address (cudaGetSymbolAddress
 *     with that device current) and keeps it for the life of the process; make that first call
 *     before any stream capture. After a cudaDeviceReset of that device the kept address is
 *     stale: do not use this entry point on a device that has been reset;
 *   - all calls in the process share the one array per device and it keeps the last call's
 *     contents (nothing in it needs to start at zero); calls whose work overlaps on the GPU, e.g.
 *     on two streams at once, race on it -- serialize them.
 * Errors: the argument checks of gptq_quantize_layer run first and give its codes (GPTQ_EINVAL,
 * GPTQ_EUNSUPPORTED); a call that passes them but needs more than the built-in scratch returns
 * GPTQ_EWORKSPACE.
 */
#define GPTQ_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)
gptq_status gptq_quantize_layer_noalloc(const void* W_dev, gptq_dtype w_dtype, int64_t rows,
                                        int64_t cols, int64_t ldw, const float* R_dev, int bits,
                                        int group, int block, float* W_hat_dev, uint8_t* codes_dev,
                                        float* scales_dev, uint8_t* zeros_dev, float* err_sq_dev,
                                        int32_t* info_dev, void* stream);

/*
 * Packed 4-bit codes -- the storage the W4A16 product reads.
 *
 * Source: "GPTQ second-order quantization" blog, "What the original results established" (GPTQ
 * is weight-only; the W4A16 runtime gains speed by moving fewer weight bytes and unpacking them
 * in its kernel) and its Vietnamese version, "Group-wise quantization" (the packed layout is chosen
 * together with the group size and the runtime kernel). The pages fix no layout; this one is:
 *   eight codes per little-endian 32-bit word, row after row: code (r, c) is held in bits
 *   4*(c % 8) .. 4*(c % 8) + 3 of word packed[r * (cols / 8) + c / 8]. Equivalently byte c / 2 of
 *   row r holds column c in its low nibble when c is even and in its high nibble when c is odd.
 *
 *   codes_dev   uint8 [rows x ldc] (columns 0..cols-1 used), e.g. gptq_quantize_layer's codes at
 *               bits <= 4. 8-byte aligned, ldc % 8 == 0.
 *   packed_dev  uint32 [rows x cols/8], dense (row stride cols / 2 bytes), 4-byte aligned; written.
 *   info_dev    status word (may be NULL): GPTQ_INFO_BAD_CODE if a code is 16 or more; its low
 *               four bits are stored.
 * rows == 0 enqueues nothing. Errors: GPTQ_EINVAL (null pointers, cols <= 0, cols % 8 != 0,
 * ldc < cols, alignment).
 */
gptq_status gptq_pack_codes_4bit(const uint8_t* codes_dev, int64_t rows, int64_t cols, int64_t ldc,
                                 uint32_t* packed_dev, int32_t* info_dev, void* stream);

/*
 * Packed 3-bit codes -- the storage for layers quantized on 3-bit grids (8 levels), 3/8 of the
 * uint8 code bytes.
 *
 * Source: as gptq_pack_codes_4bit ("GPTQ second-order quantization" blog, "What the original
 * results established"; the Vietnamese version, "Group-wise quantization"): the packed layout is
 * chosen with the bit width and the runtime kernel, and the pages fix none. This one is:
 *   32 codes per three little-endian 32-bit words, row after row: the codes of columns 32k ..
 *   32k + 31 of row r form the 96-bit little-endian number sum_i q_i 8^i held in words
 *   packed[r * (3 * cols / 32) + 3k + j], j = 0, 1, 2 (word j holding bits 32j .. 32j + 31);
 *   code (r, c) therefore sits in bits 3 (c % 32) .. 3 (c % 32) + 2, and the codes of columns
 *   32k + 10 and 32k + 21 straddle two words.
 *
 *   codes_dev   uint8 [rows x ldc] (columns 0..cols-1 used), e.g. gptq_quantize_layer's codes at
 *               bits <= 3. 8-byte aligned, ldc % 8 == 0.
 *   packed_dev  uint32 [rows x 3 cols/32], dense (row stride 3 cols / 8 bytes), 4-byte aligned;
 *               written.
 *   info_dev    status word (may be NULL): GPTQ_INFO_BAD_CODE if a code is 8 or more; its low
 *               three bits are stored.
 * rows == 0 enqueues nothing. Errors: GPTQ_EINVAL (null pointers, cols <= 0, cols % 32 != 0,
 * ldc < cols, ldc % 8 != 0, alignment).
 */
gptq_status gptq_pack_codes_3bit(const uint8_t* codes_dev, int64_t rows, int64_t cols, int64_t ldc,
                                 uint32_t* packed_dev, int32_t* info_dev, void* stream);

/*
 * W4A16 product: Y = X W_hat^T with W_hat read from packed 4-bit codes and dequantized on the fly,
 *   Y[n][r] = sum_c X[n][c] * s[r, g(c)] * (q[r][c] - z[r, g(c)]),  g(c) = c / group (0 per row).
 *
 * Source: "GPTQ second-order quantization" blog, "What the original results established" (W4A16:
 * BF16 activations, weight bytes moved packed and dequantized in the kernel) and "Group-wise
 * quantization" (scale and zero point per row or per group of input channels). One call serves a
 * decode step (n = 1, a matrix-vector product), a small batch of activation vectors (n <= 16, the
 * same kernel) or a larger batch (n > 16: a tensor-core kernel, weights as the MMA's 128-row M,
 * activation rows as its N).
 *
 *   packed_dev  codes in the layout of gptq_pack_codes_4bit, [rows x cols/8] uint32, 16-byte
 *               aligned.
 *   scales_dev  float32 [rows x G], zeros_dev uint8 [rows x G] (as gptq_quantize_layer writes
 *               them); G = 1 for group == -1, else cols / group. Zero points above 127 are not
 *               supported (4-bit quantizers produce 0..15).
 *   group       -1 (per row) or a multiple of 128 that divides cols.
 *   X_dev       activations [n x ldx], token-major, x_dtype GPTQ_BF16 only; 16-byte aligned,
 *               ldx % 8 == 0, ldx >= cols.
 *   Y_dev       float32 [n x ldy] output, ldy >= rows; fully overwritten in columns 0..rows-1.
 *   info_dev    status word (may be NULL): GPTQ_INFO_TIMEOUT if a copy wait expires.
 * Empty calls (rows == 0 or n == 0) are checked for shapes only and may pass NULL buffers.
 * Arithmetic: q - z is formed exactly in bf16 and multiplied by X on the tensor cores with fp32
 * accumulation over each 128-column chunk; the chunk sum is scaled by s in fp32 and the chunks
 * are added in a fixed order, so results are deterministic for a given device and shape. For
 * n > 16 on a layer with few 128-row tiles the columns may be split in two halves whose sums are
 * added into Y after Y is zeroed (a sum of two terms onto zero does not depend on their order).
 * rows == 0 or n == 0 enqueues nothing. Errors: GPTQ_EINVAL (null pointers, cols <= 0,
 * cols % 32 != 0, group rules, ld or alignment rules, n < 0), GPTQ_EUNSUPPORTED (x_dtype other than
 * GPTQ_BF16, n above 65535 * 128, rows above 2^27, cols above 2^22, rows * G of 2^31 or more).
 */
gptq_status gptq_w4a16_matmul(const uint32_t* packed_dev, const float* scales_dev,
                              const uint8_t* zeros_dev, int64_t rows, int64_t cols, int group,
                              const void* X_dev, gptq_dtype x_dtype, int64_t n, int64_t ldx,
                              float* Y_dev, int64_t ldy, int32_t* info_dev, void* stream);

/*
 * Data-free randomized Hadamard rotation of the input-channel axis, applied before GPTQ:
 *   Y = X Q,  Q = diag(s) (I_{n/b} (x) H_b) / sqrt(b),
 * H_b the Sylvester Hadamard matrix of order b (entry (i, j) = (-1)^popcount(i & j)), b = the
 * largest power of two dividing n, at most 4096 (gptq_hadamard_block), s_j = -1 where bit j % 32
 * of sign_bits[j / 32] is set, else +1.
 *
 * Source: "OptRot: Mitigating Weight Outliers via Data-Free Rotations for Post-Training
 * Quantization", Abstract and Figure 1 (rotations fused into the weights and, transposed, into the
 * activations leave the layer output unchanged and spread weight outliers) and Theorem 3.1 (the
 * round-to-nearest error bound grows with the weight incoherence). The page learns its rotations;
 * this is the data-free randomized Hadamard member of the family it compares against. Rotating
 * both W (rows = output channels) and the token-major calibration X with the same Q gives
 * W' X'^T = W X^T and H' = Q^T H Q, so GPTQ can then run on (W', X') unchanged.
 *
 *   X_dev      [rows x ldx], x_dtype GPTQ_BF16 or GPTQ_FP32; columns 0..n-1 rotated.
 *   n          multiple of 32.
 *   sign_bits_dev  n / 32 uint32 words (drawn by the caller), or NULL for s = +1.
 *   Y_dev      [rows x ldy], y_dtype GPTQ_BF16 (round to nearest even) or GPTQ_FP32. Y may be X
 *              itself (same dtype and ld); otherwise the two must not overlap.
 * Arithmetic: fp32 butterflies (log2 b stages), then the 1/sqrt(b) scale (exact for even log2 b);
 * deterministic. Requirements: X_dev, Y_dev 16-byte aligned; ldx and ldy times the element size
 * multiples of 16 bytes. rows == 0 enqueues nothing. Errors: GPTQ_EINVAL (shapes, dtypes,
 * alignment, null pointers, X == Y with different dtype or ld), GPTQ_EUNSUPPORTED (more than
 * 2^31 - 1 tiles of 4096 elements).
 */
int gptq_hadamard_block(int64_t n);
gptq_status gptq_hadamard_rotate(const void* X_dev, gptq_dtype x_dtype, int64_t rows, int64_t n,
                                 int64_t ldx, const uint32_t* sign_bits_dev, void* Y_dev,
                                 gptq_dtype y_dtype, int64_t ldy, void* stream);

/*
 * OBQ: greedy-order quantization of small layers with explicit inverse-Hessian downdates, the
 * reference that GPTQ's fixed left-to-right order is measured against.
 *
 * Source: "Part 2: Adaptive Rounding: Optimal Brain Quantizer (OBQ)", sections "Greedy Search"
 * (each step quantizes the remaining weight whose quantization raises the proxy loss least,
 * (w_p - q_p)^2 / H^-1[p, p] up to a factor 2), "Generalized Weight Update" (the other weights
 * move by -(w_p - q_p) H^-1[:, p] / H^-1[p, p]), "The OBS / GPTQ Trick" (H^-1 loses weight p by
 * the rank-1 downdate H^-1 - H^-1[:, p] H^-1[p, :] / H^-1[p, p]) and "Limitations of OBQ" (each row
 * needs its own H^-1, which is why this reference is limited to small layers).
 *
 *   W_dev       float32 [rows x ldw], columns 0..cols-1; not modified.
 *   cols        1 .. 128.
 *   Hinv_dev    float64 [cols x cols], ld = cols: the symmetric inverse of the damped Hessian
 *               shared by all rows (e.g. R^T R from gptq_prepare_hinv, in fp64).
 *   bits        2 .. 8; one grid per row from the original W (GPTQ's per-row grid: min/max with 0
 *               included, float32, round half to even).
 *   order_mode  GPTQ_OBQ_GREEDY (OBQ) or GPTQ_OBQ_NATURAL (left to right: GPTQ's order with the
 *               same explicit downdates).
 * Outputs (rows x cols, ld = cols): codes_dev uint8, W_hat_dev float32 = s (q - z); order_dev
 * int32 (column quantized at each step; may be NULL); loss_dev float64 [rows] = sum over the steps
 * of (w_p - q_p)^2 / H^-1[p, p], which equals (w_hat - w)^T H_d (w_hat - w) (may be NULL);
 * scales_dev float32 [rows] and zeros_dev uint8 [rows] (may be NULL).
 * Arithmetic: fp64 for the weights and H^-1, each operation rounded once in a fixed order (no fused
 * multiply-adds); greedy ties go to the lowest column. Results are reproducible operation by
 * operation. rows == 0 enqueues nothing. Errors: GPTQ_EINVAL (shapes, bits, mode, null pointers),
 * GPTQ_EUNSUPPORTED (cols > 128).
 */
#define GPTQ_OBQ_NATURAL 0
#define GPTQ_OBQ_GREEDY 1
gptq_status gptq_obq_quantize(const float* W_dev, int64_t rows, int64_t cols, int64_t ldw,
                              const double* Hinv_dev, int bits, int order_mode,
                              uint8_t* codes_dev, float* W_hat_dev, int32_t* order_dev,
                              double* loss_dev, float* scales_dev, uint8_t* zeros_dev,
                              void* stream);

/* Workspace bytes needed by one call (GPTQ_WS_PREPARE or GPTQ_WS_QUANTIZE); 0 for bad input. */
size_t gptq_workspace_size(int which, int64_t rows, int64_t cols, int block);

/* Maps a status word read back from the device to a gptq_status (0 -> GPTQ_OK,
   pivot codes -> GPTQ_ENOTPD, GPTQ_INFO_TIMEOUT -> GPTQ_ETIMEOUT, others -> GPTQ_EINVAL). */
gptq_status gptq_info_status(int32_t info);

/* Static, human-readable name of a status code. */
const char* gptq_status_string(int status);

/* Number of CUDA kernels this library has enqueued since it was loaded, over all calls and
   devices (a diagnostic counter; copies and memsets are not counted). */
uint64_t gptq_kernel_launches(void);

/*
 * Self-test of the bounded device waits (no counterpart on the pages). Enqueues one CTA that
 * waits on a shared-memory barrier nothing will ever arrive on, giving up after limit_ms
 * milliseconds (1..10000); on giving up it writes GPTQ_INFO_TIMEOUT into *info_dev and returns,
 * leaving the context usable. Lets callers check that a lost wait ends as a status, not a hang.
 */
gptq_status gptq_selftest_wait_timeout(int32_t* info_dev, int limit_ms, void* stream);

/*
 * Self-test of the bounded waits on flags in global memory, the form the fused factorization
 * step uses between its CTAs (no counterpart on the pages). Enqueues one thread that waits for
 * *flag_dev >= 1 (flag_dev: a caller-owned, 4-byte aligned device int32), reading it with acquire
 * semantics; if it has not reached 1 after limit_ms milliseconds (1..10000) the thread writes
 * GPTQ_INFO_TIMEOUT into *info_dev and returns, leaving the context usable. With *flag_dev >= 1
 * it returns at once and leaves *info_dev alone. Errors: GPTQ_EINVAL for null or misaligned
 * pointers or a limit out of range, GPTQ_ECUDA for a launch failure.
 */
gptq_status gptq_selftest_flag_timeout(const int32_t* flag_dev, int32_t* info_dev, int limit_ms,
                                       void* stream);

/*
 * Self-test of the tensor-core matrix product every S3-S5 and S8 step runs on (no counterpart on
 * the pages). Computes, in the 3xTF32 scheme (operands split into tf32 big/small parts; the
 * small*small term is dropped):
 *     C[m][n] = alpha * sum_{k = klo}^{K-1} opA[m][k] * opB[k][n] + beta * C[m][n]
 *   opA[m][k] = a_mn ? A[k * lda + m] : A[m * lda + k];  opB[k][n] = b_mn ? B[k * ldb + n]
 *   : B[n * ldb + k]; with `lower`, 128 x 128 tiles of C above the diagonal are left untouched;
 *   klo = max(0, tile row start if klo_from_m, tile column start if klo_from_n).
 * C_big / C_small (may be NULL) receive the tf32 split of the result with ld ldc.
 * ws: at least 2 * (rows_A * lda + rows_B * ldb) * 4 bytes + 1024, where rows_A = a_mn ? K : M
 * and rows_B = b_mn ? K : N. Requirements: lda, ldb, ldc multiples of 4; 16-byte aligned buffers.
 */
gptq_status gptq_selftest_gemm(const float* A_dev, int64_t lda, int a_mn, const float* B_dev,
                               int64_t ldb, int b_mn, float* C_dev, int64_t ldc, int M, int N,
                               int K, float alpha, float beta, int lower, int klo_from_m,
                               int klo_from_n, float* C_big_dev, float* C_small_dev, void* ws_dev,
                               size_t ws_bytes, int32_t* info_dev, void* stream);

/* Library version, "major.minor.patch". */
const char* gptq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GPTQ_B200_H */
