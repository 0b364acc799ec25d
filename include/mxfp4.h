/*
 * mxfp4.h -- C ABI of libmxfp4.so: MXFP4 block fake quantisation
 * (quantise-dequantise, "QDQ") and its straight-through-estimator backward on
 * NVIDIA B200 (sm_100a).
 *
 * What is computed (web pages cited by title and section):
 *   amct pull request 264, "feat: MXFP4 QAT fake-quant Linear (with STE)",
 *   mxfp4_qat/fake_quant.py:
 *     - _block_view / _block_scale: blocks of `block` consecutive elements
 *       share a power-of-two scale 2^k,
 *         PAGE  mode: k = round(log2(max(amax / scale_factor, 2^-30)))
 *       (fp32 division; round() is the exact nearest integer of log2);
 *         FLOOR mode: k = max(floor(log2 amax) - 2, -127) (the OCP-MX rule;
 *       scale_factor is not used).
 *     - _round_to_e2m1 / _quant_dequant_torch: y = x / 2^k in fp32, |y| is
 *       rounded to the E2M1 codebook {0, .5, 1, 1.5, 2, 3, 4, 6} by counting
 *       the midpoints {.25, .75, 1.25, 1.75, 2.5, 3.5, 5} that are <= |y|
 *       (ties go to the larger code, |y| >= 5 gives 6), the output is
 *       sign(y) * code * 2^k in fp32, cast to the input dtype.
 *     - mxfp4_saturation_mask: an element saturates when |x| > 6 * 2^k.
 *     - _MXFP4FakeQuantSTE.backward: grad_in = grad_out (plain STE) or
 *       grad_out with saturated positions set to +0.0 (clipped STE).
 *   MindSpore hyper-parallel, fake_w4a8_gmm_func.py, FakeW4A8GroupedLinear:
 *     - quantize_input(rowwise=, colwise=, group_list=, group_list_type=):
 *       "row-wise" blocks run along a row, "column-wise" blocks run down a
 *       column; with a group_list the column-wise blocks restart at every
 *       group start so that no block straddles two MoE groups.
 *     - normalize_group_list: type 1 = per-group counts (turned into
 *       cumulative offsets by a running sum), type 0 = cumulative end offsets.
 *   sglang mxfp4_npu.py: two E2M1 values packed per byte.
 *
 * Data layout (all row-major, element strides in elements):
 *   x, y_row, y_col, grads      [rows][cols], leading dimensions ld / ld_y /
 *                               ld_grad (>= cols); dtype fp32 or bf16.
 *   codes_row, codes_col        E2M1: [rows][ceil(cols/2)] bytes, contiguous;
 *                               the nibble of element c is the low nibble of
 *                               byte c/2 when c is even, the high one when
 *                               odd; nibble = sign << 3 | code index (E2M1
 *                               bits). E4M3 (elem_format): [rows][cols]
 *                               bytes, one E4M3 code per element.
 *   scales_row                  [rows][ceil(cols/block)] E8M0 bytes (k + 127),
 *                               row-major, or (scales_row_layout =
 *                               MXFP4_SCALES_MMA) in the scale-factor layout
 *                               that block-scaled tensor-core GEMMs read
 *                               (cuBLAS documentation, "1D block scaling
 *                               factors layout"): the [rows][nblk] matrix is
 *                               cut into atoms of 128 rows x 4 block columns,
 *                               512 bytes each, stored atom row by atom row
 *                               (atom (i, j) at byte 512 * (i * ceil(nblk/4)
 *                               + j)); inside an atom, entry (r, c) sits at
 *                               byte 16 * (r % 32) + 4 * (r / 32) + c. The
 *                               buffer holds mxfp4_scales_row_bytes() bytes;
 *                               entries past rows or nblk (the padding of the
 *                               last atoms) are not written.
 *   scales_col                  [S][cols] E8M0 bytes, S = sum over groups of
 *                               ceil(group rows / block), groups in order.
 *                               mxfp4_colwise_scale_rows() gives S from a host
 *                               copy of the group_list; allocating
 *                               mxfp4_colwise_scale_rows_bound() rows needs no
 *                               host copy (rows past S are left untouched).
 *   mask_row, mask_col          [rows][ceil(cols/8)] bytes; bit b of byte j is
 *                               the saturation flag of element 8j+b.
 * Non-finite blocks (a NaN or +-inf element, or a scale that overflows fp32)
 * write the quiet NaN 0x7FC0 / 0x7FC00000 to every output element, code 0,
 * E8M0 byte 0xFF and no saturation bits.
 *
 * Ownership: every pointer is a device pointer owned by the caller, except
 * where a parameter says "host". The library allocates no memory and keeps no
 * state between calls. Calls are asynchronous on `stream`; inputs must stay
 * valid and outputs unread until the stream reaches the call.
 *
 * Errors: argument errors are found on the host before any launch and
 * returned as a status (nothing is written). A group_list lives in device
 * memory, so its validity (non-negative counts, non-decreasing offsets, last
 * offset == rows) is checked by the kernels: with an invalid list no
 * column-wise output and no gradient is written (row-wise outputs, which do
 * not depend on the groups, may be) and, when `status` is non-NULL, the
 * kernels store MXFP4_EINVAL there (MXFP4_OK otherwise), so that a caller
 * that passes a group_list must read `status` before using any output. No
 * kernel traps or asserts.
 */
#ifndef MXFP4_H
#define MXFP4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st* mxfp4_stream_t;

typedef enum {
    MXFP4_OK = 0,
    MXFP4_EINVAL = 1,       /* invalid argument (also an invalid group_list) */
    MXFP4_EUNSUPPORTED = 2, /* valid but not supported (block other than 32/128, too many groups) */
    MXFP4_ECUDA = 3         /* a CUDA runtime call or launch failed */
} mxfp4_status;

typedef enum { MXFP4_F32 = 0, MXFP4_BF16 = 1 } mxfp4_dtype;

typedef enum {
    MXFP4_SCALE_PAGE = 0,  /* 2^round(log2(max(amax / scale_factor, 2^-30))) */
    MXFP4_SCALE_FLOOR = 1  /* 2^max(floor(log2 amax) - 2, -127) */
} mxfp4_scale_mode;

/* Direction bits for mxfp4_qdq_args.dirs and grad_dir. */
#define MXFP4_ROWWISE 1u
#define MXFP4_COLWISE 2u

/* Largest num_groups a call accepts. */
#define MXFP4_MAX_GROUPS 4096

/* Element formats (mxfp4_qdq_args.elem_format). E4M3 is the MXFP8 element of
 * the W4A8 path (MindSpore hyper-parallel fake_w4a8_gmm_func.py,
 * FakeW4A8GroupedLinear, which quantises activations and gradients to MXFP8;
 * the page names the operators only). Its reading is the OCP Microscaling
 * rule: scale 2^(floor(log2 amax) - 8) saturated below at 2^-127 (E4M3's
 * largest normal is 1.75 * 2^8 = 448), each x / scale rounded to the nearest
 * E4M3 value with ties to the even code and magnitudes above 448 saturating
 * to 448, the sign kept (-0 and negative values rounding to zero give code
 * 0x80); output decode(code) * scale in x's dtype; saturation |x| > 448 *
 * scale. E4M3 requires block 32 and MXFP4_SCALE_FLOOR (else
 * MXFP4_EUNSUPPORTED); its codes are one byte per element, [rows][cols] for
 * both directions. Non-finite blocks as for E2M1. */
#define MXFP4_ELEM_E2M1 0
#define MXFP4_ELEM_E4M3 1

/* Layouts of scales_row (mxfp4_qdq_args.scales_row_layout). */
#define MXFP4_SCALES_ROWMAJOR 0
#define MXFP4_SCALES_MMA 1

/* Layouts of codes_col and scales_col (mxfp4_qdq_args.col_layout).
 *
 * MXFP4_COLS_ROWMAJOR (0): as described at the top of this file.
 *
 * MXFP4_COLS_MMA: the column-wise result as the operand of a block-scaled
 * tensor-core GEMM that contracts over the rows, group by group -- the
 * weight-gradient GEMM of a grouped linear layer, which multiplies the
 * column-wise views of activations and gradients transposed (MindSpore
 * hyper-parallel fake_w4a8_gmm_func.py, FakeW4A8GroupedLinear._select_operands,
 * layout "TN"; the page fixes no byte layout, this is the library's). Each
 * group's K range is its rows padded to a multiple of 128 (four blocks of 32,
 * one column of scale atoms); group g starts at K slot
 * K0_g = sum_{j<g} 128 * ceil(n_j / 128), and k_alloc (a multiple of 128, at
 * least the sum over all groups; mxfp4_colwise_operand_k) is the K extent of
 * the buffers:
 *   codes_col   [cols][k_alloc / 2] bytes, 16-byte aligned: the E2M1 nibble of
 *               x[first row of g + t][c] is in byte c * k_alloc/2 + (K0_g + t)/2,
 *               the low nibble for even t; slots t >= n_g of the group's padded
 *               range hold 0. Row c is K-major: the operand as it stands.
 *   scales_col  the [cols][k_alloc / 32] E8M0 matrix whose entry
 *               (c, K0_g/32 + b) is the scale of block b of group g in column c
 *               (127 for the padding blocks of a group), in the 128 x 4 atom
 *               layout of MXFP4_SCALES_MMA; 2-byte aligned;
 *               mxfp4_colwise_operand_scale_bytes() bytes. Atom rows past cols
 *               and K slots past the last group are not written.
 * Group g's operand is then the [cols][128 ceil(n_g/128)] sub-matrix at K0_g
 * (row stride k_alloc/2 bytes) with the atom columns from K0_g/128 on.
 * Requires bf16 x, block 32, E2M1, and in PAGE mode
 * a scale_factor in [2^-64, 11] (else MXFP4_EUNSUPPORTED); no fused backward.
 * y_col and mask_col, when also given, keep their row-major layout. An
 * invalid group_list, or groups whose padded K exceeds k_alloc, write no
 * operand byte and set status to MXFP4_EINVAL.
 */
#define MXFP4_COLS_ROWMAJOR 0
#define MXFP4_COLS_MMA 1

#define MXFP4_ABI_VERSION 5

/*
 * Arguments of one QDQ call. Zero-initialise and fill what is used; every
 * NULL output is skipped.
 *   x              input [rows][cols], leading dimension ld; may be NULL only
 *                  when mxfp4_ste_bwd reads a saved mask.
 *   dtype          MXFP4_F32 or MXFP4_BF16 (x, y_* and grads share it).
 *   block          32 or 128 elements per scale.
 *   rows, cols     >= 0; a call with rows*cols == 0 does nothing.
 *   scale_factor   PAGE mode divisor (default 6.0); must be finite and > 0
 *                  in every mode (the page's check).
 *   scale_mode     mxfp4_scale_mode.
 *   dirs           MXFP4_ROWWISE, MXFP4_COLWISE or both: both directions are
 *                  computed from one read of x.
 *   group_list     optional device int64[num_groups]; applies to column-wise
 *                  blocks only; NULL means one group of all rows.
 *   group_list_type 0 = cumulative end offsets, 1 = counts.
 *   status         optional device int32 that receives the group_list check.
 *   y_row, y_col   dequantised outputs, x's dtype, leading dimension ld_y.
 *   scales_row_layout MXFP4_SCALES_ROWMAJOR (0) or MXFP4_SCALES_MMA: the
 *                  latter, with block 32, gives the E8M0 operand scales of an
 *                  MXFP4 block-scaled GEMM whose K dimension is `cols`
 *                  (codes_row is then its K-major E2M1 operand as is).
 *   elem_format    MXFP4_ELEM_E2M1 (0, MXFP4) or MXFP4_ELEM_E4M3 (MXFP8).
 *   col_layout     MXFP4_COLS_ROWMAJOR (0) or MXFP4_COLS_MMA (the K-major
 *                  GEMM operand layout of codes_col / scales_col).
 *   k_alloc        MXFP4_COLS_MMA only: K slots per codes_col row (a multiple
 *                  of 128, >= mxfp4_colwise_operand_k()).
 */
typedef struct mxfp4_qdq_args {
    const void* x;
    int32_t dtype;
    int32_t block;
    int64_t rows;
    int64_t cols;
    int64_t ld;
    float scale_factor;
    int32_t scale_mode;
    uint32_t dirs;
    int32_t group_list_type;
    const int64_t* group_list;
    int64_t num_groups;
    int32_t* status;
    void* y_row;
    void* y_col;
    int64_t ld_y;
    uint8_t* codes_row;
    uint8_t* scales_row;
    uint8_t* mask_row;
    uint8_t* codes_col;
    uint8_t* scales_col;
    uint8_t* mask_col;
    int32_t scales_row_layout;
    int32_t elem_format;
    int32_t col_layout;
    int64_t k_alloc;
} mxfp4_qdq_args;

/*
 * QDQ forward (fake_quant.py: mxfp4_quant_dequant, mxfp4_saturation_mask;
 * fake_w4a8_gmm_func.py: quantize_input with rowwise/colwise/group_list).
 * One pass over x writes every requested output of every requested direction:
 * dequantised values, packed E2M1 codes, E8M0 scales and saturation bitmasks
 * (the bitmask is what the clipped STE backward later reads, so a forward
 * with mask_row set is the fused "forward + saved mask" step).
 * Returns MXFP4_OK once the work is queued.
 */
mxfp4_status mxfp4_qdq_fwd(const mxfp4_qdq_args* args, mxfp4_stream_t stream);

/*
 * Clipped/plain STE backward (fake_quant.py: _MXFP4FakeQuantSTE.backward).
 *   geom        shape, dtype, block, scale mode/factor, and exactly one
 *               direction bit in dirs (the direction whose saturation masks
 *               the gradient), plus x and group_list when the mask is
 *               recomputed; its output pointers are ignored.
 *   grad_out    [rows][cols], leading dimension ld_grad, geom->dtype.
 *   grad_in     [rows][cols], leading dimension ld_grad; may equal grad_out.
 *   saved_mask  bit-packed mask from a forward call, or NULL to recompute the
 *               mask from x ("saved-free": one extra read of x).
 *   clip_grad   0: grad_in = grad_out. 1: grad_in = grad_out with +0.0 where
 *               the element saturated.
 */
mxfp4_status mxfp4_ste_bwd(const mxfp4_qdq_args* geom, const void* grad_out, void* grad_in,
                           int64_t ld_grad, const uint8_t* saved_mask, int32_t clip_grad,
                           mxfp4_stream_t stream);

/*
 * Fused forward + clipped-STE backward in one pass: everything mxfp4_qdq_fwd
 * writes for `args`, plus grad_in = grad_out masked by the saturation of the
 * direction grad_dir (which must be one of args->dirs). Used when the
 * incoming gradient is already known at quantisation time (recomputation in
 * the backward pass, or a measured training step).
 */
mxfp4_status mxfp4_qdq_fwd_bwd(const mxfp4_qdq_args* args, const void* grad_out, void* grad_in,
                               int64_t ld_grad, uint32_t grad_dir, mxfp4_stream_t stream);

/*
 * Number of column-wise scale rows S for a group_list held in HOST memory
 * (fake_w4a8_gmm_func.py: normalize_group_list, then sum of ceil(n_g/block)).
 * Returns -1 when the list is not a valid partition of [0, rows).
 */
int64_t mxfp4_colwise_scale_rows(const int64_t* host_group_list, int64_t num_groups,
                                 int32_t group_list_type, int64_t rows, int32_t block);

/* Upper bound on S that needs no group sizes: floor(rows/block) + num_groups
 * (ceil(rows/block) without groups). */
int64_t mxfp4_colwise_scale_rows_bound(int64_t rows, int64_t num_groups, int32_t block);

/* Bytes of a scales_row buffer for `rows` x `cols` with blocks of `block` in
 * `layout` (MXFP4_SCALES_ROWMAJOR: rows * ceil(cols/block); MXFP4_SCALES_MMA:
 * 512 * ceil(rows/128) * ceil(ceil(cols/block)/4)); -1 for invalid arguments. */
int64_t mxfp4_scales_row_bytes(int64_t rows, int64_t cols, int32_t block, int32_t layout);

/* MXFP4_COLS_MMA: the K extent sum_g 128 * ceil(n_g / 128) of a group_list
 * held in HOST memory (128 * ceil(rows / 128) for a NULL list); -1 when the
 * list is not a valid partition of [0, rows). */
int64_t mxfp4_colwise_operand_k(const int64_t* host_group_list, int64_t num_groups, int32_t group_list_type,
                                int64_t rows);

/* An upper bound on mxfp4_colwise_operand_k that needs no group sizes:
 * 128 * (floor(rows / 128) + num_groups), or 128 * ceil(rows / 128) without
 * groups; -1 for rows < 0. */
int64_t mxfp4_colwise_operand_k_bound(int64_t rows, int64_t num_groups);

/* Bytes of a MXFP4_COLS_MMA scales_col buffer: 512 * ceil(cols / 128) *
 * (k_alloc / 128); -1 for invalid arguments. */
int64_t mxfp4_colwise_operand_scale_bytes(int64_t cols, int64_t k_alloc);

/*
 * Grouped block-scaled GEMM on the tensor cores, the consumer of the
 * operands above (MindSpore hyper-parallel fake_w4a8_gmm_func.py,
 * FakeW4A8GroupedLinear.grouped_matmul over the operands _select_operands
 * picks for the layouts "NN", "NT" and "TN"):
 *   D = A B^T, D[m][n] = sum_k decode(A[m][k]) 2^(sA[m][k/32] - 127)
 *                              decode(B[n][k]) 2^(sB[n][k/32] - 127),
 * accumulated in fp32, stored as fp32 or bf16 (round to nearest even).
 *   elem_format   MXFP4_ELEM_E2M1 (codes_row / MXFP4_COLS_MMA codes: two per
 *                 byte, first element in the low nibble) or MXFP4_ELEM_E4M3
 *                 (one byte per element); both operands alike.
 *   a, lda        A [m][k] codes, K-major, row stride lda bytes (a multiple
 *                 of 16; a 16-byte aligned). k is a multiple of 128.
 *   a_scales      E8M0 scales of A in the MXFP4_SCALES_MMA layout of the
 *                 [m][k/32] scale matrix (mxfp4_scales_row_bytes(m, k, 32,
 *                 MXFP4_SCALES_MMA) bytes).
 *   b, ldb, b_scales  likewise for B.
 *   group_mode    MXFP4_GMM_GROUP_M ("NN" forward, "NT" input gradient): the
 *                 group list partitions the m rows of A and D; group g uses
 *                 B_g = rows [g n, g n + n) of b (b holds num_groups stacked
 *                 [n][k] matrices with row stride ldb) and its scale matrix
 *                 at b_scales + g * mxfp4_scales_row_bytes(n, k, 32,
 *                 MXFP4_SCALES_MMA).
 *                 MXFP4_GMM_GROUP_K ("TN" weight gradient): A [m][k] and B
 *                 [n][k] are column-wise operands in the MXFP4_COLS_MMA
 *                 layout with k = k_alloc; the group list partitions k_rows
 *                 rows (tokens) and group g contracts over its K slots
 *                 [K0_g, K0_g + 128 ceil(n_g / 128)); D holds num_groups
 *                 matrices [m][n], D_g at d + g * m * ldd; an empty group's
 *                 D_g is zero.
 *   d, ldd, d_dtype  output, row stride ldd elements (ldd * element size a
 *                 multiple of 16, d 16-byte aligned), MXFP4_F32 or
 *                 MXFP4_BF16.
 *   status        optional device int32: the group list check (MXFP4_EINVAL:
 *                 not a partition, or GROUP_K groups that need more than k
 *                 slots; nothing is written then) or MXFP4_ECUDA.
 * Argument errors are returned before any launch. Operand values are read
 * as is: NaN scales (0xFF) and the E4M3 NaN code give NaN results.
 */
#define MXFP4_GMM_GROUP_M 0
#define MXFP4_GMM_GROUP_K 1

typedef struct mxfp4_gmm_args {
    int32_t elem_format;
    int32_t group_mode;
    int64_t m, n, k;
    const uint8_t* a;
    int64_t lda;
    const uint8_t* a_scales;
    const uint8_t* b;
    int64_t ldb;
    const uint8_t* b_scales;
    const int64_t* group_list;
    int64_t num_groups;
    int32_t group_list_type;
    int32_t d_dtype;
    int64_t k_rows;
    void* d;
    int64_t ldd;
    int32_t* status;
} mxfp4_gmm_args;

mxfp4_status mxfp4_grouped_gemm(const mxfp4_gmm_args* args, mxfp4_stream_t stream);

/*
 * Dual-level MX quantisation (sglang mxfp4_npu.py, NPUMXFP4DiffusionLinearMethod:
 * npu_dynamic_dual_level_mx_quant turns a bf16 [rows, cols] tensor into E2M1
 * codes, a level-0 scale of shape [rows, cols / level0_block] and a level-1
 * scale, which npu_dual_level_quant_matmul consumes; the page names the
 * operators and their results only, so the arithmetic below is this
 * library's reading of them):
 *   level 0   blocks of level0_block consecutive elements of a row (the last
 *             one partial): s0 = fl32(amax0 / 6), the fp32 level-0 scale
 *             (1 when that quotient is 0, i.e. an all-zero block);
 *   level 1   y = fl32(x / s0) (IEEE division), quantised like one row of
 *             mxfp4_qdq_fwd with block 32: E8M0 scale 2^k1 by scale_mode /
 *             scale_factor from the block's max |y|, E2M1 code of y / 2^k1,
 *             saturation |y| > 6 * 2^k1;
 *   output    fl32((code * 2^k1) * s0) rounded to bf16 (nearest even);
 *   a level-0 block holding a NaN or +-inf writes the quiet NaN 0x7FC0 to
 *   its outputs, code 0, E8M0 bytes 0xFF, no saturation bits and s0 =
 *   0x7FC00000.
 * Arguments (zero-initialise; NULL outputs are skipped):
 *   x            bf16 [rows][cols], leading dimension ld (>= cols) elements.
 *   dtype        MXFP4_BF16 (anything else: MXFP4_EUNSUPPORTED).
 *   rows, cols   >= 0 and below 2^30 (else MXFP4_EUNSUPPORTED).
 *   level0_block 512 (other positive multiples of 32: MXFP4_EUNSUPPORTED;
 *                anything else MXFP4_EINVAL).
 *   scale_factor, scale_mode  the level-1 scale rule, as for mxfp4_qdq_fwd.
 *   y            bf16 [rows][cols], leading dimension ld_y (>= cols).
 *   codes        [rows][ceil(cols/2)] bytes, E2M1 nibbles as codes_row.
 *   scales0      fp32 [rows][ceil(cols/level0_block)], row-major.
 *   scales1      [rows][ceil(cols/32)] E8M0 bytes, row-major.
 *   mask         [rows][ceil(cols/8)] saturation bits as mask_row; the
 *                clipped STE backward reads it through mxfp4_ste_bwd
 *                (saved_mask) unchanged.
 * Device pointers owned by the caller; no allocation; asynchronous on
 * `stream`; argument errors are returned before any launch.
 */
typedef struct mxfp4_dual_level_args {
    const void* x;
    int32_t dtype;
    int32_t level0_block;
    int64_t rows;
    int64_t cols;
    int64_t ld;
    float scale_factor;
    int32_t scale_mode;
    void* y;
    int64_t ld_y;
    uint8_t* codes;
    float* scales0;
    uint8_t* scales1;
    uint8_t* mask;
} mxfp4_dual_level_args;

mxfp4_status mxfp4_dual_level_qdq(const mxfp4_dual_level_args* args, mxfp4_stream_t stream);

/* Static English text of a status; never NULL. */
const char* mxfp4_status_string(mxfp4_status status);

/* MXFP4_ABI_VERSION of the loaded library. */
int32_t mxfp4_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MXFP4_H */
