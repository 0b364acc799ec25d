/*
 * mxfp4_oracle.c -- plain scalar CPU oracle for MXFP4 block fake quantisation
 * (quantise-dequantise) and its straight-through-estimator backward.
 *
 * TEST INFRASTRUCTURE. Only the tests, the smoke check and the bench's CPU
 * baseline leg load this library. The product path (the CUDA library and its
 * Python binding) never links, imports or calls it, and this file shares no
 * code, header, table or helper with that path.
 *
 * Sources (web pages; cited by title and the function/section on the page):
 *   [QAT]  amct pull request 264, "feat: MXFP4 QAT fake-quant Linear (with
 *          STE)", file mxfp4_qat/fake_quant.py -- the numerical definition:
 *          constants, _block_view, _block_scale, _round_to_e2m1,
 *          _quant_dequant_torch, mxfp4_saturation_mask, _MXFP4FakeQuantSTE.
 *   [QATREADME] same pull request, mxfp4_qat/README_en.md, section
 *          "1. MXFP4 and STE" -- the scale formula and the plain/clipped STE.
 *   [GMM]  MindSpore hyper-parallel coverage page for fake_w4a8_gmm_func.py,
 *          FakeW4A8GroupedLinear.normalize_group_list / quantize_input --
 *          group_list types and row/column ("rowwise"/"colwise") quantisation.
 *   [NPU]  sglang mxfp4_npu.py, process_weights_after_loading comment:
 *          "float4_e2m1fn_x2 (2 FP4 packed/byte)"; NPUMXFP4DiffusionLinearMethod
 *          (npu_dynamic_dual_level_mx_quant: codes, level-0 and level-1 scales).
 *
 * Every floating-point step is done in fp32 because [QAT] casts the input to
 * float32 before any arithmetic (_block_view) and keeps all tensors in fp32.
 * The one step evaluated in double is round(log2(r)): [QAT] applies it to an
 * fp32 r, and the reading taken here is the exact mathematical value, which
 * double log2 resolves for every fp32 r (log2 r is never within 1e-8 of a
 * half-integer, far above double's error).
 *
 * Readings where the pages are silent:
 *   - scale_mode FLOOR: 2^(floor(log2 amax) - 2) saturated below at 2^-127
 *     (the E8M0 minimum), the rule of the OCP MX format; amax == 0 gives
 *     2^-127. Non-finite amax gives a non-finite scale as in PAGE mode.
 *   - Non-finite blocks: the page arithmetic makes every output NaN; the NaN
 *     written is the canonical positive quiet NaN, codes are 0, the E8M0
 *     byte is 0xFF (the E8M0 NaN encoding).
 *   - Packed layouts: element 2j in the low nibble, 2j+1 in the high nibble;
 *     nibble = sign<<3 | code index; saturation masks are bit-packed, bit b
 *     of byte j is element 8j+b of the row.
 *   - Column-wise blocks run down a column, restart at each group start and
 *     end early at a group end; scale rows are stored group after group.
 *
 * Parity status (what pins each function; the tests hold the pins):
 *   - scales, rounding, outputs, masks, STE: pinned by hand-worked blocks
 *     (tests/golden), closed forms, exhaustive bf16 sweeps, a brute-force
 *     nearest-code search and algebraic invariants;
 *   - packed layouts: the nibble values and the decode identity are pinned;
 *     the nibble order within a byte and the order of column-wise scale rows
 *     are conventions the pages do not fix: parity unpinned;
 *   - MXFP8 (oracle_qdq8_*, oracle_e4m3_*): the pages give no MXFP8
 *     arithmetic, so parity against them is unpinned; the functions are
 *     pinned against the E4M3 / OCP definitions (bit-field value set,
 *     nearest-even search over every bf16 value, torch's float8_e4m3fn cast);
 *   - dual-level MX quantisation (oracle_dual_level_rowwise): the page names
 *     the operator and its three results only, so parity against it is
 *     unpinned; the function is pinned against its stated reading: reduction
 *     to the single-level QDQ when the level-0 scale is a power of two, a
 *     brute-force restatement on small inputs, a hand-worked block
 *     (tests/golden) and the special blocks.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_F32 0
#define OR_BF16 1
#define OR_SCALE_PAGE 0
#define OR_SCALE_FLOOR 1

/* [QAT] module constants: codebook, its midpoints, saturation limit and the
 * smallest raw block scale. */
static const float E2M1_CODES[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};
static const float E2M1_MIDPOINTS[7] = {0.25f, 0.75f, 1.25f, 1.75f, 2.5f, 3.5f, 5.0f};
static const float MXFP4_E2M1_MAX = 6.0f;
static const float MIN_SCALE_RAW = 0x1p-30f;

/* ---- dtype casts ------------------------------------------------------- */

float oracle_bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16; /* bf16 is the top half of an fp32 */
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* fp32 -> bf16, round to nearest even; NaN becomes the canonical 0x7FC0. */
uint16_t oracle_f32_to_bf16(float f)
{
    uint32_t u;
    if (isnan(f))
        return 0x7FC0;
    memcpy(&u, &f, 4);
    uint32_t keep = u >> 16;
    uint32_t rest = u & 0xFFFF;
    if (rest > 0x8000 || (rest == 0x8000 && (keep & 1)))
        keep += 1;
    return (uint16_t)keep;
}

static float canonical_nan(void)
{
    uint32_t u = 0x7FC00000u;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

static float load_elem(const void* x, int dtype, int64_t i)
{
    if (dtype == OR_BF16)
        return oracle_bf16_to_f32(((const uint16_t*)x)[i]);
    return ((const float*)x)[i];
}

static void store_elem(void* y, int dtype, int64_t i, float v)
{
    if (dtype == OR_BF16) {
        ((uint16_t*)y)[i] = oracle_f32_to_bf16(v);
    } else {
        if (isnan(v))
            v = canonical_nan();
        ((float*)y)[i] = v;
    }
}

/* ---- [QAT] _block_scale -------------------------------------------------- */

/* |x|.amax over the block. Zero padding never raises it, so only the real
 * elements are visited; a NaN anywhere makes the result NaN (torch amax). */
static float block_amax(const float* v, int n)
{
    float m = 0.0f;
    for (int i = 0; i < n; ++i) {
        float a = fabsf(v[i]);
        if (isnan(a))
            return a;
        if (a > m)
            m = a;
    }
    return m;
}

/* PAGE mode: scale = exp2(round(log2(clamp(amax / scale_factor, min=2^-30)))). */
float oracle_scale_page(float amax, float scale_factor)
{
    float raw = amax / scale_factor; /* fp32 IEEE division */
    if (isnan(raw))
        return raw;                  /* clamp propagates NaN */
    if (raw < MIN_SCALE_RAW)
        raw = MIN_SCALE_RAW;
    double l = log2((double)raw);    /* +inf for raw == +inf */
    double k = nearbyint(l);         /* round half to even */
    return (float)exp2(k);           /* 2^k; +inf once k >= 128 */
}

/* FLOOR mode: scale = 2^(floor(log2 amax) - 2), saturated at 2^-127. */
float oracle_scale_floor(float amax)
{
    double e = floor(log2((double)amax)) - 2.0; /* -inf at 0, NaN at NaN */
    if (e < -127.0)
        e = -127.0;
    return (float)exp2(e);
}

static float block_scale(float amax, float scale_factor, int mode)
{
    return mode == OR_SCALE_FLOOR ? oracle_scale_floor(amax)
                                  : oracle_scale_page(amax, scale_factor);
}

/* E8M0 byte of a power-of-two scale: its exponent + 127; 0xFF when the scale
 * is not a finite number. */
static uint8_t e8m0_of(float scale)
{
    if (!isfinite(scale))
        return 0xFF;
    int e;
    frexp((double)scale, &e); /* scale = 0.5 * 2^e */
    return (uint8_t)(e - 1 + 127);
}

/* ---- [QAT] _round_to_e2m1 and _quant_dequant_torch ------------------------ */

/* bucketize(|y|, midpoints, right=True): the number of midpoints <= |y|. */
static int e2m1_index(float ay)
{
    int idx = 0;
    for (int j = 0; j < 7; ++j)
        if (E2M1_MIDPOINTS[j] <= ay)
            idx += 1;
    return idx;
}

/* torch.sign */
static float sign_of(float y)
{
    if (isnan(y))
        return y;
    if (y > 0.0f)
        return 1.0f;
    if (y < 0.0f)
        return -1.0f;
    return 0.0f;
}

/*
 * One block of n (<= block size) real elements v[0..n), already widened to
 * fp32. Writes, per element, the dequantised fp32 value, the E2M1 nibble and
 * the saturation flag, and returns the block's E8M0 byte through *e8m0.
 */
void oracle_qdq_block(const float* v, int n, float scale_factor, int mode,
                      float* out, uint8_t* nib, uint8_t* sat, uint8_t* e8m0)
{
    float scale = block_scale(block_amax(v, n), scale_factor, mode);
    float limit = MXFP4_E2M1_MAX * scale; /* mxfp4_saturation_mask */
    for (int i = 0; i < n; ++i) {
        float y = v[i] / scale;
        int idx = e2m1_index(fabsf(y));
        float q = sign_of(y) * E2M1_CODES[idx];
        float o = q * scale;
        out[i] = o;
        sat[i] = fabsf(v[i]) > limit ? 1 : 0;
        if (isnan(o))
            nib[i] = 0;
        else
            nib[i] = (uint8_t)((signbit(o) ? 8 : 0) | idx);
    }
    *e8m0 = e8m0_of(scale);
}

/* ---- packing helpers ------------------------------------------------------ */

static void put_nibble(uint8_t* row, int64_t c, uint8_t v)
{
    uint8_t* b = row + c / 2;
    if (c % 2 == 0)
        *b = (uint8_t)((*b & 0xF0) | (v & 0x0F));
    else
        *b = (uint8_t)((*b & 0x0F) | ((v & 0x0F) << 4));
}

static void put_bit(uint8_t* row, int64_t c, uint8_t v)
{
    uint8_t* b = row + c / 8;
    uint8_t m = (uint8_t)(1u << (c % 8));
    *b = v ? (uint8_t)(*b | m) : (uint8_t)(*b & ~m);
}

/* ---- [GMM] normalize_group_list ------------------------------------------ */

/*
 * group_list type 1 holds per-group counts and is turned into cumulative end
 * offsets by a running sum; type 0 already holds cumulative end offsets.
 * Returns 0 when the result is a valid partition of [0, rows) (non-decreasing
 * ends, first end >= 0, last end == rows), else -1.
 */
int oracle_group_ends(const int64_t* group_list, int64_t num_groups, int type,
                      int64_t rows, int64_t* ends)
{
    int64_t acc = 0, prev = 0;
    if (num_groups < 1 || (type != 0 && type != 1))
        return -1;
    for (int64_t g = 0; g < num_groups; ++g) {
        int64_t e;
        if (type == 1) {
            if (group_list[g] < 0)
                return -1;
            acc += group_list[g];
            e = acc;
        } else {
            e = group_list[g];
        }
        if (e < prev)
            return -1;
        ends[g] = e;
        prev = e;
    }
    return prev == rows ? 0 : -1;
}

/* Number of column-wise scale rows: sum over groups of ceil(n_g / block). */
int64_t oracle_colwise_scale_rows(const int64_t* ends, int64_t num_groups, int64_t block)
{
    int64_t s = 0, start = 0;
    for (int64_t g = 0; g < num_groups; ++g) {
        int64_t n = ends[g] - start;
        s += (n + block - 1) / block;
        start = ends[g];
    }
    return s;
}

/* ---- whole-tensor drivers ------------------------------------------------- */

/*
 * Row-wise QDQ of x[rows][cols] (leading dimension ld elements): blocks of
 * `block` consecutive elements of a row, the last one partial when cols is
 * not a multiple of block ([QAT] _block_view pads the last dim with zeros so
 * that rows never share a block).
 *   y      [rows][cols] in x's dtype, contiguous (or NULL)
 *   codes  [rows][ceil(cols/2)] nibble pairs (or NULL)
 *   scales [rows][ceil(cols/block)] E8M0 bytes (or NULL)
 *   mask   [rows][ceil(cols/8)] saturation bits (or NULL)
 */
int oracle_qdq_rowwise(const void* x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                       int block, float scale_factor, int mode,
                       void* y, uint8_t* codes, uint8_t* scales, uint8_t* mask)
{
    float* v = (float*)malloc(sizeof(float) * (size_t)block);
    float* o = (float*)malloc(sizeof(float) * (size_t)block);
    uint8_t* nb = (uint8_t*)malloc((size_t)block);
    uint8_t* st = (uint8_t*)malloc((size_t)block);
    if (!v || !o || !nb || !st) {
        free(v); free(o); free(nb); free(st);
        return -1;
    }
    int64_t nblk = (cols + block - 1) / block;
    int64_t cstride = (cols + 1) / 2, mstride = (cols + 7) / 8;
    if (codes)
        memset(codes, 0, (size_t)(rows * cstride));
    if (mask)
        memset(mask, 0, (size_t)(rows * mstride));
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < nblk; ++b) {
            int64_t c0 = b * block;
            int n = (int)((cols - c0) < block ? (cols - c0) : block);
            for (int i = 0; i < n; ++i)
                v[i] = load_elem(x, dtype, r * ld + c0 + i);
            uint8_t e8;
            oracle_qdq_block(v, n, scale_factor, mode, o, nb, st, &e8);
            for (int i = 0; i < n; ++i) {
                if (y)
                    store_elem(y, dtype, r * cols + c0 + i, o[i]);
                if (codes)
                    put_nibble(codes + r * cstride, c0 + i, nb[i]);
                if (mask)
                    put_bit(mask + r * mstride, c0 + i, st[i]);
            }
            if (scales)
                scales[r * nblk + b] = e8;
        }
    }
    free(v); free(o); free(nb); free(st);
    return 0;
}

/*
 * Column-wise QDQ: blocks of `block` consecutive rows of one column,
 * restarting at every group start (ends = cumulative end offsets, NULL for a
 * single group of all rows). Outputs keep x's orientation:
 *   y      [rows][cols] (or NULL)
 *   codes  [rows][ceil(cols/2)] (or NULL)
 *   scales [S][cols], S = sum_g ceil(n_g/block), group after group (or NULL)
 *   mask   [rows][ceil(cols/8)] (or NULL)
 */
int oracle_qdq_colwise(const void* x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                       int block, float scale_factor, int mode,
                       const int64_t* ends, int64_t num_groups,
                       void* y, uint8_t* codes, uint8_t* scales, uint8_t* mask)
{
    int64_t one_end = rows;
    if (!ends) {
        ends = &one_end;
        num_groups = 1;
    }
    float* v = (float*)malloc(sizeof(float) * (size_t)block);
    float* o = (float*)malloc(sizeof(float) * (size_t)block);
    uint8_t* nb = (uint8_t*)malloc((size_t)block);
    uint8_t* st = (uint8_t*)malloc((size_t)block);
    if (!v || !o || !nb || !st) {
        free(v); free(o); free(nb); free(st);
        return -1;
    }
    int64_t cstride = (cols + 1) / 2, mstride = (cols + 7) / 8;
    if (codes)
        memset(codes, 0, (size_t)(rows * cstride));
    if (mask)
        memset(mask, 0, (size_t)(rows * mstride));
    int64_t srow = 0, start = 0;
    for (int64_t g = 0; g < num_groups; ++g) {
        for (int64_t r0 = start; r0 < ends[g]; r0 += block, ++srow) {
            int n = (int)((ends[g] - r0) < block ? (ends[g] - r0) : block);
            for (int64_t c = 0; c < cols; ++c) {
                for (int i = 0; i < n; ++i)
                    v[i] = load_elem(x, dtype, (r0 + i) * ld + c);
                uint8_t e8;
                oracle_qdq_block(v, n, scale_factor, mode, o, nb, st, &e8);
                for (int i = 0; i < n; ++i) {
                    int64_t r = r0 + i;
                    if (y)
                        store_elem(y, dtype, r * cols + c, o[i]);
                    if (codes)
                        put_nibble(codes + r * cstride, c, nb[i]);
                    if (mask)
                        put_bit(mask + r * mstride, c, st[i]);
                }
                if (scales)
                    scales[srow * cols + c] = e8;
            }
        }
        start = ends[g];
    }
    free(v); free(o); free(nb); free(st);
    return 0;
}

/* ---- MXFP8: E4M3 elements with E8M0 block scales ------------------------- */
/*
 * [GMM] FakeW4A8GroupedLinear quantises activations and gradients to MXFP8
 * (E4M3 elements, one E8M0 scale per 32 elements) but the page only names the
 * NPU operators. Reading: the OCP Microscaling format rule, the same rule as
 * scale_mode FLOOR above with the element type's largest exponent:
 *   scale  = 2^(floor(log2 amax) - 8), saturated below at 2^-127
 *            (E4M3's largest normal is 1.75 * 2^8 = 448);
 *   code   = the E4M3 value nearest to x / scale, ties to the even code,
 *            magnitudes above 448 saturating to 448, the sign kept (so -0 and
 *            negative values that round to zero give the code 0x80);
 *   out    = decode(code) * scale, cast to the input dtype;
 *   sat    = |x| > 448 * scale.
 * Non-finite blocks follow the MXFP4 convention: NaN outputs, code 0, E8M0
 * 0xFF, no saturation.
 */

/* E4M3 (OCP "E4M3FN"): sign, 4 exponent bits (bias 7), 3 mantissa bits; no
 * infinities; S.1111.111 is NaN. Value of a code without its sign bit. */
double oracle_e4m3_value(uint8_t c)
{
    int e = (c >> 3) & 15, m = c & 7;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        return ldexp((double)m, -9);      /* subnormal: m * 2^-9 */
    return ldexp(1.0 + m / 8.0, e - 7);   /* normal: (1 + m/8) * 2^(e-7) */
}

/* Nearest E4M3 code to a finite y: search of the 127 finite magnitudes, ties
 * to the even code, saturation at 448, sign bit from y. */
uint8_t oracle_e4m3_encode(float y)
{
    double a = fabs((double)y);
    int best = 0;
    double bd = INFINITY;
    for (int c = 0; c <= 0x7E; ++c) {
        double d = fabs(a - oracle_e4m3_value((uint8_t)c));
        if (d < bd || (d == bd && (c & 1) == 0 && (best & 1) != 0)) {
            bd = d;
            best = c;
        }
    }
    if (a > 448.0)
        best = 0x7E;
    return (uint8_t)(best | (signbit(y) ? 0x80 : 0));
}

void oracle_qdq8_block(const float* v, int n, float* out, uint8_t* code, uint8_t* sat, uint8_t* e8m0)
{
    float amax = block_amax(v, n);
    double e = floor(log2((double)amax)) - 8.0; /* -inf at 0, NaN at NaN, +inf at inf */
    if (e < -127.0)
        e = -127.0;
    float scale = (float)exp2(e);
    float limit = 448.0f * scale;
    for (int i = 0; i < n; ++i) {
        if (!isfinite(scale)) {
            out[i] = canonical_nan();
            code[i] = 0;
            sat[i] = 0;
            continue;
        }
        float y = v[i] / scale; /* exact scaling by a power of two, rounded once */
        uint8_t c = oracle_e4m3_encode(y);
        double q = oracle_e4m3_value((uint8_t)(c & 0x7F));
        out[i] = (float)((c & 0x80 ? -q : q) * (double)scale); /* exact in fp32 */
        code[i] = c;
        sat[i] = fabsf(v[i]) > limit ? 1 : 0;
    }
    *e8m0 = e8m0_of(scale);
}

/* Row-wise MXFP8 QDQ, blocks of 32 along a row; codes [rows][cols] bytes,
 * the other outputs as in oracle_qdq_rowwise. */
int oracle_qdq8_rowwise(const void* x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                        void* y, uint8_t* codes, uint8_t* scales, uint8_t* mask)
{
    const int block = 32;
    float v[32], o[32];
    uint8_t cd[32], st[32];
    int64_t nblk = (cols + block - 1) / block, mstride = (cols + 7) / 8;
    if (mask)
        memset(mask, 0, (size_t)(rows * mstride));
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < nblk; ++b) {
            int64_t c0 = b * block;
            int n = (int)((cols - c0) < block ? (cols - c0) : block);
            for (int i = 0; i < n; ++i)
                v[i] = load_elem(x, dtype, r * ld + c0 + i);
            uint8_t e8;
            oracle_qdq8_block(v, n, o, cd, st, &e8);
            for (int i = 0; i < n; ++i) {
                if (y)
                    store_elem(y, dtype, r * cols + c0 + i, o[i]);
                if (codes)
                    codes[r * cols + c0 + i] = cd[i];
                if (mask)
                    put_bit(mask + r * mstride, c0 + i, st[i]);
            }
            if (scales)
                scales[r * nblk + b] = e8;
        }
    }
    return 0;
}

/* Column-wise MXFP8 QDQ, blocks of 32 rows restarting at group starts; codes
 * [rows][cols] bytes, the other outputs as in oracle_qdq_colwise. */
int oracle_qdq8_colwise(const void* x, int dtype, int64_t rows, int64_t cols, int64_t ld,
                        const int64_t* ends, int64_t num_groups,
                        void* y, uint8_t* codes, uint8_t* scales, uint8_t* mask)
{
    const int block = 32;
    float v[32], o[32];
    uint8_t cd[32], st[32];
    int64_t one_end = rows;
    if (!ends) {
        ends = &one_end;
        num_groups = 1;
    }
    int64_t mstride = (cols + 7) / 8;
    if (mask)
        memset(mask, 0, (size_t)(rows * mstride));
    int64_t srow = 0, start = 0;
    for (int64_t g = 0; g < num_groups; ++g) {
        for (int64_t r0 = start; r0 < ends[g]; r0 += block, ++srow) {
            int n = (int)((ends[g] - r0) < block ? (ends[g] - r0) : block);
            for (int64_t c = 0; c < cols; ++c) {
                for (int i = 0; i < n; ++i)
                    v[i] = load_elem(x, dtype, (r0 + i) * ld + c);
                uint8_t e8;
                oracle_qdq8_block(v, n, o, cd, st, &e8);
                for (int i = 0; i < n; ++i) {
                    int64_t r = r0 + i;
                    if (y)
                        store_elem(y, dtype, r * cols + c, o[i]);
                    if (codes)
                        codes[r * cols + c] = cd[i];
                    if (mask)
                        put_bit(mask + r * mstride, c, st[i]);
                }
                if (scales)
                    scales[srow * cols + c] = e8;
            }
        }
        start = ends[g];
    }
    return 0;
}

/*
 * [QAT] _MXFP4FakeQuantSTE.backward: plain STE returns grad_out unchanged;
 * clipped STE writes 0.0 where the saturation mask is set
 * (grad_output.masked_fill(saturated, 0.0)). grad arrays are [rows][cols]
 * contiguous in `dtype`; mask is the bit-packed [rows][ceil(cols/8)] layout.
 */
void oracle_ste_bwd(const void* grad_out, int dtype, int64_t rows, int64_t cols,
                    const uint8_t* mask, int clip_grad, void* grad_in)
{
    int64_t mstride = (cols + 7) / 8;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t c = 0; c < cols; ++c) {
            int64_t i = r * cols + c;
            int masked = clip_grad && ((mask[r * mstride + c / 8] >> (c % 8)) & 1);
            if (dtype == OR_BF16) {
                uint16_t g = ((const uint16_t*)grad_out)[i];
                ((uint16_t*)grad_in)[i] = masked ? (uint16_t)0 : g;
            } else {
                uint32_t g = ((const uint32_t*)grad_out)[i]; /* bits: NaN payloads pass */
                ((uint32_t*)grad_in)[i] = masked ? 0u : g;   /* 0u is +0.0f */
            }
        }
    }
}

/* ---- [NPU] dual-level MX quantisation -------------------------------------- */

/*
 * [NPU] NPUMXFP4DiffusionLinearMethod quantises weights and activations with
 * npu_dynamic_dual_level_mx_quant, which returns E2M1 codes, a level-0 scale
 * of shape [rows, cols / level0_block] and a level-1 scale; the page gives no
 * formula for either. Reading taken here (parity against the page unpinned):
 *   - the input is bf16 (the page's activation dtypes are bf16 and fp16, and
 *     weights of other dtypes are cast to bf16);
 *   - level 0: blocks of level0_block consecutive elements of a row (the
 *     last one partial); s0 = fl32(amax0 / 6), the fp32 level-0 scale, taken
 *     as 1 when that quotient is 0 (an all-zero block);
 *   - level 1: y = fl32(x / s0); y is quantised exactly as one row of the
 *     MXFP4 QDQ above (blocks of 32, the same scale rule, codes, E8M0 bytes
 *     and saturation |y| > 6 * 2^k1);
 *   - output fl32((code * 2^k1) * s0) (the first product is exact), cast to
 *     bf16;
 *   - a level-0 block holding a NaN or +-inf is non-finite: NaN outputs,
 *     codes 0, E8M0 bytes 0xFF, no saturation bits, s0 = NaN.
 * Layouts: y [rows][cols] (row stride cols), codes [rows][ceil(cols/2)],
 * scales0 [rows][ceil(cols/level0_block)] fp32, scales1 [rows][ceil(cols/32)],
 * mask [rows][ceil(cols/8)]; any output may be NULL. Returns -1 when
 * level0_block is not a positive multiple of 32 or memory runs out.
 */
int oracle_dual_level_rowwise(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld,
                              int level0_block, float scale_factor, int mode,
                              uint16_t* y, uint8_t* codes, float* scales0, uint8_t* scales1,
                              uint8_t* mask)
{
    if (level0_block <= 0 || level0_block % 32 != 0)
        return -1;
    float* v = (float*)malloc(sizeof(float) * (size_t)level0_block);
    if (!v)
        return -1;
    float w[32], o[32];
    uint8_t nb[32], st[32];
    int64_t nb0 = (cols + level0_block - 1) / level0_block, nb1 = (cols + 31) / 32;
    int64_t cstride = (cols + 1) / 2, mstride = (cols + 7) / 8;
    if (codes)
        memset(codes, 0, (size_t)(rows * cstride));
    if (mask)
        memset(mask, 0, (size_t)(rows * mstride));
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t j = 0; j < nb0; ++j) {
            int64_t c0 = j * level0_block;
            int n0 = (int)((cols - c0) < level0_block ? (cols - c0) : level0_block);
            for (int i = 0; i < n0; ++i)
                v[i] = oracle_bf16_to_f32(x[r * ld + c0 + i]);
            float a0 = block_amax(v, n0);
            int finite = isfinite(a0);
            float s0 = canonical_nan();
            if (finite) {
                s0 = a0 / MXFP4_E2M1_MAX; /* fp32 IEEE division */
                if (s0 == 0.0f)
                    s0 = 1.0f;
            }
            for (int b = 0; b * 32 < n0; ++b) {
                int n1 = n0 - 32 * b < 32 ? n0 - 32 * b : 32;
                int64_t cb = c0 + 32 * b;
                uint8_t e8 = 0xFF;
                if (finite) {
                    for (int i = 0; i < n1; ++i)
                        w[i] = v[32 * b + i] / s0;
                    oracle_qdq_block(w, n1, scale_factor, mode, o, nb, st, &e8);
                }
                for (int i = 0; i < n1; ++i) {
                    if (y)
                        y[r * cols + cb + i] = oracle_f32_to_bf16(finite ? o[i] * s0 : canonical_nan());
                    if (codes)
                        put_nibble(codes + r * cstride, cb + i, finite ? nb[i] : 0);
                    if (mask)
                        put_bit(mask + r * mstride, cb + i, finite ? st[i] : 0);
                }
                if (scales1)
                    scales1[r * nb1 + cb / 32] = e8;
            }
            if (scales0)
                scales0[r * nb0 + j] = s0;
        }
    }
    free(v);
    return 0;
}
