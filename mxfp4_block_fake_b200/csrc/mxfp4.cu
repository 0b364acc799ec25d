// mxfp4.cu -- sm_100a kernels and the C ABI of libmxfp4.so: MXFP4 block fake
// quantisation (quantise-dequantise) and its straight-through-estimator
// backward. The arithmetic follows amct pull request 264, "feat: MXFP4 QAT
// fake-quant Linear (with STE)", mxfp4_qat/fake_quant.py (_block_scale,
// _round_to_e2m1, _quant_dequant_torch, mxfp4_saturation_mask,
// _MXFP4FakeQuantSTE) and the grouped column-wise blocking of MindSpore's
// fake_w4a8_gmm_func.py (quantize_input, normalize_group_list).
//
// The work is a memory-bound block reduction plus an elementwise map, so no
// tensor cores are used. Design:
//  * tile kernel: a warp (block 32) or a CTA (block 128) owns a tile of
//    `block` rows x 64..128 columns held in registers as 16-byte vectors. The
//    row-wise block amax is a shuffle across the 4..32 lanes that share a
//    row block, the column-wise amax a register max over the thread's rows,
//    then a shuffle (and for block 128 a shared-memory step) across rows. One
//    read of x therefore serves both directions. Loads are 128-bit read-only
//    streaming loads, stores 128-bit streaming stores; grids are persistent
//    (SM count x resident CTAs).
//  * the block scale exponent comes from exponent/mantissa bits, with one fp32
//    divide per block in PAGE mode (round(log2 r) = e + (mantissa >= that of
//    sqrt 2), exact because no fp32 r lies on the rounding boundary);
//  * an element's code index is the count of codebook midpoints <= |x/2^k|
//    (a ladder of compares, ties up), the output sign(y)*code*2^k is formed
//    as one exact fp32 multiply and narrowed to bf16 by dropping zero bits.
//  * generic kernels (one thread per block, scalar accesses) serve shapes and
//    pointers the vector path cannot (cols or ld not a multiple of 16 bytes,
//    unaligned buffers).
#include <cuda.h>
#include <cuda_runtime.h>

#include <math.h>
#include <stdint.h>
#include <string.h>

#include <mutex>

#include "mxfp4.h"

namespace mxfp4 {

constexpr unsigned FULL = 0xFFFFFFFFu;
constexpr uint32_t QNAN32 = 0x7FC00000u;
constexpr int NTHREADS = 256;

struct KArgs {
    const void* x;
    int64_t rows, cols, ld;
    float sf;
    int32_t mode;
    int32_t grad_dir;  // 0, MXFP4_ROWWISE or MXFP4_COLWISE
    void* y_row;
    void* y_col;
    int64_t ld_y;
    uint8_t* codes_row;
    uint8_t* scales_row;
    uint8_t* mask_row;
    uint8_t* codes_col;
    uint8_t* scales_col;
    uint8_t* mask_col;
    const void* g_out;
    void* g_in;
    int64_t ld_g;
    const int64_t* group_list;
    int32_t num_groups;
    int32_t gl_type;
    int32_t* status;
    uint32_t n_ct;  // column tiles of the tile kernel
    uint32_t thr;   // PAGE mode: fp32 bits of T0 (see qparams)
    uint32_t ts_flags;  // staged kernel: column-wise outputs written by TMA stores (SG_TS_*)
    int32_t srow_mma;   // scales_row in the MMA scale-factor layout (MXFP4_SCALES_MMA)
    int32_t fmt;        // MXFP4_ELEM_E2M1 or MXFP4_ELEM_E4M3
    int64_t k_alloc;    // column-wise operand layout: K slots per codes row (MXFP4_COLS_MMA)
    // 4 and 65536, set by the host: the staged kernel scales table indices and
    // moves halves with integer multiply-adds by these run-time values, which
    // the compiler cannot turn back into shifts, so that this work runs on the
    // multiply-add pipe beside the logic ops on the ALU pipe
    uint32_t mul4, mul16;
};

// Byte offset of row-wise scale (row, b) of a [rows][nblk] scale matrix:
// row-major, or the block-scaled MMA layout (atoms of 128 rows x 4 block
// columns, 512 bytes, atom rows in order; entry (r, c) of an atom at
// 16 (r mod 32) + 4 floor(r / 32) + c).
__device__ __forceinline__ int64_t srow_off_mma(int64_t row, int64_t b, int64_t nblk)
{
    const int64_t ncb = (nblk + 3) >> 2;
    return (((row >> 7) * ncb + (b >> 2)) << 9) + ((row & 31) << 4) + (((row >> 5) & 3) << 2) + (b & 3);
}

__device__ __forceinline__ int64_t srow_off(const KArgs& a, int64_t row, int64_t b, int64_t nblk)
{
    return a.srow_mma ? srow_off_mma(row, b, nblk) : row * nblk + b;
}

// ---------------------------------------------------------------------------
// Per-block parameters
// ---------------------------------------------------------------------------

struct BP {
    float inv;      // 2^-k
    float scale;    // 2^k
    uint32_t lim;   // fp32 bits of fl(6 * 2^k); +inf bits once it overflows
    uint32_t nanm;  // all ones for a non-finite block
    uint32_t e8;    // E8M0 byte
};

// fp32 bits of 2^k for k in [-127, 127] (2^-127 is the subnormal 0x00400000).
__device__ __forceinline__ uint32_t pow2_bits(int k)
{
    return k >= -126 ? (uint32_t)(k + 127) << 23 : 0x00400000u;
}

// A = fp32 bits of the block's max |x| (integer max of sign-cleared bits, so a
// NaN anywhere gives A > 0x7F800000 and an inf gives A == 0x7F800000).
__device__ __forceinline__ BP block_params(uint32_t A, int mode, float sf)
{
    int k;
    bool special = A >= 0x7F800000u;
    if (mode == MXFP4_SCALE_FLOOR) {
        // floor(log2 amax) - 2 from the biased exponent; subnormal and zero
        // amax have a biased exponent of 0 and saturate at -127.
        k = max((int)(A >> 23) - 129, -127);
    } else {
        // r = max(fl(amax / sf), 2^-30) is a normal fp32 number; round(log2 r)
        // is its exponent plus one when its significand is at or above the
        // first fp32 significand above sqrt(2) (1.0110101000001001111001100..b;
        // fraction field 0x3504F3 < frac(sqrt 2) < 0x3504F4).
        float r = fmaxf(__fdiv_rn(__uint_as_float(A), sf), 0x1p-30f);
        uint32_t rb = __float_as_uint(r);
        k = (int)(rb >> 23) - 127 + ((rb & 0x7FFFFFu) >= 0x3504F4u ? 1 : 0);
        special = special || k > 127;  // 2^128 overflows fp32: scale = inf
    }
    if (special)
        k = 0;
    BP p;
    p.inv = __uint_as_float(pow2_bits(-k));
    p.scale = __uint_as_float(pow2_bits(k));
    p.lim = k >= 126 ? 0x7F800000u : (((uint32_t)(k + 129) << 23) | 0x00400000u);
    p.nanm = special ? 0xFFFFFFFFu : 0u;
    p.e8 = special ? 0xFFu : (uint32_t)(k + 127);
    return p;
}

// One element: returns the fp32 bits of sign(y) * code * 2^k with y = x * 2^-k
// (== fl(x / 2^k)), and the E2M1 nibble and saturation flag.
__device__ __forceinline__ uint32_t qdq_elem(uint32_t xb, const BP& p, uint32_t& nib, uint32_t& sat)
{
    const float y = __fmul_rn(__uint_as_float(xb), p.inv);
    const float a = fabsf(y);
    const uint32_t i = (uint32_t)(a >= 0.25f) + (uint32_t)(a >= 0.75f) + (uint32_t)(a >= 1.25f) +
                       (uint32_t)(a >= 1.75f) + (uint32_t)(a >= 2.5f) + (uint32_t)(a >= 3.5f) +
                       (uint32_t)(a >= 5.0f);
    // code magnitude as fp32 bits: 0, 0.5, then (i << 22) + 0x3F000000 gives
    // 1, 1.5, 2, 3, 4, 6 for i = 2..7 (two significant bits per binade)
    const uint32_t cb = i >= 2u ? (i << 22) + 0x3F000000u : (i == 1u ? 0x3F000000u : 0u);
    const uint32_t neg = y < 0.0f ? 0x80000000u : 0u;  // sign(-0) and sign(+0) are 0
    const float o = __fmul_rn(__uint_as_float(cb | neg), p.scale);
    nib = (neg >> 28) | i;
    sat = (xb & 0x7FFFFFFFu) > p.lim ? 1u : 0u;
    return __float_as_uint(o);
}

// ---------------------------------------------------------------------------
// MXFP8: E4M3 elements (scale mode FLOOR, block 32)
// ---------------------------------------------------------------------------

// k = floor(log2 amax) - 8 from the biased exponent (E4M3's largest normal is
// 1.75 * 2^8 = 448), saturated at -127 (subnormal and zero amax included).
__device__ __forceinline__ int k_e4m3(uint32_t A) { return max((int)(A >> 23) - 135, -127); }

__device__ __forceinline__ BP block_params8(uint32_t A)
{
    const bool special = A >= 0x7F800000u;
    const int k = special ? 0 : k_e4m3(A);
    BP p;
    p.inv = __uint_as_float(pow2_bits(-k));
    p.scale = __uint_as_float(pow2_bits(k));
    p.lim = ((uint32_t)(k + 135) << 23) | 0x00600000u;  // fp32 bits of 448 * 2^k = 1.75 * 2^(k + 8)
    p.nanm = special ? 0xFFFFFFFFu : 0u;
    p.e8 = special ? 0xFFu : (uint32_t)(k + 127);
    return p;
}

// One element: fp32 bits of decode(code) * 2^k (exact: codes have four
// significant bits and 2^k >= 2^-127), the E4M3 code of y = x * 2^-k by the
// hardware convert (nearest even, saturating at 448, sign kept) and the
// saturation flag.
__device__ __forceinline__ uint32_t qdq8_elem(uint32_t xb, const BP& p, uint32_t& code, uint32_t& sat)
{
    const float y = __fmul_rn(__uint_as_float(xb), p.inv);
    uint16_t q;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(q) : "f"(0.0f), "f"(y));
    uint32_t h;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(q));
    float c;
    asm("{\n\t.reg .b16 l, u;\n\tmov.b32 {l, u}, %1;\n\tcvt.f32.f16 %0, l;\n\t}" : "=f"(c) : "r"(h));
    code = q & 0xFFu;
    sat = (xb & 0x7FFFFFFFu) > p.lim ? 1u : 0u;
    return __float_as_uint(__fmul_rn(c, p.scale));
}

// fp32 bits -> the same bits rounded to bf16 (nearest even) in the top half;
// finite values only.
__device__ __forceinline__ uint32_t round_bf16_bits(uint32_t b)
{
    return (b + 0x7FFFu + ((b >> 16) & 1u)) & 0xFFFF0000u;
}

// ---------------------------------------------------------------------------
// 16-byte vectors
// ---------------------------------------------------------------------------

template <int VEC>
struct Vec;

template <>
struct Vec<8> {  // bf16 x 8
    static __device__ __forceinline__ void unpack(const uint4& v, uint32_t (&xb)[8])
    {
        xb[0] = v.x << 16; xb[1] = v.x & 0xFFFF0000u;
        xb[2] = v.y << 16; xb[3] = v.y & 0xFFFF0000u;
        xb[4] = v.z << 16; xb[5] = v.z & 0xFFFF0000u;
        xb[6] = v.w << 16; xb[7] = v.w & 0xFFFF0000u;
    }
    // The dequantised values have at most two significant bits and are >= 2^-128
    // in magnitude, so their bf16 narrowing is exact: keep the top halves.
    static __device__ __forceinline__ uint4 pack(const uint32_t (&ob)[8])
    {
        uint4 r;
        r.x = __byte_perm(ob[0], ob[1], 0x7632);
        r.y = __byte_perm(ob[2], ob[3], 0x7632);
        r.z = __byte_perm(ob[4], ob[5], 0x7632);
        r.w = __byte_perm(ob[6], ob[7], 0x7632);
        return r;
    }
    // zero the elements whose bit is set in m (8 bits)
    static __device__ __forceinline__ uint4 mask_out(const uint4& g, uint32_t m)
    {
        auto half = [](uint32_t w, uint32_t two) {
            uint32_t z = ((two & 1u) ? 0x0000FFFFu : 0u) | ((two & 2u) ? 0xFFFF0000u : 0u);
            return w & ~z;
        };
        uint4 r;
        r.x = half(g.x, m);
        r.y = half(g.y, m >> 2);
        r.z = half(g.z, m >> 4);
        r.w = half(g.w, m >> 6);
        return r;
    }
};

template <>
struct Vec<4> {  // fp32 x 4
    static __device__ __forceinline__ void unpack(const uint4& v, uint32_t (&xb)[4])
    {
        xb[0] = v.x; xb[1] = v.y; xb[2] = v.z; xb[3] = v.w;
    }
    static __device__ __forceinline__ uint4 pack(const uint32_t (&ob)[4])
    {
        return make_uint4(ob[0], ob[1], ob[2], ob[3]);
    }
    static __device__ __forceinline__ uint4 mask_out(const uint4& g, uint32_t m)
    {
        return make_uint4((m & 1u) ? 0u : g.x, (m & 2u) ? 0u : g.y, (m & 4u) ? 0u : g.z,
                          (m & 8u) ? 0u : g.w);
    }
};

__device__ __forceinline__ uint4 ld_stream(const void* p)
{
    uint4 r;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
        : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
        : "l"(p));
    return r;
}

__device__ __forceinline__ void st_stream(void* p, const uint4& v)
{
    __stcs(reinterpret_cast<uint4*>(p), v);
}

// ---------------------------------------------------------------------------
// group_list plan, built by every CTA in shared memory
// ---------------------------------------------------------------------------

// Writes s_rst[g] = sum_{j<g} n_j and s_bpre[g] = sum_{j<g} ceil(n_j / BS) for
// g = 0..G and returns S = s_bpre[G], or -1 when the list is not a partition
// of [0, rows): a negative count, a decreasing offset, or a wrong total.
// Every thread of the CTA must call it; the first NTHREADS hold the groups.
template <int BS>
__device__ int64_t build_plan(const KArgs& a, int32_t* s_bpre, int32_t* s_rst)
{
    __shared__ long long s_wr[NTHREADS / 32], s_wb[NTHREADS / 32];
    __shared__ int s_bad;
    const int G = a.num_groups;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int per = (G + NTHREADS - 1) / NTHREADS;
    const int g0 = min(G, tid * per), g1 = min(G, g0 + per);
    if (tid == 0)
        s_bad = 0;
    __syncthreads();

    long long lr = 0, lb = 0;
    bool bad = false;
    long long prev = (a.gl_type == 0 && g0 > 0) ? (long long)a.group_list[g0 - 1] : 0;
    for (int g = g0; g < g1; ++g) {
        long long v = a.group_list[g];
        long long n = a.gl_type == 1 ? v : v - prev;
        prev = v;
        if (n < 0 || n > a.rows) {
            bad = true;
            n = 0;
        }
        lr += n;
        lb += (n + BS - 1) / BS;
    }
    long long ir = lr, ib = lb;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        long long tr = __shfl_up_sync(FULL, ir, o);
        long long tb = __shfl_up_sync(FULL, ib, o);
        if (lane >= o) {
            ir += tr;
            ib += tb;
        }
    }
    if (lane == 31 && warp < NTHREADS / 32) {  // a CTA may carry extra warps: they hold no groups
        s_wr[warp] = ir;
        s_wb[warp] = ib;
    }
    if (bad)
        atomicOr(&s_bad, 1);
    __syncthreads();
    long long er = ir - lr, eb = ib - lb, tot_r = 0, tot_b = 0;
    for (int w = 0; w < NTHREADS / 32; ++w) {
        if (w < warp) {
            er += s_wr[w];
            eb += s_wb[w];
        }
        tot_r += s_wr[w];
        tot_b += s_wb[w];
    }
    prev = (a.gl_type == 0 && g0 > 0) ? (long long)a.group_list[g0 - 1] : 0;
    for (int g = g0; g < g1; ++g) {
        long long v = a.group_list[g];
        long long n = a.gl_type == 1 ? v : v - prev;
        prev = v;
        if (n < 0 || n > a.rows)
            n = 0;
        s_rst[g] = (int32_t)er;
        s_bpre[g] = (int32_t)eb;
        er += n;
        eb += (n + BS - 1) / BS;
    }
    if (tid == 0) {
        s_rst[G] = (int32_t)tot_r;
        s_bpre[G] = (int32_t)tot_b;
    }
    __syncthreads();
    const bool ok = !s_bad && tot_r == a.rows;
    return ok ? (int64_t)tot_b : -1;
}

// Row-block rb -> first row and row count, for a plan built by build_plan.
__device__ __forceinline__ void plan_lookup(const int32_t* s_bpre, const int32_t* s_rst, int G,
                                            uint32_t rb, int bs, int64_t& row0, int& nrows)
{
    int lo = 0, hi = G - 1;  // largest g with s_bpre[g] <= rb
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if ((uint32_t)s_bpre[mid] <= rb)
            lo = mid;
        else
            hi = mid - 1;
    }
    row0 = (int64_t)s_rst[lo] + (int64_t)(rb - (uint32_t)s_bpre[lo]) * bs;
    nrows = (int)min((int64_t)bs, (int64_t)s_rst[lo + 1] - row0);
}

// ---------------------------------------------------------------------------
// Tile kernel (vector path)
// ---------------------------------------------------------------------------

// Per-block parameters of the vector path: only 2^-k and 2^k are kept. A
// non-finite block (a NaN or inf element, or 2^k overflowing fp32) gets
// scale = NaN (0x7FC00000) and inv = 0, so that
//   E8M0 byte  = scale_bits >> 23   (0xFF for NaN; 0 for the subnormal 2^-127)
//   rare block = scale_bits >= 0x7E800000 (non-finite, or k >= 126 where
//                fl(6 * 2^k) overflows and nothing saturates)
struct QP {
    float inv;
    float scale;
};

// Scale exponent without a divide. PAGE mode: with T0 the smallest fp32 a for
// which fl(a / scale_factor) >= C (C = 0x3FB504F4, the first fp32 above
// sqrt 2), round(log2(fl(amax / sf))) >= j + 1 exactly when amax >= T0 * 2^j,
// because dividing by sf commutes with power-of-two scaling while the results
// stay normal. So k = floor(log2(amax / T0)) + 1, an exponent difference
// corrected by a significand compare, then clamped at -30 (the 2^-30 floor of
// the raw scale). The host computes T0 and limits scale_factor to
// [2^-64, 11] on this path so that every threshold used is a normal number.
__device__ __forceinline__ QP qparams(uint32_t A, int mode, uint32_t thr)
{
    int k;
    if (mode == MXFP4_SCALE_FLOOR) {
        k = max((int)(A >> 23) - 129, -127);
    } else {
        k = (int)(A >> 23) - (int)(thr >> 23) + 1 - ((A & 0x7FFFFFu) < (thr & 0x7FFFFFu) ? 1 : 0);
        k = max(k, -30);
    }
    QP p;
    if (A >= 0x7F800000u || k > 127) {
        p.inv = 0.0f;
        p.scale = __uint_as_float(QNAN32);
    } else {
        p.inv = __uint_as_float(pow2_bits(-k));
        p.scale = __uint_as_float(pow2_bits(k));
    }
    return p;
}

__device__ __forceinline__ uint32_t qp_e8(const QP& p) { return __float_as_uint(p.scale) >> 23; }
__device__ __forceinline__ bool qp_rare(const QP& p) { return __float_as_uint(p.scale) >= 0x7E800000u; }
__device__ __forceinline__ bool qp_nonfinite(const QP& p) { return __float_as_uint(p.scale) > 0x7F800000u; }

// E8M0 bytes of four blocks, first block in the low byte.
__device__ __forceinline__ uint32_t pack_e8(const QP& a, const QP& b, const QP& c, const QP& d)
{
    return qp_e8(a) | (qp_e8(b) << 8) | (qp_e8(c) << 16) | (qp_e8(d) << 24);
}

// Lookup entry for u = floor(4 |y|), u < 64: the code magnitude as fp32 bits
// (two significant bits, so the low half is zero). The code index is the
// number of midpoints m with 4m <= u, i.e. with m <= |y| since every 4m is an
// integer (ties go to the larger code).
__device__ __forceinline__ uint32_t lut_entry(uint32_t u)
{
    const uint32_t i = (u >= 1) + (u >= 3) + (u >= 5) + (u >= 7) + (u >= 10) + (u >= 14) + (u >= 20);
    return i >= 2u ? (i << 22) + 0x3F000000u : (i == 1u ? 0x3F000000u : 0u);
}

// One element. y = fl(x / 2^k); t = 2^23 + floor(4|y|) (one fma rounding
// down: the sum is exact below 2^24); the lookup address is
// lut_base + 4 * (t_bits - 0x4B000000) folded into one shift-add (lutb holds
// lut_base - 0x2C000000). |y| < 16 in every finite block on this path; the
// clamp (which also maps NaN to 15.75) keeps the table index inside [0, 63]
// for the non-finite blocks, whose outputs are then replaced. The sign follows
// sign(y): set only for y < 0, not for -0 (y & (0x80000000 - y) has bit 31
// set exactly then).
__device__ __forceinline__ void qfast(uint32_t xb, const QP& p, uint32_t lutb, float& cs, float& o, bool& sat)
{
    const float y = __fmul_rn(__uint_as_float(xb), p.inv);
    const float t = __fmaf_rd(fminf(fabsf(y), 15.75f), 4.0f, 8388608.0f);
    uint32_t e;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(e) : "r"(lutb + (__float_as_uint(t) << 2)));
    const uint32_t yb = __float_as_uint(y);
    const uint32_t s = yb & (0x80000000u - yb) & 0x80000000u;
    cs = __uint_as_float((e & 0xFFFF0000u) | s);
    o = __fmul_rn(cs, p.scale);
    sat = fabsf(y) > 6.0f;
}

// 8 signed code values (exact E2M1 values, so the conversion rounds nothing)
// -> 8 nibbles, element 2j in the low nibble of byte j.
__device__ __forceinline__ uint32_t e2m1x8(const float (&c)[8])
{
    uint32_t r;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(r)
        : "f"(c[0]), "f"(c[1]), "f"(c[2]), "f"(c[3]), "f"(c[4]), "f"(c[5]), "f"(c[6]), "f"(c[7]));
    return r;
}

__device__ __forceinline__ uint32_t e2m1x4(const float (&c)[4])
{
    uint32_t r;
    asm("{\n\t.reg .b8 b0, b1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "mov.b32 %0, {b0, b1, 0, 0};\n\t}"
        : "=r"(r)
        : "f"(c[0]), "f"(c[1]), "f"(c[2]), "f"(c[3]));
    return r;
}

template <int VEC>
__device__ __forceinline__ uint32_t nibbles(const float (&c)[VEC]);
template <>
__device__ __forceinline__ uint32_t nibbles<8>(const float (&c)[8]) { return e2m1x8(c); }
template <>
__device__ __forceinline__ uint32_t nibbles<4>(const float (&c)[4]) { return e2m1x4(c); }

// Quantise the VEC elements of one 16-byte chunk with one parameter set
// (row-wise: the chunk's block) or one per element (column-wise).
template <int VEC, bool PER_ELEM>
__device__ __forceinline__ void quant_chunk(const uint32_t (&xb)[VEC], const QP* p, uint32_t lutb,
                                            uint32_t (&ob)[VEC], uint32_t& nibs, uint32_t& sats)
{
    float cs[VEC];
    sats = 0;
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
        float o;
        bool sat;
        qfast(xb[e], p[PER_ELEM ? e : 0], lutb, cs[e], o, sat);
        ob[e] = __float_as_uint(o);
        sats |= (sat ? 1u : 0u) << e;
    }
    nibs = nibbles<VEC>(cs);
}

// Fix-up for rare blocks (non-finite, or k >= 126): every output NaN with code
// 0 and no saturation for a non-finite block; no saturation when 6 * 2^k
// overflows fp32.
template <int VEC>
__device__ __forceinline__ void rare_fixup(const QP& p, int e, uint32_t (&ob)[VEC], uint32_t& nibs, uint32_t& sats)
{
    if (qp_nonfinite(p)) {
        ob[e] = QNAN32;
        nibs &= ~(0xFu << (4 * e));
    }
    sats &= ~(1u << e);
}

// ---- bf16 fast path: two elements per 32-bit word ---------------------------

// Packed unsigned 16-bit max of two words.
__device__ __forceinline__ uint32_t vmax2(uint32_t a, uint32_t b)
{
    uint32_t r;
    asm("max.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// A block takes the bf16 fast path when 2^-126 <= 2^k <= 2^16. k <= 16 keeps
// every nonzero bf16 x clear of the fp32 underflow of x / 2^k (|x| >= 2^-133
// > 2^(k-150)), so sign(y) is the sign of x; k >= -126 keeps 2^k normal, so
// the bf16 bits of 6 * 2^k = 1.5 * 2^(k+2) are (scale_bits >> 16) + 0x140.
// Non-finite blocks (scale NaN) and every other k take the general path.
__device__ __forceinline__ bool qp_fast16(const QP& p)
{
    return (__float_as_uint(p.scale) - 0x00800000u) <= 0x47000000u;
}

__device__ __forceinline__ uint32_t qp_lim16(const QP& p) { return (__float_as_uint(p.scale) >> 16) + 0x140u; }

// Code of one bf16 element on the fast path, signed like x. xw holds the
// element in its top 16 bits; its low 16 bits may hold the other element of
// the word: that perturbs |x| by less than one bf16 ulp, and every quarter of
// 2^k that the rounding compares against is a bf16 number, so floor(4|y|) is
// unchanged. t = 2^21 + |x| * 2^-k rounded down once: fp32 spacing on
// [2^21, 2^22) is 1/4, so t's bit pattern is 0x4A000000 + floor(4|y|) and the
// table address is lut_base + 4 * that, folded into one shift-add (lutb16 =
// lut_base - 0x28000000). -0 inputs were cleared to +0 beforehand.
__device__ __forceinline__ float qcode16(uint32_t xw, float inv, uint32_t lutb16)
{
    const float t = __fmaf_rd(fabsf(__uint_as_float(xw)), inv, 0x1p21f);
    uint32_t e;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(e) : "r"(lutb16 + (__float_as_uint(t) << 2)));
    return __uint_as_float(e | (xw & 0x80000000u));
}

// Quantise 8 bf16 elements (4 cleaned words) on the fast path: packed bf16
// outputs and nibbles. One parameter set (row-wise) or one per element.
template <bool PER_ELEM>
__device__ __forceinline__ void quant16(const uint32_t (&wc)[4], const QP* p, uint32_t lutb16, uint32_t (&packed)[4],
                                        uint32_t& nibs)
{
    float cs[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const QP& pl = p[PER_ELEM ? 2 * j : 0];
        const QP& ph = p[PER_ELEM ? 2 * j + 1 : 0];
        cs[2 * j] = qcode16(wc[j] << 16, pl.inv, lutb16);
        cs[2 * j + 1] = qcode16(wc[j], ph.inv, lutb16);
        const float o0 = __fmul_rn(cs[2 * j], pl.scale);
        const float o1 = __fmul_rn(cs[2 * j + 1], ph.scale);
        packed[j] = __byte_perm(__float_as_uint(o0), __float_as_uint(o1), 0x7632);
    }
    nibs = e2m1x8(cs);
}

// Scale exponent k of a block from its amax bits, by the same rule as
// qparams but without building 2^k: non-finite amax yields k >= 125 here
// (scale_factor <= 11 on the vector path), which the fast-path range test
// below rejects.
__device__ __forceinline__ int block_k(uint32_t A, int mode, uint32_t thr)
{
    if (mode == MXFP4_SCALE_FLOOR)
        return max((int)(A >> 23) - 129, -127);
    const int k = (int)(A >> 23) - (int)(thr >> 23) + 1 - ((A & 0x7FFFFFu) < (thr & 0x7FFFFFu) ? 1 : 0);
    return max(k, -30);
}

// bf16 fast-path range: -126 <= k <= 16 (see qp_fast16).
__device__ __forceinline__ bool k_fast16(int k) { return (uint32_t)(k + 126) <= 142u; }

// 2^-k and 2^k for a fast-path k (both normal), as exponent-field arithmetic.
__device__ __forceinline__ QP qp_of_k(int k)
{
    QP p;
    p.inv = __uint_as_float(0x3F800000u - ((uint32_t)k << 23));
    p.scale = __uint_as_float(0x3F800000u + ((uint32_t)k << 23));
    return p;
}

// bf16 bits of 6 * 2^k = 1.5 * 2^(k+2) for a fast-path k.
__device__ __forceinline__ uint32_t lim16_of_k(int k) { return ((uint32_t)k << 7) + 0x40C0u; }

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel)
{
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

// Saturation bits of 8 elements from their abs bits (4 words) against packed
// limits: per half, 0x8000 + lim - a keeps bit 15 set exactly when a <= lim.
// A sign-replicating byte permute turns those bits into 0x00/0xFF bytes, a
// mask keeps a different bit per element, and one multiply ORs the four bytes.
__device__ __forceinline__ uint32_t sat8(const uint32_t (&aw)[4], const uint32_t (&limx)[4])
{
    const uint32_t m01 = prmt(limx[0] - aw[0], limx[1] - aw[1], 0xFDB9u);
    const uint32_t m23 = prmt(limx[2] - aw[2], limx[3] - aw[3], 0xFDB9u);
    const uint32_t keep = (m01 & 0x08040201u) | (m23 & 0x80402010u);
    return ~(keep * 0x01010101u) >> 24;
}

// |x| bits of a word and the word with -0 halves cleared to +0.
__device__ __forceinline__ void prep16(uint32_t w, uint32_t& aw, uint32_t& wc)
{
    aw = w & 0x7FFF7FFFu;
    wc = w & ((aw + 0x7FFF7FFFu) | 0x7FFF7FFFu);
}

// General path for the VEC elements of one chunk, out of line so that the
// fast path keeps its registers: exact block parameters (subnormal 2^k,
// non-finite blocks, any scale_factor within the vector-path range), the
// clamped lookup of qfast, and the rare-block fix-ups. ROWWISE: one block
// with amax bits A[0]; COLWISE: one block per element with amax bits A[e].
struct ChunkOut {
    uint4 packed;
    uint32_t nibs;
    uint32_t sats;
};

template <int VEC, bool PER_ELEM>
__device__ __noinline__ ChunkOut general_chunk(uint4 dv, const uint32_t* A, int mode, uint32_t thr, uint32_t lutb)
{
    QP p[PER_ELEM ? VEC : 1];
#pragma unroll
    for (int e = 0; e < (PER_ELEM ? VEC : 1); ++e)
        p[e] = qparams(A[e], mode, thr);
    uint32_t xb[VEC], ob[VEC];
    Vec<VEC>::unpack(dv, xb);
    ChunkOut r;
    quant_chunk<VEC, PER_ELEM>(xb, p, lutb, ob, r.nibs, r.sats);
#pragma unroll
    for (int e = 0; e < VEC; ++e)
        if (qp_rare(p[PER_ELEM ? e : 0]))
            rare_fixup<VEC>(p[PER_ELEM ? e : 0], e, ob, r.nibs, r.sats);
    r.packed = Vec<VEC>::pack(ob);
    return r;
}

// E8M0 byte of a block from its amax bits and k: 0xFF for a non-finite block
// (a NaN or inf element, or 2^k beyond fp32), else k + 127.
__device__ __forceinline__ uint32_t e8_of(uint32_t A, int k)
{
    return (A >= 0x7F800000u || k > 127) ? 0xFFu : (uint32_t)(k + 127);
}

// ESZ: 2 (bf16) or 4 (fp32) bytes. LC lanes across columns (16 bytes each),
// LR = 32/LC lanes across rows, RPT rows per thread, WR warps down the tile.
// A tile is BS rows (one column-wise block; a group tail may be shorter) by
// LC*VEC columns.
template <int ESZ, int BS, int LC, int RPT, int WR, bool ROW, bool COL, bool GROUPS, bool GRAD>
__global__ void __launch_bounds__(NTHREADS, COL ? 2 : 1) qdq_tile_kernel(const KArgs a)
{
    constexpr int VEC = 16 / ESZ;
    constexpr int LR = 32 / LC;
    constexpr int TC = LC * VEC;
    constexpr int NWG = (NTHREADS / 32) / WR;
    constexpr int BL = BS / VEC;  // lanes sharing one row-wise block
    static_assert(LR * RPT * WR == BS, "tile rows must equal the block");
    static_assert(!ROW || (LC % BL == 0), "a row-wise block must sit in one warp row");
    static_assert(WR == 1 || WR == NTHREADS / 32, "a multi-warp tile takes the whole CTA");
    using V = Vec<VEC>;

    extern __shared__ int32_t s_plan[];
    __shared__ uint32_t s_am[(COL && WR > 1) ? WR * TC : 1];
    __shared__ uint32_t s_lut[64];

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int wg = warp / WR, wr = warp - wg * WR;
    const int lc = lane % LC, lr = lane / LC;

    if (threadIdx.x < 64)
        s_lut[threadIdx.x] = lut_entry(threadIdx.x);
    uint32_t S;
    int32_t* s_bpre = s_plan;
    int32_t* s_rst = s_plan + (GROUPS ? a.num_groups + 1 : 0);
    if constexpr (GROUPS) {
        const int64_t s = build_plan<BS>(a, s_bpre, s_rst);  // contains __syncthreads
        if (blockIdx.x == 0 && threadIdx.x == 0 && a.status)
            *a.status = s < 0 ? MXFP4_EINVAL : MXFP4_OK;
        if (s < 0)
            return;
        S = (uint32_t)s;
    } else {
        __syncthreads();
        S = (uint32_t)((a.rows + BS - 1) / BS);
    }
    const uint32_t lutb = (uint32_t)__cvta_generic_to_shared(s_lut) - 0x2C000000u;
    const uint32_t lutb16 = lutb + 0x04000000u;  // lut_base - 0x28000000

    const char* xp = static_cast<const char*>(a.x);
    const int64_t cstride = a.cols / 2, mstride = (a.cols + 7) / 8, nblk = (a.cols + BS - 1) / BS;
    const uint32_t ntiles = S * a.n_ct;
    const uint32_t tstride = gridDim.x * NWG;

    for (uint32_t t = blockIdx.x * NWG + wg; t < ntiles; t += tstride) {
        const uint32_t rb = t / a.n_ct, ct = t - rb * a.n_ct;
        int64_t row0;
        int nrows;
        if constexpr (GROUPS) {
            plan_lookup(s_bpre, s_rst, a.num_groups, rb, BS, row0, nrows);
        } else {
            row0 = (int64_t)rb * BS;
            nrows = (int)min((int64_t)BS, a.rows - row0);
        }
        const int64_t col = (int64_t)ct * TC + lc * VEC;
        const bool colok = col < a.cols;

        uint4 d[RPT];
        uint4 gv[GRAD ? RPT : 1];
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
            const int r = i * (LR * WR) + wr * LR + lr;
            d[i] = make_uint4(0u, 0u, 0u, 0u);
            if (colok && r < nrows)
                d[i] = ld_stream(xp + ((row0 + r) * a.ld + col) * ESZ);
            if constexpr (GRAD) {
                gv[i] = make_uint4(0u, 0u, 0u, 0u);
                if (colok && r < nrows)
                    gv[i] = ld_stream(static_cast<const char*>(a.g_out) + ((row0 + r) * a.ld_g + col) * ESZ);
            }
        }

        // Column-wise block parameters first: a max down the thread's rows, a
        // shuffle across the LR row lanes, shared memory across warps.
        constexpr int NW = (VEC == 8) ? 4 : VEC;  // words (bf16 pairs) or elements (fp32)
        uint32_t mc[COL ? NW : 1];
        QP pc[COL ? VEC : 1];                      // fast-path 2^-k, 2^k per column
        uint32_t limxc[(COL && VEC == 8) ? 4 : 1];
        bool cgen = false;                         // some column block needs the general path
        bool csat = false;                         // some column block may saturate
        if constexpr (COL) {
#pragma unroll
            for (int j = 0; j < NW; ++j)
                mc[j] = 0;
#pragma unroll
            for (int i = 0; i < RPT; ++i) {
                const uint32_t w[4] = {d[i].x, d[i].y, d[i].z, d[i].w};
#pragma unroll
                for (int j = 0; j < NW; ++j) {
                    if constexpr (VEC == 8)
                        mc[j] = vmax2(mc[j], w[j] & 0x7FFF7FFFu);
                    else
                        mc[j] = max(mc[j], w[j] & 0x7FFFFFFFu);
                }
            }
#pragma unroll
            for (int o = LC; o < 32; o <<= 1) {
#pragma unroll
                for (int j = 0; j < NW; ++j) {
                    const uint32_t v = __shfl_xor_sync(FULL, mc[j], o);
                    if constexpr (VEC == 8)
                        mc[j] = vmax2(mc[j], v);
                    else
                        mc[j] = max(mc[j], v);
                }
            }
            if constexpr (WR > 1) {
                if (lr == 0) {
#pragma unroll
                    for (int j = 0; j < NW; ++j)
                        s_am[wr * TC + lc * VEC + j] = mc[j];
                }
                __syncthreads();
#pragma unroll
                for (int j = 0; j < NW; ++j) {
                    uint32_t m = 0;
#pragma unroll
                    for (int w = 0; w < WR; ++w) {
                        const uint32_t v = s_am[w * TC + lc * VEC + j];
                        if constexpr (VEC == 8)
                            m = vmax2(m, v);
                        else
                            m = max(m, v);
                    }
                    mc[j] = m;
                }
                __syncthreads();  // s_am is rewritten by the next tile
            }
            uint32_t e8[VEC];
#pragma unroll
            for (int e = 0; e < VEC; ++e) {
                uint32_t A;
                if constexpr (VEC == 8)
                    A = (e & 1) ? (mc[e / 2] & 0xFFFF0000u) : (mc[e / 2] << 16);
                else
                    A = mc[e];
                const int k = block_k(A, a.mode, a.thr);
                e8[e] = e8_of(A, k);
                if constexpr (VEC == 8) {
                    cgen = cgen || !k_fast16(k);
                    pc[e] = qp_of_k(k);
                    const uint32_t lim = lim16_of_k(k);
                    if (e & 1)
                        limxc[e / 2] |= (0x8000u + lim) << 16;
                    else
                        limxc[e / 2] = 0x8000u + lim;
                }
            }
            if constexpr (VEC == 8) {
#pragma unroll
                for (int j = 0; j < 4; ++j)  // both halves of limx - amax keep bit 15 when nothing saturates
                    csat = csat || (((limxc[j] - mc[j]) & 0x80008000u) != 0x80008000u);
            } else {
                cgen = true;
            }
            if (a.scales_col && lr == 0 && wr == 0 && colok) {
                uint8_t* sp = a.scales_col + (int64_t)rb * a.cols + col;
                const uint32_t lo = e8[0] | (e8[1] << 8) | (e8[2] << 16) | (e8[3] << 24);
                if constexpr (VEC == 8)
                    *reinterpret_cast<uint2*>(sp) =
                        make_uint2(lo, e8[4 % VEC] | (e8[5 % VEC] << 8) | (e8[6 % VEC] << 16) | (e8[7 % VEC] << 24));
                else
                    *reinterpret_cast<uint32_t*>(sp) = lo;
            }
        }

        // Then one pass over the rows: both directions of row i, and the
        // gradient of row i, before moving on.
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
            const int r = i * (LR * WR) + wr * LR + lr;
            const bool ok = colok && r < nrows;
            const int64_t row = row0 + r;
            const uint32_t w[4] = {d[i].x, d[i].y, d[i].z, d[i].w};
            uint32_t aw[4], wc[4];
            if constexpr (VEC == 8) {
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    prep16(w[j], aw[j], wc[j]);
            }
            uint32_t gmask = 0;
            if constexpr (ROW) {
                uint32_t am;
                if constexpr (VEC == 8) {
                    const uint32_t m2 = vmax2(vmax2(aw[0], aw[1]), vmax2(aw[2], aw[3]));
                    am = max(m2 & 0xFFFFu, m2 >> 16);
                } else {
                    am = max(max(w[0] & 0x7FFFFFFFu, w[1] & 0x7FFFFFFFu), max(w[2] & 0x7FFFFFFFu, w[3] & 0x7FFFFFFFu));
                }
#pragma unroll
                for (int o = 1; o < BL; o <<= 1)
                    am = max(am, __shfl_xor_sync(FULL, am, o));
                const uint32_t A = VEC == 8 ? am << 16 : am;
                const int k = block_k(A, a.mode, a.thr);
                uint32_t packed[4], nibs, sats;
                if (VEC == 8 && k_fast16(k)) {
                    const QP p = qp_of_k(k);
                    quant16<false>(wc, &p, lutb16, packed, nibs);
                    const uint32_t lim = lim16_of_k(k);
                    sats = 0;
                    if (am > lim) {
                        const uint32_t lx = (0x8000u + lim) * 0x10001u;
                        const uint32_t limx[4] = {lx, lx, lx, lx};
                        sats = sat8(aw, limx);
                    }
                } else {
                    const ChunkOut g = general_chunk<VEC, false>(d[i], &A, a.mode, a.thr, lutb);
                    packed[0] = g.packed.x;
                    packed[1] = g.packed.y;
                    packed[2] = g.packed.z;
                    packed[3] = g.packed.w;
                    nibs = g.nibs;
                    sats = g.sats;
                }
                if (a.grad_dir == MXFP4_ROWWISE)
                    gmask = sats;
                if constexpr (VEC == 4) {  // two lanes form one mask byte
                    const uint32_t other = __shfl_xor_sync(FULL, sats, 1);
                    sats = (lc & 1) ? 0u : (sats | (other << 4));
                }
                if (ok) {
                    if (a.y_row)
                        st_stream(static_cast<char*>(a.y_row) + (row * a.ld_y + col) * ESZ,
                                  make_uint4(packed[0], packed[1], packed[2], packed[3]));
                    if (a.codes_row) {
                        if constexpr (VEC == 8)
                            *reinterpret_cast<uint32_t*>(a.codes_row + row * cstride + col / 2) = nibs;
                        else
                            *reinterpret_cast<uint16_t*>(a.codes_row + row * cstride + col / 2) = (uint16_t)nibs;
                    }
                    if (a.mask_row && (VEC == 8 || !(lc & 1)))
                        a.mask_row[row * mstride + col / 8] = (uint8_t)sats;
                    if (a.scales_row && (lc % BL) == 0)
                        a.scales_row[srow_off(a, row, col / BS, nblk)] = (uint8_t)e8_of(A, k);
                }
            }
            if constexpr (COL) {
                uint32_t packed[4], nibs, sats;
                if (!cgen) {
                    if constexpr (VEC == 8) {
                        quant16<true>(wc, pc, lutb16, packed, nibs);
                        sats = csat ? sat8(aw, limxc) : 0u;
                    }
                } else {
                    uint32_t Ac[VEC];
#pragma unroll
                    for (int e = 0; e < VEC; ++e) {
                        if constexpr (VEC == 8)
                            Ac[e] = (e & 1) ? (mc[e / 2] & 0xFFFF0000u) : (mc[e / 2] << 16);
                        else
                            Ac[e] = mc[e];
                    }
                    const ChunkOut g = general_chunk<VEC, true>(d[i], Ac, a.mode, a.thr, lutb);
                    packed[0] = g.packed.x;
                    packed[1] = g.packed.y;
                    packed[2] = g.packed.z;
                    packed[3] = g.packed.w;
                    nibs = g.nibs;
                    sats = g.sats;
                }
                if (a.grad_dir == MXFP4_COLWISE)
                    gmask = sats;
                if constexpr (VEC == 4) {
                    const uint32_t other = __shfl_xor_sync(FULL, sats, 1);
                    sats = (lc & 1) ? 0u : (sats | (other << 4));
                }
                if (ok) {
                    if (a.y_col)
                        st_stream(static_cast<char*>(a.y_col) + (row * a.ld_y + col) * ESZ,
                                  make_uint4(packed[0], packed[1], packed[2], packed[3]));
                    if (a.codes_col) {
                        if constexpr (VEC == 8)
                            *reinterpret_cast<uint32_t*>(a.codes_col + row * cstride + col / 2) = nibs;
                        else
                            *reinterpret_cast<uint16_t*>(a.codes_col + row * cstride + col / 2) = (uint16_t)nibs;
                    }
                    if (a.mask_col && (VEC == 8 || !(lc & 1)))
                        a.mask_col[row * mstride + col / 8] = (uint8_t)sats;
                }
            }
            if constexpr (GRAD) {
                if (ok)
                    st_stream(static_cast<char*>(a.g_in) + (row * a.ld_g + col) * ESZ, V::mask_out(gv[i], gmask));
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Generic kernels (scalar path for any alignment / leading dimension)
// ---------------------------------------------------------------------------

template <int ESZ>
__device__ __forceinline__ uint32_t load_bits(const void* base, int64_t i)
{
    if (ESZ == 2)
        return (uint32_t)static_cast<const uint16_t*>(base)[i] << 16;
    return static_cast<const uint32_t*>(base)[i];
}

template <int ESZ>
__device__ __forceinline__ void store_bits(void* base, int64_t i, uint32_t v)
{
    if (ESZ == 2)
        static_cast<uint16_t*>(base)[i] = (uint16_t)(v >> 16);
    else
        static_cast<uint32_t*>(base)[i] = v;
}

// One thread per (row, row-wise block). FMT: MXFP4_ELEM_E2M1 or _E4M3.
template <int ESZ, int BS, bool GRAD, int FMT>
__global__ void __launch_bounds__(NTHREADS) generic_row_kernel(const KArgs a)
{
    const int64_t nblk = (a.cols + BS - 1) / BS;
    const int64_t total = a.rows * nblk;
    const int64_t cstride = (a.cols + 1) / 2, mstride = (a.cols + 7) / 8;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t row = idx / nblk, b = idx - row * nblk;
        const int64_t c0 = b * BS;
        const int n = (int)min((int64_t)BS, a.cols - c0);
        const int64_t xo = row * a.ld + c0;
        uint32_t am = 0;
        for (int j = 0; j < n; ++j)
            am = max(am, load_bits<ESZ>(a.x, xo + j) & 0x7FFFFFFFu);
        const BP p = FMT == MXFP4_ELEM_E4M3 ? block_params8(am) : block_params(am, a.mode, a.sf);
        uint32_t nacc = 0, sacc = 0;
        for (int j = 0; j < n; ++j) {
            uint32_t nb, st;
            uint32_t ob = FMT == MXFP4_ELEM_E4M3 ? qdq8_elem(load_bits<ESZ>(a.x, xo + j), p, nb, st)
                                                : qdq_elem(load_bits<ESZ>(a.x, xo + j), p, nb, st);
            if (FMT == MXFP4_ELEM_E4M3 && ESZ == 2)
                ob = round_bf16_bits(ob);
            if (p.nanm) {
                ob = QNAN32;
                nb = 0;
                st = 0;
            }
            if (a.y_row)
                store_bits<ESZ>(a.y_row, row * a.ld_y + c0 + j, ob);
            if (FMT == MXFP4_ELEM_E4M3 && a.codes_row)
                a.codes_row[row * a.cols + c0 + j] = (uint8_t)nb;
            nacc |= nb << (4 * (j & 1));
            sacc |= st << (j & 7);
            if (FMT == MXFP4_ELEM_E2M1 && a.codes_row && ((j & 1) || j == n - 1))
                a.codes_row[row * cstride + (c0 + j) / 2] = (uint8_t)nacc;
            if ((j & 1) || j == n - 1)
                nacc = 0;
            if (a.mask_row && ((j & 7) == 7 || j == n - 1))
                a.mask_row[row * mstride + (c0 + j) / 8] = (uint8_t)sacc;
            if ((j & 7) == 7 || j == n - 1)
                sacc = 0;
            if (GRAD && a.grad_dir == MXFP4_ROWWISE) {
                const int64_t gi = row * a.ld_g + c0 + j;
                store_bits<ESZ>(a.g_in, gi, st ? 0u : load_bits<ESZ>(a.g_out, gi));
            }
        }
        if (a.scales_row)
            a.scales_row[srow_off(a, row, b, nblk)] = (uint8_t)p.e8;
    }
}

// One thread per (column-wise block, 8 adjacent columns): whole code and mask
// bytes are owned by one thread.
template <int ESZ, int BS, bool GROUPS, bool GRAD, int FMT>
__global__ void __launch_bounds__(NTHREADS) generic_col_kernel(const KArgs a)
{
    extern __shared__ int32_t s_plan[];
    int32_t* s_bpre = s_plan;
    int32_t* s_rst = s_plan + (GROUPS ? a.num_groups + 1 : 0);
    int64_t S;
    if (GROUPS) {
        S = build_plan<BS>(a, s_bpre, s_rst);
        if (blockIdx.x == 0 && threadIdx.x == 0 && a.status)
            *a.status = S < 0 ? MXFP4_EINVAL : MXFP4_OK;
        if (S < 0)
            return;
    } else {
        S = (a.rows + BS - 1) / BS;
    }
    const int64_t noct = (a.cols + 7) / 8;
    const int64_t total = S * noct;
    const int64_t cstride = (a.cols + 1) / 2, mstride = (a.cols + 7) / 8;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t rb = idx / noct, oc = idx - rb * noct;
        int64_t row0;
        int nrows;
        if (GROUPS) {
            plan_lookup(s_bpre, s_rst, a.num_groups, (uint32_t)rb, BS, row0, nrows);
        } else {
            row0 = rb * BS;
            nrows = (int)min((int64_t)BS, a.rows - row0);
        }
        const int64_t c0 = oc * 8;
        const int nc = (int)min((int64_t)8, a.cols - c0);
        uint32_t am[8];
#pragma unroll
        for (int c = 0; c < 8; ++c)
            am[c] = 0;
        for (int r = 0; r < nrows; ++r) {
#pragma unroll
            for (int c = 0; c < 8; ++c)
                if (c < nc)
                    am[c] = max(am[c], load_bits<ESZ>(a.x, (row0 + r) * a.ld + c0 + c) & 0x7FFFFFFFu);
        }
        BP p[8];
#pragma unroll
        for (int c = 0; c < 8; ++c)
            p[c] = FMT == MXFP4_ELEM_E4M3 ? block_params8(am[c]) : block_params(am[c], a.mode, a.sf);
        for (int r = 0; r < nrows; ++r) {
            const int64_t row = row0 + r;
            uint32_t nibs = 0, sats = 0;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                if (c >= nc)
                    continue;
                uint32_t nb, st;
                uint32_t ob = FMT == MXFP4_ELEM_E4M3 ? qdq8_elem(load_bits<ESZ>(a.x, row * a.ld + c0 + c), p[c], nb, st)
                                                    : qdq_elem(load_bits<ESZ>(a.x, row * a.ld + c0 + c), p[c], nb, st);
                if (FMT == MXFP4_ELEM_E4M3 && ESZ == 2)
                    ob = round_bf16_bits(ob);
                if (p[c].nanm) {
                    ob = QNAN32;
                    nb = 0;
                    st = 0;
                }
                if (a.y_col)
                    store_bits<ESZ>(a.y_col, row * a.ld_y + c0 + c, ob);
                if (FMT == MXFP4_ELEM_E4M3 && a.codes_col)
                    a.codes_col[row * a.cols + c0 + c] = (uint8_t)nb;
                nibs |= nb << (4 * c);
                sats |= st << c;
                if (GRAD && a.grad_dir == MXFP4_COLWISE) {
                    const int64_t gi = row * a.ld_g + c0 + c;
                    store_bits<ESZ>(a.g_in, gi, st ? 0u : load_bits<ESZ>(a.g_out, gi));
                }
            }
            if (FMT == MXFP4_ELEM_E2M1 && a.codes_col) {
                for (int j = 0; j < (nc + 1) / 2; ++j)
                    a.codes_col[row * cstride + c0 / 2 + j] = (uint8_t)(nibs >> (8 * j));
            }
            if (a.mask_col)
                a.mask_col[row * mstride + oc] = (uint8_t)sats;
        }
        if (a.scales_col) {
#pragma unroll
            for (int c = 0; c < 8; ++c)
                if (c < nc)
                    a.scales_col[rb * a.cols + c0 + c] = (uint8_t)p[c].e8;
        }
    }
}

// grad_in = grad_out with +0 where the saved bit is set (mask may be NULL for
// the plain STE copy). One thread per (row, 8 columns).
template <int ESZ>
__global__ void __launch_bounds__(NTHREADS)
    ste_mask_kernel(int64_t rows, int64_t cols, const void* g_out, void* g_in, int64_t ld_g,
                    const uint8_t* mask, int vec)
{
    const int64_t noct = (cols + 7) / 8, mstride = noct;
    const int64_t total = rows * noct;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t row = idx / noct, oc = idx - row * noct;
        const uint32_t m = mask ? (uint32_t)mask[row * mstride + oc] : 0u;
        const int64_t base = row * ld_g + oc * 8;
        if (vec) {
            const char* src = static_cast<const char*>(g_out) + base * ESZ;
            char* dst = static_cast<char*>(g_in) + base * ESZ;
            if (ESZ == 2) {
                st_stream(dst, Vec<8>::mask_out(ld_stream(src), m));
            } else {
                st_stream(dst, Vec<4>::mask_out(ld_stream(src), m));
                st_stream(dst + 16, Vec<4>::mask_out(ld_stream(src + 16), m >> 4));
            }
        } else {
            const int nc = (int)min((int64_t)8, cols - oc * 8);
            for (int c = 0; c < nc; ++c)
                store_bits<ESZ>(g_in, base + c, ((m >> c) & 1u) ? 0u : load_bits<ESZ>(g_out, base + c));
        }
    }
}

}  // namespace mxfp4

#include "mxfp4_staged.cuh"
#include "mxfp4_staged8.cuh"
#include "mxfp4_operand.cuh"
#include "mxfp4_gemm.cuh"

namespace mxfp4 {

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

struct DevInfo {
    int sms = 0;
};

static std::mutex g_mu;

static int device_sms()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return -1;
    static DevInfo info[64];
    std::lock_guard<std::mutex> lk(g_mu);
    if (dev < 0 || dev >= 64)
        return -1;
    if (info[dev].sms == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return -1;
        info[dev].sms = n;
    }
    return info[dev].sms;
}

// Resident CTAs per SM of `fn` launched with `threads` per CTA, cached per
// (device, kernel).
static int occupancy(const void* fn, size_t smem, int threads = NTHREADS)
{
    struct Entry {
        const void* fn;
        int dev;
        size_t smem;
        int occ;
    };
    static Entry cache[512];
    static int n = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return -1;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        for (int i = 0; i < n; ++i)
            if (cache[i].fn == fn && cache[i].dev == dev && cache[i].smem == smem)
                return cache[i].occ;
    }
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, fn, threads, smem) != cudaSuccess)
        return -1;
    if (occ < 1)
        occ = 1;
    std::lock_guard<std::mutex> lk(g_mu);
    if (n < 512)
        cache[n++] = Entry{fn, dev, smem, occ};
    return occ;
}

static inline bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

static float f32_of(uint32_t u)
{
    float f;
    memcpy(&f, &u, 4);
    return f;
}

static uint32_t u32_of(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    return u;
}

// PAGE-mode scale_factor range of the vector path: every threshold T0 * 2^j it
// uses stays a normal fp32 number, and |x / 2^k| < 16 keeps floor(4|y|) inside
// the 64-entry lookup table.
static bool page_fast_ok(float sf) { return sf >= 0x1p-64f && sf <= 11.0f; }

// T0 = the smallest fp32 a with fl(a / sf) >= C, C = 0x3FB504F4 (the first fp32
// above sqrt 2), found by stepping from fl(C * sf) one ulp at a time with IEEE
// fp32 host division (a -> fl(a / sf) is monotone).
static uint32_t page_threshold(float sf)
{
    const float C = f32_of(0x3FB504F4u);
    volatile float a = C * sf;
    for (int i = 0; i < 64; ++i) {
        volatile float prev = nextafterf(a, 0.0f);
        volatile float q = prev / sf;
        if (!(q >= C))
            break;
        a = prev;
    }
    for (int i = 0; i < 64; ++i) {
        volatile float q = a / sf;
        if (q >= C)
            break;
        a = nextafterf(a, INFINITY);
    }
    return u32_of(a);
}

typedef void (*KernelFn)(const KArgs);

template <int ESZ, int BS, int LC, int RPT, int WR, bool GRAD>
static KernelFn pick_tile(bool row, bool col, bool groups)
{
    if (row && col)
        return groups ? qdq_tile_kernel<ESZ, BS, LC, RPT, WR, true, true, true, GRAD>
                      : qdq_tile_kernel<ESZ, BS, LC, RPT, WR, true, true, false, GRAD>;
    if (col)
        return groups ? qdq_tile_kernel<ESZ, BS, LC, RPT, WR, false, true, true, GRAD>
                      : qdq_tile_kernel<ESZ, BS, LC, RPT, WR, false, true, false, GRAD>;
    return qdq_tile_kernel<ESZ, BS, LC, RPT, WR, true, false, false, GRAD>;
}

// Tile shape per (element size, block): LC lanes across, RPT rows per thread,
// WR warps down the tile.
template <int ESZ, int BS>
struct TileShape;
template <> struct TileShape<2, 32> { static constexpr int LC = 8, RPT = 8, WR = 1; };
template <> struct TileShape<2, 128> { static constexpr int LC = 16, RPT = 8, WR = 8; };
template <> struct TileShape<4, 32> { static constexpr int LC = 8, RPT = 8, WR = 1; };
template <> struct TileShape<4, 128> { static constexpr int LC = 32, RPT = 16, WR = 8; };

template <int ESZ, int BS>
static KernelFn pick_tile_shape(bool row, bool col, bool groups, bool grad, int& tc, int& nwg)
{
    using TS = TileShape<ESZ, BS>;
    tc = TS::LC * (16 / ESZ);
    nwg = (NTHREADS / 32) / TS::WR;
    return grad ? pick_tile<ESZ, BS, TS::LC, TS::RPT, TS::WR, true>(row, col, groups)
                : pick_tile<ESZ, BS, TS::LC, TS::RPT, TS::WR, false>(row, col, groups);
}

template <int FMT>
static KernelFn pick_generic_row_f(int esz, int bs, bool grad)
{
    if (FMT == MXFP4_ELEM_E4M3)  // block 32 only
        return esz == 2 ? (grad ? generic_row_kernel<2, 32, true, FMT> : generic_row_kernel<2, 32, false, FMT>)
                        : (grad ? generic_row_kernel<4, 32, true, FMT> : generic_row_kernel<4, 32, false, FMT>);
    if (esz == 2)
        return bs == 32 ? (grad ? generic_row_kernel<2, 32, true, FMT> : generic_row_kernel<2, 32, false, FMT>)
                        : (grad ? generic_row_kernel<2, 128, true, FMT> : generic_row_kernel<2, 128, false, FMT>);
    return bs == 32 ? (grad ? generic_row_kernel<4, 32, true, FMT> : generic_row_kernel<4, 32, false, FMT>)
                    : (grad ? generic_row_kernel<4, 128, true, FMT> : generic_row_kernel<4, 128, false, FMT>);
}

static KernelFn pick_generic_row(int esz, int bs, bool grad, int fmt)
{
    return fmt == MXFP4_ELEM_E4M3 ? pick_generic_row_f<MXFP4_ELEM_E4M3>(esz, bs, grad)
                                  : pick_generic_row_f<MXFP4_ELEM_E2M1>(esz, bs, grad);
}

template <int ESZ, int BS, int FMT>
static KernelFn pick_generic_col_bs(bool groups, bool grad)
{
    if (groups)
        return grad ? generic_col_kernel<ESZ, BS, true, true, FMT> : generic_col_kernel<ESZ, BS, true, false, FMT>;
    return grad ? generic_col_kernel<ESZ, BS, false, true, FMT> : generic_col_kernel<ESZ, BS, false, false, FMT>;
}

static KernelFn pick_generic_col(int esz, int bs, bool groups, bool grad, int fmt)
{
    if (fmt == MXFP4_ELEM_E4M3)  // block 32 only
        return esz == 2 ? pick_generic_col_bs<2, 32, MXFP4_ELEM_E4M3>(groups, grad)
                        : pick_generic_col_bs<4, 32, MXFP4_ELEM_E4M3>(groups, grad);
    if (esz == 2)
        return bs == 32 ? pick_generic_col_bs<2, 32, MXFP4_ELEM_E2M1>(groups, grad)
                        : pick_generic_col_bs<2, 128, MXFP4_ELEM_E2M1>(groups, grad);
    return bs == 32 ? pick_generic_col_bs<4, 32, MXFP4_ELEM_E2M1>(groups, grad)
                    : pick_generic_col_bs<4, 128, MXFP4_ELEM_E2M1>(groups, grad);
}

static mxfp4_status launch(KernelFn fn, int64_t work_units, size_t smem, const KArgs& k, cudaStream_t s)
{
    const int sms = device_sms();
    const int occ = occupancy((const void*)fn, smem);
    if (sms <= 0 || occ <= 0)
        return MXFP4_ECUDA;
    int64_t grid = (int64_t)sms * occ;
    if (work_units < grid)
        grid = work_units < 1 ? 1 : work_units;
    fn<<<(unsigned)grid, NTHREADS, smem, s>>>(k);
    return cudaGetLastError() == cudaSuccess ? MXFP4_OK : MXFP4_ECUDA;
}

// ---- staged path: TMA tensor maps ------------------------------------------

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled through the runtime's driver entry point (the library
// does not link libcuda directly); nullptr when unavailable.
static EncodeTiledFn encode_tiled()
{
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!tried) {
        tried = true;
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
        else
            (void)cudaGetLastError();
    }
    return fn;
}

// One 2-D tiled map: inner dimension d0 (elements of esz bytes), outer d1,
// row pitch bytes, box b0 x b1.
static bool encode_2d(CUtensorMap* tm, CUtensorMapDataType dt, void* base, uint64_t d0, uint64_t d1, uint64_t pitch,
                      uint32_t b0, uint32_t b1, CUtensorMapSwizzle sw)
{
    EncodeTiledFn fn = encode_tiled();
    if (!fn)
        return false;
    const cuuint64_t dims[2] = {(cuuint64_t)d0, (cuuint64_t)d1};
    const cuuint64_t strides[1] = {(cuuint64_t)pitch};
    const cuuint32_t box[2] = {(cuuint32_t)b0, (cuuint32_t)b1};
    const cuuint32_t estr[2] = {1, 1};
    return fn(tm, dt, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Maps of the staged kernel. x: bf16 [rows, cols] with row pitch ld * 2
// bytes, 64 x 32 boxes with the 128-byte swizzle (out-of-range elements read
// as zero). Outputs of both directions, each only where TMA can address it
// (16-byte aligned base and row pitch) and the tensor holds at least one
// full tile: y as x (pitch ld_y * 2), codes [rows, cols/2] bytes in 128 x 32
// boxes with the 128-byte swizzle, masks [rows, cols/8] bytes in 32 x 32
// boxes. Returns false when the input map cannot be built.
static bool make_staged_maps(StagedMaps* m, const KArgs& k, uint32_t* ts_flags)
{
    memset(m, 0, sizeof(*m));
    *ts_flags = 0;
    if (!encode_2d(&m->x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, const_cast<void*>(k.x), (uint64_t)k.cols,
                   (uint64_t)k.rows, (uint64_t)k.ld * 2, SG_SLAB_COLS, SG_ROWS, CU_TENSOR_MAP_SWIZZLE_128B))
        return false;
    if (k.cols < SG_COLS || k.rows < SG_ROWS)
        return true;
    if (k.y_col && aligned(k.y_col, 16) && (k.ld_y * 2) % 16 == 0 &&
        encode_2d(&m->y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, k.y_col, (uint64_t)k.cols, (uint64_t)k.rows,
                  (uint64_t)k.ld_y * 2, SG_SLAB_COLS, SG_ROWS, CU_TENSOR_MAP_SWIZZLE_128B))
        *ts_flags |= SG_TS_Y;
    if (k.codes_col && aligned(k.codes_col, 16) && (k.cols / 2) % 16 == 0 &&
        encode_2d(&m->codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, k.codes_col, (uint64_t)k.cols / 2, (uint64_t)k.rows,
                  (uint64_t)k.cols / 2, SG_COLS / 2, SG_ROWS, CU_TENSOR_MAP_SWIZZLE_128B))
        *ts_flags |= SG_TS_CODES;
    if (k.mask_col && aligned(k.mask_col, 16) && (k.cols / 8) % 16 == 0 &&
        encode_2d(&m->mask, CU_TENSOR_MAP_DATA_TYPE_UINT8, k.mask_col, (uint64_t)k.cols / 8, (uint64_t)k.rows,
                  (uint64_t)k.cols / 8, SG_COLS / 8, SG_ROWS, CU_TENSOR_MAP_SWIZZLE_NONE))
        *ts_flags |= SG_TS_MASK;
    if (k.y_row && aligned(k.y_row, 16) && (k.ld_y * 2) % 16 == 0 &&
        encode_2d(&m->yr, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, k.y_row, (uint64_t)k.cols, (uint64_t)k.rows,
                  (uint64_t)k.ld_y * 2, SG_SLAB_COLS, SG_ROWS, CU_TENSOR_MAP_SWIZZLE_128B))
        *ts_flags |= SG_TS_YR;
    if (k.codes_row && aligned(k.codes_row, 16) && (k.cols / 2) % 16 == 0 &&
        encode_2d(&m->codes_r, CU_TENSOR_MAP_DATA_TYPE_UINT8, k.codes_row, (uint64_t)k.cols / 2, (uint64_t)k.rows,
                  (uint64_t)k.cols / 2, SG_COLS / 2, SG_ROWS, CU_TENSOR_MAP_SWIZZLE_128B))
        *ts_flags |= SG_TS_CODES_R;
    if (k.mask_row && aligned(k.mask_row, 16) && (k.cols / 8) % 16 == 0 &&
        encode_2d(&m->mask_r, CU_TENSOR_MAP_DATA_TYPE_UINT8, k.mask_row, (uint64_t)k.cols / 8, (uint64_t)k.rows,
                  (uint64_t)k.cols / 8, SG_COLS / 8, SG_ROWS, CU_TENSOR_MAP_SWIZZLE_NONE))
        *ts_flags |= SG_TS_MASK_R;
    return true;
}

// Maps of the block-128 staged kernel: the same tensors in 64 x 128 boxes
// (x and y, 128-byte swizzle), codes in 64-byte x 128 boxes with the 64-byte
// swizzle, masks in 16-byte x 128 boxes.
static bool make_staged128_maps(StagedMaps* m, const KArgs& k, uint32_t* ts_flags)
{
    memset(m, 0, sizeof(*m));
    *ts_flags = 0;
    if (!encode_2d(&m->x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, const_cast<void*>(k.x), (uint64_t)k.cols,
                   (uint64_t)k.rows, (uint64_t)k.ld * 2, SG_SLAB_COLS, SB_ROWS, CU_TENSOR_MAP_SWIZZLE_128B))
        return false;
    if (k.cols < SB_COLS || k.rows < SB_ROWS)
        return true;
    const bool ypitch = (k.ld_y * 2) % 16 == 0, cpitch = (k.cols / 2) % 16 == 0, mpitch = (k.cols / 8) % 16 == 0;
    if (k.y_col && aligned(k.y_col, 16) && ypitch &&
        encode_2d(&m->y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, k.y_col, (uint64_t)k.cols, (uint64_t)k.rows,
                  (uint64_t)k.ld_y * 2, SG_SLAB_COLS, SB_ROWS, CU_TENSOR_MAP_SWIZZLE_128B))
        *ts_flags |= SG_TS_Y;
    if (k.y_row && aligned(k.y_row, 16) && ypitch &&
        encode_2d(&m->yr, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, k.y_row, (uint64_t)k.cols, (uint64_t)k.rows,
                  (uint64_t)k.ld_y * 2, SG_SLAB_COLS, SB_ROWS, CU_TENSOR_MAP_SWIZZLE_128B))
        *ts_flags |= SG_TS_YR;
    if (k.codes_col && aligned(k.codes_col, 16) && cpitch &&
        encode_2d(&m->codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, k.codes_col, (uint64_t)k.cols / 2, (uint64_t)k.rows,
                  (uint64_t)k.cols / 2, SB_COLS / 2, SB_ROWS, CU_TENSOR_MAP_SWIZZLE_64B))
        *ts_flags |= SG_TS_CODES;
    if (k.codes_row && aligned(k.codes_row, 16) && cpitch &&
        encode_2d(&m->codes_r, CU_TENSOR_MAP_DATA_TYPE_UINT8, k.codes_row, (uint64_t)k.cols / 2, (uint64_t)k.rows,
                  (uint64_t)k.cols / 2, SB_COLS / 2, SB_ROWS, CU_TENSOR_MAP_SWIZZLE_64B))
        *ts_flags |= SG_TS_CODES_R;
    if (k.mask_col && aligned(k.mask_col, 16) && mpitch &&
        encode_2d(&m->mask, CU_TENSOR_MAP_DATA_TYPE_UINT8, k.mask_col, (uint64_t)k.cols / 8, (uint64_t)k.rows,
                  (uint64_t)k.cols / 8, SB_COLS / 8, SB_ROWS, CU_TENSOR_MAP_SWIZZLE_NONE))
        *ts_flags |= SG_TS_MASK;
    if (k.mask_row && aligned(k.mask_row, 16) && mpitch &&
        encode_2d(&m->mask_r, CU_TENSOR_MAP_DATA_TYPE_UINT8, k.mask_row, (uint64_t)k.cols / 8, (uint64_t)k.rows,
                  (uint64_t)k.cols / 8, SB_COLS / 8, SB_ROWS, CU_TENSOR_MAP_SWIZZLE_NONE))
        *ts_flags |= SG_TS_MASK_R;
    return true;
}

typedef void (*StagedFn)(const StagedMaps, const KArgs);

// SMMA (row-wise scales in the MMA layout) is its own instantiation, so the
// row-major kernels carry no code for it
template <bool ROW, bool COL, bool GROUPS>
static StagedFn pick_staged(int mode, bool smma)
{
    if (ROW && smma)
        return mode == MXFP4_SCALE_FLOOR ? qdq_staged_kernel<ROW, COL, GROUPS, MXFP4_SCALE_FLOOR, ROW>
                                         : qdq_staged_kernel<ROW, COL, GROUPS, MXFP4_SCALE_PAGE, ROW>;
    return mode == MXFP4_SCALE_FLOOR ? qdq_staged_kernel<ROW, COL, GROUPS, MXFP4_SCALE_FLOOR, false>
                                     : qdq_staged_kernel<ROW, COL, GROUPS, MXFP4_SCALE_PAGE, false>;
}

template <bool ROW, bool COL, bool GROUPS>
static StagedFn pick_staged128(int mode)
{
    return mode == MXFP4_SCALE_FLOOR ? qdq_staged128_kernel<ROW, COL, GROUPS, MXFP4_SCALE_FLOOR>
                                     : qdq_staged128_kernel<ROW, COL, GROUPS, MXFP4_SCALE_PAGE>;
}

static mxfp4_status launch_staged128(bool row, bool col, bool groups, const StagedMaps& maps, const KArgs& k,
                                     int64_t tiles, size_t plan_smem, cudaStream_t s)
{
    StagedFn fn = !col ? pick_staged128<true, false, false>(k.mode)
                : row  ? (groups ? pick_staged128<true, true, true>(k.mode) : pick_staged128<true, true, false>(k.mode))
                       : (groups ? pick_staged128<false, true, true>(k.mode) : pick_staged128<false, true, false>(k.mode));
    const size_t smem = sizeof(Staged128Smem) + 1024 + plan_smem;
    if (cudaFuncSetAttribute((const void*)fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return MXFP4_ECUDA;
    const int sms = device_sms();
    const int occ = occupancy((const void*)fn, smem, SB_THREADS);
    if (sms <= 0 || occ <= 0)
        return MXFP4_ECUDA;
    int64_t grid = (int64_t)sms * occ;
    if (tiles < grid)
        grid = tiles < 1 ? 1 : tiles;
    fn<<<(unsigned)grid, SB_THREADS, smem, s>>>(maps, k);
    return cudaGetLastError() == cudaSuccess ? MXFP4_OK : MXFP4_ECUDA;
}

// row-only tiles never restart at groups (the caller routes row-only calls
// with a group_list elsewhere)
static mxfp4_status launch_staged(bool row, bool col, bool groups, const StagedMaps& maps, const KArgs& k,
                                  int64_t tiles, size_t plan_smem, cudaStream_t s)
{
    const bool sm = k.srow_mma && k.scales_row;
    StagedFn fn = !col ? pick_staged<true, false, false>(k.mode, sm)
                : row  ? (groups ? pick_staged<true, true, true>(k.mode, sm) : pick_staged<true, true, false>(k.mode, sm))
                       : (groups ? pick_staged<false, true, true>(k.mode, sm) : pick_staged<false, true, false>(k.mode, sm));
    const size_t smem = sizeof(StagedSmem) + 1024 + plan_smem;
    if (cudaFuncSetAttribute((const void*)fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return MXFP4_ECUDA;
    const int sms = device_sms();
    const int occ = occupancy((const void*)fn, smem, SG_THREADS);
    if (sms <= 0 || occ <= 0)
        return MXFP4_ECUDA;
    int64_t grid = (int64_t)sms * occ;
    if (tiles < grid)
        grid = tiles < 1 ? 1 : tiles;
    fn<<<(unsigned)grid, SG_THREADS, smem, s>>>(maps, k);
    return cudaGetLastError() == cudaSuccess ? MXFP4_OK : MXFP4_ECUDA;
}

// Maps of the MXFP8 staged kernel: x as for the block-32 staged kernel;
// row-wise y (64 x 32 boxes, 128-byte swizzle; pitch ld_y * 2), row-wise
// E4M3 codes [rows, cols] bytes in 128 x 32 boxes with the 128-byte swizzle,
// masks [rows, cols/8] bytes in 32 x 32 boxes, each only where TMA can
// address it and the tensor holds a full tile (ts_flags). Returns false when
// the input map cannot be built.
static bool make_staged8_maps(StagedMaps* m, const KArgs& k, uint32_t* ts_flags)
{
    memset(m, 0, sizeof(*m));
    *ts_flags = 0;
    if (!encode_2d(&m->x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, const_cast<void*>(k.x), (uint64_t)k.cols,
                   (uint64_t)k.rows, (uint64_t)k.ld * 2, SG_SLAB_COLS, SG_ROWS, CU_TENSOR_MAP_SWIZZLE_128B))
        return false;
    if (k.cols < SG_COLS || k.rows < SG_ROWS)
        return true;
    if (k.y_row && aligned(k.y_row, 16) && (k.ld_y * 2) % 16 == 0 &&
        encode_2d(&m->yr, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, k.y_row, (uint64_t)k.cols, (uint64_t)k.rows,
                  (uint64_t)k.ld_y * 2, SG_SLAB_COLS, SG_ROWS, CU_TENSOR_MAP_SWIZZLE_128B))
        *ts_flags |= SG_TS_YR;
    if (k.codes_row && aligned(k.codes_row, 16) && k.cols % 16 == 0 &&
        encode_2d(&m->codes_r, CU_TENSOR_MAP_DATA_TYPE_UINT8, k.codes_row, (uint64_t)k.cols, (uint64_t)k.rows,
                  (uint64_t)k.cols, 128, SG_ROWS, CU_TENSOR_MAP_SWIZZLE_128B))
        *ts_flags |= SG_TS_CODES_R;
    if (k.mask_row && aligned(k.mask_row, 16) && (k.cols / 8) % 16 == 0 &&
        encode_2d(&m->mask_r, CU_TENSOR_MAP_DATA_TYPE_UINT8, k.mask_row, (uint64_t)k.cols / 8, (uint64_t)k.rows,
                  (uint64_t)k.cols / 8, SG_COLS / 8, SG_ROWS, CU_TENSOR_MAP_SWIZZLE_NONE))
        *ts_flags |= SG_TS_MASK_R;
    if (k.mask_col && aligned(k.mask_col, 16) && (k.cols / 8) % 16 == 0 &&
        encode_2d(&m->mask, CU_TENSOR_MAP_DATA_TYPE_UINT8, k.mask_col, (uint64_t)k.cols / 8, (uint64_t)k.rows,
                  (uint64_t)k.cols / 8, SG_COLS / 8, SG_ROWS, CU_TENSOR_MAP_SWIZZLE_NONE))
        *ts_flags |= SG_TS_MASK;
    return true;
}

template <bool ROW, bool GROUPS>
static StagedFn pick_staged8(bool smma)
{
    return smma ? qdq_staged8_kernel<ROW, GROUPS, true> : qdq_staged8_kernel<ROW, GROUPS, false>;
}

// MXFP8 staged kernel (both directions or column-wise alone).
static mxfp4_status launch_staged8(bool row, bool groups, const StagedMaps& maps, const KArgs& k, int64_t tiles,
                                   size_t plan_smem, cudaStream_t s)
{
    const bool sm = k.srow_mma && k.scales_row;
    StagedFn fn = row ? (groups ? pick_staged8<true, true>(sm) : pick_staged8<true, false>(sm))
                      : (groups ? pick_staged8<false, true>(sm) : pick_staged8<false, false>(sm));
    const size_t smem = sizeof(Staged8Smem) + 1024 + plan_smem;
    if (cudaFuncSetAttribute((const void*)fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return MXFP4_ECUDA;
    const int sms = device_sms();
    const int occ = occupancy((const void*)fn, smem, S8_THREADS);
    if (sms <= 0 || occ <= 0)
        return MXFP4_ECUDA;
    int64_t grid = (int64_t)sms * occ;
    if (tiles < grid)
        grid = tiles < 1 ? 1 : tiles;
    fn<<<(unsigned)grid, S8_THREADS, smem, s>>>(maps, k);
    return cudaGetLastError() == cudaSuccess ? MXFP4_OK : MXFP4_ECUDA;
}

template <bool SMMA, bool VALS>
static const void* pick_row_stream(int mode)
{
    return mode == MXFP4_SCALE_FLOOR ? (const void*)row_stream_kernel<MXFP4_SCALE_FLOOR, SMMA, VALS>
                                     : (const void*)row_stream_kernel<MXFP4_SCALE_PAGE, SMMA, VALS>;
}

static mxfp4_status launch_row_stream(const KArgs& k, int64_t blocks, cudaStream_t s)
{
    const bool sm = k.srow_mma && k.scales_row;
    const void* fn = k.y_row ? (sm ? pick_row_stream<true, true>(k.mode) : pick_row_stream<false, true>(k.mode))
                             : (sm ? pick_row_stream<true, false>(k.mode) : pick_row_stream<false, false>(k.mode));
    const int sms = device_sms();
    const int occ = occupancy(fn, 0);
    if (sms <= 0 || occ <= 0)
        return MXFP4_ECUDA;
    int64_t grid = (int64_t)sms * occ;
    if ((blocks + NTHREADS - 1) / NTHREADS < grid)
        grid = (blocks + NTHREADS - 1) / NTHREADS;
    void* args[] = {const_cast<KArgs*>(&k)};
    return cudaLaunchKernel(fn, dim3((unsigned)grid), dim3(NTHREADS), args, 0, s) == cudaSuccess ? MXFP4_OK
                                                                                               : MXFP4_ECUDA;
}

static mxfp4_status launch_row_stream8(const KArgs& k, int64_t blocks, cudaStream_t s)
{
    const void* fn = k.srow_mma && k.scales_row ? (const void*)row_stream8_kernel<true>
                                                : (const void*)row_stream8_kernel<false>;
    const int sms = device_sms();
    const int occ = occupancy(fn, 0);
    if (sms <= 0 || occ <= 0)
        return MXFP4_ECUDA;
    int64_t grid = (int64_t)sms * occ;
    if ((blocks + NTHREADS - 1) / NTHREADS < grid)
        grid = (blocks + NTHREADS - 1) / NTHREADS;
    void* args[] = {const_cast<KArgs*>(&k)};
    return cudaLaunchKernel(fn, dim3((unsigned)grid), dim3(NTHREADS), args, 0, s) == cudaSuccess ? MXFP4_OK
                                                                                               : MXFP4_ECUDA;
}

static mxfp4_status check_geometry(const mxfp4_qdq_args* a)
{
    if (!a)
        return MXFP4_EINVAL;
    if (a->dtype != MXFP4_F32 && a->dtype != MXFP4_BF16)
        return MXFP4_EINVAL;
    if (a->block <= 0)
        return MXFP4_EINVAL;
    if (a->block != 32 && a->block != 128)
        return MXFP4_EUNSUPPORTED;
    if (!(a->scale_factor > 0.0f) || !isfinite(a->scale_factor))
        return MXFP4_EINVAL;
    if (a->scale_mode != MXFP4_SCALE_PAGE && a->scale_mode != MXFP4_SCALE_FLOOR)
        return MXFP4_EINVAL;
    if (a->rows < 0 || a->cols < 0)
        return MXFP4_EINVAL;
    if (a->rows > INT32_MAX || a->cols > INT32_MAX)
        return MXFP4_EUNSUPPORTED;
    if (a->dirs == 0 || (a->dirs & ~(MXFP4_ROWWISE | MXFP4_COLWISE)))
        return MXFP4_EINVAL;
    if (a->scales_row_layout != MXFP4_SCALES_ROWMAJOR && a->scales_row_layout != MXFP4_SCALES_MMA)
        return MXFP4_EINVAL;
    if (a->elem_format != MXFP4_ELEM_E2M1 && a->elem_format != MXFP4_ELEM_E4M3)
        return MXFP4_EINVAL;
    if (a->elem_format == MXFP4_ELEM_E4M3 && (a->block != 32 || a->scale_mode != MXFP4_SCALE_FLOOR))
        return MXFP4_EUNSUPPORTED;
    if (a->col_layout != MXFP4_COLS_ROWMAJOR && a->col_layout != MXFP4_COLS_MMA)
        return MXFP4_EINVAL;
    if (a->group_list) {
        if (a->num_groups < 1)
            return MXFP4_EINVAL;
        if (a->num_groups > MXFP4_MAX_GROUPS)
            return MXFP4_EUNSUPPORTED;
        if (a->group_list_type != 0 && a->group_list_type != 1)
            return MXFP4_EINVAL;
        if (!aligned(a->group_list, 8))
            return MXFP4_EINVAL;
    }
    return MXFP4_OK;
}

// Column-wise codes and scales in the GEMM operand layout (MXFP4_COLS_MMA):
// host checks, then one launch of col_operand_kernel.
static mxfp4_status launch_col_operand(const mxfp4_qdq_args* A, cudaStream_t s)
{
    if (A->block != 32 || A->elem_format != MXFP4_ELEM_E2M1 || A->dtype != MXFP4_BF16)
        return MXFP4_EUNSUPPORTED;
    if (A->scale_mode == MXFP4_SCALE_PAGE && !page_fast_ok(A->scale_factor))
        return MXFP4_EUNSUPPORTED;
    const bool groups = A->group_list != nullptr;
    if (A->k_alloc <= 0 || A->k_alloc % OP_KPAD != 0 || A->k_alloc > (int64_t)INT32_MAX * OP_KPAD)
        return MXFP4_EINVAL;
    if (!groups && A->k_alloc < OP_KPAD * ((A->rows + OP_KPAD - 1) / OP_KPAD))
        return MXFP4_EINVAL;
    if (!A->x || A->ld < A->cols || !aligned(A->x, 2))
        return MXFP4_EINVAL;
    if ((A->codes_col && !aligned(A->codes_col, 16)) || (A->scales_col && !aligned(A->scales_col, 2)))
        return MXFP4_EINVAL;
    KArgs k;
    memset(&k, 0, sizeof(k));
    k.x = A->x;
    k.rows = A->rows;
    k.cols = A->cols;
    k.ld = A->ld;
    k.sf = A->scale_factor;
    k.mode = A->scale_mode;
    k.codes_col = A->codes_col;
    k.scales_col = A->scales_col;
    k.group_list = groups ? A->group_list : nullptr;
    k.num_groups = groups ? (int32_t)A->num_groups : 0;
    k.gl_type = A->group_list_type;
    k.status = A->status;
    k.k_alloc = A->k_alloc;
    if (A->scale_mode == MXFP4_SCALE_PAGE)
        k.thr = page_threshold(A->scale_factor);
    if (A->status && !groups && cudaMemsetAsync(A->status, 0, sizeof(int32_t), s) != cudaSuccess)
        return MXFP4_ECUDA;
    const size_t plan_bytes = groups ? (size_t)(2 * (A->num_groups + 1)) * sizeof(int32_t) : 0;
    // TMA-staged kernel where x is addressable by TMA and the outputs take
    // its 32-byte and 16-bit stores
    if (A->cols % 32 == 0 && A->ld % 8 == 0 && aligned(A->x, 16) && (!k.codes_col || aligned(k.codes_col, 32)) &&
        A->rows <= INT32_MAX - 128 && A->cols <= INT32_MAX - SG_COLS) {
        StagedMaps maps;
        memset(&maps, 0, sizeof(maps));
        const int64_t n_ct = (A->cols + SG_COLS - 1) / SG_COLS;
        const int64_t pairs = 2 * (A->k_alloc / OP_KPAD);
        if (pairs * n_ct < (int64_t)INT32_MAX &&
            encode_2d(&maps.x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, const_cast<void*>(k.x), (uint64_t)k.cols,
                      (uint64_t)k.rows, (uint64_t)k.ld * 2, SG_SLAB_COLS, SG_ROWS, CU_TENSOR_MAP_SWIZZLE_128B)) {
            k.n_ct = (uint32_t)n_ct;
            StagedFn sfn = A->scale_mode == MXFP4_SCALE_FLOOR
                               ? (groups ? col_operand_staged_kernel<MXFP4_SCALE_FLOOR, true>
                                         : col_operand_staged_kernel<MXFP4_SCALE_FLOOR, false>)
                               : (groups ? col_operand_staged_kernel<MXFP4_SCALE_PAGE, true>
                                         : col_operand_staged_kernel<MXFP4_SCALE_PAGE, false>);
            const size_t smem = sizeof(OpsSmem) + 1024 + plan_bytes;
            if (cudaFuncSetAttribute((const void*)sfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
                cudaSuccess)
                return MXFP4_ECUDA;
            const int sms = device_sms();
            const int occ = occupancy((const void*)sfn, smem, OPS_THREADS);
            if (sms <= 0 || occ <= 0)
                return MXFP4_ECUDA;
            int64_t grid = (int64_t)sms * occ;
            if (pairs * n_ct < grid)
                grid = pairs * n_ct < 1 ? 1 : pairs * n_ct;
            sfn<<<(unsigned)grid, OPS_THREADS, smem, s>>>(maps, k);
            return cudaGetLastError() == cudaSuccess ? MXFP4_OK : MXFP4_ECUDA;
        }
    }
    const void* fn;
    if (A->scale_mode == MXFP4_SCALE_FLOOR)
        fn = groups ? (const void*)col_operand_kernel<MXFP4_SCALE_FLOOR, true>
                    : (const void*)col_operand_kernel<MXFP4_SCALE_FLOOR, false>;
    else
        fn = groups ? (const void*)col_operand_kernel<MXFP4_SCALE_PAGE, true>
                    : (const void*)col_operand_kernel<MXFP4_SCALE_PAGE, false>;
    const size_t plan_smem = groups ? (size_t)(2 * (A->num_groups + 1)) * sizeof(int32_t) : 0;
    // the grid covers the K units the caller allocated: units past the real
    // groups' end exit at once
    const int64_t units = (A->k_alloc / 64) * ((A->cols + 1) / 2);
    const int sms = device_sms();
    const int occ = occupancy(fn, plan_smem);
    if (sms <= 0 || occ <= 0)
        return MXFP4_ECUDA;
    int64_t grid = (int64_t)sms * occ;
    if ((units + NTHREADS - 1) / NTHREADS < grid)
        grid = (units + NTHREADS - 1) / NTHREADS;
    void* args[] = {&k};
    return cudaLaunchKernel(fn, dim3((unsigned)grid), dim3(NTHREADS), args, plan_smem, s) == cudaSuccess
               ? MXFP4_OK
               : MXFP4_ECUDA;
}

// Validates, then queues the forward (and the fused backward when g_in is set).
static mxfp4_status run_qdq(const mxfp4_qdq_args* A, const void* g_out, void* g_in, int64_t ld_g,
                            uint32_t grad_dir, cudaStream_t s)
{
    mxfp4_status st = check_geometry(A);
    if (st != MXFP4_OK)
        return st;
    const bool row = A->dirs & MXFP4_ROWWISE, col = A->dirs & MXFP4_COLWISE;
    const bool grad = g_in != nullptr;
    const int esz = A->dtype == MXFP4_BF16 ? 2 : 4;
    if (grad) {
        if (!g_out || (grad_dir != MXFP4_ROWWISE && grad_dir != MXFP4_COLWISE) || !(A->dirs & grad_dir))
            return MXFP4_EINVAL;
        if (ld_g < A->cols || !aligned(g_out, esz) || !aligned(g_in, esz))
            return MXFP4_EINVAL;
    }
    const bool groups = col && A->group_list != nullptr;
    if (A->rows == 0 || A->cols == 0) {
        if (A->status && cudaMemsetAsync(A->status, 0, sizeof(int32_t), s) != cudaSuccess)
            return MXFP4_ECUDA;
        return MXFP4_OK;
    }
    if (col && A->col_layout == MXFP4_COLS_MMA && (A->codes_col || A->scales_col)) {
        // The operand kernel runs last, so that its group_list check (which
        // also covers k_alloc) is the last word written to status; the other
        // outputs of the call go through the usual paths first.
        if (grad)
            return MXFP4_EUNSUPPORTED;
        mxfp4_qdq_args R = *A;
        R.codes_col = R.scales_col = nullptr;
        R.col_layout = MXFP4_COLS_ROWMAJOR;
        const bool rows_out = row && (R.y_row || R.codes_row || R.scales_row || R.mask_row);
        const bool cols_out = R.y_col || R.mask_col;
        if (!cols_out)
            R.dirs &= ~MXFP4_COLWISE;
        if (!rows_out)
            R.dirs &= ~MXFP4_ROWWISE;
        if (R.dirs != 0) {
            // host checks of the operand first: nothing is queued for an invalid call
            if (A->k_alloc <= 0 || A->k_alloc % OP_KPAD != 0)
                return MXFP4_EINVAL;
            st = run_qdq(&R, nullptr, nullptr, 0, 0, s);
            if (st != MXFP4_OK)
                return st;
        }
        return launch_col_operand(A, s);
    }
    if (!A->x || A->ld < A->cols || !aligned(A->x, esz))
        return MXFP4_EINVAL;

    KArgs k;
    memset(&k, 0, sizeof(k));
    k.x = A->x;
    k.rows = A->rows;
    k.cols = A->cols;
    k.ld = A->ld;
    k.sf = A->scale_factor;
    k.mode = A->scale_mode;
    k.grad_dir = grad ? (int32_t)grad_dir : 0;
    k.mul4 = 4;
    k.mul16 = 65536;
    if (row) {
        k.y_row = A->y_row;
        k.codes_row = A->codes_row;
        k.scales_row = A->scales_row;
        k.srow_mma = A->scales_row_layout == MXFP4_SCALES_MMA;
        k.mask_row = A->mask_row;
    }
    if (col) {
        k.y_col = A->y_col;
        k.codes_col = A->codes_col;
        k.scales_col = A->scales_col;
        k.mask_col = A->mask_col;
    }
    k.ld_y = A->ld_y;
    k.fmt = A->elem_format;
    if ((k.y_row || k.y_col) && A->ld_y < A->cols)
        return MXFP4_EINVAL;
    if ((k.y_row && !aligned(k.y_row, esz)) || (k.y_col && !aligned(k.y_col, esz)))
        return MXFP4_EINVAL;
    k.g_out = g_out;
    k.g_in = g_in;
    k.ld_g = ld_g;
    k.group_list = groups ? A->group_list : nullptr;
    k.num_groups = groups ? (int32_t)A->num_groups : 0;
    k.gl_type = A->group_list_type;
    k.status = A->status;
    if (A->status && !groups && cudaMemsetAsync(A->status, 0, sizeof(int32_t), s) != cudaSuccess)
        return MXFP4_ECUDA;

    const int vec = 16 / esz;
    bool fast = aligned(A->x, 16) && A->ld % vec == 0 && A->cols % vec == 0;
    for (void* y : {k.y_row, k.y_col})
        if (y)
            fast = fast && aligned(y, 16) && A->ld_y % vec == 0;
    for (uint8_t* c : {k.codes_row, k.codes_col})
        if (c)
            fast = fast && aligned(c, vec / 2);
    if (k.scales_col)
        fast = fast && aligned(k.scales_col, vec);
    if (grad)
        fast = fast && aligned(g_out, 16) && aligned(g_in, 16) && ld_g % vec == 0;
    if (A->scale_mode == MXFP4_SCALE_PAGE) {
        fast = fast && page_fast_ok(A->scale_factor);
        if (fast)
            k.thr = page_threshold(A->scale_factor);
    }

    const int bs = A->block;
    const size_t plan_smem = groups ? (size_t)(2 * (A->num_groups + 1)) * sizeof(int32_t) : 0;
    const int64_t s_bound = groups ? A->rows / bs + A->num_groups : (A->rows + bs - 1) / bs;

    if (k.fmt == MXFP4_ELEM_E4M3 && esz == 2 && !grad && col && A->cols % 32 == 0 && A->ld % 8 == 0 &&
        aligned(A->x, 16) && (!(k.y_row || k.y_col) || A->ld_y % 8 == 0) && (!k.y_row || aligned(k.y_row, 16)) &&
        (!k.y_col || aligned(k.y_col, 16)) && (!k.codes_row || aligned(k.codes_row, 16)) &&
        (!k.codes_col || aligned(k.codes_col, 2)) && (!k.scales_col || aligned(k.scales_col, 2)) &&
        (!k.mask_row || aligned(k.mask_row, 4)) && (!k.mask_col || aligned(k.mask_col, 4)) &&
        A->rows <= INT32_MAX - 2 * SG_ROWS && A->cols <= INT32_MAX - 2 * SG_COLS) {
        // MXFP8 column-wise (and row-wise), bf16: the staged kernel, one read
        // of each tile for both directions
        StagedMaps maps;
        if (make_staged8_maps(&maps, k, &k.ts_flags)) {
            const int64_t n_ct = (A->cols + SG_COLS - 1) / SG_COLS;
            if (s_bound * n_ct >= (int64_t)INT32_MAX)
                return MXFP4_EUNSUPPORTED;
            k.n_ct = (uint32_t)n_ct;
            return launch_staged8(row, groups, maps, k, s_bound * n_ct, plan_smem, s);
        }
    }
    if (k.fmt == MXFP4_ELEM_E4M3 && esz == 2 && !grad) {
        // MXFP8, bf16: the row-wise part on the streaming kernel, the
        // column-wise part on the column-pair kernel, where their layout
        // conditions hold; the rest on the generic kernels
        const bool row8 = row && fast && A->cols % 32 == 0 && A->ld % 16 == 0 && aligned(A->x, 32) &&
                          (!k.y_row || (aligned(k.y_row, 32) && A->ld_y % 16 == 0)) &&
                          (!k.codes_row || aligned(k.codes_row, 32)) && (!k.mask_row || aligned(k.mask_row, 4)) &&
                          A->rows * (A->cols / 32) < (int64_t)UINT32_MAX;
        const bool col8 = col && A->cols % 8 == 0 && A->ld % 2 == 0 && aligned(A->x, 4) &&
                          (!k.y_col || (aligned(k.y_col, 4) && A->ld_y % 2 == 0)) &&
                          (!k.codes_col || aligned(k.codes_col, 2)) && (!k.scales_col || aligned(k.scales_col, 2));
        if (row8 || col8) {
            if (row) {
                KArgs kr = k;
                kr.y_col = nullptr;
                kr.codes_col = kr.scales_col = kr.mask_col = nullptr;
                st = row8 ? launch_row_stream8(kr, A->rows * (A->cols / 32), s)
                          : launch(pick_generic_row(esz, bs, false, k.fmt),
                                   (A->rows * ((A->cols + bs - 1) / bs) + NTHREADS - 1) / NTHREADS, 0, kr, s);
                if (st != MXFP4_OK)
                    return st;
            }
            if (col) {
                const int64_t units = s_bound * ((A->cols + 7) / 8);
                if (col8)
                    return launch(groups ? col_pair8_kernel<true> : col_pair8_kernel<false>,
                                  (s_bound * (A->cols / 2) + NTHREADS - 1) / NTHREADS, plan_smem, k, s);
                return launch(pick_generic_col(esz, bs, groups, false, k.fmt), (units + NTHREADS - 1) / NTHREADS,
                              plan_smem, k, s);
            }
            return st;
        }
    }
    if (k.fmt == MXFP4_ELEM_E4M3)
        fast = false;  // MXFP8 otherwise: the generic kernels below

    // row-wise only, bf16 block 32, with codes or masks (or without values):
    // one streaming pass, one thread per block. Values alone go to the staged
    // kernel, whose tiled stores measured faster for that traffic mix.
    if (fast && row && !col && esz == 2 && bs == 32 && !grad && (!k.y_row || k.codes_row || k.mask_row) &&
        A->cols % 32 == 0 && A->ld % 16 == 0 &&
        aligned(A->x, 32) && (!k.y_row || (aligned(k.y_row, 32) && A->ld_y % 16 == 0)) &&
        (!k.codes_row || aligned(k.codes_row, 16)) && (!k.mask_row || aligned(k.mask_row, 4)) &&
        A->rows * (A->cols / 32) < (int64_t)UINT32_MAX)
        return launch_row_stream(k, A->rows * (A->cols / 32), s);

    // TMA coordinates and the staged kernel's tile bookkeeping are 32-bit
    if (fast && esz == 2 && bs == 32 && (col || !groups) && !grad && A->rows <= INT32_MAX - 2 * SG_ROWS &&
        A->cols <= INT32_MAX - 2 * SG_COLS) {
        StagedMaps maps;
        if (make_staged_maps(&maps, k, &k.ts_flags)) {
            const int64_t n_ct = (A->cols + SG_COLS - 1) / SG_COLS;
            if (s_bound * n_ct >= (int64_t)INT32_MAX)
                return MXFP4_EUNSUPPORTED;
            k.n_ct = (uint32_t)n_ct;
            return launch_staged(row, col, groups, maps, k, s_bound * n_ct, plan_smem, s);
        }
    }
    if (fast && esz == 2 && bs == 128 && (col || !groups) && !grad && A->rows <= INT32_MAX - 2 * SB_ROWS &&
        A->cols <= INT32_MAX - 2 * SB_COLS) {
        StagedMaps maps;
        if (make_staged128_maps(&maps, k, &k.ts_flags)) {
            const int64_t n_ct = (A->cols + SB_COLS - 1) / SB_COLS;
            if (s_bound * n_ct >= (int64_t)INT32_MAX)
                return MXFP4_EUNSUPPORTED;
            k.n_ct = (uint32_t)n_ct;
            return launch_staged128(row, col, groups, maps, k, s_bound * n_ct, plan_smem, s);
        }
    }
    if (fast) {
        int tc = 0, nwg = 1;
        KernelFn fn;
        if (esz == 2)
            fn = bs == 32 ? pick_tile_shape<2, 32>(row, col, groups, grad, tc, nwg)
                          : pick_tile_shape<2, 128>(row, col, groups, grad, tc, nwg);
        else
            fn = bs == 32 ? pick_tile_shape<4, 32>(row, col, groups, grad, tc, nwg)
                          : pick_tile_shape<4, 128>(row, col, groups, grad, tc, nwg);
        const int64_t n_ct = (A->cols + tc - 1) / tc;
        if (s_bound * n_ct >= (int64_t)INT32_MAX)
            return MXFP4_EUNSUPPORTED;
        k.n_ct = (uint32_t)n_ct;
        return launch(fn, (s_bound * n_ct + nwg - 1) / nwg, plan_smem, k, s);
    }

    // generic path: one kernel per direction
    if (row) {
        KArgs kr = k;
        kr.y_col = nullptr;
        st = launch(pick_generic_row(esz, bs, grad && grad_dir == MXFP4_ROWWISE, k.fmt),
                    (A->rows * ((A->cols + bs - 1) / bs) + NTHREADS - 1) / NTHREADS, 0, kr, s);
        if (st != MXFP4_OK)
            return st;
    }
    if (col) {
        const int64_t units = s_bound * ((A->cols + 7) / 8);
        st = launch(pick_generic_col(esz, bs, groups, grad && grad_dir == MXFP4_COLWISE, k.fmt),
                    (units + NTHREADS - 1) / NTHREADS, plan_smem, k, s);
    }
    return st;
}

// ---- grouped block-scaled GEMM (mxfp4_grouped_gemm) -----------------------

template <int FMT, bool GK, bool F32>
static mxfp4_status launch_gmm_t(const GmMaps& maps, const GmArgs& g, int64_t tile_bound, cudaStream_t s)
{
    const void* fn = (const void*)gmm_kernel<FMT, GK, F32>;
    const size_t smem = sizeof(GmSmem<FMT>) + 1024 + (size_t)(2 * (g.num_groups + 1)) * sizeof(int32_t);
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return MXFP4_ECUDA;
    const int sms = device_sms();
    if (sms <= 0)
        return MXFP4_ECUDA;
    int64_t grid = sms;
    if (tile_bound < grid)
        grid = tile_bound < 1 ? 1 : tile_bound;
    GmMaps m = maps;
    GmArgs a = g;
    void* args[] = {&m, &a};
    return cudaLaunchKernel(fn, dim3((unsigned)grid), dim3(GM_THREADS), args, smem, s) == cudaSuccess ? MXFP4_OK
                                                                                                    : MXFP4_ECUDA;
}

static mxfp4_status run_gmm(const mxfp4_gmm_args* A, cudaStream_t s)
{
    if (!A)
        return MXFP4_EINVAL;
    if (A->elem_format != MXFP4_ELEM_E2M1 && A->elem_format != MXFP4_ELEM_E4M3)
        return MXFP4_EINVAL;
    if (A->group_mode != MXFP4_GMM_GROUP_M && A->group_mode != MXFP4_GMM_GROUP_K)
        return MXFP4_EINVAL;
    if (A->d_dtype != MXFP4_F32 && A->d_dtype != MXFP4_BF16)
        return MXFP4_EINVAL;
    if (A->m < 0 || A->n < 0 || A->k < 0 || A->k % GM_KU != 0)
        return MXFP4_EINVAL;
    if (A->m > INT32_MAX || A->n > INT32_MAX || A->k > INT32_MAX)
        return MXFP4_EUNSUPPORTED;
    if (!A->group_list || A->num_groups < 1 || (A->group_list_type != 0 && A->group_list_type != 1) ||
        !aligned(A->group_list, 8))
        return MXFP4_EINVAL;
    if (A->num_groups > MXFP4_MAX_GROUPS)
        return MXFP4_EUNSUPPORTED;
    const bool gk = A->group_mode == MXFP4_GMM_GROUP_K;
    if (gk && A->k_rows < 0)
        return MXFP4_EINVAL;
    if (A->m == 0 || A->n == 0) {
        if (A->status && cudaMemsetAsync(A->status, 0, sizeof(int32_t), s) != cudaSuccess)
            return MXFP4_ECUDA;
        return MXFP4_OK;
    }
    const int64_t kb = A->elem_format == MXFP4_ELEM_E2M1 ? A->k / 2 : A->k;  // bytes of a K row
    const int esz = A->d_dtype == MXFP4_F32 ? 4 : 2;
    if (!A->a || !A->b || !A->a_scales || !A->b_scales || !A->d)
        return MXFP4_EINVAL;
    if (A->lda < kb || A->ldb < kb || A->lda % 16 != 0 || A->ldb % 16 != 0 || !aligned(A->a, 16) || !aligned(A->b, 16))
        return MXFP4_EINVAL;
    if (!aligned(A->a_scales, 4) || !aligned(A->b_scales, 4) || A->ldd < A->n || !aligned(A->d, 16) ||
        (A->ldd * esz) % 16 != 0)
        return MXFP4_EINVAL;
    const bool e2 = A->elem_format == MXFP4_ELEM_E2M1;
    const int row_bytes = GM_ROW_BYTES;
    const CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B;
    GmMaps maps;
    memset(&maps, 0, sizeof(maps));
    const int64_t b_rows = gk ? A->n : A->n * A->num_groups;
    if (!encode_2d(&maps.a, CU_TENSOR_MAP_DATA_TYPE_UINT8, const_cast<uint8_t*>(A->a), (uint64_t)kb, (uint64_t)A->m,
                   (uint64_t)A->lda, (uint32_t)row_bytes, GM_BM, sw) ||
        !encode_2d(&maps.b, CU_TENSOR_MAP_DATA_TYPE_UINT8, const_cast<uint8_t*>(A->b), (uint64_t)kb, (uint64_t)b_rows,
                   (uint64_t)A->ldb, (uint32_t)row_bytes, GM_BN, sw))
        return MXFP4_ECUDA;
    GmArgs g;
    memset(&g, 0, sizeof(g));
    g.sfa = A->a_scales;
    g.sfb = A->b_scales;
    g.d = A->d;
    g.group_list = A->group_list;
    g.status = A->status;
    g.a_rows = A->m;
    g.n = A->n;
    g.k = A->k;
    g.ldd = A->ldd;
    g.sfb_group_bytes = 512 * ((A->n + 127) / 128) * ((A->k / 32 + 3) / 4);
    g.k_rows = A->k_rows;
    g.num_groups = (int32_t)A->num_groups;
    g.gl_type = A->group_list_type;
    g.d_f32 = A->d_dtype == MXFP4_F32;
    g.group_k = gk;
    const int64_t n_nt = (A->n + GM_BN - 1) / GM_BN;
    const int64_t bound = gk ? A->num_groups * ((A->m + GM_BM - 1) / GM_BM) * n_nt : (A->m / GM_BM + A->num_groups) * n_nt;
    const bool f32 = A->d_dtype == MXFP4_F32;
    if (e2)
        return gk ? (f32 ? launch_gmm_t<MXFP4_ELEM_E2M1, true, true>(maps, g, bound, s)
                         : launch_gmm_t<MXFP4_ELEM_E2M1, true, false>(maps, g, bound, s))
                  : (f32 ? launch_gmm_t<MXFP4_ELEM_E2M1, false, true>(maps, g, bound, s)
                         : launch_gmm_t<MXFP4_ELEM_E2M1, false, false>(maps, g, bound, s));
    return gk ? (f32 ? launch_gmm_t<MXFP4_ELEM_E4M3, true, true>(maps, g, bound, s)
                     : launch_gmm_t<MXFP4_ELEM_E4M3, true, false>(maps, g, bound, s))
              : (f32 ? launch_gmm_t<MXFP4_ELEM_E4M3, false, true>(maps, g, bound, s)
                     : launch_gmm_t<MXFP4_ELEM_E4M3, false, false>(maps, g, bound, s));
}

#include "mxfp4_dual.cuh"

}  // namespace mxfp4

using namespace mxfp4;

extern "C" {

mxfp4_status mxfp4_qdq_fwd(const mxfp4_qdq_args* args, mxfp4_stream_t stream)
{
    return run_qdq(args, nullptr, nullptr, 0, 0, reinterpret_cast<cudaStream_t>(stream));
}

mxfp4_status mxfp4_qdq_fwd_bwd(const mxfp4_qdq_args* args, const void* grad_out, void* grad_in,
                               int64_t ld_grad, uint32_t grad_dir, mxfp4_stream_t stream)
{
    if (!grad_in)
        return MXFP4_EINVAL;
    return run_qdq(args, grad_out, grad_in, ld_grad, grad_dir, reinterpret_cast<cudaStream_t>(stream));
}

mxfp4_status mxfp4_ste_bwd(const mxfp4_qdq_args* geom, const void* grad_out, void* grad_in,
                           int64_t ld_grad, const uint8_t* saved_mask, int32_t clip_grad,
                           mxfp4_stream_t stream)
{
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (!geom || (geom->dirs != MXFP4_ROWWISE && geom->dirs != MXFP4_COLWISE))
        return MXFP4_EINVAL;
    if (geom->dtype != MXFP4_F32 && geom->dtype != MXFP4_BF16)
        return MXFP4_EINVAL;
    if (geom->rows < 0 || geom->cols < 0)
        return MXFP4_EINVAL;
    if (geom->rows > INT32_MAX || geom->cols > INT32_MAX)
        return MXFP4_EUNSUPPORTED;
    if (geom->rows == 0 || geom->cols == 0)
        return MXFP4_OK;
    const int esz = geom->dtype == MXFP4_BF16 ? 2 : 4;
    if (!grad_out || !grad_in || ld_grad < geom->cols || !aligned(grad_out, esz) || !aligned(grad_in, esz))
        return MXFP4_EINVAL;
    if (clip_grad && !saved_mask && geom->dirs == MXFP4_ROWWISE && esz == 2 && geom->block == 32 &&
        geom->elem_format == MXFP4_ELEM_E2M1 &&
        geom->cols % 32 == 0 && geom->x && geom->ld >= geom->cols && geom->ld % 16 == 0 && ld_grad % 16 == 0 &&
        ((uintptr_t)geom->x | (uintptr_t)grad_out | (uintptr_t)grad_in) % 32 == 0 &&
        geom->rows * (geom->cols / 32) < (int64_t)UINT32_MAX &&
        (geom->scale_mode == MXFP4_SCALE_FLOOR ||
         (geom->scale_mode == MXFP4_SCALE_PAGE && page_fast_ok(geom->scale_factor)))) {
        // saved-free, row-wise, bf16 block 32: one streaming pass over x and grad_out
        KArgs k;
        memset(&k, 0, sizeof(k));
        k.x = geom->x;
        k.rows = geom->rows;
        k.cols = geom->cols;
        k.ld = geom->ld;
        k.sf = geom->scale_factor;
        k.mode = geom->scale_mode;
        k.g_out = grad_out;
        k.g_in = grad_in;
        k.ld_g = ld_grad;
        if (k.mode == MXFP4_SCALE_PAGE)
            k.thr = page_threshold(geom->scale_factor);
        const void* fn = k.mode == MXFP4_SCALE_FLOOR ? (const void*)ste_row_kernel<MXFP4_SCALE_FLOOR>
                                                      : (const void*)ste_row_kernel<MXFP4_SCALE_PAGE>;
        const int sms = device_sms();
        const int occ = occupancy(fn, 0);
        if (sms <= 0 || occ <= 0)
            return MXFP4_ECUDA;
        const int64_t blocks = geom->rows * (geom->cols / 32);
        int64_t grid = (int64_t)sms * occ;
        if ((blocks + NTHREADS - 1) / NTHREADS < grid)
            grid = (blocks + NTHREADS - 1) / NTHREADS;
        if (k.mode == MXFP4_SCALE_FLOOR)
            ste_row_kernel<MXFP4_SCALE_FLOOR><<<(unsigned)grid, NTHREADS, 0, s>>>(k);
        else
            ste_row_kernel<MXFP4_SCALE_PAGE><<<(unsigned)grid, NTHREADS, 0, s>>>(k);
        return cudaGetLastError() == cudaSuccess ? MXFP4_OK : MXFP4_ECUDA;
    }
    if (clip_grad && !saved_mask) {
        // saved-free: recompute the saturation of x in the same pass
        mxfp4_qdq_args g = *geom;
        g.y_row = g.y_col = nullptr;
        g.codes_row = g.scales_row = g.mask_row = nullptr;
        g.codes_col = g.scales_col = g.mask_col = nullptr;
        return run_qdq(&g, grad_out, grad_in, ld_grad, geom->dirs, s);
    }
    if (!clip_grad && grad_in == grad_out)
        return MXFP4_OK;
    const int vec = (((uintptr_t)grad_out | (uintptr_t)grad_in) % 16 == 0) && (ld_grad % 8 == 0) &&
                    (geom->cols % 8 == 0);
    const int64_t units = geom->rows * ((geom->cols + 7) / 8);
    const uint8_t* m = clip_grad ? saved_mask : nullptr;
    const int sms = device_sms();
    if (sms <= 0)
        return MXFP4_ECUDA;
    const void* fn = esz == 2 ? (const void*)ste_mask_kernel<2> : (const void*)ste_mask_kernel<4>;
    const int occ = occupancy(fn, 0);
    if (occ <= 0)
        return MXFP4_ECUDA;
    int64_t grid = (int64_t)sms * occ;
    const int64_t need = (units + NTHREADS - 1) / NTHREADS;
    if (need < grid)
        grid = need;
    if (esz == 2)
        ste_mask_kernel<2><<<(unsigned)grid, NTHREADS, 0, s>>>(geom->rows, geom->cols, grad_out, grad_in,
                                                              ld_grad, m, vec);
    else
        ste_mask_kernel<4><<<(unsigned)grid, NTHREADS, 0, s>>>(geom->rows, geom->cols, grad_out, grad_in,
                                                              ld_grad, m, vec);
    return cudaGetLastError() == cudaSuccess ? MXFP4_OK : MXFP4_ECUDA;
}

int64_t mxfp4_colwise_scale_rows(const int64_t* host_group_list, int64_t num_groups,
                                 int32_t group_list_type, int64_t rows, int32_t block)
{
    if (block <= 0 || rows < 0)
        return -1;
    if (!host_group_list)
        return (rows + block - 1) / block;
    if (num_groups < 1 || (group_list_type != 0 && group_list_type != 1))
        return -1;
    int64_t total = 0, prev = 0, s = 0;
    for (int64_t g = 0; g < num_groups; ++g) {
        const int64_t v = host_group_list[g];
        const int64_t n = group_list_type == 1 ? v : v - prev;
        prev = v;
        if (n < 0 || n > rows)
            return -1;
        total += n;
        s += (n + block - 1) / block;
    }
    return total == rows ? s : -1;
}

int64_t mxfp4_colwise_scale_rows_bound(int64_t rows, int64_t num_groups, int32_t block)
{
    if (block <= 0 || rows < 0)
        return -1;
    if (num_groups <= 0)
        return (rows + block - 1) / block;
    return rows / block + num_groups;
}

const char* mxfp4_status_string(mxfp4_status status)
{
    switch (status) {
    case MXFP4_OK: return "ok";
    case MXFP4_EINVAL: return "invalid argument";
    case MXFP4_EUNSUPPORTED: return "unsupported argument";
    case MXFP4_ECUDA: return "CUDA error";
    }
    return "unknown status";
}

int64_t mxfp4_scales_row_bytes(int64_t rows, int64_t cols, int32_t block, int32_t layout)
{
    if (rows < 0 || cols < 0 || block <= 0)
        return -1;
    const int64_t nblk = (cols + block - 1) / block;
    if (layout == MXFP4_SCALES_ROWMAJOR)
        return rows * nblk;
    if (layout == MXFP4_SCALES_MMA)
        return 512 * ((rows + 127) / 128) * ((nblk + 3) / 4);
    return -1;
}

int64_t mxfp4_colwise_operand_k(const int64_t* host_group_list, int64_t num_groups, int32_t group_list_type,
                                int64_t rows)
{
    if (rows < 0)
        return -1;
    if (!host_group_list)
        return OP_KPAD * ((rows + OP_KPAD - 1) / OP_KPAD);
    if (num_groups < 1 || (group_list_type != 0 && group_list_type != 1))
        return -1;
    int64_t total = 0, prev = 0, k = 0;
    for (int64_t g = 0; g < num_groups; ++g) {
        const int64_t v = host_group_list[g];
        const int64_t n = group_list_type == 1 ? v : v - prev;
        prev = v;
        if (n < 0 || n > rows)
            return -1;
        total += n;
        k += OP_KPAD * ((n + OP_KPAD - 1) / OP_KPAD);
    }
    return total == rows ? k : -1;
}

int64_t mxfp4_colwise_operand_k_bound(int64_t rows, int64_t num_groups)
{
    if (rows < 0)
        return -1;
    if (num_groups <= 0)
        return OP_KPAD * ((rows + OP_KPAD - 1) / OP_KPAD);
    return OP_KPAD * (rows / OP_KPAD + num_groups);
}

int64_t mxfp4_colwise_operand_scale_bytes(int64_t cols, int64_t k_alloc)
{
    if (cols < 0 || k_alloc < 0 || k_alloc % OP_KPAD != 0)
        return -1;
    return 512 * ((cols + 127) / 128) * (k_alloc / OP_KPAD);
}

mxfp4_status mxfp4_dual_level_qdq(const mxfp4_dual_level_args* args, mxfp4_stream_t stream)
{
    return run_dual_level(args, reinterpret_cast<cudaStream_t>(stream));
}

mxfp4_status mxfp4_grouped_gemm(const mxfp4_gmm_args* args, mxfp4_stream_t stream)
{
    return run_gmm(args, reinterpret_cast<cudaStream_t>(stream));
}

int32_t mxfp4_abi_version(void) { return MXFP4_ABI_VERSION; }

}  // extern "C"
