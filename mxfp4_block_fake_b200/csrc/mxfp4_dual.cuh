// mxfp4_dual.cuh -- dual-level MX quantisation (included by mxfp4.cu).
//
// sglang mxfp4_npu.py, NPUMXFP4DiffusionLinearMethod, quantises weights and
// activations with npu_dynamic_dual_level_mx_quant into E2M1 codes, a
// level-0 scale per level0_block elements of a row and a level-1 scale; the
// page names the operator and its results only. The reading implemented
// here: per level-0 block of 512 elements, s0 = fl32(amax0 / 6) (1 for an
// all-zero block); y = fl32(x / s0); y is quantised like one row of the
// MXFP4 QDQ of amct pull request 264 (mxfp4_qat/fake_quant.py) with blocks
// of 32; the output is fl32(code 2^k1 s0) in bf16. A level-0 block holding a
// NaN or an infinity is written as NaN (code 0, E8M0 0xFF, s0 NaN).
//
// Work layout: a warp owns one level-0 block of a row (a "unit"). Lane l
// holds elements 8l..8l+7 of each 256-element half, so each of the warp's two
// 16-byte loads (and the 16-byte stores of y) covers 512 contiguous bytes, and
// a level-1 block of 32 is four neighbouring lanes of one half. Per unit:
// level-0 amax by one warp reduction, s0 and its reciprocal, y = x / s0 by a
// corrected reciprocal product (dl_div), the level-1 amax by two shuffles,
// the scale and codes as in the single-level kernels, the output as one more
// fp32 multiply. Grid-stride over units, consecutive warps on consecutive
// units, so that the grid streams through memory in order.

constexpr int DL_BLOCK0 = 512;

struct DualArgs {
    const uint16_t* x;
    int64_t rows, cols, ld;
    uint16_t* y;
    int64_t ld_y;
    uint8_t* codes;
    float* s0;
    uint8_t* s1;
    uint8_t* mask;
    float sf;
    int32_t mode;
    int32_t vec;  // full units may use 16-byte loads / stores (host-checked alignment)
    int64_t nb0, nb1, cstride, mstride, units;
};

// fl32(x / s0) for one element, given r = fl32(1 / s0): q = fl(x r), the
// residual e = x - q s0 (exact, by one fma) and fl(q + e r). For bf16 x with
// |x| >= 2^-102 and |q| >= 2^-124 this is the IEEE quotient for every bf16
// level-0 amax (an exhaustive CPU replay of these steps checks every pair);
// x = +-0 gives +0, which quantises exactly as -0 does; every other element
// is flagged `slow` and takes the IEEE division instead.
__device__ __forceinline__ float dl_div(float x, float s0, float r, bool& slow)
{
    const float q = __fmul_rn(x, r);
    const float e = __fmaf_rn(-q, s0, x);
    const float y = __fmaf_rn(e, r, q);
    const float ax = fabsf(x);
    slow = ax != 0.0f && !(ax >= 0x1p-102f && fabsf(q) >= 0x1p-124f);
    return ax == 0.0f ? 0.0f : y;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

template <bool VEC>
__device__ __forceinline__ void dual_unit(const DualArgs& a, int64_t row, int64_t j, int lane)
{
    const int64_t c0 = j * DL_BLOCK0;
    const uint16_t* xr = a.x + row * a.ld;
    uint32_t w[2][4];  // bf16 pairs, element 2i in the low half
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int64_t c = c0 + 256 * h + 8 * lane;
        if (VEC) {
            const uint4 v = ld_stream(xr + c);
            w[h][0] = v.x;
            w[h][1] = v.y;
            w[h][2] = v.z;
            w[h][3] = v.w;
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint32_t lo = c + 2 * i < a.cols ? xr[c + 2 * i] : 0u;
                const uint32_t hi = c + 2 * i + 1 < a.cols ? xr[c + 2 * i + 1] : 0u;
                w[h][i] = lo | (hi << 16);
            }
        }
    }
    // level-0 amax: integer max of the sign-cleared bf16 bits (padding is +0,
    // which never raises it; NaN bits exceed those of inf)
    uint32_t m = 0;
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int i = 0; i < 4; ++i)
            m = vmax2(m, w[h][i] & 0x7FFF7FFFu);
    const uint32_t A0 = __reduce_max_sync(FULL, max(m & 0xFFFFu, m >> 16));
    const int64_t s1_row = row * a.nb1 + c0 / 32;

    if (A0 >= 0x7F80u) {  // non-finite level-0 block
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int64_t c = c0 + 256 * h + 8 * lane;
            if (VEC) {
                if (a.y)
                    st_stream(a.y + row * a.ld_y + c, make_uint4(0x7FC07FC0u, 0x7FC07FC0u, 0x7FC07FC0u, 0x7FC07FC0u));
                if (a.codes)
                    *reinterpret_cast<uint32_t*>(a.codes + row * a.cstride + c / 2) = 0u;
                if (a.mask)
                    a.mask[row * a.mstride + c / 8] = 0;
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    if (c + i < a.cols && a.y)
                        a.y[row * a.ld_y + c + i] = 0x7FC0;
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    if (c + 2 * i < a.cols && a.codes)
                        a.codes[row * a.cstride + c / 2 + i] = 0;
                if (c < a.cols && a.mask)
                    a.mask[row * a.mstride + c / 8] = 0;
            }
            const int64_t cb = c0 + 256 * h + 32 * (lane >> 2);
            if ((lane & 3) == 0 && cb < a.cols && a.s1)
                a.s1[s1_row + 8 * h + (lane >> 2)] = 0xFF;
        }
        if (lane == 0 && a.s0)
            a.s0[row * a.nb0 + j] = __uint_as_float(QNAN32);
        return;
    }

    float s0 = __fdiv_rn(__uint_as_float(A0 << 16), 6.0f);
    if (s0 == 0.0f)
        s0 = 1.0f;
    const float r = __frcp_rn(s0);
    uint32_t yb[2][8];
    uint32_t slow = 0;
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            bool sl;
            const float xv = (i & 1) ? bf16_hi(w[h][i >> 1]) : bf16_lo(w[h][i >> 1]);
            yb[h][i] = __float_as_uint(dl_div(xv, s0, r, sl));
            slow |= (sl ? 1u : 0u) << (8 * h + i);
        }
    if (slow) {
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int i = 0; i < 8; ++i)
                if ((slow >> (8 * h + i)) & 1u) {
                    const float xv = (i & 1) ? bf16_hi(w[h][i >> 1]) : bf16_lo(w[h][i >> 1]);
                    yb[h][i] = __float_as_uint(__fdiv_rn(xv, s0));
                }
    }

#pragma unroll
    for (int h = 0; h < 2; ++h) {
        uint32_t A1 = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i)
            A1 = max(A1, yb[h][i] & 0x7FFFFFFFu);
        A1 = max(A1, __shfl_xor_sync(FULL, A1, 1));
        A1 = max(A1, __shfl_xor_sync(FULL, A1, 2));
        const BP p = block_params(A1, a.mode, a.sf);
        uint32_t ob[8], nibs = 0, sats = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            uint32_t nib, sat;
            const uint32_t o = qdq_elem(yb[h][i], p, nib, sat);
            ob[i] = round_bf16_bits(__float_as_uint(__fmul_rn(__uint_as_float(o), s0))) >> 16;
            nibs |= nib << (4 * i);
            sats |= sat << i;
        }
        const int64_t c = c0 + 256 * h + 8 * lane;
        if (VEC) {
            if (a.y)
                st_stream(a.y + row * a.ld_y + c, make_uint4(ob[0] | (ob[1] << 16), ob[2] | (ob[3] << 16),
                                                             ob[4] | (ob[5] << 16), ob[6] | (ob[7] << 16)));
            if (a.codes)
                *reinterpret_cast<uint32_t*>(a.codes + row * a.cstride + c / 2) = nibs;
            if (a.mask)
                a.mask[row * a.mstride + c / 8] = (uint8_t)sats;
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i)
                if (c + i < a.cols && a.y)
                    a.y[row * a.ld_y + c + i] = (uint16_t)ob[i];
#pragma unroll
            for (int i = 0; i < 4; ++i)
                if (c + 2 * i < a.cols && a.codes)
                    a.codes[row * a.cstride + c / 2 + i] = (uint8_t)(nibs >> (8 * i));
            if (c < a.cols && a.mask)
                a.mask[row * a.mstride + c / 8] = (uint8_t)sats;
        }
        const int64_t cb = c0 + 256 * h + 32 * (lane >> 2);
        if ((lane & 3) == 0 && cb < a.cols && a.s1)
            a.s1[s1_row + 8 * h + (lane >> 2)] = (uint8_t)p.e8;
    }
    if (lane == 0 && a.s0)
        a.s0[row * a.nb0 + j] = s0;
}

__global__ void __launch_bounds__(NTHREADS) dual_level_kernel(const DualArgs a)
{
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = (int64_t)gridDim.x * (NTHREADS / 32);
    for (int64_t u = (int64_t)blockIdx.x * (NTHREADS / 32) + (threadIdx.x >> 5); u < a.units; u += nwarps) {
        const int64_t row = u / a.nb0, j = u - row * a.nb0;
        if (a.vec && (j + 1) * DL_BLOCK0 <= a.cols)
            dual_unit<true>(a, row, j, lane);
        else
            dual_unit<false>(a, row, j, lane);
    }
}

static mxfp4_status run_dual_level(const mxfp4_dual_level_args* A, cudaStream_t s)
{
    if (!A || A->rows < 0 || A->cols < 0)
        return MXFP4_EINVAL;
    if (A->dtype != MXFP4_F32 && A->dtype != MXFP4_BF16)
        return MXFP4_EINVAL;
    if (A->level0_block <= 0 || A->level0_block % 32 != 0)
        return MXFP4_EINVAL;
    if (!(A->scale_factor > 0.0f) || !isfinite(A->scale_factor))
        return MXFP4_EINVAL;
    if (A->scale_mode != MXFP4_SCALE_PAGE && A->scale_mode != MXFP4_SCALE_FLOOR)
        return MXFP4_EINVAL;
    if (A->dtype != MXFP4_BF16 || A->level0_block != DL_BLOCK0)
        return MXFP4_EUNSUPPORTED;
    if (A->rows == 0 || A->cols == 0)
        return MXFP4_OK;
    if (!A->x || A->ld < A->cols || (A->y && A->ld_y < A->cols))
        return MXFP4_EINVAL;
    DualArgs k;
    k.x = static_cast<const uint16_t*>(A->x);
    k.rows = A->rows;
    k.cols = A->cols;
    k.ld = A->ld;
    k.y = static_cast<uint16_t*>(A->y);
    k.ld_y = A->ld_y;
    k.codes = A->codes;
    k.s0 = A->scales0;
    k.s1 = A->scales1;
    k.mask = A->mask;
    k.sf = A->scale_factor;
    k.mode = A->scale_mode;
    k.nb0 = (A->cols + DL_BLOCK0 - 1) / DL_BLOCK0;
    k.nb1 = (A->cols + 31) / 32;
    k.cstride = (A->cols + 1) / 2;
    k.mstride = (A->cols + 7) / 8;
    k.units = A->rows * k.nb0;
    k.vec = aligned(A->x, 16) && A->ld % 8 == 0 && A->cols % 8 == 0 &&
            (!A->y || (aligned(A->y, 16) && A->ld_y % 8 == 0)) && (!A->codes || aligned(A->codes, 4));
    const int sms = device_sms();
    const int occ = occupancy((const void*)dual_level_kernel, 0);
    if (sms <= 0 || occ <= 0)
        return MXFP4_ECUDA;
    const int64_t need = (k.units + NTHREADS / 32 - 1) / (NTHREADS / 32);
    const int64_t grid = need < (int64_t)sms * occ ? need : (int64_t)sms * occ;
    dual_level_kernel<<<(unsigned)grid, NTHREADS, 0, s>>>(k);
    return cudaGetLastError() == cudaSuccess ? MXFP4_OK : MXFP4_ECUDA;
}
