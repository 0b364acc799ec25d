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
// Work layout: a warp owns one level-0 block of a row (a "unit", 1 KB of
// bf16). Grid-stride over units, consecutive warps on consecutive units, so
// that the grid streams through memory in order; each warp copies its next
// units into a private shared-memory ring (cp.async) while it works on the
// current one.
//
// Two element paths. The fast path (dual_unit_fast: full, aligned units
// whose level-1 scales are at most 1, which covers every block at the default
// scale factor 6) gives lane l the 16 consecutive elements 16l..16l+15, half
// of one level-1 block (the other half is lane l ^ 1): the level-0 amax is a
// packed 16-bit max, one shuffle and one warp reduction; s0 and 1/s0 come
// from a table; y = |x| / s0 is a corrected reciprocal product in packed
// f32x2 arithmetic (dl_div's steps); the level-1 scale is computed once per
// lane from the quotient of the block's max |x|; floor(4 |y| 2^-k1) indexes a
// 64-entry code table; the E2M1 nibbles come from the hardware convert of
// the exact signed codes and the output from one or two fp32 multiplies. It
// stores nothing before it has decided to handle the unit. The general path
// (dual_unit: lane l holds elements 8l..8l+7 of each 256-element half, a
// level-1 block is four lanes) takes every other unit: ragged or unaligned
// ones, non-finite or tiny level-0 blocks, level-1 scales above 1 (small
// PAGE scale factors); it divides with dl_div or IEEE division and quantises
// each element with the single-level element routine.

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
    int32_t vec;   // full units may use 16-byte loads / stores (host-checked alignment)
    int32_t fast;  // the fast path's scale rule is available (FLOOR, or PAGE with thr)
    uint32_t thr;  // PAGE mode: fp32 bits of the qparams threshold T0
    // 4 and 65536 (set by the host): multiply-adds by these run-time values
    // stay on the multiply-add pipe instead of becoming shifts
    uint32_t mul4, mul16;
    int64_t nb0, nb1, cstride, mstride, units;
};

// fl32(x / s0) for one element, given r = fl32(1 / s0): q = fl(x r), the
// residual e = x - q s0 (exact, by one fma) and fl(q + e r). For bf16 x with
// |x| >= 2^-102 and |q| >= 2^-124 this is the IEEE quotient for every bf16
// level-0 amax (an exhaustive CPU replay of these steps checks every pair);
// x = +-0 gives +0, which quantises exactly as -0 does; an element outside
// those bounds is flagged `slow` and takes the IEEE division instead.
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

typedef unsigned long long u64;

__device__ __forceinline__ u64 pk2(float lo, float hi)
{
    u64 d;
    asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(lo), "f"(hi));
    return d;
}

__device__ __forceinline__ void upk2(u64 v, float& lo, float& hi)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}

__device__ __forceinline__ u64 mul2(u64 a, u64 b)
{
    u64 d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

__device__ __forceinline__ u64 fma2(u64 a, u64 b, u64 c)
{
    u64 d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

__device__ __forceinline__ u64 fma2_rm(u64 a, u64 b, u64 c)
{
    u64 d;
    asm("fma.rm.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

__device__ __forceinline__ uint32_t vmin2(uint32_t a, uint32_t b)
{
    uint32_t r;
    asm("min.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// y = fl32(x / s0) of one value, r = fl32(1 / s0): the corrected reciprocal
// product where |x| >= tf (dl_div's conditions hold), the IEEE quotient
// otherwise.
__device__ __forceinline__ float dl_quot(float x, float s0, float r, float tf)
{
    if (fabsf(x) >= tf) {
        const float q = __fmul_rn(x, r);
        return __fmaf_rn(__fmaf_rn(-q, s0, x), r, q);
    }
    return __fdiv_rn(x, s0) + 0.0f;
}

// Fast path of one full, aligned unit. The lane holds w = elements
// 16 lane .. 16 lane + 15 of the unit (8 bf16 pairs): half of one level-1
// block, whose other half is the neighbouring lane. Returns false, having
// stored nothing, when the unit needs dual_unit; the decision is uniform
// across the warp.
//
// s0 = fl32(a0 / 6) and r = fl32(1 / s0) come from a table over the seven
// significand bits of the bf16 amax a0 (entries for a0 in [1, 2)), shifted by
// a0's exponent: both roundings commute with power-of-two scaling while the
// results stay normal, which holds for every a0 >= 2^-65 taken here. The
// quotients are formed from |x| (the sign is put back on the code), so
// |y| = fl32(|x| / s0) feeds both the floor and the saturation test. The
// level-1 amax is taken on x: fl32(|x| / s0) is a monotone function of |x|,
// so max |y| over a block is the quotient of max |x|. floor(4 |y 2^-k1|)
// comes from one packed fma rounding down into 2^21, where the fp32 spacing
// is 1/4 (y 2^-k1 is exact: 2^-k1 >= 1 on this path, and |y 2^-k1| < 16);
// the table entry at that index is the code magnitude. Elements whose y is
// zero (x = +-0, or a quotient that underflows) get a +0 code, as sign(y) = 0
// there. The output is (code * A) * B with (A, B) = (2^k1 s0, 1) when that
// product is a normal number (so exact), else (2^k1, s0).
__device__ __forceinline__ bool dual_unit_fast(const DualArgs& a, int row, int j, int lane, const uint32_t (&w)[8],
                                               uint32_t lutb, const float2* s0r)
{
    uint32_t aw[8], m = 0u, mn = 0x7FFF7FFFu;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        aw[i] = w[i] & 0x7FFF7FFFu;
        m = vmax2(m, aw[i]);
        mn = vmin2(mn, aw[i]);
    }
    uint32_t mb = max(m & 0xFFFFu, m >> 16);
    mb = max(mb, __shfl_xor_sync(FULL, mb, 1));  // the level-1 block's max |x| (bf16 bits)
    const uint32_t A0 = __reduce_max_sync(FULL, mb);
    if (A0 >= 0x7F80u || A0 < 0x1F00u)  // non-finite, or a0 < 2^-65 (tiny or all-zero block)
        return false;
    const float2 t0 = s0r[A0 & 0x7Fu];
    const uint32_t esh = ((A0 >> 7) - 127u) << 23;
    const float s0 = __uint_as_float(__float_as_uint(t0.x) + esh);
    const float r = __uint_as_float(__float_as_uint(t0.y) - esh);
    // |x| >= tf meets both conditions under which the corrected reciprocal
    // product is the IEEE quotient (|x| >= 2^-102, |x r| >= 2^-124); s0 2^-123
    // is exact whenever it exceeds 2^-102. tb: tf rounded up to bf16 bits.
    const float tf = fmaxf(0x1p-102f, s0 * 0x1p-123f);
    const uint32_t tb = (__float_as_uint(tf) + 0xFFFFu) >> 16;
    // a lane with an |x| below tf (zeros included) checks its elements one by one
    const bool lane_slow = min(mn & 0xFFFFu, mn >> 16) < tb;

    const QP p = qparams(__float_as_uint(dl_quot(__uint_as_float(mb << 16), s0, r, tf)), a.mode, a.thr);
    if (__any_sync(FULL, !(p.inv >= 1.0f)))  // a level-1 scale above 1: y * 2^-k1 may round
        return false;
    const float S = p.scale * s0;
    const bool exact = S >= 0x1p-126f;  // 2^k1 s0 normal, hence exact

    const u64 R2 = pk2(r, r), NS2 = pk2(-s0, -s0);
    u64 Y[8];
    uint32_t sg[8];  // sign sources: x with -0 turned into +0
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const u64 X = pk2(__uint_as_float(aw[i] * a.mul16), __uint_as_float(aw[i] & 0xFFFF0000u));
        const u64 Q = mul2(X, R2);
        Y[i] = fma2(fma2(Q, NS2, X), R2, Q);
        sg[i] = clear_neg_zero(w[i]);
    }
    if (lane_slow) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            float ylo, yhi;
            upk2(Y[i], ylo, yhi);
            const uint32_t alo = aw[i] & 0xFFFFu, ahi = aw[i] >> 16;
            if (alo - 1u < tb - 1u) {  // 0 < |x| < tf: the IEEE quotient; an underflow to 0 drops the sign
                ylo = __fdiv_rn(__uint_as_float(alo << 16), s0);
                if (ylo == 0.0f)
                    sg[i] &= 0xFFFF7FFFu;
            }
            if (ahi - 1u < tb - 1u) {
                yhi = __fdiv_rn(__uint_as_float(ahi << 16), s0);
                if (yhi == 0.0f)
                    sg[i] &= 0x7FFFFFFFu;
            }
            Y[i] = pk2(ylo, yhi);
        }
    }

    const u64 INV2 = pk2(p.inv, p.inv);
    const u64 A2 = exact ? pk2(S, S) : pk2(p.scale, p.scale);
    const u64 B2 = exact ? pk2(1.0f, 1.0f) : pk2(s0, s0);
    const uint32_t lim = __float_as_uint(p.scale * 6.0f);  // exact: 2^k1 >= 2^-127
    uint32_t ob[8], sats = 0;
    float cv[16];
#pragma unroll
    for (int i = 7; i >= 0; --i) {
        float ylo, yhi;
        upk2(Y[i], ylo, yhi);
        float tlo, thi;
        upk2(fma2_rm(Y[i], INV2, pk2(2097152.0f, 2097152.0f)), tlo, thi);
        uint32_t elo, ehi;
        asm("ld.shared.u32 %0, [%1];" : "=r"(elo) : "r"(__float_as_uint(tlo) * a.mul4 + lutb));
        asm("ld.shared.u32 %0, [%1];" : "=r"(ehi) : "r"(__float_as_uint(thi) * a.mul4 + lutb));
        cv[2 * i] = __uint_as_float(elo | ((sg[i] * a.mul16) & 0x80000000u));
        cv[2 * i + 1] = __uint_as_float(ehi | (sg[i] & 0x80000000u));
        float olo, ohi;
        upk2(mul2(mul2(pk2(cv[2 * i], cv[2 * i + 1]), A2), B2), olo, ohi);
        asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(ob[i]) : "f"(ohi), "f"(olo));
        // saturation |y| > 6 * 2^k1: the sign of lim - |y|, element 2i + 1 first
        sats = (sats << 1) | ((lim - __float_as_uint(yhi)) >> 31);
        sats = (sats << 1) | ((lim - __float_as_uint(ylo)) >> 31);
    }
    const int64_t c = (int64_t)j * DL_BLOCK0 + 16 * lane;
    if (a.y) {
        uint16_t* yp = a.y + (int64_t)row * a.ld_y + c;
        st_stream(yp, make_uint4(ob[0], ob[1], ob[2], ob[3]));
        st_stream(yp + 8, make_uint4(ob[4], ob[5], ob[6], ob[7]));
    }
    if (a.codes) {
        const float (&c0)[8] = *reinterpret_cast<const float(*)[8]>(&cv[0]);
        const float (&c1)[8] = *reinterpret_cast<const float(*)[8]>(&cv[8]);
        *reinterpret_cast<uint2*>(a.codes + (int64_t)row * a.cstride + c / 2) = make_uint2(e2m1x8(c0), e2m1x8(c1));
    }
    if (a.mask)
        *reinterpret_cast<uint16_t*>(a.mask + (int64_t)row * a.mstride + c / 8) = (uint16_t)sats;
    if ((lane & 1) == 0 && a.s1)
        a.s1[(int64_t)row * a.nb1 + c / 32] = (uint8_t)qp_e8(p);
    if (lane == 0 && a.s0)
        a.s0[(int64_t)row * a.nb0 + j] = s0;
    return true;
}

// Each warp streams its units through a private ring of DL_STAGES 1 KB
// stages in shared memory: every lane copies its own 32 bytes of a unit with
// cp.async, DL_STAGES - 1 units ahead of the one it works on, and later reads
// back only what it copied itself, so no barrier is needed (a lane's
// wait_group makes its own copies visible to it). The copies in flight per SM
// do not depend on how many registers the element work needs.
constexpr int DL_STAGES = 4;

__device__ __forceinline__ void dl_cp16(uint32_t saddr, const void* g)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(saddr), "l"(g) : "memory");
}

__device__ __forceinline__ void dl_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

__device__ __forceinline__ void dl_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(DL_STAGES - 1) : "memory"); }

__global__ void __launch_bounds__(NTHREADS) dual_level_kernel(const DualArgs a)
{
    __shared__ uint32_t s_lut[64];
    __shared__ float2 s_s0r[128];  // (fl32(a0 / 6), fl32(1 / that)) for a0 = 1 + i / 128
    __shared__ __align__(16) uint4 s_ring[NTHREADS / 32][DL_STAGES][64];
    if (threadIdx.x < 64)
        s_lut[threadIdx.x] = lut_entry(threadIdx.x);
    if (threadIdx.x < 128) {
        const float s0 = __fdiv_rn(__uint_as_float((0x3F80u + threadIdx.x) << 16), 6.0f);
        s_s0r[threadIdx.x] = make_float2(s0, __frcp_rn(s0));
    }
    __syncthreads();
    // table address of t = 2^21 + floor(4|y|) / 4: base + 4 (bits(t) - 0x4A000000)
    const uint32_t lutb = (uint32_t)__cvta_generic_to_shared(s_lut) - 0x28000000u;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t ring = (uint32_t)__cvta_generic_to_shared(&s_ring[warp][0][2 * lane]);
    // units u = row * nb0 + j (rows and nb0 below 2^30, host-checked); warp w
    // takes u = w, w + nwarps, ...; (row, j) advance by (drow, dj) with a carry
    const int nb0 = (int)a.nb0, rows = (int)a.rows;
    const int64_t nwarps = (int64_t)gridDim.x * (NTHREADS / 32);
    const int64_t u0 = (int64_t)blockIdx.x * (NTHREADS / 32) + warp;
    const int drow = (int)(nwarps / nb0), dj = (int)(nwarps % nb0);
    // units j < j_full are full and aligned: they take the ring and the fast path
    const int j_full = a.fast && a.vec ? (int)(a.cols / DL_BLOCK0) : 0;
    auto advance = [&](int& rr, int& jj) {
        rr += drow;
        jj += dj;
        if (jj >= nb0) {
            jj -= nb0;
            rr += 1;
        }
    };
    auto issue = [&](int rr, int jj, int st) {
        if (rr < rows && jj < j_full) {
            const uint16_t* g = a.x + (int64_t)rr * a.ld + jj * DL_BLOCK0 + 16 * lane;
            const uint32_t sa = ring + (uint32_t)st * 1024u;
            dl_cp16(sa, g);
            dl_cp16(sa + 16u, g + 8);
        }
        dl_commit();  // one group per unit, empty or not, so that the counting stays uniform
    };
    int row = (int)(u0 / nb0), j = (int)(u0 % nb0);  // the unit worked on (u0 < rows * nb0 when row < rows)
    int rp = row, jp = j;                            // the next unit to copy
    if (u0 >= (int64_t)rows * nb0)
        return;
#pragma unroll
    for (int st = 0; st < DL_STAGES - 1; ++st) {
        issue(rp, jp, st);
        advance(rp, jp);
    }
    for (int st = 0; row < rows; st = st + 1 == DL_STAGES ? 0 : st + 1) {
        issue(rp, jp, st == 0 ? DL_STAGES - 1 : st - 1);  // the stage used one unit ago
        advance(rp, jp);
        dl_wait();
        bool done = false;
        if (j < j_full) {
            const uint32_t sa = ring + (uint32_t)st * 1024u;
            uint32_t w[8];
            asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
                         : "r"(sa));
            asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(w[4]), "=r"(w[5]), "=r"(w[6]), "=r"(w[7])
                         : "r"(sa + 16u));
            done = dual_unit_fast(a, row, j, lane, w, lutb, s_s0r);
        }
        if (!done) {
            if (a.vec && (int64_t)(j + 1) * DL_BLOCK0 <= a.cols)
                dual_unit<true>(a, row, j, lane);
            else
                dual_unit<false>(a, row, j, lane);
        }
        advance(row, j);
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
    if (A->dtype != MXFP4_BF16 || A->level0_block != DL_BLOCK0 || A->rows >= (1 << 30) || A->cols >= (1 << 30))
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
    k.mul4 = 4;
    k.mul16 = 65536;
    k.fast = A->scale_mode == MXFP4_SCALE_FLOOR || page_fast_ok(A->scale_factor);
    k.thr = A->scale_mode == MXFP4_SCALE_PAGE && k.fast ? page_threshold(A->scale_factor) : 0u;
    // full units take 16-byte loads and y stores, 8-byte code stores and
    // 2-byte mask stores
    k.vec = aligned(A->x, 16) && A->ld % 8 == 0 && A->cols % 16 == 0 &&
            (!A->y || (aligned(A->y, 16) && A->ld_y % 8 == 0)) && (!A->codes || aligned(A->codes, 8)) &&
            (!A->mask || aligned(A->mask, 2));
    const int sms = device_sms();
    const int occ = occupancy((const void*)dual_level_kernel, 0);
    if (sms <= 0 || occ <= 0)
        return MXFP4_ECUDA;
    const int64_t need = (k.units + NTHREADS / 32 - 1) / (NTHREADS / 32);
    const int64_t grid = need < (int64_t)sms * occ ? need : (int64_t)sms * occ;
    dual_level_kernel<<<(unsigned)grid, NTHREADS, 0, s>>>(k);
    return cudaGetLastError() == cudaSuccess ? MXFP4_OK : MXFP4_ECUDA;
}
