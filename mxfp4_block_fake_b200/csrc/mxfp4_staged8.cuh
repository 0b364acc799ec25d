// mxfp4_staged8.cuh -- MXFP8 (E4M3 elements, E8M0 scales per 32) for bf16,
// column-wise or both directions from one read of each tile (included by
// mxfp4.cu after mxfp4_staged.cuh; shares their helpers).
//
// Tiles and loads as in the block-32 staged kernel: 32 rows (one column-wise
// block, shorter at a group tail) by 256 columns, brought in by TMA as four
// 64 x 32 boxes with the 128-byte swizzle, every G-th tile per CTA. The CTA has eight compute warps and one producer warp. The
// compute warps release a tile with one arrival each on its stage's "empty"
// mbarrier; the producer warp then stores the tile's row-wise outputs (TMA,
// one bulk group per tile), copies what TMA cannot address, and once the
// stores of the tile before have read their sources, releases that tile's
// staging buffer ("sfree") and refills its stage. No CTA barrier orders the
// tiles.
//
// Compute warp w owns tile columns 32w..32w+31 in both passes:
//   * column pass: lane = column pair p (lane & 15) x row half h (lane >> 4)
//     over rows 8i + 4h + q (i, q = 0..3), the conflict-free pattern of the
//     MXFP4 kernel; the amax takes one shuffle. y (one word per row) and the
//     E4M3 code pair (two bytes per row) are stored straight to global
//     memory (a half-warp writes 64 contiguous bytes of y and 32 of codes per
//     row), rows of the block only;
//   * row pass: lane = tile row, over the warp's 32 columns: y written over
//     the tile's own input words, the 32 code bytes, the row-wise and the
//     column-wise saturation words and the scale byte into the staging
//     buffer. Every row of the tile is computed, group tail or not (a row's
//     row-wise outputs depend on that row alone, so the rows past a group
//     tail get the values the tile owning them writes).
//
// Element arithmetic (both passes): y = x * 2^-k in fp32 (exact), the E4M3
// pair by the hardware convert (nearest even, saturating at 448, sign kept),
// the codes back to f16 by the hardware convert (exact) and times 2^k in fp32
// (exact: a code has at most four significant bits and every result is a
// multiple of the smallest bf16 subnormal, so bf16 keeps it). A block whose
// amax is inf or NaN gives NaN values, code 0, no saturation and scale 0xFF.
// Every wait on an mbarrier is bounded (SG_WAIT_NS); on expiry the CTA
// records MXFP4_ECUDA in the caller's status word (when given), waits
// (bounded) for its loads still in flight and for its stores, and returns.

namespace mxfp4 {

constexpr int S8_STAGES = 4;
constexpr int S8_COMPUTE_WARPS = SG_COLS / 32;            // 8
constexpr int S8_THREADS = 32 * (S8_COMPUTE_WARPS + 1);  // + the producer warp
constexpr int S8_PRODUCER = S8_COMPUTE_WARPS;            // its warp index

// Staged row-wise outputs of one tile (two buffers alternate): codes as two
// boxes of 128 columns (32 rows of 128 bytes, 128-byte swizzle), masks and
// scales as 32 rows of 32 and 8 bytes.
struct __align__(1024) Staged8Out {
    uint8_t crow[2][SG_ROWS * 128];
    uint32_t mrow[SG_MASK_WORDS];
    uint32_t mcol[SG_MASK_WORDS];
    uint8_t srow[SG_ROWS * 8];
};

struct __align__(1024) Staged8Smem {
    uint8_t tiles[S8_STAGES][SG_TILE_BYTES];  // input stages; row-wise y in place
    Staged8Out out[2];
    uint32_t limw[S8_COMPUTE_WARPS][16];  // per warp and column pair: 0x8000 + limit bits per half (0xFFFF: never)
    int4 info[S8_STAGES];                 // row0, nrows, col0, row block of each stage's tile
    unsigned long long full[S8_STAGES];   // stage loaded (TMA transaction count)
    unsigned long long empty[S8_STAGES];  // stage's tile finished by the eight compute warps
    unsigned long long sfree[2];          // staging buffer read by the stores of its last tile
    int err;
};

// Packed 0x8000 + bf16 bits of 448 * 2^k = 1.75 * 2^(k + 8) for a finite
// block (see sat8): an element saturates when its |x| bits exceed the limit.
__device__ __forceinline__ uint32_t lim8x(int k) { return 0x8000u + (((uint32_t)(k + 135) << 7) | 0x60u); }

// One word (low and high bf16 element) with the parameters of each element's
// block: returns the packed bf16 dequantised pair; code receives the E4M3
// pair (low element in the low byte).
__device__ __forceinline__ uint32_t q8word(uint32_t w, float inv_lo, float inv_hi, float sc_lo, float sc_hi,
                                          uint32_t& code)
{
    const float ylo = __fmul_rn(__uint_as_float(w << 16), inv_lo);
    const float yhi = __fmul_rn(__uint_as_float(w & 0xFFFF0000u), inv_hi);
    uint16_t q;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(q) : "f"(yhi), "f"(ylo));
    uint32_t hf;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(hf) : "h"(q));
    code = q;
    return dequant_pair(hf, sc_lo, sc_hi);
}

// Thread copies by the producer warp (lane = tile row) of a tile's staged
// outputs: rows at or past nrows and 32-column units at or past cols are
// skipped. which: SG_TS_* bits of the outputs to copy; row-wise scales are
// always copied (SMMA: the MMA layout, where a tile row's eight blocks are
// two 4-byte atom entries).
template <bool SMMA>
__device__ __forceinline__ void copy8(const KArgs& a, const Staged8Out& o, const uint8_t* tile, int row0, int nrows,
                                      int col0, uint32_t which, int lane)
{
    const int r = lane;
    if (r >= nrows)
        return;
    const int64_t row = (int64_t)row0 + r, mstride = a.cols / 8, nblk = a.cols / 32;
    const int nu = (int)min((int64_t)8, (a.cols - col0) / 32);  // 32-column units inside the tensor
    if (a.scales_row) {
        if constexpr (SMMA) {
            if (nu == 8 && ((uintptr_t)a.scales_row & 3) == 0) {
                const uint2 v = *reinterpret_cast<const uint2*>(o.srow + r * 8);
                *reinterpret_cast<uint32_t*>(a.scales_row + srow_off_mma(row, col0 / 32, nblk)) = v.x;
                *reinterpret_cast<uint32_t*>(a.scales_row + srow_off_mma(row, col0 / 32 + 4, nblk)) = v.y;
            } else {
                for (int b = 0; b < nu; ++b)
                    a.scales_row[srow_off_mma(row, col0 / 32 + b, nblk)] = o.srow[r * 8 + b];
            }
        } else {
            uint8_t* dst = a.scales_row + row * nblk + col0 / 32;
            if (nu == 8 && ((uintptr_t)dst & 7) == 0) {
                *reinterpret_cast<uint2*>(dst) = *reinterpret_cast<const uint2*>(o.srow + r * 8);
            } else {
                for (int b = 0; b < nu; ++b)
                    dst[b] = o.srow[r * 8 + b];
            }
        }
    }
    for (int u = 0; u < nu; ++u) {
        const int64_t c = col0 + 32 * u;
        if (which & SG_TS_MASK)
            *reinterpret_cast<uint32_t*>(a.mask_col + row * mstride + c / 8) = o.mcol[r * 8 + u];
        if (which & SG_TS_MASK_R)
            *reinterpret_cast<uint32_t*>(a.mask_row + row * mstride + c / 8) = o.mrow[r * 8 + u];
        if (which & SG_TS_CODES_R) {
            const uint8_t* cb = o.crow[u >> 2] + r * 128;
            uint4* dst = reinterpret_cast<uint4*>(a.codes_row + row * a.cols + c);
            dst[0] = sm_ld128(cb, ((2u * (u & 3)) ^ (uint32_t)(r & 7)) << 4);
            dst[1] = sm_ld128(cb, ((2u * (u & 3) + 1) ^ (uint32_t)(r & 7)) << 4);
        }
        if (which & SG_TS_YR) {
            char* dst = static_cast<char*>(a.y_row) + (row * a.ld_y + c) * 2;
#pragma unroll
            for (int jj = 0; jj < 4; ++jj)
                st_stream(dst + 16 * jj, sm_ld128(tile, (u >> 1) * SG_SLAB_BYTES + r * 128 +
                                                            (((4u * (u & 1) + jj) ^ (uint32_t)(r & 7)) << 4)));
        }
    }
}

// ROW: the row-wise direction too (the column-wise one always); GROUPS:
// column-wise blocks restart at group_list boundaries; SMMA: row-wise scales
// in the MMA layout. Requires cols % 32 == 0 (so a warp's 32 columns lie
// wholly inside or outside the tensor), 16-byte aligned y rows and row-wise
// codes, 4-byte aligned masks, 2-byte aligned column-wise codes and scales
// (the launcher checks). a.ts_flags: the row-wise outputs and the column-wise
// mask that TMA stores on full tiles (SG_TS_*); the others are copied.
template <bool ROW, bool GROUPS, bool SMMA>
__global__ void __launch_bounds__(S8_THREADS, 2) qdq_staged8_kernel(const __grid_constant__ StagedMaps maps,
                                                                    const KArgs a)
{
    extern __shared__ __align__(1024) uint8_t s_dyn[];
    uint8_t* s_base = s_dyn + ((1024u - (smem_addr(s_dyn) & 1023u)) & 1023u);
    Staged8Smem& sm = *reinterpret_cast<Staged8Smem*>(s_base);
    int32_t* s_plan = reinterpret_cast<int32_t*>(s_base + sizeof(Staged8Smem));
    int32_t* s_bpre = s_plan;
    int32_t* s_rst = s_plan + (GROUPS ? a.num_groups + 1 : 0);
    volatile int* err = &sm.err;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) {
        sm.err = 0;
        for (int s = 0; s < S8_STAGES; ++s) {
            mbar_init(smem_addr(&sm.full[s]), 1);
            mbar_init(smem_addr(&sm.empty[s]), S8_COMPUTE_WARPS);
        }
        mbar_init(smem_addr(&sm.sfree[0]), 1);
        mbar_init(smem_addr(&sm.sfree[1]), 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    uint32_t S;
    if constexpr (GROUPS) {
        const int64_t s = build_plan<SG_ROWS>(a, s_bpre, s_rst);  // contains __syncthreads
        if (blockIdx.x == 0 && tid == 0 && a.status)
            *a.status = s < 0 ? MXFP4_EINVAL : MXFP4_OK;
        if (s < 0)
            return;
        S = (uint32_t)s;
    } else {
        __syncthreads();
        S = (uint32_t)((a.rows + SG_ROWS - 1) / SG_ROWS);
    }
    const uint32_t ntiles = S * a.n_ct;
    // this CTA's tiles: blockIdx.x, + gridDim.x, ... (TileWalk)
    const uint32_t n = blockIdx.x < ntiles ? (ntiles - blockIdx.x + gridDim.x - 1) / gridDim.x : 0u;
    // outputs present (SG_TS_* bits): the row-wise ones, the column-wise mask
    const uint32_t outs = (ROW && a.y_row ? SG_TS_YR : 0u) | (ROW && a.codes_row ? SG_TS_CODES_R : 0u) |
                          (ROW && a.mask_row ? SG_TS_MASK_R : 0u) | (a.mask_col ? SG_TS_MASK : 0u);
    uint32_t issued = 0;  // producer lane 0: tiles whose load was issued

    if (warp == S8_PRODUCER) {
        TileWalk<GROUPS> pw;
        auto load = [&](uint32_t j) {  // lane 0: tile j (in order) into stage j mod S8_STAGES
            const int s = (int)(j % S8_STAGES);
            const int4 inf = pw.info(a, s_bpre, s_rst);
            sm.info[s] = inf;
            const uint32_t bar = smem_addr(&sm.full[s]);
            mbar_expect_tx(bar, SG_TILE_BYTES);
#pragma unroll
            for (int sl = 0; sl < 4; ++sl)
                tma_load_slab(smem_addr(sm.tiles[s] + sl * SG_SLAB_BYTES), &maps.x, inf.z + sl * SG_SLAB_COLS, inf.x,
                              bar);
            ++issued;
            pw.next(a, s_bpre);
        };
        if (lane == 0 && n > 0) {
            pw.start(a, s_bpre, blockIdx.x, gridDim.x);
            for (uint32_t j = 0; j < n && j < (uint32_t)S8_STAGES; ++j)
                load(j);
        }
        for (uint32_t j = 0; j < n; ++j) {
            const int s = (int)(j % S8_STAGES);
            // every lane waits (and so acquires the compute warps' writes)
            const bool ok = __all_sync(FULL, mbar_wait(smem_addr(&sm.empty[s]), (j / S8_STAGES) & 1u));
            if (!ok || *err) {
                if (lane == 0)
                    *err = 1;
                break;
            }
            const int4 inf = sm.info[s];
            const int row0 = inf.x, nrows = inf.y, col0 = inf.z;
            const Staged8Out& o = sm.out[j & 1];
            // full tiles: TMA for what it can address; short tiles: the
            // row-wise outputs by TMA (the rows past nrows hold the values
            // their owner writes), the column-wise mask copied
            const uint32_t tma = outs & a.ts_flags & (nrows == SG_ROWS ? ~0u : ~SG_TS_MASK);
            if (lane == 0) {
                const uint32_t ybase = smem_addr(sm.tiles[s]);
#pragma unroll
                for (int sl = 0; sl < 4; ++sl)
                    if ((tma & SG_TS_YR) && col0 + sl * SG_SLAB_COLS < a.cols)
                        tma_store_box(&maps.yr, ybase + sl * SG_SLAB_BYTES, col0 + sl * SG_SLAB_COLS, row0);
#pragma unroll
                for (int b = 0; b < 2; ++b)
                    if ((tma & SG_TS_CODES_R) && col0 + 128 * b < a.cols)
                        tma_store_box(&maps.codes_r, smem_addr(o.crow[b]), col0 + 128 * b, row0);
                if (tma & SG_TS_MASK_R)
                    tma_store_box(&maps.mask_r, smem_addr(o.mrow), col0 / 8, row0);
                if (tma & SG_TS_MASK)
                    tma_store_box(&maps.mask, smem_addr(o.mcol), col0 / 8, row0);
                bulk_commit();  // this tile's group
            }
            copy8<SMMA>(a, o, sm.tiles[s], row0, nrows, col0, outs & ~tma, lane);
            __syncwarp();
            if (lane == 0 && j > 0) {
                // tile j - 1's stores have read its staging buffer and its
                // stage: release the buffer to tile j + 1 and refill the stage
                bulk_wait_read_but1();
                mbar_arrive(smem_addr(&sm.sfree[(j - 1) & 1]));
                if (j - 1 + S8_STAGES < n)
                    load(j - 1 + S8_STAGES);
            }
            __syncwarp();
        }
    } else {
        // column pass: this lane's column pair and rows (as the MXFP4 kernel)
        const int p = lane & 15, h = lane >> 4;
        const int cpair = 32 * warp + 2 * p;
        const uint32_t cchunk = 4 * (warp & 1) + (p >> 2);
        uint32_t yo[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint32_t rq = 4 * h + q;
            yo[q] = (uint32_t)(warp >> 1) * SG_SLAB_BYTES + rq * 128 + ((cchunk ^ rq) << 4) + 4 * (p & 3);
        }
        // row pass: tile row rr; 16-byte chunks jj of the warp's 32 columns
        // in the stage; its two 16-byte code chunks in box w / 4; its mask
        // word and scale byte
        const int rr = lane;
        uint32_t ro[4];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj)
            ro[jj] = (uint32_t)(warp >> 1) * SG_SLAB_BYTES + rr * 128 +
                     ((uint32_t)((4 * (warp & 1) + jj) ^ (rr & 7)) << 4);
        const uint32_t rc0 = rr * 128 + (((2u * (warp & 3)) ^ (uint32_t)(rr & 7)) << 4);
        const uint32_t rc1 = rr * 128 + (((2u * (warp & 3) + 1) ^ (uint32_t)(rr & 7)) << 4);
        const int rw = rr * 8 + warp;

        for (uint32_t j = 0; j < n; ++j) {
            const int s = (int)(j % S8_STAGES);
            if (!__all_sync(FULL, mbar_wait(smem_addr(&sm.full[s]), (j / S8_STAGES) & 1u))) {
                if (lane == 0)
                    *err = 1;
                break;
            }
            const int4 inf = sm.info[s];
            const int row0 = inf.x, nrows = inf.y, col0 = inf.z;
            const uint32_t rb = (uint32_t)inf.w;
            uint8_t* tile = sm.tiles[s];
            Staged8Out& o = sm.out[j & 1];
            // the warp's 32 columns lie wholly inside or outside the tensor
            if (col0 + 32 * warp < a.cols) {
                // ---- column pass
                uint32_t cw[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    cw[i] = sm_ld32(tile, yo[i & 3] + (i >> 2) * 1024);
                if (nrows < SG_ROWS) {
                    // rows past a group tail belong to the next group
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        if (8 * (i >> 2) + 4 * h + (i & 3) >= nrows)
                            cw[i] = 0u;
                }
                uint32_t m2 = 0;
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    m2 = vmax2(m2, cw[i] & 0x7FFF7FFFu);
                m2 = vmax2(m2, __shfl_xor_sync(FULL, m2, 16));
                const uint32_t A_lo = m2 << 16, A_hi = m2 & 0xFFFF0000u;
                const bool sp_lo = A_lo >= 0x7F800000u, sp_hi = A_hi >= 0x7F800000u;
                const int k_lo = sp_lo ? 0 : k_e4m3(A_lo), k_hi = sp_hi ? 0 : k_e4m3(A_hi);
                const float inv_lo = __uint_as_float(pow2_bits(-k_lo)), inv_hi = __uint_as_float(pow2_bits(-k_hi));
                const float sc_lo = __uint_as_float(pow2_bits(k_lo)), sc_hi = __uint_as_float(pow2_bits(k_hi));
                // special halves: NaN values and code 0
                const uint32_t nanw = (sp_lo ? 0x0000FFFFu : 0u) | (sp_hi ? 0xFFFF0000u : 0u);
                const uint32_t ckeep = (sp_lo ? 0u : 0x00FFu) | (sp_hi ? 0u : 0xFF00u);
                if (h == 0) {
                    sm.limw[warp][p] = (sp_lo ? 0xFFFFu : lim8x(k_lo)) | ((sp_hi ? 0xFFFFu : lim8x(k_hi)) << 16);
                    if (a.scales_col)
                        *reinterpret_cast<uint16_t*>(a.scales_col + (int64_t)rb * a.cols + col0 + cpair) =
                            (uint16_t)((sp_lo ? 0xFFu : (uint32_t)(k_lo + 127)) |
                                       ((sp_hi ? 0xFFu : (uint32_t)(k_hi + 127)) << 8));
                }
                char* yb = a.y_col ? static_cast<char*>(a.y_col) + (((int64_t)row0 + 4 * h) * a.ld_y + col0 + cpair) * 2
                                   : nullptr;
                uint8_t* cb = a.codes_col ? a.codes_col + ((int64_t)row0 + 4 * h) * a.cols + col0 + cpair : nullptr;
                const int64_t ys = a.ld_y * 2, cs = a.cols;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int r = 8 * (i >> 2) + (i & 3);  // tile row - 4h
                    uint32_t code;
                    uint32_t yw = q8word(cw[i], inv_lo, inv_hi, sc_lo, sc_hi, code);
                    yw = (yw & ~nanw) | (0x7FC07FC0u & nanw);
                    if (r + 4 * h < nrows) {
                        if (yb)
                            *reinterpret_cast<uint32_t*>(yb + r * ys) = yw;
                        if (cb)
                            *reinterpret_cast<uint16_t*>(cb + r * cs) = (uint16_t)(code & ckeep);
                    }
                }
                // staging buffer j & 1 was last filled by tile j - 2, whose
                // stores the producer saw read at tile j - 1 (the k-th
                // release of a buffer completes its phase k - 1)
                if (!__all_sync(FULL, j < 2 || mbar_wait(smem_addr(&sm.sfree[j & 1]), ((j >> 1) + 1) & 1u))) {
                    if (lane == 0)
                        *err = 1;
                    break;
                }
                // limw of this warp -> its row pass (the __all_sync above
                // also orders the warp)

                // ---- row pass: every row of the tile
                uint32_t w[16];
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    const uint4 c = sm_ld128(tile, ro[jj]);
                    w[4 * jj + 0] = c.x;
                    w[4 * jj + 1] = c.y;
                    w[4 * jj + 2] = c.z;
                    w[4 * jj + 3] = c.w;
                }
                if (a.mask_col) {
                    // rows past a group tail are not copied out; their word is don't-care
                    uint32_t cm = 0;
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        const uint4 L = *reinterpret_cast<const uint4*>(&sm.limw[warp][4 * jj]);
                        const uint32_t lx[4] = {L.x, L.y, L.z, L.w};
                        const uint32_t a4w[4] = {w[4 * jj] & 0x7FFF7FFFu, w[4 * jj + 1] & 0x7FFF7FFFu,
                                                 w[4 * jj + 2] & 0x7FFF7FFFu, w[4 * jj + 3] & 0x7FFF7FFFu};
                        cm |= sat8(a4w, lx) << (8 * jj);
                    }
                    o.mcol[rw] = cm;
                }
                if constexpr (ROW) {
                    uint32_t r2 = 0;
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        r2 = vmax2(r2, w[i] & 0x7FFF7FFFu);
                    const uint32_t A = max(r2 & 0xFFFFu, r2 >> 16) << 16;
                    const bool sp = A >= 0x7F800000u;
                    const int k = sp ? 0 : k_e4m3(A);
                    const float inv = __uint_as_float(pow2_bits(-k)), sc = __uint_as_float(pow2_bits(k));
                    uint32_t yv[16], cv[8], sats = 0;
                    if (!sp) {
                        const uint32_t lx = lim8x(k) * 0x10001u;
                        const uint32_t limx[4] = {lx, lx, lx, lx};
#pragma unroll
                        for (int jj = 0; jj < 4; ++jj) {
                            uint32_t q[4];
#pragma unroll
                            for (int u = 0; u < 4; ++u)
                                yv[4 * jj + u] = q8word(w[4 * jj + u], inv, inv, sc, sc, q[u]);
                            cv[2 * jj] = q[0] | (q[1] << 16);
                            cv[2 * jj + 1] = q[2] | (q[3] << 16);
                            const uint32_t a4w[4] = {w[4 * jj] & 0x7FFF7FFFu, w[4 * jj + 1] & 0x7FFF7FFFu,
                                                     w[4 * jj + 2] & 0x7FFF7FFFu, w[4 * jj + 3] & 0x7FFF7FFFu};
                            sats |= sat8(a4w, limx) << (8 * jj);
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            yv[i] = 0x7FC07FC0u;
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            cv[i] = 0u;
                    }
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj)
                        *reinterpret_cast<uint4*>(tile + ro[jj]) =
                            make_uint4(yv[4 * jj], yv[4 * jj + 1], yv[4 * jj + 2], yv[4 * jj + 3]);
                    uint8_t* cbx = o.crow[warp >> 2];
                    *reinterpret_cast<uint4*>(cbx + rc0) = make_uint4(cv[0], cv[1], cv[2], cv[3]);
                    *reinterpret_cast<uint4*>(cbx + rc1) = make_uint4(cv[4], cv[5], cv[6], cv[7]);
                    o.mrow[rw] = sats;
                    o.srow[rw] = (uint8_t)(sp ? 0xFFu : (uint32_t)(k + 127));
                }
            }
            fence_async_smem();  // y in the stage and the staged outputs -> visible to the TMA stores
            __syncwarp();
            if (lane == 0)
                mbar_arrive(smem_addr(&sm.empty[s]));  // this warp is done with tile j
        }
    }

    __syncthreads();
    if (warp == S8_PRODUCER && lane == 0) {
        if (*err) {
            if (a.status)
                *a.status = MXFP4_ECUDA;
            // loads still in flight land in shared memory: wait (bounded) for
            // the last S8_STAGES issued before the CTA releases it (load i
            // completes phase (i / S8_STAGES) of its stage's barrier)
            for (uint32_t i = issued > (uint32_t)S8_STAGES ? issued - S8_STAGES : 0u; i < issued; ++i)
                (void)mbar_wait(smem_addr(&sm.full[i % S8_STAGES]), (i / S8_STAGES) & 1u);
        }
        bulk_wait_all();
    }
}

}  // namespace mxfp4
