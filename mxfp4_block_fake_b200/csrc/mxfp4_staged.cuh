// mxfp4_staged.cuh -- the shared-memory-staged forward for bf16, block 32,
// column-wise or both directions (included by mxfp4.cu; shares its helpers),
// and the other kernels of the bf16 fast paths.
//
// A tile is one column-wise block of 32 rows (shorter at a group tail) by 256
// columns. CTA b takes every G-th tile from tile b in row-block-major order
// (TileWalk), so the grid sweeps the tensor a run of whole rows at a time.
// TMA (cp.async.bulk.tensor, 2-D, no multicast) brings each tile into shared
// memory as four 64-column slabs with the 128-byte swizzle, SG_STAGES tiles
// ahead of the computation. The thread that issues the loads also writes the
// tile's coordinates next to the stage, so the other threads never search the
// group plan.
//
// Per tile warp w owns tile columns 32w..32w+31 in both passes:
//   * column pass: lanes l and l ^ 16 share one column pair over 16 rows each
//     (rows with bit 2 clear / set), so the column amax takes one shuffle and
//     each thread derives the two columns' parameters itself. Element core:
//     the nudged hardware convert (qword_cvt). Its y and codes go to a
//     staging tile in shared memory, which TMA stores write to global memory
//     once the tile is complete;
//   * row pass: one row-wise block per lane (32 elements of one row).
//     Element core: the floor(4|y|) code table (qword). Its y is written over
//     the tile's own input words; codes, masks and scales are staged.
// The two cores load different pipes (the converter and the table's integer
// work), which is why the passes use different ones. Group-tail and ragged
// tiles, and outputs whose layout TMA cannot address, are copied out by the
// threads instead. Shared-memory accesses of the passes are conflict-free by
// construction: the two half-warps of the column pass read rows whose
// swizzle phases differ by 4, i.e. disjoint 64-byte halves of the bank space.
//
// One CTA barrier per tile (tile done). Staging buffers alternate between
// tiles; a buffer and the tile's stage are released once the tile's TMA
// stores have read them (an mbarrier per buffer), and the freed stage is
// refilled. Every wait on an mbarrier is bounded; on expiry the CTA records
// MXFP4_ECUDA in the caller's status word (when given), waits (bounded) for
// its own loads still in flight and for its stores, and returns.

namespace mxfp4 {

constexpr int SG_ROWS = 32;                                // rows per tile (= the block)
constexpr int SG_COLS = 256;                               // columns per tile
constexpr int SG_SLAB_COLS = 64;                           // columns per TMA box (128 bytes of bf16)
constexpr int SG_SLAB_BYTES = SG_SLAB_COLS * 2 * SG_ROWS;  // 4096
constexpr int SG_TILE_BYTES = 4 * SG_SLAB_BYTES;           // 16384
constexpr int SG_CODE_BYTES = SG_ROWS * SG_COLS / 2;       // 4096: e2m1 codes of a tile
constexpr int SG_MASK_WORDS = SG_ROWS * SG_COLS / 32;      // 256: saturation bits of a tile
constexpr int SG_STAGES = 3;
constexpr uint64_t SG_WAIT_NS = 4000000000ull;             // an mbarrier wait gives up after 4 s

// which outputs leave through TMA stores on full tiles (the others, and every
// output of a group-tail or ragged tile, are copied out by the threads)
constexpr uint32_t SG_TS_Y = 1u, SG_TS_CODES = 2u, SG_TS_MASK = 4u;              // column-wise
constexpr uint32_t SG_TS_YR = 8u, SG_TS_CODES_R = 16u, SG_TS_MASK_R = 32u;       // row-wise

// Staged outputs of one tile; two buffers alternate between consecutive
// tiles. y tiles use the input's layout (four 4 KB slabs of 64 columns with
// the 128-byte swizzle); codes are 32 rows of 128 bytes with the 128-byte
// swizzle; masks are 32 rows of 32 bytes; row-wise scales are 32 rows of 8
// bytes. Row-wise y is written over the tile's input stage instead.
struct __align__(1024) StagedOut {
    uint8_t ycol[SG_TILE_BYTES];
    uint8_t ccol[SG_CODE_BYTES];
    uint8_t crow[SG_CODE_BYTES];
    uint32_t mcol[SG_MASK_WORDS];
    uint32_t mrow[SG_MASK_WORDS];
    uint8_t srow[SG_ROWS * SG_COLS / 32];
};

struct __align__(1024) StagedSmem {
    uint8_t tiles[SG_STAGES][SG_TILE_BYTES];  // input stages (1024-aligned swizzle atoms); row-wise y in place
    StagedOut out[2];                         // staged outputs of tiles j (j even) and j (j odd)
    uint32_t limw[8][16];                     // per warp and column pair: 0x8000 + limit bits of each column
    int4 info[SG_STAGES];                     // row0, nrows, col0, row block of each stage's tile
    uint32_t lut[64];
    unsigned long long full[SG_STAGES];       // mbarriers: stage loaded (TMA transaction count)
    unsigned long long sfree[2];              // mbarriers: the stores of staging buffer b's last tile have read it
    int err;
};

constexpr int SG_THREADS = NTHREADS;
// Thread SG_ASYNC (lane 0 of warp 1) issues every TMA load and store of the
// CTA and waits for the stores; its warp copies the row-wise scales.
constexpr int SG_ASYNC = 32;

// TMA descriptors: the input and the outputs (an output map is only read
// when its SG_TS_* flag is set).
struct StagedMaps {
    CUtensorMap x, y, codes, mask, yr, codes_r, mask_r;
};

__device__ __forceinline__ uint32_t smem_addr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }


__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity)
{
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    return done != 0;
}

__device__ __forceinline__ uint64_t global_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wait for the phase of the given parity to complete; false after SG_WAIT_NS
// of global time (the caller then records an error and stops).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity)
{
    if (mbar_try(bar, parity))
        return true;
    const uint64_t t0 = global_ns();
    while (!mbar_try(bar, parity))
        if (global_ns() - t0 > SG_WAIT_NS)
            return false;
    return true;
}

// One 64 x 32 box of bf16 from global memory into a 4 KB swizzled slab. The
// inner coordinate is a multiple of 64 elements (128 bytes).
__device__ __forceinline__ void tma_load_slab(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(map), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

// One box from shared memory to global memory (bulk-group completion). The
// box lies wholly inside the tensor and its inner coordinate is a multiple of
// 16 bytes.
__device__ __forceinline__ void tma_store_box(const CUtensorMap* map, uint32_t src, int x, int y)
{
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(map), "r"(src),
                 "r"(x), "r"(y)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_but1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// A code-table entry. Not volatile: the table does not change once built, so
// the compiler may schedule these loads freely among the surrounding work.
__device__ __forceinline__ uint32_t lut_load(uint32_t addr)
{
    uint32_t v;
    asm("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

// Typed views of shared memory by byte offset (ordinary loads and stores, so
// that the compiler orders them against the barriers and schedules them
// freely among themselves).
__device__ __forceinline__ uint32_t sm_ld32(const uint8_t* base, uint32_t off)
{
    return *reinterpret_cast<const uint32_t*>(base + off);
}
__device__ __forceinline__ uint4 sm_ld128(const uint8_t* base, uint32_t off)
{
    return *reinterpret_cast<const uint4*>(base + off);
}

__device__ __forceinline__ uint32_t hmul2_bf16(uint32_t a, uint32_t b)
{
    uint32_t r;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// E2M1 nibbles of four words of signed packed bf16 codes (8 elements).
__device__ __forceinline__ uint32_t e2m1_word(const uint32_t* P)
{
    uint32_t r;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %1, %2;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %3, %4;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %5, %6;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %7, %8;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(r)
        : "f"(__uint_as_float(P[0])), "f"(__uint_as_float(P[0] << 16)), "f"(__uint_as_float(P[1])),
          "f"(__uint_as_float(P[1] << 16)), "f"(__uint_as_float(P[2])), "f"(__uint_as_float(P[2] << 16)),
          "f"(__uint_as_float(P[3])), "f"(__uint_as_float(P[3] << 16)));
    return r;
}

// Block exponent for a scale mode fixed at compile time (block_k's rule).
template <int MODE>
__device__ __forceinline__ int block_kt(uint32_t A, uint32_t thr)
{
    if constexpr (MODE == MXFP4_SCALE_FLOOR) {
        return max((int)(A >> 23) - 129, -127);
    } else {
        const int k = (int)(A >> 23) - (int)(thr >> 23) + 1 - ((A & 0x7FFFFFu) < (thr & 0x7FFFFFu) ? 1 : 0);
        return max(k, -30);
    }
}

// Fast-path exponent range of this kernel: 2^k and every code * 2^k are
// normal bf16 numbers (k >= -125), and the limit bits of lim16_of_k stay
// below 0x8000 (k <= 16).
__device__ __forceinline__ bool k_fast_bf(int k) { return (uint32_t)(k + 125) <= 141u; }

// bf16 bits of 2^k for a fast-path k.
__device__ __forceinline__ uint32_t bf16_pow2(int k) { return (uint32_t)(k + 127) << 7; }

// A word with its -0 halves turned into +0 (x + 0 in bf16 arithmetic, which
// changes nothing else: nonzero values, subnormals and infinities pass
// unchanged, a NaN stays a NaN). After this the sign bit of a half is set
// exactly when the codebook's sign rule keeps a sign: sign(y) of a nonzero x.
__device__ __forceinline__ uint32_t clear_neg_zero(uint32_t w)
{
    uint32_t r;
    asm("add.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(w), "r"(0u));
    return r;
}

// One word (two bf16 elements) of fast-path blocks; wc has no -0 halves
// (clear_neg_zero). inv_*: 2^-k of each element's block; s2: packed bf16
// 2^k of each element's block; mul4, mul16: 4 and 65536 (KArgs).
// t = 2^21 + |x| * 2^-k rounded down (fp32 spacing on [2^21, 2^22) is 1/4),
// so t's bits are 0x4A000000 + floor(4|y|); lutb16 = table base - 0x28000000
// folds that offset into the address multiply-add. Both halves take one
// packed fma (fma.rm.f32x2) on (|low| as fp32, |word| as fp32): the high
// element is indexed from the whole word, since the low element's magnitude
// lies below its last bf16 bit and cannot carry it across a quarter of 2^k.
// Returns the dequantised packed bf16 pair; P receives the signed codes.
__device__ __forceinline__ uint32_t qword(uint32_t wc, float inv_lo, float inv_hi, uint32_t s2, uint32_t lutb16,
                                          uint32_t mul4, uint32_t mul16, uint32_t& P)
{
    const uint32_t aw = wc & 0x7FFF7FFFu;
    unsigned long long t;
    const unsigned long long src = ((unsigned long long)aw << 32) | (unsigned long long)(aw * mul16);
    const unsigned long long inv2 = ((unsigned long long)__float_as_uint(inv_hi) << 32) | __float_as_uint(inv_lo);
    asm("fma.rm.f32x2 %0, %1, %2, %3;" : "=l"(t) : "l"(src), "l"(inv2), "l"(0x4A0000004A000000ull));
    const uint32_t el = lut_load((uint32_t)t * mul4 + lutb16);
    const uint32_t eh = lut_load((uint32_t)(t >> 32) * mul4 + lutb16);
    P = __byte_perm(el, eh, 0x7632) | (wc & 0x80008000u);
    return hmul2_bf16(P, s2);
}

// ---- E2M1 rounding by the hardware convert ---------------------------------
// The convert rounds to nearest with ties to even; the codebook's rule sends
// ties up (away from zero). Multiplying y by (1 + 2^-20) first moves exact
// midpoints above themselves and nothing else across one: y is a bf16 value
// times 2^-k (8 significant bits), so a y below a midpoint lies at least one
// bf16 ulp (2^-8 relative) below it, and the one rounding of the product
// changes it by at most 2^-24 relative. The product is formed as
// x * (2^-k (1 + 2^-20)) + 0 in one fma: adding +0 turns -0 into +0 (the
// codebook's sign rule for zero inputs) and keeps the sign of every nonzero
// product, however small. Codes above 6 saturate to 6 in the convert, as in
// the codebook. Checked against the table path for every finite bf16 value
// and every fast-path k.

// 2^-k (1 + 2^-20) for a fast-path k (mantissa bit 3 set).
__device__ __forceinline__ float inv_nudged(int k) { return __uint_as_float((0x3F800000u - ((uint32_t)k << 23)) | 8u); }

// 2^k for a fast-path k.
__device__ __forceinline__ float pow2f_k(int k) { return __uint_as_float(0x3F800000u + ((uint32_t)k << 23)); }

// Nudged scaled values of both halves of a bf16 word.
__device__ __forceinline__ void nudged_pair(uint32_t w, float invn_lo, float invn_hi, float& ylo, float& yhi)
{
    asm("fma.rn.f32 %0, %1, %2, 0f00000000;" : "=f"(ylo) : "f"(__uint_as_float(w << 16)), "f"(invn_lo));
    asm("fma.rn.f32 %0, %1, %2, 0f00000000;" : "=f"(yhi) : "f"(__uint_as_float(w & 0xFFFF0000u)), "f"(invn_hi));
}

// code * 2^k of both halves from the f16x2 codes, as packed bf16 (exact).
__device__ __forceinline__ uint32_t dequant_pair(uint32_t h, float sc_lo, float sc_hi)
{
    float clo, chi;
    asm("{\n\t.reg .b16 l, u;\n\tmov.b32 {l, u}, %2;\n\tcvt.f32.f16 %0, l;\n\tcvt.f32.f16 %1, u;\n\t}"
        : "=f"(clo), "=f"(chi)
        : "r"(h));
    return __byte_perm(__float_as_uint(clo * sc_lo), __float_as_uint(chi * sc_hi), 0x7632);
}

// One word: its E2M1 byte (low element in the low nibble) and its
// dequantised packed bf16 pair.
__device__ __forceinline__ uint32_t qword_cvt(uint32_t w, float invn_lo, float invn_hi, float sc_lo, float sc_hi,
                                              uint32_t& byte)
{
    float ylo, yhi;
    nudged_pair(w, invn_lo, invn_hi, ylo, yhi);
    uint32_t h;
    asm("{\n\t.reg .b8 q;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q, %2, %3;\n\t"
        "cvt.u32.u8 %0, q;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, q;\n\t}"
        : "=r"(byte), "=r"(h)
        : "f"(yhi), "f"(ylo));
    return dequant_pair(h, sc_lo, sc_hi);
}

// Four words with one scale: the 32-bit E2M1 nibble word and four
// dequantised packed bf16 pairs.
__device__ __forceinline__ uint32_t qword4_cvt(const uint32_t* w, float invn, float sc, uint32_t* o)
{
    float y[8];
#pragma unroll
    for (int u = 0; u < 4; ++u)
        nudged_pair(w[u], invn, invn, y[2 * u], y[2 * u + 1]);
    uint32_t nibs, h[4];
    asm("{\n\t.reg .b8 q0, q1, q2, q3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q0, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q1, %8, %7;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q2, %10, %9;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q3, %12, %11;\n\t"
        "mov.b32 %0, {q0, q1, q2, q3};\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, q0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, q1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, q2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %4, q3;\n\t}"
        : "=r"(nibs), "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
        : "f"(y[0]), "f"(y[1]), "f"(y[2]), "f"(y[3]), "f"(y[4]), "f"(y[5]), "f"(y[6]), "f"(y[7]));
#pragma unroll
    for (int u = 0; u < 4; ++u)
        o[u] = dequant_pair(h[u], sc, sc);
    return nibs;
}

// The general element path with block amaxes passed by value: a column pair
// (lo, hi alternating over the eight elements of a chunk) or one block. The
// array general_chunk reads lives in these functions' frames, so a kernel
// keeps nothing in local memory on its fast path.
__device__ __noinline__ ChunkOut general_chunk_pair(uint4 dv, uint32_t A_lo, uint32_t A_hi, int mode, uint32_t thr,
                                                    uint32_t lutb)
{
    const uint32_t Ac[8] = {A_lo, A_hi, A_lo, A_hi, A_lo, A_hi, A_lo, A_hi};
    return general_chunk<8, true>(dv, Ac, mode, thr, lutb);
}

__device__ __noinline__ ChunkOut general_chunk_one(uint4 dv, uint32_t A, int mode, uint32_t thr, uint32_t lutb)
{
    return general_chunk<8, false>(dv, &A, mode, thr, lutb);
}

// Tile sequence of one CTA. Tiles are TR rows (one column-wise block) by TC
// columns, numbered row block major (tile t is column tile t mod n_ct of row
// block t / n_ct). CTA b takes tiles b, b + G, b + 2G, ... (G CTAs), so the
// tiles in flight at any moment are a contiguous run of the numbering: whole
// rows of the tensor are read and written at about the same time, and the
// rows a group-tail tile reads past its group's end (the next row block's)
// are read again by another CTA while they are still in L2. g tracks the
// group that holds rb (largest g with s_bpre[g] <= rb, which skips empty
// groups).
template <bool GROUPS, int TR = SG_ROWS, int TC = SG_COLS>
struct TileWalk {
    uint32_t t, stride, rb, ct;
    int g;

    __device__ void start(const KArgs& a, const int32_t* s_bpre, uint32_t t0, uint32_t step)
    {
        t = t0;
        stride = step;
        rb = t / a.n_ct;
        ct = t - rb * a.n_ct;
        g = 0;
        if constexpr (GROUPS) {
            int lo = 0, hi = a.num_groups - 1;
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if ((uint32_t)s_bpre[mid] <= rb)
                    lo = mid;
                else
                    hi = mid - 1;
            }
            g = lo;
        }
    }

    __device__ void next(const KArgs& a, const int32_t* s_bpre)
    {
        t += stride;
        rb = t / a.n_ct;
        ct = t - rb * a.n_ct;
        if constexpr (GROUPS) {
            while (g + 1 < a.num_groups && (uint32_t)s_bpre[g + 1] <= rb)
                ++g;
        }
    }

    // row0, nrows, col0, rb
    __device__ int4 info(const KArgs& a, const int32_t* s_bpre, const int32_t* s_rst) const
    {
        int r0, nr;
        if constexpr (GROUPS) {
            r0 = s_rst[g] + (int)(rb - (uint32_t)s_bpre[g]) * TR;
            nr = min(TR, s_rst[g + 1] - r0);
        } else {
            r0 = (int)rb * TR;
            nr = (int)min((int64_t)TR, a.rows - r0);
        }
        return make_int4(r0, nr, (int)ct * TC, (int)rb);
    }
};

// Copy staged outputs of a tile to global memory with the threads of the CTA
// (group tails, outputs TMA cannot address). The flags select the outputs;
// rows at or past nrows and columns at or past cols are skipped.
__device__ __forceinline__ void copy_outputs(const KArgs& a, const StagedOut& o, const uint8_t* yrow, int row0,
                                             int nrows, int col0, uint32_t which)
{
    const int tid = threadIdx.x;
    const int64_t cstride = a.cols / 2, mstride = (a.cols + 7) / 8;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const int q = tid + NTHREADS * m;  // 0..1023
        const int r = q >> 5, u = q & 31;
        if (r >= nrows)
            continue;
        const int64_t row = row0 + r;
        const int col = col0 + 8 * u;  // y chunk u / codes word u / mask byte u: columns col..col+7
        if (col >= a.cols)
            continue;
        const uint32_t yoff = (u >> 3) * SG_SLAB_BYTES + r * 128 + (((u & 7) ^ (r & 7)) << 4);
        const uint32_t coff = r * 128 + (((u >> 2) ^ (r & 7)) << 4) + 4 * (u & 3);
        if (which & SG_TS_Y)
            st_stream(static_cast<char*>(a.y_col) + (row * a.ld_y + col) * 2, sm_ld128(o.ycol, yoff));
        if (which & SG_TS_YR)
            st_stream(static_cast<char*>(a.y_row) + (row * a.ld_y + col) * 2, sm_ld128(yrow, yoff));
        if (which & SG_TS_CODES)
            *reinterpret_cast<uint32_t*>(a.codes_col + row * cstride + col / 2) = sm_ld32(o.ccol, coff);
        if (which & SG_TS_CODES_R)
            *reinterpret_cast<uint32_t*>(a.codes_row + row * cstride + col / 2) = sm_ld32(o.crow, coff);
        if (which & SG_TS_MASK)
            a.mask_col[row * mstride + col / 8] = reinterpret_cast<const uint8_t*>(o.mcol)[r * 32 + u];
        if (which & SG_TS_MASK_R)
            a.mask_row[row * mstride + col / 8] = reinterpret_cast<const uint8_t*>(o.mrow)[r * 32 + u];
    }
}

// Row-wise scales of a tile (32 rows x 8 blocks) from staging: one row per
// lane. SMMA: the MMA layout, where a tile's row holds two 4-byte atom
// entries (its first block is a multiple of 8).
template <bool SMMA>
__device__ __forceinline__ void copy_row_scales(const KArgs& a, const StagedOut& o, int row0, int nrows, int col0,
                                                int lane)
{
    const int r = lane;
    if (r >= nrows)
        return;
    const int64_t nblk = (a.cols + 31) / 32;
    if constexpr (SMMA) {
        const int64_t b0 = col0 / 32, row = (int64_t)row0 + r;
        const int nb = (int)min((int64_t)8, nblk - b0);
        if (nb == 8 && ((uintptr_t)a.scales_row & 3) == 0) {
            const uint2 v = *reinterpret_cast<const uint2*>(o.srow + r * 8);
            *reinterpret_cast<uint32_t*>(a.scales_row + srow_off_mma(row, b0, nblk)) = v.x;
            *reinterpret_cast<uint32_t*>(a.scales_row + srow_off_mma(row, b0 + 4, nblk)) = v.y;
        } else {
            for (int b = 0; b < nb; ++b)
                a.scales_row[srow_off_mma(row, b0 + b, nblk)] = o.srow[r * 8 + b];
        }
        return;
    }
    uint8_t* dst = a.scales_row + (int64_t)(row0 + r) * nblk + col0 / 32;
    const int nb = (int)min((int64_t)8, nblk - col0 / 32);
    if (nb == 8 && ((uintptr_t)dst & 7) == 0) {
        *reinterpret_cast<uint2*>(dst) = *reinterpret_cast<const uint2*>(o.srow + r * 8);
    } else {
        for (int b = 0; b < nb; ++b)
            dst[b] = o.srow[r * 8 + b];
    }
}

// ORs a warp's column-pass saturation bits into the staged mask words (one
// 32-bit word per tile row and warp, bit 2p + e for column pair p). Called
// by the whole warp, after the words were written by other lanes.
__device__ __forceinline__ void col_sat_store(uint32_t* mwords, uint32_t bits, int h, int p, int warp)
{
    __syncwarp();
    while (bits) {
        const int i = (__ffs(bits) - 1) >> 1;
        const uint32_t two = (bits >> (2 * i)) & 3u;
        bits &= ~(3u << (2 * i));
        atomicOr(&mwords[(8 * (i >> 2) + 4 * h + (i & 3)) * 8 + warp], two << (2 * p));
    }
}

// ROW / COL: the directions computed (at least one); GROUPS: column-wise
// blocks restart at group_list boundaries; MODE: the scale rule; SMMA:
// row-wise scales in the MMA layout.
template <bool ROW, bool COL, bool GROUPS, int MODE, bool SMMA>
__global__ void __launch_bounds__(SG_THREADS, 2) qdq_staged_kernel(const __grid_constant__ StagedMaps maps, const KArgs a)
{
    extern __shared__ __align__(1024) uint8_t s_dyn[];
    // the swizzle pattern follows absolute shared-memory address bits, so the
    // slabs are placed on a 1024-byte boundary (1 KB of slack is requested)
    uint8_t* s_base = s_dyn + ((1024u - (smem_addr(s_dyn) & 1023u)) & 1023u);
    StagedSmem& sm = *reinterpret_cast<StagedSmem*>(s_base);
    int32_t* s_plan = reinterpret_cast<int32_t*>(s_base + sizeof(StagedSmem));
    int32_t* s_bpre = s_plan;
    int32_t* s_rst = s_plan + (GROUPS ? a.num_groups + 1 : 0);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const bool async_thread = tid == SG_ASYNC;
    if (tid < 64)
        sm.lut[tid] = lut_entry(tid);
    if (tid == 0) {
        sm.err = 0;
        for (int s = 0; s < SG_STAGES; ++s)
            mbar_init(smem_addr(&sm.full[s]), 1);
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
    // this CTA's tiles in sequence order 0..t_end-1 (TileWalk maps them)
    const uint32_t t_begin = 0;
    const uint32_t t_end = blockIdx.x < ntiles ? (ntiles - blockIdx.x + gridDim.x - 1) / gridDim.x : 0u;
    const uint32_t lutb = smem_addr(sm.lut) - 0x2C000000u;
    const uint32_t lutb16 = lutb + 0x04000000u;
    // outputs present, as SG_TS_* bits; those TMA cannot address are copied
    const uint32_t col_out = COL ? (a.y_col ? SG_TS_Y : 0u) | (a.codes_col ? SG_TS_CODES : 0u) |
                                       (a.mask_col ? SG_TS_MASK : 0u)
                                 : 0u;
    const uint32_t row_out = (ROW && a.y_row ? SG_TS_YR : 0u) | (ROW && a.codes_row ? SG_TS_CODES_R : 0u) |
                             (ROW && a.mask_row ? SG_TS_MASK_R : 0u);

    // producer state (the async thread): the next tile to load
    TileWalk<GROUPS> pw;
    uint32_t t_issue = t_begin;
    auto issue = [&](int s) {
        const int4 inf = pw.info(a, s_bpre, s_rst);
        sm.info[s] = inf;
        const uint32_t bar = smem_addr(&sm.full[s]);
        mbar_expect_tx(bar, SG_TILE_BYTES);
#pragma unroll
        for (int sl = 0; sl < 4; ++sl)
            tma_load_slab(smem_addr(sm.tiles[s] + sl * SG_SLAB_BYTES), &maps.x, inf.z + sl * SG_SLAB_COLS, inf.x, bar);
        ++t_issue;
        pw.next(a, s_bpre);
    };
    if (async_thread && t_begin < t_end) {
        pw.start(a, s_bpre, blockIdx.x, gridDim.x);
        for (int s = 0; s < SG_STAGES && t_issue < t_end; ++s)
            issue(s);
    }

    // column pass: warp w owns tile columns 32w..32w+31 (slab w/2); lane =
    // column pair p (columns 32w+2p, +1) x row half h: rows 8i'+4h+q for
    // i' = 0..3, q = 0..3 (word i = 4i' + q)
    const int p = lane & 15, h = lane >> 4;
    const int cpair = 32 * warp + 2 * p;  // first tile column of the pair
    const uint32_t cchunk = 4 * (warp & 1) + (p >> 2);
    uint32_t yo[4], co[4];  // per q: byte offset of word (i' = 0) in a y tile / in a codes tile
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint32_t rq = 4 * h + q;  // row mod 8 (and row for i' = 0)
        yo[q] = (uint32_t)(warp >> 1) * SG_SLAB_BYTES + rq * 128 + ((cchunk ^ rq) << 4) + 4 * (p & 3);
        co[q] = rq * 128 + (((uint32_t)warp ^ rq) << 4) + p;
    }
    // row pass: warp w takes the row-wise blocks of columns 32w..32w+31 (the
    // columns of its column pass), one tile row per lane. Byte offsets of the
    // lane's block: chunks of a y tile, its 16 code bytes; word rr*8 + w of
    // a mask tile; byte rr*8 + w of the scales.
    const int rr = lane;
    uint32_t ro[4];
#pragma unroll
    for (int jj = 0; jj < 4; ++jj)
        ro[jj] = (uint32_t)(warp >> 1) * SG_SLAB_BYTES + rr * 128 +
                 ((uint32_t)((4 * (warp & 1) + jj) ^ (rr & 7)) << 4);
    const uint32_t rco = rr * 128 + (((uint32_t)warp ^ (uint32_t)(rr & 7)) << 4);
    const int rw = rr * 8 + warp;

    int s = 0;
    uint32_t phase = 0;
    uint32_t t = t_begin;
    for (uint32_t j = 0; t < t_end; ++t, ++j) {
        int row0 = 0, nrows = 0, col0 = 0;
        // the warp decides together, so that its shuffles and votes below
        // always see all 32 lanes
        const bool ok = __all_sync(FULL, mbar_wait(smem_addr(&sm.full[s]), phase));
        uint8_t* tile = sm.tiles[s];
        StagedOut& out = sm.out[j & 1];
        uint32_t cw[16];  // the column pass's words
        int k_lo = 0, k_hi = 0;
        uint32_t A_lo = 0, A_hi = 0;
        bool fast = true;
        if (!ok) {
            sm.err = 1;
        } else {
            const int4 inf = sm.info[s];
            row0 = inf.x;
            nrows = inf.y;
            col0 = inf.z;
            const uint32_t rb = (uint32_t)inf.w;
            const bool rows_full = nrows == SG_ROWS;

            // ---- column pass, part 1: amax and parameters of the column pair
            if constexpr (COL) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                cw[i] = sm_ld32(tile, yo[i & 3] + (i >> 2) * 1024);
            }
            if (!rows_full) {
                // rows past a group tail belong to the next group: neither
                // their values nor their amax take part
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
            A_lo = m2 << 16;
            A_hi = m2 & 0xFFFF0000u;
            k_lo = block_kt<MODE>(A_lo, a.thr);
            k_hi = block_kt<MODE>(A_hi, a.thr);
            fast = k_fast_bf(k_lo) && k_fast_bf(k_hi);
            if (h == 0) {
                // the row pass of this warp tests its elements against these
                // limits (0xFFFF: never; the general path reports its own)
                sm.limw[warp][p] = fast ? (0x8000u + lim16_of_k(k_lo)) | ((0x8000u + lim16_of_k(k_hi)) << 16)
                                        : 0xFFFFFFFFu;
                if (a.scales_col && col0 + cpair < a.cols) {
                    // fast-path blocks are finite with k <= 16: the byte is k + 127
                    const uint32_t e8p = fast ? (uint32_t)(k_lo + 127) | ((uint32_t)(k_hi + 127) << 8)
                                              : e8_of(A_lo, k_lo) | (e8_of(A_hi, k_hi) << 8);
                    *reinterpret_cast<uint16_t*>(a.scales_col + (int64_t)rb * a.cols + col0 + cpair) =
                        (uint16_t)e8p;
                }
            }
            }  // COL
        }
        // Staging buffer j & 1 was last filled by tile j - 2; the async
        // thread arrived on sfree[j & 1] at the end of tile j - 1, once the
        // stores of tile j - 2 had read it (the k-th arrival on a buffer's
        // barrier completes its phase k - 1).
        const bool go = ok && (j < 2 || __all_sync(FULL, mbar_wait(smem_addr(&sm.sfree[j & 1]), ((j >> 1) + 1) & 1u)));
        if (!go)
            sm.err = 1;
        __syncwarp();  // limw of this warp

        // ---- column pass, part 2: y and codes of the column pair
        uint32_t gsat = 0;  // saturation bits of a general-path column pair (bits 2i, 2i+1: word i)
        if (COL && go) {
            uint32_t* yq[4];
            uint8_t* cq[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                yq[q] = reinterpret_cast<uint32_t*>(out.ycol + yo[q]);
                cq[q] = out.ccol + co[q];
            }
            auto col_fast = [&]() {
                const float invn_lo = inv_nudged(k_lo), invn_hi = inv_nudged(k_hi);
                const float sc_lo = pow2f_k(k_lo), sc_hi = pow2f_k(k_hi);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    uint32_t byte;
                    yq[i & 3][(i >> 2) * 256] = qword_cvt(cw[i], invn_lo, invn_hi, sc_lo, sc_hi, byte);
                    cq[i & 3][(i >> 2) * 1024] = (uint8_t)byte;
                }
            };
            if (__all_sync(FULL, fast)) {
                col_fast();  // the common case, straight-line
            } else if (fast) {
                col_fast();
            } else {
#pragma unroll
                for (int i0 = 0; i0 < 16; i0 += 4) {
                    const uint4 dv = make_uint4(cw[i0], cw[i0 + 1], cw[i0 + 2], cw[i0 + 3]);
                    const ChunkOut gch = general_chunk_pair(dv, A_lo, A_hi, a.mode, a.thr, lutb);
                    gsat |= (gch.sats & 0xFFu) << (2 * i0);
                    const uint32_t ov[4] = {gch.packed.x, gch.packed.y, gch.packed.z, gch.packed.w};
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int i = i0 + u;
                        yq[i & 3][(i >> 2) * 256] = ov[u];
                        cq[i & 3][(i >> 2) * 1024] = (uint8_t)(gch.nibs >> (8 * u));
                    }
                }
            }
        }


        // ---- row pass: the lane's row-wise block (tile row rr, columns
        // 32w..32w+31): row-wise outputs (y over the block's own input words:
        // the column pass of this warp, the only other reader of these
        // columns, is done), and the column-wise saturation word of the same
        // 32 elements
        if (go) {
            uint32_t rw16[16];  // the lane's block, -0 cleared
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                const uint4 c = sm_ld128(tile, ro[jj]);
                rw16[4 * jj + 0] = c.x;
                rw16[4 * jj + 1] = c.y;
                rw16[4 * jj + 2] = c.z;
                rw16[4 * jj + 3] = c.w;
            }
#pragma unroll
            for (int i = 0; i < 16; ++i)
                rw16[i] = clear_neg_zero(rw16[i]);
            if (COL && a.mask_col) {
                // rows past a group tail are not copied out; their word is don't-care
                uint32_t cm = 0;
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    const uint4 L = *reinterpret_cast<const uint4*>(&sm.limw[warp][4 * jj]);
                    const uint32_t lx[4] = {L.x, L.y, L.z, L.w};
                    const uint32_t a4w[4] = {rw16[4 * jj] & 0x7FFF7FFFu, rw16[4 * jj + 1] & 0x7FFF7FFFu,
                                             rw16[4 * jj + 2] & 0x7FFF7FFFu, rw16[4 * jj + 3] & 0x7FFF7FFFu};
                    cm |= sat8(a4w, lx) << (8 * jj);
                }
                out.mcol[rw] = cm;
            }
            if constexpr (ROW) {
                // every row of the tile is computed, group tail or not: a
                // row's row-wise outputs depend on that row alone
                uint32_t m2 = 0;
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    m2 = vmax2(m2, rw16[i] & 0x7FFF7FFFu);
                const uint32_t am = max(m2 & 0xFFFFu, m2 >> 16);
                const uint32_t A = am << 16;
                const int k = block_kt<MODE>(A, a.thr);
                const bool rfast = k_fast_bf(k);
                uint32_t nib[4], sats = 0;
                auto row_fast = [&]() {
                    const float inv = __uint_as_float(0x3F800000u - ((uint32_t)k << 23));
                    const uint32_t s2 = bf16_pow2(k) * 0x10001u;
                    const uint32_t lx = (0x8000u + lim16_of_k(k)) * 0x10001u;
                    const uint32_t limx[4] = {lx, lx, lx, lx};
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        uint32_t P[4], o[4], a4w[4];
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            a4w[u] = rw16[4 * jj + u] & 0x7FFF7FFFu;
                            o[u] = qword(rw16[4 * jj + u], inv, inv, s2, lutb16, a.mul4, a.mul16, P[u]);
                        }
                        *reinterpret_cast<uint4*>(tile + ro[jj]) = make_uint4(o[0], o[1], o[2], o[3]);
                        nib[jj] = e2m1_word(P);
                        sats |= sat8(a4w, limx) << (8 * jj);
                    }
                };
                if (__all_sync(FULL, rfast)) {
                    row_fast();  // the common case, straight-line
                } else if (rfast) {
                    row_fast();
                } else {
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        const uint4 dv = make_uint4(rw16[4 * jj], rw16[4 * jj + 1], rw16[4 * jj + 2], rw16[4 * jj + 3]);
                        const ChunkOut gch = general_chunk_one(dv, A, a.mode, a.thr, lutb);
                        *reinterpret_cast<uint4*>(tile + ro[jj]) = gch.packed;
                        nib[jj] = gch.nibs;
                        sats |= gch.sats << (8 * jj);
                    }
                }
                *reinterpret_cast<uint4*>(out.crow + rco) = make_uint4(nib[0], nib[1], nib[2], nib[3]);
                out.mrow[rw] = sats;
                // fast-path blocks are finite with k <= 16: the byte is k + 127
                out.srow[rw] = (uint8_t)(rfast ? (uint32_t)(k + 127) : e8_of(A, k));
            }
        }
        // column pairs of the general path add their exact saturation bits
        if (COL && go && __any_sync(FULL, gsat != 0u))
            col_sat_store(out.mcol, gsat, h, p, warp);
        fence_async_smem();  // staged outputs and the stage's y -> visible to the TMA stores and loads
        __syncthreads();     // stage s consumed; staged outputs complete; errors visible
        if (sm.err)
            break;

        // Column-wise outputs of a group tail are copied (the rows past it
        // belong to the next group); row-wise outputs always leave by TMA
        // where it can address them, the rows past a group tail included:
        // they equal what the tile that owns those rows writes. TMA clips
        // rows and columns outside the tensor.
        const uint32_t tma = (nrows == SG_ROWS ? col_out : 0u) | row_out;
        const uint32_t copy = (col_out | row_out) & ~(tma & a.ts_flags);
        if (async_thread) {
            const uint32_t st = tma & a.ts_flags;
            const uint32_t ybase_c = smem_addr(out.ycol), ybase_r = smem_addr(tile);
#pragma unroll
            for (int sl = 0; sl < 4; ++sl)
                if ((st & SG_TS_Y) && col0 + sl * SG_SLAB_COLS < a.cols)
                    tma_store_box(&maps.y, ybase_c + sl * SG_SLAB_BYTES, col0 + sl * SG_SLAB_COLS, row0);
            if (st & SG_TS_CODES)
                tma_store_box(&maps.codes, smem_addr(out.ccol), col0 / 2, row0);
            if (st & SG_TS_MASK)
                tma_store_box(&maps.mask, smem_addr(out.mcol), col0 / 8, row0);
#pragma unroll
            for (int sl = 0; sl < 4; ++sl)
                if ((st & SG_TS_YR) && col0 + sl * SG_SLAB_COLS < a.cols)
                    tma_store_box(&maps.yr, ybase_r + sl * SG_SLAB_BYTES, col0 + sl * SG_SLAB_COLS, row0);
            if (st & SG_TS_CODES_R)
                tma_store_box(&maps.codes_r, smem_addr(out.crow), col0 / 2, row0);
            if (st & SG_TS_MASK_R)
                tma_store_box(&maps.mask_r, smem_addr(out.mrow), col0 / 8, row0);
            bulk_commit();  // this tile's group
            if (j > 0) {
                // tile j - 1's stores have read its staging buffer and its
                // stage (they had this tile's time to do so): release the
                // buffer to tile j + 1 and load tile j + 2 into the stage
                bulk_wait_read_but1();
                mbar_arrive(smem_addr(&sm.sfree[(j - 1) & 1]));
                if (t_issue < t_end)
                    issue(s == 0 ? SG_STAGES - 1 : s - 1);
            }
        }
        if (ROW && a.scales_row && warp == SG_ASYNC / 32)
            copy_row_scales<SMMA>(a, out, row0, nrows, col0, lane);
        // (tile j + 1 writes the other staging buffer and stage: no barrier
        // is needed before the next tile)
        if (copy)
            copy_outputs(a, out, tile, row0, nrows, col0, copy);
        if (++s == SG_STAGES) {
            s = 0;
            phase ^= 1u;
        }
    }

    if (async_thread) {
        if (sm.err) {
            if (a.status)
                *a.status = MXFP4_ECUDA;
            // loads still in flight land in shared memory: wait for them
            // (bounded) before the CTA releases it. They are the tiles from
            // the one this loop stopped at (index t) up to t_issue, in stages
            // s, s + 1, ... with the phase of their turn.
            uint32_t ss = (uint32_t)s, ph = phase;
            for (uint32_t k = t; k < t_issue; ++k) {
                (void)mbar_wait(smem_addr(&sm.full[ss]), ph);
                if (++ss == SG_STAGES) {
                    ss = 0;
                    ph ^= 1u;
                }
            }
        }
        bulk_wait_all();
    }
}

// ---------------------------------------------------------------------------
// Block 128 (bf16): the staged scheme on tiles of 128 rows (one column-wise
// block) by 128 columns (one row-wise block), 16 compute warps and one
// producer warp, one CTA per SM. Per tile every compute thread owns 32
// elements of each pass:
//   * column pass: warp w owns tile columns 8w..8w+7; lane = column pair p
//     (lane & 3) x row group g (lane >> 2) over rows 8i + g, i = 0..15, so
//     the eight row groups of a 16-byte chunk hit eight different swizzle
//     phases; the column amax takes three shuffles;
//   * row pass: warp w owns tile rows 8w..8w+7; lanes 0-15 take the first
//     half of each row's block (slab 0), lanes 16-31 the second (slab 1),
//     32 elements per lane; the row amax takes two shuffles (xor 1, 16).
// Inputs arrive as two 64 x 128 TMA boxes per tile (128-byte swizzle), four
// stages deep. Row-wise y is written over the tile's own stage; row-wise codes
// go straight from registers to global memory (a lane's 32 elements are 16
// contiguous code bytes of its row), which leaves room for the fourth stage;
// the other outputs go to one of two staging buffers (column-wise codes with
// the 64-byte swizzle, masks as 16-byte rows) and leave by TMA stores, issued
// by the producer warp once the compute warps have released the tile (one
// arrival each on its stage's "empty" mbarrier); the producer warp also
// copies the row-wise scales and the group-tail column-wise outputs, and once
// the stores of the tile before have read their sources, releases that
// staging buffer ("sfree") and refills its stage. One barrier among the compute warps per tile (named
// barrier 1): every column pass has read its words from the stage (which
// the row pass then overwrites with y) and published its column limits.
// ---------------------------------------------------------------------------

constexpr int SB_ROWS = 128, SB_COLS = 128;
constexpr int SB_SLAB_BYTES = SG_SLAB_COLS * 2 * SB_ROWS;  // 16384
constexpr int SB_TILE_BYTES = 2 * SB_SLAB_BYTES;           // 32768
constexpr int SB_CODE_BYTES = SB_ROWS * SB_COLS / 2;       // 8192: 64-byte rows
constexpr int SB_MASK_WORDS = SB_ROWS * SB_COLS / 32;      // 512: 16-byte rows
constexpr int SB_STAGES = 4;
constexpr int SB_COMPUTE_WARPS = 16;
constexpr int SB_COMPUTE = 32 * SB_COMPUTE_WARPS;      // 512
constexpr int SB_THREADS = SB_COMPUTE + 32;           // + the producer warp
constexpr int SB_PRODUCER = SB_COMPUTE_WARPS;

struct __align__(1024) StagedOut128 {
    uint8_t ycol[SB_TILE_BYTES];
    uint8_t ccol[SB_CODE_BYTES];
    uint32_t mcol[SB_MASK_WORDS];
    uint32_t mrow[SB_MASK_WORDS];
    uint8_t srow[SB_ROWS];  // row-wise scale byte of each tile row
};

struct __align__(1024) Staged128Smem {
    uint8_t tiles[SB_STAGES][SB_TILE_BYTES];  // input stages; row-wise y in place
    StagedOut128 out[2];
    uint32_t limw[2][SB_COLS / 2];  // per tile parity and column pair: 0x8000 + limit bits of each column (0xFFFF: never)
    uint32_t gm[2][SB_MASK_WORDS];  // per tile parity: column-wise saturation bits of general-path column pairs
    int4 info[SB_STAGES];
    uint32_t lut[64];
    unsigned long long full[SB_STAGES];
    unsigned long long empty[SB_STAGES];
    unsigned long long sfree[2];
    int err;
};

// Copies of a block-128 tile's staged outputs by the producer warp (group
// tails, layouts TMA cannot address): rows at or past nrows and columns at
// or past cols skipped. yrow: the tile's stage (row-wise y).
__device__ __forceinline__ void copy_outputs128(const KArgs& a, const StagedOut128& o, const uint8_t* yrow, int row0,
                                                int nrows, int col0, uint32_t which, int lane)
{
    const int64_t cstride = a.cols / 2, mstride = (a.cols + 7) / 8;
#pragma unroll 1
    for (int q = lane; q < SB_ROWS * 16; q += 32) {
        const int r = q >> 4, u = q & 15;  // row r, 8-column unit u
        if (r >= nrows)
            break;
        const int col = col0 + 8 * u;
        if (col >= a.cols)
            continue;
        const int64_t row = row0 + r;
        const uint32_t yoff = (u >> 3) * SB_SLAB_BYTES + r * 128 + (((u & 7) ^ (r & 7)) << 4);
        const uint32_t coff = r * 64 + ((((uint32_t)u >> 2) ^ ((r >> 1) & 3)) << 4) + 4 * (u & 3);
        if (which & SG_TS_Y)
            st_stream(static_cast<char*>(a.y_col) + (row * a.ld_y + col) * 2, sm_ld128(o.ycol, yoff));
        if (which & SG_TS_YR)
            st_stream(static_cast<char*>(a.y_row) + (row * a.ld_y + col) * 2, sm_ld128(yrow, yoff));
        if (which & SG_TS_CODES)
            *reinterpret_cast<uint32_t*>(a.codes_col + row * cstride + col / 2) = sm_ld32(o.ccol, coff);
        if (which & SG_TS_MASK)
            a.mask_col[row * mstride + col / 8] = reinterpret_cast<const uint8_t*>(o.mcol)[r * 16 + u];
        if (which & SG_TS_MASK_R)
            a.mask_row[row * mstride + col / 8] = reinterpret_cast<const uint8_t*>(o.mrow)[r * 16 + u];
    }
}

// Barrier 1 among the compute warps; returns whether any of their threads
// passed true (the same answer in every thread, so they leave together).
__device__ __forceinline__ bool compute_bar_any(bool p)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred pi, po;\n\t"
        "setp.ne.u32 pi, %1, 0;\n\t"
        "bar.red.or.pred po, 1, %2, pi;\n\t"
        "selp.u32 %0, 1, 0, po;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)p), "n"(SB_COMPUTE)
        : "memory");
    return r != 0;
}

template <bool ROW, bool COL, bool GROUPS, int MODE>
__global__ void __launch_bounds__(SB_THREADS, 1) qdq_staged128_kernel(const __grid_constant__ StagedMaps maps,
                                                                       const KArgs a)
{
    extern __shared__ __align__(1024) uint8_t s_dyn[];
    uint8_t* s_base = s_dyn + ((1024u - (smem_addr(s_dyn) & 1023u)) & 1023u);
    Staged128Smem& sm = *reinterpret_cast<Staged128Smem*>(s_base);
    int32_t* s_plan = reinterpret_cast<int32_t*>(s_base + sizeof(Staged128Smem));
    int32_t* s_bpre = s_plan;
    int32_t* s_rst = s_plan + (GROUPS ? a.num_groups + 1 : 0);
    volatile int* err = &sm.err;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid < 64)
        sm.lut[tid] = lut_entry(tid);
    for (int i = tid; i < 2 * SB_MASK_WORDS; i += SB_THREADS)
        (&sm.gm[0][0])[i] = 0u;
    if (tid == 0) {
        sm.err = 0;
        for (int s = 0; s < SB_STAGES; ++s) {
            mbar_init(smem_addr(&sm.full[s]), 1);
            mbar_init(smem_addr(&sm.empty[s]), SB_COMPUTE_WARPS);
        }
        mbar_init(smem_addr(&sm.sfree[0]), 1);
        mbar_init(smem_addr(&sm.sfree[1]), 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    uint32_t S;
    if constexpr (GROUPS) {
        const int64_t s = build_plan<SB_ROWS>(a, s_bpre, s_rst);  // contains __syncthreads
        if (blockIdx.x == 0 && tid == 0 && a.status)
            *a.status = s < 0 ? MXFP4_EINVAL : MXFP4_OK;
        if (s < 0)
            return;
        S = (uint32_t)s;
    } else {
        __syncthreads();
        S = (uint32_t)((a.rows + SB_ROWS - 1) / SB_ROWS);
    }
    const uint32_t ntiles = S * a.n_ct;
    // this CTA's tiles: blockIdx.x, + gridDim.x, ... (TileWalk)
    const uint32_t n = blockIdx.x < ntiles ? (ntiles - blockIdx.x + gridDim.x - 1) / gridDim.x : 0u;
    const uint32_t col_out = COL ? (a.y_col ? SG_TS_Y : 0u) | (a.codes_col ? SG_TS_CODES : 0u) |
                                       (a.mask_col ? SG_TS_MASK : 0u)
                                 : 0u;
    const uint32_t row_out = (ROW && a.y_row ? SG_TS_YR : 0u) |
                             (ROW && a.mask_row ? SG_TS_MASK_R : 0u);
    uint32_t issued = 0;  // producer lane 0: tiles whose load was issued

    if (warp == SB_PRODUCER) {
        TileWalk<GROUPS, SB_ROWS, SB_COLS> pw;
        auto load = [&](uint32_t j) {  // lane 0: tile j (in order) into stage j mod SB_STAGES
            const int s = (int)(j % SB_STAGES);
            const int4 inf = pw.info(a, s_bpre, s_rst);
            sm.info[s] = inf;
            const uint32_t bar = smem_addr(&sm.full[s]);
            mbar_expect_tx(bar, SB_TILE_BYTES);
#pragma unroll
            for (int sl = 0; sl < 2; ++sl)
                tma_load_slab(smem_addr(sm.tiles[s] + sl * SB_SLAB_BYTES), &maps.x, inf.z + sl * SG_SLAB_COLS, inf.x,
                              bar);
            ++issued;
            pw.next(a, s_bpre);
        };
        if (lane == 0 && n > 0) {
            pw.start(a, s_bpre, blockIdx.x, gridDim.x);
            for (uint32_t j = 0; j < n && j < (uint32_t)SB_STAGES; ++j)
                load(j);
        }
        for (uint32_t j = 0; j < n; ++j) {
            const int s = (int)(j % SB_STAGES);
            const bool ok = __all_sync(FULL, mbar_wait(smem_addr(&sm.empty[s]), (j / SB_STAGES) & 1u));
            if (!ok || *err) {
                if (lane == 0)
                    *err = 1;
                break;
            }
            const int4 inf = sm.info[s];
            const int row0 = inf.x, nrows = inf.y, col0 = inf.z;
            const StagedOut128& o = sm.out[j & 1];
            // column-wise outputs of a group tail are copied; row-wise ones
            // leave by TMA, the rows past a group tail included (they equal
            // what the tile owning those rows writes)
            const uint32_t st = ((nrows == SB_ROWS ? col_out : 0u) | row_out) & a.ts_flags;
            if (lane == 0) {
#pragma unroll
                for (int sl = 0; sl < 2; ++sl) {
                    if ((st & SG_TS_Y) && col0 + sl * SG_SLAB_COLS < a.cols)
                        tma_store_box(&maps.y, smem_addr(o.ycol) + sl * SB_SLAB_BYTES, col0 + sl * SG_SLAB_COLS, row0);
                    if ((st & SG_TS_YR) && col0 + sl * SG_SLAB_COLS < a.cols)
                        tma_store_box(&maps.yr, smem_addr(sm.tiles[s]) + sl * SB_SLAB_BYTES, col0 + sl * SG_SLAB_COLS,
                                      row0);
                }
                if (st & SG_TS_CODES)
                    tma_store_box(&maps.codes, smem_addr(o.ccol), col0 / 2, row0);
                if (st & SG_TS_MASK)
                    tma_store_box(&maps.mask, smem_addr(o.mcol), col0 / 8, row0);
                if (st & SG_TS_MASK_R)
                    tma_store_box(&maps.mask_r, smem_addr(o.mrow), col0 / 8, row0);
                bulk_commit();  // this tile's group
            }
            const uint32_t copy = (col_out | row_out) & ~st;
            if (copy)
                copy_outputs128(a, o, sm.tiles[s], row0, nrows, col0, copy, lane);
            if (ROW && a.scales_row) {
                const int64_t nblk = (a.cols + 127) / 128;
                for (int r = lane; r < nrows; r += 32)
                    a.scales_row[srow_off(a, (int64_t)row0 + r, col0 / 128, nblk)] = o.srow[r];
            }
            __syncwarp();
            if (lane == 0 && j > 0) {
                // tile j - 1's stores have read its staging buffer and its
                // stage: release the buffer to tile j + 1 and refill the stage
                bulk_wait_read_but1();
                mbar_arrive(smem_addr(&sm.sfree[(j - 1) & 1]));
                if (j - 1 + SB_STAGES < n)
                    load(j - 1 + SB_STAGES);
            }
            __syncwarp();
        }
    } else {
        const uint32_t lutb = smem_addr(sm.lut) - 0x2C000000u;
        // column pass: warp w -> tile columns 8w..8w+7 (slab w/8, chunk w%8);
        // lane -> pair p, row group g (rows 8i + g)
        const int p = lane & 3, g = lane >> 2;
        const int cpair = 8 * warp + 2 * p;
        const uint32_t yo = (uint32_t)(warp >> 3) * SB_SLAB_BYTES + g * 128 + ((uint32_t)((warp & 7) ^ g) << 4) + 4 * p;
        const uint32_t co =
            g * 64 + ((((uint32_t)warp >> 2) ^ (uint32_t)((g >> 1) & 3)) << 4) + ((4 * warp + p) & 15);
        // row pass: warp w -> tile rows 8w..8w+7; lanes 0-15 the block's first
        // 64 columns (q = lane & 1 picks 32 of them), lanes 16-31 the last 64
        const int hq = lane >> 4, q = 2 * hq + (lane & 1);
        const int rr = 8 * warp + ((lane & 15) >> 1);
        uint32_t ro[4];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj)
            ro[jj] = (uint32_t)hq * SB_SLAB_BYTES + rr * 128 + ((uint32_t)((4 * (q & 1) + jj) ^ (rr & 7)) << 4);
        const int rw = rr * 4 + q;  // mask word of (row rr, columns 32q..32q+31)

        for (uint32_t j = 0; j < n; ++j) {
            const int s = (int)(j % SB_STAGES);
            const int par = (int)(j & 1);
            int row0 = 0, nrows = 0, col0 = 0;
            uint32_t rb = 0;
            uint8_t* tile = sm.tiles[s];
            StagedOut128& out = sm.out[par];
            uint32_t* limw = sm.limw[par];
            uint32_t* gm = sm.gm[par];
            uint32_t cw[16];
            int k_lo = 0, k_hi = 0;
            uint32_t A_lo = 0, A_hi = 0;
            bool fast = true;
            // waits never break out before the barrier below: a warp that
            // gives up records the error, and all compute warps leave together
            bool ok = __all_sync(FULL, mbar_wait(smem_addr(&sm.full[s]), (j / SB_STAGES) & 1u));
            if (ok) {
                const int4 inf = sm.info[s];
                row0 = inf.x;
                nrows = inf.y;
                col0 = inf.z;
                rb = (uint32_t)inf.w;
                if constexpr (COL) {
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        cw[i] = sm_ld32(tile, yo + i * 1024);
                    if (nrows < SB_ROWS) {
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            if (8 * i + g >= nrows)
                                cw[i] = 0u;
                    }
                    uint32_t m2 = 0;
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        m2 = vmax2(m2, cw[i] & 0x7FFF7FFFu);
                    m2 = vmax2(m2, __shfl_xor_sync(FULL, m2, 4));
                    m2 = vmax2(m2, __shfl_xor_sync(FULL, m2, 8));
                    m2 = vmax2(m2, __shfl_xor_sync(FULL, m2, 16));
                    A_lo = m2 << 16;
                    A_hi = m2 & 0xFFFF0000u;
                    k_lo = block_kt<MODE>(A_lo, a.thr);
                    k_hi = block_kt<MODE>(A_hi, a.thr);
                    fast = k_fast_bf(k_lo) && k_fast_bf(k_hi);
                    if (!fast && a.mask_col) {
                        // general-path column pair (rare): its exact saturation
                        // bits go to gm before the barrier; the row pass ORs
                        // them into its words. Word i of lane (p, g) is row
                        // 8i + g, columns 8w + 2p, +1.
#pragma unroll
                        for (int i0 = 0; i0 < 16; i0 += 4) {
                            const ChunkOut gch = general_chunk_pair(
                                make_uint4(cw[i0], cw[i0 + 1], cw[i0 + 2], cw[i0 + 3]), A_lo, A_hi, a.mode, a.thr, lutb);
                            for (int u = 0; u < 4; ++u) {
                                const uint32_t two = (gch.sats >> (2 * u)) & 3u;
                                if (two)
                                    atomicOr(&gm[(8 * (i0 + u) + g) * 4 + (warp >> 2)],
                                             two << ((8 * warp + 2 * p) & 31));
                            }
                        }
                    }
                    if (g == 0) {
                        limw[4 * warp + p] =
                            fast ? (0x8000u + lim16_of_k(k_lo)) | ((0x8000u + lim16_of_k(k_hi)) << 16) : 0xFFFFFFFFu;
                        if (a.scales_col && col0 + cpair < a.cols) {
                            const uint32_t e8p = fast ? (uint32_t)(k_lo + 127) | ((uint32_t)(k_hi + 127) << 8)
                                                      : e8_of(A_lo, k_lo) | (e8_of(A_hi, k_hi) << 8);
                            *reinterpret_cast<uint16_t*>(a.scales_col + (int64_t)rb * a.cols + col0 + cpair) =
                                (uint16_t)e8p;
                        }
                    }
                }
                // staging buffer par was last filled by tile j - 2, whose
                // stores the producer saw read at tile j - 1
                ok = __all_sync(FULL, j < 2 || mbar_wait(smem_addr(&sm.sfree[par]), ((j >> 1) + 1) & 1u));
            }
            if (!ok && lane == 0)
                *err = 1;
            // column words read, limits published, staging free (or an error)
            if (compute_bar_any(!ok))
                break;

            if constexpr (COL) {
                auto col_fast = [&]() {
                    const float invn_lo = inv_nudged(k_lo), invn_hi = inv_nudged(k_hi);
                    const float sc_lo = pow2f_k(k_lo), sc_hi = pow2f_k(k_hi);
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        uint32_t byte;
                        *reinterpret_cast<uint32_t*>(out.ycol + yo + i * 1024) =
                            qword_cvt(cw[i], invn_lo, invn_hi, sc_lo, sc_hi, byte);
                        out.ccol[co + i * 512] = (uint8_t)byte;
                    }
                };
                if (__all_sync(FULL, fast)) {
                    col_fast();
                } else if (fast) {
                    col_fast();
                } else {
#pragma unroll
                    for (int i0 = 0; i0 < 16; i0 += 4) {
                        const uint4 dv = make_uint4(cw[i0], cw[i0 + 1], cw[i0 + 2], cw[i0 + 3]);
                        const ChunkOut gch = general_chunk_pair(dv, A_lo, A_hi, a.mode, a.thr, lutb);
                        const uint32_t ov[4] = {gch.packed.x, gch.packed.y, gch.packed.z, gch.packed.w};
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            *reinterpret_cast<uint32_t*>(out.ycol + yo + (i0 + u) * 1024) = ov[u];
                            out.ccol[co + (i0 + u) * 512] = (uint8_t)(gch.nibs >> (8 * u));
                        }
                    }
                }
            }

            // ---- row pass: the lane's 32 elements of row rr's block (q-th
            // quarter), the block amax over its four lanes; y over the stage
            {
                uint32_t rw16[16];
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    const uint4 c = sm_ld128(tile, ro[jj]);
                    rw16[4 * jj + 0] = c.x;
                    rw16[4 * jj + 1] = c.y;
                    rw16[4 * jj + 2] = c.z;
                    rw16[4 * jj + 3] = c.w;
                }
                if (COL && a.mask_col) {
                    uint32_t cm = 0;
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        const uint4 L = *reinterpret_cast<const uint4*>(&limw[16 * q + 4 * jj]);
                        const uint32_t lx[4] = {L.x, L.y, L.z, L.w};
                        const uint32_t a4w[4] = {rw16[4 * jj] & 0x7FFF7FFFu, rw16[4 * jj + 1] & 0x7FFF7FFFu,
                                                 rw16[4 * jj + 2] & 0x7FFF7FFFu, rw16[4 * jj + 3] & 0x7FFF7FFFu};
                        cm |= sat8(a4w, lx) << (8 * jj);
                    }
                    out.mcol[rw] = cm | gm[rw];
                    gm[rw] = 0u;  // this thread alone reads the word: clear it for tile j + 2
                }
                if constexpr (ROW) {
                    uint32_t m2 = 0;
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        m2 = vmax2(m2, rw16[i] & 0x7FFF7FFFu);
                    m2 = vmax2(m2, __shfl_xor_sync(FULL, m2, 1));
                    m2 = vmax2(m2, __shfl_xor_sync(FULL, m2, 16));
                    const uint32_t am = max(m2 & 0xFFFFu, m2 >> 16);
                    const uint32_t A = am << 16;
                    const int k = block_kt<MODE>(A, a.thr);
                    const bool rfast = k_fast_bf(k);
                    uint32_t nib[4], sats = 0;
                    auto row_fast = [&]() {
                        const float invn = inv_nudged(k), sc = pow2f_k(k);
                        const uint32_t lx = (0x8000u + lim16_of_k(k)) * 0x10001u;
                        const uint32_t limx[4] = {lx, lx, lx, lx};
#pragma unroll
                        for (int jj = 0; jj < 4; ++jj) {
                            uint32_t o[4];
                            nib[jj] = qword4_cvt(rw16 + 4 * jj, invn, sc, o);
                            *reinterpret_cast<uint4*>(tile + ro[jj]) = make_uint4(o[0], o[1], o[2], o[3]);
                            const uint32_t a4w[4] = {rw16[4 * jj] & 0x7FFF7FFFu, rw16[4 * jj + 1] & 0x7FFF7FFFu,
                                                     rw16[4 * jj + 2] & 0x7FFF7FFFu, rw16[4 * jj + 3] & 0x7FFF7FFFu};
                            sats |= sat8(a4w, limx) << (8 * jj);
                        }
                    };
                    if (__all_sync(FULL, rfast)) {
                        row_fast();
                    } else if (rfast) {
                        row_fast();
                    } else {
#pragma unroll
                        for (int jj = 0; jj < 4; ++jj) {
                            const uint4 dv =
                                make_uint4(rw16[4 * jj], rw16[4 * jj + 1], rw16[4 * jj + 2], rw16[4 * jj + 3]);
                            const ChunkOut gch = general_chunk_one(dv, A, a.mode, a.thr, lutb);
                            *reinterpret_cast<uint4*>(tile + ro[jj]) = gch.packed;
                            nib[jj] = gch.nibs;
                            sats |= gch.sats << (8 * jj);
                        }
                    }
                    if (a.codes_row && (int64_t)row0 + rr < a.rows) {
                        // row-wise codes straight from registers: the lane's 32
                        // elements are 16 contiguous code bytes of its row
                        const int gcol = col0 + 32 * q;
                        uint8_t* cp = a.codes_row + ((int64_t)row0 + rr) * (a.cols / 2) + gcol / 2;
                        if (gcol + 32 <= a.cols && (a.ts_flags & SG_TS_CODES_R)) {
                            st_stream(cp, make_uint4(nib[0], nib[1], nib[2], nib[3]));
                        } else {
#pragma unroll
                            for (int jj = 0; jj < 4; ++jj)
                                if (gcol + 8 * jj < a.cols)
                                    *reinterpret_cast<uint32_t*>(cp + 4 * jj) = nib[jj];
                        }
                    }
                    out.mrow[rw] = sats;
                    if (q == 0)
                        out.srow[rr] = (uint8_t)(rfast ? (uint32_t)(k + 127) : e8_of(A, k));
                }
            }
            fence_async_smem();  // staged outputs and the stage's y -> visible to the TMA stores
            __syncwarp();
            if (lane == 0)
                mbar_arrive(smem_addr(&sm.empty[s]));  // this warp is done with tile j
        }
    }

    __syncthreads();
    if (warp == SB_PRODUCER && lane == 0) {
        if (*err) {
            if (a.status)
                *a.status = MXFP4_ECUDA;
            for (uint32_t i = issued > (uint32_t)SB_STAGES ? issued - SB_STAGES : 0u; i < issued; ++i)
                (void)mbar_wait(smem_addr(&sm.full[i % SB_STAGES]), (i / SB_STAGES) & 1u);
        }
        bulk_wait_all();
    }
}

// ---------------------------------------------------------------------------
// Saved-free clipped STE backward, row-wise, bf16, block 32: grad_in =
// grad_out with +0.0 where |x| exceeds its block's limit, the mask recomputed
// from x in the same pass. One thread per block: two 32-byte loads of x and of
// grad_out (one sector each, every sector used), the block amax and exponent,
// a packed compare per word turned into a keep mask by a sign-replicating
// byte permute, two 32-byte stores. Blocks off the fast range take the
// general element path for their saturation bits. Requires cols % 32 == 0,
// 32-byte aligned pointers and leading dimensions that are multiples of 16.
// ---------------------------------------------------------------------------

__device__ __forceinline__ void ld_nc_v8(const void* p, uint32_t* v)
{
    asm volatile("ld.global.nc.L1::no_allocate.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
                 : "l"(p));
}

__device__ __forceinline__ void st_cs_v8(void* p, const uint32_t* v)
{
    asm volatile("st.global.cs.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(v[0]), "r"(v[1]),
                 "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
                 : "memory");
}

template <int MODE>
__global__ void __launch_bounds__(NTHREADS) ste_row_kernel(const KArgs a)
{
    const uint32_t nb = (uint32_t)(a.cols / 32);
    const uint32_t total = (uint32_t)a.rows * nb;
    __shared__ uint32_t s_lut[64];
    if (threadIdx.x < 64)
        s_lut[threadIdx.x] = lut_entry(threadIdx.x);
    __syncthreads();
    const uint32_t glutb = smem_addr(s_lut) - 0x2C000000u;
    for (uint32_t u = blockIdx.x * blockDim.x + threadIdx.x; u < total; u += gridDim.x * blockDim.x) {
        const uint32_t row = u / nb, blk = u - row * nb;
        const char* xp = static_cast<const char*>(a.x) + ((int64_t)row * a.ld + 32 * blk) * 2;
        uint32_t w[16];
        ld_nc_v8(xp, w);
        ld_nc_v8(xp + 32, w + 8);
        uint32_t m2 = 0;
#pragma unroll
        for (int i = 0; i < 16; ++i)
            m2 = vmax2(m2, w[i] & 0x7FFF7FFFu);
        const uint32_t am = max(m2 & 0xFFFFu, m2 >> 16);
        const uint32_t A = am << 16;
        const int k = block_kt<MODE>(A, a.thr);
        uint32_t keep[16];
        if (k_fast_bf(k)) {
            const uint32_t lx = (0x8000u + lim16_of_k(k)) * 0x10001u;
#pragma unroll
            for (int i = 0; i < 16; ++i)  // bit 15 / 31 of lx - |x| set: that half does not saturate
                keep[i] = prmt(lx - (w[i] & 0x7FFF7FFFu), 0u, 0xBB99u);
        } else {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const ChunkOut gch = general_chunk_one(
                    make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]), A, a.mode, a.thr, glutb);
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    keep[4 * c + j] = ((gch.sats >> (2 * j)) & 1u ? 0u : 0xFFFFu) |
                                      ((gch.sats >> (2 * j + 1)) & 1u ? 0u : 0xFFFF0000u);
            }
        }
        const int64_t goff = ((int64_t)row * a.ld_g + 32 * blk) * 2;
        uint32_t g[16];
        ld_nc_v8(static_cast<const char*>(a.g_out) + goff, g);
        ld_nc_v8(static_cast<const char*>(a.g_out) + goff + 32, g + 8);
#pragma unroll
        for (int i = 0; i < 16; ++i)
            g[i] &= keep[i];
        st_cs_v8(static_cast<char*>(a.g_in) + goff, g);
        st_cs_v8(static_cast<char*>(a.g_in) + goff + 32, g + 8);
    }
}

// ---------------------------------------------------------------------------
// Row-wise bf16 block 32, one streaming pass: one thread per block, two
// 32-byte loads (the next block's issued before this block is worked on),
// amax, k, the codes by the nudged hardware convert, then the
// outputs asked for: dequantised values (VALS: two 32-byte streaming
// stores), one 16-byte code store, one 4-byte mask word and one scale byte
// (SMMA: in the MMA layout). Without values this is the real-quantisation
// producer. Blocks off the fast k range take the general element path.
// ---------------------------------------------------------------------------

// E2M1 bytes of four words sharing one scale, as one 32-bit nibble word.
__device__ __forceinline__ uint32_t nibs4_cvt(const uint32_t* w, float invn)
{
    float y[8];
#pragma unroll
    for (int u = 0; u < 4; ++u)
        nudged_pair(w[u], invn, invn, y[2 * u], y[2 * u + 1]);
    uint32_t nibs;
    asm("{\n\t.reg .b8 q0, q1, q2, q3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q3, %8, %7;\n\t"
        "mov.b32 %0, {q0, q1, q2, q3};\n\t}"
        : "=r"(nibs)
        : "f"(y[0]), "f"(y[1]), "f"(y[2]), "f"(y[3]), "f"(y[4]), "f"(y[5]), "f"(y[6]), "f"(y[7]));
    return nibs;
}

template <int MODE, bool SMMA, bool VALS>
__global__ void __launch_bounds__(NTHREADS) row_stream_kernel(const KArgs a)
{
    const uint32_t nb = (uint32_t)(a.cols / 32);
    const uint32_t total = (uint32_t)a.rows * nb;
    __shared__ uint32_t s_lut[64];
    if (threadIdx.x < 64)
        s_lut[threadIdx.x] = lut_entry(threadIdx.x);
    __syncthreads();
    const uint32_t glutb = smem_addr(s_lut) - 0x2C000000u;
    const uint32_t stride = gridDim.x * blockDim.x;
    auto load = [&](uint32_t uu, uint32_t (&ww)[16]) {
        const uint32_t rr = uu / nb, bb = uu - rr * nb;
        const char* xp = static_cast<const char*>(a.x) + ((int64_t)rr * a.ld + 32 * bb) * 2;
        ld_nc_v8(xp, ww);
        ld_nc_v8(xp + 32, ww + 8);
    };
    uint32_t w[16];
    uint32_t u = blockIdx.x * blockDim.x + threadIdx.x;
    if (u < total)
        load(u, w);
    for (; u < total; u += stride) {
        const uint32_t row = u / nb, blk = u - row * nb;
        uint32_t wn[16];
        const bool more = u + stride < total;
        if (more)
            load(u + stride, wn);  // the next block's loads are in flight while this one is worked on
        uint32_t m2 = 0;
#pragma unroll
        for (int i = 0; i < 16; ++i)
            m2 = vmax2(m2, w[i] & 0x7FFF7FFFu);
        const uint32_t am = max(m2 & 0xFFFFu, m2 >> 16);
        const uint32_t A = am << 16;
        const int k = block_kt<MODE>(A, a.thr);
        uint32_t nib[4], sats = 0, e8, yv[VALS ? 16 : 1];
        if (k_fast_bf(k)) {
            const float invn = inv_nudged(k);
            const uint32_t lx = (0x8000u + lim16_of_k(k)) * 0x10001u;
            const uint32_t limx[4] = {lx, lx, lx, lx};
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                if constexpr (VALS)
                    nib[c] = qword4_cvt(w + 4 * c, invn, pow2f_k(k), yv + 4 * c);
                else
                    nib[c] = nibs4_cvt(w + 4 * c, invn);
                const uint32_t a4w[4] = {w[4 * c] & 0x7FFF7FFFu, w[4 * c + 1] & 0x7FFF7FFFu,
                                         w[4 * c + 2] & 0x7FFF7FFFu, w[4 * c + 3] & 0x7FFF7FFFu};
                sats |= sat8(a4w, limx) << (8 * c);
            }
            e8 = (uint32_t)(k + 127);
        } else {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const ChunkOut gch = general_chunk_one(
                    make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]), A, a.mode, a.thr, glutb);
                nib[c] = gch.nibs;
                sats |= gch.sats << (8 * c);
                if constexpr (VALS) {
                    yv[4 * c] = gch.packed.x;
                    yv[4 * c + 1] = gch.packed.y;
                    yv[4 * c + 2] = gch.packed.z;
                    yv[4 * c + 3] = gch.packed.w;
                }
            }
            e8 = e8_of(A, k);
        }
        if constexpr (VALS) {
            char* yp = static_cast<char*>(a.y_row) + ((int64_t)row * a.ld_y + 32 * blk) * 2;
            st_cs_v8(yp, yv);
            st_cs_v8(yp + 32, yv + 8);
        }
        if (a.codes_row)
            st_stream(a.codes_row + (int64_t)row * (a.cols / 2) + 16 * blk, make_uint4(nib[0], nib[1], nib[2], nib[3]));
        if (a.mask_row)
            *reinterpret_cast<uint32_t*>(a.mask_row + (int64_t)row * (a.cols / 8) + 4 * blk) = sats;
        if (a.scales_row)
            a.scales_row[SMMA ? srow_off_mma(row, blk, nb) : (int64_t)row * nb + blk] = (uint8_t)e8;
        if (more) {
#pragma unroll
            for (int i = 0; i < 16; ++i)
                w[i] = wn[i];
        }
    }
}

// ---------------------------------------------------------------------------
// MXFP8 row-wise, bf16, block 32, one streaming pass: one thread per block,
// two 32-byte loads (the next block's issued before this block is worked
// on), amax and k (floor(log2 amax) - 8, at least -127), per
// pair of elements one E4M3 convert (nearest even, saturating at 448) and one
// back to exact f16 codes, widened and multiplied by 2^k (exact), then the
// outputs asked for: two 32-byte stores of values, one 32-byte store of codes,
// a 4-byte mask word, a scale byte (SMMA: MMA layout). Non-finite blocks:
// NaN values, codes 0, no saturation, E8M0 0xFF.
// ---------------------------------------------------------------------------

template <bool SMMA>
__global__ void __launch_bounds__(NTHREADS) row_stream8_kernel(const KArgs a)
{
    const uint32_t nb = (uint32_t)(a.cols / 32);
    const uint32_t total = (uint32_t)a.rows * nb;
    const uint32_t stride = gridDim.x * blockDim.x;
    auto load = [&](uint32_t uu, uint32_t (&ww)[16]) {
        const uint32_t rr = uu / nb, bb = uu - rr * nb;
        const char* xp = static_cast<const char*>(a.x) + ((int64_t)rr * a.ld + 32 * bb) * 2;
        ld_nc_v8(xp, ww);
        ld_nc_v8(xp + 32, ww + 8);
    };
    uint32_t w[16];
    uint32_t u = blockIdx.x * blockDim.x + threadIdx.x;
    if (u < total)
        load(u, w);
    for (; u < total; u += stride) {
        const uint32_t row = u / nb, blk = u - row * nb;
        uint32_t wn[16];
        const bool more = u + stride < total;
        if (more)
            load(u + stride, wn);  // the next block's loads are in flight while this one is worked on
        uint32_t m2 = 0;
#pragma unroll
        for (int i = 0; i < 16; ++i)
            m2 = vmax2(m2, w[i] & 0x7FFF7FFFu);
        const uint32_t A = max(m2 & 0xFFFFu, m2 >> 16) << 16;
        uint32_t yv[16], cw[8], sats = 0, e8;
        if (A < 0x7F800000u) {
            const int k = k_e4m3(A);
            const float inv = __uint_as_float(pow2_bits(-k)), sc = __uint_as_float(pow2_bits(k));
            uint32_t q[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float ylo = __fmul_rn(__uint_as_float(w[i] << 16), inv);
                const float yhi = __fmul_rn(__uint_as_float(w[i] & 0xFFFF0000u), inv);
                uint16_t qq;
                asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(qq) : "f"(yhi), "f"(ylo));
                uint32_t h;
                asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(qq));
                float clo, chi;
                asm("{\n\t.reg .b16 l, u;\n\tmov.b32 {l, u}, %2;\n\tcvt.f32.f16 %0, l;\n\tcvt.f32.f16 %1, u;\n\t}"
                    : "=f"(clo), "=f"(chi)
                    : "r"(h));
                // exact products with at most four significant bits: bf16 keeps them
                yv[i] = __byte_perm(__float_as_uint(__fmul_rn(clo, sc)), __float_as_uint(__fmul_rn(chi, sc)), 0x7632);
                q[i] = qq;
            }
#pragma unroll
            for (int j = 0; j < 8; ++j)
                cw[j] = q[2 * j] | (q[2 * j + 1] << 16);
            // bf16 bits of 448 * 2^k = 1.75 * 2^(k + 8)
            const uint32_t lx = (0x8000u + (((uint32_t)(k + 135) << 7) | 0x60u)) * 0x10001u;
            const uint32_t limx[4] = {lx, lx, lx, lx};
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const uint32_t a4w[4] = {w[4 * c] & 0x7FFF7FFFu, w[4 * c + 1] & 0x7FFF7FFFu,
                                         w[4 * c + 2] & 0x7FFF7FFFu, w[4 * c + 3] & 0x7FFF7FFFu};
                sats |= sat8(a4w, limx) << (8 * c);
            }
            e8 = (uint32_t)(k + 127);
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i)
                yv[i] = 0x7FC07FC0u;
#pragma unroll
            for (int j = 0; j < 8; ++j)
                cw[j] = 0u;
            e8 = 0xFFu;
        }
        if (a.y_row) {
            char* yp = static_cast<char*>(a.y_row) + ((int64_t)row * a.ld_y + 32 * blk) * 2;
            st_cs_v8(yp, yv);
            st_cs_v8(yp + 32, yv + 8);
        }
        if (a.codes_row)
            st_cs_v8(a.codes_row + (int64_t)row * a.cols + 32 * blk, cw);
        if (a.mask_row)
            *reinterpret_cast<uint32_t*>(a.mask_row + (int64_t)row * (a.cols / 8) + 4 * blk) = sats;
        if (a.scales_row)
            a.scales_row[SMMA ? srow_off_mma(row, blk, nb) : (int64_t)row * nb + blk] = (uint8_t)e8;
        if (more) {
#pragma unroll
            for (int i = 0; i < 16; ++i)
                w[i] = wn[i];
        }
    }
}

// ---------------------------------------------------------------------------
// MXFP8 column-wise, bf16, block 32 with group restarts: one thread per
// (column-wise block, column pair). Consecutive lanes take consecutive column
// pairs of the same block, so every load and store of a warp is one
// contiguous row segment (128 bytes of x or y). A lane keeps its 32 words in
// registers: amax of both columns, k, then per row the E4M3 pair convert, the
// exact dequantisation, the 2-byte code store; the saturation bits of four
// lanes (8 columns) are OR-ed by two shuffles into the mask byte of each row.
// Requires cols % 8 == 0 (a mask byte's four lanes share a block), 4-byte
// aligned x / y rows and 2-byte aligned codes and scales.
// ---------------------------------------------------------------------------

template <bool GROUPS>
__global__ void __launch_bounds__(NTHREADS, 2) col_pair8_kernel(const KArgs a)
{
    extern __shared__ int32_t s_plan8[];
    int32_t* s_bpre = s_plan8;
    int32_t* s_rst = s_plan8 + (GROUPS ? a.num_groups + 1 : 0);
    int64_t S;
    if constexpr (GROUPS) {
        S = build_plan<32>(a, s_bpre, s_rst);  // contains __syncthreads
        if (blockIdx.x == 0 && threadIdx.x == 0 && a.status)
            *a.status = S < 0 ? MXFP4_EINVAL : MXFP4_OK;
        if (S < 0)
            return;
    } else {
        S = (a.rows + 31) / 32;
    }
    const int lane = threadIdx.x & 31;
    const int64_t npairs = a.cols / 2, mstride = a.cols / 8;
    const int64_t total = S * npairs;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    // tile of a warp iteration: this lane's column pair and block rows
    auto locate = [&](int64_t base, int64_t& rb, int64_t& pr, int64_t& row0, int& nrows) {
        const int64_t idx = base + lane;
        const bool on = idx < total;
        rb = on ? idx / npairs : 0;
        pr = on ? idx - rb * npairs : 0;
        row0 = 0;
        nrows = 0;
        if (on) {
            if constexpr (GROUPS) {
                plan_lookup(s_bpre, s_rst, a.num_groups, (uint32_t)rb, 32, row0, nrows);
            } else {
                row0 = rb * 32;
                nrows = (int)min((int64_t)32, a.rows - row0);
            }
        }
        return on;
    };
    auto load = [&](int64_t row0, int nrows, int64_t pr, uint32_t (&w)[32]) {
#pragma unroll
        for (int r = 0; r < 32; ++r)
            w[r] = r < nrows ? *reinterpret_cast<const uint32_t*>(static_cast<const uint16_t*>(a.x) +
                                                                   (row0 + r) * a.ld + 2 * pr)
                             : 0u;
    };
    // the loop runs per warp, so that all lanes take part in the shuffles; the
    // next tile's words are loaded before this tile's are converted
    int64_t base = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) & ~31ll;
    int64_t rb, pr, row0;
    int nrows;
    bool on = locate(base, rb, pr, row0, nrows);
    uint32_t w[32];
    load(row0, nrows, pr, w);
    for (; base < total; base += stride) {
        int64_t rb_n, pr_n, row0_n;
        int nrows_n;
        const bool on_n = locate(base + stride, rb_n, pr_n, row0_n, nrows_n);
        uint32_t wn[32];
        load(row0_n, nrows_n, pr_n, wn);

        const int64_t c = 2 * pr;
        uint32_t m2 = 0;
#pragma unroll
        for (int r = 0; r < 32; ++r)
            m2 = vmax2(m2, w[r] & 0x7FFF7FFFu);
        const uint32_t A_lo = m2 << 16, A_hi = m2 & 0xFFFF0000u;
        const bool sp_lo = A_lo >= 0x7F800000u, sp_hi = A_hi >= 0x7F800000u;
        const int k_lo = sp_lo ? 0 : k_e4m3(A_lo), k_hi = sp_hi ? 0 : k_e4m3(A_hi);
        const float inv_lo = __uint_as_float(pow2_bits(-k_lo)), inv_hi = __uint_as_float(pow2_bits(-k_hi));
        const float sc_lo = __uint_as_float(pow2_bits(k_lo)), sc_hi = __uint_as_float(pow2_bits(k_hi));
        // 0x8000 + bf16 bits of 448 * 2^k per half; 0xFFFF: never (non-finite block)
        const uint32_t lx = (sp_lo ? 0xFFFFu : 0x8000u + (((uint32_t)(k_lo + 135) << 7) | 0x60u)) |
                            ((sp_hi ? 0xFFFFu : 0x8000u + (((uint32_t)(k_hi + 135) << 7) | 0x60u)) << 16);
        const uint32_t nanw = (sp_lo ? 0x0000FFFFu : 0u) | (sp_hi ? 0xFFFF0000u : 0u);
        const int sh = 2 * (int)(pr & 3);
        uint32_t satw = 0;  // 4 rows at a time: byte j = row 4m + j's bits of the 8 columns
#pragma unroll
        for (int r = 0; r < 32; ++r) {
            const float ylo = __fmul_rn(__uint_as_float(w[r] << 16), inv_lo);
            const float yhi = __fmul_rn(__uint_as_float(w[r] & 0xFFFF0000u), inv_hi);
            uint16_t qq;
            asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(qq) : "f"(yhi), "f"(ylo));
            uint32_t h;
            asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(qq));
            float clo, chi;
            asm("{\n\t.reg .b16 l, u;\n\tmov.b32 {l, u}, %2;\n\tcvt.f32.f16 %0, l;\n\tcvt.f32.f16 %1, u;\n\t}"
                : "=f"(clo), "=f"(chi)
                : "r"(h));
            uint32_t yw = __byte_perm(__float_as_uint(__fmul_rn(clo, sc_lo)), __float_as_uint(__fmul_rn(chi, sc_hi)),
                                      0x7632);
            yw = (yw & ~nanw) | (0x7FC07FC0u & nanw);
            const uint32_t qw = (uint32_t)qq & ~(nanw & 0x00FF00FFu) & ~((nanw >> 8) & 0x0000FF00u);
            const uint32_t keep = lx - (w[r] & 0x7FFF7FFFu);  // bit 15 / 31 set: that half does not saturate
            const uint32_t two = ((~keep >> 15) & 1u) | ((~keep >> 30) & 2u);
            satw |= two << (sh + 8 * (r & 3));
            if (r < nrows) {
                const int64_t row = row0 + r;
                if (a.y_col)
                    *reinterpret_cast<uint32_t*>(static_cast<uint16_t*>(a.y_col) + row * a.ld_y + c) = yw;
                if (a.codes_col)
                    *reinterpret_cast<uint16_t*>(a.codes_col + row * a.cols + c) = (uint16_t)qw;
            }
            if ((r & 3) == 3) {
                satw |= __shfl_xor_sync(FULL, satw, 1);
                satw |= __shfl_xor_sync(FULL, satw, 2);
                if (a.mask_col && on && (pr & 3) == 0) {
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        if (r - 3 + j < nrows)
                            a.mask_col[(row0 + r - 3 + j) * mstride + c / 8] = (uint8_t)(satw >> (8 * j));
                }
                satw = 0;
            }
        }
        if (a.scales_col && on)
            *reinterpret_cast<uint16_t*>(a.scales_col + rb * a.cols + c) =
                (uint16_t)((sp_lo ? 0xFFu : (uint32_t)(k_lo + 127)) | ((sp_hi ? 0xFFu : (uint32_t)(k_hi + 127)) << 8));
#pragma unroll
        for (int r = 0; r < 32; ++r)
            w[r] = wn[r];
        rb = rb_n;
        pr = pr_n;
        row0 = row0_n;
        nrows = nrows_n;
        on = on_n;
    }
}

}  // namespace mxfp4
