// mxfp4_gemm.cuh -- grouped block-scaled GEMM on the fifth-generation tensor
// cores (tcgen05, accumulators in tensor memory), the consumer of the
// operands this library emits (included by mxfp4.cu; shares its helpers and
// the staged kernels' TMA and mbarrier wrappers).
//
// MindSpore hyper-parallel fake_w4a8_gmm_func.py, FakeW4A8GroupedLinear:
// grouped_matmul multiplies, per MoE group, a left and a right operand that
// _select_operands picks from the row-wise and column-wise quantised views
// (layouts "NN", "NT", "TN"). Each operand here is a K-major matrix of E2M1
// codes (two per byte, first element in the low nibble) or E4M3 codes (one
// byte), with one E8M0 scale per 32 elements along K in the 128 x 4 atom
// layout of MXFP4_SCALES_MMA:
//   D[m][n] = sum_k decode(A[m][k]) 2^(sA[m][k/32]-127) decode(B[n][k]) 2^(sB[n][k/32]-127)
// Two ways of grouping:
//   GROUP_M ("NN" forward, "NT" input gradient): the rows of A (tokens) are
//     split by the group list; group g multiplies its rows by its own B_g
//     [N][K] (the expert's weight), into its rows of D [M][N].
//   GROUP_K ("TN" weight gradient): the K slots of A [M][k_alloc] and B
//     [N][k_alloc] are split by the group list as in the column-wise operand
//     layout (each group padded to 128 K slots, MXFP4_COLS_MMA); group g
//     writes D_g [M][N] (D + g * M * ldd); an empty group writes zeros.
//
// Design (one CTA per SM, persistent over output tiles of 128 x 128):
//   warp 0: producer. Lane 0 loads the A and B tiles of one K stage (128-byte
//     rows: 256 E2M1 or 128 E4M3 K elements) with TMA into shared memory
//     with the 128-byte swizzle; the warp gathers the 128 rows' scale bytes
//     of A and of B for the stage into 512-byte atoms (one per 128 K; A's
//     rows of a group need not start on a multiple of 128)
//     with asynchronous 4-byte copies (cp.async, zero-filled past the last
//     row), whose completion each lane signals on the stage's barrier, so
//     the producer never waits for them.
//   warp 1: allocates the tensor memory; lane 0 copies a stage's scale atoms
//     into tensor memory (tcgen05.cp 32x128b.warpx4) and issues the block-
//     scaled MMAs (tcgen05.mma kind::mxf4 K = 64, or kind::mxf8f6f4 K = 32;
//     a group's K range that ends halfway through a stage takes half of them),
//     releasing the stage with tcgen05.commit; two accumulators of 128 fp32
//     columns alternate between tiles.
//   warps 2-5: epilogue. Each warp reads its 32 lanes (rows) of the
//     finished accumulator (tcgen05.ld 32x32b), converts and stores the
//     valid rows and columns of the tile, and hands the accumulator back.
//   warps 6-7 only help build the group plan.
// Every wait on an mbarrier gives up after 4 s of global time; the CTA then
// records MXFP4_ECUDA, waits (bounded) for its loads and MMAs in flight,
// frees the tensor memory and exits.

namespace mxfp4 {

constexpr int GM_BM = 128, GM_BN = 128;  // tile rows, tile columns
constexpr int GM_KU = 128;               // K elements per scale atom column (4 blocks of 32): the unit of K ranges
constexpr int GM_THREADS = 256;  // 8 warps: producer, MMA, 4 epilogue, 2 that only build the group plan
constexpr uint32_t GM_TMEM_COLS = 512;  // 2 accumulators x 128 + scale atoms of every stage
constexpr uint32_t GM_SF_COL0 = 256;    // first tensor-memory column of the scale atoms

template <int FMT>
struct GmFmt;
template <>
struct GmFmt<MXFP4_ELEM_E2M1> {
    static constexpr int BK = 256;         // K elements per stage (128-byte rows)
    static constexpr int STAGES = 6;
    static constexpr int MMA_K = 64;       // kind::mxf4: K = 64 (32 bytes) per MMA
    static constexpr uint32_t AB_FMT = 1;  // E2M1 in the kind::mxf4 encoding
};
template <>
struct GmFmt<MXFP4_ELEM_E4M3> {
    static constexpr int BK = 128;
    static constexpr int STAGES = 5;
    static constexpr int MMA_K = 32;       // kind::mxf8f6f4: K = 32 (32 bytes) per MMA
    static constexpr uint32_t AB_FMT = 0;  // E4M3
};
constexpr int GM_ROW_BYTES = 128;       // bytes of a tile row per stage, both formats
constexpr uint64_t GM_LAYOUT = 2;       // 128-byte swizzle (smem descriptor layout type)
constexpr uint32_t GM_SBO = 1024;       // 8 rows x 128 bytes

template <int FMT>
struct __align__(1024) GmSmem {
    static constexpr int S = GmFmt<FMT>::STAGES, TB = GM_BM * GM_ROW_BYTES, ATOMS = GmFmt<FMT>::BK / GM_KU;
    uint8_t a[S][TB];             // swizzled A tiles (1024-aligned)
    uint8_t b[S][TB];             // swizzled B tiles
    uint8_t sfa[S][512 * ATOMS];  // A's scale atoms of each stage
    uint8_t sfb[S][512 * ATOMS];  // B's scale atoms of each stage
    unsigned long long full[S], empty[S], acc_full[2], acc_empty[2], done;
    uint32_t tmem_base;
    int err;
};

// Kernel arguments (device pointers; byte strides).
struct GmArgs {
    const uint8_t* sfa;   // A scales, MMA layout of [a_rows][k_blocks]
    const uint8_t* sfb;   // B scales (GROUP_M: per group, sfb_group_bytes apart)
    void* d;
    const int64_t* group_list;
    int32_t* status;
    int64_t a_rows;       // rows of A (GROUP_M: tokens; GROUP_K: M)
    int64_t n;            // N (columns of D, rows of one B)
    int64_t k;            // GROUP_M: K; GROUP_K: k_alloc
    int64_t ldd;          // D row stride in elements
    int64_t sfb_group_bytes;
    int64_t k_rows;       // GROUP_K: the rows (tokens) the group list partitions
    int32_t num_groups;
    int32_t gl_type;
    int32_t d_f32;        // D is fp32 (else bf16)
    int32_t group_k;      // 1: GROUP_K, 0: GROUP_M
};

struct GmMaps {
    CUtensorMap a, b;     // A [a_rows][k bytes]; B [G * N or N][k bytes]
};

__device__ __forceinline__ uint64_t gm_smem_desc(uint32_t saddr, uint64_t layout, uint32_t sbo)
{
    // start address, leading byte offset 16 (unused by swizzled K-major
    // layouts), stride byte offset between 8-row groups, descriptor version 1
    // (sm_100), base offset 0, layout type in the top three bits
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) |
           ((uint64_t)1 << 46) | (layout << 61);
}

// The 512-byte scale atom (32 rows of 16 bytes, no swizzle) as the source of
// a tcgen05.cp 32x128b: core matrices of 8 rows x 16 bytes, 128 bytes apart.
__device__ __forceinline__ uint64_t gm_sf_desc(uint32_t saddr)
{
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(128 >> 4) << 32) | ((uint64_t)1 << 46);
}

// Block-scaled instruction descriptor: E8M0 scales, K-major A and B, M = 128,
// N = 128, the scale bytes sf_id of each 32-bit tensor-memory word.
__device__ __forceinline__ uint32_t gm_idesc(uint32_t ab_fmt, uint32_t sf_id)
{
    return (sf_id << 4) | (ab_fmt << 7) | (ab_fmt << 10) | ((uint32_t)(GM_BN >> 3) << 17) | (1u << 23) |
           ((uint32_t)(GM_BM >> 4) << 24) | (sf_id << 29);
}

template <int FMT>
__device__ __forceinline__ void gm_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t acc)
{
    if constexpr (FMT == MXFP4_ELEM_E2M1) {
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
            "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc), "r"(sfa_tmem), "r"(sfb_tmem)
            : "memory");
    } else {
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
            "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc), "r"(sfa_tmem), "r"(sfb_tmem)
            : "memory");
    }
}

__device__ __forceinline__ void gm_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void gm_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void gm_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 consecutive fp32 accumulator columns of this thread's tensor-memory lane.
__device__ __forceinline__ void gm_ld32(uint32_t taddr, uint32_t (&v)[32])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
          "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]),
          "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
          "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// 2-D TMA load of a byte tile (box of 128 bytes x 128 rows, 128-byte
// swizzle); the inner coordinate is a multiple of 64 bytes.
__device__ __forceinline__ void gm_tma_load(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(map), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

// Tile t of the CTA's sequence -> (group g, first row of A, A rows of the
// tile that are valid, first column n0, D base row, K range of the group).
struct GmTile {
    int g;
    int64_t a_row0;   // first A row of the tile
    int64_t d_row0;   // first D row (GROUP_K: within D_g)
    int rows;         // valid rows (<= 128)
    int64_t n0;
    int64_t k0;       // first K element of the group's range
    int ku;           // K units (GM_KU elements) of the range
};

// The plan (GROUP_M): s_tpre[g] = sum_{j<g} ceil(m_j / 128) row tiles,
// s_rst[g] = the group's first row (build_plan<128>); GROUP_K: s_tpre[g] =
// sum_{j<g} ceil(n_j / 128) = K0_g / 128, s_rst unused.
__device__ __forceinline__ GmTile gm_tile(const GmArgs& a, const int32_t* s_tpre, const int32_t* s_rst,
                                          int64_t t, int64_t n_nt, int64_t n_mt)
{
    GmTile r;
    const int64_t nt = t % n_nt, mt = t / n_nt;
    r.n0 = nt * GM_BN;
    if (a.group_k) {
        const int64_t g = mt / n_mt, mi = mt - g * n_mt;
        r.g = (int)g;
        r.a_row0 = mi * GM_BM;
        r.d_row0 = mi * GM_BM;
        r.rows = (int)min((int64_t)GM_BM, a.a_rows - r.a_row0);
        r.k0 = (int64_t)s_tpre[g] * GM_KU;
        r.ku = s_tpre[g + 1] - s_tpre[g];
    } else {
        int lo = 0, hi = a.num_groups - 1;  // largest g with s_tpre[g] <= mt (skips empty groups)
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if ((int64_t)s_tpre[mid] <= mt)
                lo = mid;
            else
                hi = mid - 1;
        }
        r.g = lo;
        r.a_row0 = (int64_t)s_rst[lo] + (mt - s_tpre[lo]) * GM_BM;
        r.d_row0 = r.a_row0;
        r.rows = (int)min((int64_t)GM_BM, (int64_t)s_rst[lo + 1] - r.a_row0);
        r.k0 = 0;
        r.ku = (int)(a.k / GM_KU);
    }
    return r;
}

template <int FMT, bool GROUP_K, bool F32OUT>
__global__ void __launch_bounds__(GM_THREADS, 1) gmm_kernel(const __grid_constant__ GmMaps maps, const GmArgs a)
{
    using F = GmFmt<FMT>;
    constexpr int S = F::STAGES;
    constexpr int ATOMS = F::BK / GM_KU;               // scale atom columns per stage
    constexpr int MMA_PER_UNIT = GM_KU / F::MMA_K;     // MMAs per K unit
    constexpr uint32_t TB = GM_BM * GM_ROW_BYTES;
    extern __shared__ __align__(1024) uint8_t gm_dyn[];
    uint8_t* base = gm_dyn + ((1024u - (smem_addr(gm_dyn) & 1023u)) & 1023u);
    GmSmem<FMT>& sm = *reinterpret_cast<GmSmem<FMT>*>(base);
    int32_t* s_tpre = reinterpret_cast<int32_t*>(base + sizeof(GmSmem<FMT>));
    int32_t* s_rst = s_tpre + a.num_groups + 1;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) {
        sm.err = 0;
        for (int s = 0; s < S; ++s) {
            mbar_init(smem_addr(&sm.full[s]), 1 + 32);  // the TMA transaction + each producer lane's copies
            mbar_init(smem_addr(&sm.empty[s]), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_addr(&sm.acc_full[i]), 1);
            mbar_init(smem_addr(&sm.acc_empty[i]), 4);
        }
        mbar_init(smem_addr(&sm.done), 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(&sm.tmem_base)),
                     "r"(GM_TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
        gm_fence_before();
    }
    // the group plan: a KArgs view of the group list for build_plan
    KArgs pa;
    memset(&pa, 0, sizeof(pa));
    pa.group_list = a.group_list;
    pa.num_groups = a.num_groups;
    pa.gl_type = a.gl_type;
    pa.rows = GROUP_K ? a.k_rows : a.a_rows;
    // s_tpre[g] = sum_{j<g} ceil(n_j / 128); valid iff the list partitions pa.rows
    const int64_t units = build_plan<128>(pa, s_tpre, s_rst);  // contains __syncthreads
    gm_fence_after();
    const uint32_t tmem = sm.tmem_base;
    // GROUP_K: the groups' padded K slots must fit in k
    const bool ok = units >= 0 && (!GROUP_K || units * GM_KU <= a.k);
    if (blockIdx.x == 0 && tid == 0 && a.status)
        *a.status = ok ? MXFP4_OK : MXFP4_EINVAL;

    const int64_t n_nt = (a.n + GM_BN - 1) / GM_BN;
    const int64_t n_mt = (a.a_rows + GM_BM - 1) / GM_BM;
    const int64_t tiles = !ok ? 0 : GROUP_K ? (int64_t)a.num_groups * n_mt * n_nt : units * n_nt;
    const int64_t kblocks = a.k / 32;

    if (warp == 0) {
        // ---- producer
        int s = 0;
        uint32_t ph = 0, issued = 0;  // issued: bit s = stage s has had a load
        for (int64_t t = blockIdx.x; t < tiles && !sm.err; t += gridDim.x) {
            const GmTile tl = gm_tile(a, s_tpre, s_rst, t, n_nt, n_mt);
            const int64_t brow0 = GROUP_K ? tl.n0 : (int64_t)tl.g * a.n + tl.n0;
            const uint8_t* sfb = a.sfb + (GROUP_K ? 0 : (int64_t)tl.g * a.sfb_group_bytes);
            // this lane's rows r = lane + 32q of the tile: the address of
            // their four scale bytes in atom column 0 (MMA layout), or a
            // zero-filled copy past the last row
            const uint8_t* pa[4];
            const uint8_t* pb[4];
            uint32_t na = 0, nb = 0;  // bit q: row of A / B inside the matrix
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int r = lane + 32 * q;
                const int64_t ra = tl.a_row0 + r, rb = tl.n0 + r;
                pa[q] = a.sfa + (ra < a.a_rows ? srow_off_mma(ra, 0, kblocks) : 0);
                pb[q] = sfb + (rb < a.n ? srow_off_mma(rb, 0, kblocks) : 0);
                na |= (ra < a.a_rows ? 1u : 0u) << q;
                nb |= (rb < a.n ? 1u : 0u) << q;
            }
            const int nst = (tl.ku + ATOMS - 1) / ATOMS;  // stages of the tile
            for (int ks = 0; ks < nst; ++ks) {
                if (!__all_sync(FULL, mbar_wait(smem_addr(&sm.empty[s]), ph ^ 1u))) {
                    sm.err = 1;
                    break;
                }
                const int64_t kel = tl.k0 + (int64_t)ks * F::BK;  // first K element of the stage
                const int nu = min(ATOMS, tl.ku - ks * ATOMS);     // K units of the stage
                // tile row r's four bytes at 16 (r % 32) + 4 (r / 32) of each of
                // the stage's atoms (atom column kel / 128 + i, 512 bytes apart)
#pragma unroll
                for (int i = 0; i < ATOMS; ++i) {
                    const int64_t jo = (kel / GM_KU + i) * 512;
                    const uint32_t da = smem_addr(sm.sfa[s]) + 512 * i + 16 * lane;
                    const uint32_t db = smem_addr(sm.sfb[s]) + 512 * i + 16 * lane;
                    const uint32_t ua = i < nu ? na : 0u, ub = i < nu ? nb : 0u;  // a unit past the range: zeros
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(da + 4 * q),
                                     "l"(pa[q] + ((ua >> q) & 1u ? jo : 0)), "r"((ua >> q) & 1u ? 4u : 0u)
                                     : "memory");
                        asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(db + 4 * q),
                                     "l"(pb[q] + ((ub >> q) & 1u ? jo : 0)), "r"((ub >> q) & 1u ? 4u : 0u)
                                     : "memory");
                    }
                }
                asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_addr(&sm.full[s]))
                             : "memory");
                if (lane == 0) {
                    const uint32_t bar = smem_addr(&sm.full[s]);
                    mbar_expect_tx(bar, 2 * TB);
                    const int kx = (int)(kel * GM_ROW_BYTES / F::BK);
                    gm_tma_load(smem_addr(sm.a[s]), &maps.a, kx, (int)tl.a_row0, bar);
                    gm_tma_load(smem_addr(sm.b[s]), &maps.b, kx, (int)brow0, bar);
                }
                issued |= 1u << s;
                if (++s == S) {
                    s = 0;
                    ph ^= 1u;
                }
            }
        }
        // every load issued lands before the CTA leaves: the last load of
        // stage i had the parity of its turn (i < s: this round, else the
        // previous one); waits on consumed stages return at once
        if (lane == 0)
            for (int i = 0; i < S; ++i)
                if (issued & (1u << i))
                    (void)mbar_wait(smem_addr(&sm.full[i]), i < s ? ph : ph ^ 1u);
        __syncwarp();
    } else if (warp == 1) {
        // ---- MMA issuer (lane 0)
        if (lane == 0) {
            int s = 0, acc = 0;
            uint32_t ph = 0, aph = 0;
            for (int64_t t = blockIdx.x; t < tiles && !sm.err; t += gridDim.x) {
                const GmTile tl = gm_tile(a, s_tpre, s_rst, t, n_nt, n_mt);
                if (!mbar_wait(smem_addr(&sm.acc_empty[acc]), aph ^ 1u)) {
                    sm.err = 1;
                    break;
                }
                gm_fence_after();
                const uint32_t d_tmem = tmem + (uint32_t)(acc * GM_BN);
                const int nst = (tl.ku + ATOMS - 1) / ATOMS;
                for (int ks = 0; ks < nst; ++ks) {
                    if (!mbar_wait(smem_addr(&sm.full[s]), ph)) {
                        sm.err = 1;
                        break;
                    }
                    gm_fence_after();
                    // the scale atoms were written by the producer's copies
                    // (generic proxy); tcgen05.cp reads them in the async proxy
                    fence_async_smem();
                    const uint32_t sf_col = tmem + GM_SF_COL0 + (uint32_t)(8 * ATOMS * s);
#pragma unroll
                    for (int i = 0; i < ATOMS; ++i) {
                        asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(sf_col + 4u * i),
                                     "l"(gm_sf_desc(smem_addr(sm.sfa[s]) + 512 * i))
                                     : "memory");
                        asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(sf_col + 4u * (ATOMS + i)),
                                     "l"(gm_sf_desc(smem_addr(sm.sfb[s]) + 512 * i))
                                     : "memory");
                    }
                    const uint64_t ad = gm_smem_desc(smem_addr(sm.a[s]), GM_LAYOUT, GM_SBO);
                    const uint64_t bd = gm_smem_desc(smem_addr(sm.b[s]), GM_LAYOUT, GM_SBO);
                    const int nmma = min(ATOMS, tl.ku - ks * ATOMS) * MMA_PER_UNIT;
                    for (int kk = 0; kk < nmma; ++kk) {
                        // 32 bytes of K per MMA: the start address moves by 2 units of 16
                        // bytes; its first scale block kk * MMA_K / 32 is byte (block % 4)
                        // of atom (block / 4)
                        const int blk = kk * (F::MMA_K / 32);
                        const uint32_t ai = (uint32_t)(blk >> 2);
                        gm_mma<FMT>(d_tmem, ad + 2u * kk, bd + 2u * kk, gm_idesc(F::AB_FMT, (uint32_t)(blk & 3)),
                                    sf_col + 4u * ai, sf_col + 4u * (ATOMS + ai), (ks > 0 || kk > 0) ? 1u : 0u);
                    }
                    gm_commit(smem_addr(&sm.empty[s]));  // the stage is free once these MMAs have read it
                    if (++s == S) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                gm_commit(smem_addr(&sm.acc_full[acc]));  // ku == 0: completes at once, D of the tile is zero
                if (++acc == 2) {
                    acc = 0;
                    aph ^= 1u;
                }
            }
            // every MMA issued has completed before the tensor memory is freed
            gm_commit(smem_addr(&sm.done));
            (void)mbar_wait(smem_addr(&sm.done), 0);
        }
        __syncwarp();
    } else if (warp < 6) {
        // ---- epilogue: warp w reads tensor-memory lanes 32 (w % 4) .. + 31
        // (exactly four warps: acc_empty counts four arrivals per tile)
        const int quad = warp & 3;
        const int r = 32 * quad + lane;  // tile row of this thread
        int acc = 0;
        uint32_t aph = 0;
        for (int64_t t = blockIdx.x; t < tiles && !sm.err; t += gridDim.x) {
            const GmTile tl = gm_tile(a, s_tpre, s_rst, t, n_nt, n_mt);
            if (!__all_sync(FULL, mbar_wait(smem_addr(&sm.acc_full[acc]), aph))) {
                sm.err = 1;
                break;
            }
            gm_fence_after();
            const bool zero = tl.ku == 0;
            const bool row_ok = r < tl.rows;
            const int64_t drow = (GROUP_K ? (int64_t)tl.g * a.a_rows : 0) + tl.d_row0 + r;
#pragma unroll 1
            for (int c = 0; c < GM_BN / 32; ++c) {
                uint32_t v[32];
                __syncwarp();  // tcgen05.ld is warp-collective
                gm_ld32(tmem + ((uint32_t)(32 * quad) << 16) + (uint32_t)(acc * GM_BN + 32 * c), v);
                const int64_t col = tl.n0 + 32 * c;
                if (!row_ok || col >= a.n)
                    continue;
                if (zero) {
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        v[i] = 0u;
                }
                const int ncol = (int)min((int64_t)32, a.n - col);
                if constexpr (F32OUT) {
                    float* dp = static_cast<float*>(a.d) + drow * a.ldd + col;
                    if (ncol == 32) {
#pragma unroll
                        for (int i = 0; i < 32; i += 4)
                            *reinterpret_cast<uint4*>(dp + i) = make_uint4(v[i], v[i + 1], v[i + 2], v[i + 3]);
                    } else {
                        for (int i = 0; i < ncol; ++i)
                            dp[i] = __uint_as_float(v[i]);
                    }
                } else {
                    uint16_t* dp = static_cast<uint16_t*>(a.d) + drow * a.ldd + col;
                    uint32_t h[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(h[i]) : "f"(__uint_as_float(v[2 * i + 1])),
                            "f"(__uint_as_float(v[2 * i])));
                    if (ncol == 32) {
#pragma unroll
                        for (int i = 0; i < 16; i += 4)
                            *reinterpret_cast<uint4*>(dp + 2 * i) = make_uint4(h[i], h[i + 1], h[i + 2], h[i + 3]);
                    } else {
                        for (int i = 0; i < ncol; ++i)
                            dp[i] = (uint16_t)(h[i >> 1] >> (16 * (i & 1)));
                    }
                }
            }
            gm_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(smem_addr(&sm.acc_empty[acc]));
            if (++acc == 2) {
                acc = 0;
                aph ^= 1u;
            }
        }
    }

    __syncthreads();
    if (tid == 0 && sm.err && a.status)
        *a.status = MXFP4_ECUDA;
    if (warp == 1) {
        gm_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(GM_TMEM_COLS) : "memory");
    }
}

}  // namespace mxfp4
