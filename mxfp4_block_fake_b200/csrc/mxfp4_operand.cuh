// mxfp4_operand.cuh -- the column-wise MXFP4 operand of a block-scaled GEMM
// that contracts over the rows (included by mxfp4.cu; shares its helpers).
//
// A grouped linear layer's weight-gradient GEMM multiplies, per MoE group,
// the column-wise quantised activations and gradients, contracting over the
// group's tokens (MindSpore hyper-parallel fake_w4a8_gmm_func.py,
// FakeW4A8GroupedLinear._select_operands, layout "TN": both operands are the
// column-wise views, transposed). A tensor-core operand must be K-major, so
// the column-wise codes are written transposed: for column c, the 32 codes
// of a column-wise block follow each other along a row of the output, two
// per byte (the first row in the low nibble). Each group's K range is padded
// to a multiple of 128 rows (four blocks, one column of 128 x 4 scale atoms),
// so that every group starts on an atom boundary:
//   codes   [cols][k_alloc / 2] bytes; group g's rows start at K slot
//           K0_g = sum_{j<g} 128 ceil(n_j / 128); slots past n_g hold 0;
//   scales  the [cols][k_alloc / 32] E8M0 matrix in the MMA scale-factor
//           layout (atoms of 128 x 4, 512 bytes, atom rows in order); the
//           padding blocks of a group get 127 (2^0: their codes are 0).
// The per-group sub-matrices are then ordinary block-scaled operands at a
// row stride of k_alloc / 2 bytes.
//
// One thread per (block pair, column pair): 64 rows of one 32-bit word (two
// bf16 columns; two 16-bit loads when x's rows are not 4-byte aligned); a
// warp covers 64 adjacent columns, so every load instruction of the warp
// reads one 128-byte row segment. Per column and
// block: the amax, the scale exponent, the codes of 32 rows by the nudged
// hardware convert (the same argument as the row-wise producer: the nudge
// turns the convert's ties-to-even into the codebook's ties-up for bf16
// inputs with -125 <= k <= 16), written as one 32-byte row segment per
// column and block pair. Blocks off that k range (non-finite, huge or
// subnormal scales) take the table path of the general kernels.

namespace mxfp4 {

constexpr int OP_KPAD = 128;  // rows per padded K unit (one scale-atom column)

// The halves of eight words of one column pair (rows 8m..8m+7) as two
// 8-element bf16 vectors: the low halves (column c) and the high halves
// (column c + 1), in row order.
__device__ __forceinline__ void split_pair_rows(const uint32_t* w, uint4& lo, uint4& hi)
{
    lo = make_uint4(__byte_perm(w[0], w[1], 0x5410), __byte_perm(w[2], w[3], 0x5410), __byte_perm(w[4], w[5], 0x5410),
                    __byte_perm(w[6], w[7], 0x5410));
    hi = make_uint4(__byte_perm(w[0], w[1], 0x7632), __byte_perm(w[2], w[3], 0x7632), __byte_perm(w[4], w[5], 0x7632),
                    __byte_perm(w[6], w[7], 0x7632));
}

template <int MODE, bool GROUPS>
__global__ void __launch_bounds__(NTHREADS) col_operand_kernel(const KArgs a)
{
    extern __shared__ int32_t s_op_plan[];
    __shared__ uint32_t s_lut[64];
    if (threadIdx.x < 64)
        s_lut[threadIdx.x] = lut_entry(threadIdx.x);
    // s_apre[g]: group g's first atom column (K0_g / 128); s_rst[g]: its first row
    int32_t* s_apre = s_op_plan;
    int32_t* s_rst = s_op_plan + (GROUPS ? a.num_groups + 1 : 0);
    int64_t natoms;
    if constexpr (GROUPS) {
        natoms = build_plan<OP_KPAD>(a, s_apre, s_rst);  // contains __syncthreads
        const bool ok = natoms >= 0 && natoms * OP_KPAD <= a.k_alloc;
        if (blockIdx.x == 0 && threadIdx.x == 0 && a.status)
            *a.status = ok ? MXFP4_OK : MXFP4_EINVAL;
        if (!ok)
            return;
    } else {
        __syncthreads();
        natoms = (a.rows + OP_KPAD - 1) / OP_KPAD;
    }
    const uint32_t glutb = smem_addr(s_lut) - 0x2C000000u;
    const int64_t npairs = (a.cols + 1) / 2;
    const int64_t total = natoms * (OP_KPAD / 64) * npairs;
    const int64_t kbytes = a.k_alloc / 2;   // bytes per codes row
    const int64_t nsc = a.k_alloc / 32;     // scale columns
    const uint16_t* xb = static_cast<const uint16_t*>(a.x);
    // a column pair is one aligned 32-bit word when x is 4-byte aligned and ld
    // even; otherwise it is read as two 16-bit elements
    const bool words = ((uintptr_t)a.x & 3u) == 0 && (a.ld & 1) == 0;
    for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u < total; u += (int64_t)gridDim.x * blockDim.x) {
        const int64_t bp = u / npairs, cp = u - bp * npairs;
        const int64_t c = 2 * cp;
        const bool two = c + 1 < a.cols;
        int64_t row0, gend;
        if constexpr (GROUPS) {
            const int32_t at = (int32_t)(bp >> 1);
            int lo = 0, hi = a.num_groups - 1;  // largest g with s_apre[g] <= at (skips empty groups)
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (s_apre[mid] <= at)
                    lo = mid;
                else
                    hi = mid - 1;
            }
            row0 = (int64_t)s_rst[lo] + (bp - 2 * (int64_t)s_apre[lo]) * 64;
            gend = s_rst[lo + 1];
        } else {
            row0 = bp * 64;
            gend = a.rows;
        }
        uint32_t q[2][8];  // [column][block * 4 + word]: the 32-byte code segment of each column
        uint32_t e8[2][2];
#pragma unroll
        for (int b = 0; b < 2; ++b) {
            const int64_t r0 = row0 + 32 * b;
            const int n = (int)max((int64_t)0, min((int64_t)32, gend - r0));
            if (n == 0) {  // a padding block of the group
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    q[0][4 * b + i] = q[1][4 * b + i] = 0u;
                e8[0][b] = e8[1][b] = 127u;
                continue;
            }
            uint32_t w[32];
#pragma unroll
            for (int r = 0; r < 32; ++r) {
                const uint16_t* p = xb + (r0 + r) * a.ld + c;
                w[r] = r >= n ? 0u
                       : !two ? (uint32_t)__ldcs(p)
                       : words ? __ldcs(reinterpret_cast<const unsigned int*>(p))
                               : (uint32_t)__ldcs(p) | ((uint32_t)__ldcs(p + 1) << 16);
            }
            uint32_t m2 = 0;
#pragma unroll
            for (int r = 0; r < 32; ++r)
                m2 = vmax2(m2, w[r] & 0x7FFF7FFFu);
            const uint32_t A[2] = {m2 << 16, m2 & 0xFFFF0000u};
            int k[2];
            bool fast[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                k[h] = block_kt<MODE>(A[h], a.thr);
                fast[h] = k_fast_bf(k[h]);
                e8[h][b] = fast[h] ? (uint32_t)(k[h] + 127) : e8_of(A[h], k[h]);
            }
            if (fast[0] && fast[1]) {
                const float invn_lo = inv_nudged(k[0]), invn_hi = inv_nudged(k[1]);
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    float ylo[8], yhi[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        nudged_pair(w[8 * m + i], invn_lo, invn_hi, ylo[i], yhi[i]);
                    q[0][4 * b + m] = e2m1x8(ylo);
                    q[1][4 * b + m] = e2m1x8(yhi);
                }
            } else {
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    uint4 vlo, vhi;
                    split_pair_rows(w + 8 * m, vlo, vhi);
                    q[0][4 * b + m] = general_chunk_one(vlo, A[0], a.mode, a.thr, glutb).nibs;
                    q[1][4 * b + m] = general_chunk_one(vhi, A[1], a.mode, a.thr, glutb).nibs;
                }
            }
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            if (h == 1 && !two)
                break;
            uint4* dst = reinterpret_cast<uint4*>(a.codes_col + (c + h) * kbytes + 32 * bp);
            if (a.codes_col) {
                __stcs(dst, make_uint4(q[h][0], q[h][1], q[h][2], q[h][3]));
                __stcs(dst + 1, make_uint4(q[h][4], q[h][5], q[h][6], q[h][7]));
            }
            if (a.scales_col)
                *reinterpret_cast<uint16_t*>(a.scales_col + srow_off_mma(c + h, 2 * bp, nsc)) =
                    (uint16_t)(e8[h][0] | (e8[h][1] << 8));
        }
    }
}


// ---------------------------------------------------------------------------
// The same operand from TMA-staged tiles (bf16, cols % 32 == 0, x addressable
// by TMA): a tile is one pair of 32-row blocks of the padded K numbering (64
// rows; fewer, or none, at a group's end) by 256 columns, CTA b taking tiles
// b, b + G, ... . Warp OPS_PRODUCER's lane 0 loads each block of a tile as
// four 64 x 32 boxes (128-byte swizzle) into a ring of OPS_STAGES stages;
// the eight compute warps release a stage with one arrival each on its
// "empty" mbarrier. Compute warp w owns tile columns 32w..32w+31: lane =
// column pair p (lane & 15) x row half h (lane >> 4) over rows 8i + 4h + q
// (i = 0..7, q = 0..3), the two blocks' amaxes by one shuffle each. Four
// consecutive rows of one column give one 16-bit piece of the K-major codes
// (nudged hardware convert); after one exchange of pieces between the two
// half-warps, lane h writes column 2p + h's 32 bytes (both blocks, one
// sector) with one 32-byte store and its two scale bytes with one 16-bit
// store. Every wait is bounded (SG_WAIT_NS).
// ---------------------------------------------------------------------------

constexpr int OPS_STAGES = 3;
constexpr int OPS_COMPUTE_WARPS = SG_COLS / 32;                 // 8
constexpr int OPS_THREADS = 32 * (OPS_COMPUTE_WARPS + 1);      // + the producer warp
constexpr int OPS_PRODUCER = OPS_COMPUTE_WARPS;
constexpr int OPS_TILE_BYTES = 2 * SG_TILE_BYTES;              // two blocks of 32 rows x 256 columns

struct __align__(1024) OpsSmem {
    uint8_t tiles[OPS_STAGES][OPS_TILE_BYTES];  // [block][slab][32 rows][128 bytes], swizzled
    int4 info[OPS_STAGES];                      // row0, rows (0..64), col0, block pair of each stage's tile
    uint32_t lut[64];
    unsigned long long full[OPS_STAGES];
    unsigned long long empty[OPS_STAGES];
    int err;
};

// 32-byte store (eight words) to global memory, streaming.
__device__ __forceinline__ void st_cs_v8w(void* p, const uint32_t (&v)[8])
{
    asm volatile("st.global.cs.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(v[0]), "r"(v[1]),
                 "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
                 : "memory");
}

template <int MODE, bool GROUPS>
__global__ void __launch_bounds__(OPS_THREADS, 2) col_operand_staged_kernel(const __grid_constant__ StagedMaps maps,
                                                                            const KArgs a)
{
    extern __shared__ __align__(1024) uint8_t s_dyn[];
    uint8_t* s_base = s_dyn + ((1024u - (smem_addr(s_dyn) & 1023u)) & 1023u);
    OpsSmem& sm = *reinterpret_cast<OpsSmem*>(s_base);
    int32_t* s_apre = reinterpret_cast<int32_t*>(s_base + sizeof(OpsSmem));  // group g's first atom column
    int32_t* s_rst = s_apre + (GROUPS ? a.num_groups + 1 : 0);              // group g's first row
    volatile int* err = &sm.err;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid < 64)
        sm.lut[tid] = lut_entry(tid);
    if (tid == 0) {
        sm.err = 0;
        for (int s = 0; s < OPS_STAGES; ++s) {
            mbar_init(smem_addr(&sm.full[s]), 1);
            mbar_init(smem_addr(&sm.empty[s]), OPS_COMPUTE_WARPS);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    int64_t natoms;
    if constexpr (GROUPS) {
        natoms = build_plan<OP_KPAD>(a, s_apre, s_rst);  // contains __syncthreads
        const bool ok = natoms >= 0 && natoms * OP_KPAD <= a.k_alloc;
        if (blockIdx.x == 0 && tid == 0 && a.status)
            *a.status = ok ? MXFP4_OK : MXFP4_EINVAL;
        if (!ok)
            return;
    } else {
        __syncthreads();
        natoms = (a.rows + OP_KPAD - 1) / OP_KPAD;
    }
    const uint32_t ntiles = (uint32_t)(2 * natoms) * a.n_ct;  // block pairs x column tiles
    const uint32_t n = blockIdx.x < ntiles ? (ntiles - blockIdx.x + gridDim.x - 1) / gridDim.x : 0u;
    uint32_t issued = 0;

    if (warp == OPS_PRODUCER) {
        // tile t -> (block pair, column tile) and its rows
        auto locate = [&](uint32_t t) {
            const uint32_t bp = t / a.n_ct, ct = t - bp * a.n_ct;
            int64_t row0, gend;
            if constexpr (GROUPS) {
                const int32_t at = (int32_t)(bp >> 1);
                int lo = 0, hi = a.num_groups - 1;  // largest g with s_apre[g] <= at (skips empty groups)
                while (lo < hi) {
                    const int mid = (lo + hi + 1) >> 1;
                    if (s_apre[mid] <= at)
                        lo = mid;
                    else
                        hi = mid - 1;
                }
                row0 = (int64_t)s_rst[lo] + ((int64_t)bp - 2 * (int64_t)s_apre[lo]) * 64;
                gend = s_rst[lo + 1];
            } else {
                row0 = (int64_t)bp * 64;
                gend = a.rows;
            }
            const int rows = (int)max((int64_t)0, min((int64_t)64, gend - row0));
            return make_int4((int)(rows > 0 ? row0 : 0), rows, (int)(ct * SG_COLS), (int)bp);
        };
        auto load = [&](uint32_t j) {  // lane 0: the CTA's j-th tile into stage j mod OPS_STAGES
            const int s = (int)(j % OPS_STAGES);
            const int4 inf = locate(blockIdx.x + j * gridDim.x);
            sm.info[s] = inf;
            const uint32_t bar = smem_addr(&sm.full[s]);
            const int nb = (inf.y + 31) >> 5;  // blocks with rows: 0, 1 or 2
            if (nb == 0) {
                mbar_arrive(bar);  // a padding pair: nothing to load
            } else {
                mbar_expect_tx(bar, (uint32_t)(nb * SG_TILE_BYTES));
                for (int b = 0; b < nb; ++b)
                    for (int sl = 0; sl < 4; ++sl)
                        tma_load_slab(smem_addr(sm.tiles[s] + b * SG_TILE_BYTES + sl * SG_SLAB_BYTES), &maps.x,
                                      inf.z + sl * SG_SLAB_COLS, inf.x + 32 * b, bar);
            }
            ++issued;
        };
        if (lane == 0) {
            for (uint32_t j = 0; j < n && j < (uint32_t)OPS_STAGES; ++j)
                load(j);
            for (uint32_t j = OPS_STAGES; j < n; ++j) {
                // round r >= 1 of a stage waits for the release of round r - 1
                if (*err || !mbar_wait(smem_addr(&sm.empty[j % OPS_STAGES]), ((j / OPS_STAGES) - 1) & 1u)) {
                    *err = 1;
                    break;
                }
                load(j);
            }
        }
    } else {
        const uint32_t glutb = smem_addr(sm.lut) - 0x2C000000u;
        const int p = lane & 15, h = lane >> 4;
        const int cpair = 32 * warp + 2 * p;
        const uint32_t cchunk = 4 * (warp & 1) + (p >> 2);
        uint32_t yo[4];  // per q: byte offset of row 4h + q of block 0 in a stage
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint32_t rq = 4 * h + q;
            yo[q] = (uint32_t)(warp >> 1) * SG_SLAB_BYTES + rq * 128 + ((cchunk ^ rq) << 4) + 4 * (p & 3);
        }
        const int64_t kbytes = a.k_alloc / 2, nsc = a.k_alloc / 32;
        for (uint32_t j = 0; j < n; ++j) {
            const int s = (int)(j % OPS_STAGES);
            if (!__all_sync(FULL, mbar_wait(smem_addr(&sm.full[s]), (j / OPS_STAGES) & 1u))) {
                if (lane == 0)
                    *err = 1;
                break;
            }
            const int4 inf = sm.info[s];
            const int rows = inf.y, col0 = inf.z;
            const int64_t bp = inf.w;
            const uint8_t* tile = sm.tiles[s];
            if (col0 + 32 * warp < a.cols) {
                // the lane's 32 words: word 4i + q is row 8i + 4h + q of the pair
                uint32_t w[32];
#pragma unroll
                for (int i = 0; i < 8; ++i)
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        w[4 * i + q] = 8 * i + 4 * h + q < rows
                                           ? sm_ld32(tile, (uint32_t)((i >> 2) * SG_TILE_BYTES + (i & 3) * 1024) + yo[q])
                                           : 0u;
                uint32_t pc[2][2][4];  // [column lo/hi][block][i & 3]: 16-bit pieces (rows 8i + 4h .. + 3)
                uint32_t e8[2][2];     // [column][block]
#pragma unroll
                for (int b = 0; b < 2; ++b) {
                    uint32_t m2 = 0;
#pragma unroll
                    for (int i = 16 * b; i < 16 * b + 16; ++i)
                        m2 = vmax2(m2, w[i] & 0x7FFF7FFFu);
                    m2 = vmax2(m2, __shfl_xor_sync(FULL, m2, 16));
                    const uint32_t A_lo = m2 << 16, A_hi = m2 & 0xFFFF0000u;
                    const int k_lo = block_kt<MODE>(A_lo, a.thr), k_hi = block_kt<MODE>(A_hi, a.thr);
                    const bool blk = 32 * b < rows;  // a padding block: codes 0, scale 2^0
                    const bool fast = k_fast_bf(k_lo) && k_fast_bf(k_hi);
                    e8[0][b] = !blk ? 127u : fast ? (uint32_t)(k_lo + 127) : e8_of(A_lo, k_lo);
                    e8[1][b] = !blk ? 127u : fast ? (uint32_t)(k_hi + 127) : e8_of(A_hi, k_hi);
                    if (!blk) {
#pragma unroll
                        for (int m = 0; m < 4; ++m)
                            pc[0][b][m] = pc[1][b][m] = 0u;
                    } else if (fast) {
                        const float invn_lo = inv_nudged(k_lo), invn_hi = inv_nudged(k_hi);
#pragma unroll
                        for (int m = 0; m < 4; ++m) {
                            float ylo[4], yhi[4];
#pragma unroll
                            for (int q = 0; q < 4; ++q)
                                nudged_pair(w[16 * b + 4 * m + q], invn_lo, invn_hi, ylo[q], yhi[q]);
                            pc[0][b][m] = e2m1x4(ylo);
                            pc[1][b][m] = e2m1x4(yhi);
                        }
                    } else {
#pragma unroll
                        for (int m = 0; m < 4; m += 2) {
                            uint4 vlo, vhi;
                            split_pair_rows(w + 16 * b + 4 * m, vlo, vhi);
                            const uint32_t nlo = general_chunk_one(vlo, A_lo, a.mode, a.thr, glutb).nibs;
                            const uint32_t nhi = general_chunk_one(vhi, A_hi, a.mode, a.thr, glutb).nibs;
                            pc[0][b][m] = nlo & 0xFFFFu;
                            pc[0][b][m + 1] = nlo >> 16;
                            pc[1][b][m] = nhi & 0xFFFFu;
                            pc[1][b][m + 1] = nhi >> 16;
                        }
                    }
                }
                // lane h writes column cpair + h: it keeps its own pieces of
                // that column and receives the partner's (the partner sends
                // the pieces of the column it does not write)
                uint32_t give[4], got[4];
#pragma unroll
                for (int b = 0; b < 2; ++b)
#pragma unroll
                    for (int m = 0; m < 4; m += 2) {
                        const int o = h ^ 1;  // the column the partner writes
                        give[2 * b + m / 2] = (o == 0 ? pc[0][b][m] : pc[1][b][m]) |
                                              ((o == 0 ? pc[0][b][m + 1] : pc[1][b][m + 1]) << 16);
                    }
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    got[u] = __shfl_xor_sync(FULL, give[u], 16);
                // word m of block b: bytes 4m .. 4m + 3 = rows 8m .. 8m + 7:
                // the h = 0 half's piece then the h = 1 half's
                uint32_t out[8];
#pragma unroll
                for (int b = 0; b < 2; ++b)
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        const uint32_t mine = h == 0 ? pc[0][b][m] : pc[1][b][m];
                        const uint32_t theirs = (got[2 * b + m / 2] >> (16 * (m & 1))) & 0xFFFFu;
                        out[4 * b + m] = h == 0 ? (mine | (theirs << 16)) : (theirs | (mine << 16));
                    }
                const int64_t c = col0 + cpair + h;
                if (a.codes_col)
                    st_cs_v8w(a.codes_col + c * kbytes + 32 * bp, out);
                if (a.scales_col)
                    *reinterpret_cast<uint16_t*>(a.scales_col + srow_off_mma(c, 2 * bp, nsc)) =
                        (uint16_t)(h == 0 ? (e8[0][0] | (e8[0][1] << 8)) : (e8[1][0] | (e8[1][1] << 8)));
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(smem_addr(&sm.empty[s]));
        }
    }

    __syncthreads();
    if (warp == OPS_PRODUCER && lane == 0 && *err) {
        if (a.status)
            *a.status = MXFP4_ECUDA;
        for (uint32_t i = issued > (uint32_t)OPS_STAGES ? issued - OPS_STAGES : 0u; i < issued; ++i)
            (void)mbar_wait(smem_addr(&sm.full[i % OPS_STAGES]), (i / OPS_STAGES) & 1u);
    }
}

}  // namespace mxfp4
