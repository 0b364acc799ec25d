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

}  // namespace mxfp4
