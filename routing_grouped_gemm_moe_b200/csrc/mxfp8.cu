// MXFP8 block quantisation ("Ai2 rebuilds Olmo's training stack for
// trillion-parameter MoEs", "MXFP8 reduces compute and memory costs": an 8-bit
// float format with separate scaling for small blocks of values).
//
// Rule (OCP Microscaling Formats v1.0): a block of 32 values shares
// X = clamp(floor(log2(amax)) - 8, -127, 127), 8 being the largest exponent of
// E4M3 (X = 0 for an all-zero block); the scale byte is X + 127 (E8M0) and each
// value is stored as E4M3 of v * 2^-X, round-to-nearest-even, saturated to
// +-448.  floor(log2(amax)) is read from the exponent bits of the bf16 amax,
// so no logarithm is evaluated; v * 2^-X is exact in fp32.
#include "common.cuh"
#include "mx_encode.cuh"

namespace moe {

// axis = 1: one lane per 32-value block of a row (64 input bytes).
__global__ void __launch_bounds__(256) mx_rowwise_kernel(const uint16_t* __restrict__ x,
                                                         int64_t rows, int64_t cols,
                                                         uint8_t* __restrict__ codes,
                                                         uint8_t* __restrict__ scales) {
    const int64_t nblk_row = cols / 32;
    const int64_t total = rows * nblk_row;
    for (int64_t b = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; b < total;
         b += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t r = b / nblk_row, j = b - r * nblk_row;
        const uint4* src = reinterpret_cast<const uint4*>(x + r * cols + j * 32);
        uint32_t h[16];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint4 v = __ldg(src + q);
            h[4 * q] = v.x; h[4 * q + 1] = v.y; h[4 * q + 2] = v.z; h[4 * q + 3] = v.w;
        }
        scales[r * nblk_row + j] = mx_encode_row32(h, codes + r * cols + j * 32);
    }
}

// axis = 0 with groups: a CTA takes one 32-row block (restarted at each group
// start) x 256 columns.  The block is read row by row (each warp a contiguous
// 512-byte row segment) into shared memory, each thread then owns 2 columns
// (amax over the block's rows with one 16-bit-pair max per row, codes back
// into shared memory), and the codes leave row by row again.  Scales: one
// byte per (block, column).  The kernels are bound by instruction issue, not
// by DRAM, so their rate follows the SM clock.
constexpr int kMaxGroups = 1024;
constexpr int kColTile = 256;
constexpr int kColThreads = 128;

// Staged rows hold their 16-byte chunks (8 bf16) swizzled within each 128-byte
// group: chunk c sits at c ^ ((c >> 2) & 7).  The row-wise reads (8 threads on
// chunks 4j + q of one row, j = 0..7) and the column reads (consecutive column
// pairs) then fall on distinct banks.
__device__ __forceinline__ int tile_col(int col) {
    const int c = col >> 3;
    return 8 * (c ^ ((c >> 2) & 7)) + (col & 7);
}

// ROW: also the row-wise encoding of the same staged tile (each thread two
// (row, 32-column block) items), so that a tensor needed in both layouts is
// read once.
template <bool ROW>
__global__ void __launch_bounds__(kColThreads) mx_colwise_kernel(const uint16_t* __restrict__ x,
                                                                 int64_t rows, int64_t cols,
                                                                 const int32_t* __restrict__ goff,
                                                                 int ngroups, uint8_t* __restrict__ codes,
                                                                 uint8_t* __restrict__ scales,
                                                                 int32_t* status,
                                                                 uint8_t* __restrict__ rcodes,
                                                                 uint8_t* __restrict__ rscales) {
    __shared__ int s_off[kMaxGroups + 1];
    __shared__ int s_base[kMaxGroups + 1];
    __shared__ __align__(16) uint16_t tile[32][kColTile];
    __shared__ __align__(16) uint8_t ctile[32][kColTile];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp == 0) {
        load_group_offsets(goff, ngroups, rows, s_off, status);
        const int seg = (ngroups + 31) / 32;
        const int lo = min(ngroups, lane * seg), hi = min(ngroups, lo + seg);
        int local = 0;
        for (int g = lo; g < hi; ++g) local += max(0, s_off[g + 1] - s_off[g] + 31) / 32;
        int incl = local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        int run = incl - local;
        for (int g = lo; g < hi; ++g) {
            s_base[g] = run;
            run += max(0, s_off[g + 1] - s_off[g] + 31) / 32;
        }
        if (lane == 31) s_base[ngroups] = incl;
    }
    __syncthreads();
    const int nblk = s_base[ngroups];
    const int64_t nct = (cols + kColTile - 1) / kColTile;
    const int64_t total = static_cast<int64_t>(nblk) * nct;
    // work item w: block b (32 rows r0 .. r0 + nr of one group) x columns c0 ..
    struct Item { int b, r0, nr, ncol; int64_t c0; };
    auto locate = [&](int64_t w) {
        Item it;
        it.b = static_cast<int>(w / nct);
        it.c0 = (w - static_cast<int64_t>(it.b) * nct) * kColTile;
        int lo = 0, hi = ngroups - 1;
        while (lo < hi) {  // largest g with s_base[g] <= b
            const int mid = (lo + hi + 1) >> 1;
            if (s_base[mid] <= it.b) lo = mid; else hi = mid - 1;
        }
        it.r0 = s_off[lo] + (it.b - s_base[lo]) * 32;
        it.nr = min(s_off[lo + 1], it.r0 + 32) - it.r0;
        it.ncol = static_cast<int>(cols - it.c0 < kColTile ? cols - it.c0 : kColTile);  // multiple of 32
        return it;
    };
    // rows in as 16-byte vectors (a warp per 512-byte row segment); the next
    // item's vectors are loaded into registers while this one is encoded
    constexpr int kVec = 32 * (kColTile / 8) / kColThreads;
    uint4 pre[kVec];
    auto fetch = [&](const Item& it) {
#pragma unroll
        for (int j = 0; j < kVec; ++j) {
            const int i = threadIdx.x + kColThreads * j;
            const int r = i / (kColTile / 8), v = i % (kColTile / 8);
            pre[j] = (r < it.nr && 8 * v < it.ncol)
                         ? __ldg(reinterpret_cast<const uint4*>(x + static_cast<int64_t>(it.r0 + r) * cols + it.c0) + v)
                         : make_uint4(0, 0, 0, 0);
        }
    };
    if (blockIdx.x < total) fetch(locate(blockIdx.x));
    for (int64_t w = blockIdx.x; w < total; w += gridDim.x) {
        const Item it = locate(w);
        const int b = it.b, r0 = it.r0, nr = it.nr, ncol = it.ncol;
        const int64_t c0 = it.c0;
#pragma unroll
        for (int j = 0; j < kVec; ++j) {
            const int i = threadIdx.x + kColThreads * j;
            *reinterpret_cast<uint4*>(&tile[i / (kColTile / 8)][tile_col(8 * (i % (kColTile / 8)))]) = pre[j];
        }
        __syncthreads();
        if (w + gridDim.x < total) fetch(locate(w + gridDim.x));
        {
            const int c = 2 * threadIdx.x;  // this thread's two columns
            uint32_t m = 0;
            const int tc = tile_col(c);
#pragma unroll 8
            for (int r = 0; r < 32; ++r) m = mag_max2(m, *reinterpret_cast<const uint32_t*>(&tile[r][tc]));
            const int X0 = block_exponent(m & 0xFFFFu), X1 = block_exponent(m >> 16);
            const float s0 = pow2_neg(X0), s1 = pow2_neg(X1);
#pragma unroll 8
            for (int r = 0; r < 32; ++r) {
                const uint32_t v = *reinterpret_cast<const uint32_t*>(&tile[r][tc]);
                *reinterpret_cast<uint16_t*>(&ctile[r][c]) = e4m3x2(bf16_lo(v) * s0, bf16_hi(v) * s1);
            }
            if (c < ncol) {
                scales[static_cast<int64_t>(b) * cols + c0 + c] = static_cast<uint8_t>(X0 + 127);
                scales[static_cast<int64_t>(b) * cols + c0 + c + 1] = static_cast<uint8_t>(X1 + 127);
            }
        }
        if (ROW) {
            // row-wise: item = (row r, block j of 32 columns), codes straight out
#pragma unroll
            for (int it = 0; it < 2; ++it) {
                const int i = threadIdx.x + kColThreads * it;
                const int r = i >> 3, j = i & 7;
                if (r < nr && 32 * j < ncol) {
                    uint32_t h[16];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint4 v = *reinterpret_cast<const uint4*>(&tile[r][tile_col(32 * j + 8 * q)]);
                        h[4 * q] = v.x; h[4 * q + 1] = v.y; h[4 * q + 2] = v.z; h[4 * q + 3] = v.w;
                    }
                    const int64_t at = static_cast<int64_t>(r0 + r) * cols + c0 + 32 * j;
                    rscales[at / 32] = mx_encode_row32(h, rcodes + at);
                }
            }
        }
        __syncthreads();
        // codes out: 16-byte vectors, row segments
        for (int i = threadIdx.x; i < 32 * (kColTile / 16); i += kColThreads) {
            const int r = i / (kColTile / 16), v = i % (kColTile / 16);
            if (r < nr && 16 * v < ncol)
                *(reinterpret_cast<uint4*>(codes + static_cast<int64_t>(r0 + r) * cols + c0) + v) =
                    *reinterpret_cast<const uint4*>(&ctile[r][16 * v]);
        }
        __syncthreads();  // the tiles are refilled by the next item
    }
}

int mxfp8_quantize_impl(const uint16_t* x, int64_t rows, int64_t cols, int axis,
                        const int32_t* goff, int ngroups, uint8_t* codes, uint8_t* scales,
                        int32_t* status, cudaStream_t st) {
    if (rows == 0) return MOE_OK;
    const int grid = num_sms() * 8;
    if (axis == 1) {
        mx_rowwise_kernel<<<grid, 256, 0, st>>>(x, rows, cols, codes, scales);
    } else {
        mx_colwise_kernel<false><<<num_sms() * 6, kColThreads, 0, st>>>(
            x, rows, cols, goff, goff ? ngroups : 1, codes, scales, status, nullptr, nullptr);
    }
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}

}  // namespace moe

namespace moe {

int mxfp8_quantize_rowcol_impl(const uint16_t* x, int64_t rows, int64_t cols, const int32_t* goff,
                               int ngroups, uint8_t* rcodes, uint8_t* rscales, uint8_t* ccodes,
                               uint8_t* cscales, int32_t* status, cudaStream_t st) {
    if (rows == 0) return MOE_OK;
    mx_colwise_kernel<true><<<num_sms() * 6, kColThreads, 0, st>>>(
        x, rows, cols, goff, goff ? ngroups : 1, ccodes, cscales, status, rcodes, rscales);
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}

}  // namespace moe
