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

// axis = 0 with groups: a warp takes one 32-row block (restarted at each
// group start; rows past the group count as zero) x 64 columns, held in
// registers: lane l owns the 8 columns 8 (l % 8) .. +8 of rows l / 8 + 4 j
// (j = 0..7), read as one 16-byte vector per row.  Column maxima: per lane
// over its 8 rows (one max.u16x2 per column pair), then across the 4 lanes of
// a column group (two shuffles); the codes of a row's 8 columns leave as one
// 8-byte store.  Scales: one byte per (block, column).  No shared memory and
// no block barriers; each warp loads its next item while it encodes this one.
// (Measured on 262144 x 4096 bf16 with 128 groups, one B200: column-wise 771
// -> 551 us, row + column 1033 -> 846 us against a CTA-per-32x256-tile
// version staged in shared memory.)
constexpr int kMaxGroups = 1024;
constexpr int kColWarps = 8;   // warps per CTA
// CTAs per SM (up to 128 registers a thread: this item's and the next item's
// vectors; 3 CTAs spilled and ran at 0.6x)
constexpr int col_ctas(bool) { return 2; }

__device__ __forceinline__ uint32_t mag2(uint32_t w) { return w & 0x7FFF7FFFu; }
// 2^-X as bf16 bits (X in [-127, 127]; 2^-127 is the one subnormal case)
__device__ __forceinline__ uint32_t bf16_pow2_neg(int X) {
    const int e = 127 - X;
    return e >= 1 ? static_cast<uint32_t>(e << 7) : 0x0040u;
}
// E4M3 codes of a packed bf16 pair scaled by a packed pair of powers of two:
// the bf16 product is exact wherever a code can be nonzero (and a product
// that underflows keeps its sign, as its code, +-0, does), so this equals
// encoding the fp32 products.
__device__ __forceinline__ uint32_t enc_pair(uint32_t v, uint32_t s2) {
    uint32_t p;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(p) : "r"(v), "r"(s2));
    return e4m3x2(bf16_lo(p), bf16_hi(p));
}
__device__ __forceinline__ uint32_t umax2(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("max.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// ROW: also the row-wise encoding of the same registers (a row's 32-column
// block is 4 lanes' 8 columns: l % 8 = 0..3 or 4..7), so that a tensor needed
// in both layouts is read once.
template <bool ROW>
__global__ void __launch_bounds__(kColWarps * 32, col_ctas(ROW))
    mx_colwise_kernel(const uint16_t* __restrict__ x, int64_t rows, int64_t cols,
                      const int32_t* __restrict__ goff, int ngroups, uint8_t* __restrict__ codes,
                      uint8_t* __restrict__ scales, int32_t* status, uint8_t* __restrict__ rcodes,
                      uint8_t* __restrict__ rscales) {
    __shared__ int s_off[kMaxGroups + 1];
    __shared__ int s_base[kMaxGroups + 1];
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
    const int64_t nch = (cols + 63) / 64;
    const int64_t total = static_cast<int64_t>(nblk) * nch;
    const int cg = lane & 7;   // column group: columns 8 cg .. 8 cg + 7 of the chunk
    const int rq = lane >> 3;  // rows rq + 4 j
    // item w: block b (rows r0 .. r0 + nr of one group) x this lane's columns c ..
    struct Item { int b, r0, nr; int64_t c; };
    auto locate = [&](int64_t w) {
        Item it;
        it.b = static_cast<int>(w / nch);
        it.c = (w - static_cast<int64_t>(it.b) * nch) * 64 + 8 * cg;
        int lo = 0, hi = ngroups - 1;
        while (lo < hi) {  // largest g with s_base[g] <= b
            const int mid = (lo + hi + 1) >> 1;
            if (s_base[mid] <= it.b) lo = mid; else hi = mid - 1;
        }
        it.r0 = s_off[lo] + (it.b - s_base[lo]) * 32;
        it.nr = min(s_off[lo + 1], it.r0 + 32) - it.r0;
        return it;
    };
    // cols % 32 == 0: a lane's 8 columns are all in or all out
    auto fetch = [&](const Item& it, uint4 (&v)[8]) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int r = rq + 4 * j;
            v[j] = (it.c < cols && r < it.nr)
                       ? __ldg(reinterpret_cast<const uint4*>(x + static_cast<int64_t>(it.r0 + r) * cols + it.c))
                       : make_uint4(0, 0, 0, 0);
        }
    };
    const int64_t wstep = static_cast<int64_t>(gridDim.x) * kColWarps;
    int64_t w = static_cast<int64_t>(blockIdx.x) * kColWarps + warp;
    Item nxt = locate(w);
    uint4 vn[8];
    if (w < total) fetch(nxt, vn);
    for (; w < total; w += wstep) {
        // this item's vectors; the next item's are loaded while it is encoded
        const Item it = nxt;
        uint4 v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = vn[j];
        if (w + wstep < total) {
            nxt = locate(w + wstep);
            fetch(nxt, vn);
        }
        const int b = it.b, r0 = it.r0, nr = it.nr;
        const int64_t c = it.c;
        const bool cok = c < cols;
        // column maxima of this lane's 8 columns over the block's 32 rows
        uint32_t m[4] = {0, 0, 0, 0};
        uint32_t rm[8];  // per row: maximum over this lane's 8 columns (two halves)
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint32_t a0 = mag2(v[j].x), a1 = mag2(v[j].y), a2 = mag2(v[j].z), a3 = mag2(v[j].w);
            m[0] = umax2(m[0], a0);
            m[1] = umax2(m[1], a1);
            m[2] = umax2(m[2], a2);
            m[3] = umax2(m[3], a3);
            rm[j] = umax2(umax2(a0, a1), umax2(a2, a3));
        }
        // Column blocks: the 4 lanes of a column group (rq = 0..3) share 4
        // words of column-pair maxima; a reduce-scatter over them (partners
        // lane ^ 16, then lane ^ 8) leaves lane rq with the block maximum of
        // pair rq only, whose two exponents it alone computes; the pairs'
        // scales then travel back by shuffles.
        const bool h1 = (lane >> 4) & 1, h0 = (lane >> 3) & 1;
        uint32_t k0 = h1 ? m[2] : m[0], k1 = h1 ? m[3] : m[1];
        k0 = umax2(k0, __shfl_xor_sync(0xffffffffu, h1 ? m[0] : m[2], 16));
        k1 = umax2(k1, __shfl_xor_sync(0xffffffffu, h1 ? m[1] : m[3], 16));
        const uint32_t cw = umax2(h0 ? k1 : k0, __shfl_xor_sync(0xffffffffu, h0 ? k0 : k1, 8));
        const int cX0 = block_exponent(cw & 0xFFFFu), cX1 = block_exponent(cw >> 16);
        const uint32_t s_own = bf16_pow2_neg(cX0) | (bf16_pow2_neg(cX1) << 16);
        uint32_t s[4];  // per column pair: the two scales as bf16x2
#pragma unroll
        for (int i = 0; i < 4; ++i) s[i] = __shfl_sync(0xffffffffu, s_own, (lane & 7) | (i << 3));
        if (ROW) {
            // Row blocks: a row's 32-column block spans the 4 lanes l ^ 0..3
            // (same l / 4; lanes past the columns hold zeros).  Reduce-scatter
            // of the 8 rows' maxima (partners lane ^ 2, then lane ^ 1): lane
            // k = l % 4 keeps rows 2k, 2k + 1, computes their exponents and
            // stores their scale bytes; the scales travel back by shuffles.
            const bool g1 = (lane >> 1) & 1, g0 = lane & 1;
            uint32_t t4[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
                t4[i] = umax2(g1 ? rm[4 + i] : rm[i], __shfl_xor_sync(0xffffffffu, g1 ? rm[i] : rm[4 + i], 2));
            uint32_t t2[2];
#pragma unroll
            for (int i = 0; i < 2; ++i)
                t2[i] = umax2(g0 ? t4[2 + i] : t4[i], __shfl_xor_sync(0xffffffffu, g0 ? t4[i] : t4[2 + i], 1));
            const int kq = lane & 3;  // this lane's rows: 2 kq, 2 kq + 1
            int rX[2];
            uint32_t rs_own = 0;
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                rX[i] = block_exponent(max(t2[i] & 0xFFFFu, t2[i] >> 16));
                rs_own |= bf16_pow2_neg(rX[i]) << (16 * i);
                const int r = rq + 4 * (2 * kq + i);
                if (cok && r < nr)
                    rscales[(static_cast<int64_t>(r0 + r) * cols + c) / 32] = static_cast<uint8_t>(rX[i] + 127);
            }
#pragma unroll
            for (int jp = 0; jp < 4; ++jp) {
                const uint32_t w = __shfl_sync(0xffffffffu, rs_own, (lane & ~3) | jp);
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const int j = 2 * jp + i;
                    const int r = rq + 4 * j;
                    const uint32_t sr = ((w >> (16 * i)) & 0xFFFFu) * 0x10001u;
                    if (cok && r < nr) {
                        const uint4 q = v[j];
                        const uint32_t c01 = enc_pair(q.x, sr);
                        const uint32_t c23 = enc_pair(q.y, sr);
                        const uint32_t c45 = enc_pair(q.z, sr);
                        const uint32_t c67 = enc_pair(q.w, sr);
                        *reinterpret_cast<uint2*>(rcodes + static_cast<int64_t>(r0 + r) * cols + c) =
                            make_uint2(c01 | (c23 << 16), c45 | (c67 << 16));
                    }
                }
            }
        }
        if (cok) {
            // this lane's column pair 2 rq, 2 rq + 1 of its 8 columns
            *reinterpret_cast<uint16_t*>(scales + static_cast<int64_t>(b) * cols + c + 2 * rq) =
                static_cast<uint16_t>((cX0 + 127) | ((cX1 + 127) << 8));
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int r = rq + 4 * j;
                if (r < nr) {
                    const uint4 q = v[j];
                    const uint32_t c01 = enc_pair(q.x, s[0]);
                    const uint32_t c23 = enc_pair(q.y, s[1]);
                    const uint32_t c45 = enc_pair(q.z, s[2]);
                    const uint32_t c67 = enc_pair(q.w, s[3]);
                    *reinterpret_cast<uint2*>(codes + static_cast<int64_t>(r0 + r) * cols + c) =
                        make_uint2(c01 | (c23 << 16), c45 | (c67 << 16));
                }
            }
        }
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
        mx_colwise_kernel<false><<<num_sms() * col_ctas(false), kColWarps * 32, 0, st>>>(
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
    mx_colwise_kernel<true><<<num_sms() * col_ctas(true), kColWarps * 32, 0, st>>>(
        x, rows, cols, goff, goff ? ngroups : 1, ccodes, cscales, status, rcodes, rscales);
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}

}  // namespace moe
