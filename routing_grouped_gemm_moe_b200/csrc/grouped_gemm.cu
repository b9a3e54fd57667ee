// Device-scheduled grouped GEMM on the 5th-generation tensor cores (sm_100a).
//
// Combines the many small expert matmuls of the MoE layer into one persistent
// launch ("Ai2 rebuilds Olmo's training stack for trillion-parameter MoEs",
// "Routing work stays on the GPU", third bullet; "Supercharging Olmo-core for
// Efficient and Scalable MoE Training", Summary: device-scheduled grouped
// GEMMs), in BF16 or in MXFP8 ("MXFP8 reduces compute and memory costs":
// E4M3 operands with one E8M0 scale per 32 values along the reduction axis).
// The group sizes are read from device memory (`offsets`) by every CTA; the
// host never learns them.
//
// Kernel anatomy (one CTA per SM, or one CTA pair per two SMs):
//   warp 0      TMA producer: fills a ring of shared-memory stages (A tile
//               128 rows x 128 bytes of K, B tile BN rows x 128 bytes, 128-byte
//               swizzle), signalling `full[s]` through the transaction count of
//               an mbarrier.  Ragged-M loads of the weight operand carry an L2
//               evict-last policy (an expert's weight block is read again by
//               each of its row tiles).
//   warp 1      allocates TMEM; one thread issues the MMAs (tcgen05.mma,
//               kind::f16 128xBNx16 for bf16, kind::mxf8f6f4.block_scale
//               128xBNx32 for MXFP8, cta_group::2 256xBNx16 on a CTA pair) into
//               an fp32 accumulator in TMEM and releases stages / publishes
//               accumulators with tcgen05.commit.  For MXFP8 on single CTAs it
//               first moves the stage's scale factors from shared memory to
//               TMEM with tcgen05.cp.  On the peer of a ragged-K pair it zeroes
//               the rows of the next expert in its own last K stage instead.
//   warps 2..9  epilogue: tcgen05.ld of the accumulator (two warps per
//               32-lane TMEM quadrant, each taking half of the columns), fused
//               SwiGLU / SwiGLU-backward (optionally with the MXFP8 encoding
//               of its output), bf16 stores.
//   warps 10-11 MXFP8 pairs only: scale-atom loader and copier (below).
// Accumulators: two in TMEM, so that the epilogue of one tile overlaps the
// main loop of the next; MXFP8 tiles 256 wide keep one (two would not fit
// next to the per-stage scales) and the epilogue frees it as soon as its
// columns are in registers.
// CTA pairs (BF16, 256 x 256 tiles): each CTA loads its 128 rows of A and
// half of B; the leader's barrier counts both CTAs' bytes and the leader
// issues the MMAs for both.
// MXFP8 scales: before the GEMM, two small kernels rewrite the row- or
// column-wise scale arrays into 512-byte "atoms", one per (128-row tile,
// 4 K-blocks) of an operand, in the order tcgen05.cp 32x128b.warpx4 places in
// TMEM (byte 16*(r%32) + 4*(r/32) + b holds the scale of row r, K-block b).
// Single CTAs: the producer bulk-copies the stage's atoms (one for A, one per
// 128 rows of B) next to its operand tiles and the MMA thread copies them
// into TMEM.  CTA pairs: a loader warp brings the atoms of kSfGroup
// consecutive K stages at once (two tensor loads per CTA and group, on the
// leader's barrier) into a ring of kSfSlots slots of their own, and a copier
// warp of the leader moves each landed group into TMEM (one column set per K
// stage and slot) and signals the MMA thread, which only waits for it at a
// group's first stage.  Per-stage atom loads next to the operands and copies
// issued by the MMA thread held the MMAs back (ncu: tensor pipe 60 % busy
// against 96 % for cuBLAS's kernel moving the same bytes; this arrangement
// took the layer's MXFP8 GEMM1 and GEMM2 9-10 % faster, outputs unchanged).
// Tiles are handed out round-robin (tile = blockIdx.x + i * gridDim.x, per
// pair on pairs) from a per-expert tile prefix sum each CTA builds in shared
// memory from `offsets`; within an expert, row tiles advance fastest (column
// tiles for the SwiGLU-backward GEMM and the ragged-K ones).
//
// Modes
//   RAGGED_M : C[R_e, :] = A[R_e, :] . B_e^T   (forward GEMMs, dA, dX)
//   RAGGED_K : C_e = A[R_e, :]^T . B[R_e, :]   (dW GEMMs; K = rows of expert e;
//              rows of the last K tile that belong to the next expert are
//              zeroed in shared memory before the MMA reads them)
#include <cuda.h>

#include <atomic>
#include <cstdlib>
#include <mutex>

#include "common.cuh"
#include "mx_encode.cuh"
#include "ptx.cuh"

namespace moe {

int mxfp8_quantize_impl(const uint16_t*, int64_t, int64_t, int, const int32_t*, int, uint8_t*,
                        uint8_t*, int32_t*, cudaStream_t);

namespace gg {

constexpr int BM = 128;
constexpr int ROW_BYTES = 128;  // bytes of K per tile row per stage (one swizzle atom)
constexpr int MAX_E = 1024;
constexpr int kEpiWarps = 8;

enum { kRaggedM = 0, kRaggedK = 1 };
enum { kEpiNone = 0, kEpiSwiglu = 1, kEpiSwigluBwd = 2 };

struct Params {
    // MXFP8 on CTA pairs: the scale-atom arrays (sfa / sfb) as 3-D tensors
    // of whole atoms (see make_atom_map), so that each CTA's group loads can
    // complete on the leader's barrier (cta_group::2 tensor loads); unused
    // otherwise.
    CUtensorMap sfa_map;
    CUtensorMap sfb_map;
    const int32_t* offsets;
    int E;
    int M_total;
    int M;  // RAGGED_K: output rows per expert
    int N;  // output columns (RAGGED_M SWIGLU: 2f)
    int K;  // RAGGED_M reduction width
    int f;  // SwiGLU half width
    uint16_t* c;
    int64_t ldc;
    uint16_t* aux;       // SWIGLU: A out [M_total, f]
    const uint16_t* gu;  // SWIGLU_BWD: [G | U] [M_total, 2f]
    const uint8_t* sfa;  // MXFP8 scale atoms of A / B (see sf_rows_kernel / sf_cols_kernel)
    const uint8_t* sfb;
    int32_t* status;
    // fused MXFP8 quantisation of the epilogue output (SWIGLU: A, width f;
    // SWIGLU_BWD: dH, width 2f): row-wise and column-wise (32-row blocks per
    // expert), NULL when not requested
    uint8_t* qr_codes;
    uint8_t* qr_scales;
    uint8_t* qc_codes;
    uint8_t* qc_scales;
    int b_evict_normal;  // ragged-M: load B with the normal L2 priority instead of evict-last
    int m_fastest;       // ragged-M: an expert's row tiles advance fastest (A evict-last, B normal)
    // ragged-K (BF16): per expert e, tensor maps of A and B whose row extent
    // ends at the expert's last row (kmaps[2 e], kmaps[2 e + 1]): the last K
    // tile's rows past the expert then arrive as TMA zero fill.  NULL: those
    // rows are zeroed in shared memory instead.
    const CUtensorMap* kmaps;
    // Keeping the persistent CTAs in step: every CTA (pair) counts the tiles
    // it starts in *sync_done; a producer about to start its j-th tile first
    // waits, for a bounded time, until all of them have started their
    // (j - sync_slack)-th.  Without it, CTAs drift apart over the hundreds of
    // tiles each takes, the tiles in flight span several experts and their
    // operands no longer fit L2 (see the DRAM-traffic profile).  The last CTA
    // to leave zeroes the counters.  NULL: off.
    unsigned int* sync_done;
    unsigned int* sync_exit;
    int sync_slack;
    // BF16 ragged-M pairs: an expert's last row tile with at most 128 rows
    // runs as an M = 128 pair MMA (64 rows per CTA) instead of M = 256
    int half_tiles;
};

constexpr int kSyncSlots = 64;           // counter pairs, used in turn by the launches
constexpr int kSyncSpinNs = 50000;       // longest wait for the other CTAs per tile
__device__ unsigned int g_sync[2 * kSyncSlots];

constexpr int kAtomBytes = 512;  // scales of 128 rows x 4 K-blocks
constexpr int kSfGroup = 4;      // MXFP8 pairs: K stages whose atoms one group load brings
constexpr int kSfSlots = 2;      // MXFP8 pairs: groups in shared memory at a time

// BN = accumulator columns (the MMA's N).  C2: a CTA pair computes a 256-row
// tile with tcgen05 cta_group::2; each CTA holds 128 rows of A and BN/2 rows of B.
// Coalescing buffers of the SwiGLU-backward epilogue: per warp, G and U of a
// 32-row x 32-column chunk, 64 bytes per row, whose four 16-byte segments are
// stored XOR-swizzled by row (epi_seg): both the row-segment accesses (two
// rows x four segments per 8-thread phase) and the one-row-per-thread
// accesses (eight rows, one segment) then cover all eight 16-byte bank groups.
constexpr int kEpiPitch = 64;
constexpr int kEpiWarpBytes = 2 * 32 * kEpiPitch;
// plain bf16 stores stage one 32 x 32 chunk per warp (C rows leave as 64-byte
// segments instead of 16-byte pieces of 32 different rows)
constexpr int kEpiPlainWarpBytes = 32 * kEpiPitch;
__device__ __forceinline__ int epi_seg(int row, int seg) {
    return row * kEpiPitch + 16 * (seg ^ ((row >> 1) & 3));
}
constexpr int kEpiStageBytes = kEpiWarps * kEpiWarpBytes;
constexpr int kEpiPlainBytes = kEpiWarps * kEpiPlainWarpBytes;
constexpr int kStaticSmemReserve = 17 * 1024;  // group tables and barriers of the kernel

template <int BN, bool MX, bool C2 = false, int ESM = 0>
struct Shape {
    static constexpr int BK = MX ? 128 : 64;       // K elements per stage
    static constexpr int KPI = MX ? 32 : 16;       // K per MMA instruction
    static constexpr int TM = C2 ? 256 : 128;      // tile rows (ragged-M)
    static constexpr int B_ROWS = C2 ? BN / 2 : BN;
    static constexpr int A_BYTES = BM * ROW_BYTES;
    static constexpr int B_BYTES = B_ROWS * ROW_BYTES;
    // MXFP8 scale atoms (512 bytes per 128 rows per stage): each CTA holds the
    // atom of its own 128 rows of A and the atoms of ALL BN columns of B --
    // in a CTA pair too, where each CTA computes its 128 rows against the
    // whole 256-column tile and reads B's scales from its own TMEM only.
    static constexpr int B_ATOMS = BN / 128;
    // CTA pairs take their atoms in groups (see the scale-atom loader and
    // copier warps), single CTAs with each stage
    static constexpr bool SF_GRP = MX && C2;
    static constexpr int SF_BYTES = (MX && !SF_GRP) ? (1 + B_ATOMS) * kAtomBytes : 0;
    static constexpr int SFG_BYTES = SF_GRP ? (1 + B_ATOMS) * kSfGroup * kAtomBytes : 0;
    static constexpr int SF_RING = kSfSlots * SFG_BYTES;
    static constexpr int STAGE_BYTES = ((A_BYTES + B_BYTES + SF_BYTES + 1023) / 1024) * 1024;
    static constexpr int BASE_STAGES = (MX && BN == 128) ? 6 : ((A_BYTES + B_BYTES > 32768) ? 4 : 6);
    static constexpr int FIT_STAGES = (227 * 1024 - 1024 - ESM - SF_RING - kStaticSmemReserve) / STAGE_BYTES;
    static constexpr int STAGES = BASE_STAGES < FIT_STAGES ? BASE_STAGES : FIT_STAGES;
    // MXFP8 with 256-wide tiles: TMEM cannot hold two 256-column accumulators
    // next to the scales, so the accumulator is single-buffered and the
    // epilogue frees it as soon as it has moved it into registers.
    static constexpr int ACC_BUFS = (MX && BN == 256) ? 1 : 2;
    static constexpr int ACC_COLS = ACC_BUFS * BN;
    static constexpr int TMEM_COLS = MX ? 512 : 2 * BN;
    static constexpr int SF_COL0 = ACC_COLS;      // MXFP8: per-stage scale columns after the accumulators
    static constexpr int SF_STRIDE = B_ATOMS == 1 ? 8 : 16;  // per stage: A at +0 (4), B at +SF_B (4 per atom)
    static constexpr int SF_B = B_ATOMS == 1 ? 4 : 8;
    // TMEM scale column sets: one per pipeline stage, or (pairs) one per K
    // stage of each group slot
    static constexpr int SF_SETS = SF_GRP ? kSfSlots * kSfGroup : STAGES;
    static constexpr int SF_RING_OFF = STAGES * STAGE_BYTES + ESM;  // 1024-aligned (ESM is)
    static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + ESM + SF_RING + 1024;
    static constexpr int THREADS = (2 + kEpiWarps + (SF_GRP ? 2 : 0)) * 32;
    static constexpr int MN_BOX_BYTES = ROW_BYTES * BK;  // one MN-major box: BK rows x 128 bytes
    static constexpr int MN_BOX_ELEMS = MX ? 128 : 64;   // MN elements per MN-major box
    static_assert(!MX || BN == 128 || BN == 256, "MXFP8 tiles are 128 x 128 or 128 x 256");
    static_assert(!MX || ACC_COLS + SF_SETS * SF_STRIDE <= 512, "TMEM budget");
    static_assert(SMEM_BYTES + kStaticSmemReserve <= 227 * 1024, "shared memory budget");
    static_assert(STAGES >= 3, "pipeline depth");
    static_assert(ESM % 1024 == 0, "scale-atom ring alignment");
    static_assert(!C2 || BN == 256, "CTA pairs: 128 x 256 halves of 256 x 256 tiles");
};

// The SwiGLU-backward epilogue stages G, U and dH through shared memory
// (coalesced row segments) on MXFP8 tiles and on CTA pairs, whose pipeline
// stages are small enough to leave room for the buffers; single BF16 CTAs
// keep one row per thread (the buffers would cost them a pipeline stage).
constexpr bool staged_epilogue(int epi, bool mx, bool c2, bool fq) {
    return epi == kEpiSwigluBwd && !fq && (mx || c2);
}
// BF16 tiles with two accumulators store plain outputs through a per-warp
// staging buffer as well (16 KB, which costs no pipeline stage).
constexpr bool staged_plain(int epi, bool mx) { return epi == kEpiNone && !mx; }
constexpr int epi_smem_bytes(int epi, bool mx, bool c2, bool fq) {
    return staged_epilogue(epi, mx, c2, fq) ? kEpiStageBytes : (staged_plain(epi, mx) ? kEpiPlainBytes : 0);
}

struct Tile {
    int e;
    int m0;       // RAGGED_M: first routed row; RAGGED_K: first output row
    int row_end;  // RAGGED_M: end of expert rows; RAGGED_K: output rows
    int n0;       // first output column (SWIGLU: first f column)
    int k0;       // RAGGED_K: first routed row of the expert
    int kiters;
    int k_last;   // RAGGED_K: valid rows in the last K tile
};

struct Sched {
    int* off;   // [E+1]
    int* pref;  // [E+1] tile prefix
    int* rt;    // [E+1] MXFP8: prefix of ceil(rows_e / 128) (scale-atom rows)
    int* bb;    // [E+1] SwiGLU epilogues: prefix of ceil(rows_e / 32) (column-wise MXFP8 blocks)
    int n_tiles;
    int m_tiles;  // RAGGED_K
};

// A pair tile whose expert has at most 128 rows left runs as an M = 128
// pair MMA: half the MMA work of an M = 256 tile whose second half would be
// padding.  Each CTA then holds 64 rows of A (rows 64 rank ..) and of the
// accumulator, whose 64 x BN values lie folded over the 128 TMEM lanes
// (measured): lanes 0-63 hold the CTA's rows 0-63 in accumulator columns
// [0, BN/2) = tile columns [0, BN/2), lanes 64-127 the same rows' tile
// columns [BN/2, BN).
__device__ __forceinline__ bool half_tile(const Tile& t, const Params& p) {
    return p.half_tiles && t.row_end - t.m0 <= BM;
}
// What the epilogue warp of TMEM lane quadrant q and column half `half`
// takes: CTA-local first row (32 rows), first accumulator column, number of
// accumulator columns, and the tile column of accumulator column 0.
template <int BN>
__device__ __forceinline__ void epi_part(bool halft, int q, int half, int* row_first, int* acc_beg,
                                         int* acc_n, int* col_shift) {
    if (!halft) {
        *row_first = 32 * q; *acc_beg = half * (BN / 2); *acc_n = BN / 2; *col_shift = 0;
    } else {
        *row_first = 32 * (q & 1); *acc_beg = half * (BN / 4); *acc_n = BN / 4; *col_shift = (q >> 1) * (BN / 2);
    }
}

template <int MODE, int BK, int TM = BM>
__device__ __forceinline__ Tile decode(const Sched& s, const Params& p, int tile, int bn_out) {
    Tile t;
    if (MODE == kRaggedM) {
        int lo = 0, hi = p.E;
        while (lo < hi) {  // largest e with pref[e] <= tile
            int mid = (lo + hi + 1) >> 1;
            if (s.pref[mid] <= tile) lo = mid; else hi = mid - 1;
        }
        t.e = lo;
        int local = tile - s.pref[lo];
        int mt = local / s.n_tiles, nt = local - mt * s.n_tiles;
        if (p.m_fastest) {
            const int mtiles = (s.off[lo + 1] - s.off[lo] + TM - 1) / TM;
            nt = local / mtiles;
            mt = local - nt * mtiles;
        }
        t.m0 = s.off[lo] + mt * TM;
        t.row_end = s.off[lo + 1];
        t.n0 = nt * bn_out;
        t.k0 = 0;
        t.kiters = (p.K + BK - 1) / BK;
        t.k_last = BK;
    } else {
        int per = s.m_tiles * s.n_tiles;
        t.e = tile / per;
        int local = tile - t.e * per;
        int mt = local / s.n_tiles, nt = local - mt * s.n_tiles;
        t.m0 = mt * TM;
        t.row_end = p.M;
        t.n0 = nt * bn_out;
        t.k0 = s.off[t.e];
        const int me = max(0, s.off[t.e + 1] - s.off[t.e]);
        t.kiters = (me + BK - 1) / BK;
        t.k_last = me - (t.kiters - 1) * BK;
    }
    return t;
}

// ---- epilogue stores of 32 accumulator columns (fp32 bit patterns) of one row

__device__ __forceinline__ void store_row32(uint16_t* crow, int col, int ncols, const uint32_t* v) {
    if (col >= ncols) return;
    if (col + 32 <= ncols) {
        uint4* dst = reinterpret_cast<uint4*>(crow + col);
#pragma unroll
        for (int j = 0; j < 4; ++j)
            dst[j] = make_uint4(pack_bf16x2(__uint_as_float(v[8 * j + 0]), __uint_as_float(v[8 * j + 1])),
                                pack_bf16x2(__uint_as_float(v[8 * j + 2]), __uint_as_float(v[8 * j + 3])),
                                pack_bf16x2(__uint_as_float(v[8 * j + 4]), __uint_as_float(v[8 * j + 5])),
                                pack_bf16x2(__uint_as_float(v[8 * j + 6]), __uint_as_float(v[8 * j + 7])));
    } else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
            if (col + j < ncols) crow[col + j] = f32_to_bf16(__uint_as_float(v[j]));
    }
}

// [G | U] row segment and A = silu(G) U for f-columns col .. col+31
__device__ __forceinline__ void store_swiglu32(uint16_t* gurow, uint16_t* arow, int col, int f,
                                               const uint32_t* g, const uint32_t* u) {
    if (col >= f) return;
    if (col + 32 <= f) {
        uint4* dg = reinterpret_cast<uint4*>(gurow + col);
        uint4* du = reinterpret_cast<uint4*>(gurow + f + col);
        uint4* da = reinterpret_cast<uint4*>(arow + col);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float gf[8], uf[8], af[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                gf[i] = __uint_as_float(g[8 * j + i]);
                uf[i] = __uint_as_float(u[8 * j + i]);
                af[i] = silu_f(gf[i]) * uf[i];
            }
            dg[j] = pack8(gf);
            du[j] = pack8(uf);
            da[j] = pack8(af);
        }
    } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            if (col + j >= f) continue;
            const float gv = __uint_as_float(g[j]), uv = __uint_as_float(u[j]);
            gurow[col + j] = f32_to_bf16(gv);
            gurow[f + col + j] = f32_to_bf16(uv);
            arow[col + j] = f32_to_bf16(silu_f(gv) * uv);
        }
    }
}

// store_swiglu32 for a whole chunk (col + 32 <= f) that also returns A as 16
// packed bf16 words (for the fused MXFP8 quantisation); stores only when `store`.
__device__ __forceinline__ void swiglu_pack32(uint16_t* gurow, uint16_t* arow, int col, int f,
                                              const uint32_t* g, const uint32_t* u, bool store,
                                              uint32_t (&ha)[16]) {
    uint4* dg = reinterpret_cast<uint4*>(gurow + col);
    uint4* du = reinterpret_cast<uint4*>(gurow + f + col);
    uint4* da = reinterpret_cast<uint4*>(arow + col);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        float gf[8], uf[8], af[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            gf[i] = __uint_as_float(g[8 * j + i]);
            uf[i] = __uint_as_float(u[8 * j + i]);
            af[i] = silu_f(gf[i]) * uf[i];
        }
        const uint4 a4 = pack8(af);
        ha[4 * j] = a4.x; ha[4 * j + 1] = a4.y; ha[4 * j + 2] = a4.z; ha[4 * j + 3] = a4.w;
        if (store) {
            dg[j] = pack8(gf);
            du[j] = pack8(uf);
            da[j] = a4;
        }
    }
}

// dH = [dG | dU] row segment for f-columns col .. col+31 from dA and the saved
// G, U (gb / ub: the 32 G and U values, already loaded when col + 32 <= f)
__device__ __forceinline__ void store_swiglu_bwd32(uint16_t* dhrow, const uint16_t* gurow, int col,
                                                   int f, const uint32_t* da, const uint4 (&gb)[4],
                                                   const uint4 (&ub)[4]) {
    if (col >= f) return;
    if (col + 32 <= f) {
        uint4* dg = reinterpret_cast<uint4*>(dhrow + col);
        uint4* du = reinterpret_cast<uint4*>(dhrow + f + col);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float gf[8], uf[8], dgf[8], duf[8];
            unpack8(gb[j], gf);
            unpack8(ub[j], uf);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float a = __uint_as_float(da[8 * j + i]);
                const float sg = sigmoid_f(gf[i]);
                dgf[i] = a * uf[i] * sg * (1.0f + gf[i] * (1.0f - sg));
                duf[i] = a * gf[i] * sg;
            }
            dg[j] = pack8(dgf);
            du[j] = pack8(duf);
        }
    } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            if (col + j >= f) continue;
            const float a = __uint_as_float(da[j]);
            const float gv = bf16_to_f32(gurow[col + j]);
            const float uv = bf16_to_f32(gurow[f + col + j]);
            const float sg = sigmoid_f(gv);
            dhrow[col + j] = f32_to_bf16(a * uv * sg * (1.0f + gv * (1.0f - sg)));
            dhrow[f + col + j] = f32_to_bf16(a * gv * sg);
        }
    }
}

// FQ: the epilogue also quantises its output to MXFP8 (SwiGLU: A, SwiGLU
// backward: dH); a separate instantiation keeps the plain epilogues' register
// budget.
template <int BN, int MODE, bool A_MN, bool B_MN, int EPI, bool MX, bool C2, bool FQ = false>
__global__ void __launch_bounds__(Shape<BN, MX, C2>::THREADS, 1)
    gg_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
              const __grid_constant__ Params p) {
    // SwiGLU backward on MXFP8 tiles: the 2x faster main loop leaves the
    // epilogue's row-per-thread G / U / dH accesses as the bound, so they are
    // staged through shared memory (measured: MXFP8 dA 7.3 -> 6.7 ms per step;
    // on BF16 tiles the pipeline stage it costs made dA slower)
    constexpr bool STAGED = staged_epilogue(EPI, MX, C2, FQ);
    // M = 128 pair MMAs for an expert's last <= 128 rows (see half_tile): BF16
    // ragged-M pairs whose epilogue neither quantises (its column-wise blocks
    // are a warp's 32 rows) nor pairs G with U (they fall in different lanes)
    constexpr bool kHalfOK = C2 && !MX && MODE == kRaggedM && !FQ && EPI != kEpiSwiglu;
    constexpr bool STAGED_PLAIN = staged_plain(EPI, MX);
    using S = Shape<BN, MX, C2, epi_smem_bytes(EPI, MX, C2, FQ)>;
    constexpr int BK = S::BK;
    constexpr int TM = S::TM;
    constexpr int BN_OUT = (EPI == kEpiSwiglu) ? BN / 2 : BN;
    static_assert(!(EPI == kEpiSwiglu && B_MN), "SwiGLU GEMM takes K-major weights");
    static_assert(MODE == kRaggedM || (A_MN && B_MN && EPI == kEpiNone), "RAGGED_K layout");

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint8_t* epi_smem = smem + S::STAGES * S::STAGE_BYTES;  // SwiGLU-backward coalescing buffers
    __shared__ __align__(8) uint64_t full_bar[S::STAGES];
    __shared__ __align__(8) uint64_t empty_bar[S::STAGES];
    // ragged-K on a CTA pair: the peer's loads of a K tile that ends past the
    // expert land on its own barrier, so that the peer can zero those rows
    // before the leader's MMA reads them
    constexpr bool kPairK = C2 && MODE == kRaggedK;
    __shared__ __align__(8) uint64_t pfull_bar[kPairK ? S::STAGES : 1];
    __shared__ __align__(8) uint64_t tfull_bar[S::ACC_BUFS];
    __shared__ __align__(8) uint64_t tempty_bar[S::ACC_BUFS];
    // MXFP8 pairs: scale-atom group slots (loaded: the leader's sf_full
    // counts both CTAs' bytes; consumed: the MMAs' commit to both sf_empty)
    __shared__ __align__(8) uint64_t sf_full_bar[S::SF_GRP ? kSfSlots : 1];
    __shared__ __align__(8) uint64_t sf_empty_bar[S::SF_GRP ? kSfSlots : 1];
    __shared__ __align__(8) uint64_t sf_ready_bar[S::SF_GRP ? kSfSlots : 1];
    __shared__ uint32_t tmem_base_sh;
    __shared__ int s_off[MAX_E + 1];
    __shared__ int s_pref[MAX_E + 1];
    __shared__ int s_rt[MX ? MAX_E + 1 : 1];
    __shared__ int s_bb[EPI != kEpiNone ? MAX_E + 1 : 1];
    __shared__ volatile int s_abort;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // CTA pairs: both CTAs walk the same tile sequence, one pair per tile
    const uint32_t rank = C2 ? ptx::cluster_ctarank() : 0u;
    const int tile0 = C2 ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
    const int tstep = C2 ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);

    Sched sch;
    sch.off = s_off;
    sch.pref = s_pref;
    sch.rt = s_rt;
    sch.bb = s_bb;
    if (MODE == kRaggedM) {
        const int n_eff = (EPI == kEpiSwiglu) ? p.f : p.N;
        sch.n_tiles = (n_eff + BN_OUT - 1) / BN_OUT;
        sch.m_tiles = 0;
    } else {
        sch.n_tiles = (p.N + BN - 1) / BN;
        sch.m_tiles = (p.M + TM - 1) / TM;
    }

    if (threadIdx.x == 0) {
        for (int s = 0; s < S::STAGES; ++s) {
            // kPairK: the leader's arrival plus one from the peer (after its
            // loads, or after it zeroed the rows past the expert)
            ptx::mbar_init(&full_bar[s], kPairK ? 2 : 1);
            ptx::mbar_init(&empty_bar[s], 1);
            if (kPairK) ptx::mbar_init(&pfull_bar[s], 1);
        }
        if (S::SF_GRP) {
            for (int s = 0; s < kSfSlots; ++s) {
                ptx::mbar_init(&sf_full_bar[s], 1);
                ptx::mbar_init(&sf_empty_bar[s], 1);
                ptx::mbar_init(&sf_ready_bar[s], 1);
            }
        }
        for (int a = 0; a < S::ACC_BUFS; ++a) {
            ptx::mbar_init(&tfull_bar[a], 1);
            ptx::mbar_init(&tempty_bar[a], C2 ? 2 * kEpiWarps : kEpiWarps);
        }
        s_abort = 0;
        ptx::fence_mbar_init();
        ptx::prefetch_tmap(&tmA);
        ptx::prefetch_tmap(&tmB);
    }
    if (warp == 1) {
        if (C2) {
            ptx::tmem_alloc_pair(&tmem_base_sh, S::TMEM_COLS);
            ptx::tmem_relinquish_pair();
        } else {
            ptx::tmem_alloc(&tmem_base_sh, S::TMEM_COLS);
            ptx::tmem_relinquish();
        }
    }
    if (warp == 2) {
        // Group table and per-expert tile prefix sum (warp-wide scan); for
        // MXFP8 also the prefix of ceil(rows / 128) that indexes scale atoms.
        // offsets out of [0, M_total] or going down: flagged, clamped and
        // replaced by their running maximum (the MXFP8 scale tables use the
        // same groups)
        const int E = p.E;
        load_group_offsets(p.offsets, E, p.M_total, s_off, p.status);
        const int per = (E + 31) / 32;
        const int beg = min(E, lane * per), end = min(E, beg + per);
        int local = 0, lblk = 0, l32 = 0;
        for (int e = beg; e < end; ++e) {
            const int me = s_off[e + 1] - s_off[e];
            local += (MODE == kRaggedM) ? ((me + TM - 1) / TM) * sch.n_tiles
                                        : sch.m_tiles * sch.n_tiles;
            lblk += (me + 127) / 128;
            l32 += (me + 31) / 32;
        }
        int incl = local, iblk = lblk, i32 = l32;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            const int vb = __shfl_up_sync(0xffffffffu, iblk, o);
            const int v32 = __shfl_up_sync(0xffffffffu, i32, o);
            if (lane >= o) { incl += v; iblk += vb; i32 += v32; }
        }
        int run = incl - local, rb = iblk - lblk, r32 = i32 - l32;
        for (int e = beg; e < end; ++e) {
            s_pref[e] = run;
            const int me = max(0, s_off[e + 1] - s_off[e]);
            run += (MODE == kRaggedM) ? ((me + TM - 1) / TM) * sch.n_tiles
                                      : sch.m_tiles * sch.n_tiles;
            if (MX) s_rt[e] = rb;
            rb += (me + 127) / 128;
            if (EPI != kEpiNone) s_bb[e] = r32;
            r32 += (me + 31) / 32;
        }
        if (lane == 31) {
            s_pref[E] = incl;
            if (MX) s_rt[E] = iblk;
            if (EPI != kEpiNone) s_bb[E] = i32;
        }
    }
    __syncthreads();
    if (C2) ptx::cluster_sync();  // the peer's barriers are initialised before any remote signal
    ptx::tc_fence_after();
    const uint32_t tmem_base = tmem_base_sh;
    const int total = s_pref[p.E];

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            constexpr uint32_t TX = S::A_BYTES + S::B_BYTES + S::SF_BYTES;
            // ragged-M: the operand that later tiles of the same expert read
            // again stays in L2 (evict-last): the activations when row tiles
            // advance fastest, else the expert's weight block (large layer,
            // ncu: GEMM1 DRAM reads 16.1 -> 12.0 GB, dX 17.0 -> 12.5 GB
            // against no hint; marking A evict-first as well doubled them)
            const uint64_t pol_a = p.m_fastest ? ptx::policy_evict_last() : ptx::policy_evict_normal();
            const uint64_t pol_b = (p.b_evict_normal || p.m_fastest) ? ptx::policy_evict_normal()
                                                                     : ptx::policy_evict_last();
            int jt = 0;  // tiles this CTA has started
            bool in_step = p.sync_done != nullptr;
            const unsigned int units = C2 ? gridDim.x / 2 : gridDim.x;
            for (int tile = tile0; ok && tile < total; tile += tstep) {
                const Tile t = decode<MODE, BK, TM>(sch, p, tile, BN_OUT);
                if (in_step) {
                    if (jt >= p.sync_slack) {
                        // (capped: every tile is started exactly once)
                        unsigned int target = static_cast<unsigned int>(jt - p.sync_slack + 1) * units;
                        if (target > static_cast<unsigned int>(total)) target = static_cast<unsigned int>(total);
                        const uint64_t t0 = ptx::globaltimer();
                        while (*reinterpret_cast<volatile unsigned int*>(p.sync_done) < target) {
                            if (ptx::globaltimer() - t0 > kSyncSpinNs) { in_step = false; break; }
                            __nanosleep(200);
                        }
                    }
                    if (!C2 || rank == 0) atomicAdd(p.sync_done, 1u);
                    ++jt;
                }
                // ragged-K with per-expert maps: rows past the expert read as zeros
                const CUtensorMap* mapA = &tmA;
                const CUtensorMap* mapB = &tmB;
                if (MODE == kRaggedK && p.kmaps && t.kiters > 0) {
                    mapA = p.kmaps + 2 * t.e;
                    mapB = p.kmaps + 2 * t.e + 1;
                    ptx::tmap_acquire(mapA);
                    ptx::tmap_acquire(mapB);
                }
                for (int kt = 0; kt < t.kiters; ++kt) {
                    if (!ptx::mbar_wait(&empty_bar[stage], phase ^ 1u, &s_abort)) { ok = false; break; }
                    uint8_t* sa = smem + stage * S::STAGE_BYTES;
                    uint8_t* sb = sa + S::A_BYTES;
                    uint64_t* fb = &full_bar[stage];
                    if (kPairK) {
                        // A: this CTA's 128 output rows, B: its half of the N
                        // columns; both K-row boxes start at the same routed row
                        const uint32_t fbc = ptx::mapa_shared(ptx::smem_addr(fb), 0);
                        const bool tail = !p.kmaps && kt == t.kiters - 1 && t.k_last < BK;
                        const int krow = t.k0 + kt * BK;
                        const int am = t.m0 + BM * static_cast<int>(rank);
                        const int bn0 = t.n0 + S::B_ROWS * static_cast<int>(rank);
                        if (rank == 0) ptx::mbar_arrive_expect_tx(fb, tail ? TX : 2 * TX);
                        if (rank == 1 && tail) {
                            uint64_t* pb = &pfull_bar[stage];
                            ptx::mbar_arrive_expect_tx(pb, TX);
#pragma unroll
                            for (int j = 0; j < BM / S::MN_BOX_ELEMS; ++j)
                                ptx::tma_load_2d(sa + j * S::MN_BOX_BYTES, &tmA, pb, am + S::MN_BOX_ELEMS * j, krow);
#pragma unroll
                            for (int j = 0; j < S::B_ROWS / S::MN_BOX_ELEMS; ++j)
                                ptx::tma_load_2d(sb + j * S::MN_BOX_BYTES, &tmB, pb, bn0 + S::MN_BOX_ELEMS * j, krow);
                        } else {
#pragma unroll
                            for (int j = 0; j < BM / S::MN_BOX_ELEMS; ++j)
                                ptx::tma_load_2d_pair(sa + j * S::MN_BOX_BYTES, mapA, fbc, am + S::MN_BOX_ELEMS * j, krow);
#pragma unroll
                            for (int j = 0; j < S::B_ROWS / S::MN_BOX_ELEMS; ++j)
                                ptx::tma_load_2d_pair(sb + j * S::MN_BOX_BYTES, mapB, fbc, bn0 + S::MN_BOX_ELEMS * j, krow);
                            if (rank == 1) ptx::mbar_arrive_cluster_relaxed(fbc);
                        }
                        if (++stage == S::STAGES) { stage = 0; phase ^= 1u; }
                        continue;
                    }
                    if (C2) {
                        // both CTAs' bytes are counted on the leader's barrier
                        const uint32_t fbc = ptx::mapa_shared(ptx::smem_addr(fb), 0);
                        if (rank == 0) ptx::mbar_arrive_expect_tx(fb, 2 * TX);
                        const int a_rows = (kHalfOK && half_tile(t, p)) ? BM / 2 : BM;
                        ptx::tma_load_2d_pair_h(sa, &tmA, fbc, kt * BK, t.m0 + a_rows * static_cast<int>(rank), pol_a);
                        if (!B_MN) {
                            const int brow = (EPI == kEpiSwiglu) ? (rank ? p.f : 0) + t.n0
                                                                 : t.n0 + static_cast<int>(rank) * S::B_ROWS;
                            ptx::tma_load_3d_pair_h(sb, &tmB, fbc, kt * BK, brow, t.e, pol_b);
                        } else {
#pragma unroll
                            for (int j = 0; j < S::B_ROWS / S::MN_BOX_ELEMS; ++j)
                                ptx::tma_load_3d_pair_h(sb + j * S::MN_BOX_BYTES, &tmB, fbc,
                                                        t.n0 + static_cast<int>(rank) * S::B_ROWS + S::MN_BOX_ELEMS * j,
                                                        kt * BK, t.e, pol_b);
                        }
                        if (++stage == S::STAGES) { stage = 0; phase ^= 1u; }
                        continue;
                    }
                    ptx::mbar_arrive_expect_tx(fb, TX);
                    if (MODE == kRaggedM) {
                        ptx::tma_load_2d_h(sa, &tmA, fb, kt * BK, t.m0, pol_a);
                        if (!B_MN) {
                            if (EPI == kEpiSwiglu) {
                                ptx::tma_load_3d_h(sb, &tmB, fb, kt * BK, t.n0, t.e, pol_b);
                                ptx::tma_load_3d_h(sb + S::B_BYTES / 2, &tmB, fb, kt * BK, p.f + t.n0, t.e, pol_b);
                            } else {
                                ptx::tma_load_3d_h(sb, &tmB, fb, kt * BK, t.n0, t.e, pol_b);
                            }
                        } else {
#pragma unroll
                            for (int j = 0; j < BN / S::MN_BOX_ELEMS; ++j)
                                ptx::tma_load_3d_h(sb + j * S::MN_BOX_BYTES, &tmB, fb,
                                                   t.n0 + S::MN_BOX_ELEMS * j, kt * BK, t.e, pol_b);
                        }
                    } else {
                        const int krow = t.k0 + kt * BK;
#pragma unroll
                        for (int j = 0; j < BM / S::MN_BOX_ELEMS; ++j)
                            ptx::tma_load_2d(sa + j * S::MN_BOX_BYTES, mapA, fb, t.m0 + S::MN_BOX_ELEMS * j, krow);
#pragma unroll
                        for (int j = 0; j < BN / S::MN_BOX_ELEMS; ++j)
                            ptx::tma_load_2d(sb + j * S::MN_BOX_BYTES, mapB, fb, t.n0 + S::MN_BOX_ELEMS * j, krow);
                    }
                    if (MX) {
                        // scale atoms of this stage: A, then the B_ATOMS atoms of
                        // B (one per 128 rows of the B tile), after the B tile
                        int64_t ia, ib;
                        const int nsub = S::B_ATOMS;  // B atoms per tile
                        const int nct = sch.n_tiles * nsub;  // B atom columns of 128 rows (padded to tiles)
                        if (MODE == kRaggedM) {
                            const int ks = t.kiters;
                            const int mt = (t.m0 - sch.off[t.e]) / BM;
                            const int nt = t.n0 / BN_OUT;
                            ia = (static_cast<int64_t>(sch.rt[t.e] + mt) * ks + kt);
                            if (EPI == kEpiSwiglu)  // atoms per (expert, tile, sub-atom)
                                ib = ((static_cast<int64_t>(t.e) * sch.n_tiles + nt) * nsub) * ks + kt;
                            else if (B_MN)
                                ib = (static_cast<int64_t>(t.e) * ks + kt) * nct + nt * nsub;
                            else
                                ib = (static_cast<int64_t>(t.e) * nct + nt * nsub) * ks + kt;
                        } else {
                            const int64_t slot = sch.rt[t.e] + kt;
                            ia = slot * sch.m_tiles + t.m0 / BM;
                            ib = slot * nct + (t.n0 / BN) * nsub;
                        }
                        ptx::bulk_load(sb + S::B_BYTES, p.sfa + ia * kAtomBytes, kAtomBytes, fb);
#pragma unroll
                        for (int j = 0; j < S::B_ATOMS; ++j) {
                            // consecutive sub-atoms: stride ks (K-major weights) or 1
                            const int64_t stride = (MODE == kRaggedM && !B_MN) ? t.kiters : 1;
                            ptx::bulk_load(sb + S::B_BYTES + (1 + j) * kAtomBytes,
                                           p.sfb + (ib + j * stride) * kAtomBytes, kAtomBytes, fb);
                        }
                    }
                    if (++stage == S::STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            if (!ok) {
                s_abort = 1;
                flag_status(p.status, MOE_ERR_DEVICE_TIMEOUT);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (the leader CTA of a pair)
        if (!C2 || rank == 0) {
        int stage = 0;
        uint32_t phase = 0;
        int acc = 0;
        uint32_t acc_phase = 0;
        int sgi = 0;  // scale-atom groups consumed (MXFP8 pairs)
        bool ok = true;
        for (int tile = tile0; ok && tile < total; tile += tstep) {
            const Tile t = decode<MODE, BK, TM>(sch, p, tile, BN_OUT);
            if (!ptx::mbar_wait(&tempty_bar[acc], acc_phase ^ 1u, &s_abort)) { ok = false; break; }
            ptx::tc_fence_after();
            const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
            for (int kt = 0; kt < t.kiters; ++kt) {
                if (!ptx::mbar_wait(&full_bar[stage], phase, &s_abort)) { ok = false; break; }
                if constexpr (S::SF_GRP) {
                    if (kt % kSfGroup == 0 &&
                        !ptx::mbar_wait(&sf_ready_bar[sgi % kSfSlots], (sgi / kSfSlots) & 1u, &s_abort)) {
                        ok = false;
                        break;
                    }
                }
                ptx::tc_fence_after();
                uint8_t* sa = smem + stage * S::STAGE_BYTES;
                uint8_t* sb = sa + S::A_BYTES;
                if (MODE == kRaggedK && !p.kmaps && kt == t.kiters - 1 && t.k_last < BK) {
                    // Rows k_last..BK-1 of this K tile belong to the next expert
                    // (or lie past the buffer): zero them in every box of A and B.
                    const int nbytes = (BK - t.k_last) * ROW_BYTES;
                    constexpr int NA = BM / S::MN_BOX_ELEMS, NB = S::B_ROWS / S::MN_BOX_ELEMS;
                    for (int j = 0; j < NA + NB; ++j) {
                        uint8_t* box = (j < NA) ? sa + j * S::MN_BOX_BYTES : sb + (j - NA) * S::MN_BOX_BYTES;
                        uint4* z = reinterpret_cast<uint4*>(box + t.k_last * ROW_BYTES);
                        for (int i = lane; i < nbytes / 16; i += 32) z[i] = make_uint4(0, 0, 0, 0);
                    }
                    ptx::fence_proxy_async_smem();
                }
                __syncwarp();
                if (lane == 0) {
                    const uint32_t a_addr = ptx::smem_addr(sa);
                    const uint32_t b_addr = ptx::smem_addr(sb);
                    // per-MMA start-address advance along K
                    constexpr uint32_t MN_STEP = S::KPI * ROW_BYTES;  // KPI rows of 128 bytes
                    constexpr uint32_t K_STEP = 32;                  // KPI elements = 32 bytes
                    if (MX) {
                        const int sf_set = S::SF_GRP ? (sgi % kSfSlots) * kSfGroup + kt % kSfGroup : stage;
                        const uint32_t sf_col = tmem_base + S::SF_COL0 + sf_set * S::SF_STRIDE;
                        if constexpr (C2) {
                            // (the group's atoms were copied into TMEM by the copier warp)
                        } else {
                            const uint32_t sf_smem = ptx::smem_addr(sb + S::B_BYTES);
                            ptx::tmem_cp_32x128b_x4(sf_col, ptx::sdesc_plain(sf_smem, 128, 128));
#pragma unroll
                            for (int j = 0; j < S::B_ATOMS; ++j)
                                ptx::tmem_cp_32x128b_x4(sf_col + S::SF_B + 4 * j,
                                                        ptx::sdesc_plain(sf_smem + (1 + j) * kAtomBytes, 128, 128));
                        }
#pragma unroll
                        for (int kk = 0; kk < BK / S::KPI; ++kk) {
                            const uint64_t ad = A_MN ? ptx::sdesc_sw128(a_addr + kk * MN_STEP, S::MN_BOX_BYTES, 1024)
                                                     : ptx::sdesc_sw128(a_addr + kk * K_STEP, 16, 1024);
                            const uint64_t bd = B_MN ? ptx::sdesc_sw128(b_addr + kk * MN_STEP, S::MN_BOX_BYTES, 1024)
                                                     : ptx::sdesc_sw128(b_addr + kk * K_STEP, 16, 1024);
                            // the scale byte of K block kk in each TMEM word: the
                            // descriptor's A / B scale-factor ids
                            const uint32_t id = ptx::idesc_mxf8(C2 ? 2 * BM : BM, BN, A_MN, B_MN, kk, kk);
                            if constexpr (C2)
                                ptx::mma_mxf8_pair(d_tmem, ad, bd, id, sf_col, sf_col + S::SF_B,
                                                   (kt | kk) != 0 ? 1u : 0u);
                            else
                                ptx::mma_mxf8(d_tmem, ad, bd, id, sf_col, sf_col + S::SF_B,
                                              (kt | kk) != 0 ? 1u : 0u);
                        }
                    } else {
                        constexpr uint32_t IDESC = ptx::idesc_bf16(C2 ? 2 * BM : BM, BN, A_MN, B_MN);
                        // (M = 128 pair MMA for a half tile)
                        constexpr uint32_t IDESC_HALF = ptx::idesc_bf16(BM, BN, A_MN, B_MN);
                        const uint32_t idesc = (kHalfOK && half_tile(t, p)) ? IDESC_HALF : IDESC;
#pragma unroll
                        for (int kk = 0; kk < BK / S::KPI; ++kk) {
                            const uint64_t ad = A_MN ? ptx::sdesc_sw128(a_addr + kk * MN_STEP, S::MN_BOX_BYTES, 1024)
                                                     : ptx::sdesc_sw128(a_addr + kk * K_STEP, 16, 1024);
                            const uint64_t bd = B_MN ? ptx::sdesc_sw128(b_addr + kk * MN_STEP, S::MN_BOX_BYTES, 1024)
                                                     : ptx::sdesc_sw128(b_addr + kk * K_STEP, 16, 1024);
                            if (C2) ptx::mma_f16_pair(d_tmem, ad, bd, idesc, (kt | kk) != 0 ? 1u : 0u);
                            else ptx::mma_f16(d_tmem, ad, bd, IDESC, (kt | kk) != 0 ? 1u : 0u);
                        }
                    }
                    if (C2) ptx::mma_commit_pair(&empty_bar[stage], 0x3);
                    else ptx::mma_commit(&empty_bar[stage]);
                }
                __syncwarp();
                if (S::SF_GRP && (kt % kSfGroup == kSfGroup - 1 || kt == t.kiters - 1)) {
                    if (lane == 0) ptx::mma_commit_pair(&sf_empty_bar[sgi % kSfSlots], 0x3);
                    __syncwarp();
                    ++sgi;
                }
                if (++stage == S::STAGES) { stage = 0; phase ^= 1u; }
            }
            if (!ok) break;
            if (lane == 0) {
                if (C2) ptx::mma_commit_pair(&tfull_bar[acc], 0x3);
                else if (t.kiters > 0) ptx::mma_commit(&tfull_bar[acc]);
                else ptx::mbar_arrive(&tfull_bar[acc]);
            }
            __syncwarp();
            if (++acc == S::ACC_BUFS) { acc = 0; acc_phase ^= 1u; }
        }
        if (!ok && lane == 0) {
            s_abort = 1;
            flag_status(p.status, MOE_ERR_DEVICE_TIMEOUT);
        }
        } else if constexpr (kPairK) {
            // The peer of a ragged-K pair: for each tile's last K stage that
            // reaches past the expert, wait for this CTA's own loads, zero the
            // rows past the expert in its A and B boxes, and give the leader's
            // full barrier its second arrival.
            int stage = 0;
            uint32_t pphase = 0;  // bit s: parity of pfull_bar[s]
            bool ok = true;
            for (int tile = tile0; ok && tile < total; tile += tstep) {
                const Tile t = decode<MODE, BK, TM>(sch, p, tile, BN_OUT);
                if (!p.kmaps && t.kiters > 0 && t.k_last < BK) {
                    const int st = (stage + t.kiters - 1) % S::STAGES;
                    if (!ptx::mbar_wait(&pfull_bar[st], (pphase >> st) & 1u, &s_abort)) { ok = false; break; }
                    pphase ^= 1u << st;
                    uint8_t* sa = smem + st * S::STAGE_BYTES;
                    uint8_t* sb = sa + S::A_BYTES;
                    const int nbytes = (BK - t.k_last) * ROW_BYTES;
                    constexpr int NA = BM / S::MN_BOX_ELEMS, NB = S::B_ROWS / S::MN_BOX_ELEMS;
                    for (int j = 0; j < NA + NB; ++j) {
                        uint8_t* box = (j < NA) ? sa + j * S::MN_BOX_BYTES : sb + (j - NA) * S::MN_BOX_BYTES;
                        uint4* z = reinterpret_cast<uint4*>(box + t.k_last * ROW_BYTES);
                        for (int i = lane; i < nbytes / 16; i += 32) z[i] = make_uint4(0, 0, 0, 0);
                    }
                    ptx::fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive_cluster(ptx::mapa_shared(ptx::smem_addr(&full_bar[st]), 0));
                    __syncwarp();
                }
                stage = (stage + max(t.kiters, 0)) % S::STAGES;
            }
            if (!ok && lane == 0) {
                s_abort = 1;
                flag_status(p.status, MOE_ERR_DEVICE_TIMEOUT);
            }
        }
    } else if (S::SF_GRP && warp == 2 + kEpiWarps) {
        // ------------------------------------------------ scale-atom loader (MXFP8 pairs)
        // Each CTA loads, per group of kSfGroup K stages, the atoms of its 128
        // rows of A (map [row tile][K stage][atom]) and those of the tile's
        // B_ATOMS x 128 B columns into the next ring slot, as soon as the MMAs
        // of the slot's previous group have completed (sf_empty); both CTAs'
        // bytes land on the leader's sf_full.
        if (lane == 0) {
            int gi = 0;
            bool ok = true;
            for (int tile = tile0; ok && tile < total; tile += tstep) {
                const Tile t = decode<MODE, BK, TM>(sch, p, tile, BN_OUT);
                const int ks = t.kiters;
                const int mt = (t.m0 + BM * static_cast<int>(rank) - sch.off[t.e]) / BM;
                const int nt = t.n0 / BN_OUT;
                const int nct = sch.n_tiles * S::B_ATOMS;
                for (int kt0 = 0; kt0 < ks; kt0 += kSfGroup, ++gi) {
                    const int slot = gi % kSfSlots;
                    if (!ptx::mbar_wait(&sf_empty_bar[slot], ((gi / kSfSlots) & 1u) ^ 1u, &s_abort)) {
                        ok = false;
                        break;
                    }
                    uint8_t* dst = smem + S::SF_RING_OFF + slot * S::SFG_BYTES;
                    const uint32_t fbc = ptx::mapa_shared(ptx::smem_addr(&sf_full_bar[slot]), 0);
                    if (rank == 0) ptx::mbar_arrive_expect_tx(&sf_full_bar[slot], 2 * S::SFG_BYTES);
                    // map coordinates (x: the atom's words): ragged-M A [row tile][K
                    // stage], B [expert x atom column][K stage] or, MN-major, [expert
                    // x K stage][atom column]; ragged-K (dW) A [K slot][128-row output
                    // tile], B [K slot][atom column]
                    int ay, az, by, bz;
                    if (MODE == kRaggedK) {
                        ay = (t.m0 + BM * static_cast<int>(rank)) / BM; az = sch.rt[t.e] + kt0;
                        by = (t.n0 / BN) * S::B_ATOMS; bz = sch.rt[t.e] + kt0;
                    } else {
                        ay = kt0; az = sch.rt[t.e] + mt;
                        if (B_MN) { by = nt * S::B_ATOMS; bz = t.e * ks + kt0; }
                        else { by = kt0; bz = t.e * nct + nt * S::B_ATOMS; }
                    }
                    ptx::tma_load_3d_pair(dst, &p.sfa_map, fbc, 0, ay, az);
                    ptx::tma_load_3d_pair(dst + kSfGroup * kAtomBytes, &p.sfb_map, fbc, 0, by, bz);
                }
            }
            if (!ok) {
                s_abort = 1;
                flag_status(p.status, MOE_ERR_DEVICE_TIMEOUT);
            }
        }
    } else if (S::SF_GRP && warp == 3 + kEpiWarps) {
        // ------------------------------------------------ scale-atom copier (MXFP8 pairs)
        // The leader moves each landed group's atoms, both CTAs' (same shared-
        // memory offsets, each into its own TMEM), into the slot's column sets,
        // then signals sf_ready.  The sets were last read by the MMAs of the
        // slot's previous group, which completed before its loads were issued.
        if (lane == 0 && rank == 0) {
            int gi = 0;
            bool ok = true;
            for (int tile = tile0; ok && tile < total; tile += tstep) {
                const Tile t = decode<MODE, BK, TM>(sch, p, tile, BN_OUT);
                for (int kt0 = 0; kt0 < t.kiters; kt0 += kSfGroup, ++gi) {
                    const int slot = gi % kSfSlots;
                    if (!ptx::mbar_wait(&sf_full_bar[slot], (gi / kSfSlots) & 1u, &s_abort)) { ok = false; break; }
                    ptx::tc_fence_after();
                    const uint32_t ring = ptx::smem_addr(smem + S::SF_RING_OFF + slot * S::SFG_BYTES);
                    const int ng = min(kSfGroup, t.kiters - kt0);
                    for (int g = 0; g < ng; ++g) {
                        const uint32_t col = tmem_base + S::SF_COL0 + (slot * kSfGroup + g) * S::SF_STRIDE;
                        ptx::tmem_cp_32x128b_x4_pair(col, ptx::sdesc_plain(ring + g * kAtomBytes, 128, 128));
#pragma unroll
                        for (int j = 0; j < S::B_ATOMS; ++j) {
                            const int bi = (B_MN || MODE == kRaggedK) ? g * S::B_ATOMS + j : j * kSfGroup + g;
                            ptx::tmem_cp_32x128b_x4_pair(col + S::SF_B + 4 * j,
                                                         ptx::sdesc_plain(ring + (kSfGroup + bi) * kAtomBytes, 128, 128));
                        }
                    }
                    ptx::mma_commit_pair(&sf_ready_bar[slot], 0x1);
                }
            }
            if (!ok) { s_abort = 1; flag_status(p.status, MOE_ERR_DEVICE_TIMEOUT); }
        }
    } else {
        // ------------------------------------------------ epilogue (8 warps)
        // Two warps per TMEM lane quadrant (warp % 4 selects the quadrant a
        // warp may access); the two split the tile's columns in halves.
        const int q = warp & 3;
        const int half = (warp - 2) >> 2;
        const int r = q * 32 + lane;
        int acc = 0;
        uint32_t acc_phase = 0;
        bool ok = true;
        for (int tile = tile0; tile < total; tile += tstep) {
            const Tile t = decode<MODE, BK, TM>(sch, p, tile, BN_OUT);
            const bool halft = kHalfOK && half_tile(t, p);
            int q_first, acc_beg, acc_n, col_shift;
            epi_part<BN>(halft, q, half, &q_first, &acc_beg, &acc_n, &col_shift);
            const int cta_row0 = t.m0 + (halft ? BM / 2 : BM) * static_cast<int>(rank);
            const int row = cta_row0 + q_first + lane;
            const bool row_ok = row < t.row_end;
            if constexpr (S::ACC_BUFS == 1) {
                // Single accumulator: move this warp's 128 columns into
                // registers, free the accumulator for the next tile's MMAs,
                // then convert and store.  Columns: NONE / SWIGLU_BWD
                // [128 half, +128); SWIGLU G [64 half, +64) and U [128 + 64 half, +64).
                const uint16_t* gurow = (EPI == kEpiSwigluBwd) ? p.gu + static_cast<int64_t>(row) * 2 * p.f : nullptr;
                const int c_out = (EPI == kEpiSwiglu) ? t.n0 + 64 * half : t.n0 + 128 * half;
                uint4 gb[4], ub[4];
                auto fetch = [&](int col) {
                    if (EPI == kEpiSwigluBwd && row_ok && col + 32 <= p.f) {
                        const uint4* sg = reinterpret_cast<const uint4*>(gurow + col);
                        const uint4* su = reinterpret_cast<const uint4*>(gurow + p.f + col);
#pragma unroll
                        for (int j = 0; j < 4; ++j) { gb[j] = __ldg(sg + j); ub[j] = __ldg(su + j); }
                    }
                };
                fetch(c_out);
                if (!ptx::mbar_wait(&tfull_bar[0], acc_phase, &s_abort)) { ok = false; break; }
                ptx::tc_fence_after();
                const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
                const bool zero = (MODE == kRaggedK) && t.kiters <= 0;  // empty expert
                uint32_t v[128];
                if (!zero) {
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int c = (EPI == kEpiSwiglu) ? (j < 2 ? 64 * half + 32 * j : 128 + 64 * half + 32 * (j - 2))
                                                          : 128 * half + 32 * j;
                        ptx::tmem_ld_32x32b_x32(tb + c, *reinterpret_cast<uint32_t(*)[32]>(v + 32 * j));
                    }
                    ptx::tmem_wait_ld();
                } else {
#pragma unroll
                    for (int j = 0; j < 128; ++j) v[j] = 0u;
                }
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    if (C2 && rank != 0) ptx::mbar_arrive_cluster_relaxed(ptx::mapa_shared(ptx::smem_addr(&tempty_bar[0]), 0));
                    else ptx::mbar_arrive(&tempty_bar[0]);
                }
                if constexpr (EPI == kEpiSwiglu && FQ) {
                    // A is also quantised to MXFP8 here (f % 32 == 0: every
                    // chunk is whole or past f): row-wise per 32 columns of a
                    // row, column-wise per 32 rows of the expert (this warp's
                    // TMEM quadrant is one such block; rows past the expert
                    // count as zero).
                    uint16_t* gurow_o = p.c + static_cast<int64_t>(row) * p.ldc;
                    uint16_t* arow = p.aux + static_cast<int64_t>(row) * p.f;
                    const int qrow0 = t.m0 + BM * static_cast<int>(rank) + 32 * q;
                    const bool blk = qrow0 < t.row_end;
                    const int64_t bidx = blk ? sch.bb[t.e] + (qrow0 - sch.off[t.e]) / 32 : 0;
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        const int col = c_out + 32 * j;
                        if (col >= p.f) continue;
                        uint32_t ha[16];
                        swiglu_pack32(gurow_o, arow, col, p.f, v + 32 * j, v + 64 + 32 * j, row_ok, ha);
                        const int64_t at = static_cast<int64_t>(row) * p.f + col;
                        if (p.qr_codes && row_ok)
                            p.qr_scales[at / 32] = mx_encode_row32(ha, p.qr_codes + at);
                        if (p.qc_codes) {
                            const uint8_t sc = mx_encode_col32(ha, row_ok, p.qc_codes + at);
                            if (blk) p.qc_scales[bidx * p.f + col + lane] = sc;
                        }
                    }
                } else if (row_ok) {
                    if (EPI == kEpiSwiglu) {
                        uint16_t* gurow_o = p.c + static_cast<int64_t>(row) * p.ldc;
                        uint16_t* arow = p.aux + static_cast<int64_t>(row) * p.f;
#pragma unroll
                        for (int j = 0; j < 2; ++j)
                            store_swiglu32(gurow_o, arow, c_out + 32 * j, p.f, v + 32 * j, v + 64 + 32 * j);
                    } else if (EPI == kEpiSwigluBwd) {
                        uint16_t* dhrow = p.c + static_cast<int64_t>(row) * p.ldc;
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            store_swiglu_bwd32(dhrow, gurow, c_out + 32 * j, p.f, v + 32 * j, gb, ub);
                            if (j < 3) fetch(c_out + 32 * (j + 1));
                        }
                    } else {
                        uint16_t* crow = (MODE == kRaggedK)
                                             ? p.c + (static_cast<int64_t>(t.e) * p.M + row) * p.ldc
                                             : p.c + static_cast<int64_t>(row) * p.ldc;
#pragma unroll
                        for (int j = 0; j < 4; ++j) store_row32(crow, c_out + 32 * j, p.N, v + 32 * j);
                    }
                }
                if (++acc == S::ACC_BUFS) { acc = 0; acc_phase ^= 1u; }
                continue;
            }
            if (EPI == kEpiSwigluBwd) {
                // G and U do not depend on the accumulator: fetch them while
                // the MMAs of this tile are still running.
                const int NCH = acc_n / 32;
                const int cbase = acc_beg;
                const uint16_t* gurow = p.gu + static_cast<int64_t>(row) * 2 * p.f;
                uint16_t* dhrow = p.c + static_cast<int64_t>(row) * p.ldc;
                uint4 gb[4], ub[4];
                auto fetch = [&](int col, uint4 (&g)[4], uint4 (&u)[4]) {  // FQ: one row per thread
                    if (row_ok && col + 32 <= p.f) {
                        const uint4* sg = reinterpret_cast<const uint4*>(gurow + col);
                        const uint4* su = reinterpret_cast<const uint4*>(gurow + p.f + col);
#pragma unroll
                        for (int j = 0; j < 4; ++j) { g[j] = __ldg(sg + j); u[j] = __ldg(su + j); }
                    }
                };
                // without FQ: the warp's 32 rows x 32 columns as coalesced row
                // segments, lane = (row 8 i + lane / 4, 16-byte segment lane % 4)
                uint4 cgb[4], cub[4];
                auto cfetch = [&](int col) {
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int rr = cta_row0 + q_first + 8 * i + (lane >> 2);
                        const bool use = rr < t.row_end && col + 32 <= p.f;
                        const uint16_t* src = p.gu + static_cast<int64_t>(rr) * 2 * p.f + col + 8 * (lane & 3);
                        cgb[i] = use ? __ldg(reinterpret_cast<const uint4*>(src)) : make_uint4(0, 0, 0, 0);
                        cub[i] = use ? __ldg(reinterpret_cast<const uint4*>(src + p.f)) : make_uint4(0, 0, 0, 0);
                    }
                };
                if constexpr (!STAGED) fetch(t.n0 + col_shift + cbase, gb, ub);
                else cfetch(t.n0 + col_shift + cbase);
                if (!ptx::mbar_wait(&tfull_bar[acc], acc_phase, &s_abort)) { ok = false; break; }
                ptx::tc_fence_after();
                const uint32_t tb = tmem_base + static_cast<uint32_t>(acc * BN) + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll 1
                for (int ci = 0; ci < NCH; ++ci) {
                    const int c0 = cbase + ci * 32;
                    const int col = t.n0 + col_shift + c0;
                    uint32_t v[32];
                    ptx::tmem_ld_32x32b_x32(tb + c0, v);
                    uint4 gn[4], un[4];
                    if constexpr (!STAGED) {
                        if (ci + 1 < NCH) fetch(col + 32, gn, un);
                    }
                    ptx::tmem_wait_ld();
                    if constexpr (FQ) {
                        if (col >= p.f) continue;
                        // dH is also quantised to MXFP8 here (f % 32 == 0):
                        // row-wise per 32 columns, column-wise per 32 rows of
                        // the expert (this warp's TMEM quadrant).
                        uint32_t hg[16], hu[16];
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            float gf[8], uf[8], dgf[8], duf[8];
                            unpack8(gb[j], gf);
                            unpack8(ub[j], uf);
#pragma unroll
                            for (int i = 0; i < 8; ++i) {
                                const float da = __uint_as_float(v[8 * j + i]);
                                const float sg = sigmoid_f(gf[i]);
                                dgf[i] = da * uf[i] * sg * (1.0f + gf[i] * (1.0f - sg));
                                duf[i] = da * gf[i] * sg;
                            }
                            const uint4 g4 = pack8(dgf), u4 = pack8(duf);
                            hg[4 * j] = g4.x; hg[4 * j + 1] = g4.y; hg[4 * j + 2] = g4.z; hg[4 * j + 3] = g4.w;
                            hu[4 * j] = u4.x; hu[4 * j + 1] = u4.y; hu[4 * j + 2] = u4.z; hu[4 * j + 3] = u4.w;
                            if (row_ok) {
                                reinterpret_cast<uint4*>(dhrow + col)[j] = g4;
                                reinterpret_cast<uint4*>(dhrow + p.f + col)[j] = u4;
                            }
                        }
                        const int64_t w2 = 2 * static_cast<int64_t>(p.f);
                        const int64_t at = static_cast<int64_t>(row) * w2 + col;
                        if (p.qr_codes && row_ok) {
                            p.qr_scales[at / 32] = mx_encode_row32(hg, p.qr_codes + at);
                            p.qr_scales[(at + p.f) / 32] = mx_encode_row32(hu, p.qr_codes + at + p.f);
                        }
                        if (p.qc_codes) {
                            const int qrow0 = t.m0 + BM * static_cast<int>(rank) + 32 * q;
                            const bool blk = qrow0 < t.row_end;
                            const int64_t bidx = blk ? sch.bb[t.e] + (qrow0 - sch.off[t.e]) / 32 : 0;
                            const uint8_t sg_ = mx_encode_col32(hg, row_ok, p.qc_codes + at);
                            const uint8_t su_ = mx_encode_col32(hu, row_ok, p.qc_codes + at + p.f);
                            if (blk) {
                                p.qc_scales[bidx * w2 + col + lane] = sg_;
                                p.qc_scales[bidx * w2 + p.f + col + lane] = su_;
                            }
                        }
                    } else if (STAGED && col + 32 <= p.f) {
                        // Full chunk, staged through this warp's shared buffer:
                        // G / U arrive as coalesced row segments (8 rows of 64
                        // bytes per instruction), each thread takes its row,
                        // writes dG / dU back in place, and the chunk leaves as
                        // coalesced row segments again.
                        uint8_t* sG = epi_smem + (warp - 2) * kEpiWarpBytes;
                        uint8_t* sU = sG + 32 * kEpiPitch;
                        const int lr = lane >> 2, ls = lane & 3;
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            *reinterpret_cast<uint4*>(sG + epi_seg(8 * i + lr, ls)) = cgb[i];
                            *reinterpret_cast<uint4*>(sU + epi_seg(8 * i + lr, ls)) = cub[i];
                        }
                        __syncwarp();
                        if (ci + 1 < NCH) cfetch(col + 32);
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            uint4* pg = reinterpret_cast<uint4*>(sG + epi_seg(lane, j));
                            uint4* pu = reinterpret_cast<uint4*>(sU + epi_seg(lane, j));
                            float gf[8], uf[8], dgf[8], duf[8];
                            unpack8(*pg, gf);
                            unpack8(*pu, uf);
#pragma unroll
                            for (int i = 0; i < 8; ++i) {
                                const float da = __uint_as_float(v[8 * j + i]);
                                const float sg = sigmoid_f(gf[i]);
                                dgf[i] = da * uf[i] * sg * (1.0f + gf[i] * (1.0f - sg));
                                duf[i] = da * gf[i] * sg;
                            }
                            *pg = pack8(dgf);
                            *pu = pack8(duf);
                        }
                        __syncwarp();
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const int rr = cta_row0 + q_first + 8 * i + lr;
                            if (rr < t.row_end) {
                                uint16_t* drow = p.c + static_cast<int64_t>(rr) * p.ldc;
                                *reinterpret_cast<uint4*>(drow + col + 8 * ls) =
                                    *reinterpret_cast<const uint4*>(sG + epi_seg(8 * i + lr, ls));
                                *reinterpret_cast<uint4*>(drow + p.f + col + 8 * ls) =
                                    *reinterpret_cast<const uint4*>(sU + epi_seg(8 * i + lr, ls));
                            }
                        }
                        __syncwarp();  // the buffers are refilled by the next chunk
                    } else if (!STAGED && row_ok && col + 32 <= p.f) {
                        // full chunk, one row per thread (G / U prefetched per row)
                        uint4* dg = reinterpret_cast<uint4*>(dhrow + col);
                        uint4* du = reinterpret_cast<uint4*>(dhrow + p.f + col);
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            float gf[8], uf[8], dgf[8], duf[8];
                            unpack8(gb[j], gf);
                            unpack8(ub[j], uf);
#pragma unroll
                            for (int i = 0; i < 8; ++i) {
                                const float da = __uint_as_float(v[8 * j + i]);
                                const float sg = sigmoid_f(gf[i]);
                                dgf[i] = da * uf[i] * sg * (1.0f + gf[i] * (1.0f - sg));
                                duf[i] = da * gf[i] * sg;
                            }
                            dg[j] = pack8(dgf);
                            du[j] = pack8(duf);
                        }
                    } else if (row_ok && col < p.f && col + 32 > p.f) {
                        // partial chunk at the end of f: per-row scalar path
                        {
#pragma unroll
                            for (int j = 0; j < 32; ++j) {
                                if (col + j >= p.f) continue;
                                const float da = __uint_as_float(v[j]);
                                const float gv = bf16_to_f32(gurow[col + j]);
                                const float uv = bf16_to_f32(gurow[p.f + col + j]);
                                const float sg = sigmoid_f(gv);
                                dhrow[col + j] = f32_to_bf16(da * uv * sg * (1.0f + gv * (1.0f - sg)));
                                dhrow[p.f + col + j] = f32_to_bf16(da * gv * sg);
                            }
                        }
                    }
                    if constexpr (!STAGED) {
                        if (ci + 1 < NCH) {
#pragma unroll
                            for (int j = 0; j < 4; ++j) { gb[j] = gn[j]; ub[j] = un[j]; }
                        }
                    }
                }
            } else {
                if (!ptx::mbar_wait(&tfull_bar[acc], acc_phase, &s_abort)) { ok = false; break; }
                ptx::tc_fence_after();
                const uint32_t tb = tmem_base + static_cast<uint32_t>(acc * BN) + (static_cast<uint32_t>(q * 32) << 16);
                if (EPI == kEpiSwiglu) {
                    // accumulator columns [0, BN/2) = G, [BN/2, BN) = U of f columns n0..
                    uint16_t* gurow = p.c + static_cast<int64_t>(row) * p.ldc;
                    uint16_t* arow = p.aux + static_cast<int64_t>(row) * p.f;
                    for (int c0 = half * (BN / 4); c0 < (half + 1) * (BN / 4); c0 += 32) {
                        uint32_t g[32], u[32];
                        ptx::tmem_ld_32x32b_x32(tb + c0, g);
                        ptx::tmem_ld_32x32b_x32(tb + BN / 2 + c0, u);
                        ptx::tmem_wait_ld();
                        const int col = t.n0 + c0;
                        if (row_ok && col < p.f) {
                            if (col + 32 <= p.f) {
                                uint4* dg = reinterpret_cast<uint4*>(gurow + col);
                                uint4* du = reinterpret_cast<uint4*>(gurow + p.f + col);
                                uint4* da = reinterpret_cast<uint4*>(arow + col);
#pragma unroll
                                for (int j = 0; j < 4; ++j) {
                                    float gf[8], uf[8], af[8];
#pragma unroll
                                    for (int i = 0; i < 8; ++i) {
                                        gf[i] = __uint_as_float(g[8 * j + i]);
                                        uf[i] = __uint_as_float(u[8 * j + i]);
                                        af[i] = silu_f(gf[i]) * uf[i];
                                    }
                                    dg[j] = pack8(gf);
                                    du[j] = pack8(uf);
                                    da[j] = pack8(af);
                                }
                            } else {
#pragma unroll
                                for (int j = 0; j < 32; ++j) {
                                    if (col + j >= p.f) continue;
                                    float gv = __uint_as_float(g[j]), uv = __uint_as_float(u[j]);
                                    gurow[col + j] = f32_to_bf16(gv);
                                    gurow[p.f + col + j] = f32_to_bf16(uv);
                                    arow[col + j] = f32_to_bf16(silu_f(gv) * uv);
                                }
                            }
                        }
                    }
                } else if (STAGED_PLAIN) {
                    // plain bf16 store, RAGGED_M rows of C or RAGGED_K rows of
                    // C_e: the next 32 accumulator columns are read from TMEM
                    // while this chunk is packed into the warp's buffer (one
                    // row per thread) and leaves as 64-byte row segments
                    // (4 lanes per row, 8 rows per instruction)
                    const bool zero = (MODE == kRaggedK) && t.kiters <= 0;  // empty expert
                    const int row0 = cta_row0 + q_first;
                    uint8_t* sbuf = epi_smem + (warp - 2) * kEpiPlainWarpBytes;
                    const int lr = lane >> 2, ls = lane & 3;
                    uint32_t va[32], vb[32];
                    auto tload = [&](uint32_t (&v)[32], int c0) {
                        if (!zero) {
                            ptx::tmem_ld_32x32b_x32(tb + c0, v);
                        } else {
#pragma unroll
                            for (int j = 0; j < 32; ++j) v[j] = 0u;
                        }
                    };
                    auto chunk_out = [&](const uint32_t (&v)[32], int c0) {
                        const int col = t.n0 + col_shift + c0;
                        if (col >= p.N) return;
                        if (col + 32 <= p.N) {
#pragma unroll
                            for (int j = 0; j < 4; ++j)
                                *reinterpret_cast<uint4*>(sbuf + epi_seg(lane, j)) = make_uint4(
                                    pack_bf16x2(__uint_as_float(v[8 * j + 0]), __uint_as_float(v[8 * j + 1])),
                                    pack_bf16x2(__uint_as_float(v[8 * j + 2]), __uint_as_float(v[8 * j + 3])),
                                    pack_bf16x2(__uint_as_float(v[8 * j + 4]), __uint_as_float(v[8 * j + 5])),
                                    pack_bf16x2(__uint_as_float(v[8 * j + 6]), __uint_as_float(v[8 * j + 7])));
                            __syncwarp();
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const int rr = row0 + 8 * i + lr;
                                if (rr < t.row_end) {
                                    uint16_t* cr = (MODE == kRaggedK)
                                                       ? p.c + (static_cast<int64_t>(t.e) * p.M + rr) * p.ldc
                                                       : p.c + static_cast<int64_t>(rr) * p.ldc;
                                    *reinterpret_cast<uint4*>(cr + col + 8 * ls) =
                                        *reinterpret_cast<const uint4*>(sbuf + epi_seg(8 * i + lr, ls));
                                }
                            }
                            __syncwarp();  // the buffer is refilled by the next chunk
                        } else if (row_ok) {
                            uint16_t* crow = (MODE == kRaggedK)
                                                 ? p.c + (static_cast<int64_t>(t.e) * p.M + row) * p.ldc
                                                 : p.c + static_cast<int64_t>(row) * p.ldc;
#pragma unroll
                            for (int j = 0; j < 32; ++j)
                                if (col + j < p.N) crow[col + j] = f32_to_bf16(__uint_as_float(v[j]));
                        }
                    };
                    const int cbeg = acc_beg;
                    const int NCH = acc_n / 32;
                    tload(va, cbeg);
                    ptx::tmem_wait_ld();
#pragma unroll 1
                    for (int ci = 0; ci < NCH; ci += 2) {
                        if (ci + 1 < NCH) tload(vb, cbeg + 32 * (ci + 1));
                        chunk_out(va, cbeg + 32 * ci);
                        ptx::tmem_wait_ld();
                        if (ci + 1 < NCH) {
                            if (ci + 2 < NCH) tload(va, cbeg + 32 * (ci + 2));
                            chunk_out(vb, cbeg + 32 * (ci + 1));
                            ptx::tmem_wait_ld();
                        }
                    }
                } else {
                    // plain bf16 store: RAGGED_M rows of C, or RAGGED_K rows of C_e
                    uint16_t* crow = (MODE == kRaggedK)
                                         ? p.c + (static_cast<int64_t>(t.e) * p.M + row) * p.ldc
                                         : p.c + static_cast<int64_t>(row) * p.ldc;
                    const bool zero = (MODE == kRaggedK) && t.kiters <= 0;  // empty expert
                    for (int c0 = half * (BN / 2); c0 < (half + 1) * (BN / 2); c0 += 32) {
                        uint32_t v[32];
                        if (!zero) {
                            ptx::tmem_ld_32x32b_x32(tb + c0, v);
                            ptx::tmem_wait_ld();
                        } else {
#pragma unroll
                            for (int j = 0; j < 32; ++j) v[j] = 0u;
                        }
                        const int col = t.n0 + c0;
                        if (row_ok && col < p.N) {
                            if (col + 32 <= p.N) {
                                uint4* dst = reinterpret_cast<uint4*>(crow + col);
#pragma unroll
                                for (int j = 0; j < 4; ++j)
                                    dst[j] = make_uint4(
                                        pack_bf16x2(__uint_as_float(v[8 * j + 0]), __uint_as_float(v[8 * j + 1])),
                                        pack_bf16x2(__uint_as_float(v[8 * j + 2]), __uint_as_float(v[8 * j + 3])),
                                        pack_bf16x2(__uint_as_float(v[8 * j + 4]), __uint_as_float(v[8 * j + 5])),
                                        pack_bf16x2(__uint_as_float(v[8 * j + 6]), __uint_as_float(v[8 * j + 7])));
                            } else {
#pragma unroll
                                for (int j = 0; j < 32; ++j)
                                    if (col + j < p.N) crow[col + j] = f32_to_bf16(__uint_as_float(v[j]));
                            }
                        }
                    }
                }
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                // the arrival orders only this warp's accumulator reads (done:
                // tcgen05.wait::ld, then the tcgen05 fence); a release would
                // also wait for every output store of the tile
                if (C2 && rank != 0) ptx::mbar_arrive_cluster_relaxed(ptx::mapa_shared(ptx::smem_addr(&tempty_bar[acc]), 0));
                else ptx::mbar_arrive(&tempty_bar[acc]);
            }
            if (++acc == S::ACC_BUFS) { acc = 0; acc_phase ^= 1u; }
        }
        if (!ok && lane == 0) {
            s_abort = 1;
            flag_status(p.status, MOE_ERR_DEVICE_TIMEOUT);
        }
    }

    __syncthreads();
    if (threadIdx.x == 0 && p.sync_done) {
        __threadfence();
        if (atomicAdd(p.sync_exit, 1u) == gridDim.x - 1) {
            atomicExch(p.sync_done, 0u);
            atomicExch(p.sync_exit, 0u);
        }
    }
    if (C2) ptx::cluster_sync();  // the pair's MMAs and remote signals are done
    if (warp == 1) {
        if (s_abort) {
            // Let in-flight tensor-core and TMA work drain before TMEM is freed.
            const uint64_t t0 = ptx::globaltimer();
            while (ptx::globaltimer() - t0 < 20000000ull) { }
        }
        ptx::tc_fence_after();
        if (C2) ptx::tmem_dealloc_pair(tmem_base, S::TMEM_COLS);
        else ptx::tmem_dealloc(tmem_base, S::TMEM_COLS);
    }
}

// ------------------------------------------------------------------ MXFP8 scale atoms
//
// An atom holds the E8M0 scales of one 128-row (or 128-column) tile of an
// operand for 4 consecutive K-blocks of 32: 32-bit word 4 i + j (byte
// 16 i + 4 j) carries the four block scales of row i + 32 j, in K order.
// Scales outside the operand (rows past the buffer or the group, K-blocks past
// the end) are 127, i.e. 2^0, so that zero-filled codes stay zero.

enum { kSfRowsGrouped = 0, kSfRowsWeight = 1, kSfRowsWeightSwiglu = 2, kSfRowsWeightSwiglu2 = 3 };
enum { kSfColsWeight = 0, kSfColsGrouped = 1 };

struct SfRowsArgs {
    const uint8_t* canon;  // [rows][nblk] row-wise scales
    int64_t rows;
    int nblk;              // K / 32
    int ks;                // K stages of 4 blocks = ceil(nblk / 4)
    int mode;
    int E, N, f;           // weights: E groups of N rows (SwiGLU: N = 2f)
    int tiles_per_group;   // weights
    const int32_t* offsets;
    uint32_t* atoms;
    int32_t* status;       // grouped: MOE_ERR_DEVICE_BOUNDS for offsets out of range or going down
};

struct SfColsArgs {
    const uint8_t* canon;  // [blocks][cols] column-wise scales
    int64_t cols;
    int nct;               // column tiles = ceil(cols / 128)
    int mode;
    int E, K;              // weights: E groups of K rows
    int64_t rows;          // grouped: rows of the operand the offsets index
    const int32_t* offsets;
    uint32_t* atoms;
    int32_t* status;       // grouped: MOE_ERR_DEVICE_BOUNDS for offsets out of range or going down
};

// group table of `offsets` in shared memory: off, prefix of ceil(m/128) (rt),
// prefix of ceil(m/32) (bb); built by warp 0
__device__ void sf_group_table(const int32_t* offsets, int E, int64_t rows, int* s_off, int* s_rt,
                               int* s_bb, int32_t* status) {
    const int lane = threadIdx.x & 31;
    if (threadIdx.x >= 32) return;
    load_group_offsets(offsets, E, rows, s_off, status);
    const int per = (E + 31) / 32;
    const int lo = min(E, lane * per), hi = min(E, lo + per);
    int a = 0, b = 0;
    for (int g = lo; g < hi; ++g) {
        const int m = max(0, s_off[g + 1] - s_off[g]);
        a += (m + 127) / 128;
        b += (m + 31) / 32;
    }
    int ia = a, ib = b;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int va = __shfl_up_sync(0xffffffffu, ia, o), vb = __shfl_up_sync(0xffffffffu, ib, o);
        if (lane >= o) { ia += va; ib += vb; }
    }
    int ra = ia - a, rb = ib - b;
    for (int g = lo; g < hi; ++g) {
        s_rt[g] = ra;
        s_bb[g] = rb;
        const int m = max(0, s_off[g + 1] - s_off[g]);
        ra += (m + 127) / 128;
        rb += (m + 31) / 32;
    }
    if (lane == 31) { s_rt[E] = ia; s_bb[E] = ib; }
}

__device__ __forceinline__ int largest_le(const int* pref, int n, int v) {
    int lo = 0, hi = n;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (pref[mid] <= v) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// Row of the canonical scale array that holds row r (0..127) of row tile
// `tile` of the operand; false when that row lies past the group / operand.
__device__ __forceinline__ bool sf_row_of(const SfRowsArgs& a, const int* s_off, const int* s_rt,
                                          int64_t tile, int r, int64_t* row) {
    if (a.mode == kSfRowsGrouped) {
        const int g = largest_le(s_rt, a.E, static_cast<int>(tile));
        *row = s_off[g] + (tile - s_rt[g]) * 128 + r;
        return *row < a.rows;  // rows past the expert belong to the next one
    }
    const int g = static_cast<int>(tile / a.tiles_per_group);
    const int t = static_cast<int>(tile - static_cast<int64_t>(g) * a.tiles_per_group);
    int n;
    bool valid;
    if (a.mode == kSfRowsWeight) {
        n = 128 * t + r;
        valid = n < a.N;
    } else if (a.mode == kSfRowsWeightSwiglu) {  // 64 gate rows then the 64 matching up rows
        const int c = 64 * t + (r & 63);
        n = r < 64 ? c : a.f + c;
        valid = c < a.f;
    } else {  // 256-wide SwiGLU tile t / 2: atom 0 = 128 gate rows, atom 1 = the up rows
        const int c = 128 * (t >> 1) + r;
        n = (t & 1) ? a.f + c : c;
        valid = c < a.f;
    }
    *row = static_cast<int64_t>(g) * a.N + n;
    return valid;
}

// A block stages one row tile x up to kSfStages K stages of the canonical
// scales in shared memory (each row's 4-scale words read contiguously), then
// writes the tile's atoms, which are consecutive in memory.
constexpr int kSfStages = 16;

__global__ void __launch_bounds__(256) sf_rows_kernel(const SfRowsArgs a) {
    __shared__ int s_off[MAX_E + 1], s_rt[MAX_E + 1], s_bb[MAX_E + 1];
    __shared__ uint32_t sw[128][kSfStages + 1];
    if (a.mode == kSfRowsGrouped) sf_group_table(a.offsets, a.E, a.rows, s_off, s_rt, s_bb, a.status);
    __syncthreads();
    const int64_t tiles = (a.mode == kSfRowsGrouped) ? s_rt[a.E]
                                                     : static_cast<int64_t>(a.E) * a.tiles_per_group;
    const int nch = (a.ks + kSfStages - 1) / kSfStages;
    // a stage's 4 scales form an aligned 32-bit word
    const bool words = (a.nblk % 4) == 0 && (reinterpret_cast<uintptr_t>(a.canon) & 3) == 0;
    // 16 stages start 16-byte aligned in every row
    const bool quads = (a.nblk % 16) == 0 && (reinterpret_cast<uintptr_t>(a.canon) & 15) == 0;
    for (int64_t item = blockIdx.x; item < tiles * nch; item += gridDim.x) {
        const int64_t tile = item / nch;
        const int k0 = static_cast<int>(item - tile * nch) * kSfStages;
        const int nst = min(kSfStages, a.ks - k0);
        // thread = (row r, 8 stages from s0): the row is located once and its
        // 8 stage words (32 contiguous bytes) read with two 16-byte loads
        // where the canonical rows allow it
        {
            static_assert(kSfStages == 16, "two threads per row, 8 stages each");
            const int r = threadIdx.x >> 1, s0 = (threadIdx.x & 1) * 8;
            uint32_t v[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) v[j] = 0x7F7F7F7Fu;  // 2^0: zero-filled codes stay zero
            int64_t row;
            if (s0 < nst && sf_row_of(a, s_off, s_rt, tile, r, &row)) {
                const uint8_t* src = a.canon + row * a.nblk + 4 * (k0 + s0);
                if (quads && s0 + 8 <= nst) {
                    const uint4 x0 = __ldg(reinterpret_cast<const uint4*>(src));
                    const uint4 x1 = __ldg(reinterpret_cast<const uint4*>(src) + 1);
                    v[0] = x0.x; v[1] = x0.y; v[2] = x0.z; v[3] = x0.w;
                    v[4] = x1.x; v[5] = x1.y; v[6] = x1.z; v[7] = x1.w;
                } else {
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        if (s0 + j >= nst) break;
                        const int blk = 4 * (k0 + s0 + j);
                        if (words) {
                            v[j] = __ldg(reinterpret_cast<const uint32_t*>(a.canon + row * a.nblk + blk));
                        } else {
                            uint32_t x = 0;
#pragma unroll
                            for (int b = 0; b < 4; ++b) {
                                const uint32_t y = blk + b < a.nblk ? a.canon[row * a.nblk + blk + b] : 127u;
                                x |= y << (8 * b);
                            }
                            v[j] = x;
                        }
                    }
                }
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) sw[r][s0 + j] = v[j];
        }
        __syncthreads();
        uint32_t* out = a.atoms + (tile * a.ks + k0) * 128;
        for (int i = threadIdx.x; i < nst * 128; i += blockDim.x) {
            const int st = i >> 7, w = i & 127;
            out[i] = sw[(w >> 2) + 32 * (w & 3)][st];  // word 4 i + j: row i + 32 j
        }
        __syncthreads();
    }
}

// A block stages the 4 canonical block rows of one K stage (slot) for up to
// 8 column tiles in shared memory (read as contiguous row segments), then
// writes those atoms, which are consecutive in memory.
constexpr int kSfColTiles = 8;

__global__ void __launch_bounds__(256) sf_cols_kernel(const SfColsArgs a) {
    __shared__ int s_off[MAX_E + 1], s_rt[MAX_E + 1], s_bb[MAX_E + 1];
    __shared__ __align__(16) uint8_t sb[4][kSfColTiles * 128];
    if (a.mode == kSfColsGrouped) sf_group_table(a.offsets, a.E, a.rows, s_off, s_rt, s_bb, a.status);
    __syncthreads();
    const int ksw = (a.K / 32 + 3) / 4;  // weights: stages per expert
    const int64_t slots = (a.mode == kSfColsGrouped) ? s_rt[a.E] : static_cast<int64_t>(a.E) * ksw;
    const int nch = (a.nct + kSfColTiles - 1) / kSfColTiles;
    const bool vec = (a.cols % 16) == 0 && (reinterpret_cast<uintptr_t>(a.canon) & 15) == 0;
    for (int64_t item = blockIdx.x; item < slots * nch; item += gridDim.x) {
        const int64_t slot = item / nch;
        const int ct0 = static_cast<int>(item - slot * nch) * kSfColTiles;
        const int nct = min(kSfColTiles, a.nct - ct0);
        int64_t bb;
        int nb, ks;
        if (a.mode == kSfColsGrouped) {
            const int g = largest_le(s_rt, a.E, static_cast<int>(slot));
            ks = static_cast<int>(slot - s_rt[g]);
            bb = s_bb[g];
            nb = (max(0, s_off[g + 1] - s_off[g]) + 31) / 32;
        } else {
            const int g = static_cast<int>(slot / ksw);
            ks = static_cast<int>(slot - static_cast<int64_t>(g) * ksw);
            nb = a.K / 32;
            bb = static_cast<int64_t>(g) * nb;
        }
        const int64_t col0 = 128 * static_cast<int64_t>(ct0);
        // 4 block rows x nct * 128 columns, 16 bytes per thread step
        for (int i = threadIdx.x; i < 4 * kSfColTiles * 8; i += blockDim.x) {
            const int b = i / (kSfColTiles * 8), v = i % (kSfColTiles * 8);
            const int blk = 4 * ks + b;
            const int64_t c = col0 + 16 * v;
            uint4 val = make_uint4(0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu);
            if (blk < nb && 16 * v < nct * 128) {
                const uint8_t* src = a.canon + (bb + blk) * a.cols + c;
                if (vec && c + 16 <= a.cols) {
                    val = __ldg(reinterpret_cast<const uint4*>(src));
                } else {
                    uint8_t tmp[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) tmp[j] = (c + j < a.cols) ? src[j] : 127u;
                    val = *reinterpret_cast<const uint4*>(tmp);
                }
            }
            *reinterpret_cast<uint4*>(&sb[b][16 * v]) = val;
        }
        __syncthreads();
        uint32_t* out = a.atoms + (slot * a.nct + ct0) * 128;
        for (int i = threadIdx.x; i < nct * 128; i += blockDim.x) {
            const int ct = i >> 7, w = i & 127;
            const int c = 128 * ct + (w >> 2) + 32 * (w & 3);
            out[i] = static_cast<uint32_t>(sb[0][c]) | (static_cast<uint32_t>(sb[1][c]) << 8) |
                     (static_cast<uint32_t>(sb[2][c]) << 16) | (static_cast<uint32_t>(sb[3][c]) << 24);
        }
        __syncthreads();
    }
}

// ------------------------------------------------------------------ host side

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// Tensor map (bf16 or bytes), 128-byte swizzle, zero fill outside the tensor.
// dims / strides are in elements of `esize` bytes.
static int make_map(CUtensorMap* m, const void* base, int esize, int rank, const uint64_t* dims,
                    const uint64_t* strides_elems, const uint32_t* box) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return MOE_ERR_CUDA;
    cuuint64_t gd[3], gs[2];
    cuuint32_t bx[3], es[3] = {1, 1, 1};
    for (int i = 0; i < rank; ++i) { gd[i] = dims[i]; bx[i] = box[i]; }
    for (int i = 0; i < rank - 1; ++i) gs[i] = strides_elems[i] * esize;
    const CUtensorMapDataType dt = esize == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
    CUresult r = fn(m, dt, rank, const_cast<void*>(base), gd, gs, bx, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MOE_OK : MOE_ERR_CUDA;
}

// Tensor map of a scale-atom array: `atoms` rows of 512 bytes (128 x 32-bit
// words), one atom per box.
// A scale-atom array as a 3-D tensor [d2][d1][atom] of 32-bit words, rows of
// dim 2 `stride2` atoms apart, boxes of b2 x b1 whole atoms (MXFP8 pairs load
// kSfGroup K stages per box; boxes that reach past d1 or d2 read zeros there).
static int make_atom_map(CUtensorMap* m, const void* base, int64_t d1, int64_t d2, int64_t stride2,
                         int b1, int b2) {
    EncodeTiledFn fn = encode_fn();
    if (!fn || d1 < 1 || d2 < 1 || d1 > INT32_MAX || d2 > INT32_MAX || stride2 < d1) return MOE_ERR_CUDA;
    cuuint64_t gd[3] = {kAtomBytes / 4, static_cast<cuuint64_t>(d1), static_cast<cuuint64_t>(d2)};
    cuuint64_t gs[2] = {kAtomBytes, static_cast<cuuint64_t>(stride2) * kAtomBytes};
    cuuint32_t bx[3] = {kAtomBytes / 4, static_cast<cuuint32_t>(b1), static_cast<cuuint32_t>(b2)};
    cuuint32_t es[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<void*>(base), gd, gs, bx, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MOE_OK : MOE_ERR_CUDA;
}

template <int BN, int MODE, bool A_MN, bool B_MN, int EPI, bool MX, bool C2 = false, bool FQ = false>
static int launch(const CUtensorMap& ma, const CUtensorMap& mb, const Params& p, int grid,
                  cudaStream_t st) {
    using S = Shape<BN, MX, C2, epi_smem_bytes(EPI, MX, C2, FQ)>;
    auto kern = gg_kernel<BN, MODE, A_MN, B_MN, EPI, MX, C2, FQ>;
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [&] {
        attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::SMEM_BYTES);
    });
    if (attr_err != cudaSuccess) return MOE_ERR_CUDA;
    if (!C2) {
        kern<<<grid, S::THREADS, S::SMEM_BYTES, st>>>(ma, mb, p);
    } else {
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.gridDim = dim3(grid & ~1, 1, 1);
        cfg.blockDim = dim3(S::THREADS, 1, 1);
        cfg.dynamicSmemBytes = S::SMEM_BYTES;
        cfg.stream = st;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&cfg, kern, ma, mb, p) != cudaSuccess) return MOE_ERR_CUDA;
    }
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}

// fq: the epilogue quantises its output itself (only where the kernel can:
// the single-accumulator SwiGLU epilogue and the SwiGLU-backward one).
template <int BN, bool MX, bool C2 = false>
static bool can_fuse_q(int epi) {
    if (epi == kEpiSwiglu) return Shape<BN, MX, C2>::ACC_BUFS == 1;
    return epi == kEpiSwigluBwd && Shape<BN, MX, C2>::ACC_BUFS == 2;
}

template <int BN, bool MX, bool C2 = false>
static int launch_ragged_m(bool b_mn, int epi, const CUtensorMap& ma, const CUtensorMap& mb,
                           const Params& p, int grid, cudaStream_t st, bool fq = false) {
    if (epi == kEpiSwiglu) {
        if constexpr (Shape<BN, MX, C2>::ACC_BUFS == 1)
            if (fq) return launch<BN, kRaggedM, false, false, kEpiSwiglu, MX, C2, true>(ma, mb, p, grid, st);
        if (fq) return MOE_ERR_UNSUPPORTED;
        return launch<BN, kRaggedM, false, false, kEpiSwiglu, MX, C2>(ma, mb, p, grid, st);
    }
    // The SwiGLU-backward epilogue needs two accumulators: with one, its 128
    // columns plus the G / U operands exceed the 168 registers a thread of a
    // 10-warp CTA can hold.
    constexpr bool kBwdOk = Shape<BN, MX, C2>::ACC_BUFS == 2;
    if (epi == kEpiSwigluBwd) {
        if constexpr (kBwdOk) {
            if (fq) {
                if (!b_mn) return launch<BN, kRaggedM, false, false, kEpiSwigluBwd, MX, C2, true>(ma, mb, p, grid, st);
                return launch<BN, kRaggedM, false, true, kEpiSwigluBwd, MX, C2, true>(ma, mb, p, grid, st);
            }
            if (!b_mn) return launch<BN, kRaggedM, false, false, kEpiSwigluBwd, MX, C2>(ma, mb, p, grid, st);
            return launch<BN, kRaggedM, false, true, kEpiSwigluBwd, MX, C2>(ma, mb, p, grid, st);
        }
        return MOE_ERR_UNSUPPORTED;
    }
    if (fq) return MOE_ERR_UNSUPPORTED;
    if (!b_mn) return launch<BN, kRaggedM, false, false, kEpiNone, MX, C2>(ma, mb, p, grid, st);
    return launch<BN, kRaggedM, false, true, kEpiNone, MX, C2>(ma, mb, p, grid, st);
}

// MOE_GG_NO_PAIRS=1 in the environment keeps the BF16 ragged-M GEMMs on single
// CTAs (128 x 256 tiles) instead of CTA pairs; MOE_GG_MX_NARROW=1 keeps the
// MXFP8 GEMMs on 128 x 128 tiles.  Read once per process.
static bool env_flag(const char* name) {
    const char* v = getenv(name);
    return v && v[0] == '1';
}
static const bool g_no_pairs = env_flag("MOE_GG_NO_PAIRS");
static const bool g_mx_narrow = env_flag("MOE_GG_MX_NARROW");
// MOE_GG_MX_NO_PAIRS=1: the 256-wide MXFP8 ragged-M GEMMs run on single CTAs
static const bool g_mx_no_pairs = env_flag("MOE_GG_MX_NO_PAIRS");
// MOE_GG_SYNC_SLACK=n: how many tiles a CTA may start ahead of the others
// (Params::sync_done; default 1, 0 = off)
static int env_int(const char* name, int dflt) {
    const char* v = getenv(name);
    return (v && v[0]) ? atoi(v) : dflt;
}
static const int g_sync_slack = env_int("MOE_GG_SYNC_SLACK", 1);
// MOE_GG_NO_HALF_TILES=1: BF16 ragged-M pairs run M = 256 MMAs on every tile
// (Params::half_tiles off)
static const bool g_no_half_tiles = env_flag("MOE_GG_NO_HALF_TILES");
// MOE_GG_SINGLE_BWD=1: the BF16 SwiGLU-backward GEMM runs on single CTAs
// (one row per thread in the epilogue) instead of CTA pairs
static const bool g_single_bwd = env_flag("MOE_GG_SINGLE_BWD");
// MOE_GG_B_EVICT_NORMAL=1: ragged-M GEMMs load the weights with the normal L2
// priority (for measuring what the evict-last hint does)
static const bool g_b_evict_normal = env_flag("MOE_GG_B_EVICT_NORMAL");
// Ragged-M GEMMs other than the SwiGLU-backward one walk an expert's tiles
// row tile fastest and keep the activations in L2 (evict-last) rather than
// the weights: the rows a wave of tiles shares with the next are then the
// expert's activations (16 MB on the large layer) instead of its weight block
// (32 MB).  Large layer, one box: GEMM1 DRAM reads 11.4 -> 8.1 GB, dX 12.6 ->
// 10.7 GB, GEMM2 4.6 -> 4.4 GB per launch, 1-2 % less time; the
// SwiGLU-backward GEMM read 4 % more that way and keeps column tiles fastest.
// MOE_GG_N_FASTEST=1 restores column tiles fastest for all of them.
static const bool g_n_fastest = env_flag("MOE_GG_N_FASTEST");


// MXFP8 GEMMs run 128 x 256 tiles when the output is at least 256 wide
// (SwiGLU: 128 f-columns of G and of U), 128 x 128 tiles otherwise and for the
// SwiGLU-backward epilogue (see launch_ragged_m).
static bool mx_wide(const moe_gg_args* a) {
    if (g_mx_narrow || a->epilogue == MOE_EPI_SWIGLU_BWD) return false;
    return a->epilogue == MOE_EPI_SWIGLU ? a->N / 2 >= 128 : a->N >= 256;
}

// Atom columns of the B operand (one atom per 128 rows / columns of B per K
// stage), padded to whole tiles: tiles x atoms per tile.
static int64_t mx_b_atom_cols(const moe_gg_args* a) {
    const bool wide = mx_wide(a);
    if (a->mode == MOE_GG_RAGGED_M && a->epilogue == MOE_EPI_SWIGLU)
        return wide ? 2 * cdiv(a->N / 2, 128) : cdiv(a->N / 2, 64);
    return wide ? 2 * cdiv(a->N, 256) : cdiv(a->N, 128);
}

// Bytes of scale atoms the MXFP8 GEMM needs for its A and B operands.
static void mx_atom_bytes(const moe_gg_args* a, size_t* A, size_t* B) {
    const int64_t rtiles = a->M_total / BM + a->E;  // >= sum_e ceil(m_e / 128)
    if (a->mode == MOE_GG_RAGGED_M) {
        const int64_t ks = cdiv(a->K, 128);
        *A = static_cast<size_t>(rtiles * ks * kAtomBytes);
        *B = static_cast<size_t>(static_cast<int64_t>(a->E) * mx_b_atom_cols(a) *
                                 ks * kAtomBytes);
    } else {
        *A = static_cast<size_t>(rtiles * cdiv(a->M, 128) * kAtomBytes);
        *B = static_cast<size_t>(rtiles * mx_b_atom_cols(a) * kAtomBytes);
    }
}

static size_t al256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Per-expert copies of the ragged-K operand maps with the row extent cut at
// the expert's last row (see Params::kmaps).  Empty experts keep one row
// (their maps are never used); offsets are clamped to [1, rows].
__global__ void kmap_kernel(const __grid_constant__ CUtensorMap tmA,
                            const __grid_constant__ CUtensorMap tmB, const int32_t* offsets,
                            int E, int64_t rows, CUtensorMap* maps) {
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e < E) {
        int64_t end = offsets[e + 1];
        end = end < 1 ? 1 : (end > rows ? rows : end);
        maps[2 * e] = tmA;
        maps[2 * e + 1] = tmB;
        ptx::tmap_replace_dim1(&maps[2 * e], static_cast<uint32_t>(end));
        ptx::tmap_replace_dim1(&maps[2 * e + 1], static_cast<uint32_t>(end));
    }
    ptx::tmap_release();
}

static size_t kmap_bytes(int E) { return al256(static_cast<size_t>(2) * E * sizeof(CUtensorMap)); }


}  // namespace gg

size_t grouped_gemm_workspace_bytes(const moe_gg_args* a) {
    if (!a) return 0;
    if (a->dtype == MOE_DTYPE_BF16 && a->mode == MOE_GG_RAGGED_K && a->E >= 1 && a->E <= gg::MAX_E)
        return gg::kmap_bytes(a->E);  // optional: per-expert tensor maps
    if (a->dtype != MOE_DTYPE_MXFP8) return 0;
    size_t A = 0, B = 0;
    gg::mx_atom_bytes(a, &A, &B);
    return gg::al256(A) + gg::al256(B);
}

int grouped_gemm(const moe_gg_args* a, cudaStream_t st) {
    using namespace gg;
    const int mode = a->mode, epi = a->epilogue;
    const bool mx = a->dtype == MOE_DTYPE_MXFP8;
    if (!mx && a->dtype != MOE_DTYPE_BF16) return MOE_ERR_INVALID_ARG;
    const int es = mx ? 1 : 2;  // element size of A / B
    if (a->E < 1 || a->E > MAX_E || a->N < 1 || a->M_total < 0 || a->M_total >= (1ll << 31))
        return MOE_ERR_INVALID_ARG;
    if (!a->offsets || !a->a || !a->b || !a->c) return MOE_ERR_INVALID_ARG;
    if (!aligned16(a->a) || !aligned16(a->b) || !aligned16(a->c)) return MOE_ERR_INVALID_ARG;
    if (a->N % (mx ? 32 : 8)) return MOE_ERR_INVALID_ARG;
    if (mx && (!a->a_scales || !a->b_scales)) return MOE_ERR_INVALID_ARG;
    if (mx && (!a->workspace || !aligned16(a->workspace) ||
               a->workspace_bytes < grouped_gemm_workspace_bytes(a)))
        return MOE_ERR_INVALID_ARG;

    Params p{};
    if (g_sync_slack > 0) {
        // the next counter pair of this device's slots
        static unsigned int* base[64] = {nullptr};
        static std::atomic<unsigned int> seq{0};
        int dev = 0;
        if (cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < 64) {
            if (!base[dev]) {
                void* a = nullptr;
                if (cudaGetSymbolAddress(&a, g_sync) == cudaSuccess) base[dev] = static_cast<unsigned int*>(a);
            }
            if (base[dev]) {
                const unsigned int slot = seq.fetch_add(1u) % kSyncSlots;
                p.sync_done = base[dev] + 2 * slot;
                p.sync_exit = base[dev] + 2 * slot + 1;
                p.sync_slack = g_sync_slack;
            }
        }
    }
    p.b_evict_normal = g_b_evict_normal ? 1 : 0;
    p.half_tiles = g_no_half_tiles ? 0 : 1;
    p.m_fastest = (a->mode == MOE_GG_RAGGED_M && a->epilogue != MOE_EPI_SWIGLU_BWD && !g_n_fastest) ? 1 : 0;
    p.offsets = a->offsets;
    p.E = a->E;
    p.M_total = static_cast<int>(a->M_total);
    p.M = a->M;
    p.N = a->N;
    p.K = a->K;
    p.c = static_cast<uint16_t*>(a->c);
    if (mx) {
        size_t A = 0, B = 0;
        mx_atom_bytes(a, &A, &B);
        p.sfa = static_cast<const uint8_t*>(a->workspace);
        p.sfb = static_cast<const uint8_t*>(a->workspace) + al256(A);
    }
    p.status = a->status;
    const int sms = num_sms();
    const uint32_t box_k = mx ? 128 : 64;  // 128 bytes of K (or of MN for MN-major boxes)
    CUtensorMap ma, mb;

    const bool want_qr = a->q_row_codes || a->q_row_scales;
    const bool want_qc = a->q_col_codes || a->q_col_scales;
    if (want_qr || want_qc) {
        // fused MXFP8 quantisation of the SwiGLU / SwiGLU-backward output
        if (mode != MOE_GG_RAGGED_M || (epi != MOE_EPI_SWIGLU && epi != MOE_EPI_SWIGLU_BWD))
            return MOE_ERR_INVALID_ARG;
        const int64_t W = epi == MOE_EPI_SWIGLU ? a->N / 2 : 2 * static_cast<int64_t>(a->N);
        if (W % 32 || a->N % (epi == MOE_EPI_SWIGLU ? 64 : 32)) return MOE_ERR_INVALID_ARG;
        if (want_qr && (!a->q_row_codes || !a->q_row_scales || !aligned16(a->q_row_codes) ||
                        !aligned16(a->q_row_scales)))
            return MOE_ERR_INVALID_ARG;
        if (want_qc && (!a->q_col_codes || !a->q_col_scales || !aligned16(a->q_col_codes) ||
                        !aligned16(a->q_col_scales)))
            return MOE_ERR_INVALID_ARG;
    }

    if (mode == MOE_GG_RAGGED_M) {
        if (a->K < 1 || a->K % (mx ? 32 : 8)) return MOE_ERR_INVALID_ARG;
        if (a->M_total == 0) return MOE_OK;
        const uint64_t K = a->K, N = a->N, E = a->E, Mt = a->M_total;
        {
            uint64_t d[2] = {K, Mt}, s[1] = {K};
            uint32_t b[2] = {box_k, 128};
            MOE_TRY(make_map(&ma, a->a, es, 2, d, s, b));
        }
        const bool wide = mx && mx_wide(a);
        const int bn = mx ? (wide ? 256 : 128) : ((epi == MOE_EPI_SWIGLU || a->N >= 256) ? 256 : 128);
        if (epi == MOE_EPI_SWIGLU) {
            if (a->b_mn_major || !a->aux || !aligned16(a->aux) || a->N % 16) return MOE_ERR_INVALID_ARG;
            p.f = a->N / 2;
            p.ldc = a->N;
            p.aux = static_cast<uint16_t*>(a->aux);
        } else if (epi == MOE_EPI_SWIGLU_BWD) {
            if (!a->gu || !aligned16(a->gu)) return MOE_ERR_INVALID_ARG;
            p.f = a->N;
            p.ldc = 2 * static_cast<int64_t>(a->N);
            p.gu = static_cast<const uint16_t*>(a->gu);
        } else if (epi == MOE_EPI_NONE) {
            p.ldc = a->N;
        } else {
            return MOE_ERR_INVALID_ARG;
        }
        // BF16 with 256-wide tiles runs on CTA pairs (cta_group::2, 256 x 256
        // tiles).  A pair waits for the slower of its two epilogues, so the
        // SwiGLU-backward one (G/U reads, a sigmoid per element) stages G, U
        // and dH through shared memory as coalesced row segments there; with
        // one row per thread instead it made the paired GEMM slower than a
        // single CTA (large layer: 5.3-5.7 ms against 4.4-4.7; staged 4.2-4.3).
        // MXFP8 with 256-wide tiles: CTA pairs as well (each CTA loads half of
        // B and one scale atom of it: a stage is 33 KB instead of 49 KB, six
        // stages instead of four, for a main loop twice as fast as BF16's)
        const bool pair = (mx ? (wide && !g_mx_no_pairs)
                              : (bn == 256 && (epi != MOE_EPI_SWIGLU_BWD || !g_single_bwd))) &&
                          !g_no_pairs;
        // the epilogues that quantise their output themselves: the wide MXFP8
        // SwiGLU one and every SwiGLU-backward one; otherwise the output is
        // quantised after the GEMM (quantise_after)
        const int ge0 = epi == MOE_EPI_SWIGLU ? kEpiSwiglu : (epi == MOE_EPI_SWIGLU_BWD ? kEpiSwigluBwd : kEpiNone);
        const bool can_fuse = mx ? (pair ? can_fuse_q<256, true, true>(ge0)
                                         : (wide ? can_fuse_q<256, true>(ge0) : can_fuse_q<128, true>(ge0)))
                                 : (pair ? can_fuse_q<256, false, true>(ge0)
                                         : (bn == 256 ? can_fuse_q<256, false>(ge0) : can_fuse_q<128, false>(ge0)));
        const bool fuse_q = (want_qr || want_qc) && can_fuse;
        if (fuse_q) {
            p.qr_codes = static_cast<uint8_t*>(a->q_row_codes);
            p.qr_scales = static_cast<uint8_t*>(a->q_row_scales);
            p.qc_codes = static_cast<uint8_t*>(a->q_col_codes);
            p.qc_scales = static_cast<uint8_t*>(a->q_col_scales);
        }
        auto quantise_after = [&](int rc) -> int {
            if (rc != MOE_OK || fuse_q || !(want_qr || want_qc)) return rc;
            const uint16_t* out = static_cast<const uint16_t*>(epi == MOE_EPI_SWIGLU ? a->aux : a->c);
            const int64_t W = epi == MOE_EPI_SWIGLU ? a->N / 2 : 2 * static_cast<int64_t>(a->N);
            if (want_qr)
                MOE_TRY(mxfp8_quantize_impl(out, a->M_total, W, 1, nullptr, 0,
                                            static_cast<uint8_t*>(a->q_row_codes),
                                            static_cast<uint8_t*>(a->q_row_scales), a->status, st));
            if (want_qc)
                MOE_TRY(mxfp8_quantize_impl(out, a->M_total, W, 0, a->offsets, a->E,
                                            static_cast<uint8_t*>(a->q_col_codes),
                                            static_cast<uint8_t*>(a->q_col_scales), a->status, st));
            return MOE_OK;
        };
        if (!a->b_mn_major) {
            uint64_t d[3] = {K, N, E}, s[2] = {K, N * K};
            uint32_t b[3] = {box_k, static_cast<uint32_t>((epi == MOE_EPI_SWIGLU || pair) ? bn / 2 : bn), 1};
            MOE_TRY(make_map(&mb, a->b, es, 3, d, s, b));
        } else {
            uint64_t d[3] = {N, K, E}, s[2] = {N, K * N};
            uint32_t b[3] = {box_k, box_k, 1};
            MOE_TRY(make_map(&mb, a->b, es, 3, d, s, b));
        }
        const int64_t n_tiles = (epi == MOE_EPI_SWIGLU) ? cdiv(p.f, bn / 2) : cdiv(a->N, bn);
        const int64_t bound = (Mt / (pair ? 2 * BM : BM) + E) * n_tiles * (pair ? 2 : 1);
        const int grid = static_cast<int>(bound < sms ? bound : sms);
        const int ge = epi == MOE_EPI_SWIGLU ? kEpiSwiglu : (epi == MOE_EPI_SWIGLU_BWD ? kEpiSwigluBwd : kEpiNone);
        if (mx) {
            const int cgrid = sms * 4;
            SfRowsArgs ra{};
            ra.canon = a->a_scales; ra.rows = a->M_total; ra.nblk = a->K / 32;
            ra.ks = static_cast<int>(cdiv(a->K, 128)); ra.mode = kSfRowsGrouped; ra.E = a->E;
            ra.offsets = a->offsets; ra.atoms = reinterpret_cast<uint32_t*>(const_cast<uint8_t*>(p.sfa));
            ra.status = a->status;
            sf_rows_kernel<<<cgrid, 256, 0, st>>>(ra);
            MOE_LAUNCH_CHECK();
            if (!a->b_mn_major) {
                SfRowsArgs rb{};
                rb.canon = a->b_scales; rb.rows = static_cast<int64_t>(a->E) * a->N;
                rb.nblk = a->K / 32; rb.ks = ra.ks; rb.E = a->E; rb.N = a->N; rb.f = p.f;
                rb.mode = epi != MOE_EPI_SWIGLU ? kSfRowsWeight
                                                : (wide ? kSfRowsWeightSwiglu2 : kSfRowsWeightSwiglu);
                rb.tiles_per_group = static_cast<int>(mx_b_atom_cols(a));
                rb.atoms = reinterpret_cast<uint32_t*>(const_cast<uint8_t*>(p.sfb));
                sf_rows_kernel<<<cgrid, 256, 0, st>>>(rb);
            } else {
                SfColsArgs cb{};
                cb.canon = a->b_scales; cb.cols = a->N; cb.nct = static_cast<int>(mx_b_atom_cols(a));
                cb.mode = kSfColsWeight; cb.E = a->E; cb.K = a->K;
                cb.atoms = reinterpret_cast<uint32_t*>(const_cast<uint8_t*>(p.sfb));
                sf_cols_kernel<<<cgrid, 256, 0, st>>>(cb);
            }
            MOE_LAUNCH_CHECK();
            if (pair) {
                size_t A = 0, B = 0;
                mx_atom_bytes(a, &A, &B);
                // A: [row tile][K stage][atom]; B: [expert x atom column][K
                // stage][atom], or [expert x K stage][atom column][atom] when
                // MN-major (the orders sf_rows_kernel / sf_cols_kernel write)
                const int64_t ks = cdiv(a->K, 128), nct = mx_b_atom_cols(a);
                MOE_TRY(make_atom_map(&p.sfa_map, p.sfa, ks, static_cast<int64_t>(A / kAtomBytes) / ks, ks,
                                      kSfGroup, 1));
                if (a->b_mn_major)
                    MOE_TRY(make_atom_map(&p.sfb_map, p.sfb, nct, static_cast<int64_t>(a->E) * ks, nct, 2,
                                          kSfGroup));
                else
                    MOE_TRY(make_atom_map(&p.sfb_map, p.sfb, ks, static_cast<int64_t>(a->E) * nct, ks,
                                          kSfGroup, 2));
                return quantise_after(launch_ragged_m<256, true, true>(a->b_mn_major, ge, ma, mb, p,
                                                                       grid < 2 ? 2 : grid, st, fuse_q));
            }
            return quantise_after(wide ? launch_ragged_m<256, true>(a->b_mn_major, ge, ma, mb, p, grid, st, fuse_q)
                                       : launch_ragged_m<128, true>(a->b_mn_major, ge, ma, mb, p, grid, st, fuse_q));
        }
        if (pair)
            return quantise_after(launch_ragged_m<256, false, true>(a->b_mn_major, ge, ma, mb, p,
                                                                    grid < 2 ? 2 : grid, st, fuse_q));
        return quantise_after(bn == 256 ? launch_ragged_m<256, false>(a->b_mn_major, ge, ma, mb, p, grid, st, fuse_q)
                                        : launch_ragged_m<128, false>(a->b_mn_major, ge, ma, mb, p, grid, st, fuse_q));
    }
    if (mode == MOE_GG_RAGGED_K) {
        if (epi != MOE_EPI_NONE || a->M < 1 || a->M % (mx ? 32 : 8)) return MOE_ERR_INVALID_ARG;
        const uint64_t M = a->M, N = a->N, E = a->E, Mt = a->M_total;
        if (Mt == 0) {
            if (cudaMemsetAsync(a->c, 0, E * M * N * 2, st) != cudaSuccess) return MOE_ERR_CUDA;
            return MOE_OK;
        }
        p.ldc = a->N;
        {
            uint64_t d[2] = {M, Mt}, s[1] = {M};
            uint32_t b[2] = {box_k, box_k};
            MOE_TRY(make_map(&ma, a->a, es, 2, d, s, b));
        }
        {
            uint64_t d[2] = {N, Mt}, s[1] = {N};
            uint32_t b[2] = {box_k, box_k};
            MOE_TRY(make_map(&mb, a->b, es, 2, d, s, b));
        }
        if (!mx && a->workspace && (reinterpret_cast<uintptr_t>(a->workspace) & 127) == 0 &&
            a->workspace_bytes >= kmap_bytes(a->E)) {
            CUtensorMap* maps = static_cast<CUtensorMap*>(a->workspace);
            kmap_kernel<<<static_cast<unsigned>(cdiv(a->E, 128)), 128, 0, st>>>(ma, mb, a->offsets, a->E,
                                                                                a->M_total, maps);
            MOE_LAUNCH_CHECK();
            p.kmaps = maps;
        }
        const bool big = mx ? mx_wide(a) : a->N >= 256;
        const int bn = big ? 256 : 128;
        // BF16 with 256-wide tiles: CTA pairs, 256 x 256 output tiles
        // 256-wide tiles: CTA pairs, 256 x 256 output tiles
        const bool pair = big && (!mx || !g_mx_no_pairs) && a->M >= 256 && !g_no_pairs;
        const int64_t bound = E * cdiv(a->M, pair ? 2 * BM : BM) * cdiv(a->N, bn) * (pair ? 2 : 1);
        const int grid = static_cast<int>(bound < sms ? bound : sms);
        if (mx) {
            const int cgrid = sms * 4;
            SfColsArgs ca{};
            ca.canon = a->a_scales; ca.cols = a->M; ca.nct = static_cast<int>(cdiv(a->M, 128));
            ca.mode = kSfColsGrouped; ca.E = a->E; ca.offsets = a->offsets;
            ca.rows = a->M_total; ca.status = a->status;
            ca.atoms = reinterpret_cast<uint32_t*>(const_cast<uint8_t*>(p.sfa));
            sf_cols_kernel<<<cgrid, 256, 0, st>>>(ca);
            MOE_LAUNCH_CHECK();
            SfColsArgs cb = ca;
            cb.canon = a->b_scales; cb.cols = a->N; cb.nct = static_cast<int>(mx_b_atom_cols(a));
            cb.atoms = reinterpret_cast<uint32_t*>(const_cast<uint8_t*>(p.sfb));
            sf_cols_kernel<<<cgrid, 256, 0, st>>>(cb);
            MOE_LAUNCH_CHECK();
            if (pair) {
                // the pair's scale-atom loader: A [K slot][row tile][atom], B [K
                // slot][atom column][atom], boxes of kSfGroup K slots
                size_t A = 0, B = 0;
                mx_atom_bytes(a, &A, &B);
                const int64_t mt = cdiv(a->M, 128), nct = mx_b_atom_cols(a);
                MOE_TRY(make_atom_map(&p.sfa_map, p.sfa, mt, static_cast<int64_t>(A / kAtomBytes) / mt, mt, 1,
                                      kSfGroup));
                MOE_TRY(make_atom_map(&p.sfb_map, p.sfb, nct, static_cast<int64_t>(B / kAtomBytes) / nct, nct, 2,
                                      kSfGroup));
                return launch<256, kRaggedK, true, true, kEpiNone, true, true>(ma, mb, p, grid < 2 ? 2 : grid, st);
            }
            return big ? launch<256, kRaggedK, true, true, kEpiNone, true>(ma, mb, p, grid, st)
                       : launch<128, kRaggedK, true, true, kEpiNone, true>(ma, mb, p, grid, st);
        }
        if (pair) return launch<256, kRaggedK, true, true, kEpiNone, false, true>(ma, mb, p, grid < 2 ? 2 : grid, st);
        return big ? launch<256, kRaggedK, true, true, kEpiNone, false>(ma, mb, p, grid, st)
                   : launch<128, kRaggedK, true, true, kEpiNone, false>(ma, mb, p, grid, st);
    }
    return MOE_ERR_INVALID_ARG;
}

}  // namespace moe
