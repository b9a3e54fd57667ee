// Device-scheduled grouped GEMM on the 5th-generation tensor cores (sm_100a).
//
// Combines the many small expert matmuls of the MoE layer into one persistent
// launch ("Ai2 rebuilds Olmo's training stack for trillion-parameter MoEs",
// "Routing work stays on the GPU", third bullet; "Supercharging Olmo-core for
// Efficient and Scalable MoE Training", Summary: device-scheduled grouped
// GEMMs).  The group sizes are read from device memory (`offsets`) by every
// CTA; the host never learns them.
//
// Kernel anatomy (one CTA per SM, 320 threads):
//   warp 0      TMA producer: fills a ring of shared-memory stages (A tile
//               128 x 64, B tile BN x 64, bf16, 128-byte swizzle), signalling
//               `full[s]` through the transaction count of an mbarrier.
//   warp 1      allocates TMEM; one thread issues tcgen05.mma (128 x BN x 16)
//               into a double-buffered fp32 accumulator in TMEM and releases
//               smem stages / publishes accumulators with tcgen05.commit.
//   warps 2..9  epilogue: tcgen05.ld of the accumulator (two warps per
//               32-lane TMEM quadrant, each taking half of the columns), fused
//               SwiGLU / SwiGLU-backward, bf16 stores.
// Tiles are handed out round-robin (tile = blockIdx.x + i * gridDim.x) from a
// per-expert tile prefix sum each CTA builds in shared memory from `offsets`.
//
// Modes
//   RAGGED_M : C[R_e, :] = A[R_e, :] . B_e^T   (forward GEMMs, dA, dX)
//   RAGGED_K : C_e = A[R_e, :]^T . B[R_e, :]   (dW GEMMs; K = rows of expert e;
//              rows of the last K tile that belong to the next expert are
//              zeroed in shared memory before the MMA reads them)
#include <cuda.h>

#include <mutex>

#include "common.cuh"
#include "ptx.cuh"

namespace moe {
namespace gg {

constexpr int BM = 128;
constexpr int BK = 64;  // 64 bf16 = one 128-byte swizzle atom along K
constexpr int MAX_E = 1024;
constexpr int kThreads = 320;  // 10 warps
constexpr int kEpiWarps = 8;
constexpr int BOX_BYTES = 64 * BK * 2;  // one [BK rows x 64 elements] MN-major box

enum { kRaggedM = 0, kRaggedK = 1 };
enum { kEpiNone = 0, kEpiSwiglu = 1, kEpiSwigluBwd = 2 };

struct Params {
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
    int32_t* status;
};

template <int BN>
struct Shape {
    static constexpr int A_BYTES = BM * BK * 2;
    static constexpr int B_BYTES = BN * BK * 2;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int STAGES = (BN == 256) ? 4 : 6;
    static constexpr int TMEM_COLS = 2 * BN;
    static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024;
};

struct Tile {
    int e;
    int m0;       // RAGGED_M: first routed row; RAGGED_K: first output row
    int row_end;  // RAGGED_M: end of expert rows
    int n0;       // first output column (SWIGLU: first f column)
    int k0;       // RAGGED_K: first routed row of the expert
    int kiters;
    int k_last;   // RAGGED_K: valid rows in the last K tile
};

struct Sched {
    int* off;   // [E+1]
    int* pref;  // [E+1] tile prefix
    int n_tiles;
    int m_tiles;  // RAGGED_K
};

template <int MODE>
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
        t.m0 = s.off[lo] + mt * BM;
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
        t.m0 = mt * BM;
        t.row_end = p.M;
        t.n0 = nt * bn_out;
        t.k0 = s.off[t.e];
        const int me = max(0, s.off[t.e + 1] - s.off[t.e]);
        t.kiters = (me + BK - 1) / BK;
        t.k_last = me - (t.kiters - 1) * BK;
    }
    return t;
}

template <int BN, int MODE, bool A_MN, bool B_MN, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    gg_bf16_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const Params p) {
    using S = Shape<BN>;
    constexpr int BN_OUT = (EPI == kEpiSwiglu) ? BN / 2 : BN;
    constexpr uint32_t IDESC = ptx::idesc_bf16(BM, BN, A_MN, B_MN);
    static_assert(!(EPI == kEpiSwiglu && B_MN), "SwiGLU GEMM takes K-major weights");
    static_assert(MODE == kRaggedM || (A_MN && B_MN && EPI == kEpiNone), "RAGGED_K layout");

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    __shared__ __align__(8) uint64_t full_bar[S::STAGES];
    __shared__ __align__(8) uint64_t empty_bar[S::STAGES];
    __shared__ __align__(8) uint64_t tfull_bar[2];
    __shared__ __align__(8) uint64_t tempty_bar[2];
    __shared__ uint32_t tmem_base_sh;
    __shared__ int s_off[MAX_E + 1];
    __shared__ int s_pref[MAX_E + 1];
    __shared__ volatile int s_abort;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    Sched sch;
    sch.off = s_off;
    sch.pref = s_pref;
    if (MODE == kRaggedM) {
        const int n_eff = (EPI == kEpiSwiglu) ? p.f : p.N;
        sch.n_tiles = (n_eff + BN_OUT - 1) / BN_OUT;
        sch.m_tiles = 0;
    } else {
        sch.n_tiles = (p.N + BN - 1) / BN;
        sch.m_tiles = (p.M + BM - 1) / BM;
    }

    if (threadIdx.x == 0) {
        for (int s = 0; s < S::STAGES; ++s) {
            ptx::mbar_init(&full_bar[s], 1);
            ptx::mbar_init(&empty_bar[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            ptx::mbar_init(&tfull_bar[a], 1);
            ptx::mbar_init(&tempty_bar[a], kEpiWarps);
        }
        s_abort = 0;
        ptx::fence_mbar_init();
        ptx::prefetch_tmap(&tmA);
        ptx::prefetch_tmap(&tmB);
    }
    if (warp == 1) {
        ptx::tmem_alloc(&tmem_base_sh, S::TMEM_COLS);
        ptx::tmem_relinquish();
    }
    if (warp == 2) {
        // Group table and per-expert tile prefix sum (warp-wide scan).
        const int E = p.E;
        bool bad = false;
        for (int i = lane; i <= E; i += 32) {
            int v = p.offsets[i];
            if (v < 0 || v > p.M_total) { bad = true; v = v < 0 ? 0 : p.M_total; }
            s_off[i] = v;
        }
        __syncwarp();
        const int per = (E + 31) / 32;
        const int beg = min(E, lane * per), end = min(E, beg + per);
        int local = 0;
        for (int e = beg; e < end; ++e) {
            int me = s_off[e + 1] - s_off[e];
            if (me < 0) { bad = true; me = 0; }
            local += (MODE == kRaggedM) ? ((me + BM - 1) / BM) * sch.n_tiles
                                        : sch.m_tiles * sch.n_tiles;
        }
        int incl = local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        int run = incl - local;
        for (int e = beg; e < end; ++e) {
            s_pref[e] = run;
            const int me = max(0, s_off[e + 1] - s_off[e]);
            run += (MODE == kRaggedM) ? ((me + BM - 1) / BM) * sch.n_tiles
                                      : sch.m_tiles * sch.n_tiles;
        }
        if (lane == 31) s_pref[E] = incl;
        if (__any_sync(0xffffffffu, bad) && lane == 0) flag_status(p.status, MOE_ERR_DEVICE_BOUNDS);
    }
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_base = tmem_base_sh;
    const int total = s_pref[p.E];

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
                const Tile t = decode<MODE>(sch, p, tile, BN_OUT);
                for (int kt = 0; kt < t.kiters; ++kt) {
                    if (!ptx::mbar_wait(&empty_bar[stage], phase ^ 1u, &s_abort)) { ok = false; break; }
                    uint8_t* sa = smem + stage * S::STAGE_BYTES;
                    uint8_t* sb = sa + S::A_BYTES;
                    uint64_t* fb = &full_bar[stage];
                    ptx::mbar_arrive_expect_tx(fb, S::STAGE_BYTES);
                    if (MODE == kRaggedM) {
                        ptx::tma_load_2d(sa, &tmA, fb, kt * BK, t.m0);
                        if (!B_MN) {
                            if (EPI == kEpiSwiglu) {
                                ptx::tma_load_3d(sb, &tmB, fb, kt * BK, t.n0, t.e);
                                ptx::tma_load_3d(sb + S::B_BYTES / 2, &tmB, fb, kt * BK, p.f + t.n0, t.e);
                            } else {
                                ptx::tma_load_3d(sb, &tmB, fb, kt * BK, t.n0, t.e);
                            }
                        } else {
#pragma unroll
                            for (int j = 0; j < BN / 64; ++j)
                                ptx::tma_load_3d(sb + j * BOX_BYTES, &tmB, fb, t.n0 + 64 * j, kt * BK, t.e);
                        }
                    } else {
                        const int krow = t.k0 + kt * BK;
#pragma unroll
                        for (int j = 0; j < BM / 64; ++j)
                            ptx::tma_load_2d(sa + j * BOX_BYTES, &tmA, fb, t.m0 + 64 * j, krow);
#pragma unroll
                        for (int j = 0; j < BN / 64; ++j)
                            ptx::tma_load_2d(sb + j * BOX_BYTES, &tmB, fb, t.n0 + 64 * j, krow);
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
        // ------------------------------------------------ MMA issuer
        int stage = 0;
        uint32_t phase = 0;
        int acc = 0;
        uint32_t acc_phase = 0;
        bool ok = true;
        for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
            const Tile t = decode<MODE>(sch, p, tile, BN_OUT);
            if (!ptx::mbar_wait(&tempty_bar[acc], acc_phase ^ 1u, &s_abort)) { ok = false; break; }
            ptx::tc_fence_after();
            const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
            for (int kt = 0; kt < t.kiters; ++kt) {
                if (!ptx::mbar_wait(&full_bar[stage], phase, &s_abort)) { ok = false; break; }
                ptx::tc_fence_after();
                uint8_t* sa = smem + stage * S::STAGE_BYTES;
                uint8_t* sb = sa + S::A_BYTES;
                if (MODE == kRaggedK && kt == t.kiters - 1 && t.k_last < BK) {
                    // Rows k_last..BK-1 of this K tile belong to the next expert
                    // (or lie past the buffer): zero them in every box of A and B.
                    const int nbytes = (BK - t.k_last) * 128;
                    for (int j = 0; j < BM / 64 + BN / 64; ++j) {
                        uint8_t* box = (j < BM / 64) ? sa + j * BOX_BYTES : sb + (j - BM / 64) * BOX_BYTES;
                        uint4* z = reinterpret_cast<uint4*>(box + t.k_last * 128);
                        for (int i = lane; i < nbytes / 16; i += 32) z[i] = make_uint4(0, 0, 0, 0);
                    }
                    ptx::fence_proxy_async_smem();
                }
                __syncwarp();
                if (lane == 0) {
                    const uint32_t a_addr = ptx::smem_addr(sa);
                    const uint32_t b_addr = ptx::smem_addr(sb);
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        const uint64_t ad = A_MN ? ptx::sdesc_sw128(a_addr + kk * 2048, BOX_BYTES, 1024)
                                                 : ptx::sdesc_sw128(a_addr + kk * 32, 16, 1024);
                        const uint64_t bd = B_MN ? ptx::sdesc_sw128(b_addr + kk * 2048, BOX_BYTES, 1024)
                                                 : ptx::sdesc_sw128(b_addr + kk * 32, 16, 1024);
                        ptx::mma_f16(d_tmem, ad, bd, IDESC, (kt | kk) != 0 ? 1u : 0u);
                    }
                    ptx::mma_commit(&empty_bar[stage]);
                }
                __syncwarp();
                if (++stage == S::STAGES) { stage = 0; phase ^= 1u; }
            }
            if (!ok) break;
            if (lane == 0) {
                if (t.kiters > 0) ptx::mma_commit(&tfull_bar[acc]);
                else ptx::mbar_arrive(&tfull_bar[acc]);
            }
            __syncwarp();
            if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
        }
        if (!ok && lane == 0) {
            s_abort = 1;
            flag_status(p.status, MOE_ERR_DEVICE_TIMEOUT);
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
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
            const Tile t = decode<MODE>(sch, p, tile, BN_OUT);
            const int row = t.m0 + r;
            const bool row_ok = row < t.row_end;
            if (EPI == kEpiSwigluBwd) {
                // G and U do not depend on the accumulator: fetch them while
                // the MMAs of this tile are still running.
                constexpr int NCH = BN / 2 / 32;
                const int cbase = half * (BN / 2);
                const uint16_t* gurow = p.gu + static_cast<int64_t>(row) * 2 * p.f;
                uint16_t* dhrow = p.c + static_cast<int64_t>(row) * p.ldc;
                uint4 gb[4], ub[4];
                auto fetch = [&](int col, uint4 (&g)[4], uint4 (&u)[4]) {
                    if (row_ok && col + 32 <= p.f) {
                        const uint4* sg = reinterpret_cast<const uint4*>(gurow + col);
                        const uint4* su = reinterpret_cast<const uint4*>(gurow + p.f + col);
#pragma unroll
                        for (int j = 0; j < 4; ++j) { g[j] = __ldg(sg + j); u[j] = __ldg(su + j); }
                    }
                };
                fetch(t.n0 + cbase, gb, ub);
                if (!ptx::mbar_wait(&tfull_bar[acc], acc_phase, &s_abort)) { ok = false; break; }
                ptx::tc_fence_after();
                const uint32_t tb = tmem_base + static_cast<uint32_t>(acc * BN) + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll 1
                for (int ci = 0; ci < NCH; ++ci) {
                    const int c0 = cbase + ci * 32;
                    const int col = t.n0 + c0;
                    uint32_t v[32];
                    ptx::tmem_ld_32x32b_x32(tb + c0, v);
                    uint4 gn[4], un[4];
                    if (ci + 1 < NCH) fetch(col + 32, gn, un);
                    ptx::tmem_wait_ld();
                    if (row_ok && col < p.f) {
                        if (col + 32 <= p.f) {
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
                        } else {
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
                    if (ci + 1 < NCH) {
#pragma unroll
                        for (int j = 0; j < 4; ++j) { gb[j] = gn[j]; ub[j] = un[j]; }
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
            if (lane == 0) ptx::mbar_arrive(&tempty_bar[acc]);
            if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
        }
        if (!ok && lane == 0) {
            s_abort = 1;
            flag_status(p.status, MOE_ERR_DEVICE_TIMEOUT);
        }
    }

    __syncthreads();
    if (warp == 1) {
        if (s_abort) {
            // Let in-flight tensor-core and TMA work drain before TMEM is freed.
            const uint64_t t0 = ptx::globaltimer();
            while (ptx::globaltimer() - t0 < 20000000ull) { }
        }
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem_base, S::TMEM_COLS);
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

// bf16 tensor map, 128-byte swizzle, zero fill outside the tensor.
static int make_map(CUtensorMap* m, const void* base, int rank, const uint64_t* dims,
                    const uint64_t* strides_bytes, const uint32_t* box) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return MOE_ERR_CUDA;
    cuuint64_t gd[3], gs[2];
    cuuint32_t bx[3], es[3] = {1, 1, 1};
    for (int i = 0; i < rank; ++i) { gd[i] = dims[i]; bx[i] = box[i]; }
    for (int i = 0; i < rank - 1; ++i) gs[i] = strides_bytes[i];
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), gd, gs, bx,
                    es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MOE_OK : MOE_ERR_CUDA;
}

template <int BN, int MODE, bool A_MN, bool B_MN, int EPI>
static int launch(const CUtensorMap& ma, const CUtensorMap& mb, const Params& p, int grid,
                  cudaStream_t st) {
    using S = Shape<BN>;
    auto kern = gg_bf16_kernel<BN, MODE, A_MN, B_MN, EPI>;
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [&] {
        attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::SMEM_BYTES);
    });
    if (attr_err != cudaSuccess) return MOE_ERR_CUDA;
    kern<<<grid, kThreads, S::SMEM_BYTES, st>>>(ma, mb, p);
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}

}  // namespace gg

int grouped_gemm_bf16(const moe_gg_args* a, cudaStream_t st) {
    using namespace gg;
    const int mode = a->mode, epi = a->epilogue;
    if (a->E < 1 || a->E > MAX_E || a->N < 1 || a->M_total < 0 || a->M_total >= (1ll << 31))
        return MOE_ERR_INVALID_ARG;
    if (!a->offsets || !a->a || !a->b || !a->c) return MOE_ERR_INVALID_ARG;
    if (!aligned16(a->a) || !aligned16(a->b) || !aligned16(a->c)) return MOE_ERR_INVALID_ARG;
    if (a->N % 8) return MOE_ERR_INVALID_ARG;

    Params p{};
    p.offsets = a->offsets;
    p.E = a->E;
    p.M_total = static_cast<int>(a->M_total);
    p.M = a->M;
    p.N = a->N;
    p.K = a->K;
    p.c = static_cast<uint16_t*>(a->c);
    p.status = a->status;
    const int sms = num_sms();
    CUtensorMap ma, mb;

    if (mode == MOE_GG_RAGGED_M) {
        if (a->K < 1 || a->K % 8) return MOE_ERR_INVALID_ARG;
        if (a->M_total == 0) return MOE_OK;
        const uint64_t K = a->K, N = a->N, E = a->E, Mt = a->M_total;
        {
            uint64_t d[2] = {K, Mt}, s[1] = {K * 2};
            uint32_t b[2] = {64, 128};
            MOE_TRY(make_map(&ma, a->a, 2, d, s, b));
        }
        if (epi == MOE_EPI_SWIGLU) {
            if (a->b_mn_major || !a->aux || !aligned16(a->aux) || a->N % 16) return MOE_ERR_INVALID_ARG;
            p.f = a->N / 2;
            p.ldc = a->N;
            p.aux = static_cast<uint16_t*>(a->aux);
            uint64_t d[3] = {K, N, E}, s[2] = {K * 2, N * K * 2};
            uint32_t b[3] = {64, 128, 1};
            MOE_TRY(make_map(&mb, a->b, 3, d, s, b));
            const int64_t bound = (Mt / BM + E) * cdiv(p.f, 128);
            const int grid = static_cast<int>(bound < sms ? bound : sms);
            return launch<256, kRaggedM, false, false, kEpiSwiglu>(ma, mb, p, grid, st);
        }
        const bool bwd = (epi == MOE_EPI_SWIGLU_BWD);
        if (bwd) {
            if (!a->gu || !aligned16(a->gu)) return MOE_ERR_INVALID_ARG;
            p.f = a->N;
            p.ldc = 2 * static_cast<int64_t>(a->N);
            p.gu = static_cast<const uint16_t*>(a->gu);
        } else if (epi == MOE_EPI_NONE) {
            p.ldc = a->N;
        } else {
            return MOE_ERR_INVALID_ARG;
        }
        const bool big = a->N >= 256;
        const int bn = big ? 256 : 128;
        if (!a->b_mn_major) {
            uint64_t d[3] = {K, N, E}, s[2] = {K * 2, N * K * 2};
            uint32_t b[3] = {64, static_cast<uint32_t>(bn), 1};
            MOE_TRY(make_map(&mb, a->b, 3, d, s, b));
        } else {
            uint64_t d[3] = {N, K, E}, s[2] = {N * 2, K * N * 2};
            uint32_t b[3] = {64, 64, 1};
            MOE_TRY(make_map(&mb, a->b, 3, d, s, b));
        }
        const int64_t bound = (Mt / BM + E) * cdiv(a->N, bn);
        const int grid = static_cast<int>(bound < sms ? bound : sms);
        if (!a->b_mn_major) {
            if (bwd) return big ? launch<256, kRaggedM, false, false, kEpiSwigluBwd>(ma, mb, p, grid, st)
                                : launch<128, kRaggedM, false, false, kEpiSwigluBwd>(ma, mb, p, grid, st);
            return big ? launch<256, kRaggedM, false, false, kEpiNone>(ma, mb, p, grid, st)
                       : launch<128, kRaggedM, false, false, kEpiNone>(ma, mb, p, grid, st);
        }
        if (bwd) return big ? launch<256, kRaggedM, false, true, kEpiSwigluBwd>(ma, mb, p, grid, st)
                            : launch<128, kRaggedM, false, true, kEpiSwigluBwd>(ma, mb, p, grid, st);
        return big ? launch<256, kRaggedM, false, true, kEpiNone>(ma, mb, p, grid, st)
                   : launch<128, kRaggedM, false, true, kEpiNone>(ma, mb, p, grid, st);
    }
    if (mode == MOE_GG_RAGGED_K) {
        if (epi != MOE_EPI_NONE || a->M < 1 || a->M % 8) return MOE_ERR_INVALID_ARG;
        const uint64_t M = a->M, N = a->N, E = a->E, Mt = a->M_total;
        if (Mt == 0) {
            if (cudaMemsetAsync(a->c, 0, E * M * N * 2, st) != cudaSuccess) return MOE_ERR_CUDA;
            return MOE_OK;
        }
        p.ldc = a->N;
        {
            uint64_t d[2] = {M, Mt}, s[1] = {M * 2};
            uint32_t b[2] = {64, 64};
            MOE_TRY(make_map(&ma, a->a, 2, d, s, b));
        }
        const bool big = a->N >= 256;
        {
            uint64_t d[2] = {N, Mt}, s[1] = {N * 2};
            uint32_t b[2] = {64, 64};
            MOE_TRY(make_map(&mb, a->b, 2, d, s, b));
        }
        const int bn = big ? 256 : 128;
        const int64_t bound = E * cdiv(a->M, BM) * cdiv(a->N, bn);
        const int grid = static_cast<int>(bound < sms ? bound : sms);
        return big ? launch<256, kRaggedK, true, true, kEpiNone>(ma, mb, p, grid, st)
                   : launch<128, kRaggedK, true, true, kEpiNone>(ma, mb, p, grid, st);
    }
    return MOE_ERR_INVALID_ARG;
}

}  // namespace moe
