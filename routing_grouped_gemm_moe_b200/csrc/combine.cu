// Weighted unpermute / combine (the k expert outputs of a token summed with
// its routing weights), its backward, the unpermute-sum of the input
// gradient, and the standalone SwiGLU forward / backward.
//
// All kernels are HBM-bound: one warp per token, 16-byte vectors, fp32 sums in
// slot order 0..k-1 (deterministic), one bf16 rounding per output.
#include "common.cuh"
#include "ptx.cuh"

namespace moe {

static int warp_grid(int64_t warps) {
    int64_t blocks = (warps + 7) / 8;
    const int64_t cap = static_cast<int64_t>(num_sms()) * 8;
    if (blocks > cap) blocks = cap;
    return static_cast<int>(blocks < 1 ? 1 : blocks);
}

// out[t] = sum_i w[t, i] y_perm[dest[t, i]]
__global__ void __launch_bounds__(256) combine_kernel(const uint16_t* __restrict__ y,
                                                      const int32_t* __restrict__ dest,
                                                      const float* __restrict__ w, int T, int d,
                                                      int k, int64_t M, uint16_t* __restrict__ out) {
    const int lane = threadIdx.x & 31;
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    const int nvec = d / 8;
    for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += nwarps) {
        int my_p = -1;
        float my_w = 0.f;
        if (lane < k) {
            my_p = dest[static_cast<int64_t>(t) * k + lane];
            my_w = w[static_cast<int64_t>(t) * k + lane];
            if (my_p < 0 || my_p >= M) { my_p = -1; }
        }
        uint4* o = reinterpret_cast<uint4*>(out + static_cast<int64_t>(t) * d);
        // every lane runs the same trip count: the shuffles below need the full warp
        for (int v0 = 0; v0 < nvec; v0 += 32) {
            const int v = v0 + lane;
            const bool act = v < nvec;
            float acc[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[j] = 0.f;
            for (int i = 0; i < k; ++i) {
                const int p = __shfl_sync(0xffffffffu, my_p, i);
                const float wi = __shfl_sync(0xffffffffu, my_w, i);
                if (p < 0 || !act) continue;
                float f[8];
                unpack8(__ldg(reinterpret_cast<const uint4*>(y + static_cast<int64_t>(p) * d) + v), f);
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[j] = fmaf(wi, f[j], acc[j]);
            }
            if (act) o[v] = pack8(acc);
        }
    }
}

// dy_perm[dest[t, i]] = bf16(w_i dout[t]);  dw[t, i] = sum_c dout[t, c] y_perm[dest[t, i], c]
template <int KMAX>
__global__ void __launch_bounds__(256) combine_bwd_kernel(
    const uint16_t* __restrict__ dout, const uint16_t* __restrict__ y,
    const int32_t* __restrict__ dest, const float* __restrict__ w, int T, int d, int k, int64_t M,
    uint16_t* __restrict__ dy, float* __restrict__ dw) {
    const int lane = threadIdx.x & 31;
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    const int nvec = d / 8;
    for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += nwarps) {
        int my_p = -1;
        float my_w = 0.f;
        if (lane < k) {
            my_p = dest[static_cast<int64_t>(t) * k + lane];
            my_w = w[static_cast<int64_t>(t) * k + lane];
            if (my_p < 0 || my_p >= M) my_p = -1;
        }
        float part[KMAX];
#pragma unroll
        for (int i = 0; i < KMAX; ++i) part[i] = 0.f;
        const uint4* g = reinterpret_cast<const uint4*>(dout + static_cast<int64_t>(t) * d);
        for (int v0 = 0; v0 < nvec; v0 += 32) {
            const int v = v0 + lane;
            const bool act = v < nvec;
            float gf[8];
            if (act) {
                unpack8(__ldg(g + v), gf);
            } else {
#pragma unroll
                for (int j = 0; j < 8; ++j) gf[j] = 0.f;
            }
#pragma unroll
            for (int i = 0; i < KMAX; ++i) {
                if (i >= k) break;
                const int p = __shfl_sync(0xffffffffu, my_p, i);
                const float wi = __shfl_sync(0xffffffffu, my_w, i);
                if (p < 0 || !act) continue;
                float yf[8], o[8];
                unpack8(__ldg(reinterpret_cast<const uint4*>(y + static_cast<int64_t>(p) * d) + v), yf);
                float s = 0.f;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    s = fmaf(gf[j], yf[j], s);
                    o[j] = wi * gf[j];
                }
                part[i] += s;
                reinterpret_cast<uint4*>(dy + static_cast<int64_t>(p) * d)[v] = pack8(o);
            }
        }
#pragma unroll
        for (int i = 0; i < KMAX; ++i) {
            if (i >= k) break;
            const float s = warp_sum(part[i]);
            if (lane == 0) dw[static_cast<int64_t>(t) * k + i] = s;
        }
    }
}

// unpermute_sum: rows of up to kBatch slots are loaded before any is used, so
// that a warp keeps kBatch 512-byte loads in flight per chunk (measured: 414
// -> 365 us per launch at the large workload; the same batching made
// combine and combine_bwd slower, 409 -> 489 and 848 -> 874 us, so they keep
// one slot per step).
constexpr int kBatch = 8;

// dx[t] = sum_i dx_perm[dest[t, i]]: one warp per token, 16-byte vectors
__global__ void __launch_bounds__(256) unpermute_sum_kernel(
    const uint16_t* __restrict__ dxp, const int32_t* __restrict__ dest, int T, int d, int k,
    int64_t M, uint16_t* __restrict__ dx) {
    const int lane = threadIdx.x & 31;
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    const int nvec = d / 8;
    for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += nwarps) {
        int my_p = -1;
        if (lane < k) {
            my_p = dest[static_cast<int64_t>(t) * k + lane];
            if (my_p < 0 || my_p >= M) my_p = -1;
        }
        uint4* o = reinterpret_cast<uint4*>(dx + static_cast<int64_t>(t) * d);
        for (int v0 = 0; v0 < nvec; v0 += 32) {
            const int v = v0 + lane;
            const bool act = v < nvec;
            float acc[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[j] = 0.f;
            for (int i0 = 0; i0 < k; i0 += kBatch) {
                uint4 xv[kBatch];
                bool use[kBatch];
#pragma unroll
                for (int u = 0; u < kBatch; ++u) {
                    const int p = __shfl_sync(0xffffffffu, my_p, (i0 + u) & 31);
                    use[u] = i0 + u < k && p >= 0 && act;
                    xv[u] = use[u] ? __ldg(reinterpret_cast<const uint4*>(dxp + static_cast<int64_t>(p) * d) + v)
                                   : make_uint4(0, 0, 0, 0);
                }
#pragma unroll
                for (int u = 0; u < kBatch; ++u) {  // slot order; skipped slots add nothing
                    if (!use[u]) continue;
                    float f[8];
                    unpack8(xv[u], f);
#pragma unroll
                    for (int j = 0; j < 8; ++j) acc[j] += f[j];
                }
            }
            if (act) o[v] = pack8(acc);
        }
    }
}

// unpermute_sum with the router-projection term, as tiles of 64 tokens x 32
// columns: sum_e d_logits[t, e] W_r[c, e] over experts in chunks of 32 staged
// in shared memory as fp32 (ascending e), then the k routed rows of dX_perm in
// slot order, one bf16 rounding.  Thread = 2 tokens x 8 consecutive columns.
__global__ void __launch_bounds__(128) unpermute_sum_router_kernel(
    const uint16_t* __restrict__ dxp, const int32_t* __restrict__ dest, int T, int d, int k,
    int64_t M, const float* __restrict__ dl, const uint16_t* __restrict__ wr, int E,
    uint16_t* __restrict__ dx) {
    __shared__ __align__(16) float gs[32][64 + 2];  // d_logits tile, [expert][token]
    __shared__ __align__(16) float ws[32][32];      // W_r tile, [expert][column]
    const int tid = threadIdx.x, tg = tid & 31, cg = tid >> 5;
    const int t0 = blockIdx.x * 64, c0 = blockIdx.y * 32;
    float acc[2][8];
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[a][j] = 0.f;
    for (int e0 = 0; e0 < E; e0 += 32) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int i = tid + 128 * j;
            const int r = i >> 3, v = i & 7, e = e0 + 4 * v;
            const int t = t0 + r;
            float g[4] = {0.f, 0.f, 0.f, 0.f};
            if (t < T) {
                const float* src = dl + static_cast<int64_t>(t) * E + e;
#pragma unroll
                for (int m = 0; m < 4; ++m) g[m] = e + m < E ? __ldg(src + m) : 0.f;
            }
#pragma unroll
            for (int m = 0; m < 4; ++m) gs[4 * v + m][r] = g[m];
        }
        {
            const int cc = tid >> 2, v = tid & 3, c = c0 + cc;
            float f[8];
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                const int e = e0 + 8 * v + m;
                f[m] = (c < d && e < E) ? bf16_to_f32(__ldg(wr + static_cast<int64_t>(c) * E + e)) : 0.f;
            }
#pragma unroll
            for (int m = 0; m < 8; ++m) ws[8 * v + m][cc] = f[m];
        }
        __syncthreads();
#pragma unroll 4
        for (int e = 0; e < 32; ++e) {
            const float2 g = *reinterpret_cast<const float2*>(&gs[e][2 * tg]);
            const float4 w0 = *reinterpret_cast<const float4*>(&ws[e][8 * cg]);
            const float4 w1 = *reinterpret_cast<const float4*>(&ws[e][8 * cg + 4]);
            const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                acc[0][j] = fmaf(g.x, wv[j], acc[0][j]);
                acc[1][j] = fmaf(g.y, wv[j], acc[1][j]);
            }
        }
        __syncthreads();
    }
    const int c = c0 + 8 * cg;
    if (c >= d) return;
#pragma unroll
    for (int a = 0; a < 2; ++a) {
        const int t = t0 + 2 * tg + a;
        if (t >= T) continue;
        for (int i = 0; i < k; ++i) {
            const int p = __ldg(dest + static_cast<int64_t>(t) * k + i);
            if (p < 0 || p >= M) continue;
            float f[8];
            unpack8(__ldg(reinterpret_cast<const uint4*>(dxp + static_cast<int64_t>(p) * d + c)), f);
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[a][j] += f[j];
        }
        *reinterpret_cast<uint4*>(dx + static_cast<int64_t>(t) * d + c) = pack8(acc[a]);
    }
}

// Bulk-load engine of the token-side kernels.  A CTA has kCombWarps consumer
// warps and one producer warp, and NS shared-memory stages, each holding the
// rows one token needs: its k routed rows (combine, unpermute-sum) or dOut[t]
// followed by its k rows of Y_perm (combine backward).  The producer reads a
// token's row positions and weights, then its lanes load the rows with one
// bulk copy each (cp.async.bulk, completion on the stage's mbarrier), NS tokens
// ahead of the consumers; the consumers compute from shared memory, store
// with 16-byte vectors and release the stage.  Few instructions move the
// rows, so the kernels keep their rate when the SM clock drops.  A stage
// holds a whole token (64 KB at k = 8, d = 4096), so one CTA fills an SM:
// 16 consumer warps (one 16-byte vector each per row at d = 4096) rather
// than 8 took the combine 533 -> 402 us and the unpermute-sum 535 -> 385 us
// inside the large layer's step (isolated 396 -> 366 us each).
constexpr int kCombWarps = 16;
constexpr int kCombThreads = 32 * (kCombWarps + 1);
constexpr int kCombMaxStages = 8;
constexpr size_t kCombSmem = 200 * 1024;

// BWD = false: out[t] = sum_i w_i rows[dest[t, i]] (w == nullptr: unit weights,
// the unpermute-sum).  BWD = true: dy[dest[t, i]] = bf16(w_i dout[t]) and
// dw[t, i] = sum_c dout[t, c] rows[dest[t, i], c].
template <bool BWD>
__global__ void __launch_bounds__(kCombThreads) combine_bulk_kernel(
    const uint16_t* __restrict__ rows, const uint16_t* __restrict__ dout,
    const int32_t* __restrict__ dest, const float* __restrict__ w, int T, int d, int k, int64_t M,
    int NS, uint16_t* __restrict__ out, float* __restrict__ dw, int32_t* status) {
    extern __shared__ __align__(128) uint8_t stage_mem[];
    __shared__ __align__(8) uint64_t full[kCombMaxStages];
    __shared__ __align__(8) uint64_t empty[kCombMaxStages];
    __shared__ int sp[kCombMaxStages][32];
    __shared__ float sw[kCombMaxStages][32];
    // backward: per-warp partial dot products of each stage's token, and a
    // barrier on which the warps post them for warp 0 to add
    __shared__ float red[BWD ? kCombMaxStages : 1][kCombWarps][32];
    __shared__ __align__(8) uint64_t red_bar[kCombMaxStages];
    __shared__ volatile int abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int lead = BWD ? 1 : 0;  // rows before the routed ones in a stage
    const uint32_t row_bytes = static_cast<uint32_t>(d) * 2u;
    const size_t stage_bytes = static_cast<size_t>(k + lead) * row_bytes;
    if (threadIdx.x == 0) {
        for (int q = 0; q < NS; ++q) {
            ptx::mbar_init(&full[q], 1);
            ptx::mbar_init(&empty[q], kCombWarps);
            ptx::mbar_init(&red_bar[q], kCombWarps);
        }
        abort_flag = 0;
        ptx::fence_mbar_init();
    }
    __syncthreads();
    const int n = blockIdx.x < T ? (T - 1 - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x) + 1 : 0;
    bool ok = true;
    if (warp == kCombWarps) {
        // ------------------------------------------------ producer
        // a token's row positions and weights are read one token ahead, so
        // that their load latency overlaps the wait for a free stage
        auto meta = [&](int i, int& p, float& wi) {
            p = -1;
            wi = 0.f;
            if (i < n && lane < k) {
                const int64_t t = blockIdx.x + static_cast<int64_t>(i) * gridDim.x;
                p = __ldg(dest + t * k + lane);
                wi = w ? __ldg(w + t * k + lane) : 1.0f;
            }
        };
        int p_next;
        float w_next;
        meta(0, p_next, w_next);
        for (int i = 0; i < n && ok; ++i) {
            const int q = i % NS;
            int p = p_next;
            const float wi = w_next;
            meta(i + 1, p_next, w_next);
            if (i >= NS && !ptx::mbar_wait(&empty[q], static_cast<uint32_t>((i / NS - 1) & 1), &abort_flag)) {
                ok = false;
                break;
            }
            const int64_t t = blockIdx.x + static_cast<int64_t>(i) * gridDim.x;
            if (p < 0 || p >= M) p = -1;
            if (lane < k) {
                sp[q][lane] = p;
                sw[q][lane] = wi;
            }
            const uint32_t nvalid = __popc(__ballot_sync(0xffffffffu, p >= 0));
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive_expect_tx(&full[q], (nvalid + lead) * row_bytes);
            __syncwarp();
            uint8_t* st = stage_mem + q * stage_bytes;
            if (p >= 0) ptx::bulk_load(st + (lead + lane) * row_bytes, rows + p * static_cast<int64_t>(d), row_bytes, &full[q]);
            if (BWD && lane == 0) ptx::bulk_load(st, dout + t * d, row_bytes, &full[q]);
        }
    } else {
        // ------------------------------------------------ consumers
        const int nvec = d / 8;
        const int tid = threadIdx.x;
        for (int i = 0; i < n; ++i) {
            const int q = i % NS;
            if (!ptx::mbar_wait(&full[q], static_cast<uint32_t>((i / NS) & 1), &abort_flag)) {
                ok = false;
                break;
            }
            const int64_t t = blockIdx.x + static_cast<int64_t>(i) * gridDim.x;
            const uint8_t* st = stage_mem + q * stage_bytes;
            if (!BWD) {
                for (int v = tid; v < nvec; v += 32 * kCombWarps) {
                    float acc[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) acc[j] = 0.f;
                    for (int r = 0; r < k; ++r) {  // slot order
                        if (sp[q][r] < 0) continue;
                        const float wr = sw[q][r];
                        float f[8];
                        unpack8(*reinterpret_cast<const uint4*>(st + r * row_bytes + 16 * v), f);
#pragma unroll
                        for (int j = 0; j < 8; ++j) acc[j] = fmaf(wr, f[j], acc[j]);
                    }
                    reinterpret_cast<uint4*>(out + t * d)[v] = pack8(acc);
                }
            } else {
                for (int r = 0; r < k; ++r) {
                    const int p = sp[q][r];
                    const float wr = sw[q][r];
                    float s = 0.f;
                    if (p >= 0) {
                        for (int v = tid; v < nvec; v += 32 * kCombWarps) {
                            float g[8], y[8], o[8];
                            unpack8(*reinterpret_cast<const uint4*>(st + 16 * v), g);
                            unpack8(*reinterpret_cast<const uint4*>(st + (1 + r) * row_bytes + 16 * v), y);
#pragma unroll
                            for (int j = 0; j < 8; ++j) {
                                s = fmaf(g[j], y[j], s);
                                o[j] = wr * g[j];
                            }
                            reinterpret_cast<uint4*>(out + static_cast<int64_t>(p) * d)[v] = pack8(o);
                        }
                    }
                    s = warp_sum(s);
                    if (lane == 0) red[BWD ? q : 0][warp][r] = s;
                }
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&red_bar[q]);
                // warp 0 adds the warps' partials in warp order (deterministic)
                // before it releases the stage: red[q] is rewritten only for
                // the token that refills stage q
                if (warp == 0) {
                    if (!ptx::mbar_wait(&red_bar[q], static_cast<uint32_t>((i / NS) & 1), &abort_flag)) {
                        ok = false;
                        break;
                    }
                    if (lane < k) {
                        float s = 0.f;
#pragma unroll
                        for (int q2 = 0; q2 < kCombWarps; ++q2) s += red[BWD ? q : 0][q2][lane];
                        dw[t * k + lane] = s;
                    }
                }
            }
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&empty[q]);
        }
    }
    if (!ok) {
        abort_flag = 1;
        if (lane == 0) flag_status(status, MOE_ERR_DEVICE_TIMEOUT);
    }
}

// Stages for a token of `rows_per_token` rows of d bf16, or 0 when the rows
// do not fit the bulk engine (the warp-per-token kernels take those).
static int comb_stages(int rows_per_token, int d) {
    const size_t stage = static_cast<size_t>(rows_per_token) * d * 2;
    size_t ns = kCombSmem / stage;
    if (ns > kCombMaxStages) ns = kCombMaxStages;
    return ns < 2 ? 0 : static_cast<int>(ns);
}

template <bool BWD>
static int launch_comb(int NS, int rows_per_token, const uint16_t* rows, const uint16_t* dout,
                       const int32_t* dest, const float* w, int T, int d, int k, uint16_t* out,
                       float* dw, cudaStream_t st) {
    static int configured_dev = -1;  // opt-in above 48 KB, once per device
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_dev != dev) {
        if (cudaFuncSetAttribute(combine_bulk_kernel<BWD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(kCombSmem)) != cudaSuccess)
            return MOE_ERR_CUDA;
        configured_dev = dev;
    }
    const size_t smem = static_cast<size_t>(NS) * rows_per_token * d * 2;
    // two CTAs per SM when two fit
    const int per_sm = 2 * (smem + 8192) <= 227 * 1024 ? 2 : 1;
    int64_t grid = static_cast<int64_t>(num_sms()) * per_sm;
    if (grid > T) grid = T;
    combine_bulk_kernel<BWD><<<static_cast<int>(grid), kCombThreads, smem, st>>>(
        rows, dout, dest, w, T, d, k, static_cast<int64_t>(T) * k, NS, out, dw, nullptr);
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}

__global__ void swiglu_kernel(const uint16_t* __restrict__ gu, uint16_t* __restrict__ a, int64_t M,
                              int f) {
    const int64_t nv = M * (f / 8);
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < nv;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t r = i / (f / 8);
        const int c = static_cast<int>(i - r * (f / 8)) * 8;
        float g[8], u[8], o[8];
        unpack8(*reinterpret_cast<const uint4*>(gu + r * 2 * f + c), g);
        unpack8(*reinterpret_cast<const uint4*>(gu + r * 2 * f + f + c), u);
#pragma unroll
        for (int j = 0; j < 8; ++j) o[j] = silu_f(g[j]) * u[j];
        *reinterpret_cast<uint4*>(a + r * f + c) = pack8(o);
    }
}

__global__ void swiglu_bwd_kernel(const uint16_t* __restrict__ gu, const uint16_t* __restrict__ da,
                                  uint16_t* __restrict__ dh, int64_t M, int f) {
    const int64_t nv = M * (f / 8);
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < nv;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t r = i / (f / 8);
        const int c = static_cast<int>(i - r * (f / 8)) * 8;
        float g[8], u[8], d8[8], og[8], ou[8];
        unpack8(*reinterpret_cast<const uint4*>(gu + r * 2 * f + c), g);
        unpack8(*reinterpret_cast<const uint4*>(gu + r * 2 * f + f + c), u);
        unpack8(*reinterpret_cast<const uint4*>(da + r * f + c), d8);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float s = sigmoid_f(g[j]);
            og[j] = d8[j] * u[j] * s * (1.0f + g[j] * (1.0f - s));
            ou[j] = d8[j] * g[j] * s;
        }
        *reinterpret_cast<uint4*>(dh + r * 2 * f + c) = pack8(og);
        *reinterpret_cast<uint4*>(dh + r * 2 * f + f + c) = pack8(ou);
    }
}

int combine(const uint16_t* y, const int32_t* dest, const float* w, int T, int d, int k,
            uint16_t* out, cudaStream_t st) {
    if (T == 0) return MOE_OK;
    if (const int ns = comb_stages(k, d))
        return launch_comb<false>(ns, k, y, nullptr, dest, w, T, d, k, out, nullptr, st);
    combine_kernel<<<warp_grid(T), 256, 0, st>>>(y, dest, w, T, d, k, static_cast<int64_t>(T) * k, out);
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}

int combine_bwd(const uint16_t* dout, const uint16_t* y, const int32_t* dest, const float* w,
                int T, int d, int k, uint16_t* dy, float* dw, cudaStream_t st) {
    if (T == 0) return MOE_OK;
    const int64_t M = static_cast<int64_t>(T) * k;
    if (const int ns = comb_stages(k + 1, d))
        return launch_comb<true>(ns, k + 1, y, dout, dest, w, T, d, k, dy, dw, st);
    const int g = warp_grid(T);
    if (k <= 2) combine_bwd_kernel<2><<<g, 256, 0, st>>>(dout, y, dest, w, T, d, k, M, dy, dw);
    else if (k <= 4) combine_bwd_kernel<4><<<g, 256, 0, st>>>(dout, y, dest, w, T, d, k, M, dy, dw);
    else if (k <= 8) combine_bwd_kernel<8><<<g, 256, 0, st>>>(dout, y, dest, w, T, d, k, M, dy, dw);
    else if (k <= 16) combine_bwd_kernel<16><<<g, 256, 0, st>>>(dout, y, dest, w, T, d, k, M, dy, dw);
    else combine_bwd_kernel<32><<<g, 256, 0, st>>>(dout, y, dest, w, T, d, k, M, dy, dw);
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}

int unpermute_sum(const uint16_t* dxp, const int32_t* dest, int T, int d, int k, const float* dl,
                  const uint16_t* wr, int E, uint16_t* dx, cudaStream_t st) {
    if (T == 0) return MOE_OK;
    const int64_t M = static_cast<int64_t>(T) * k;
    if (dl && wr) {
        dim3 grid(static_cast<unsigned>(cdiv(T, 64)), static_cast<unsigned>(cdiv(d, 32)));
        unpermute_sum_router_kernel<<<grid, 128, 0, st>>>(dxp, dest, T, d, k, M, dl, wr, E, dx);
    } else if (const int ns = comb_stages(k, d)) {
        // unit weights: fmaf(1, x, acc) is the correctly rounded acc + x
        return launch_comb<false>(ns, k, dxp, nullptr, dest, nullptr, T, d, k, dx, nullptr, st);
    } else {
        unpermute_sum_kernel<<<warp_grid(T), 256, 0, st>>>(dxp, dest, T, d, k, M, dx);
    }
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}

int swiglu(const uint16_t* gu, uint16_t* a, int64_t M, int f, cudaStream_t st) {
    if (M == 0) return MOE_OK;
    swiglu_kernel<<<num_sms() * 8, 256, 0, st>>>(gu, a, M, f);
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}

int swiglu_bwd(const uint16_t* gu, const uint16_t* da, uint16_t* dh, int64_t M, int f,
               cudaStream_t st) {
    if (M == 0) return MOE_OK;
    swiglu_bwd_kernel<<<num_sms() * 8, 256, 0, st>>>(gu, da, dh, M, f);
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}

}  // namespace moe
