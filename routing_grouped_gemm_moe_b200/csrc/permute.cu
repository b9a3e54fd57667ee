// Rowwise dispatch: routed token rows are written straight into contiguous
// per-expert input buffers, and the routing metadata (counts, offsets, row
// positions) is built and kept on the device ("Ai2 rebuilds Olmo's training
// stack for trillion-parameter MoEs", "Routing work stays on the GPU", first
// two bullets; "Supercharging Olmo-core ...", Summary).
//
// Four launches, no host round trip:
//   count : per 128-token task, an E-bin histogram (shared-memory atomics;
//           counts do not depend on order)
//   scan  : one block; per expert an exclusive scan over tasks, counts, and
//           the exclusive scan over experts (offsets)
//   rank  : per task, each (t, i) gets dest = offsets[e] + task base +
//           rank among earlier tokens of the task, from per-warp 32-bit
//           token masks (popc of lower lanes) -- deterministic, ascending
//           token order inside each expert
//   copy  : one warp per token reads x[t] once (16-byte vectors) and writes
//           its k copies (and, for an MXFP8 GEMM1, the row-wise MXFP8
//           encoding of x[t] to the same k rows)
#include "common.cuh"
#include "mx_encode.cuh"
#include "ptx.cuh"

namespace moe {

constexpr int kTaskTokens = 128;  // tokens per task = threads per block
constexpr size_t kBulkCopySmem = 200 * 1024;  // dynamic shared memory opt-in of the bulk copy

size_t permute_scratch_bytes(int T, int E) {
    const int64_t ntasks = cdiv(T, kTaskTokens);
    return static_cast<size_t>(ntasks) * E * sizeof(int32_t);
}

__global__ void __launch_bounds__(kTaskTokens) permute_count_kernel(
    const int32_t* __restrict__ idx, int T, int E, int k, int32_t* __restrict__ task_hist,
    int32_t* status) {
    extern __shared__ int hist[];
    for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
    __syncthreads();
    const int t = blockIdx.x * kTaskTokens + threadIdx.x;
    bool bad = false;
    if (t < T) {
        for (int i = 0; i < k; ++i) {
            const int e = idx[static_cast<int64_t>(t) * k + i];
            if (e >= 0 && e < E) atomicAdd(&hist[e], 1);
            else bad = true;
        }
    }
    if (bad) flag_status(status, MOE_ERR_DEVICE_BOUNDS);
    __syncthreads();
    int32_t* out = task_hist + static_cast<int64_t>(blockIdx.x) * E;
    for (int e = threadIdx.x; e < E; e += blockDim.x) out[e] = hist[e];
}

// One CTA per expert e: the exclusive prefix of the expert's count over the
// tasks (task_hist column e, in place) and counts[e] = its total.  Thread j
// sums a contiguous range of tasks; the ranges are stitched with a warp scan
// of the per-warp totals.
constexpr int kScanThreads = 256;

__device__ __forceinline__ int warp_incl_scan(int v, int lane) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
    }
    return v;
}

__global__ void __launch_bounds__(kScanThreads) permute_scan_kernel(int32_t* __restrict__ task_hist,
                                                                    int ntasks, int E,
                                                                    int32_t* __restrict__ counts) {
    ptx::grid_dependency_wait();
    __shared__ int warp_tot[kScanThreads / 32];
    const int e = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int per = (ntasks + kScanThreads - 1) / kScanThreads;
    const int b = min(ntasks, tid * per), en = min(ntasks, b + per);
    int s = 0;
    for (int task = b; task < en; ++task) s += task_hist[static_cast<int64_t>(task) * E + e];
    const int incl = warp_incl_scan(s, lane);
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int wt = lane < kScanThreads / 32 ? warp_tot[lane] : 0;
        const int wi = warp_incl_scan(wt, lane);
        if (lane < kScanThreads / 32) warp_tot[lane] = wi - wt;
        if (lane == kScanThreads / 32 - 1) counts[e] = wi;
    }
    __syncthreads();
    ptx::grid_dependents_launch();
    int run = warp_tot[warp] + incl - s;
    for (int task = b; task < en; ++task) {
        int32_t* q = task_hist + static_cast<int64_t>(task) * E + e;
        const int c = *q;
        *q = run;
        run += c;
    }
}

// Also the offsets: every CTA forms the exclusive scan of counts over the
// experts in shared memory (E <= 1024 values); CTA 0 writes it out.
__global__ void __launch_bounds__(kTaskTokens) permute_rank_kernel(
    const int32_t* __restrict__ idx, int T, int E, int k, const int32_t* __restrict__ task_base,
    const int32_t* __restrict__ counts, int32_t* __restrict__ offsets, int32_t* __restrict__ dest_pos,
    int32_t* __restrict__ src_token) {
    constexpr int W = kTaskTokens / 32;
    extern __shared__ uint32_t masks[];  // [E][W], then offsets [E + 1]
    int* s_off = reinterpret_cast<int*>(masks + E * W);
    __shared__ int warp_tot[W];
    for (int i = threadIdx.x; i < E * W; i += blockDim.x) masks[i] = 0u;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * kTaskTokens + threadIdx.x;
    ptx::grid_dependency_wait();
    int sel[32];
    const int kk = min(k, 32);
#pragma unroll
    for (int i = 0; i < 32; ++i) sel[i] = (i < kk && t < T) ? __ldg(idx + static_cast<int64_t>(t) * k + i) : -1;
    {   // offsets = exclusive scan of counts: thread j sums a contiguous range
        const int per = (E + kTaskTokens - 1) / kTaskTokens;
        const int b = min(E, static_cast<int>(threadIdx.x) * per), en = min(E, b + per);
        int sum = 0;
        for (int e = b; e < en; ++e) sum += counts[e];
        const int incl = warp_incl_scan(sum, lane);
        if (lane == 31) warp_tot[warp] = incl;
        __syncthreads();
        int base = 0;
        for (int w2 = 0; w2 < warp; ++w2) base += warp_tot[w2];
        int run = base + incl - sum;
        for (int e = b; e < en; ++e) {
            s_off[e] = run;
            run += counts[e];
        }
        if (threadIdx.x == kTaskTokens - 1) s_off[E] = run;
        __syncthreads();
        if (blockIdx.x == 0)
            for (int e = threadIdx.x; e <= E; e += blockDim.x) offsets[e] = s_off[e];
    }
    if (t < T) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const int e = sel[i];
            if (i < kk && e >= 0 && e < E) atomicOr(&masks[e * W + warp], 1u << lane);
        }
    }
    __syncthreads();
    ptx::grid_dependents_launch();
    if (t < T) {
        const int32_t* base = task_base + static_cast<int64_t>(blockIdx.x) * E;
        const uint32_t lt = (1u << lane) - 1u;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            if (i >= kk) break;
            const int e = sel[i];
            int pos = -1;
            if (e >= 0 && e < E) {
                pos = s_off[e] + base[e] + __popc(masks[e * W + warp] & lt);
                for (int w = 0; w < warp; ++w) pos += __popc(masks[e * W + w]);
                src_token[pos] = t;
            }
            dest_pos[static_cast<int64_t>(t) * k + i] = pos;
        }
    }
}

// One warp per token: x[t] is read once and stored to its k rows.  With
// `codes` (MXFP8 dispatch), the row's row-wise MXFP8 encoding is also stored
// to its k rows: a 32-value block is 4 consecutive 16-byte vectors, held by 4
// consecutive lanes, so its maximum takes two shuffles, and each token is
// encoded once for all of its rows.
template <bool MX>
__global__ void __launch_bounds__(256) permute_copy_kernel(const uint16_t* __restrict__ x,
                                                           const int32_t* __restrict__ dest_pos,
                                                           int T, int d, int k, int64_t M,
                                                           uint16_t* __restrict__ x_perm,
                                                           uint8_t* __restrict__ codes,
                                                           uint8_t* __restrict__ scales) {
    const int lane = threadIdx.x & 31;
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    const int nvec = d / 8;
    for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += nwarps) {
        const int my_dest = lane < k ? dest_pos[static_cast<int64_t>(t) * k + lane] : -1;
        const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<int64_t>(t) * d);
        // warp-uniform trip count (the shuffles need every lane); 4 vectors
        // per lane in flight before the k stores
        for (int v0 = 0; v0 < nvec; v0 += 128) {
            uint4 a[4];
            bool act[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int v = v0 + lane + 32 * u;
                act[u] = v < nvec;
                a[u] = act[u] ? __ldg(src + v) : make_uint4(0, 0, 0, 0);
            }
            uint2 q[4];      // MX: E4M3 codes of the lane's 8 values per vector
            uint32_t sc[4];  // MX: scale byte of the vector's block
            if constexpr (MX) {
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    uint32_t m = mag_max2(mag_max2(mag_max2(mag_max2(0u, a[u].x), a[u].y), a[u].z), a[u].w);
                    m = max(m & 0xFFFFu, m >> 16);
                    m = max(m, __shfl_xor_sync(0xffffffffu, m, 1));
                    m = max(m, __shfl_xor_sync(0xffffffffu, m, 2));
                    const int X = block_exponent(m);
                    const float s = pow2_neg(X);
                    q[u].x = static_cast<uint32_t>(e4m3x2(bf16_lo(a[u].x) * s, bf16_hi(a[u].x) * s)) |
                             (static_cast<uint32_t>(e4m3x2(bf16_lo(a[u].y) * s, bf16_hi(a[u].y) * s)) << 16);
                    q[u].y = static_cast<uint32_t>(e4m3x2(bf16_lo(a[u].z) * s, bf16_hi(a[u].z) * s)) |
                             (static_cast<uint32_t>(e4m3x2(bf16_lo(a[u].w) * s, bf16_hi(a[u].w) * s)) << 16);
                    sc[u] = static_cast<uint32_t>(X + 127);
                }
            }
            for (int i = 0; i < k; ++i) {
                const int p = __shfl_sync(0xffffffffu, my_dest, i);
                if (p < 0 || p >= M) continue;
                uint4* dst = reinterpret_cast<uint4*>(x_perm + static_cast<int64_t>(p) * d);
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    if (act[u]) dst[v0 + lane + 32 * u] = a[u];
                if constexpr (MX) {
                    uint2* cdst = reinterpret_cast<uint2*>(codes + static_cast<int64_t>(p) * d);
                    uint8_t* sdst = scales + static_cast<int64_t>(p) * (d / 32);
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int v = v0 + lane + 32 * u;
                        if (act[u]) {
                            cdst[v] = q[u];
                            if ((v & 3) == 0) sdst[v >> 2] = static_cast<uint8_t>(sc[u]);
                        }
                    }
                }
            }
        }
    }
}

// Bulk-copy dispatch: a CTA is one warp with kCopyStages shared-memory row
// stages.  Lane 0 loads x[t] into a stage with one bulk copy (cp.async.bulk,
// completion on the stage's mbarrier), kCopyAhead tokens before it is used;
// lanes 0..k-1 then store the stage to the token's k destination rows with one
// bulk copy each and commit a bulk group.  A stage is reloaded once the
// stores that read it are done (each lane waits for its own groups).  Data
// moves without passing through registers: a few instructions per 8 KB row
// instead of one per 16 bytes, so the rate does not fall with the SM clock.
template <int NS>
__global__ void __launch_bounds__(32) permute_bulk_copy_kernel(const uint16_t* __restrict__ x,
                                                               const int32_t* __restrict__ dest_pos,
                                                               int T, int d, int k, int64_t M,
                                                               uint16_t* __restrict__ x_perm,
                                                               int32_t* status) {
    constexpr int AHEAD = NS / 2;
    extern __shared__ __align__(128) uint8_t rows[];  // [NS][d] bf16
    __shared__ __align__(8) uint64_t full[NS];
    __shared__ int sdest[NS][32];
    __shared__ volatile int abort_flag;
    const int lane = threadIdx.x;
    const uint32_t row_bytes = static_cast<uint32_t>(d) * 2u;
    if (lane == 0) {
        for (int q = 0; q < NS; ++q) ptx::mbar_init(&full[q], 1);
        abort_flag = 0;
        ptx::fence_mbar_init();
    }
    __syncwarp();
    ptx::grid_dependency_wait();
    const int n = blockIdx.x < T ? (T - 1 - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x) + 1 : 0;
    auto issue = [&](int i) {  // token i of this CTA into stage i % NS
        const int q = i % NS;
        const int64_t t = blockIdx.x + static_cast<int64_t>(i) * gridDim.x;
        if (lane < k) sdest[q][lane] = dest_pos[t * k + lane];
        if (lane == 0) {
            ptx::mbar_arrive_expect_tx(&full[q], row_bytes);
            ptx::bulk_load(rows + static_cast<size_t>(q) * row_bytes, x + t * d, row_bytes, &full[q]);
        }
    };
    for (int i = 0; i < AHEAD && i < n; ++i) issue(i);
    bool ok = true;
    for (int i = 0; i < n; ++i) {
        if (i + AHEAD < n) {
            // stage (i + AHEAD) % NS last held token i + AHEAD - NS, whose
            // store group is followed by NS - AHEAD - 1 newer ones
            ptx::bulk_wait_group_read<NS - AHEAD - 1>();
            __syncwarp();
            issue(i + AHEAD);
        }
        const int q = i % NS;
        if (!ptx::mbar_wait(&full[q], static_cast<uint32_t>((i / NS) & 1), &abort_flag)) {
            ok = false;
            break;
        }
        if (lane < k) {
            const int p = sdest[q][lane];
            if (p >= 0 && p < M)
                ptx::bulk_store(x_perm + static_cast<int64_t>(p) * d, rows + static_cast<size_t>(q) * row_bytes,
                                row_bytes);
        }
        ptx::bulk_commit_group();
    }
    ptx::bulk_wait_group_all();
    if (!ok && lane == 0) flag_status(status, MOE_ERR_DEVICE_TIMEOUT);
}

// Launch with programmatic stream serialisation: the kernel may start while
// the previous one on the stream finishes; it calls griddepcontrol.wait before
// it reads anything that one wrote.
template <typename... KArgs, typename... Args>
static int launch_pdl(void (*kern)(KArgs...), int grid, int block, size_t smem, cudaStream_t st,
                      Args... args) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
    cfg.blockDim = dim3(static_cast<unsigned>(block), 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, args...) != cudaSuccess) return MOE_ERR_CUDA;
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}

template <int NS>
static int launch_bulk_copy(const uint16_t* x, const int32_t* dest_pos, int T, int d, int k,
                            uint16_t* x_perm, int32_t* status, cudaStream_t st) {
    const size_t smem = static_cast<size_t>(NS) * d * 2;
    static int configured_dev = -1;  // opt-in above 48 KB, once per device
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_dev != dev) {
        if (cudaFuncSetAttribute(permute_bulk_copy_kernel<NS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kBulkCopySmem) != cudaSuccess)
            return MOE_ERR_CUDA;
        configured_dev = dev;
    }
    // CTAs per SM that the shared memory admits (at most 8)
    int per_sm = static_cast<int>(kBulkCopySmem / (smem + 1024));
    per_sm = per_sm < 1 ? 1 : (per_sm > 8 ? 8 : per_sm);
    int64_t grid = static_cast<int64_t>(num_sms()) * per_sm;
    if (grid > T) grid = T;
    return launch_pdl(permute_bulk_copy_kernel<NS>, static_cast<int>(grid), 32, smem, st, x, dest_pos, T,
                      d, k, static_cast<int64_t>(T) * k, x_perm, status);
}

int permute_rows(const uint16_t* x, const int32_t* idx, int T, int d, int E, int k,
                 int32_t* counts, int32_t* offsets, int32_t* dest_pos, int32_t* src_token,
                 uint16_t* x_perm, int32_t* task_hist, int32_t* status, cudaStream_t st,
                 uint8_t* mx_codes, uint8_t* mx_scales) {
    const int ntasks = static_cast<int>(cdiv(T, kTaskTokens));
    if (T == 0) {
        if (cudaMemsetAsync(counts, 0, sizeof(int32_t) * E, st) != cudaSuccess) return MOE_ERR_CUDA;
        if (cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (E + 1), st) != cudaSuccess) return MOE_ERR_CUDA;
        return MOE_OK;
    }
    permute_count_kernel<<<ntasks, kTaskTokens, E * sizeof(int), st>>>(idx, T, E, k, task_hist, status);
    MOE_LAUNCH_CHECK();
    MOE_TRY(launch_pdl(permute_scan_kernel, E, kScanThreads, 0, st, task_hist, ntasks, E, counts));
    const size_t rank_smem = (static_cast<size_t>(E) * (kTaskTokens / 32) + E + 1) * sizeof(uint32_t);
    MOE_TRY(launch_pdl(permute_rank_kernel, ntasks, kTaskTokens, rank_smem, st, idx, T, E, k,
                       static_cast<const int32_t*>(task_hist), static_cast<const int32_t*>(counts),
                       offsets, dest_pos, src_token));
    if (!mx_codes) {
        // rows of at most 24 KB take the bulk-copy engine with 8 stages,
        // rows up to 96 KB with 2
        const size_t row = static_cast<size_t>(d) * 2;
        if (row * 8 <= kBulkCopySmem / 2) return launch_bulk_copy<8>(x, dest_pos, T, d, k, x_perm, status, st);
        if (row * 2 <= kBulkCopySmem) return launch_bulk_copy<2>(x, dest_pos, T, d, k, x_perm, status, st);
    }
    int64_t blocks = cdiv(T, 8);
    const int64_t cap = static_cast<int64_t>(num_sms()) * 8;
    if (blocks > cap) blocks = cap;
    if (mx_codes)
        permute_copy_kernel<true><<<static_cast<int>(blocks), 256, 0, st>>>(
            x, dest_pos, T, d, k, static_cast<int64_t>(T) * k, x_perm, mx_codes, mx_scales);
    else
        permute_copy_kernel<false><<<static_cast<int>(blocks), 256, 0, st>>>(
            x, dest_pos, T, d, k, static_cast<int64_t>(T) * k, x_perm, nullptr, nullptr);
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}

}  // namespace moe
