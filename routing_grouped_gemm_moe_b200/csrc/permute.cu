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

namespace moe {

constexpr int kTaskTokens = 128;  // tokens per task = threads per block

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

// One block of 1024 threads.  Thread (e, part) scans a contiguous range of
// tasks for expert e; parts = 1024 / E ranges are stitched through shared
// memory.  task_hist becomes the exclusive per-expert prefix over tasks.
__global__ void __launch_bounds__(1024) permute_scan_kernel(int32_t* __restrict__ task_hist,
                                                            int ntasks, int E,
                                                            int32_t* __restrict__ counts,
                                                            int32_t* __restrict__ offsets) {
    __shared__ int part_sum[1024];
    __shared__ int tot[1024];
    const int parts = max(1, 1024 / E);
    const int tid = threadIdx.x;
    const int e = tid % E;
    const int part = tid / E;
    const bool active = part < parts && tid < parts * E;
    const int per = (ntasks + parts - 1) / parts;
    const int b = min(ntasks, part * per), en = min(ntasks, b + per);
    int s = 0;
    if (active)
        for (int task = b; task < en; ++task) s += task_hist[static_cast<int64_t>(task) * E + e];
    part_sum[tid] = s;
    __syncthreads();
    if (active) {
        int run = 0;
        for (int q = 0; q < part; ++q) run += part_sum[q * E + e];
        for (int task = b; task < en; ++task) {
            int32_t* p = task_hist + static_cast<int64_t>(task) * E + e;
            const int c = *p;
            *p = run;
            run += c;
        }
        if (part == parts - 1) tot[e] = run;
    }
    __syncthreads();
    // exclusive scan of tot[0..E) -> offsets (E <= 1024): warp 0 does it in
    // segments of ceil(E / 32)
    if (tid < 32) {
        const int seg = (E + 31) / 32;
        const int lo = min(E, tid * seg), hi = min(E, lo + seg);
        int local = 0;
        for (int i = lo; i < hi; ++i) local += tot[i];
        int incl = local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (tid >= o) incl += v;
        }
        int run = incl - local;
        for (int i = lo; i < hi; ++i) {
            offsets[i] = run;
            counts[i] = tot[i];
            run += tot[i];
        }
        if (tid == 31) offsets[E] = incl;
    }
}

__global__ void __launch_bounds__(kTaskTokens) permute_rank_kernel(
    const int32_t* __restrict__ idx, int T, int E, int k, const int32_t* __restrict__ task_base,
    const int32_t* __restrict__ offsets, int32_t* __restrict__ dest_pos,
    int32_t* __restrict__ src_token) {
    constexpr int W = kTaskTokens / 32;
    extern __shared__ uint32_t masks[];  // [E][W]
    for (int i = threadIdx.x; i < E * W; i += blockDim.x) masks[i] = 0u;
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * kTaskTokens + threadIdx.x;
    if (t < T) {
        for (int i = 0; i < k; ++i) {
            const int e = idx[static_cast<int64_t>(t) * k + i];
            if (e >= 0 && e < E) atomicOr(&masks[e * W + warp], 1u << lane);
        }
    }
    __syncthreads();
    if (t < T) {
        const int32_t* base = task_base + static_cast<int64_t>(blockIdx.x) * E;
        const uint32_t lt = (1u << lane) - 1u;
        for (int i = 0; i < k; ++i) {
            const int e = idx[static_cast<int64_t>(t) * k + i];
            int pos = -1;
            if (e >= 0 && e < E) {
                pos = offsets[e] + base[e] + __popc(masks[e * W + warp] & lt);
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
    permute_scan_kernel<<<1, 1024, 0, st>>>(task_hist, ntasks, E, counts, offsets);
    MOE_LAUNCH_CHECK();
    permute_rank_kernel<<<ntasks, kTaskTokens, E * (kTaskTokens / 32) * sizeof(uint32_t), st>>>(
        idx, T, E, k, task_hist, offsets, dest_pos, src_token);
    MOE_LAUNCH_CHECK();
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
