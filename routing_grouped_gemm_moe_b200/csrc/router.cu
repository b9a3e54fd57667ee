// Router: fp32 softmax / top-k with renormalisation, its backward, and the
// optional router projection logits = x W_r.
//
// "Ai2 rebuilds Olmo's training stack for trillion-parameter MoEs",
// introduction: a router sends each token to only a small selection of
// feed-forward experts; "Supercharging Olmo-core ...", Summary: 4 experts per
// token.  Reading: softmax over all E logits, keep the k largest (ties to the
// lower expert index), renormalise over them.
#include <math.h>

#include "common.cuh"

namespace moe {

__device__ __forceinline__ bool better(float av, int ai, float bv, int bi) {
    return av > bv || (av == bv && ai < bi);
}

// One warp per token.  Lane l holds logits l, l+32, ..., so EPL = ceil(E/32)
// values live in registers; k rounds of a shuffle argmax on (value, index)
// pick the experts in selection order.
template <int EPL>
__global__ void __launch_bounds__(256) router_topk_kernel(const float* __restrict__ logits, int T,
                                                          int E, int k, int32_t* __restrict__ idx,
                                                          float* __restrict__ w) {
    const int lane = threadIdx.x & 31;
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += nwarps) {
        const float* row = logits + static_cast<int64_t>(t) * E;
        float v[EPL];
        uint32_t taken = 0;
#pragma unroll
        for (int j = 0; j < EPL; ++j) {
            const int e = lane + 32 * j;
            if (e < E) v[j] = row[e];
            else { v[j] = -INFINITY; taken |= 1u << j; }
        }
        float my_v = 0.f;
        int my_i = 0;
        for (int i = 0; i < k; ++i) {
            float bv = -INFINITY;
            int bi = 0x7fffffff;
#pragma unroll
            for (int j = 0; j < EPL; ++j)
                if (!((taken >> j) & 1u) && better(v[j], lane + 32 * j, bv, bi)) { bv = v[j]; bi = lane + 32 * j; }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
                const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
                if (better(ov, oi, bv, bi)) { bv = ov; bi = oi; }
            }
            if (lane == (bi & 31)) taken |= 1u << (bi >> 5);
            if (lane == i) { my_v = bv; my_i = bi; }
        }
        const float lmax = __shfl_sync(0xffffffffu, my_v, 0);
        const float ex = lane < k ? expf(my_v - lmax) : 0.f;
        const float sum = warp_sum(ex);
        if (lane < k) {
            idx[static_cast<int64_t>(t) * k + lane] = my_i;
            w[static_cast<int64_t>(t) * k + lane] = ex / sum;
        }
    }
}

// logits[t, e] = sum_c x[t, c] W_r[c, e]; 32 tokens x 64 experts per block,
// d in chunks of 64 staged in shared memory; fp32 sum in ascending c.
__global__ void __launch_bounds__(256) router_proj_kernel(const uint16_t* __restrict__ x,
                                                          const uint16_t* __restrict__ wr, int T,
                                                          int d, int E, float* __restrict__ logits) {
    __shared__ float xs[32][65];
    __shared__ float ws[64][65];
    const int t0 = blockIdx.x * 32, e0 = blockIdx.y * 64;
    const int tid = threadIdx.x;
    const int ti = tid >> 3, ej = tid & 7;
    float acc[8];
#pragma unroll
    for (int m = 0; m < 8; ++m) acc[m] = 0.f;
    for (int c0 = 0; c0 < d; c0 += 64) {
        {   // x tile: 32 tokens x 64 columns, one 16-byte vector per thread
            const int row = tid >> 3, col = (tid & 7) * 8;
            const int t = t0 + row, c = c0 + col;
            float f8[8];
            if (t < T && c < d) {
                unpack8(*reinterpret_cast<const uint4*>(x + static_cast<int64_t>(t) * d + c), f8);
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) f8[i] = 0.f;
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) xs[row][col + i] = f8[i];
        }
        for (int i = tid; i < 64 * 64; i += 256) {
            const int cc = i >> 6, e = i & 63;
            const int c = c0 + cc;
            ws[cc][e] = (c < d && e0 + e < E) ? bf16_to_f32(wr[static_cast<int64_t>(c) * E + e0 + e]) : 0.f;
        }
        __syncthreads();
#pragma unroll 8
        for (int cc = 0; cc < 64; ++cc) {
            const float xv = xs[ti][cc];
#pragma unroll
            for (int m = 0; m < 8; ++m) acc[m] = fmaf(xv, ws[cc][ej + 8 * m], acc[m]);
        }
        __syncthreads();
    }
    const int t = t0 + ti;
    if (t < T) {
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            const int e = e0 + ej + 8 * m;
            if (e < E) logits[static_cast<int64_t>(t) * E + e] = acc[m];
        }
    }
}

// d_logits[t, idx[t, j]] = w_j (dw_j - sum_i w_i dw_i); zero elsewhere.
__global__ void __launch_bounds__(256) router_bwd_kernel(const int32_t* __restrict__ idx,
                                                         const float* __restrict__ w,
                                                         const float* __restrict__ dw, int T, int E,
                                                         int k, float* __restrict__ dl) {
    const int lane = threadIdx.x & 31;
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += nwarps) {
        float* row = dl + static_cast<int64_t>(t) * E;
        for (int e = lane; e < E; e += 32) row[e] = 0.f;
        float wi = 0.f, dwi = 0.f;
        int ei = -1;
        if (lane < k) {
            wi = w[static_cast<int64_t>(t) * k + lane];
            dwi = dw[static_cast<int64_t>(t) * k + lane];
            ei = idx[static_cast<int64_t>(t) * k + lane];
        }
        const float inner = warp_sum(wi * dwi);
        __syncwarp();
        if (lane < k && ei >= 0 && ei < E) row[ei] = wi * (dwi - inner);
    }
}

// dW_r[c, e] = sum_t x[t, c] d_logits[t, e]: 64 columns x 64 experts per
// block, tokens in chunks of 32 through shared memory, fp32 sum in token order.
__global__ void __launch_bounds__(256) router_proj_bwd_kernel(const uint16_t* __restrict__ x,
                                                              const float* __restrict__ dl, int T,
                                                              int d, int E,
                                                              uint16_t* __restrict__ dwr) {
    __shared__ float xs[32][65];
    __shared__ float ds[32][65];
    const int c0 = blockIdx.x * 64, e0 = blockIdx.y * 64;
    const int tid = threadIdx.x;
    const int ci = tid >> 2;        // 0..63 column
    const int eg = tid & 3;         // experts eg, eg+4, ... (16 of them)
    float acc[16];
#pragma unroll
    for (int m = 0; m < 16; ++m) acc[m] = 0.f;
    for (int t0 = 0; t0 < T; t0 += 32) {
        {
            const int row = tid >> 3, col = (tid & 7) * 8;
            const int t = t0 + row, c = c0 + col;
            float f8[8];
            if (t < T && c < d) {
                unpack8(*reinterpret_cast<const uint4*>(x + static_cast<int64_t>(t) * d + c), f8);
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) f8[i] = 0.f;
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) xs[row][col + i] = f8[i];
        }
        for (int i = tid; i < 32 * 64; i += 256) {
            const int row = i >> 6, e = i & 63;
            const int t = t0 + row;
            ds[row][e] = (t < T && e0 + e < E) ? dl[static_cast<int64_t>(t) * E + e0 + e] : 0.f;
        }
        __syncthreads();
#pragma unroll 4
        for (int r = 0; r < 32; ++r) {
            const float xv = xs[r][ci];
#pragma unroll
            for (int m = 0; m < 16; ++m) acc[m] = fmaf(xv, ds[r][eg + 4 * m], acc[m]);
        }
        __syncthreads();
    }
    const int c = c0 + ci;
    if (c < d) {
#pragma unroll
        for (int m = 0; m < 16; ++m) {
            const int e = e0 + eg + 4 * m;
            if (e < E) dwr[static_cast<int64_t>(c) * E + e] = f32_to_bf16(acc[m]);
        }
    }
}

static int grid_for_warps(int64_t warps) {
    int64_t blocks = (warps + 7) / 8;
    const int64_t cap = static_cast<int64_t>(num_sms()) * 16;
    if (blocks > cap) blocks = cap;
    return static_cast<int>(blocks < 1 ? 1 : blocks);
}

int router_topk(const float* logits, int T, int E, int k, int32_t* idx, float* w, cudaStream_t st) {
    if (T == 0) return MOE_OK;
    const int grid = grid_for_warps(T);
    const int epl = (E + 31) / 32;
    if (epl <= 1) router_topk_kernel<1><<<grid, 256, 0, st>>>(logits, T, E, k, idx, w);
    else if (epl <= 2) router_topk_kernel<2><<<grid, 256, 0, st>>>(logits, T, E, k, idx, w);
    else if (epl <= 4) router_topk_kernel<4><<<grid, 256, 0, st>>>(logits, T, E, k, idx, w);
    else if (epl <= 8) router_topk_kernel<8><<<grid, 256, 0, st>>>(logits, T, E, k, idx, w);
    else if (epl <= 16) router_topk_kernel<16><<<grid, 256, 0, st>>>(logits, T, E, k, idx, w);
    else router_topk_kernel<32><<<grid, 256, 0, st>>>(logits, T, E, k, idx, w);
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}

int router_proj(const uint16_t* x, const uint16_t* wr, int T, int d, int E, float* logits,
                cudaStream_t st) {
    if (T == 0) return MOE_OK;
    dim3 grid(static_cast<unsigned>(cdiv(T, 32)), static_cast<unsigned>(cdiv(E, 64)));
    router_proj_kernel<<<grid, 256, 0, st>>>(x, wr, T, d, E, logits);
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}

int router_bwd(const int32_t* idx, const float* w, const float* dw, int T, int E, int k,
               float* dl, cudaStream_t st) {
    if (T == 0) return MOE_OK;
    router_bwd_kernel<<<grid_for_warps(T), 256, 0, st>>>(idx, w, dw, T, E, k, dl);
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}

int router_proj_bwd(const uint16_t* x, const float* dl, int T, int d, int E, uint16_t* dwr,
                    cudaStream_t st) {
    dim3 grid(static_cast<unsigned>(cdiv(d, 64)), static_cast<unsigned>(cdiv(E, 64)));
    router_proj_bwd_kernel<<<grid, 256, 0, st>>>(x, dl, T, d, E, dwr);
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}

}  // namespace moe

// ------------------------------------------------------------------ routing balance
//
// "Ai2 rebuilds Olmo's training stack for trillion-parameter MoEs", "Four
// failure modes from the report", first bullet: a routing-balance score can
// improve while the actual workload gets less balanced.  Reading (the pages
// give no formula): the auxiliary balance loss L = E * sum_e f_e P_e with
// f_e = counts_e / (T k) and P_e the mean over tokens of the full softmax,
// reported next to the actual imbalance of the counts.  All sums run in a
// fixed order (deterministic).

namespace moe {

constexpr int kBalTokens = 256;  // tokens per block (8 warps x 32 tokens)

// partial[b][e] = sum over the block's tokens of softmax(l_t)_e
template <int EPL>
__global__ void __launch_bounds__(256) balance_partial_kernel(const float* __restrict__ logits,
                                                              int T, int E,
                                                              float* __restrict__ partial) {
    __shared__ float wsum[8][1024];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float acc[EPL];
#pragma unroll
    for (int j = 0; j < EPL; ++j) acc[j] = 0.f;
    const int t0 = blockIdx.x * kBalTokens + warp * 32;
    for (int i = 0; i < 32; ++i) {
        const int t = t0 + i;
        if (t >= T) break;
        const float* row = logits + static_cast<int64_t>(t) * E;
        float v[EPL];
        float mx = -INFINITY;
#pragma unroll
        for (int j = 0; j < EPL; ++j) {
            const int e = lane + 32 * j;
            v[j] = e < E ? row[e] : -INFINITY;
            mx = fmaxf(mx, v[j]);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        float s = 0.f;
#pragma unroll
        for (int j = 0; j < EPL; ++j) {
            v[j] = (lane + 32 * j < E) ? expf(v[j] - mx) : 0.f;
            s += v[j];
        }
        s = warp_sum(s);
        const float inv = 1.0f / s;
#pragma unroll
        for (int j = 0; j < EPL; ++j) acc[j] += v[j] * inv;
    }
#pragma unroll
    for (int j = 0; j < EPL; ++j)
        if (lane + 32 * j < E) wsum[warp][lane + 32 * j] = acc[j];
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        float s = 0.f;
        for (int w = 0; w < 8; ++w) s += wsum[w][e];
        partial[static_cast<int64_t>(blockIdx.x) * E + e] = s;
    }
}

// One block: P_e, f_e and the statistics.
__global__ void __launch_bounds__(1024) balance_final_kernel(const float* __restrict__ partial,
                                                             int nblk, const int32_t* __restrict__ counts,
                                                             int T, int E, int k,
                                                             float* __restrict__ stats,
                                                             float* __restrict__ probs_mean) {
    __shared__ float s_fp[1024];
    __shared__ float s_c[1024];
    const int tid = threadIdx.x;
    for (int e = tid; e < E; e += blockDim.x) {
        float s = 0.f;
        for (int b = 0; b < nblk; ++b) s += partial[static_cast<int64_t>(b) * E + e];
        const float P = s / static_cast<float>(T);
        const float c = static_cast<float>(counts[e]);
        if (probs_mean) probs_mean[e] = P;
        s_fp[e] = (c / (static_cast<float>(T) * k)) * P;
        s_c[e] = c;
    }
    __syncthreads();
    if (tid == 0) {
        double aux = 0.0, sum = 0.0, mx = 0.0, empty = 0.0;
        for (int e = 0; e < E; ++e) {
            aux += s_fp[e];
            sum += s_c[e];
            mx = s_c[e] > mx ? s_c[e] : mx;
            empty += s_c[e] == 0.f ? 1.0 : 0.0;
        }
        const double mean = sum / E;
        double var = 0.0;
        for (int e = 0; e < E; ++e) var += (s_c[e] - mean) * (s_c[e] - mean);
        var /= E;
        stats[0] = static_cast<float>(E * aux);
        stats[1] = mean > 0 ? static_cast<float>(mx / mean) : 0.f;
        stats[2] = mean > 0 ? static_cast<float>(sqrt(var) / mean) : 0.f;
        stats[3] = static_cast<float>(empty / E);
    }
}

// d_logits[t, j] += scale * (E / T) * p_tj * (f_j - sum_e f_e p_te)
template <int EPL>
__global__ void __launch_bounds__(256) balance_bwd_kernel(const float* __restrict__ logits,
                                                          const int32_t* __restrict__ counts, int T,
                                                          int E, int k, float scale,
                                                          float* __restrict__ dl) {
    const int lane = threadIdx.x & 31;
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    const float fk = 1.0f / (static_cast<float>(T) * k);
    for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += nwarps) {
        const float* row = logits + static_cast<int64_t>(t) * E;
        float v[EPL], f[EPL];
        float mx = -INFINITY;
#pragma unroll
        for (int j = 0; j < EPL; ++j) {
            const int e = lane + 32 * j;
            v[j] = e < E ? row[e] : -INFINITY;
            f[j] = e < E ? static_cast<float>(counts[e]) * fk : 0.f;
            mx = fmaxf(mx, v[j]);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        float s = 0.f;
#pragma unroll
        for (int j = 0; j < EPL; ++j) {
            v[j] = (lane + 32 * j < E) ? expf(v[j] - mx) : 0.f;
            s += v[j];
        }
        s = warp_sum(s);
        const float inv = 1.0f / s;
        float inner = 0.f;
#pragma unroll
        for (int j = 0; j < EPL; ++j) {
            v[j] *= inv;
            inner += f[j] * v[j];
        }
        inner = warp_sum(inner);
        const float c = scale * static_cast<float>(E) / static_cast<float>(T);
        float* drow = dl + static_cast<int64_t>(t) * E;
#pragma unroll
        for (int j = 0; j < EPL; ++j) {
            const int e = lane + 32 * j;
            if (e < E) drow[e] += c * v[j] * (f[j] - inner);
        }
    }
}

size_t balance_scratch_bytes(int T, int E) {
    return static_cast<size_t>(cdiv(T, kBalTokens)) * E * sizeof(float);
}

int router_balance(const float* logits, const int32_t* counts, int T, int E, int k, float* stats,
                   float* probs_mean, float* partial, cudaStream_t st) {
    const int nblk = static_cast<int>(cdiv(T, kBalTokens));
    const int epl = (E + 31) / 32;
    if (T > 0) {
        if (epl <= 1) balance_partial_kernel<1><<<nblk, 256, 0, st>>>(logits, T, E, partial);
        else if (epl <= 2) balance_partial_kernel<2><<<nblk, 256, 0, st>>>(logits, T, E, partial);
        else if (epl <= 4) balance_partial_kernel<4><<<nblk, 256, 0, st>>>(logits, T, E, partial);
        else if (epl <= 8) balance_partial_kernel<8><<<nblk, 256, 0, st>>>(logits, T, E, partial);
        else if (epl <= 16) balance_partial_kernel<16><<<nblk, 256, 0, st>>>(logits, T, E, partial);
        else balance_partial_kernel<32><<<nblk, 256, 0, st>>>(logits, T, E, partial);
        MOE_LAUNCH_CHECK();
    }
    balance_final_kernel<<<1, 1024, 0, st>>>(partial, nblk, counts, T > 0 ? T : 1, E, k, stats, probs_mean);
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}

int router_balance_bwd(const float* logits, const int32_t* counts, int T, int E, int k,
                       float scale, float* dl, cudaStream_t st) {
    if (T == 0) return MOE_OK;
    const int grid = grid_for_warps(T);
    const int epl = (E + 31) / 32;
    if (epl <= 1) balance_bwd_kernel<1><<<grid, 256, 0, st>>>(logits, counts, T, E, k, scale, dl);
    else if (epl <= 2) balance_bwd_kernel<2><<<grid, 256, 0, st>>>(logits, counts, T, E, k, scale, dl);
    else if (epl <= 4) balance_bwd_kernel<4><<<grid, 256, 0, st>>>(logits, counts, T, E, k, scale, dl);
    else if (epl <= 8) balance_bwd_kernel<8><<<grid, 256, 0, st>>>(logits, counts, T, E, k, scale, dl);
    else if (epl <= 16) balance_bwd_kernel<16><<<grid, 256, 0, st>>>(logits, counts, T, E, k, scale, dl);
    else balance_bwd_kernel<32><<<grid, 256, 0, st>>>(logits, counts, T, E, k, scale, dl);
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}

}  // namespace moe
