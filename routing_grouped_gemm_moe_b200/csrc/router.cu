// Router: fp32 softmax / top-k with renormalisation, its backward, and the
// optional router projection logits = x W_r.
//
// "Ai2 rebuilds Olmo's training stack for trillion-parameter MoEs",
// introduction: a router sends each token to only a small selection of
// feed-forward experts; "Supercharging Olmo-core ...", Summary: 4 experts per
// token.  Reading: softmax over all E logits, keep the k largest (ties to the
// lower expert index), renormalise over them.
#include <math.h>

#include <mutex>

#include "common.cuh"
#include "ptx.cuh"

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

// Warp per token with single-instruction warp reductions (k <= 8, E <= 256).
// Lane l holds the EPL = E / 32 logits l, l + 32, ... as order-preserving
// 32-bit keys (-0 and +0 share one key, so they tie), sorted in registers by
// key descending; equal keys stay in expert order.  Each of the k rounds takes
// the warp maximum of the lanes' heads (redux.sync.max), then the lowest
// expert index among the heads equal to it (redux.sync.min): exactly the
// (value descending, index ascending) order.  The winning lane drops its head.
__device__ __forceinline__ uint32_t order_key(float v) {
    const uint32_t b = __float_as_uint(v + 0.0f);  // -0 -> +0
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t key) {
    return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

template <int EPL>
__global__ void __launch_bounds__(256) router_topk_redux_kernel(const float* __restrict__ logits,
                                                               int T, int E, int k,
                                                               int32_t* __restrict__ idx,
                                                               float* __restrict__ w) {
    const int lane = threadIdx.x & 31;
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += nwarps) {
        const float* row = logits + static_cast<int64_t>(t) * E;
        uint32_t key[EPL];
        int ex[EPL];
#pragma unroll
        for (int j = 0; j < EPL; ++j) {
            const int e = lane + 32 * j;
            key[j] = e < E ? order_key(__ldg(row + e)) : 0u;  // 0: below every real key
            ex[j] = e;
        }
        // insertion sort by key descending; equal keys keep expert order
#pragma unroll
        for (int i = 1; i < EPL; ++i) {
#pragma unroll
            for (int j = i; j > 0; --j) {
                const bool sw = key[j] > key[j - 1];
                const uint32_t k0 = key[j - 1], k1 = key[j];
                const int e0 = ex[j - 1], e1 = ex[j];
                key[j - 1] = sw ? k1 : k0;
                key[j] = sw ? k0 : k1;
                ex[j - 1] = sw ? e1 : e0;
                ex[j] = sw ? e0 : e1;
            }
        }
        uint32_t my_key = 0;
        int my_e = 0;
        for (int i = 0; i < k; ++i) {
            const uint32_t m = __reduce_max_sync(0xffffffffu, key[0]);
            const uint32_t cand = key[0] == m ? static_cast<uint32_t>(ex[0]) : 0xffffffffu;
            const uint32_t e_win = __reduce_min_sync(0xffffffffu, cand);
            if (lane == i) { my_key = m; my_e = static_cast<int>(e_win); }
            if (cand == e_win) {  // the winning lane drops its head
#pragma unroll
                for (int j = 0; j + 1 < EPL; ++j) { key[j] = key[j + 1]; ex[j] = ex[j + 1]; }
                key[EPL - 1] = 0u;
            }
        }
        const float my_v = key_value(my_key);
        const float lmax = __shfl_sync(0xffffffffu, my_v, 0);
        const float e_w = lane < k ? expf(my_v - lmax) : 0.f;
        const float sum = warp_sum(e_w);
        if (lane < k) {
            idx[static_cast<int64_t>(t) * k + lane] = my_e;
            w[static_cast<int64_t>(t) * k + lane] = e_w / sum;
        }
    }
}

// Thread per token (E in {32, 64, 128}, k in {2, 4, 8}): the warp-wide
// rounds above cost about 300 instructions per token, which made the kernel
// issue-bound at a fraction of HBM bandwidth.  Here a warp stages the logits
// of 32 tokens in shared memory with coalesced 16-byte copies (rows padded by
// 16 bytes, so that each lane reading its own row is conflict-free), and each
// lane then selects its own token's top-k with no cross-lane work:
//   1. G = 2k group maxima over a fixed partition of the E logits; their k-th
//      largest, L, is a lower bound of the k-th largest logit (k distinct
//      groups hold a value >= L), so every selected expert has logit >= L;
//   2. the experts with logit >= L (about 10 of 128 for k = 8) are inserted,
//      in expert order, into a sorted list of k (value, expert) pairs; an
//      element moves ahead only of strictly smaller values, so equal logits
//      keep the lower expert index first -- the (value descending, index
//      ascending) order, with -0 == +0 as in any float comparison.
// Weights as above: exp(l_i - l_0) over their sum (summed in slot order).
constexpr int kRtWarps = 2;  // warps per block, 32 tokens per warp

template <int E_>
constexpr int rt_pitch() { return E_ + 4; }  // floats per staged row
template <int E_>
constexpr int rt_smem_bytes() { return kRtWarps * 32 * rt_pitch<E_>() * 4; }

template <int N>
__device__ __forceinline__ void sort_desc(float (&v)[N]) {  // bitonic, N a power of 2
#pragma unroll
    for (int size = 2; size <= N; size <<= 1) {
#pragma unroll
        for (int stride = size / 2; stride > 0; stride >>= 1) {
#pragma unroll
            for (int i = 0; i < N; ++i) {
                const int j = i ^ stride;
                if (j > i) {
                    const float hi = fmaxf(v[i], v[j]), lo = fminf(v[i], v[j]);
                    const bool desc = (i & size) == 0;
                    v[i] = desc ? hi : lo;
                    v[j] = desc ? lo : hi;
                }
            }
        }
    }
}

template <int E_, int K_>
__global__ void __launch_bounds__(kRtWarps * 32) router_topk_thread_kernel(const float* __restrict__ logits,
                                                                         int T, int32_t* __restrict__ idx,
                                                                         float* __restrict__ w) {
    constexpr int NC = E_ / 4;  // 16-byte chunks per row
    constexpr int PITCH = rt_pitch<E_>();
    constexpr int G = 2 * K_;
    constexpr int GS = E_ / G;  // logits per group
    constexpr int NW = (E_ + 63) / 64;  // 64-bit candidate-mask words
    // E_ <= 128: the compiler keeps the row in registers between the passes
    static_assert(E_ % 32 == 0 && E_ <= 128 && GS >= 1 && (K_ & (K_ - 1)) == 0, "shape");
    extern __shared__ float4 rt_smem[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t t0 = (static_cast<int64_t>(blockIdx.x) * kRtWarps + warp) * 32;
    if (t0 >= T) return;
    const int nt = static_cast<int>(T - t0 < 32 ? T - t0 : 32);
    float* rows = reinterpret_cast<float*>(rt_smem) + warp * 32 * PITCH;
    const float* src = logits + t0 * E_;
    {
        // the warp copies 32 consecutive chunks (32 / NC rows) per step: lane
        // `lane` always copies chunk lane % NC of row step * 32 / NC + lane / NC
        constexpr int RPS = 32 / NC;  // rows per step
        const int r0 = lane / NC, c0 = lane % NC;
        float* dst = rows + r0 * PITCH + c0 * 4;
        const float* s0 = src + r0 * E_ + c0 * 4;
#pragma unroll
        for (int i = 0; i < NC; ++i)
            if (i * RPS + r0 < nt) ptx::cp_async_16(dst + i * RPS * PITCH, s0 + i * RPS * E_);
    }
    ptx::cp_async_wait_all();
    __syncwarp();
    if (lane >= nt) return;
    const float* row = rows + lane * PITCH;

    // 1. group maxima and the bound L
    float a[K_], b[K_];
#pragma unroll
    for (int g = 0; g < K_; ++g) { a[g] = -INFINITY; b[g] = -INFINITY; }
#pragma unroll
    for (int c = 0; c < NC; ++c) {
        const float4 v = reinterpret_cast<const float4*>(row)[c];
        const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int g = (4 * c + i) / GS;
            if (g < K_) a[g] = fmaxf(a[g], vv[i]);
            else b[g - K_] = fmaxf(b[g - K_], vv[i]);
        }
    }
    sort_desc(a);
    sort_desc(b);
    float L = INFINITY;  // k-th largest of the 2k maxima (bitonic merge of two sorted lists)
#pragma unroll
    for (int i = 0; i < K_; ++i) L = fminf(L, fmaxf(a[i], b[K_ - 1 - i]));

    // 2. candidates (logit >= L) as a bit mask in expert order
    uint32_t m32[2 * NW];
#pragma unroll
    for (int j = 0; j < 2 * NW; ++j) m32[j] = 0u;
#pragma unroll
    for (int c = 0; c < NC; ++c) {
        const float4 v = reinterpret_cast<const float4*>(row)[c];
        const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
            if (vv[i] >= L) m32[(4 * c + i) >> 5] |= 1u << ((4 * c + i) & 31);
    }
    uint64_t q[NW];
#pragma unroll
    for (int j = 0; j < NW; ++j) q[j] = (static_cast<uint64_t>(m32[2 * j + 1]) << 32) | m32[2 * j];
    float sk[K_];
    int si[K_];
#pragma unroll
    for (int i = 0; i < K_; ++i) { sk[i] = -INFINITY; si[i] = 0; }
    int base = 0;
    while (true) {
        if (q[0] == 0) {  // next non-empty word (the words shift down)
            bool more = false;
#pragma unroll
            for (int j = 1; j < NW; ++j) more |= q[j] != 0;
            if (!more) break;
            do {
#pragma unroll
                for (int j = 0; j + 1 < NW; ++j) q[j] = q[j + 1];
                q[NW - 1] = 0;
                base += 64;
            } while (q[0] == 0);
        }
        const int e = base + __ffsll(static_cast<long long>(q[0])) - 1;
        q[0] &= q[0] - 1;
        const float v = row[e];
        bool gt[K_];
#pragma unroll
        for (int i = 0; i < K_; ++i) gt[i] = v > sk[i];
#pragma unroll
        for (int i = K_ - 1; i > 0; --i) {
            sk[i] = gt[i - 1] ? sk[i - 1] : (gt[i] ? v : sk[i]);
            si[i] = gt[i - 1] ? si[i - 1] : (gt[i] ? e : si[i]);
        }
        sk[0] = gt[0] ? v : sk[0];
        si[0] = gt[0] ? e : si[0];
    }

    float ex[K_], sum = 0.f;
#pragma unroll
    for (int i = 0; i < K_; ++i) { ex[i] = expf(sk[i] - sk[0]); sum += ex[i]; }
    const int64_t t = t0 + lane;
    int32_t* io = idx + t * K_;
    float* wo = w + t * K_;
    if constexpr (K_ >= 4) {
#pragma unroll
        for (int i = 0; i < K_; i += 4) {
            *reinterpret_cast<int4*>(io + i) = make_int4(si[i], si[i + 1], si[i + 2], si[i + 3]);
            *reinterpret_cast<float4*>(wo + i) =
                make_float4(ex[i] / sum, ex[i + 1] / sum, ex[i + 2] / sum, ex[i + 3] / sum);
        }
    } else {
#pragma unroll
        for (int i = 0; i < K_; ++i) { io[i] = si[i]; wo[i] = ex[i] / sum; }
    }
}

template <int E_, int K_>
static int launch_topk_thread(const float* logits, int T, int32_t* idx, float* w, cudaStream_t st) {
    auto kern = router_topk_thread_kernel<E_, K_>;
    constexpr int smem = rt_smem_bytes<E_>();
    if (smem > 48 * 1024) {
        static std::once_flag once;
        static cudaError_t err = cudaSuccess;
        std::call_once(once, [&] { err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem); });
        if (err != cudaSuccess) return MOE_ERR_CUDA;
    }
    const int64_t blocks = cdiv(T, kRtWarps * 32);
    kern<<<static_cast<unsigned>(blocks), kRtWarps * 32, smem, st>>>(logits, T, idx, w);
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}

template <int E_>
static int topk_thread_k(const float* logits, int T, int k, int32_t* idx, float* w, cudaStream_t st) {
    switch (k) {
        case 2: return launch_topk_thread<E_, 2>(logits, T, idx, w, st);
        case 4: return launch_topk_thread<E_, 4>(logits, T, idx, w, st);
        default: return launch_topk_thread<E_, 8>(logits, T, idx, w, st);
    }
}

// Router projection and its weight gradient: small dense products whose
// reduction axis (d, or T) is long.  A cluster of kSplit CTAs shares one
// 64 x 32 output tile and splits the reduction axis into slices; a CTA walks
// its slice in pieces of 64 staged in shared memory as fp32 (the next
// piece's loads are issued before the current piece is used).  Thread = 4 x 4
// outputs, so each FMA costs 1/8 of a shared-memory vector load.  The kSplit
// partial tiles are added in rank order through distributed shared memory,
// each CTA finishing 64 / kSplit rows: deterministic, no workspace, kSplit x
// more CTAs than output tiles.
constexpr int kProjThreads = 128;  // thread: rows 4 (tid % 16) .. +4, columns 4 (tid / 16) .. +4
constexpr int kSplit = 8;
constexpr int kPiece = 64;         // reduction elements per staged piece
constexpr int kTileR = 64, kTileC = 32;

// Cluster sum of the partial tiles `red` (fp32 [kTileR][kTileC + 1] in every CTA).
template <typename Store>
__device__ __forceinline__ void cluster_tile_sum(float (&red)[kTileR][kTileC + 1], Store store) {
    ptx::cluster_sync();
    const uint32_t rank = ptx::cluster_ctarank();
    constexpr int ROWS = kTileR / kSplit;
    for (int i = threadIdx.x; i < ROWS * kTileC; i += blockDim.x) {
        const int r = static_cast<int>(rank) * ROWS + i / kTileC, c = i % kTileC;
        const uint32_t local = ptx::smem_addr(&red[r][c]);
        float s = 0.f;
#pragma unroll
        for (int q = 0; q < kSplit; ++q) s += ptx::ld_shared_cluster_f32(ptx::mapa_shared(local, q));
        store(r, c, s);
    }
    ptx::cluster_sync();  // peers may still read this CTA's tile
}

// Eight bf16 of W_r row `c`, experts e0 + 8 v .. +8 (zero past E).
__device__ __forceinline__ uint4 load_wr8(const uint16_t* __restrict__ wr, int c, int E, int e0, int v,
                                          bool full_e) {
    const uint16_t* src = wr + static_cast<int64_t>(c) * E + e0 + 8 * v;
    if (full_e) return __ldg(reinterpret_cast<const uint4*>(src));
    uint32_t h[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int e = e0 + 8 * v + 2 * j;
        const uint32_t lo = e < E ? __ldg(src + 2 * j) : 0u;
        const uint32_t hi = e + 1 < E ? __ldg(src + 2 * j + 1) : 0u;
        h[j] = lo | (hi << 16);
    }
    return make_uint4(h[0], h[1], h[2], h[3]);
}

__device__ __forceinline__ void fma4x4(float (&acc)[4][4], const float4& a, const float4& b) {
    const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
}

// logits[t, e] = sum_c x[t, c] W_r[c, e]: tile 64 tokens x 32 experts; CTA q
// of the cluster takes the q-th slice of d.
__global__ void __launch_bounds__(kProjThreads) router_proj_kernel(
    const uint16_t* __restrict__ x, const uint16_t* __restrict__ wr, int T, int d, int E,
    float* __restrict__ logits) {
    __shared__ __align__(16) float xs[kPiece][kTileR + 4];  // [column][token]
    __shared__ __align__(16) float ws[kPiece][kTileC];      // [column][expert]
    __shared__ float red[kTileR][kTileC + 1];
    const int tid = threadIdx.x, tg = tid & 15, eg = tid >> 4;
    const int q = static_cast<int>(ptx::cluster_ctarank());
    const int t0 = (blockIdx.x / kSplit) * kTileR, e0 = blockIdx.y * kTileC;
    const bool full_e = e0 + kTileC <= E && (E % 8) == 0;
    const int64_t nch = d / 8;
    const int c_lo = static_cast<int>(nch * q / kSplit) * 8;
    const int c_hi = static_cast<int>(nch * (q + 1) / kSplit) * 8;
    // a piece: x 64 tokens x 8 vectors (4 per thread), W_r 64 rows x 4 vectors (2 per thread)
    uint4 xv[4], wv[2];
    auto fetch = [&](int cp) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int i = tid + kProjThreads * j;
            const int r = i & 63, c = cp + 8 * (i >> 6);
            xv[j] = (t0 + r < T && c < c_hi)
                        ? __ldg(reinterpret_cast<const uint4*>(x + static_cast<int64_t>(t0 + r) * d + c))
                        : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int i = tid + kProjThreads * j;
            const int cc = i >> 2;
            wv[j] = (cp + cc < c_hi) ? load_wr8(wr, cp + cc, E, e0, i & 3, full_e) : make_uint4(0, 0, 0, 0);
        }
    };
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
    if (c_lo < c_hi) fetch(c_lo);
    for (int cp = c_lo; cp < c_hi; cp += kPiece) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int i = tid + kProjThreads * j;
            float f[8];
            unpack8(xv[j], f);
#pragma unroll
            for (int m = 0; m < 8; ++m) xs[8 * (i >> 6) + m][i & 63] = f[m];
        }
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int i = tid + kProjThreads * j;
            float f[8];
            unpack8(wv[j], f);
            float4* dst = reinterpret_cast<float4*>(&ws[i >> 2][8 * (i & 3)]);
            dst[0] = make_float4(f[0], f[1], f[2], f[3]);
            dst[1] = make_float4(f[4], f[5], f[6], f[7]);
        }
        __syncthreads();
        if (cp + kPiece < c_hi) fetch(cp + kPiece);
        const int n = min(kPiece, c_hi - cp);
#pragma unroll 4
        for (int cc = 0; cc < n; ++cc)
            fma4x4(acc, *reinterpret_cast<const float4*>(&xs[cc][4 * tg]),
                   *reinterpret_cast<const float4*>(&ws[cc][4 * eg]));
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) red[4 * tg + i][4 * eg + j] = acc[i][j];
    cluster_tile_sum(red, [&](int r, int c, float s) {
        if (t0 + r < T && e0 + c < E) logits[static_cast<int64_t>(t0 + r) * E + e0 + c] = s;
    });
}

// dW_r[c, e] = sum_t x[t, c] d_logits[t, e]: tile 64 columns x 32 experts;
// CTA q of the cluster takes the q-th slice of the tokens.
__global__ void __launch_bounds__(kProjThreads) router_proj_bwd_kernel(
    const uint16_t* __restrict__ x, const float* __restrict__ dl, int T, int d, int E,
    uint16_t* __restrict__ dwr) {
    __shared__ __align__(16) float xs[kPiece][kTileR + 4];  // [token][column]
    __shared__ __align__(16) float gs[kPiece][kTileC];      // [token][expert]
    __shared__ float red[kTileR][kTileC + 1];
    const int tid = threadIdx.x, cg = tid & 15, eg = tid >> 4;
    const int q = static_cast<int>(ptx::cluster_ctarank());
    const int c0 = (blockIdx.x / kSplit) * kTileR, e0 = blockIdx.y * kTileC;
    const bool full_e = e0 + kTileC <= E && (E % 4) == 0;
    const int t_lo = static_cast<int>(static_cast<int64_t>(T) * q / kSplit);
    const int t_hi = static_cast<int>(static_cast<int64_t>(T) * (q + 1) / kSplit);
    // a piece: x 64 tokens x 8 vectors (4 per thread), d_logits 64 tokens x 8 float4 (4 per thread)
    uint4 xv[4];
    float4 gv[4];
    auto fetch = [&](int tp) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int i = tid + kProjThreads * j;
            const int r = i >> 3, c = c0 + 8 * (i & 7);
            xv[j] = (tp + r < t_hi && c < d)
                        ? __ldg(reinterpret_cast<const uint4*>(x + static_cast<int64_t>(tp + r) * d + c))
                        : make_uint4(0, 0, 0, 0);
            const int e = e0 + 4 * (i & 7);
            const float* src = dl + static_cast<int64_t>(tp + r) * E + e;
            if (tp + r >= t_hi) {
                gv[j] = make_float4(0.f, 0.f, 0.f, 0.f);
            } else if (full_e) {
                gv[j] = __ldg(reinterpret_cast<const float4*>(src));
            } else {
                gv[j] = make_float4(e < E ? __ldg(src) : 0.f, e + 1 < E ? __ldg(src + 1) : 0.f,
                                    e + 2 < E ? __ldg(src + 2) : 0.f, e + 3 < E ? __ldg(src + 3) : 0.f);
            }
        }
    };
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
    if (t_lo < t_hi) fetch(t_lo);
    for (int tp = t_lo; tp < t_hi; tp += kPiece) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int i = tid + kProjThreads * j;
            float f[8];
            unpack8(xv[j], f);
            float4* dst = reinterpret_cast<float4*>(&xs[i >> 3][8 * (i & 7)]);
            dst[0] = make_float4(f[0], f[1], f[2], f[3]);
            dst[1] = make_float4(f[4], f[5], f[6], f[7]);
            *reinterpret_cast<float4*>(&gs[i >> 3][4 * (i & 7)]) = gv[j];
        }
        __syncthreads();
        if (tp + kPiece < t_hi) fetch(tp + kPiece);
        const int n = min(kPiece, t_hi - tp);
#pragma unroll 4
        for (int r = 0; r < n; ++r)
            fma4x4(acc, *reinterpret_cast<const float4*>(&xs[r][4 * cg]),
                   *reinterpret_cast<const float4*>(&gs[r][4 * eg]));
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) red[4 * cg + i][4 * eg + j] = acc[i][j];
    cluster_tile_sum(red, [&](int r, int e, float s) {
        if (c0 + r < d && e0 + e < E) dwr[static_cast<int64_t>(c0 + r) * E + e0 + e] = f32_to_bf16(s);
    });
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

// E % 4 == 0: the row is written once, as 16-byte vectors -- lane l owns
// entries 4 l .. 4 l + 3 of every 128-entry chunk and fills in the selected
// experts' values it holds (broadcast by shuffles) -- instead of zeroing the
// row and then storing the k values over it.
__global__ void __launch_bounds__(256) router_bwd_vec_kernel(const int32_t* __restrict__ idx,
                                                             const float* __restrict__ w,
                                                             const float* __restrict__ dw, int T,
                                                             int E, int k, float* __restrict__ dl) {
    const int lane = threadIdx.x & 31;
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += nwarps) {
        float wi = 0.f, dwi = 0.f;
        int ei = -1;
        if (lane < k) {
            wi = __ldg(w + static_cast<int64_t>(t) * k + lane);
            dwi = __ldg(dw + static_cast<int64_t>(t) * k + lane);
            ei = __ldg(idx + static_cast<int64_t>(t) * k + lane);
        }
        const float inner = warp_sum(wi * dwi);
        const float gi = wi * (dwi - inner);
        float4* row = reinterpret_cast<float4*>(dl + static_cast<int64_t>(t) * E);
        for (int c = 0; c < E; c += 128) {
            const int e0 = c + 4 * lane;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int i = 0; i < k; ++i) {
                const int o = __shfl_sync(0xffffffffu, ei, i) - e0;
                const float g = __shfl_sync(0xffffffffu, gi, i);
                v.x = o == 0 ? g : v.x;
                v.y = o == 1 ? g : v.y;
                v.z = o == 2 ? g : v.z;
                v.w = o == 3 ? g : v.w;
            }
            if (e0 < E) row[e0 >> 2] = v;
        }
    }
}

// Thread per token (E % 4 == 0, E <= 256, k <= 8): a warp builds the dense
// d_logits rows of its 32 tokens in shared memory -- zeroed with 16-byte
// stores, then each lane writes its token's k values -- and one bulk copy
// stores the 32 contiguous rows.  The warp-per-token kernel above spends
// about 10 instructions per (token, selected expert) on shuffles and selects
// and was issue-bound at a fraction of HBM bandwidth.
constexpr int kRbWarps = 2;

__global__ void __launch_bounds__(kRbWarps * 32) router_bwd_thread_kernel(const int32_t* __restrict__ idx,
                                                                        const float* __restrict__ w,
                                                                        const float* __restrict__ dw, int T,
                                                                        int E, int k, float* __restrict__ dl) {
    extern __shared__ float4 rb_smem[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t t0 = (static_cast<int64_t>(blockIdx.x) * kRbWarps + warp) * 32;
    if (t0 >= T) return;
    const int nt = static_cast<int>(T - t0 < 32 ? T - t0 : 32);
    float* rows = reinterpret_cast<float*>(rb_smem) + static_cast<int64_t>(warp) * 32 * E;
    float4* r4 = reinterpret_cast<float4*>(rows);
    const int n4 = nt * E / 4;
    for (int i = lane; i < n4; i += 32) r4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    __syncwarp();
    if (lane < nt) {
        const int64_t t = t0 + lane;
        float wi[8], dwi[8];
        int ei[8];
        float inner = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if (i < k) {
                wi[i] = __ldg(w + t * k + i);
                dwi[i] = __ldg(dw + t * k + i);
                ei[i] = __ldg(idx + t * k + i);
                inner += wi[i] * dwi[i];
            }
        }
#pragma unroll
        for (int i = 0; i < 8; ++i)
            if (i < k && ei[i] >= 0 && ei[i] < E) rows[lane * E + ei[i]] = wi[i] * (dwi[i] - inner);
    }
    ptx::fence_proxy_async_smem();  // the rows are read by the bulk copy (async proxy)
    __syncwarp();
    if (lane == 0) {
        ptx::bulk_store(dl + t0 * E, rows, static_cast<uint32_t>(nt) * E * 4);
        ptx::bulk_commit_group();
        ptx::bulk_wait_group_read<0>();
    }
}

// Cluster launch of a projection kernel: kSplit CTAs per output tile.
template <typename... KArgs, typename... Args>
static int launch_proj(void (*kern)(KArgs...), int tiles_x, int tiles_y, cudaStream_t st,
                       Args... args) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kSplit;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(static_cast<unsigned>(tiles_x) * kSplit, static_cast<unsigned>(tiles_y), 1);
    cfg.blockDim = dim3(kProjThreads, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, args...) != cudaSuccess) return MOE_ERR_CUDA;
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}

static int grid_for_warps(int64_t warps) {
    int64_t blocks = (warps + 7) / 8;
    const int64_t cap = static_cast<int64_t>(num_sms()) * 16;
    if (blocks > cap) blocks = cap;
    return static_cast<int>(blocks < 1 ? 1 : blocks);
}

int router_topk(const float* logits, int T, int E, int k, int32_t* idx, float* w, cudaStream_t st) {
    if (T == 0) return MOE_OK;
    const bool aligned = ((reinterpret_cast<uintptr_t>(logits) | reinterpret_cast<uintptr_t>(idx) |
                           reinterpret_cast<uintptr_t>(w)) & 15) == 0;
    if (aligned && (k == 2 || k == 4 || k == 8)) {
        switch (E) {
            case 32: return topk_thread_k<32>(logits, T, k, idx, w, st);
            case 64: return topk_thread_k<64>(logits, T, k, idx, w, st);
            case 128: return topk_thread_k<128>(logits, T, k, idx, w, st);
            default: break;
        }
    }
    const int grid = grid_for_warps(T);
    if (E <= 256 && k <= 8) {
        const int epl = (E + 31) / 32;
        if (epl <= 1) router_topk_redux_kernel<1><<<grid, 256, 0, st>>>(logits, T, E, k, idx, w);
        else if (epl <= 2) router_topk_redux_kernel<2><<<grid, 256, 0, st>>>(logits, T, E, k, idx, w);
        else if (epl <= 4) router_topk_redux_kernel<4><<<grid, 256, 0, st>>>(logits, T, E, k, idx, w);
        else router_topk_redux_kernel<8><<<grid, 256, 0, st>>>(logits, T, E, k, idx, w);
        MOE_LAUNCH_CHECK();
        return MOE_OK;
    }
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
    return launch_proj(router_proj_kernel, static_cast<int>(cdiv(T, kTileR)),
                       static_cast<int>(cdiv(E, kTileC)), st, x, wr, T, d, E, logits);
}

int router_bwd(const int32_t* idx, const float* w, const float* dw, int T, int E, int k,
               float* dl, cudaStream_t st) {
    if (T == 0) return MOE_OK;
    if (E % 4 == 0 && E <= 256 && k <= 8 && (reinterpret_cast<uintptr_t>(dl) & 15) == 0) {
        const int smem = kRbWarps * 32 * E * 4;
        if (smem > 48 * 1024) {
            static std::once_flag once;
            static cudaError_t err = cudaSuccess;
            std::call_once(once, [] {
                err = cudaFuncSetAttribute(router_bwd_thread_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           kRbWarps * 32 * 256 * 4);
            });
            if (err != cudaSuccess) return MOE_ERR_CUDA;
        }
        router_bwd_thread_kernel<<<static_cast<unsigned>(cdiv(T, kRbWarps * 32)), kRbWarps * 32, smem, st>>>(
            idx, w, dw, T, E, k, dl);
    } else if (E % 4 == 0 && (reinterpret_cast<uintptr_t>(dl) & 15) == 0)
        router_bwd_vec_kernel<<<grid_for_warps(T), 256, 0, st>>>(idx, w, dw, T, E, k, dl);
    else
        router_bwd_kernel<<<grid_for_warps(T), 256, 0, st>>>(idx, w, dw, T, E, k, dl);
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}

int router_proj_bwd(const uint16_t* x, const float* dl, int T, int d, int E, uint16_t* dwr,
                    cudaStream_t st) {
    return launch_proj(router_proj_bwd_kernel, static_cast<int>(cdiv(d, kTileR)),
                       static_cast<int>(cdiv(E, kTileC)), st, x, dl, T, d, E, dwr);
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
