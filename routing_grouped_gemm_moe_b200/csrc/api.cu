// extern "C" entry points: host-side validation, then the launchers.  Each
// compute entry point is an NVTX range of its own name (free unless a
// profiler such as Nsight Systems is attached), so a timeline shows the
// library's calls around their kernels.
#include <atomic>
#include <mutex>

#include "common.cuh"
#include "nvtx_range.cuh"

namespace moe {

int router_topk(const float*, int, int, int, int32_t*, float*, cudaStream_t);
int router_proj(const uint16_t*, const uint16_t*, int, int, int, float*, cudaStream_t);
int router_bwd(const int32_t*, const float*, const float*, int, int, int, float*, cudaStream_t);
int router_proj_bwd(const uint16_t*, const float*, int, int, int, uint16_t*, cudaStream_t);
size_t permute_scratch_bytes(int T, int E);
int permute_rows(const uint16_t*, const int32_t*, int, int, int, int, int32_t*, int32_t*, int32_t*,
                 int32_t*, uint16_t*, int32_t*, int32_t*, cudaStream_t, uint8_t* = nullptr,
                 uint8_t* = nullptr);
int combine(const uint16_t*, const int32_t*, const float*, int, int, int, uint16_t*, cudaStream_t);
int combine_bwd(const uint16_t*, const uint16_t*, const int32_t*, const float*, int, int, int,
                uint16_t*, float*, cudaStream_t);
int unpermute_sum(const uint16_t*, const int32_t*, int, int, int, const float*, const uint16_t*,
                  int, uint16_t*, cudaStream_t);
int swiglu(const uint16_t*, uint16_t*, int64_t, int, cudaStream_t);
size_t balance_scratch_bytes(int T, int E);
int router_balance(const float*, const int32_t*, int, int, int, float*, float*, float*, cudaStream_t);
int router_balance_bwd(const float*, const int32_t*, int, int, int, float, float*, cudaStream_t);
int swiglu_bwd(const uint16_t*, const uint16_t*, uint16_t*, int64_t, int, cudaStream_t);
int grouped_gemm(const moe_gg_args*, cudaStream_t);
size_t grouped_gemm_workspace_bytes(const moe_gg_args*);
int mxfp8_quantize_impl(const uint16_t*, int64_t, int64_t, int, const int32_t*, int, uint8_t*,
                        uint8_t*, int32_t*, cudaStream_t);
int mxfp8_quantize_rowcol_impl(const uint16_t*, int64_t, int64_t, const int32_t*, int, uint8_t*,
                               uint8_t*, uint8_t*, uint8_t*, int32_t*, cudaStream_t);
size_t layer_workspace_bytes(const moe_layer_desc*);
int layer_fwd(const moe_layer_desc*, const moe_layer_params*, const moe_layer_saved*, uint16_t*,
              void*, size_t, cudaStream_t);
int layer_bwd(const moe_layer_desc*, const moe_layer_params*, const moe_layer_saved*,
              const uint16_t*, const moe_layer_grads*, void*, size_t, cudaStream_t);

static std::atomic<uint64_t> g_launches{0};
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

int num_sms() {
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        cache[dev] = n;
    }
    return cache[dev];
}

static bool ok_ptr(const void* p) { return p && aligned16(p); }

static bool ok_router_shape(int T, int E, int k) {
    return T >= 0 && E >= 1 && E <= 1024 && k >= 1 && k <= E && k <= 32 &&
           static_cast<int64_t>(T) * k < (1ll << 31);
}

}  // namespace moe

using namespace moe;

extern "C" {

const char* moe_status_string(int status) {
    switch (status) {
        case MOE_OK: return "MOE_OK";
        case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
        case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
        case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
        case MOE_ERR_DEVICE_TIMEOUT: return "MOE_ERR_DEVICE_TIMEOUT";
        case MOE_ERR_DEVICE_BOUNDS: return "MOE_ERR_DEVICE_BOUNDS";
        default: return "MOE_ERR_UNKNOWN";
    }
}

int moe_version(void) { return 100; }

uint64_t moe_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

int moe_read_device_status(const int32_t* device_status, int clear, int32_t* host_out,
                           void* stream) {
    if (!device_status || !host_out) return MOE_ERR_INVALID_ARG;
    cudaStream_t st = as_stream(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaMemcpy(host_out, device_status, sizeof(int32_t), cudaMemcpyDeviceToHost) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (clear && cudaMemset(const_cast<int32_t*>(device_status), 0, sizeof(int32_t)) != cudaSuccess)
        return MOE_ERR_CUDA;
    return MOE_OK;
}

int moe_router_topk(const float* logits, int T, int E, int k, int32_t* topk_idx, float* topk_w,
                    void* stream) {
    MOE_NVTX_RANGE();
    if (!ok_router_shape(T, E, k)) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!ok_ptr(logits) || !ok_ptr(topk_idx) || !ok_ptr(topk_w))) return MOE_ERR_INVALID_ARG;
    return router_topk(logits, T, E, k, topk_idx, topk_w, as_stream(stream));
}

int moe_router_topk_proj(const uint16_t* x, const uint16_t* w_r, int T, int d, int E, int k,
                         float* logits_out, int32_t* topk_idx, float* topk_w, void* stream) {
    MOE_NVTX_RANGE();
    if (!ok_router_shape(T, E, k) || d < 8 || d % 8) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!ok_ptr(x) || !ok_ptr(w_r) || !ok_ptr(logits_out) || !ok_ptr(topk_idx) ||
                  !ok_ptr(topk_w)))
        return MOE_ERR_INVALID_ARG;
    MOE_TRY(router_proj(x, w_r, T, d, E, logits_out, as_stream(stream)));
    return router_topk(logits_out, T, E, k, topk_idx, topk_w, as_stream(stream));
}

int moe_router_bwd(const int32_t* topk_idx, const float* topk_w, const float* dw, int T, int E,
                   int k, float* d_logits, void* stream) {
    MOE_NVTX_RANGE();
    if (!ok_router_shape(T, E, k)) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!ok_ptr(topk_idx) || !ok_ptr(topk_w) || !ok_ptr(dw) || !ok_ptr(d_logits)))
        return MOE_ERR_INVALID_ARG;
    return router_bwd(topk_idx, topk_w, dw, T, E, k, d_logits, as_stream(stream));
}

int moe_router_proj_bwd(const uint16_t* x, const float* d_logits, int T, int d, int E,
                        uint16_t* dw_r, void* stream) {
    MOE_NVTX_RANGE();
    if (T < 0 || d < 8 || d % 8 || E < 1 || E > 1024) return MOE_ERR_INVALID_ARG;
    if (!ok_ptr(dw_r) || (T > 0 && (!ok_ptr(x) || !ok_ptr(d_logits)))) return MOE_ERR_INVALID_ARG;
    return router_proj_bwd(x, d_logits, T, d, E, dw_r, as_stream(stream));
}

size_t moe_router_balance_workspace_bytes(int T, int E) {
    if (T < 0 || E < 1) return 0;
    return balance_scratch_bytes(T > 0 ? T : 1, E);
}

int moe_router_balance(const float* logits, const int32_t* counts, int T, int E, int k,
                       float* stats, float* probs_mean, void* workspace, size_t workspace_bytes,
                       void* stream) {
    MOE_NVTX_RANGE();
    if (!ok_router_shape(T, E, k)) return MOE_ERR_INVALID_ARG;
    if (!ok_ptr(counts) || !ok_ptr(stats) || !ok_ptr(workspace)) return MOE_ERR_INVALID_ARG;
    if (T > 0 && !ok_ptr(logits)) return MOE_ERR_INVALID_ARG;
    if (probs_mean && !ok_ptr(probs_mean)) return MOE_ERR_INVALID_ARG;
    if (workspace_bytes < moe_router_balance_workspace_bytes(T, E)) return MOE_ERR_INVALID_ARG;
    return router_balance(logits, counts, T, E, k, stats, probs_mean,
                          static_cast<float*>(workspace), as_stream(stream));
}

int moe_router_balance_bwd(const float* logits, const int32_t* counts, int T, int E, int k,
                           float scale, float* d_logits, void* stream) {
    MOE_NVTX_RANGE();
    if (!ok_router_shape(T, E, k)) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!ok_ptr(logits) || !ok_ptr(counts) || !ok_ptr(d_logits))) return MOE_ERR_INVALID_ARG;
    return router_balance_bwd(logits, counts, T, E, k, scale, d_logits, as_stream(stream));
}

size_t moe_permute_workspace_bytes(int T, int E) {
    if (T < 0 || E < 1) return 0;
    return 256 + permute_scratch_bytes(T, E);
}

int moe_permute_rows(const uint16_t* x, const int32_t* topk_idx, int T, int d, int E, int k,
                     int32_t* counts, int32_t* offsets, int32_t* dest_pos, int32_t* src_token,
                     uint16_t* x_perm, void* workspace, size_t workspace_bytes, void* stream) {
    MOE_NVTX_RANGE();
    if (!ok_router_shape(T, E, k) || d < 8 || d % 8) return MOE_ERR_INVALID_ARG;
    if (!ok_ptr(counts) || !ok_ptr(offsets) || !ok_ptr(workspace)) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!ok_ptr(x) || !ok_ptr(topk_idx) || !ok_ptr(dest_pos) || !ok_ptr(src_token) ||
                  !ok_ptr(x_perm)))
        return MOE_ERR_INVALID_ARG;
    if (workspace_bytes < moe_permute_workspace_bytes(T, E)) return MOE_ERR_INVALID_ARG;
    uint8_t* w = static_cast<uint8_t*>(workspace);
    return permute_rows(x, topk_idx, T, d, E, k, counts, offsets, dest_pos, src_token, x_perm,
                        reinterpret_cast<int32_t*>(w + 256), reinterpret_cast<int32_t*>(w),
                        as_stream(stream));
}

int moe_permute_rows_mxfp8(const uint16_t* x, const int32_t* topk_idx, int T, int d, int E, int k,
                           int32_t* counts, int32_t* offsets, int32_t* dest_pos,
                           int32_t* src_token, uint16_t* x_perm, uint8_t* x_perm_codes,
                           uint8_t* x_perm_scales, void* workspace, size_t workspace_bytes,
                           void* stream) {
    MOE_NVTX_RANGE();
    if (!ok_router_shape(T, E, k) || d < 32 || d % 32) return MOE_ERR_INVALID_ARG;
    if (!ok_ptr(counts) || !ok_ptr(offsets) || !ok_ptr(workspace)) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!ok_ptr(x) || !ok_ptr(topk_idx) || !ok_ptr(dest_pos) || !ok_ptr(src_token) ||
                  !ok_ptr(x_perm) || !ok_ptr(x_perm_codes) || !ok_ptr(x_perm_scales)))
        return MOE_ERR_INVALID_ARG;
    if (workspace_bytes < moe_permute_workspace_bytes(T, E)) return MOE_ERR_INVALID_ARG;
    uint8_t* w = static_cast<uint8_t*>(workspace);
    return permute_rows(x, topk_idx, T, d, E, k, counts, offsets, dest_pos, src_token, x_perm,
                        reinterpret_cast<int32_t*>(w + 256), reinterpret_cast<int32_t*>(w),
                        as_stream(stream), x_perm_codes, x_perm_scales);
}

size_t moe_grouped_gemm_workspace_bytes(const moe_gg_args* args) {
    return grouped_gemm_workspace_bytes(args);
}

int moe_grouped_gemm(const moe_gg_args* args, void* stream) {
    MOE_NVTX_RANGE();
    if (!args) return MOE_ERR_INVALID_ARG;
    return grouped_gemm(args, as_stream(stream));
}

int moe_swiglu(const uint16_t* gu, uint16_t* a, int64_t M, int f, void* stream) {
    MOE_NVTX_RANGE();
    if (M < 0 || f < 8 || f % 8) return MOE_ERR_INVALID_ARG;
    if (M > 0 && (!ok_ptr(gu) || !ok_ptr(a))) return MOE_ERR_INVALID_ARG;
    return swiglu(gu, a, M, f, as_stream(stream));
}

int moe_swiglu_bwd(const uint16_t* gu, const uint16_t* da, uint16_t* dh, int64_t M, int f,
                   void* stream) {
    MOE_NVTX_RANGE();
    if (M < 0 || f < 8 || f % 8) return MOE_ERR_INVALID_ARG;
    if (M > 0 && (!ok_ptr(gu) || !ok_ptr(da) || !ok_ptr(dh))) return MOE_ERR_INVALID_ARG;
    return swiglu_bwd(gu, da, dh, M, f, as_stream(stream));
}

int moe_unpermute_combine(const uint16_t* y_perm, const int32_t* dest_pos, const float* topk_w,
                          int T, int d, int k, uint16_t* out, void* stream) {
    MOE_NVTX_RANGE();
    if (T < 0 || d < 8 || d % 8 || k < 1 || k > 32) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!ok_ptr(y_perm) || !ok_ptr(dest_pos) || !ok_ptr(topk_w) || !ok_ptr(out)))
        return MOE_ERR_INVALID_ARG;
    return combine(y_perm, dest_pos, topk_w, T, d, k, out, as_stream(stream));
}

int moe_unpermute_combine_bwd(const uint16_t* dout, const uint16_t* y_perm,
                              const int32_t* dest_pos, const float* topk_w, int T, int d, int k,
                              uint16_t* dy_perm, float* dw, void* stream) {
    MOE_NVTX_RANGE();
    if (T < 0 || d < 8 || d % 8 || k < 1 || k > 32) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!ok_ptr(dout) || !ok_ptr(y_perm) || !ok_ptr(dest_pos) || !ok_ptr(topk_w) ||
                  !ok_ptr(dy_perm) || !ok_ptr(dw)))
        return MOE_ERR_INVALID_ARG;
    return combine_bwd(dout, y_perm, dest_pos, topk_w, T, d, k, dy_perm, dw, as_stream(stream));
}

int moe_unpermute_sum(const uint16_t* dx_perm, const int32_t* dest_pos, int T, int d, int k,
                      const float* d_logits, const uint16_t* w_r, int E, uint16_t* dx,
                      void* stream) {
    MOE_NVTX_RANGE();
    if (T < 0 || d < 8 || d % 8 || k < 1 || k > 32) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!ok_ptr(dx_perm) || !ok_ptr(dest_pos) || !ok_ptr(dx))) return MOE_ERR_INVALID_ARG;
    if (d_logits && w_r && (E < 1 || E > 1024)) return MOE_ERR_INVALID_ARG;
    return unpermute_sum(dx_perm, dest_pos, T, d, k, d_logits, w_r, E, dx, as_stream(stream));
}

int mxfp8_quantize(const uint16_t* x, int64_t rows, int64_t cols, int axis,
                   const int32_t* group_offsets, int ngroups, uint8_t* codes, uint8_t* scales,
                   uint8_t* hw_scales, void* stream) {
    MOE_NVTX_RANGE();
    if (rows < 0 || rows >= (1ll << 31) || cols < 32 || cols % 32) return MOE_ERR_INVALID_ARG;
    if (axis != 0 && axis != 1) return MOE_ERR_INVALID_ARG;
    if (hw_scales) return MOE_ERR_UNSUPPORTED;
    if (axis == 0 && group_offsets && (ngroups < 1 || ngroups > 1024)) return MOE_ERR_INVALID_ARG;
    if (rows > 0 && (!ok_ptr(x) || !ok_ptr(codes) || !ok_ptr(scales))) return MOE_ERR_INVALID_ARG;
    return mxfp8_quantize_impl(x, rows, cols, axis, group_offsets, ngroups, codes, scales, nullptr,
                               as_stream(stream));
}

int mxfp8_quantize_rowcol(const uint16_t* x, int64_t rows, int64_t cols,
                          const int32_t* group_offsets, int ngroups, uint8_t* row_codes,
                          uint8_t* row_scales, uint8_t* col_codes, uint8_t* col_scales,
                          void* stream) {
    MOE_NVTX_RANGE();
    if (rows < 0 || rows >= (1ll << 31) || cols < 32 || cols % 32) return MOE_ERR_INVALID_ARG;
    if (group_offsets && (ngroups < 1 || ngroups > 1024)) return MOE_ERR_INVALID_ARG;
    if (rows > 0 && (!ok_ptr(x) || !ok_ptr(row_codes) || !ok_ptr(row_scales) ||
                     !ok_ptr(col_codes) || !ok_ptr(col_scales)))
        return MOE_ERR_INVALID_ARG;
    return mxfp8_quantize_rowcol_impl(x, rows, cols, group_offsets, ngroups, row_codes, row_scales,
                                      col_codes, col_scales, nullptr, as_stream(stream));
}

size_t moe_layer_workspace_bytes(const moe_layer_desc* desc) { return layer_workspace_bytes(desc); }

int moe_layer_fwd(const moe_layer_desc* desc, const moe_layer_params* params,
                  const moe_layer_saved* saved, uint16_t* out, void* workspace,
                  size_t workspace_bytes, void* stream) {
    MOE_NVTX_RANGE();
    return layer_fwd(desc, params, saved, out, workspace, workspace_bytes, as_stream(stream));
}

int moe_layer_bwd(const moe_layer_desc* desc, const moe_layer_params* params,
                  const moe_layer_saved* saved, const uint16_t* dout,
                  const moe_layer_grads* grads, void* workspace, size_t workspace_bytes,
                  void* stream) {
    MOE_NVTX_RANGE();
    return layer_bwd(desc, params, saved, dout, grads, workspace, workspace_bytes,
                     as_stream(stream));
}

}  // extern "C"
