// moe_permute_rows_noalloc: the rowwise dispatch of moe_permute_rows for
// callers that cannot hand the library a device workspace.
//
// Who needs it: code that has no device allocator it may call at this point --
// for example a plugin running inside a host framework that has already
// reserved all device memory for its own pool (a cudaMalloc there fails or
// fragments the pool), or a runtime that forbids allocation after start-up
// because cudaMalloc can synchronise the device.  Such callers still own and
// pass every input and output buffer; only the scratch space comes from here.
//
// The scratch (per-task expert histograms, then their per-expert prefix) lives
// in a file-scope __device__ array of fixed size, so every GPU that loads this
// library holds kScratchInts * 4 bytes (1 MiB) until the process exits.  In
// host code the array's name is only a host-side stand-in, never a device
// address: its device address is looked up once per device with
// cudaGetSymbolAddress while that device is current, and cached.
#include <mutex>

#include "common.cuh"
#include "nvtx_range.cuh"

namespace moe {

int permute_rows(const uint16_t*, const int32_t*, int, int, int, int, int32_t*, int32_t*, int32_t*,
                 int32_t*, uint16_t*, int32_t*, int32_t*, cudaStream_t, uint8_t* = nullptr,
                 uint8_t* = nullptr);
size_t permute_scratch_bytes(int T, int E);

namespace {

constexpr int64_t kScratchInts = 1 << 18;  // 262144 int32 = 1 MiB

__device__ __align__(256) int32_t g_noalloc_scratch[kScratchInts];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
int32_t* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up on the
// first call per device).  Returns nullptr on failure.  The cached address
// belongs to the device's primary context (the one the CUDA runtime uses); it
// is not valid in another context and does not survive cudaDeviceReset.
int32_t* scratch_on_current_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return nullptr;
        g_scratch_ptr[dev] = static_cast<int32_t*>(p);
    }
    return g_scratch_ptr[dev];
}

}  // namespace
}  // namespace moe

extern "C" int moe_permute_rows_noalloc(const uint16_t* x, const int32_t* topk_idx, int T, int d,
                                        int E, int k, int32_t* counts, int32_t* offsets,
                                        int32_t* dest_pos, int32_t* src_token, uint16_t* x_perm,
                                        void* stream) {
    MOE_NVTX_RANGE();
    using namespace moe;
    if (T < 0 || E < 1 || E > 1024 || k < 1 || k > E || k > 32 || d < 8 || d % 8 ||
        static_cast<int64_t>(T) * k >= (1ll << 31))
        return MOE_ERR_INVALID_ARG;
    // the dispatch's own scratch size for (T, E) must fit the fixed array
    if (permute_scratch_bytes(T, E) > sizeof(g_noalloc_scratch)) return MOE_ERR_INVALID_ARG;
    const void* outs[] = {counts, offsets};
    for (const void* q : outs)
        if (!q || !aligned16(q)) return MOE_ERR_INVALID_ARG;
    if (T > 0) {
        const void* ins[] = {x, topk_idx, dest_pos, src_token, x_perm};
        for (const void* q : ins)
            if (!q || !aligned16(q)) return MOE_ERR_INVALID_ARG;
    }
    int32_t* scratch = scratch_on_current_device();
    if (!scratch) return MOE_ERR_CUDA;
    // Every histogram entry the later kernels read is first written by the
    // count kernel of the same call, so stale contents from an earlier call
    // need no clearing.  No status word: an expert index outside [0, E) is
    // skipped and reported as dest_pos = -1.
    return permute_rows(x, topk_idx, T, d, E, k, counts, offsets, dest_pos, src_token, x_perm,
                        scratch, nullptr, as_stream(stream));
}
