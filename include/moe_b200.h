/*
 * moe_b200.h -- C ABI of a single-GPU MoE expert layer for NVIDIA B200 (sm_100a).
 *
 * The layer is the expert block of a mixture-of-experts transformer as
 * described in "Ai2 rebuilds Olmo's training stack for trillion-parameter
 * MoEs" (alphasignal.ai; introduction, "Routing work stays on the GPU",
 * "MXFP8 reduces compute and memory costs") and "Supercharging Olmo-core for
 * Efficient and Scalable MoE Training" (papers.projxon.ai; Summary):
 *
 *   router top-k -> rowwise dispatch into contiguous per-expert buffers ->
 *   SwiGLU expert FFNs as device-scheduled grouped GEMMs -> weighted combine,
 *   forward and backward, with an optional MXFP8 (E4M3, 1x32 blocks, E8M0
 *   scales) grouped-GEMM path.
 *
 * Conventions for every entry point
 * ---------------------------------
 *  - Pointers named as device buffers are CUDA device pointers; they must be
 *    16-byte aligned.  Host pointers are marked "host".
 *  - bf16 tensors are passed as uint16_t bit patterns; all tensors are dense
 *    row-major with the stated shapes.
 *  - Every call is asynchronous on `stream` (a cudaStream_t, NULL = legacy
 *    default stream).  The library never allocates, frees or synchronises,
 *    except moe_read_device_status, which is a documented sync point.
 *  - Routing metadata (counts, offsets, row positions) stays in device memory;
 *    kernels read it there and no count is ever copied to the host.
 *  - Return value: a moe_status.  Host-side validation happens before any
 *    launch; on an error nothing is launched.  Failures detected on the device
 *    (an out-of-range expert index, a pipeline wait that exceeded its time
 *    limit) are OR-ed into a caller-owned int32 device status word (bit
 *    values = 1 << moe_status), read back with moe_read_device_status.
 *  - Buffers the caller passes are owned by the caller.  The library keeps no
 *    state between calls other than a per-process cache of kernel attributes.
 *  - Shapes: T tokens, d model width, E experts, k experts per token,
 *    f expert hidden width, M = T*k routed rows.  Limits: 1 <= k <= E <= 1024,
 *    k <= 32, M < 2^31, d % 8 == 0, f % 8 == 0 (MXFP8: d % 32 == 0 and
 *    f % 32 == 0).
 *  - Weights use the out x in convention: W13 [E, 2f, d] holds the gate W1 in
 *    rows 0..f-1 and the up projection W3 in rows f..2f-1; W2 [E, d, f];
 *    router projection W_r [d, E].
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum moe_status {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,    /* null / misaligned pointer, bad shape */
    MOE_ERR_UNSUPPORTED = 2,    /* valid request the library does not implement */
    MOE_ERR_CUDA = 3,           /* a CUDA runtime / driver call failed */
    MOE_ERR_DEVICE_TIMEOUT = 4, /* a device-side wait exceeded its time limit */
    MOE_ERR_DEVICE_BOUNDS = 5   /* a device-side index was out of range */
} moe_status;

typedef enum moe_dtype { MOE_DTYPE_BF16 = 0, MOE_DTYPE_MXFP8 = 1 } moe_dtype;

/* Human-readable name of a status code (static storage). */
const char* moe_status_string(int status);

/* Library ABI version (major * 100 + minor). */
int moe_version(void);

/* Number of kernels this library has launched in this process (all devices,
 * all streams); a monotonically increasing counter for launch accounting. */
uint64_t moe_kernel_launches(void);

/* Reads the device status word `device_status` (int32, device) after
 * synchronising `stream`; writes it to *host_out and, if `clear` != 0, resets
 * it to zero.  This is the library's only synchronising call; it is never
 * called from inside another entry point. */
int moe_read_device_status(const int32_t* device_status, int clear, int32_t* host_out,
                           void* stream);

/* Diagnostic of the device-side failure detection: runs the library's bounded
 * pipeline wait on an mbarrier nothing arrives on.  The wait must give up after
 * limit_ns nanoseconds of global time (1e3 .. 1e10) and OR 1 << MOE_ERR_DEVICE_TIMEOUT
 * into device_status (int32, device); the time actually waited is written to
 * device_elapsed_ns (uint64, device, may be NULL).  No fault, no hang: the
 * context stays usable.  The pages have no counterpart (library diagnostics).  */
int moe_selftest_bounded_wait(int32_t* device_status, uint64_t limit_ns,
                              uint64_t* device_elapsed_ns, void* stream);

/* ------------------------------------------------------------------------ *
 * Router (introduction of the alphasignal.ai page: a router sends each token
 * to a small selection of experts; Summary of the projxon page: 4 experts per
 * token).  Reading taken: softmax over E, keep the k largest, renormalise.
 * ------------------------------------------------------------------------ */

/* topk_idx[t, i], i < k: experts ordered by fp32 logit descending, equal
 * values (+0 == -0) to the lower index.  topk_w[t, i] =
 * exp(l_i - l_max) / sum_{j in top-k} exp(l_j - l_max) in fp32.
 *   logits   device fp32 [T, E]        (NaN / Inf are outside the contract)
 *   topk_idx device int32 [T, k]  (out)
 *   topk_w   device fp32 [T, k]   (out)                                     */
int moe_router_topk(const float* logits, int T, int E, int k, int32_t* topk_idx,
                    float* topk_w, void* stream);

/* Same, with the logits computed first as logits = x W_r (bf16 inputs, fp32
 * accumulation), written to logits_out (device fp32 [T, E]).
 *   x device bf16 [T, d], w_r device bf16 [d, E]                           */
int moe_router_topk_proj(const uint16_t* x, const uint16_t* w_r, int T, int d, int E, int k,
                         float* logits_out, int32_t* topk_idx, float* topk_w, void* stream);

/* Router backward (softmax over the selected logits):
 *   d_logits[t, topk_idx[t, j]] = w_j (dw_j - sum_i w_i dw_i), zero elsewhere.
 *   dw device fp32 [T, k]; d_logits device fp32 [T, E] (out, fully written). */
int moe_router_bwd(const int32_t* topk_idx, const float* topk_w, const float* dw, int T, int E,
                   int k, float* d_logits, void* stream);

/* Router projection backward: dw_r = x^T d_logits (bf16 out, fp32 accumulation).
 *   x device bf16 [T, d], d_logits device fp32 [T, E], dw_r device bf16 [d, E] */
int moe_router_proj_bwd(const uint16_t* x, const float* d_logits, int T, int d, int E,
                        uint16_t* dw_r, void* stream);

/* Routing balance ("Four failure modes from the report", first bullet of the
 * alphasignal.ai page: a routing-balance score can improve while the actual
 * load gets less balanced -- "token gerrymandering").  Reading (no formula on
 * the pages): the auxiliary balance loss L = E * sum_e f_e P_e with
 * f_e = counts[e] / (T k) and P_e = mean_t softmax(logits[t])_e, next to the
 * actual imbalance of the counts.
 *   stats (device fp32 [4], out): L, max_e counts / mean counts, coefficient of
 *          variation of counts, fraction of experts with no token.
 *   probs_mean (device fp32 [E], out, may be NULL): P.
 *   workspace: device scratch of moe_router_balance_workspace_bytes(T, E).    */
size_t moe_router_balance_workspace_bytes(int T, int E);
int moe_router_balance(const float* logits, const int32_t* counts, int T, int E, int k,
                       float* stats, float* probs_mean, void* workspace, size_t workspace_bytes,
                       void* stream);
/* Gradient of scale * L with the counts held fixed, ADDED into d_logits:
 *   d_logits[t, j] += scale * (E / T) * p_tj * (f_j - sum_e f_e p_te).       */
int moe_router_balance_bwd(const float* logits, const int32_t* counts, int T, int E, int k,
                           float scale, float* d_logits, void* stream);

/* ------------------------------------------------------------------------ *
 * Rowwise dispatch ("Routing work stays on the GPU": routed token rows are
 * written directly into expert input buffers; routing metadata stays on the
 * device).
 * ------------------------------------------------------------------------ */

/* Device scratch needed by moe_permute_rows (bytes). */
size_t moe_permute_workspace_bytes(int T, int E);

/* counts[e]   = number of (t, i) with topk_idx[t, i] == e          (int32 [E])
 * offsets     = exclusive prefix sum of counts, offsets[E] = T*k    (int32 [E+1])
 * dest_pos[t, i] = offsets[e] + #{t' < t : e in top-k(t')}          (int32 [T, k])
 * src_token[dest_pos[t, i]] = t                                     (int32 [T*k])
 * x_perm[dest_pos[t, i], :] = x[t, :]                               (bf16 [T*k, d])
 * Rows inside an expert are in ascending token order (deterministic).
 * `workspace` (device, >= moe_permute_workspace_bytes) is scratch; its first
 * int32 is the device status word (MOE_ERR_DEVICE_BOUNDS on an expert index
 * outside [0, E), whose row is then skipped).  A token must not list the same
 * expert twice.                                                             */
int moe_permute_rows(const uint16_t* x, const int32_t* topk_idx, int T, int d, int E, int k,
                     int32_t* counts, int32_t* offsets, int32_t* dest_pos, int32_t* src_token,
                     uint16_t* x_perm, void* workspace, size_t workspace_bytes, void* stream);

/* moe_permute_rows for an MXFP8 GEMM1 ("MXFP8 reduces compute and memory
 * costs": the routed rows are GEMM1's K-contiguous operand): the dispatch
 * also writes the row-wise MXFP8 encoding of every routed row, so that no
 * separate pass reads x_perm to quantise it.
 *   x_perm_codes  uint8 [T*k, d]        E4M3 codes, x_perm_codes[r, c] of x_perm[r, c]
 *   x_perm_scales uint8 [T*k, d / 32]   E8M0 scale byte of each 32-value block of a row
 * Byte for byte what mxfp8_quantize(x_perm, axis = 1) writes (same rule).
 * d % 32 == 0; both pointers non-NULL and 16-byte aligned; everything else as
 * moe_permute_rows.  Each token is encoded once and its codes stored to all
 * of its k rows.                                                            */
int moe_permute_rows_mxfp8(const uint16_t* x, const int32_t* topk_idx, int T, int d, int E, int k,
                           int32_t* counts, int32_t* offsets, int32_t* dest_pos,
                           int32_t* src_token, uint16_t* x_perm, uint8_t* x_perm_codes,
                           uint8_t* x_perm_scales, void* workspace, size_t workspace_bytes,
                           void* stream);

/* Allocation-free variant of moe_permute_rows (no counterpart in the source
 * pages; it exists for callers, not for the method).  Same arguments and
 * results, minus the workspace: for callers that cannot allocate device
 * memory at the point of the call -- e.g. a plugin inside a host that already
 * reserved all device memory for its own pool, or a runtime that forbids
 * cudaMalloc after start-up because it can synchronise the device.
 *   - Scratch comes from a fixed 1 MiB array inside the library (held on
 *     every GPU that loads the library until the process exits).  Limit:
 *     ceil(T / 128) * E <= 262144, else MOE_ERR_INVALID_ARG.
 *   - The first call on a device looks up that array's device address
 *     (cudaGetSymbolAddress, with the device current); make that first call
 *     before any stream capture.  The address is cached for the process and
 *     belongs to the device's primary context (the runtime's): do not call
 *     this from another context, or after cudaDeviceReset.
 *   - The call allocates nothing (no cudaMalloc / cudaFree / allocating
 *     library routine).
 *   - All calls share the one array and it keeps the last call's contents:
 *     calls that can overlap on the GPU (other streams, other host threads
 *     on the same device) race and must be serialised by the caller.
 *   - No status word: an expert index outside [0, E) is skipped and its
 *     dest_pos is -1.                                                       */
int moe_permute_rows_noalloc(const uint16_t* x, const int32_t* topk_idx, int T, int d, int E,
                             int k, int32_t* counts, int32_t* offsets, int32_t* dest_pos,
                             int32_t* src_token, uint16_t* x_perm, void* stream);

/* ------------------------------------------------------------------------ *
 * Device-scheduled grouped GEMM ("Routing work stays on the GPU", third
 * bullet; projxon Summary).  One persistent launch covers all experts; the
 * tile scheduler reads `offsets` from device memory.  tcgen05 tensor cores,
 * TMA-fed shared-memory pipeline, TMEM accumulators.
 * ------------------------------------------------------------------------ */

typedef enum moe_gg_mode {
    /* For each expert e, rows R_e = [offsets[e], offsets[e+1]):
     *   C[R_e, 0:N] = A[R_e, 0:K] . B_e^T
     * A  [M_total, K] (K contiguous).
     * B  per expert [N, K]: stored [E][N][K] (b_mn_major = 0) or [E][K][N]
     *    (b_mn_major = 1).
     * C  [M_total, N].  Rows of C outside every group are not written. */
    MOE_GG_RAGGED_M = 0,
    /* For each expert e:
     *   C_e[0:M, 0:N] = A[R_e, 0:M]^T . B[R_e, 0:N]
     * A [M_total, M], B [M_total, N] (row-major, so both are MN-major),
     * C [E][M][N].  An expert with no rows gets C_e = 0 exactly.            */
    MOE_GG_RAGGED_K = 1
} moe_gg_mode;

typedef enum moe_gg_epilogue {
    MOE_EPI_NONE = 0,
    /* RAGGED_M, N = 2f: the product's columns [0, f) are G and [f, 2f) are U.
     * C receives [G | U] (bf16) and aux = A = silu(G) * U (bf16 [M_total, f]),
     * computed from the fp32 accumulators.                                 */
    MOE_EPI_SWIGLU = 1,
    /* RAGGED_M, N = f: the product is dA.  gu = saved [G | U] (bf16
     * [M_total, 2f]).  C receives dH = [dG | dU] (bf16 [M_total, 2f]) with
     * s = sigmoid(G): dG = dA U s (1 + G (1 - s)), dU = dA silu(G).          */
    MOE_EPI_SWIGLU_BWD = 2
} moe_gg_epilogue;

typedef struct moe_gg_args {
    int mode;               /* moe_gg_mode */
    int dtype;              /* MOE_DTYPE_BF16 (MXFP8 operands: see mxfp8 below) */
    int epilogue;           /* moe_gg_epilogue */
    int E;                  /* number of groups */
    int64_t M_total;        /* rows of the routed buffers (= offsets[E]) */
    int M;                  /* RAGGED_K: output rows per expert; unused for RAGGED_M */
    int N;                  /* output columns */
    int K;                  /* RAGGED_M: reduction width; unused for RAGGED_K */
    const int32_t* offsets; /* device int32 [E+1], nondecreasing, offsets[0] = 0;
                             * values out of [0, M_total] or going down set
                             * MOE_ERR_DEVICE_BOUNDS in *status (MXFP8 scale
                             * tables use the clamped running maximum)     */
    const void* a;          /* device bf16, layout per mode */
    const void* b;          /* device bf16, layout per mode */
    int b_mn_major;         /* RAGGED_M only */
    void* c;                /* device bf16 output */
    void* aux;              /* SWIGLU: A out [M_total, f] */
    const void* gu;         /* SWIGLU_BWD: [G | U] in [M_total, 2f] */
    /* MXFP8 (dtype == MOE_DTYPE_MXFP8): a and b hold E4M3 codes in the same
     * layouts as the bf16 operands, blocks of 32 along the reduction axis, and
     * a_scales / b_scales their E8M0 scales as mxfp8_quantize writes them:
     *   RAGGED_M A: row-wise, [M_total][K/32].
     *   RAGGED_M B, b_mn_major = 0: row-wise over [E*N][K], i.e. [E*N][K/32].
     *   RAGGED_M B, b_mn_major = 1: column-wise over [E*K][N] with K % 32 == 0
     *              (one block run per expert), i.e. [E*K/32][N].
     *   RAGGED_K A / B: column-wise per expert group (group_offsets =
     *              offsets), i.e. [blocks][M] and [blocks][N].
     * K, N (and M) must be multiples of 32. */
    const uint8_t* a_scales;
    const uint8_t* b_scales;
    /* Device scratch of moe_grouped_gemm_workspace_bytes bytes.  MXFP8
     * (required): the scales rearranged per tile for the tensor cores.  BF16
     * RAGGED_K (optional, 128-byte aligned): per-expert copies of the operand
     * tensor maps whose row extent ends at the expert's last row, so that the
     * last K tile's rows of the next expert arrive as zeros; without it the
     * kernel zeroes those rows in shared memory (slower).  Otherwise unused. */
    void* workspace;
    size_t workspace_bytes;
    int32_t* status;        /* device status word (may be NULL) */
    /* Optional MXFP8 quantisation of the epilogue's bf16 output, for a
     * following MXFP8 GEMM ("MXFP8 reduces compute and memory costs"): the
     * output is SWIGLU: A [M_total, W = f]; SWIGLU_BWD: dH [M_total, W = 2f].
     * Codes and scales equal what mxfp8_quantize writes for that bf16 tensor:
     *   q_row_codes / q_row_scales: axis = 1, [M_total][W] and [M_total][W/32];
     *   q_col_codes / q_col_scales: axis = 0 with group_offsets = offsets,
     *              [M_total][W] and [blocks][W].
     * Either pair may be NULL (not produced).  Requires W % 32 == 0 and the
     * SWIGLU or SWIGLU_BWD epilogue; 16-byte aligned device buffers.  Where
     * the chosen kernel cannot quantise in its epilogue, the call quantises
     * the stored output right after the GEMM on the same stream. */
    void* q_row_codes;
    void* q_row_scales;
    void* q_col_codes;
    void* q_col_scales;
} moe_gg_args;

/* Device scratch moe_grouped_gemm uses for these arguments (see workspace;
 * 0 for BF16 RAGGED_M). */
size_t moe_grouped_gemm_workspace_bytes(const moe_gg_args* args);

/* The persistent CTAs of a grouped GEMM keep within one tile of each other
 * through a counter pair in the library's device memory (64 pairs per GPU,
 * taken in turn by the calls, each zeroed by the last CTA of its call).  A
 * wait on the others is bounded (50 us per tile, then the CTA stops
 * waiting): more than 64 grouped GEMMs running at once on one GPU, or CTAs
 * that cannot all be resident, cost speed, never a result or an error.
 * MOE_GG_SYNC_SLACK=0 in the environment turns it off. */
int moe_grouped_gemm(const moe_gg_args* args, void* stream);

/* Standalone SwiGLU (the fused epilogues, for testing):
 *   a[r, j] = silu(g) * u with g = gu[r, j], u = gu[r, f + j]     (bf16)
 * and its backward, dh = [dG | dU] from da [M, f] and gu.                  */
int moe_swiglu(const uint16_t* gu, uint16_t* a, int64_t M, int f, void* stream);
int moe_swiglu_bwd(const uint16_t* gu, const uint16_t* da, uint16_t* dh, int64_t M, int f,
                   void* stream);

/* ------------------------------------------------------------------------ *
 * Weighted unpermute / combine and their backward.
 * ------------------------------------------------------------------------ */

/* out[t] = sum_{i<k} topk_w[t, i] * y_perm[dest_pos[t, i]]  (fp32 sum in slot
 * order, one bf16 rounding).  y_perm bf16 [T*k, d], out bf16 [T, d].       */
int moe_unpermute_combine(const uint16_t* y_perm, const int32_t* dest_pos, const float* topk_w,
                          int T, int d, int k, uint16_t* out, void* stream);

/* dy_perm[dest_pos[t, i]] = bf16(topk_w[t, i] * dout[t]);
 * dw[t, i] = sum_c dout[t, c] * y_perm[dest_pos[t, i], c]   (fp32).          */
int moe_unpermute_combine_bwd(const uint16_t* dout, const uint16_t* y_perm,
                              const int32_t* dest_pos, const float* topk_w, int T, int d, int k,
                              uint16_t* dy_perm, float* dw, void* stream);

/* dx[t] = sum_i dx_perm[dest_pos[t, i]] (+ sum_e d_logits[t, e] w_r[:, e] when
 * d_logits and w_r are both non-NULL; E is then their width).  bf16 out.    */
int moe_unpermute_sum(const uint16_t* dx_perm, const int32_t* dest_pos, int T, int d, int k,
                      const float* d_logits, const uint16_t* w_r, int E, uint16_t* dx,
                      void* stream);

/* ------------------------------------------------------------------------ *
 * MXFP8 block quantisation ("MXFP8 reduces compute and memory costs":
 * separate scaling for small blocks), OCP MX v1.0 rule: per block of 32
 * values X = clamp(floor(log2(amax)) - 8, -127, 127) (X = 0 for an all-zero
 * block), scale byte = X + 127, code = E4M3 round-to-nearest-even of
 * v / 2^X with saturation to +-448.
 * ------------------------------------------------------------------------ */

/* x device bf16 [rows, cols].  codes (out) uint8 [rows, cols], same layout.
 * axis = 1: blocks of 32 along a row; scales uint8 [rows, cols/32]
 *           (cols % 32 == 0).
 * axis = 0: blocks of 32 down a column, restarting at every group start
 *           group_offsets[g] (device int32 [ngroups+1]; NULL = one group);
 *           the last block of a group holds its remaining rows.  scales uint8
 *           [rows/32 + ngroups, cols]; the block of row r in group g is
 *           base[g] + (r - group_offsets[g]) / 32 with
 *           base[g] = sum_{g' < g} ceil(m_g' / 32).
 *           group_offsets must be non-decreasing with values in [0, rows].
 *           Other values are not an error of the call (it cannot read device
 *           memory): the kernel clamps them to [0, rows] and replaces each by
 *           the running maximum, so the groups never overlap and no scale
 *           row past rows/32 + ngroups is written.  (The grouped GEMM, which
 *           has a status word, also flags such offsets.)
 * hw_scales: reserved, must be NULL (the grouped GEMM rearranges the scales
 * itself).                                                                  */
int mxfp8_quantize(const uint16_t* x, int64_t rows, int64_t cols, int axis,
                   const int32_t* group_offsets, int ngroups, uint8_t* codes, uint8_t* scales,
                   uint8_t* hw_scales, void* stream);

/* Both encodings of x from one read of it: row_codes / row_scales as
 * mxfp8_quantize with axis = 1, col_codes / col_scales as axis = 0 with the
 * same group_offsets / ngroups.  Same argument rules; four separate
 * 16-byte aligned device outputs.                                          */
int mxfp8_quantize_rowcol(const uint16_t* x, int64_t rows, int64_t cols,
                          const int32_t* group_offsets, int ngroups, uint8_t* row_codes,
                          uint8_t* row_scales, uint8_t* col_codes, uint8_t* col_scales,
                          void* stream);

/* ------------------------------------------------------------------------ *
 * Whole layer, forward and backward.
 * ------------------------------------------------------------------------ */

typedef enum moe_router_mode {
    MOE_ROUTER_LOGITS = 0, /* fp32 logits are given */
    MOE_ROUTER_PROJ = 1    /* logits = x W_r computed by the layer */
} moe_router_mode;

#define MOE_FWD_STAGES 5 /* router, dispatch, GEMM1+SwiGLU, GEMM2, combine */
#define MOE_BWD_STAGES 8 /* recompute (GEMM1+SwiGLU again, recompute mode only),
                            combine-bwd, dA+SwiGLU-bwd, dW2, dX, dW13, router-bwd,
                            unpermute-sum (+ router projection backward) */

/* Bits of moe_layer_desc.mx_gemms: which grouped GEMMs take MXFP8 operands
 * when dtype == MOE_DTYPE_MXFP8 (0 = all six). */
#define MOE_MX_GEMM1 (1 << 0)
#define MOE_MX_GEMM2 (1 << 1)
#define MOE_MX_DA (1 << 2)
#define MOE_MX_DW2 (1 << 3)
#define MOE_MX_DX (1 << 4)
#define MOE_MX_DW13 (1 << 5)

typedef struct moe_layer_desc {
    int T, d, E, k, f;
    int dtype;        /* moe_dtype of the grouped GEMMs */
    int router_mode;  /* moe_router_mode */
    /* Per-layer activation recompute ("Supercharging Olmo-core ...", Summary:
     * activation recompute): when non-zero the forward keeps [G | U] and A
     * only in the workspace (saved->gu and saved->a may be NULL) and the
     * backward runs GEMM1 + SwiGLU again before its own GEMMs. */
    int recompute;
    /* Selective MXFP8 ("MXFP8 reduces compute and memory costs": selective
     * MXFP8 use): MOE_MX_* bits of the GEMMs that run in MXFP8 when dtype is
     * MOE_DTYPE_MXFP8; 0 selects all six.  The others run in BF16. */
    int mx_gemms;
    /* MXFP8 weights quantised once per step: when non-zero, moe_layer_fwd
     * reads each weight tensor once for both of its MXFP8 layouts (row-wise
     * for its forward GEMM, column-wise for its backward GEMM) and keeps the
     * column-wise one in the workspace; moe_layer_bwd then uses it instead of
     * quantising the weights again.  The backward must follow the forward of
     * the same step with the same weights and the same workspace. */
    int mx_keep_weights;
    /* Optional tracing: NULL, or an array of cudaEvent_t (created by the
     * caller) that the call records on `stream` at its stage boundaries --
     * MOE_FWD_STAGES + 1 events for moe_layer_fwd, MOE_BWD_STAGES + 1 for
     * moe_layer_bwd (event i before stage i, the last one after the last
     * stage).  Recording adds no synchronisation. */
    void* const* stage_events;
} moe_layer_desc;

typedef struct moe_layer_params {
    const uint16_t* x;     /* bf16 [T, d] */
    const float* logits;   /* fp32 [T, E] (LOGITS mode) */
    const uint16_t* w_r;   /* bf16 [d, E] (PROJ mode) */
    const uint16_t* w13;   /* bf16 [E, 2f, d] */
    const uint16_t* w2;    /* bf16 [E, d, f] */
} moe_layer_params;

/* Caller-owned buffers written by the forward and read by the backward. */
typedef struct moe_layer_saved {
    float* logits;         /* fp32 [T, E]: PROJ mode output (LOGITS mode: unused) */
    int32_t* topk_idx;     /* [T, k] */
    float* topk_w;         /* [T, k] */
    int32_t* counts;       /* [E] */
    int32_t* offsets;      /* [E+1] */
    int32_t* dest_pos;     /* [T, k] */
    int32_t* src_token;    /* [T*k] */
    uint16_t* x_perm;      /* bf16 [T*k, d] */
    uint16_t* gu;          /* bf16 [T*k, 2f]  (NULL allowed in recompute mode) */
    uint16_t* a;           /* bf16 [T*k, f]   (NULL allowed in recompute mode) */
    uint16_t* y_perm;      /* bf16 [T*k, d] */
} moe_layer_saved;

typedef struct moe_layer_grads {
    uint16_t* dx;          /* bf16 [T, d] */
    uint16_t* dw13;        /* bf16 [E, 2f, d] */
    uint16_t* dw2;         /* bf16 [E, d, f] */
    uint16_t* dw_r;        /* bf16 [d, E] (PROJ mode; else NULL) */
    float* d_logits;       /* fp32 [T, E] */
} moe_layer_grads;

/* Device workspace of moe_layer_fwd / moe_layer_bwd (bytes).  Its first
 * int32 is the device status word, which the caller zeroes once before use. */
size_t moe_layer_workspace_bytes(const moe_layer_desc* desc);

/* Forward: router -> dispatch -> GEMM1 + SwiGLU -> GEMM2 -> combine.  */
int moe_layer_fwd(const moe_layer_desc* desc, const moe_layer_params* params,
                  const moe_layer_saved* saved, uint16_t* out, void* workspace,
                  size_t workspace_bytes, void* stream);

/* Backward from dout (bf16 [T, d]) = dL/dout.  */
int moe_layer_bwd(const moe_layer_desc* desc, const moe_layer_params* params,
                  const moe_layer_saved* saved, const uint16_t* dout,
                  const moe_layer_grads* grads, void* workspace, size_t workspace_bytes,
                  void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
