// The whole expert layer, forward and backward, as one host function each that
// enqueues the kernels on the caller's stream.  Nothing is allocated and
// nothing is synchronised: every buffer is caller-owned, and routing metadata
// never leaves the device ("Routing work stays on the GPU": the CPU queues
// work without waiting for a copy back from the GPU).
//
// Options: MXFP8 operands for a chosen subset of the six grouped GEMMs
// ("MXFP8 reduces compute and memory costs": selective MXFP8 use) and
// per-layer activation recompute ("Supercharging Olmo-core ...", Summary).
#include "common.cuh"

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
int grouped_gemm(const moe_gg_args*, cudaStream_t);
size_t grouped_gemm_workspace_bytes(const moe_gg_args*);
int mxfp8_quantize_impl(const uint16_t*, int64_t, int64_t, int, const int32_t*, int, uint8_t*,
                        uint8_t*, int32_t*, cudaStream_t);
int mxfp8_quantize_rowcol_impl(const uint16_t*, int64_t, int64_t, const int32_t*, int, uint8_t*,
                               uint8_t*, uint8_t*, uint8_t*, int32_t*, cudaStream_t);

namespace {

size_t al256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

constexpr int kAllMx = MOE_MX_GEMM1 | MOE_MX_GEMM2 | MOE_MX_DA | MOE_MX_DW2 | MOE_MX_DX | MOE_MX_DW13;

// MOE_MX_* bits of the GEMMs that take MXFP8 operands under this descriptor.
int mx_mask(const moe_layer_desc* d) {
    if (d->dtype != MOE_DTYPE_MXFP8) return 0;
    return d->mx_gemms ? (d->mx_gemms & kAllMx) : kAllMx;
}

// Weights quantised by the forward in both layouts (mx_keep_weights): W13 when
// GEMM1 and dX are MXFP8, W2 when GEMM2 and dA are.
bool keep_w13(const moe_layer_desc* d, int mx) {
    return d->mx_keep_weights && (mx & MOE_MX_GEMM1) && (mx & MOE_MX_DX);
}
bool keep_w2(const moe_layer_desc* d, int mx) {
    return d->mx_keep_weights && (mx & MOE_MX_GEMM2) && (mx & MOE_MX_DA);
}

// Records the caller's stage event i (if any) on the stream.
int mark(const moe_layer_desc* d, int i, cudaStream_t st) {
    if (!d->stage_events || !d->stage_events[i]) return MOE_OK;
    return cudaEventRecord(static_cast<cudaEvent_t>(d->stage_events[i]), st) == cudaSuccess
               ? MOE_OK : MOE_ERR_CUDA;
}

// One MXFP8 operand in the workspace: E4M3 codes plus E8M0 scales.
struct MxBuf {
    size_t codes, scales;
};

struct WsLayout {
    size_t hist, dy, dh, dw;
    size_t kmaps, kmaps_bytes;  // per-expert tensor maps of the BF16 dW GEMMs
    size_t gu, a;  // recompute mode: [G | U] and A live here instead of in `saved`
    // MXFP8 (forward and backward regions alias: they never live together)
    MxBuf xr, w13r, ar, w2r;                          // forward, rowwise
    MxBuf dyr, w2c, dyc, ac, dhr, w13c, dhc, xc;      // backward
    size_t atoms, atoms_bytes;                        // per-GEMM scale atoms (reused)
    size_t total;
};

WsLayout ws_layout(const moe_layer_desc* d) {
    const size_t M = static_cast<size_t>(d->T) * d->k;
    const size_t E = d->E, dm = d->d, f = d->f;
    WsLayout L{};
    size_t off = 256;  // device status word
    L.hist = off; off += al256(permute_scratch_bytes(d->T, d->E));
    L.dy = off;   off += al256(M * dm * 2);        // dY_perm, later reused for dX_perm
    L.dh = off;   off += al256(M * 2 * f * 2);
    L.dw = off;   off += al256(static_cast<size_t>(d->T) * d->k * 4);
    if (d->recompute) {
        L.gu = off; off += al256(M * 2 * f * 2);
        L.a = off;  off += al256(M * f * 2);
    }
    {
        moe_gg_args g{};
        g.mode = MOE_GG_RAGGED_K; g.dtype = MOE_DTYPE_BF16; g.E = d->E;
        L.kmaps_bytes = grouped_gemm_workspace_bytes(&g);
        L.kmaps = off; off += al256(L.kmaps_bytes);
    }
    const int mx = mx_mask(d);
    if (mx) {
        auto row = [&](size_t& o, MxBuf& b, size_t rows, size_t cols) {
            b.codes = o; o += al256(rows * cols);
            b.scales = o; o += al256(rows * (cols / 32));
        };
        auto col = [&](size_t& o, MxBuf& b, size_t rows, size_t cols, size_t groups) {
            b.codes = o; o += al256(rows * cols);
            b.scales = o; o += al256((rows / 32 + groups) * cols);
        };
        // column-wise weights kept from the forward for the backward live
        // outside the two aliased regions
        if (keep_w2(d, mx)) col(off, L.w2c, E * dm, f, 1);
        if (keep_w13(d, mx)) col(off, L.w13c, E * 2 * f, dm, 1);
        // only the operands of the selected GEMMs get space; the backward's
        // recompute of GEMM1 may reuse the forward region: its operands are
        // dead (stream order) before the first backward quantisation
        size_t fo = off, bo = off;
        if (mx & MOE_MX_GEMM1) { row(fo, L.xr, M, dm); row(fo, L.w13r, E * 2 * f, dm); }
        if (mx & MOE_MX_GEMM2) { row(fo, L.ar, M, f); row(fo, L.w2r, E * dm, f); }
        if (mx & MOE_MX_DA) {
            row(bo, L.dyr, M, dm);
            if (!keep_w2(d, mx)) col(bo, L.w2c, E * dm, f, 1);
        }
        if (mx & MOE_MX_DW2) { col(bo, L.dyc, M, dm, E); col(bo, L.ac, M, f, E); }
        if (mx & MOE_MX_DX) {
            row(bo, L.dhr, M, 2 * f);
            if (!keep_w13(d, mx)) col(bo, L.w13c, E * 2 * f, dm, 1);
        }
        if (mx & MOE_MX_DW13) { col(bo, L.dhc, M, 2 * f, E); col(bo, L.xc, M, dm, E); }
        off = fo > bo ? fo : bo;
        // the GEMMs run one after the other: one atom area of the largest size
        size_t need = 0;
        auto gemm = [&](int bit, int mode, int epi, int N, int K, int Mo) {
            if (!(mx & bit)) return;
            moe_gg_args g{};
            g.mode = mode; g.dtype = MOE_DTYPE_MXFP8; g.epilogue = epi; g.E = d->E;
            g.M_total = static_cast<int64_t>(M); g.N = N; g.K = K; g.M = Mo;
            const size_t b = grouped_gemm_workspace_bytes(&g);
            need = b > need ? b : need;
        };
        gemm(MOE_MX_GEMM1, MOE_GG_RAGGED_M, MOE_EPI_SWIGLU, 2 * d->f, d->d, 0);
        gemm(MOE_MX_GEMM2, MOE_GG_RAGGED_M, MOE_EPI_NONE, d->d, d->f, 0);
        gemm(MOE_MX_DA, MOE_GG_RAGGED_M, MOE_EPI_SWIGLU_BWD, d->f, d->d, 0);
        gemm(MOE_MX_DX, MOE_GG_RAGGED_M, MOE_EPI_NONE, d->d, 2 * d->f, 0);
        gemm(MOE_MX_DW2, MOE_GG_RAGGED_K, MOE_EPI_NONE, d->f, 0, d->d);
        gemm(MOE_MX_DW13, MOE_GG_RAGGED_K, MOE_EPI_NONE, d->d, 0, 2 * d->f);
        L.atoms = off;
        L.atoms_bytes = need;
        off += al256(need);
    }
    L.total = off;
    return L;
}

// Both encodings of x [rows, cols] from one read: row-wise into r, column-wise
// per expert into c.
int quant_rowcol(uint8_t* w, const MxBuf& r, const MxBuf& c, const uint16_t* x, int64_t rows,
                 int64_t cols, const int32_t* goff, int ngroups, cudaStream_t st) {
    return mxfp8_quantize_rowcol_impl(x, rows, cols, goff, ngroups, w + r.codes, w + r.scales,
                                      w + c.codes, w + c.scales, nullptr, st);
}

// Quantise x [rows, cols] (bf16) into the workspace operand b.
int quant(uint8_t* w, const MxBuf& b, const uint16_t* x, int64_t rows, int64_t cols, int axis,
          const int32_t* goff, int ngroups, cudaStream_t st) {
    return mxfp8_quantize_impl(x, rows, cols, axis, goff, ngroups, w + b.codes, w + b.scales,
                               nullptr, st);
}

int validate(const moe_layer_desc* d, const moe_layer_params* p, const moe_layer_saved* s,
             void* ws, size_t ws_bytes) {
    if (!d || !p || !s || !ws) return MOE_ERR_INVALID_ARG;
    if (d->T < 0 || d->d < 8 || d->d % 8 || d->f < 8 || d->f % 8 || d->E < 1 || d->E > 1024 ||
        d->k < 1 || d->k > d->E || d->k > 32)
        return MOE_ERR_INVALID_ARG;
    if (static_cast<int64_t>(d->T) * d->k >= (1ll << 31)) return MOE_ERR_INVALID_ARG;
    if (d->dtype != MOE_DTYPE_BF16 && d->dtype != MOE_DTYPE_MXFP8) return MOE_ERR_INVALID_ARG;
    if (d->dtype == MOE_DTYPE_MXFP8 && (d->d % 32 || d->f % 32)) return MOE_ERR_INVALID_ARG;
    if (d->mx_gemms & ~kAllMx) return MOE_ERR_INVALID_ARG;
    if (d->router_mode == MOE_ROUTER_PROJ) {
        if (!p->w_r || !s->logits || !aligned16(p->w_r) || !aligned16(s->logits)) return MOE_ERR_INVALID_ARG;
    } else if (d->router_mode == MOE_ROUTER_LOGITS) {
        if (!p->logits || !aligned16(p->logits)) return MOE_ERR_INVALID_ARG;
    } else {
        return MOE_ERR_INVALID_ARG;
    }
    const void* ptrs[] = {p->x, p->w13, p->w2, s->topk_idx, s->topk_w, s->counts, s->offsets,
                          s->dest_pos, s->src_token, s->x_perm, s->y_perm, ws};
    for (const void* q : ptrs)
        if (!q || !aligned16(q)) return MOE_ERR_INVALID_ARG;
    if (!d->recompute && (!s->gu || !aligned16(s->gu) || !s->a || !aligned16(s->a)))
        return MOE_ERR_INVALID_ARG;
    if (ws_bytes < ws_layout(d).total) return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

// What every grouped GEMM of the layer shares besides its own operands.
struct Ctx {
    const moe_layer_desc* d;
    const WsLayout* L;
    uint8_t* w;
    int32_t* status;
    const int32_t* offsets;
    int mx;
    cudaStream_t st;

    moe_gg_args args(int mode, bool in_mx) const {
        moe_gg_args g{};
        g.mode = mode;
        g.dtype = in_mx ? MOE_DTYPE_MXFP8 : MOE_DTYPE_BF16;
        g.epilogue = MOE_EPI_NONE;
        g.E = d->E;
        g.M_total = static_cast<int64_t>(d->T) * d->k;
        g.offsets = offsets;
        g.status = status;
        if (in_mx) {
            g.workspace = w + L->atoms;
            g.workspace_bytes = L->atoms_bytes;
        } else if (mode == MOE_GG_RAGGED_K) {
            g.workspace = w + L->kmaps;
            g.workspace_bytes = L->kmaps_bytes;
        }
        return g;
    }
    void mx_a(moe_gg_args& g, const MxBuf& b) const {
        g.a = w + b.codes;
        g.a_scales = w + b.scales;
    }
    void mx_b(moe_gg_args& g, const MxBuf& b) const {
        g.b = w + b.codes;
        g.b_scales = w + b.scales;
    }
};

// GEMM1 + SwiGLU: [G | U] = x_perm W13_e^T, A = silu(G) * U; with `a_row`,
// A's row-wise MXFP8 codes / scales for GEMM2 come out of the same launch.
// `x_done`: x_perm's row-wise MXFP8 operand was written by the dispatch.
int run_gemm1(const Ctx& c, const uint16_t* x_perm, const uint16_t* w13, uint16_t* gu, uint16_t* a,
              const MxBuf* a_row = nullptr, bool w13_both = false, bool x_done = false) {
    const moe_layer_desc* d = c.d;
    const bool mx = c.mx & MOE_MX_GEMM1;
    moe_gg_args g = c.args(MOE_GG_RAGGED_M, mx);
    g.epilogue = MOE_EPI_SWIGLU;
    g.N = 2 * d->f;
    g.K = d->d;
    g.a = x_perm;
    g.b = w13;
    if (mx) {
        if (!x_done) MOE_TRY(quant(c.w, c.L->xr, x_perm, g.M_total, d->d, 1, nullptr, 0, c.st));
        const int64_t rows13 = static_cast<int64_t>(d->E) * 2 * d->f;
        if (w13_both)  // also W13's column-wise encoding for dX, kept for the backward
            MOE_TRY(quant_rowcol(c.w, c.L->w13r, c.L->w13c, w13, rows13, d->d, nullptr, 1, c.st));
        else
            MOE_TRY(quant(c.w, c.L->w13r, w13, rows13, d->d, 1, nullptr, 0, c.st));
        c.mx_a(g, c.L->xr);
        c.mx_b(g, c.L->w13r);
    }
    g.c = gu;
    g.aux = a;
    if (a_row) {
        g.q_row_codes = c.w + a_row->codes;
        g.q_row_scales = c.w + a_row->scales;
    }
    return grouped_gemm(&g, c.st);
}

}  // namespace

size_t layer_workspace_bytes(const moe_layer_desc* d) { return d ? ws_layout(d).total : 0; }

int layer_fwd(const moe_layer_desc* d, const moe_layer_params* p, const moe_layer_saved* s,
              uint16_t* out, void* ws, size_t ws_bytes, cudaStream_t st) {
    MOE_TRY(validate(d, p, s, ws, ws_bytes));
    if (!out || !aligned16(out)) return MOE_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(d);
    uint8_t* w = static_cast<uint8_t*>(ws);
    int32_t* status = reinterpret_cast<int32_t*>(w);
    const int T = d->T, E = d->E, k = d->k, f = d->f, dm = d->d;
    const Ctx c{d, &L, w, status, s->offsets, mx_mask(d), st};
    uint16_t* gu = d->recompute ? reinterpret_cast<uint16_t*>(w + L.gu) : s->gu;
    uint16_t* a = d->recompute ? reinterpret_cast<uint16_t*>(w + L.a) : s->a;

    const float* logits = p->logits;
    MOE_TRY(mark(d, 0, st));
    if (d->router_mode == MOE_ROUTER_PROJ) {
        MOE_TRY(router_proj(p->x, p->w_r, T, dm, E, s->logits, st));
        logits = s->logits;
    }
    MOE_TRY(router_topk(logits, T, E, k, s->topk_idx, s->topk_w, st));
    MOE_TRY(mark(d, 1, st));
    // with an MXFP8 GEMM1 the dispatch also writes x_perm's row-wise encoding
    const bool x_mx = c.mx & MOE_MX_GEMM1;
    MOE_TRY(permute_rows(p->x, s->topk_idx, T, dm, E, k, s->counts, s->offsets, s->dest_pos,
                         s->src_token, s->x_perm, reinterpret_cast<int32_t*>(w + L.hist), status, st,
                         x_mx ? w + L.xr.codes : nullptr, x_mx ? w + L.xr.scales : nullptr));
    MOE_TRY(mark(d, 2, st));
    // A's row-wise MXFP8 operand of GEMM2 comes from GEMM1's epilogue
    MOE_TRY(run_gemm1(c, s->x_perm, p->w13, gu, a, (c.mx & MOE_MX_GEMM2) ? &L.ar : nullptr,
                      keep_w13(d, c.mx), x_mx));
    MOE_TRY(mark(d, 3, st));
    {   // GEMM2: Y = A W2_e^T
        const bool mx = c.mx & MOE_MX_GEMM2;
        moe_gg_args g = c.args(MOE_GG_RAGGED_M, mx);
        g.N = dm;
        g.K = f;
        g.a = a;
        g.b = p->w2;
        if (mx) {
            if (keep_w2(d, c.mx))  // also W2's column-wise encoding for dA, kept for the backward
                MOE_TRY(quant_rowcol(w, L.w2r, L.w2c, p->w2, static_cast<int64_t>(E) * dm, f, nullptr, 1, st));
            else
                MOE_TRY(quant(w, L.w2r, p->w2, static_cast<int64_t>(E) * dm, f, 1, nullptr, 0, st));
            c.mx_a(g, L.ar);
            c.mx_b(g, L.w2r);
        }
        g.c = s->y_perm;
        MOE_TRY(grouped_gemm(&g, st));
    }
    MOE_TRY(mark(d, 4, st));
    MOE_TRY(combine(s->y_perm, s->dest_pos, s->topk_w, T, dm, k, out, st));
    return mark(d, 5, st);
}

int layer_bwd(const moe_layer_desc* d, const moe_layer_params* p, const moe_layer_saved* s,
              const uint16_t* dout, const moe_layer_grads* gr, void* ws, size_t ws_bytes,
              cudaStream_t st) {
    MOE_TRY(validate(d, p, s, ws, ws_bytes));
    if (!dout || !gr || !gr->dx || !gr->dw13 || !gr->dw2 || !gr->d_logits) return MOE_ERR_INVALID_ARG;
    if (!aligned16(dout) || !aligned16(gr->dx) || !aligned16(gr->dw13) || !aligned16(gr->dw2) ||
        !aligned16(gr->d_logits))
        return MOE_ERR_INVALID_ARG;
    const bool proj = d->router_mode == MOE_ROUTER_PROJ;
    if (proj && (!gr->dw_r || !aligned16(gr->dw_r))) return MOE_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(d);
    uint8_t* w = static_cast<uint8_t*>(ws);
    int32_t* status = reinterpret_cast<int32_t*>(w);
    uint16_t* dY = reinterpret_cast<uint16_t*>(w + L.dy);
    uint16_t* dH = reinterpret_cast<uint16_t*>(w + L.dh);
    float* dw = reinterpret_cast<float*>(w + L.dw);
    const int T = d->T, E = d->E, k = d->k, f = d->f, dm = d->d;
    const int64_t M = static_cast<int64_t>(T) * k;
    const int64_t EK2 = static_cast<int64_t>(E) * dm, EK13 = static_cast<int64_t>(E) * 2 * f;
    const Ctx c{d, &L, w, status, s->offsets, mx_mask(d), st};
    const uint16_t* gu = s->gu;
    const uint16_t* a = s->a;

    MOE_TRY(mark(d, 0, st));
    if (d->recompute) {
        // [G | U] and A again from the saved x_perm, into the workspace
        uint16_t* gu_ws = reinterpret_cast<uint16_t*>(w + L.gu);
        uint16_t* a_ws = reinterpret_cast<uint16_t*>(w + L.a);
        MOE_TRY(run_gemm1(c, s->x_perm, p->w13, gu_ws, a_ws));
        gu = gu_ws;
        a = a_ws;
    }
    MOE_TRY(mark(d, 1, st));
    MOE_TRY(combine_bwd(dout, s->y_perm, s->dest_pos, s->topk_w, T, dm, k, dY, dw, st));
    MOE_TRY(mark(d, 2, st));
    // dY and dH are each needed row-wise (dA, dX) and column-wise per expert
    // (dW2, dW13): where both are MXFP8, one pass writes both encodings
    const bool dy_both = (c.mx & MOE_MX_DA) && (c.mx & MOE_MX_DW2);
    const bool dh_both = (c.mx & MOE_MX_DX) && (c.mx & MOE_MX_DW13);
    if (dy_both) MOE_TRY(quant_rowcol(w, L.dyr, L.dyc, dY, M, dm, s->offsets, E, st));
    {   // dA = dY W2_e, fused SwiGLU backward -> dH = [dG | dU]
        const bool mx = c.mx & MOE_MX_DA;
        moe_gg_args g = c.args(MOE_GG_RAGGED_M, mx);
        g.epilogue = MOE_EPI_SWIGLU_BWD;
        g.N = f;
        g.K = dm;
        g.a = dY;
        g.b = p->w2;  // [E][d][f] = [E][K][N]
        g.b_mn_major = 1;
        if (mx) {
            if (!dy_both) MOE_TRY(quant(w, L.dyr, dY, M, dm, 1, nullptr, 0, st));
            if (!keep_w2(d, c.mx)) MOE_TRY(quant(w, L.w2c, p->w2, EK2, f, 0, nullptr, 1, st));
            c.mx_a(g, L.dyr);
            c.mx_b(g, L.w2c);
        }
        g.c = dH;
        g.gu = gu;
        MOE_TRY(grouped_gemm(&g, st));
    }
    if (dh_both) MOE_TRY(quant_rowcol(w, L.dhr, L.dhc, dH, M, 2 * f, s->offsets, E, st));
    MOE_TRY(mark(d, 3, st));
    {   // dW2_e = dY_e^T A_e
        const bool mx = c.mx & MOE_MX_DW2;
        moe_gg_args g = c.args(MOE_GG_RAGGED_K, mx);
        g.M = dm;
        g.N = f;
        g.a = dY;
        g.b = a;
        if (mx) {
            if (!dy_both) MOE_TRY(quant(w, L.dyc, dY, M, dm, 0, s->offsets, E, st));
            MOE_TRY(quant(w, L.ac, a, M, f, 0, s->offsets, E, st));
            c.mx_a(g, L.dyc);
            c.mx_b(g, L.ac);
        }
        g.c = gr->dw2;
        MOE_TRY(grouped_gemm(&g, st));
    }
    MOE_TRY(mark(d, 4, st));
    uint16_t* dX = dY;  // dY's space is free again
    {   // dX_perm = dH W13_e
        const bool mx = c.mx & MOE_MX_DX;
        moe_gg_args g = c.args(MOE_GG_RAGGED_M, mx);
        g.N = dm;
        g.K = 2 * f;
        g.a = dH;
        g.b = p->w13;  // [E][2f][d] = [E][K][N]
        g.b_mn_major = 1;
        if (mx) {
            if (!dh_both) MOE_TRY(quant(w, L.dhr, dH, M, 2 * f, 1, nullptr, 0, st));
            if (!keep_w13(d, c.mx)) MOE_TRY(quant(w, L.w13c, p->w13, EK13, dm, 0, nullptr, 1, st));
            c.mx_a(g, L.dhr);
            c.mx_b(g, L.w13c);
        }
        g.c = dX;
        MOE_TRY(grouped_gemm(&g, st));
    }
    MOE_TRY(mark(d, 5, st));
    {   // dW13_e = dH_e^T x_perm_e
        const bool mx = c.mx & MOE_MX_DW13;
        moe_gg_args g = c.args(MOE_GG_RAGGED_K, mx);
        g.M = 2 * f;
        g.N = dm;
        g.a = dH;
        g.b = s->x_perm;
        if (mx) {
            if (!dh_both) MOE_TRY(quant(w, L.dhc, dH, M, 2 * f, 0, s->offsets, E, st));
            MOE_TRY(quant(w, L.xc, s->x_perm, M, dm, 0, s->offsets, E, st));
            c.mx_a(g, L.dhc);
            c.mx_b(g, L.xc);
        }
        g.c = gr->dw13;
        MOE_TRY(grouped_gemm(&g, st));
    }
    MOE_TRY(mark(d, 6, st));
    MOE_TRY(router_bwd(s->topk_idx, s->topk_w, dw, T, E, k, gr->d_logits, st));
    MOE_TRY(mark(d, 7, st));
    MOE_TRY(unpermute_sum(dX, s->dest_pos, T, dm, k, proj ? gr->d_logits : nullptr,
                          proj ? p->w_r : nullptr, E, gr->dx, st));
    if (proj) MOE_TRY(router_proj_bwd(p->x, gr->d_logits, T, dm, E, gr->dw_r, st));
    return mark(d, 8, st);
}

}  // namespace moe
