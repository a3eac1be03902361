// lm_mlp.cu -- the non-gated relu^2 MLP, forward and backward, composed from
// the cast and GEMM kernels on one stream with no host synchronisation.
//
// Model: hidden_act relu2, gated_mlp false, intermediate 4x (decomputer.nl,
// "Het trainen van een 3.8B LLM tot 0.384 CORE voor $998", "Appendix: De
// configuratie", and section "Doorvoer (Throughput) verhogen", bullet
// "Niet-gated MLPs": two matmuls instead of three).  All six GEMMs (forward,
// dgrad and wgrad of both linears) run in FP8 with dynamic tensorwise scaling
// (same page, section "Vroege experimenten" item 4).  Each tensor is
// quantised once per call, to row-major codes only; the backward reuses the
// forward's codes and scales, reading them MN-major where a GEMM contracts
// over their rows.  The workspace's first lm_fp8_gemm_workspace_size() bytes
// let the GEMMs split an under-filled last wave of tiles.
#include "lm_internal.h"

namespace {

constexpr size_t kAlign = 256;

size_t round_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

bool mlp_shape_ok(int64_t M, int64_t d, int64_t f) {
    return M >= 0 && d > 0 && f > 0 && M % 16 == 0 && d % 16 == 0 && f % 16 == 0;
}

// scale block layout: 4 floats per tensor {amax, scale, inv_scale, unused}
enum { S_X = 0, S_WU = 4, S_WD = 8, S_H = 12 };  // in lm_mlp_saved::scales
enum { S_DY = 0, S_DH = 4 };                      // in the backward workspace

struct BwdWorkspace {
    void* split;  // the GEMMs' split-K scratch (lm_fp8_gemm_workspace_size bytes)
    uint8_t *dYq, *dHq;
    void* dH;
    float* scales;
};

size_t bwd_layout(int64_t M, int64_t d, int64_t f, uint8_t* base, BwdWorkspace* w) {
    const size_t Md = (size_t)M * (size_t)d, Mf = (size_t)M * (size_t)f;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        uint8_t* p = base ? base + off : nullptr;
        off += round_up(bytes);
        return p;
    };
    uint8_t* split = take(lm::gemm_split_workspace_bytes());
    uint8_t* dYq = take(Md);
    uint8_t* dH = take(Mf * 2);
    uint8_t* dHq = take(Mf);
    uint8_t* sc = take(8 * sizeof(float));
    if (w) *w = BwdWorkspace{split, dYq, dHq, dH, reinterpret_cast<float*>(sc)};
    return off;
}

size_t saved_layout(int64_t M, int64_t d, int64_t f, uint8_t* base, lm_mlp_saved* s) {
    const size_t Md = (size_t)M * (size_t)d, Mf = (size_t)M * (size_t)f,
                 fd = (size_t)f * (size_t)d;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        uint8_t* p = base ? base + off : nullptr;
        off += round_up(bytes);
        return p;
    };
    lm_mlp_saved o;
    o.Xq = take(Md);
    o.Wuq = take(fd);
    o.Wdq = take(fd);
    o.H = take(Mf * 2);
    o.hq = take(Mf);
    o.scales = reinterpret_cast<float*>(take(16 * sizeof(float)));
    if (s) *s = o;
    return off;
}

#define LM_TRY(expr)                       \
    do {                                   \
        lm_status _st = (expr);            \
        if (_st != LM_OK) return _st;      \
    } while (0)

}  // namespace

extern "C" {

size_t lm_relu2_mlp_saved_bytes(int64_t M, int64_t d, int64_t f) {
    if (!mlp_shape_ok(M, d, f)) return 0;
    return saved_layout(M, d, f, nullptr, nullptr);
}

lm_status lm_relu2_mlp_saved_carve(void* base, size_t bytes, int64_t M, int64_t d, int64_t f,
                                   lm_mlp_saved* out) {
    if (!base || !out) return LM_ERR_INVALID_ARG;
    if (!mlp_shape_ok(M, d, f)) return LM_ERR_UNSUPPORTED_SHAPE;
    if ((reinterpret_cast<uintptr_t>(base) % kAlign) != 0) return LM_ERR_ALIGNMENT;
    if (bytes < saved_layout(M, d, f, nullptr, nullptr)) return LM_ERR_INVALID_ARG;
    saved_layout(M, d, f, static_cast<uint8_t*>(base), out);
    return LM_OK;
}

size_t lm_relu2_mlp_workspace_size(int64_t M, int64_t d, int64_t f) {
    if (!mlp_shape_ok(M, d, f)) return 0;
    return bwd_layout(M, d, f, nullptr, nullptr);
}

lm_status lm_relu2_mlp_fwd_ex(const void* X, const void* W_up, const void* W_down, int64_t M,
                              int64_t d, int64_t f, void* Y, lm_mlp_saved* sv, void* workspace,
                              size_t ws_bytes, uint32_t flags, lm_stream_t stream) {
    if (!mlp_shape_ok(M, d, f)) return LM_ERR_UNSUPPORTED_SHAPE;
    if (flags & ~LM_MLP_REUSE_WEIGHT_CASTS) return LM_ERR_INVALID_ARG;
    if (workspace && (reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0)
        return LM_ERR_ALIGNMENT;
    const bool reuse = (flags & LM_MLP_REUSE_WEIGHT_CASTS) != 0;
    // tensors with M rows may be NULL when M == 0 (an empty micro-batch)
    if (!sv || (M > 0 && (!X || !Y)) || (!reuse && (!W_up || !W_down))) return LM_ERR_INVALID_ARG;
    if (!sv->Wuq || !sv->Wdq || !sv->scales || (M > 0 && (!sv->Xq || !sv->H || !sv->hq)))
        return LM_ERR_INVALID_ARG;
    if (!lm::all_aligned16({X, W_up, W_down, Y, sv->Xq, sv->Wuq, sv->Wdq, sv->H, sv->hq}))
        return LM_ERR_ALIGNMENT;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // the workspace, when given, holds the GEMMs' split-K scratch at its start
    const size_t split_bytes = lm::gemm_split_workspace_bytes();
    void* split = workspace && ws_bytes >= split_bytes ? workspace : nullptr;
    const size_t sb = split ? split_bytes : 0;
    float* S = sv->scales;
    if (reuse) {  // keep the weights' scale blocks; reset X's and h's
        if (cudaMemsetAsync(S + S_X, 0, 4 * sizeof(float), s) != cudaSuccess ||
            cudaMemsetAsync(S + S_H, 0, 4 * sizeof(float), s) != cudaSuccess)
            return LM_ERR_CUDA;
    } else if (cudaMemsetAsync(S, 0, 16 * sizeof(float), s) != cudaSuccess) {
        return LM_ERR_CUDA;
    }
    // X, W_up and W_down (or X alone): one amax launch for all three (their
    // amax slots were zeroed above) and one cast launch for X and W_up.
    // W_down is cast beside the up GEMM, which does not read it.  Row-major
    // codes only: the backward reads them MN-major where it needs the
    // transpose.
    const lm::CastItem in[3] = {
        {X, M, d, d, nullptr, S + S_X, S + S_X + 1, S + S_X + 2, sv->Xq, nullptr},
        {W_up, f, d, d, nullptr, S + S_WU, S + S_WU + 1, S + S_WU + 2, sv->Wuq, nullptr},
        {W_down, d, f, f, nullptr, S + S_WD, S + S_WD + 1, S + S_WD + 2, nullptr, nullptr,
         true}};
    LM_TRY(lm::cast_set(in, reuse ? 1 : 3, LM_FP8_E4M3, 0, true, s));
    const lm::SideCast wd = {W_down, d, f, LM_FP8_E4M3, S + S_WD, S + S_WD, S + S_WD + 1,
                             S + S_WD + 2, sv->Wdq};
    // H = X W_up^T (bf16) and amax of h = bf16(relu(H)^2); W_down's codes
    LM_TRY(lm::gemm_dispatch(sv->Xq, LM_FP8_E4M3, sv->Wuq, LM_FP8_E4M3, M, f, d, 0u, S + S_X + 2,
                             S + S_WU + 2, LM_EPI_RELU2_FWD, nullptr, sv->H, nullptr, S + S_H,
                             split, sb, stream, reuse ? nullptr : &wd));
    // Y = h W_down^T, with h = bf16(relu(H)^2) cast to its codes (the amax came
    // from the up GEMM's epilogue) by the down GEMM's side warps, unit by unit
    // ahead of the tiles that read them (its own launch first where that
    // cannot be done: no workspace, a thin M or a multi-part split tail)
    lm::SideCast hc = {sv->H, M, f, LM_FP8_E4M3, S + S_H, S + S_H, S + S_H + 1, S + S_H + 2,
                       sv->hq};
    hc.relu2 = 1;
    hc.feeds_a = 1;
    LM_TRY(lm::gemm_dispatch(sv->hq, LM_FP8_E4M3, sv->Wdq, LM_FP8_E4M3, M, d, f, 0u, S + S_H + 2,
                             S + S_WD + 2, LM_EPI_NONE, nullptr, Y, nullptr, nullptr, split, sb,
                             stream, &hc));
    return LM_OK;
}

lm_status lm_relu2_mlp_fwd(const void* X, const void* W_up, const void* W_down, int64_t M,
                           int64_t d, int64_t f, void* Y, lm_mlp_saved* sv, void* workspace,
                           size_t ws_bytes, lm_stream_t stream) {
    return lm_relu2_mlp_fwd_ex(X, W_up, W_down, M, d, f, Y, sv, workspace, ws_bytes, 0u, stream);
}

lm_status lm_relu2_mlp_bwd_ex(const void* dY, const lm_mlp_saved* sv, int64_t M, int64_t d,
                              int64_t f, void* dX, void* dW_up, void* dW_down, void* workspace,
                              size_t ws_bytes, uint32_t flags, lm_stream_t stream) {
    if (!mlp_shape_ok(M, d, f)) return LM_ERR_UNSUPPORTED_SHAPE;
    if (flags & ~LM_MLP_ACCUMULATE_WGRAD) return LM_ERR_INVALID_ARG;
    // tensors with M rows may be NULL when M == 0 (an empty micro-batch: the
    // weight gradients are then zero, or left as they were when accumulating)
    if (!sv || !dW_up || !dW_down || !workspace || (M > 0 && (!dY || !dX)))
        return LM_ERR_INVALID_ARG;
    if (ws_bytes < bwd_layout(M, d, f, nullptr, nullptr)) return LM_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0) return LM_ERR_ALIGNMENT;
    if (!sv->Wuq || !sv->Wdq || !sv->scales || (M > 0 && (!sv->Xq || !sv->H || !sv->hq)))
        return LM_ERR_INVALID_ARG;
    if (!lm::all_aligned16({dY, dX, dW_up, dW_down, sv->Xq, sv->Wuq, sv->Wdq, sv->H, sv->hq}))
        return LM_ERR_ALIGNMENT;
    const lm_epilogue wgrad_epi =
        (flags & LM_MLP_ACCUMULATE_WGRAD) ? LM_EPI_ACCUM_F32 : LM_EPI_NONE;
    BwdWorkspace w;
    bwd_layout(M, d, f, static_cast<uint8_t*>(workspace), &w);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const float* S = sv->scales;
    float* G = w.scales;
    if (cudaMemsetAsync(G, 0, 8 * sizeof(float), s) != cudaSuccess) return LM_ERR_CUDA;
    const lm::CastItem dy = {dY, M, d, d, nullptr, G + S_DY, G + S_DY + 1, G + S_DY + 2,
                             w.dYq, nullptr};
    LM_TRY(lm::cast_set(&dy, 1, LM_FP8_E5M2, 0, true, s));  // slot zeroed above
    constexpr uint32_t B_MN = LM_GEMM_B_MN_MAJOR, AB_MN = LM_GEMM_A_MN_MAJOR | LM_GEMM_B_MN_MAJOR;
    const size_t sb = lm::gemm_split_workspace_bytes();
    // dH = bf16(bf16(dY W_down) * 2 relu(H)), and its amax; B = W_down [d x f]
    // read MN-major as the [f x d] operand
    LM_TRY(lm_fp8_gemm_ex(w.dYq, LM_FP8_E5M2, sv->Wdq, LM_FP8_E4M3, M, f, d, B_MN, G + S_DY + 2,
                          S + S_WD + 2, LM_EPI_RELU2_BWD, sv->H, w.dH, G + S_DH, w.split, sb,
                          stream));
    // dW_down = dY^T h (K = M): dY [M x d] and h [M x f] read MN-major; the
    // cast of dH (its amax came from the epilogue above) runs beside it
    const lm::SideCast dh = {w.dH, M, f, LM_FP8_E5M2, G + S_DH, G + S_DH, G + S_DH + 1,
                             G + S_DH + 2, w.dHq};
    LM_TRY(lm::gemm_dispatch(w.dYq, LM_FP8_E5M2, sv->hq, LM_FP8_E4M3, d, f, M, AB_MN,
                             G + S_DY + 2, S + S_H + 2, wgrad_epi, nullptr, dW_down, nullptr,
                             nullptr, w.split, sb, stream, &dh));
    // dX = dH W_up (W_up [f x d] read MN-major);  dW_up = dH^T X (K = M)
    LM_TRY(lm_fp8_gemm_ex(w.dHq, LM_FP8_E5M2, sv->Wuq, LM_FP8_E4M3, M, d, f, B_MN, G + S_DH + 2,
                          S + S_WU + 2, LM_EPI_NONE, nullptr, dX, nullptr, w.split, sb, stream));
    LM_TRY(lm_fp8_gemm_ex(w.dHq, LM_FP8_E5M2, sv->Xq, LM_FP8_E4M3, f, d, M, AB_MN, G + S_DH + 2,
                          S + S_X + 2, wgrad_epi, nullptr, dW_up, nullptr, w.split, sb, stream));
    return LM_OK;
}

lm_status lm_relu2_mlp_bwd(const void* dY, const lm_mlp_saved* sv, int64_t M, int64_t d,
                           int64_t f, void* dX, void* dW_up, void* dW_down, void* workspace,
                           size_t ws_bytes, lm_stream_t stream) {
    return lm_relu2_mlp_bwd_ex(dY, sv, M, d, f, dX, dW_up, dW_down, workspace, ws_bytes, 0u,
                               stream);
}

}  // extern "C"
