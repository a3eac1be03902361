// lm_linear.cu -- a plain linear layer Y = X W^T, forward and backward, with
// all three GEMMs in FP8 and dynamic tensorwise scaling (decomputer.nl, "Het
// trainen van een 3.8B LLM tot 0.384 CORE voor $998", section "Vroege
// experimenten" item 4: forward, dgrad and wgrad of every linear in FP8).
// The attention projections and the LM head of the model are such linears.
//
// Composed from the cast and GEMM kernels on one stream with no host
// synchronisation, like the MLP: X and W are cast in one amax launch and one
// cast launch, to row-major codes only; the backward casts dY and reads the
// saved codes MN-major where a GEMM contracts over their rows.
#include "lm_internal.h"

namespace {

constexpr size_t kAlign = 256;

size_t round_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

bool linear_shape_ok(int64_t M, int64_t K, int64_t N) {
    return M >= 0 && K > 0 && N > 0 && M % 16 == 0 && K % 16 == 0 && N % 16 == 0;
}

// scale blocks: 4 floats per tensor {amax, scale, inv_scale, unused}
enum { S_X = 0, S_W = 4 };  // in lm_linear_saved::scales

size_t saved_layout(int64_t M, int64_t K, int64_t N, uint8_t* base, lm_linear_saved* s) {
    size_t off = 0;
    auto take = [&](size_t bytes) {
        uint8_t* p = base ? base + off : nullptr;
        off += round_up(bytes);
        return p;
    };
    lm_linear_saved o;
    o.Xq = take((size_t)M * (size_t)K);
    o.Wq = take((size_t)N * (size_t)K);
    o.scales = reinterpret_cast<float*>(take(8 * sizeof(float)));
    if (s) *s = o;
    return off;
}

// backward scratch: the GEMMs' split-K region, dY's codes, dY's scale block
size_t bwd_layout(int64_t M, int64_t N, uint8_t* base, void** split, uint8_t** dYq,
                  float** sc) {
    size_t off = 0;
    auto take = [&](size_t bytes) {
        uint8_t* p = base ? base + off : nullptr;
        off += round_up(bytes);
        return p;
    };
    uint8_t* sp = take(lm::gemm_split_workspace_bytes());
    uint8_t* q = take((size_t)M * (size_t)N);
    uint8_t* g = take(4 * sizeof(float));
    if (split) *split = sp;
    if (dYq) *dYq = q;
    if (sc) *sc = reinterpret_cast<float*>(g);
    return off;
}

#define LM_TRY(expr)                       \
    do {                                   \
        lm_status _st = (expr);            \
        if (_st != LM_OK) return _st;      \
    } while (0)

}  // namespace

extern "C" {

size_t lm_fp8_linear_saved_bytes(int64_t M, int64_t K, int64_t N) {
    if (!linear_shape_ok(M, K, N)) return 0;
    return saved_layout(M, K, N, nullptr, nullptr);
}

lm_status lm_fp8_linear_saved_carve(void* base, size_t bytes, int64_t M, int64_t K, int64_t N,
                                    lm_linear_saved* out) {
    if (!base || !out) return LM_ERR_INVALID_ARG;
    if (!linear_shape_ok(M, K, N)) return LM_ERR_UNSUPPORTED_SHAPE;
    if ((reinterpret_cast<uintptr_t>(base) % kAlign) != 0) return LM_ERR_ALIGNMENT;
    if (bytes < saved_layout(M, K, N, nullptr, nullptr)) return LM_ERR_INVALID_ARG;
    saved_layout(M, K, N, static_cast<uint8_t*>(base), out);
    return LM_OK;
}

size_t lm_fp8_linear_workspace_size(int64_t M, int64_t K, int64_t N) {
    if (!linear_shape_ok(M, K, N)) return 0;
    return bwd_layout(M, N, nullptr, nullptr, nullptr, nullptr);
}

lm_status lm_fp8_linear_fwd(const void* X, const void* W, int64_t M, int64_t K, int64_t N,
                            void* Y, lm_linear_saved* sv, void* workspace, size_t ws_bytes,
                            uint32_t flags, lm_stream_t stream) {
    if (!linear_shape_ok(M, K, N)) return LM_ERR_UNSUPPORTED_SHAPE;
    if (flags & ~LM_LINEAR_REUSE_WEIGHT_CAST) return LM_ERR_INVALID_ARG;
    if (workspace && (reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0)
        return LM_ERR_ALIGNMENT;
    const bool reuse = (flags & LM_LINEAR_REUSE_WEIGHT_CAST) != 0;
    // with M == 0 there is no X or Y to touch (W is still cast)
    if (!sv || (M > 0 && (!X || !Y)) || (!reuse && !W)) return LM_ERR_INVALID_ARG;
    if (!sv->Xq || !sv->Wq || !sv->scales) return LM_ERR_INVALID_ARG;
    if (!lm::all_aligned16({X, W, Y, sv->Xq, sv->Wq})) return LM_ERR_ALIGNMENT;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const size_t split_bytes = lm::gemm_split_workspace_bytes();
    void* split = workspace && ws_bytes >= split_bytes ? workspace : nullptr;
    const size_t sb = split ? split_bytes : 0;
    float* S = sv->scales;
    // zero the amax slots the casts reduce into (X's alone when W's codes are reused)
    if (cudaMemsetAsync(S, 0, (reuse ? 4 : 8) * sizeof(float), s) != cudaSuccess)
        return LM_ERR_CUDA;
    const lm::CastItem in[2] = {
        {X, M, K, K, nullptr, S + S_X, S + S_X + 1, S + S_X + 2, sv->Xq, nullptr},
        {W, N, K, K, nullptr, S + S_W, S + S_W + 1, S + S_W + 2, sv->Wq, nullptr}};
    LM_TRY(lm::cast_set(in, reuse ? 1 : 2, LM_FP8_E4M3, 0, true, s));
    // Y = Xq Wq^T (both K-major)
    return lm_fp8_gemm_ex(sv->Xq, LM_FP8_E4M3, sv->Wq, LM_FP8_E4M3, M, N, K, 0u, S + S_X + 2,
                          S + S_W + 2, LM_EPI_NONE, nullptr, Y, nullptr, split, sb, stream);
}

lm_status lm_fp8_linear_bwd(const void* dY, const lm_linear_saved* sv, int64_t M, int64_t K,
                            int64_t N, void* dX, void* dW, void* workspace, size_t ws_bytes,
                            uint32_t flags, lm_stream_t stream) {
    if (!linear_shape_ok(M, K, N)) return LM_ERR_UNSUPPORTED_SHAPE;
    if (flags & ~LM_LINEAR_ACCUMULATE_WGRAD) return LM_ERR_INVALID_ARG;
    if (!sv || !dW || !workspace || (M > 0 && !dY)) return LM_ERR_INVALID_ARG;
    if (!sv->Xq || !sv->Wq || !sv->scales) return LM_ERR_INVALID_ARG;
    if (ws_bytes < bwd_layout(M, N, nullptr, nullptr, nullptr, nullptr))
        return LM_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0) return LM_ERR_ALIGNMENT;
    if (!lm::all_aligned16({dY, dX, dW, sv->Xq, sv->Wq})) return LM_ERR_ALIGNMENT;
    void* split;
    uint8_t* dYq;
    float* G;
    bwd_layout(M, N, static_cast<uint8_t*>(workspace), &split, &dYq, &G);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const float* S = sv->scales;
    if (cudaMemsetAsync(G, 0, 4 * sizeof(float), s) != cudaSuccess) return LM_ERR_CUDA;
    const lm::CastItem dy = {dY, M, N, N, nullptr, G, G + 1, G + 2, dYq, nullptr};
    LM_TRY(lm::cast_set(&dy, 1, LM_FP8_E5M2, 0, true, s));  // slot zeroed above
    const size_t sb = lm::gemm_split_workspace_bytes();
    // dX = dY W: A = dYq [M x N], B = W [N x K] read MN-major as the [K x N] operand
    if (dX) {
        LM_TRY(lm_fp8_gemm_ex(dYq, LM_FP8_E5M2, sv->Wq, LM_FP8_E4M3, M, K, N, LM_GEMM_B_MN_MAJOR,
                              G + 2, S + S_W + 2, LM_EPI_NONE, nullptr, dX, nullptr, split, sb,
                              stream));
    }
    // dW = dY^T X (reduction over the M tokens): dYq [M x N] and Xq [M x K] read MN-major
    const lm_epilogue wgrad_epi =
        (flags & LM_LINEAR_ACCUMULATE_WGRAD) ? LM_EPI_ACCUM_F32 : LM_EPI_NONE;
    return lm_fp8_gemm_ex(dYq, LM_FP8_E5M2, sv->Xq, LM_FP8_E4M3, N, K, M,
                          LM_GEMM_A_MN_MAJOR | LM_GEMM_B_MN_MAJOR, G + 2, S + S_X + 2, wgrad_epi,
                          nullptr, dW, nullptr, split, sb, stream);
}

}  // extern "C"
