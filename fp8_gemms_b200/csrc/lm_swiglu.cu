// lm_swiglu.cu -- the gated (SwiGLU) MLP, the comparison workload of the
// non-gated relu^2 MLP (decomputer.nl, "Het trainen van een 3.8B LLM tot
// 0.384 CORE voor $998", section "Doorvoer (Throughput) verhogen", bullet
// "Niet-gated MLPs": SwiGLU needs three matmuls where relu^2 needs two; its
// intermediate ratio 2.75).  Same FP8 dynamic tensorwise scaling on all
// GEMMs.
//
//   G|U = X W_gu^T           one GEMM, W_gu = gate and up rows interleaved in
//                            128-row blocks; its epilogue also writes
//                            h = bf16(silu(G) U) and amax(h)
//   Y   = h W_down^T
//   g   = dY W_down          (dgrad of the down projection, plain epilogue)
//   dG  = bf16(g U silu'(G)), dU = bf16(g silu(G))   elementwise, with amax
//   dX  = dGU W_gu           one GEMM over the interleaved 2f dimension
//   dW_gu = dGU^T X, dW_down = dY^T h
#include <cuda_bf16.h>

#include "lm_internal.h"

namespace lm {
namespace {

constexpr size_t kAlign = 256;
size_t round_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

bool shape_ok(int64_t M, int64_t d, int64_t f) {
    return M >= 0 && d > 0 && f > 0 && M % 16 == 0 && d % 16 == 0 && f % 128 == 0;
}

enum { S_X = 0, S_WGU = 4, S_WD = 8, S_H = 12 };  // lm_swiglu_saved::scales
enum { S_DY = 0, S_DGU = 4 };                     // backward workspace scales

size_t saved_layout(int64_t M, int64_t d, int64_t f, uint8_t* base, lm_swiglu_saved* out) {
    const size_t Md = (size_t)M * d, Mf = (size_t)M * f, fd = (size_t)f * d;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        uint8_t* p = base ? base + off : nullptr;
        off += round_up(bytes);
        return p;
    };
    lm_swiglu_saved o;
    o.Xq = take(Md);
    o.Wguq = take(2 * fd);
    o.Wdq = take(fd);
    o.GU = take(2 * Mf * 2);
    o.h = take(Mf * 2);
    o.hq = take(Mf);
    o.scales = reinterpret_cast<float*>(take(16 * sizeof(float)));
    if (out) *out = o;
    return off;
}

struct BwdWs {
    void* split;  // the GEMMs' split-K scratch
    uint8_t *dYq, *dGUq;
    void *g, *dGU;
    float* scales;
};

size_t bwd_layout(int64_t M, int64_t d, int64_t f, uint8_t* base, BwdWs* w) {
    const size_t Md = (size_t)M * d, Mf = (size_t)M * f;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        uint8_t* p = base ? base + off : nullptr;
        off += round_up(bytes);
        return p;
    };
    BwdWs o;
    o.split = take(gemm_split_workspace_bytes());
    o.dYq = take(Md);
    o.g = take(Mf * 2);
    o.dGU = take(2 * Mf * 2);
    o.dGUq = take(2 * Mf);
    o.scales = reinterpret_cast<float*>(take(8 * sizeof(float)));
    if (w) *w = o;
    return off;
}

__device__ __forceinline__ float sigmoid_f32(float x) {
    return __fdiv_rn(1.0f, __fadd_rn(1.0f, expf(-x)));
}

// dG = bf16(g U silu'(G)), dU = bf16(g silu(G)) for 8 consecutive columns per
// thread (16-byte loads of g, G, U), amax of dG|dU max-reduced into amax_bits.
__global__ void __launch_bounds__(256) swiglu_bwd_kernel(const uint16_t* __restrict__ g,
                                                         const uint16_t* __restrict__ GU,
                                                         int64_t M, int64_t f,
                                                         uint16_t* __restrict__ dGU,
                                                         unsigned int* __restrict__ amax_bits) {
    const int64_t vpr = f >> 3;
    const int64_t n = M * vpr;
    uint32_t m2 = 0;
    for (int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; v < n;
         v += (int64_t)gridDim.x * blockDim.x) {
        const int64_t row = v / vpr, j = (v - row * vpr) << 3;
        const int64_t gi = row * 2 * f + (j >> 7) * 256 + (j & 127);
        const uint4 gv = *reinterpret_cast<const uint4*>(g + row * f + j);
        const uint4 Gv = *reinterpret_cast<const uint4*>(GU + gi);
        const uint4 Uv = *reinterpret_cast<const uint4*>(GU + gi + 128);
        const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w}, Gw[4] = {Gv.x, Gv.y, Gv.z, Gv.w},
                       Uw[4] = {Uv.x, Uv.y, Uv.z, Uv.w};
        uint32_t dg[4], du[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float2 gg = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&gw[i]));
            float2 GG = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&Gw[i]));
            float2 UU = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&Uw[i]));
            const float s0 = sigmoid_f32(GG.x), s1 = sigmoid_f32(GG.y);
            const float ds0 = __fmul_rn(s0, __fadd_rn(1.0f, __fmul_rn(GG.x, __fsub_rn(1.0f, s0))));
            const float ds1 = __fmul_rn(s1, __fadd_rn(1.0f, __fmul_rn(GG.y, __fsub_rn(1.0f, s1))));
            const __nv_bfloat162 a = __floats2bfloat162_rn(__fmul_rn(__fmul_rn(gg.x, UU.x), ds0),
                                                           __fmul_rn(__fmul_rn(gg.y, UU.y), ds1));
            const __nv_bfloat162 b = __floats2bfloat162_rn(__fmul_rn(gg.x, __fmul_rn(GG.x, s0)),
                                                           __fmul_rn(gg.y, __fmul_rn(GG.y, s1)));
            dg[i] = *reinterpret_cast<const uint32_t*>(&a);
            du[i] = *reinterpret_cast<const uint32_t*>(&b);
            m2 = __vmaxu2(m2, dg[i] & 0x7FFF7FFFu);
            m2 = __vmaxu2(m2, du[i] & 0x7FFF7FFFu);
        }
        *reinterpret_cast<uint4*>(dGU + gi) = make_uint4(dg[0], dg[1], dg[2], dg[3]);
        *reinterpret_cast<uint4*>(dGU + gi + 128) = make_uint4(du[0], du[1], du[2], du[3]);
    }
    uint32_t m = max(m2 & 0xFFFFu, m2 >> 16);
    m = __reduce_max_sync(0xFFFFFFFFu, m);
    __shared__ uint32_t wm[8];
    if ((threadIdx.x & 31) == 0) wm[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t b = 0;
        for (int i = 0; i < 8; ++i) b = max(b, wm[i]);
        if (b) atomicMax(amax_bits, b << 16);
    }
}

#define LM_TRY(expr)                  \
    do {                              \
        lm_status _st = (expr);       \
        if (_st != LM_OK) return _st; \
    } while (0)

}  // namespace
}  // namespace lm

extern "C" {

size_t lm_swiglu_mlp_saved_bytes(int64_t M, int64_t d, int64_t f) {
    if (!lm::shape_ok(M, d, f)) return 0;
    return lm::saved_layout(M, d, f, nullptr, nullptr);
}

lm_status lm_swiglu_mlp_saved_carve(void* base, size_t bytes, int64_t M, int64_t d, int64_t f,
                                    lm_swiglu_saved* out) {
    if (!base || !out) return LM_ERR_INVALID_ARG;
    if (!lm::shape_ok(M, d, f)) return LM_ERR_UNSUPPORTED_SHAPE;
    if (reinterpret_cast<uintptr_t>(base) % lm::kAlign) return LM_ERR_ALIGNMENT;
    if (bytes < lm::saved_layout(M, d, f, nullptr, nullptr)) return LM_ERR_INVALID_ARG;
    lm::saved_layout(M, d, f, static_cast<uint8_t*>(base), out);
    return LM_OK;
}

size_t lm_swiglu_mlp_workspace_size(int64_t M, int64_t d, int64_t f) {
    if (!lm::shape_ok(M, d, f)) return 0;
    return lm::bwd_layout(M, d, f, nullptr, nullptr);
}

lm_status lm_swiglu_mlp_fwd(const void* X, const void* W_gu, const void* W_down, int64_t M,
                            int64_t d, int64_t f, void* Y, lm_swiglu_saved* sv, void* workspace,
                            size_t ws_bytes, lm_stream_t stream) {
    using namespace lm;
    if (!shape_ok(M, d, f)) return LM_ERR_UNSUPPORTED_SHAPE;
    if (workspace && reinterpret_cast<uintptr_t>(workspace) % kAlign) return LM_ERR_ALIGNMENT;
    // the workspace, when given, holds the GEMMs' split-K scratch at its start
    void* split = workspace && ws_bytes >= gemm_split_workspace_bytes() ? workspace : nullptr;
    const size_t sb = split ? gemm_split_workspace_bytes() : 0;
    // tensors with M rows may be NULL when M == 0 (an empty micro-batch)
    if (!W_gu || !W_down || !sv || !sv->Wguq || !sv->Wdq || !sv->scales ||
        (M > 0 && (!X || !Y || !sv->Xq || !sv->GU || !sv->h || !sv->hq)))
        return LM_ERR_INVALID_ARG;
    if (!all_aligned16({X, W_gu, W_down, Y, sv->Xq, sv->Wguq, sv->Wdq, sv->GU, sv->h, sv->hq}))
        return LM_ERR_ALIGNMENT;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    float* S = sv->scales;
    if (cudaMemsetAsync(S, 0, 16 * sizeof(float), s) != cudaSuccess) return LM_ERR_CUDA;
    // X, W_gu, W_down: one amax launch, one cast launch (slots zeroed above)
    const CastItem in[3] = {
        {X, M, d, d, nullptr, S + S_X, S + S_X + 1, S + S_X + 2, sv->Xq, nullptr},
        {W_gu, 2 * f, d, d, nullptr, S + S_WGU, S + S_WGU + 1, S + S_WGU + 2, sv->Wguq,
         nullptr},
        {W_down, d, f, f, nullptr, S + S_WD, S + S_WD + 1, S + S_WD + 2, sv->Wdq, nullptr}};
    LM_TRY(cast_set(in, 3, LM_FP8_E4M3, 0, true, s));
    if (M > 0)
        LM_TRY(gemm_dispatch(sv->Xq, LM_FP8_E4M3, sv->Wguq, LM_FP8_E4M3, M, 2 * f, d, 0u,
                             S + S_X + 2, S + S_WGU + 2, kEpiSwigluFwd, nullptr, sv->GU, sv->h,
                             S + S_H, nullptr, 0, stream));
    // Y = h W_down^T, h's codes cast (amax from the epilogue above) by the down
    // GEMM's side warps unit by unit ahead of its tiles, or by their own launch
    // first where that cannot be done
    SideCast hc = {sv->h, M, f, LM_FP8_E4M3, S + S_H, S + S_H, S + S_H + 1, S + S_H + 2, sv->hq};
    hc.feeds_a = 1;
    LM_TRY(gemm_dispatch(sv->hq, LM_FP8_E4M3, sv->Wdq, LM_FP8_E4M3, M, d, f, 0u, S + S_H + 2,
                         S + S_WD + 2, LM_EPI_NONE, nullptr, Y, nullptr, nullptr, split, sb,
                         stream, &hc));
    return LM_OK;
}

lm_status lm_swiglu_mlp_bwd(const void* dY, const lm_swiglu_saved* sv, int64_t M, int64_t d,
                            int64_t f, void* dX, void* dW_gu, void* dW_down, void* workspace,
                            size_t ws_bytes, lm_stream_t stream) {
    using namespace lm;
    if (!shape_ok(M, d, f)) return LM_ERR_UNSUPPORTED_SHAPE;
    // tensors with M rows may be NULL when M == 0 (the weight gradients are then zero)
    if (!sv || !dW_gu || !dW_down || !workspace || (M > 0 && (!dY || !dX)))
        return LM_ERR_INVALID_ARG;
    if (ws_bytes < bwd_layout(M, d, f, nullptr, nullptr)) return LM_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(workspace) % kAlign) return LM_ERR_ALIGNMENT;
    if (!sv->Wguq || !sv->Wdq || !sv->scales ||
        (M > 0 && (!sv->Xq || !sv->GU || !sv->h || !sv->hq)))
        return LM_ERR_INVALID_ARG;
    if (!all_aligned16({dY, dX, dW_gu, dW_down, sv->Xq, sv->Wguq, sv->Wdq, sv->GU, sv->h,
                        sv->hq}))
        return LM_ERR_ALIGNMENT;
    BwdWs w;
    bwd_layout(M, d, f, static_cast<uint8_t*>(workspace), &w);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const float* S = sv->scales;
    float* G = w.scales;
    if (cudaMemsetAsync(G, 0, 8 * sizeof(float), s) != cudaSuccess) return LM_ERR_CUDA;
    const CastItem dy = {dY, M, d, d, nullptr, G + S_DY, G + S_DY + 1, G + S_DY + 2, w.dYq,
                         nullptr};
    LM_TRY(cast_set(&dy, 1, LM_FP8_E5M2, 0, true, s));  // slot zeroed above
    // g = dY W_down (plain bf16), dW_down = dY^T h
    // (row-major codes read MN-major where the transpose is the operand)
    constexpr uint32_t B_MN = LM_GEMM_B_MN_MAJOR, AB_MN = LM_GEMM_A_MN_MAJOR | LM_GEMM_B_MN_MAJOR;
    const size_t sb = gemm_split_workspace_bytes();
    LM_TRY(lm_fp8_gemm_ex(w.dYq, LM_FP8_E5M2, sv->Wdq, LM_FP8_E4M3, M, f, d, B_MN, G + S_DY + 2,
                          S + S_WD + 2, LM_EPI_NONE, nullptr, w.g, nullptr, w.split, sb, stream));
    LM_TRY(lm_fp8_gemm_ex(w.dYq, LM_FP8_E5M2, sv->hq, LM_FP8_E4M3, d, f, M, AB_MN, G + S_DY + 2,
                          S + S_H + 2, LM_EPI_NONE, nullptr, dW_down, nullptr, w.split, sb,
                          stream));
    if (M > 0) {
        int grid = sm_count() * 8;
        if (grid <= 0) return LM_ERR_CUDA;
        timing_mark(s, 'w');
        swiglu_bwd_kernel<<<grid, 256, 0, s>>>(
            static_cast<const uint16_t*>(w.g), static_cast<const uint16_t*>(sv->GU), M, f,
            static_cast<uint16_t*>(w.dGU), reinterpret_cast<unsigned int*>(G + S_DGU));
        if (launch_status() != LM_OK) return LM_ERR_CUDA;
    }
    // dX = dGU W_gu (K = 2f), dGU's codes (amax from the elementwise kernel)
    // cast by the GEMM's side warps ahead of its tiles;  dW_gu = dGU^T X (K = M)
    SideCast gc = {w.dGU, M, 2 * f, LM_FP8_E5M2, G + S_DGU, G + S_DGU, G + S_DGU + 1,
                   G + S_DGU + 2, w.dGUq};
    gc.feeds_a = 1;
    LM_TRY(gemm_dispatch(w.dGUq, LM_FP8_E5M2, sv->Wguq, LM_FP8_E4M3, M, d, 2 * f, B_MN,
                         G + S_DGU + 2, S + S_WGU + 2, LM_EPI_NONE, nullptr, dX, nullptr, nullptr,
                         w.split, sb, stream, &gc));
    LM_TRY(lm_fp8_gemm_ex(w.dGUq, LM_FP8_E5M2, sv->Xq, LM_FP8_E4M3, 2 * f, d, M, AB_MN,
                          G + S_DGU + 2, S + S_X + 2, LM_EPI_NONE, nullptr, dW_gu, nullptr,
                          w.split, sb, stream));
    return LM_OK;
}

}  // extern "C"
