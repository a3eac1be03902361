// lm_cast_math.cuh -- the arithmetic of the dynamic tensorwise FP8 cast,
// shared by the cast kernels and by the GEMM kernel's side cast (a cast that
// runs in extra warps of a GEMM launch):
//   scale = fp32(fmax / max(amax, 1e-12))   (one IEEE division)
//   code  = fp8_satfinite_rne(fp32(x * scale))   (one fp32 multiply)
// with e4m3 (fmax 448) for activations and weights and e5m2 (fmax 57344)
// for gradients (decomputer.nl, "Het trainen van een 3.8B LLM tot 0.384
// CORE voor $998", section "Vroege experimenten" item 4: FP8 with dynamic
// tensorwise scaling).
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "lm_fp8.h"

namespace lm {
namespace {

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}


// Two packed bf16 x -> two packed h = bf16(relu(x)^2): a NaN-propagating max
// with 0 (relu(NaN) stays NaN), then one bf16x2 multiply, which rounds the
// exact square once to bf16.
__device__ __forceinline__ uint32_t relu2_bf16x2(uint32_t w) {
    const __nv_bfloat162 x = *reinterpret_cast<const __nv_bfloat162*>(&w);
    const __nv_bfloat162 r = __hmax2_nan(x, __float2bfloat162_rn(0.0f));
    const __nv_bfloat162 h = __hmul2(r, r);
    return *reinterpret_cast<const uint32_t*>(&h);
}

// Two fp32 values -> two saturated RNE FP8 codes (lo in the low byte).
template <int FMT>
__device__ __forceinline__ uint32_t cvt_pair(float lo, float hi) {
    uint16_t r;
    if (FMT == LM_FP8_E4M3)
        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    else
        asm("cvt.rn.satfinite.e5m2x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// Two packed bf16 -> two fp32 products fp32(v * scale), one packed f32x2
// multiply (two IEEE round-to-nearest fp32 multiplies); scale2 = {scale, scale}.
__device__ __forceinline__ void mul_bf16x2_f32(uint32_t w, uint64_t scale2, float& lo, float& hi) {
    uint64_t x, r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(x) : "r"(w << 16), "r"(w & 0xFFFF0000u));
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(x), "l"(scale2));
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(r));
}

__device__ __forceinline__ uint64_t splat_f32x2(float s) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %1};" : "=l"(r) : "f"(s));
    return r;
}

// 8 bf16 (16 bytes) -> 8 codes (8 bytes), code = fp8(fp32(v * scale)).
template <int FMT, bool RELU2>
__device__ __forceinline__ uint2 convert8(uint4 v, float scale) {
    const uint64_t scale2 = splat_f32x2(scale);
    uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t p[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float lo, hi;
        mul_bf16x2_f32(RELU2 ? relu2_bf16x2(w[i]) : w[i], scale2, lo, hi);
        p[i] = cvt_pair<FMT>(lo, hi);
    }
    return make_uint2(p[0] | (p[1] << 16), p[2] | (p[3] << 16));
}

// fp32 scale of a tensor from its amax (a NaN amax gives a NaN scale).
__device__ __forceinline__ float scale_from_amax(float amax, float fmax) {
    const float a = amax < 1e-12f ? 1e-12f : amax;
    return __fdiv_rn(fmax, a);
}

}  // namespace
}  // namespace lm
