// lm_lmhead_ce.cu -- the LM head in FP8 inside a chunked, softcapped fused
// linear cross-entropy: the B*T x V logits never exist in full.
//
// The run's loss is Liger's fused linear cross-entropy with softcap 15,
// which chunks the head matmul so the logits are never materialised
// (decomputer.nl, "Het trainen van een 3.8B LLM tot 0.384 CORE voor $998",
// section "Doorvoer (Throughput) verhogen", fused linear cross-entropy
// bullet; "Appendix: De configuratie", loss).  Here the head's three GEMMs
// run in FP8 with dynamic tensorwise scaling like every other linear:
//
//   once:      W -> e4m3; amax/scale of X (whole tensor)
//   per chunk: X_c -> e4m3 at X's scale
//              logits_c = X_c W^T (bf16)
//              CE: z = c tanh(l / c), row loss, dlogits (bf16, in place) + amax
//              dlogits_c -> e5m2, no reduction pass
//              dX_c = dlogits_c W        (K = V; W's codes read MN-major)
//              dW  += fp32(dlogits_c^T X_c)   (both read MN-major; TMA
//                                              reduce-add epilogue)
// Only row-major codes are written: the GEMMs that contract over a tensor's
// rows read its codes MN-major.
//   end:       mean loss = deterministic fp64 sum of the row losses / M
#include <cuda_bf16.h>

#include "lm_internal.h"

namespace lm {
namespace {

constexpr size_t kAlign = 256;
size_t round_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }
constexpr int kCeThreads = 512;

struct Ws {
    float* scales;  // {amax, scale, inv, 0} for X, W, dlogits
    uint8_t *Wq, *Xq, *dLq;
    uint16_t* logits;
    float* loss_rows;
    // the dX GEMM's ready bits, one per 256-row x 128-column unit of the
    // dlogits codes that its side warps cast ahead of its tiles
    unsigned int* ready;
    size_t ready_bytes;
};

size_t layout(int64_t M, int64_t d, int64_t V, int64_t C, uint8_t* base, Ws* w) {
    size_t off = 0;
    auto take = [&](size_t bytes) {
        uint8_t* p = base ? base + off : nullptr;
        off += round_up(bytes);
        return p;
    };
    Ws o;
    o.scales = reinterpret_cast<float*>(take(16 * sizeof(float)));
    o.Wq = take((size_t)V * d);
    o.Xq = take((size_t)C * d);
    o.logits = reinterpret_cast<uint16_t*>(take((size_t)C * V * 2));
    o.dLq = take((size_t)C * V);
    // ready words of (C / 256) x (V / 128) units, then an 8-byte-aligned
    // 64-bit counter (the GEMM's layout for a side cast feeding A)
    const int64_t ready_words = ((C + 255) / 256) * ((((V + 127) / 128) + 31) / 32);
    o.ready_bytes = (size_t)(((ready_words + 1) & ~int64_t(1)) + 2) * 4;
    o.ready = reinterpret_cast<unsigned int*>(take(o.ready_bytes));
    o.loss_rows = reinterpret_cast<float*>(take((size_t)M * sizeof(float)));  // the tail
    if (w) *w = o;
    return off;
}

bool shapes_ok(int64_t M, int64_t d, int64_t V, int64_t C) {
    return M >= 0 && d > 0 && V > 0 && C > 0 && M % 16 == 0 && d % 16 == 0 && V % 16 == 0 &&
           C % 16 == 0 && V < (int64_t(1) << 31) && C < (int64_t(1) << 31);
}

__device__ __forceinline__ float softcap_f(float l, float c) {
    return __fmul_rn(c, tanhf(__fdiv_rn(l, c)));
}

// combine two (max, sum of exp(z - max)) pairs
__device__ __forceinline__ void lse_combine(float& m, float& s, float m2, float s2) {
    const float mm = fmaxf(m, m2);
    if (mm == -INFINITY) return;
    s = __fadd_rn(__fmul_rn(s, expf(m - mm)), __fmul_rn(s2, expf(m2 - mm)));
    m = mm;
}

// One block per row of bf16 logits (V entries, V % 8 == 0).  Writes the row
// loss and, in place, dlogits = bf16((p - onehot) (1 - (z/c)^2) inv_count);
// max |dlogits| is max-reduced into amax_bits.
__global__ void __launch_bounds__(kCeThreads)
    softcap_ce_kernel(uint16_t* __restrict__ logits, const int32_t* __restrict__ labels, int V,
                      float c, float inv_count, float* __restrict__ loss_rows,
                      unsigned int* __restrict__ amax_bits, unsigned int* err) {
    const int64_t row = blockIdx.x;
    uint4* lv = reinterpret_cast<uint4*>(logits + row * (int64_t)V);
    const int nv = V >> 3;
    int label = labels[row];
    const bool label_ok = (unsigned)label < (unsigned)V;  // never read outside the row
    if (!label_ok) {
        if (threadIdx.x == 0) atomicCAS(err, 0u, 0x401u);
        label = -1;  // no target: loss = lse, no one-hot term
    }
    float m = -INFINITY, s = 0.f;
    for (int v = threadIdx.x; v < nv; v += kCeThreads) {
        const uint4 x = lv[v];
        const uint32_t w[4] = {x.x, x.y, x.z, x.w};
        float z[8], zm = -INFINITY;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            z[2 * i] = softcap_f(__uint_as_float(w[i] << 16), c);
            z[2 * i + 1] = softcap_f(__uint_as_float(w[i] & 0xFFFF0000u), c);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) zm = fmaxf(zm, z[i]);
        float zs = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) zs = __fadd_rn(zs, expf(z[i] - zm));
        lse_combine(m, s, zm, zs);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float m2 = __shfl_xor_sync(0xFFFFFFFFu, m, o);
        const float s2 = __shfl_xor_sync(0xFFFFFFFFu, s, o);
        lse_combine(m, s, m2, s2);
    }
    __shared__ float sm[kCeThreads / 32], ss[kCeThreads / 32];
    __shared__ float s_lse;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) {
        sm[warp] = m;
        ss[warp] = s;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        float M0 = sm[0], S0 = ss[0];
        for (int i = 1; i < kCeThreads / 32; ++i) lse_combine(M0, S0, sm[i], ss[i]);
        const float lse = __fadd_rn(M0, logf(S0));
        s_lse = lse;
        const float zl =
            label_ok ? softcap_f(__uint_as_float((uint32_t)logits[row * (int64_t)V + label] << 16), c)
                     : 0.0f;
        loss_rows[row] = __fsub_rn(lse, zl);
    }
    __syncthreads();
    const float lse = s_lse;
    const float inv_c = __fdiv_rn(1.0f, c);
    uint32_t m2 = 0;
    for (int v = threadIdx.x; v < nv; v += kCeThreads) {
        const uint4 x = lv[v];
        const uint32_t w[4] = {x.x, x.y, x.z, x.w};
        uint32_t o[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float r[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const float l = __uint_as_float(h ? (w[i] & 0xFFFF0000u) : (w[i] << 16));
                const float z = softcap_f(l, c);
                float p = expf(z - lse);
                if (8 * v + 2 * i + h == label) p = __fsub_rn(p, 1.0f);
                const float t = __fmul_rn(z, inv_c);
                r[h] = __fmul_rn(__fmul_rn(p, __fsub_rn(1.0f, __fmul_rn(t, t))), inv_count);
            }
            const __nv_bfloat162 b = __floats2bfloat162_rn(r[0], r[1]);
            o[i] = *reinterpret_cast<const uint32_t*>(&b);
            m2 = __vmaxu2(m2, o[i] & 0x7FFF7FFFu);
        }
        lv[v] = make_uint4(o[0], o[1], o[2], o[3]);
    }
    uint32_t mm = max(m2 & 0xFFFFu, m2 >> 16);
    mm = __reduce_max_sync(0xFFFFFFFFu, mm);
    __shared__ uint32_t wm[kCeThreads / 32];
    if (lane == 0) wm[warp] = mm;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t b = 0;
        for (int i = 0; i < kCeThreads / 32; ++i) b = max(b, wm[i]);
        if (b) atomicMax(amax_bits, b << 16);
    }
}

// ---------------------------------------------------------------------
// The same computation with the softcap written through r = sigmoid(-2y),
// y = l / c: then tanh(y) = 1 - 2r, z = c - 2cr, exp(z - c) = exp(-2cr) and
// the softcap's derivative 1 - tanh(y)^2 = 4r(1 - r).  Every term exp(z - c)
// is at most 1, so the row's log-sum-exp needs no running maximum:
// lse = c + log(sum exp(-2cr)).  Per logit and pass that is two hardware
// transcendentals (a base-2 exponential and a reciprocal) and one base-2
// exponential on the FMA pipe (ex2_fma) instead of a division, tanhf and expf.  Used for softcaps up to kFastCeMaxCap, where
// exp(-2c) stays a normal fp32 number (no term can flush to zero) and the
// exponent of every exp(z - c) term lies in [-2 log2(e) kFastCeMaxCap, 0] =
// [-115.4, 0], inside the range of ex2_fma.
constexpr float kFastCeMaxCap = 40.0f;

__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Two fp32 lanes in one 64-bit register, and the packed f32x2 arithmetic of
// sm_100 on them: each lane is one IEEE round-to-nearest operation, exactly
// the scalar __fadd_rn / __fsub_rn / __fmul_rn / __fmaf_rn, at half the
// instructions.
__device__ __forceinline__ uint64_t pk2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void up2(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t sub2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}

// 2^x for x in [-116, 0] on the FMA and integer pipes, two lanes at a time.
// x = n + f with n = rint(x) and f in [-1/2, 1/2]: adding 1.5 * 2^23 + 127
// leaves n + 127 in the sum's low bits, which shifted into the exponent field
// are the bits of 2^n; 2^f from a degree-5 polynomial, a Remez minimax fit of
// the relative error on [-1/2, 1/2] made for this kernel (at most 1.6e-7 with
// these fp32 coefficients); 2^f 2^n is one exact multiply.  The
// kernel's exp(z - c) terms, whose argument lies in [-2 log2(e) c, 0], use it
// instead of ex2.approx, so that the transcendental pipe (left with the
// softcap's ex2 and rcp) and the FMA pipe share the work.
constexpr float kExp2C0 = 1.0000001192092896f, kExp2C1 = 0.6931469440460205f,
                kExp2C2 = 0.24022120237350464f, kExp2C3 = 0.05550713092088699f,
                kExp2C4 = 0.009675540961325169f, kExp2C5 = 0.0013276472454890609f;

__device__ __forceinline__ uint64_t ex2_fma2(uint64_t x) {
    const uint64_t magic = pk2(12583039.0f, 12583039.0f);  // 1.5 * 2^23 + 127
    const uint64_t t = add2(x, magic);  // rint(x) + 127 in the low bits of each lane
    const uint64_t f = sub2(x, sub2(t, magic));
    uint64_t p = fma2(pk2(kExp2C5, kExp2C5), f, pk2(kExp2C4, kExp2C4));
    p = fma2(p, f, pk2(kExp2C3, kExp2C3));
    p = fma2(p, f, pk2(kExp2C2, kExp2C2));
    p = fma2(p, f, pk2(kExp2C1, kExp2C1));
    p = fma2(p, f, pk2(kExp2C0, kExp2C0));
    float t0, t1;
    up2(t, t0, t1);
    return mul2(p, pk2(__int_as_float(__float_as_int(t0) << 23),
                       __int_as_float(__float_as_int(t1) << 23)));
}

// r = 1 / (exp(2 l / c) + 1) for the two logits of a bf16 pair w (low half
// first); k2 = {2 log2(e) / c} in both lanes
__device__ __forceinline__ uint64_t softcap_r2(uint32_t w, uint64_t k2, uint64_t one) {
    float e0, e1;
    up2(mul2(pk2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u)), k2), e0, e1);
    float d0, d1;
    up2(add2(pk2(ex2_approx(e0), ex2_approx(e1)), one), d0, d1);
    return pk2(rcp_approx(d0), rcp_approx(d1));
}

// r = 1 / (exp(2 l / c) + 1); k2 = 2 log2(e) / c
__device__ __forceinline__ float softcap_r(float l, float k2) {
    return rcp_approx(__fadd_rn(ex2_approx(__fmul_rn(l, k2)), 1.0f));
}

__global__ void __launch_bounds__(kCeThreads)
    softcap_ce_fast_kernel(uint16_t* __restrict__ logits, const int32_t* __restrict__ labels,
                           int V, float c, float inv_count, float* __restrict__ loss_rows,
                           unsigned int* __restrict__ amax_bits, unsigned int* err) {
    const int64_t row = blockIdx.x;
    uint4* lv = reinterpret_cast<uint4*>(logits + row * (int64_t)V);
    const int nv = V >> 3;
    int label = labels[row];
    const bool label_ok = (unsigned)label < (unsigned)V;  // never read outside the row
    if (!label_ok) {
        if (threadIdx.x == 0) atomicCAS(err, 0u, 0x401u);
        label = -1;  // no target: loss = lse, no one-hot term
    }
    const float log2e = 1.4426950408889634f;
    const float k2 = __fdiv_rn(2.0f * log2e, c);  // exp(2y) = 2^(l k2)
    const float kz = -2.0f * log2e * c;           // exp(z - c) = 2^(kz r)
    const uint64_t k2x2 = pk2(k2, k2), kzx2 = pk2(kz, kz), one2 = pk2(1.0f, 1.0f);
    // each thread keeps two partial sums (even and odd logits), added at the end
    uint64_t sum2 = pk2(0.f, 0.f);
    for (int v = threadIdx.x; v < nv; v += kCeThreads) {
        const uint4 x = lv[v];
        const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
            sum2 = add2(sum2, ex2_fma2(mul2(kzx2, softcap_r2(w[i], k2x2, one2))));
    }
    float s0, s1;
    up2(sum2, s0, s1);
    float sum = __fadd_rn(s0, s1);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum = __fadd_rn(sum, __shfl_xor_sync(0xFFFFFFFFu, sum, o));
    __shared__ float ws[kCeThreads / 32];
    __shared__ float s_inv_sum;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) ws[warp] = sum;
    __syncthreads();
    if (threadIdx.x == 0) {
        float S = 0.f;
        for (int i = 0; i < kCeThreads / 32; ++i) S = __fadd_rn(S, ws[i]);
        const float lse = __fadd_rn(c, logf(S));
        float zl = 0.0f;
        if (label_ok) {
            const float l = __uint_as_float((uint32_t)logits[row * (int64_t)V + label] << 16);
            zl = __fsub_rn(c, __fmul_rn(2.0f * c, softcap_r(l, k2)));
        }
        loss_rows[row] = __fsub_rn(lse, zl);
        s_inv_sum = __fdiv_rn(1.0f, S);
    }
    __syncthreads();
    const float inv_sum = s_inv_sum;
    const float g4 = 4.0f * inv_count;  // (1 - t^2) = 4 r (1 - r), times 1/M
    const uint64_t invx2 = pk2(inv_sum, inv_sum), g4x2 = pk2(g4, g4);
    uint32_t m2 = 0;
    for (int v = threadIdx.x; v < nv; v += kCeThreads) {
        const uint4 x = lv[v];
        const uint32_t w[4] = {x.x, x.y, x.z, x.w};
        uint32_t o[4];
        const bool target_here = (unsigned)(label - 8 * v) < 8u;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint64_t r = softcap_r2(w[i], k2x2, one2);
            uint64_t p = mul2(ex2_fma2(mul2(kzx2, r)), invx2);  // exp(z - lse)
            const int base = 8 * v + 2 * i;
            if (target_here && (unsigned)(label - base) < 2u) {  // the target logit: p - 1
                float p0, p1;
                up2(p, p0, p1);
                if (label == base) p0 = __fsub_rn(p0, 1.0f);
                else p1 = __fsub_rn(p1, 1.0f);
                p = pk2(p0, p1);
            }
            float g0, g1;
            up2(mul2(mul2(p, mul2(r, sub2(one2, r))), g4x2), g0, g1);
            const __nv_bfloat162 b = __floats2bfloat162_rn(g0, g1);
            o[i] = *reinterpret_cast<const uint32_t*>(&b);
            m2 = __vmaxu2(m2, o[i] & 0x7FFF7FFFu);
        }
        lv[v] = make_uint4(o[0], o[1], o[2], o[3]);
    }
    uint32_t mm = max(m2 & 0xFFFFu, m2 >> 16);
    mm = __reduce_max_sync(0xFFFFFFFFu, mm);
    __shared__ uint32_t wm[kCeThreads / 32];
    if (lane == 0) wm[warp] = mm;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t b = 0;
        for (int i = 0; i < kCeThreads / 32; ++i) b = max(b, wm[i]);
        if (b) atomicMax(amax_bits, b << 16);
    }
}

// mean of the row losses: fixed-order fp64 sum in one block (deterministic)
__global__ void __launch_bounds__(1024) mean_loss_kernel(const float* __restrict__ rows, int64_t n,
                                                         float* __restrict__ out) {
    __shared__ double part[1024];
    double acc = 0.0;
    for (int64_t i = threadIdx.x; i < n; i += 1024) acc += (double)rows[i];
    part[threadIdx.x] = acc;
    __syncthreads();
    for (int w = 512; w > 0; w >>= 1) {
        if ((int)threadIdx.x < w) part[threadIdx.x] += part[threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x == 0) *out = n ? (float)(part[0] / (double)n) : 0.0f;
}

#define LM_TRY(expr)                  \
    do {                              \
        lm_status _st = (expr);       \
        if (_st != LM_OK) return _st; \
    } while (0)

}  // namespace
}  // namespace lm

extern "C" {

size_t lm_fp8_lmhead_ce_workspace_size(int64_t M, int64_t d, int64_t V, int64_t chunk) {
    if (!lm::shapes_ok(M, d, V, chunk)) return 0;
    return lm::layout(M, d, V, chunk, nullptr, nullptr);
}

lm_status lm_fp8_lmhead_ce(const void* X, const void* W, const int32_t* labels, int64_t M,
                           int64_t d, int64_t V, int64_t chunk, float softcap, float* loss_out,
                           void* dX, float* dW, void* workspace, size_t ws_bytes,
                           lm_stream_t stream) {
    using namespace lm;
    if (!shapes_ok(M, d, V, chunk)) return LM_ERR_UNSUPPORTED_SHAPE;
    // X, labels and dX may be NULL when M == 0 (no tokens: loss 0, dW unchanged)
    if (!W || !loss_out || !dW || !workspace || (M > 0 && (!X || !labels || !dX)))
        return LM_ERR_INVALID_ARG;
    if (!(softcap > 0.f)) return LM_ERR_INVALID_ARG;
    if (ws_bytes < layout(M, d, V, chunk, nullptr, nullptr)) return LM_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(workspace) % kAlign) return LM_ERR_ALIGNMENT;
    if (!aligned16(X) || !aligned16(W) || !aligned16(dX) || !aligned16(dW)) return LM_ERR_ALIGNMENT;
    unsigned int* err = device_error_word();
    if (!err) return LM_ERR_CUDA;
    Ws w;
    layout(M, d, V, chunk, static_cast<uint8_t*>(workspace), &w);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    float* SX = w.scales;
    float* SW = w.scales + 4;
    float* SL = w.scales + 8;
    if (cudaMemsetAsync(w.scales, 0, 16 * sizeof(float), s) != cudaSuccess) return LM_ERR_CUDA;
    // W cast, and X's amax and scale over the whole tensor (no codes yet), with
    // one amax launch for both (slots zeroed above)
    const CastItem in[2] = {{W, V, d, d, nullptr, SW, SW + 1, SW + 2, w.Wq, nullptr},
                            {X, M, d, d, nullptr, SX, SX + 1, SX + 2, nullptr, nullptr}};
    LM_TRY(cast_set(in, 2, LM_FP8_E4M3, 0, true, s));
    const uint16_t* Xb = static_cast<const uint16_t*>(X);
    uint16_t* dXb = static_cast<uint16_t*>(dX);
    for (int64_t c0 = 0; c0 < M; c0 += chunk) {
        const int64_t rows = (M - c0) < chunk ? (M - c0) : chunk;
        LM_TRY(lm_fp8_amax_scale_cast(Xb + c0 * d, rows, d, d, LM_FP8_E4M3, 0, SX, SX, SX + 1,
                                      SX + 2, w.Xq, nullptr, stream));
        LM_TRY(lm_fp8_gemm(w.Xq, LM_FP8_E4M3, w.Wq, LM_FP8_E4M3, rows, V, d, SX + 2, SW + 2,
                           LM_EPI_NONE, nullptr, w.logits, nullptr, stream));
        if (cudaMemsetAsync(SL, 0, 4 * sizeof(float), s) != cudaSuccess) return LM_ERR_CUDA;
        timing_mark(s, 'e');
        if (softcap <= kFastCeMaxCap)
            softcap_ce_fast_kernel<<<(unsigned)rows, kCeThreads, 0, s>>>(
                w.logits, labels + c0, (int)V, softcap, (float)(1.0 / (double)M),
                w.loss_rows + c0, reinterpret_cast<unsigned int*>(SL), err);
        else
            softcap_ce_kernel<<<(unsigned)rows, kCeThreads, 0, s>>>(
                w.logits, labels + c0, (int)V, softcap, (float)(1.0 / (double)M),
                w.loss_rows + c0, reinterpret_cast<unsigned int*>(SL), err);
        if (launch_status() != LM_OK) return LM_ERR_CUDA;
        // dX = dL W (W [V x d] read MN-major), dL's codes cast by the GEMM's side
        // warps unit by unit ahead of its tiles (the workspace holds only their
        // ready bits, so no split tail); dW += dL^T X (both read MN-major)
        SideCast lc = {w.logits, rows, V, LM_FP8_E5M2, SL, SL, SL + 1, SL + 2, w.dLq};
        lc.feeds_a = 1;
        LM_TRY(gemm_dispatch(w.dLq, LM_FP8_E5M2, w.Wq, LM_FP8_E4M3, rows, d, V,
                             LM_GEMM_B_MN_MAJOR, SL + 2, SW + 2, LM_EPI_NONE, nullptr,
                             dXb + c0 * d, nullptr, nullptr, w.ready, w.ready_bytes, stream,
                             &lc));
        LM_TRY(lm_fp8_gemm_ex(w.dLq, LM_FP8_E5M2, w.Xq, LM_FP8_E4M3, V, d, rows,
                              LM_GEMM_A_MN_MAJOR | LM_GEMM_B_MN_MAJOR, SL + 2, SX + 2,
                              LM_EPI_ACCUM_F32, nullptr, dW, nullptr, nullptr, 0, stream));
    }
    timing_mark(s, 'l');
    mean_loss_kernel<<<1, 1024, 0, s>>>(w.loss_rows, M, loss_out);
    return launch_status();
}

}  // extern "C"
