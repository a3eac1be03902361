// lm_rmsnorm.cu -- the producer of the FP8 GEMM input: RMSNorm -> amax ->
// dynamic e4m3 cast (row-major codes, and the transposed copy on request).
//
// The model normalises with RMSNorm (rms_norm_eps 1e-6; PyTorch's
// F.rms_norm) before its linears (decomputer.nl, "Het trainen van een 3.8B
// LLM tot 0.384 CORE voor $998", "Appendix: De configuratie"; section "Wat
// niet werkte", Liger RMSNorm bullet).  Producing X's amax in the same pass
// that writes X lets the cast skip its reduction pass: 8 bytes per element
// move instead of 10 (norm 2+2, cast 2+2+1+1 with the transposed copy; 7
// instead of 9 without it), and the cast re-reads X while much of it is
// still in L2.
//
// One warp per row: a first sweep sums squares in fp32, the second (the row
// is then in L1) writes X = bf16(x * inv_rms * w) with 16-byte stores and
// keeps the max |X|; one atomicMax per block.
#include <cuda_bf16.h>

#include "lm_internal.h"

namespace lm {
namespace {

constexpr int kRowsPerBlock = 8;

__device__ __forceinline__ float lo_f(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float hi_f(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__global__ void __launch_bounds__(32 * kRowsPerBlock)
    rmsnorm_amax_kernel(const uint16_t* __restrict__ R, const uint16_t* __restrict__ w, int rows,
                        int cols, float eps, uint16_t* __restrict__ X,
                        unsigned int* __restrict__ amax_bits) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row = blockIdx.x * kRowsPerBlock + warp;
    uint32_t m = 0;
    if (row < rows) {
        const uint4* src = reinterpret_cast<const uint4*>(R + (int64_t)row * cols);
        const int nv = cols >> 3;
        float ss = 0.f;
        for (int v = lane; v < nv; v += 32) {
            const uint4 x = src[v];
            const uint32_t xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float a = lo_f(xs[i]), b = hi_f(xs[i]);
                ss = __fmaf_rn(a, a, ss);
                ss = __fmaf_rn(b, b, ss);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, o);
        const float inv = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(__fdiv_rn(ss, (float)cols), eps)));
        const uint4* wv = reinterpret_cast<const uint4*>(w);
        uint4* dst = reinterpret_cast<uint4*>(X + (int64_t)row * cols);
        for (int v = lane; v < nv; v += 32) {
            const uint4 x = src[v];
            const uint32_t xs[4] = {x.x, x.y, x.z, x.w};
            uint32_t ws[4] = {0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u};  // 1.0
            if (w) {
                const uint4 g = wv[v];
                ws[0] = g.x, ws[1] = g.y, ws[2] = g.z, ws[3] = g.w;
            }
            uint32_t o[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const __nv_bfloat162 y = __floats2bfloat162_rn(
                    __fmul_rn(__fmul_rn(lo_f(xs[i]), inv), lo_f(ws[i])),
                    __fmul_rn(__fmul_rn(hi_f(xs[i]), inv), hi_f(ws[i])));
                o[i] = *reinterpret_cast<const uint32_t*>(&y);
                m = __vmaxu2(m, o[i] & 0x7FFF7FFFu);
            }
            dst[v] = make_uint4(o[0], o[1], o[2], o[3]);
        }
    }
    m = max(m & 0xFFFFu, m >> 16);
    m = __reduce_max_sync(0xFFFFFFFFu, m);
    __shared__ uint32_t wm[kRowsPerBlock];
    if (lane == 0) wm[warp] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t b = 0;
#pragma unroll
        for (int i = 0; i < kRowsPerBlock; ++i) b = max(b, wm[i]);
        if (b) atomicMax(amax_bits, b << 16);
    }
}

}  // namespace
}  // namespace lm

extern "C" lm_status lm_rmsnorm_fp8_cast(const void* R, const void* weight, int64_t rows,
                                         int64_t cols, float eps, lm_fp8_format fmt, void* X,
                                         float* amax_out, float* scale_out,
                                         float* inv_scale_out, uint8_t* q, uint8_t* qT,
                                         lm_stream_t stream) {
    using namespace lm;
    if (fmt != LM_FP8_E4M3 && fmt != LM_FP8_E5M2) return LM_ERR_UNSUPPORTED_FORMAT;
    if (rows < 0 || cols <= 0 || !(eps >= 0.f)) return LM_ERR_INVALID_ARG;
    if (!amax_out || !scale_out || !inv_scale_out || (rows > 0 && (!R || !X)))
        return LM_ERR_INVALID_ARG;
    if (cols % 16 != 0 || (qT && rows % 16 != 0)) return LM_ERR_UNSUPPORTED_SHAPE;
    if (rows >= (int64_t(1) << 31) || cols >= (int64_t(1) << 31)) return LM_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(R) || !aligned16(weight) || !aligned16(X) || !aligned16(q) || !aligned16(qT))
        return LM_ERR_ALIGNMENT;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (rows > 0) timing_mark(s, 'n');
    if (cudaMemsetAsync(amax_out, 0, sizeof(float), s) != cudaSuccess) return LM_ERR_CUDA;
    if (rows > 0) {
        const int grid = (int)((rows + kRowsPerBlock - 1) / kRowsPerBlock);
        rmsnorm_amax_kernel<<<grid, 32 * kRowsPerBlock, 0, s>>>(
            static_cast<const uint16_t*>(R), static_cast<const uint16_t*>(weight), (int)rows,
            (int)cols, eps, static_cast<uint16_t*>(X), reinterpret_cast<unsigned int*>(amax_out));
        if (launch_status() != LM_OK) return LM_ERR_CUDA;
    }
    return lm_fp8_amax_scale_cast(X, rows, cols, cols, fmt, 0, amax_out, amax_out, scale_out,
                                  inv_scale_out, q, qT, stream);
}
