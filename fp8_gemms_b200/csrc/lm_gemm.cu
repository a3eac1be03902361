// lm_gemm.cu -- FP8 GEMM on sm_100a tensor cores (tcgen05), D = epi(A B^T s).
//
// The pages run all three GEMMs of each linear in FP8 with one fp32 scale
// per operand, bf16 out (decomputer.nl, "Het trainen van een 3.8B LLM tot
// 0.384 CORE voor $998", section "Doorvoer (Throughput) verhogen", FP8
// bullet; manulx.blog names the library call, torch._scaled_mm).  This is
// a kernel of our own for B200 instead of that library call:
//
//  * persistent grid, one CTA per SM, tiles of 128 x 256 outputs visited in
//    groups of 16 M-blocks so that concurrently running CTAs share A and B
//    panels in L2;
//  * warp 0: one thread issues TMA tile loads (128-byte swizzle, K-major) into
//    a 4-stage shared-memory ring guarded by full/empty mbarriers;
//  * warp 1: one thread issues tcgen05.mma kind::f8f6f4 (128 x 256 x 32 per
//    instruction) into a TMEM fp32 accumulator; two accumulators of 256
//    columns (all 512 TMEM columns) let the epilogue of one tile overlap the
//    main loop of the next;
//  * warps 2-5: epilogue -- tcgen05.ld of 32 columns at a time, dequant scale,
//    relu^2 (forward) or 2 relu(H) g (backward), bf16 stores, and the amax of
//    what the next cast consumes (atomicMax on fp32 bits, order independent).
#include <cuda_bf16.h>

#include "lm_internal.h"
#include "lm_ptx.cuh"

namespace lm {
namespace {

constexpr int BM = 128, BN = 256, BK = 128;  // BK in bytes = FP8 elements
constexpr int UMMA_K = 32;                   // K per tcgen05.mma for 8-bit inputs
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK;
constexpr int B_BYTES = BN * BK;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int NUM_THREADS = 192;
constexpr int NUM_EPI_THREADS = 128;
constexpr uint32_t TMEM_COLS = 2 * BN;
constexpr int GROUP_M = 16;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 256;

// codes recorded in the device error word when a bounded wait runs out
enum : unsigned { W_EMPTY = 0x101, W_TEMPTY = 0x102, W_FULL = 0x103, W_DRAIN = 0x104,
                  W_TFULL = 0x105, W_LOADS = 0x106 };

struct GemmArgs {
    int M, N, num_mb, num_nb, num_kb, num_tiles;
    const float* inv_a;
    const float* inv_b;
    const uint16_t* aux;
    uint16_t* D;
    float* amax_out;
    unsigned int* err;
    uint32_t idesc;
};

__device__ __forceinline__ void tile_coords(int t, int num_mb, int num_nb, int& mb, int& nb) {
    const int per_group = GROUP_M * num_nb;
    const int g = t / per_group;
    const int first = g * GROUP_M;
    const int gsize = min(GROUP_M, num_mb - first);
    const int local = t - g * per_group;
    mb = first + local % gsize;
    nb = local / gsize;
}

__device__ __forceinline__ uint32_t bf16_bits(float v) {
    return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v));
}

template <int EPI>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_fp8_kernel(const __grid_constant__ CUtensorMap tmA,
                    const __grid_constant__ CUtensorMap tmB, const GemmArgs args) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
    uint8_t* sA = smem;
    uint8_t* sB = smem + STAGES * A_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
    uint64_t* full = bars;
    uint64_t* empty = bars + STAGES;
    uint64_t* tfull = bars + 2 * STAGES;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], NUM_EPI_THREADS);
        }
        mbar_init(drain, 1);
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------------------------------------- TMA producer
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < args.num_tiles && ok; t += gridDim.x) {
                int mb, nb;
                tile_coords(t, args.num_mb, args.num_nb, mb, nb);
                for (int kb = 0; kb < args.num_kb; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, args.err, W_EMPTY)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[stage], STAGE_BYTES);
                    tma_load_2d(smem_addr(sA + stage * A_BYTES), &tmA, &full[stage], kb * BK,
                                mb * BM);
                    tma_load_2d(smem_addr(sB + stage * B_BYTES), &tmB, &full[stage], kb * BK,
                                nb * BN);
                    ++issued;
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // every load this CTA issued has landed before shared memory is
            // released (already true on the normal path: the MMA waited)
            for (int s = 0; s < STAGES; ++s) {
                const uint32_t n = issued / STAGES + ((uint32_t)s < issued % STAGES ? 1u : 0u);
                if (n) mbar_wait(&full[s], (n - 1) & 1u, args.err, W_LOADS);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------ MMA issuer
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < args.num_tiles && ok; t += gridDim.x) {
                if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, args.err, W_TEMPTY)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
                for (int kb = 0; kb < args.num_kb; ++kb) {
                    if (!mbar_wait(&full[stage], phase, args.err, W_FULL)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t ad = smem_desc_k128(smem_addr(sA + stage * A_BYTES));
                    const uint64_t bd = smem_desc_k128(smem_addr(sB + stage * B_BYTES));
#pragma unroll
                    for (int kk = 0; kk < BK / UMMA_K; ++kk)
                        mma_fp8(d_tmem, ad + (uint64_t)(kk * UMMA_K / 16),
                                bd + (uint64_t)(kk * UMMA_K / 16), args.idesc,
                                (kb | kk) != 0 ? 1u : 0u);
                    mma_commit(&empty[stage]);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                mma_commit(&tfull[acc]);
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1u;
            }
            // all MMAs retired before TMEM is deallocated
            mma_commit(drain);
            mbar_wait(drain, 0, args.err, W_DRAIN);
        }
    } else {
        // ---------------------------------------------------- epilogue
        const int quarter = warp & 3;  // TMEM lanes this warp may access
        const float s = __fmul_rn(*args.inv_a, *args.inv_b);
        uint32_t amax = 0;  // bf16 bits of the running max
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int t = blockIdx.x; t < args.num_tiles; t += gridDim.x) {
            int mb, nb;
            tile_coords(t, args.num_mb, args.num_nb, mb, nb);
            if (!mbar_wait(&tfull[acc], acc_phase, args.err, W_TFULL)) break;
            tc_fence_after();
            const int row = mb * BM + quarter * 32 + lane;
            const bool row_ok = row < args.M;
            const uint32_t tbase =
                tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * BN);
            for (int c = 0; c < BN / 32; ++c) {
                const int col0 = nb * BN + c * 32;
                if (col0 >= args.N) break;  // warp-uniform
                uint32_t r[32];
                tmem_ld_32x32b_x32(tbase + (uint32_t)(c * 32), r);
                tmem_ld_wait();
                if (!row_ok) continue;
                const int64_t off = (int64_t)row * args.N + col0;
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    if (col0 + v * 8 >= args.N) break;
                    uint32_t hb[8];
                    if (EPI == LM_EPI_RELU2_BWD) {
                        const uint4 a4 = *reinterpret_cast<const uint4*>(args.aux + off + v * 8);
                        const uint32_t aw[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            hb[2 * i] = aw[i] & 0xFFFFu;
                            hb[2 * i + 1] = aw[i] >> 16;
                        }
                    }
                    uint32_t ob[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float y = __fmul_rn(__uint_as_float(r[v * 8 + i]), s);
                        uint32_t b = bf16_bits(y);
                        if (EPI == LM_EPI_RELU2_BWD) {
                            const float g = __uint_as_float(b << 16);
                            const float h = __uint_as_float(hb[i] << 16);
                            const float rh = h > 0.f ? h : 0.f;
                            b = bf16_bits(__fmul_rn(__fmul_rn(g, 2.0f), rh));
                        }
                        ob[i] = b;
                        if (EPI == LM_EPI_RELU2_FWD)
                            amax = (b & 0x8000u) ? amax : max(amax, b);
                        else
                            amax = max(amax, b & 0x7FFFu);
                    }
                    *reinterpret_cast<uint4*>(args.D + off + v * 8) =
                        make_uint4(ob[0] | (ob[1] << 16), ob[2] | (ob[3] << 16),
                                   ob[4] | (ob[5] << 16), ob[6] | (ob[7] << 16));
                }
            }
            tc_fence_before();
            mbar_arrive(&tempty[acc]);
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1u;
        }
        if (args.amax_out) {
            uint32_t m = __reduce_max_sync(0xFFFFFFFFu, amax);
            if (lane == 0 && m) {
                uint32_t bits = m << 16;
                if (EPI == LM_EPI_RELU2_FWD) {
                    // max h = bf16(max(relu H)^2): squaring and rounding are monotone
                    const float r = __uint_as_float(bits);
                    bits = bf16_bits(__fmul_rn(r, r)) << 16;
                }
                atomicMax(reinterpret_cast<unsigned int*>(args.amax_out), bits);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

template <int EPI>
lm_status launch_gemm(const CUtensorMap& ta, const CUtensorMap& tb, const GemmArgs& a,
                      cudaStream_t s) {
    static bool configured = false;  // the attribute is per kernel, not per call
    if (!configured) {
        if (cudaFuncSetAttribute(gemm_fp8_kernel<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 SMEM_BYTES) != cudaSuccess)
            return LM_ERR_CUDA;
        configured = true;
    }
    const int sms = sm_count();
    if (sms <= 0) return LM_ERR_CUDA;
    const int grid = a.num_tiles < sms ? a.num_tiles : sms;
    gemm_fp8_kernel<EPI><<<grid, NUM_THREADS, SMEM_BYTES, s>>>(ta, tb, a);
    return launch_status();
}

}  // namespace
}  // namespace lm

extern "C" lm_status lm_fp8_gemm(const uint8_t* A, lm_fp8_format fa, const uint8_t* B,
                                 lm_fp8_format fb, int64_t M, int64_t N, int64_t K,
                                 const float* inv_scale_a, const float* inv_scale_b,
                                 lm_epilogue epi, const void* aux, void* D, float* amax_out,
                                 lm_stream_t stream) {
    using namespace lm;
    if ((fa != LM_FP8_E4M3 && fa != LM_FP8_E5M2) || (fb != LM_FP8_E4M3 && fb != LM_FP8_E5M2))
        return LM_ERR_UNSUPPORTED_FORMAT;
    if (fa == LM_FP8_E5M2 && fb == LM_FP8_E5M2) return LM_ERR_UNSUPPORTED_FORMAT;
    if (epi != LM_EPI_NONE && epi != LM_EPI_RELU2_FWD && epi != LM_EPI_RELU2_BWD)
        return LM_ERR_UNSUPPORTED_FORMAT;
    if (M < 0 || N < 0 || K < 0) return LM_ERR_INVALID_ARG;
    if (M == 0 || N == 0) return LM_OK;
    if (!D || !inv_scale_a || !inv_scale_b) return LM_ERR_INVALID_ARG;
    if (K > 0 && (!A || !B)) return LM_ERR_INVALID_ARG;
    if (epi == LM_EPI_RELU2_BWD && !aux) return LM_ERR_INVALID_ARG;
    if (K % 16 != 0 || N % 8 != 0) return LM_ERR_UNSUPPORTED_SHAPE;
    if (M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31) || K >= (int64_t(1) << 31))
        return LM_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(A) || !aligned16(B) || !aligned16(D) || !aligned16(aux))
        return LM_ERR_ALIGNMENT;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (K == 0) {  // empty reduction: D = epi(0) = 0, amax unchanged
        if (cudaMemsetAsync(D, 0, (size_t)M * (size_t)N * 2, s) != cudaSuccess)
            return LM_ERR_CUDA;
        return LM_OK;
    }
    CUtensorMap ta, tb;
    if (!encode_tmap_u8(&ta, A, (uint64_t)M, (uint64_t)K, (uint64_t)K, BM, BK) ||
        !encode_tmap_u8(&tb, B, (uint64_t)N, (uint64_t)K, (uint64_t)K, BN, BK))
        return LM_ERR_CUDA;
    unsigned int* err = device_error_word();
    if (!err) return LM_ERR_CUDA;

    GemmArgs a;
    a.M = (int)M;
    a.N = (int)N;
    a.num_mb = (int)((M + BM - 1) / BM);
    a.num_nb = (int)((N + BN - 1) / BN);
    a.num_kb = (int)((K + BK - 1) / BK);
    a.num_tiles = a.num_mb * a.num_nb;
    a.inv_a = inv_scale_a;
    a.inv_b = inv_scale_b;
    a.aux = static_cast<const uint16_t*>(aux);
    a.D = static_cast<uint16_t*>(D);
    a.amax_out = amax_out;
    a.err = err;
    a.idesc = idesc_f8((uint32_t)fa, (uint32_t)fb, BM, BN);
    switch (epi) {
        case LM_EPI_NONE: return launch_gemm<LM_EPI_NONE>(ta, tb, a, s);
        case LM_EPI_RELU2_FWD: return launch_gemm<LM_EPI_RELU2_FWD>(ta, tb, a, s);
        default: return launch_gemm<LM_EPI_RELU2_BWD>(ta, tb, a, s);
    }
}
