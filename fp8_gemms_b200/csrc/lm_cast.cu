// lm_cast.cu -- dynamic tensorwise FP8 scaling: amax reduction, scale, and
// the saturating round-to-nearest-even cast (row-major codes, and on request
// the transposed copy).
//
// Method: one fp32 scale per tensor per cast, computed from that tensor's
// current amax (decomputer.nl, "Het trainen van een 3.8B LLM tot 0.384 CORE
// voor $998", section "Vroege experimenten" item 4 -- FP8 with dynamic
// tensorwise scaling on all three GEMMs).  e4m3 (max 448) for activations and
// weights, e5m2 (max 57344) for gradients.
//
// The passes are HBM-bound and take up to three tensors per launch:
//  - amax: 16-byte loads, eight in flight per thread, packed bf16 maxima;
//  - cast: a persistent TMA-fed kernel (tensor maps per tensor) whose
//    consumer warps convert 8 bf16 at a time (packed f32x2 scaling, paired
//    satfinite conversions) and store the row-major codes; the optional
//    transpose is built in shared memory and stored by TMA;
//  - a plain per-tile kernel for the row-major codes of tensors whose row
//    count is not a multiple of 16.
#include <cuda_bf16.h>

#include "lm_cast_math.cuh"
#include "lm_internal.h"
#include "lm_ptx.cuh"

namespace lm {
namespace {

constexpr int kCastRows = 256;  // tile rows (the qT segment written per column)
constexpr int kCastCols = 128;  // tile columns (bytes of codes per smem row)
constexpr int kThreads = 256;

// max over the 8 bf16 of v of |x| (or of h = bf16(relu(x)^2)), as bf16 bits.
// Non-negative bf16 values order like their bits; NaN sorts above infinity.
template <bool RELU2>
__device__ __forceinline__ uint32_t absmax8(uint4 v, uint32_t m) {
    if (!RELU2) {
        m = __vmaxu2(m, v.x & 0x7FFF7FFFu);
        m = __vmaxu2(m, v.y & 0x7FFF7FFFu);
        m = __vmaxu2(m, v.z & 0x7FFF7FFFu);
        m = __vmaxu2(m, v.w & 0x7FFF7FFFu);
        return m;
    }
    m = __vmaxu2(m, relu2_bf16x2(v.x) & 0x7FFF7FFFu);
    m = __vmaxu2(m, relu2_bf16x2(v.y) & 0x7FFF7FFFu);
    m = __vmaxu2(m, relu2_bf16x2(v.z) & 0x7FFF7FFFu);
    m = __vmaxu2(m, relu2_bf16x2(v.w) & 0x7FFF7FFFu);
    return m;
}

// Up to kMaxSet tensors handled by one launch of a pass.  Per-tensor values
// are picked with compile-time indices (no dynamic indexing of a kernel
// parameter, which would copy it to local memory).
constexpr int kMaxSet = kMaxCastSet;

template <typename T>
__device__ __forceinline__ T pick(int j, T a, T b, T c) {
    return j == 0 ? a : (j == 1 ? b : c);
}

struct AmaxSet {
    int n;
    const uint16_t* x[kMaxSet];
    int64_t rows[kMaxSet], cols[kMaxSet], ld[kMaxSet];
    unsigned int* out[kMaxSet];  // fp32 bits of the amax, zeroed beforehand
    int block_end[kMaxSet];      // blocks [block_end[j-1], block_end[j]) reduce tensor j
};

// Pass 1: amax of each tensor of the set into its *out (fp32 bit pattern of
// a non-negative value, max-reduced with atomicMax).  Each block reduces one
// tensor; blocks are shared out in proportion to the tensors' sizes.
template <bool RELU2>
__global__ void __launch_bounds__(kThreads) amax_kernel(const AmaxSet set) {
    const int b = (int)blockIdx.x;
    const int j = b < set.block_end[0] ? 0 : (b < set.block_end[1] ? 1 : 2);
    const int b0 = pick(j, 0, set.block_end[0], set.block_end[1]);
    const int nblocks = pick(j, set.block_end[0], set.block_end[1], set.block_end[2]) - b0;
    const uint16_t* x = pick(j, set.x[0], set.x[1], set.x[2]);
    const int64_t rows = pick(j, set.rows[0], set.rows[1], set.rows[2]);
    const int64_t cols = pick(j, set.cols[0], set.cols[1], set.cols[2]);
    const int64_t ld = pick(j, set.ld[0], set.ld[1], set.ld[2]);
    uint32_t m = 0;
    const int64_t vpr = cols >> 3;  // 16-byte vectors per row
    const int64_t nvec = rows * vpr;
    const int64_t stride = (int64_t)nblocks * kThreads;
    int64_t i = (int64_t)(b - b0) * kThreads + threadIdx.x;
    if (ld == cols) {
        const uint4* xv = reinterpret_cast<const uint4*>(x);
        // eight independent 16-byte loads in flight per thread, the last batch
        // predicated (a vector past the end counts as zeros), so that a small
        // tensor's few vectors per thread are fetched together, not one
        // dependent load after another
        for (; i < nvec; i += 8 * stride) {
            uint4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                v[u] = i + u * stride < nvec ? ld_stream_v4(xv + i + u * stride)
                                             : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int u = 0; u < 8; ++u) m = absmax8<RELU2>(v[u], m);
        }
    } else {
        for (; i < nvec; i += stride) {
            const int64_t r = i / vpr, c = (i - r * vpr) << 3;
            m = absmax8<RELU2>(ld_stream_v4(x + r * ld + c), m);
        }
    }
    m = max(m & 0xFFFFu, m >> 16);
    m = __reduce_max_sync(0xFFFFFFFFu, m);
    __shared__ uint32_t warp_max[kThreads / 32];
    if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t bm = 0;
#pragma unroll
        for (int w = 0; w < kThreads / 32; ++w) bm = max(bm, warp_max[w]);
        if (bm) atomicMax(pick(j, set.out[0], set.out[1], set.out[2]), bm << 16);
    }
}

// The scales of a tensor from its amax.  A NaN or infinite amax (the tensor
// holds a NaN or an infinity) still yields the scales the formula gives -- a
// NaN or zero scale -- and records kErrNonfiniteAmax in the error word, which
// lm_get_error reports as LM_ERR_NONFINITE.
__device__ __forceinline__ void write_scales(float amax, float fmax, float* amax_out,
                                             float* scale_out, float* inv_out, float* scale_reg,
                                             unsigned int* err) {
    const float scale = scale_from_amax(amax, fmax);
    *scale_reg = scale;
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        *amax_out = amax;
        *scale_out = scale;
        *inv_out = __fdiv_rn(1.0f, scale);
        if (!(amax <= 3.40282347e38f)) atomicCAS(err, 0u, kErrNonfiniteAmax);
    }
}

__global__ void scales_only_kernel(const float* amax_src, float fmax, float* amax_out,
                                   float* scale_out, float* inv_out, unsigned int* err) {
    float s;
    write_scales(*amax_src, fmax, amax_out, scale_out, inv_out, &s, err);
}

// Pass 2: scale, cast and transpose one 256 x 128 tile per block.  Tiles are
// taken in reverse memory order so the first blocks re-read the tail of the
// tensor, the part pass 1 left in L2.
template <int FMT, bool RELU2>
__global__ void __launch_bounds__(kThreads) cast_kernel(
    const uint16_t* __restrict__ x, int rows, int cols, int64_t ld, const float* amax_src,
    float* amax_out, float* scale_out, float* inv_out, uint8_t* __restrict__ q,
    uint8_t* __restrict__ qT, int tiles_c, int num_tiles, unsigned int* err) {
    __shared__ __align__(16) uint32_t tile[kCastRows][kCastCols / 4];
    const float fmax = FMT == LM_FP8_E4M3 ? 448.0f : 57344.0f;
    float scale;
    write_scales(*amax_src, fmax, amax_out, scale_out, inv_out, &scale, err);

    const int t = num_tiles - 1 - (int)blockIdx.x;
    const int r0 = (t / tiles_c) * kCastRows;
    const int c0 = (t % tiles_c) * kCastCols;
    const int tid = threadIdx.x;

    // all sixteen 16-byte loads of this thread in flight, then convert:
    // 8 bf16 -> 8 codes per load; row-major codes straight to q
    constexpr int kIters = (kCastRows * kCastCols / 8) / kThreads;
    uint4 xin[kIters];
#pragma unroll
    for (int it = 0; it < kIters; ++it) {
        const int idx = it * kThreads + tid;
        const int r = r0 + (idx >> 4), c = c0 + (idx & 15) * 8;
        xin[it] = (r < rows && c < cols) ? ld_stream_v4(x + (int64_t)r * ld + c)
                                       : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int it = 0; it < kIters; ++it) {
        const int idx = it * kThreads + tid;
        const int rr = idx >> 4, ch = idx & 15;
        const int r = r0 + rr, c = c0 + ch * 8;
        const uint2 codes = convert8<FMT, RELU2>(xin[it], scale);
        if (q && r < rows && c < cols) *reinterpret_cast<uint2*>(q + (int64_t)r * cols + c) = codes;
        *reinterpret_cast<uint2*>(&tile[rr][ch * 2]) = codes;
    }
    if (!qT) return;
    __syncthreads();

    // warp w owns tile rows [32w, 32w+32), lane l owns tile columns [4l, 4l+4)
    const int w = tid >> 5, l = tid & 31;
    uint32_t v[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = tile[w * 32 + i][l];
    uint32_t o[4][8];  // o[j][k]: column 4l+j, tile rows 32w+4k .. +3
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const uint32_t t0 = __byte_perm(v[4 * k], v[4 * k + 1], 0x5140);
        const uint32_t t1 = __byte_perm(v[4 * k + 2], v[4 * k + 3], 0x5140);
        const uint32_t t2 = __byte_perm(v[4 * k], v[4 * k + 1], 0x7362);
        const uint32_t t3 = __byte_perm(v[4 * k + 2], v[4 * k + 3], 0x7362);
        o[0][k] = __byte_perm(t0, t1, 0x5410);
        o[1][k] = __byte_perm(t0, t1, 0x7632);
        o[2][k] = __byte_perm(t2, t3, 0x5410);
        o[3][k] = __byte_perm(t2, t3, 0x7632);
    }
    const int rb = r0 + w * 32;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int c = c0 + 4 * l + j;
        if (c >= cols) continue;
        uint8_t* dst = qT + (int64_t)c * rows + rb;
        if (rb + 16 <= rows)
            *reinterpret_cast<uint4*>(dst) = make_uint4(o[j][0], o[j][1], o[j][2], o[j][3]);
        if (rb + 32 <= rows)
            *reinterpret_cast<uint4*>(dst + 16) = make_uint4(o[j][4], o[j][5], o[j][6], o[j][7]);
    }
}


// Pass 2, TMA-fed: a persistent kernel, two CTAs per SM.  Warp 8 streams
// 128 x 128 bf16 tiles (32 KB) into a shared ring with TMA; warps 0-7 convert
// each tile (16-byte shared loads; 8-byte stores of the row-major codes
// straight to q).  The TRANS instantiation (2 stages) also builds each
// tile's transpose in shared memory, which one thread writes to qT with a
// single TMA store; without it the ring has 3 stages.
//  - codes tile: word w of tile row r sits at r*32 + (w ^ 4*((r >> 4) & 7)),
//    so both the row-major writes and the column-quad reads of the
//    transpose are free of bank conflicts;
//  - transposed tile: tile column c is a 128-byte row, its 16-byte chunk k
//    at ((k ^ (c & 7)) * 16) -- the 128-byte swizzle the qT tensor map
//    uses -- so the 16-byte writes are conflict-free too.
// Tiles are taken in reverse memory order so the first ones re-read what the
// amax pass left in L2.  Waits are bounded; after a timeout a thread stops
// waiting but keeps the loop's barrier sequence, so no barrier can hang.
namespace tmac {
constexpr int TR = 128, TC = 128;
constexpr int IN_BYTES = TR * TC * 2;
constexpr int CODE_BYTES = TR * TC;
constexpr int CONSUMERS = 256;
constexpr int THREADS = CONSUMERS + 32;
// With transposes: 2 input stages plus the codes and transposed tiles.
// Without (row-major codes only): the same shared memory holds 3 stages.
// Either way two CTAs fit on an SM.
__host__ __device__ constexpr int stages(bool trans) { return trans ? 2 : 3; }
__host__ __device__ constexpr int smem_bytes(bool trans) {
    return 1024 + (trans ? 2 * CODE_BYTES : 0) + stages(trans) * IN_BYTES + 64;
}
enum : unsigned { W_CAST_EMPTY = 0x201, W_CAST_FULL = 0x202, W_CAST_LOADS = 0x203 };
}  // namespace tmac

__device__ __forceinline__ void consumers_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(tmac::CONSUMERS) : "memory");
}

// The tensors of one launch of the TMA-fed cast.  Global tile indices
// [tile_end[j-1], tile_end[j]) belong to tensor j; unused entries repeat the
// total.  Each tensor has its own tensor maps (kernel parameters tmX<j>,
// tmQT<j>), scale and outputs.
struct CastSet {
    int n, num_tiles;
    int want_qT;  // bit j: write tensor j's transposed codes
    int tile_end[kMaxSet];
    int rows[kMaxSet], cols[kMaxSet], tiles_c[kMaxSet];
    const float* amax_src[kMaxSet];
    float* amax_out[kMaxSet];
    float* scale_out[kMaxSet];
    float* inv_out[kMaxSet];
    uint8_t* q[kMaxSet];
};

__device__ __forceinline__ int set_member(const CastSet& set, int t) {
    return t < set.tile_end[0] ? 0 : (t < set.tile_end[1] ? 1 : 2);
}

template <int FMT, bool RELU2, bool TRANS>
__global__ void __launch_bounds__(tmac::THREADS) cast_tma_kernel(
    const __grid_constant__ CUtensorMap tmX0, const __grid_constant__ CUtensorMap tmX1,
    const __grid_constant__ CUtensorMap tmX2, const __grid_constant__ CUtensorMap tmQT0,
    const __grid_constant__ CUtensorMap tmQT1, const __grid_constant__ CUtensorMap tmQT2,
    const CastSet set, unsigned int* err) {
    using namespace tmac;
    constexpr int STAGES = stages(TRANS);
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
    uint8_t* sT = smem;                                   // transposed codes, 1024-aligned
    uint8_t* sIn = smem + (TRANS ? CODE_BYTES : 0);       // STAGES x 32 KB
    uint32_t* sCode = reinterpret_cast<uint32_t*>(sIn + STAGES * IN_BYTES);  // [TR][TC/4]
    uint64_t* full =
        reinterpret_cast<uint64_t*>(sIn + STAGES * IN_BYTES + (TRANS ? CODE_BYTES : 0));
    uint64_t* empty = full + STAGES;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], CONSUMERS / 32);
        }
        fence_barrier_init();
    }
    __syncthreads();
    const int num_tiles = set.num_tiles;

    if (warp == CONSUMERS / 32) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0, issued = 0;
            for (int i = blockIdx.x; i < num_tiles; i += gridDim.x) {
                const int t = num_tiles - 1 - i;
                const int j = set_member(set, t);
                const int lt = t - pick(j, 0, set.tile_end[0], set.tile_end[1]);
                const int tc = pick(j, set.tiles_c[0], set.tiles_c[1], set.tiles_c[2]);
                if (!mbar_wait(&empty[s], ph ^ 1u, err, W_CAST_EMPTY)) break;
                mbar_arrive_expect_tx(&full[s], IN_BYTES);
                tma_load_2d(smem_addr(sIn + s * IN_BYTES), pick(j, &tmX0, &tmX1, &tmX2), &full[s],
                            (lt % tc) * TC, (lt / tc) * TR);
                ++issued;
                if (++s == STAGES) {
                    s = 0;
                    ph ^= 1u;
                }
            }
            for (int st = 0; st < STAGES; ++st) {  // every issued load has landed
                const uint32_t n = issued / STAGES + ((uint32_t)st < issued % STAGES ? 1u : 0u);
                if (n) mbar_wait(&full[st], (n - 1) & 1u, err, W_CAST_LOADS);
            }
        }
        return;
    }

    // ---------------------------------------------------- consumers
    // the scales, while the producer's first loads are in flight
    const float fmax = FMT == LM_FP8_E4M3 ? 448.0f : 57344.0f;
    float sc[kMaxSet] = {0.f, 0.f, 0.f};
#pragma unroll
    for (int j = 0; j < kMaxSet; ++j)
        if (j < set.n)
            write_scales(*set.amax_src[j], fmax, set.amax_out[j], set.scale_out[j], set.inv_out[j],
                         &sc[j], err);
    int s = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (int i = blockIdx.x; i < num_tiles; i += gridDim.x) {
        const int t = num_tiles - 1 - i;
        const int j = set_member(set, t);
        const int lt = t - pick(j, 0, set.tile_end[0], set.tile_end[1]);
        const int tc = pick(j, set.tiles_c[0], set.tiles_c[1], set.tiles_c[2]);
        const int rows = pick(j, set.rows[0], set.rows[1], set.rows[2]);
        const int cols = pick(j, set.cols[0], set.cols[1], set.cols[2]);
        uint8_t* q = pick(j, set.q[0], set.q[1], set.q[2]);
        const float scale = pick(j, sc[0], sc[1], sc[2]);
        const int r0 = (lt / tc) * TR, c0 = (lt % tc) * TC;
        if (ok) ok = mbar_wait(&full[s], ph, err, W_CAST_FULL);
        const uint8_t* in = sIn + s * IN_BYTES;
#pragma unroll
        for (int it = 0; it < (TR * TC / 8) / CONSUMERS; ++it) {
            const int idx = it * CONSUMERS + tid;
            const int rr = idx >> 4, ch = idx & 15;
            const uint4 v = *reinterpret_cast<const uint4*>(in + rr * (TC * 2) + ch * 16);
            const uint2 codes = convert8<FMT, RELU2>(v, scale);
            const int r = r0 + rr, c = c0 + ch * 8;
            if (q && r < rows && c < cols)
                *reinterpret_cast<uint2*>(q + (int64_t)r * cols + c) = codes;
            if (TRANS) {
                const int wpos = (2 * ch) ^ (4 * ((rr >> 4) & 7));
                *reinterpret_cast<uint2*>(&sCode[rr * (TC / 4) + wpos]) = codes;
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);  // this warp is done with the stage
        if (++s == STAGES) {
            s = 0;
            ph ^= 1u;
        }
        if (!TRANS || !((set.want_qT >> j) & 1)) continue;
        if (tid == 0) bulk_wait_group_read<0>();  // the previous tile's store has read sT
        consumers_sync();                           // codes tile complete, sT free
        // lane: tile rows [16k, 16k+16) with k = lane % 8; tile columns
        // [4q, 4q+4) with q = 4 * warp + lane / 8
        const int k = lane & 7, qd = 4 * warp + (lane >> 3);
        uint32_t v[16];
#pragma unroll
        for (int i2 = 0; i2 < 16; ++i2) v[i2] = sCode[(16 * k + i2) * (TC / 4) + (qd ^ (4 * k))];
        uint32_t o[4][4];  // o[j][m]: column 4q+j, rows 16k+4m .. +3
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const uint32_t t0 = __byte_perm(v[4 * m], v[4 * m + 1], 0x5140);
            const uint32_t t1 = __byte_perm(v[4 * m + 2], v[4 * m + 3], 0x5140);
            const uint32_t t2 = __byte_perm(v[4 * m], v[4 * m + 1], 0x7362);
            const uint32_t t3 = __byte_perm(v[4 * m + 2], v[4 * m + 3], 0x7362);
            o[0][m] = __byte_perm(t0, t1, 0x5410);
            o[1][m] = __byte_perm(t0, t1, 0x7632);
            o[2][m] = __byte_perm(t2, t3, 0x5410);
            o[3][m] = __byte_perm(t2, t3, 0x7632);
        }
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            const int c = 4 * qd + jj;
            *reinterpret_cast<uint4*>(sT + c * 128 + ((k ^ (c & 7)) << 4)) =
                make_uint4(o[jj][0], o[jj][1], o[jj][2], o[jj][3]);
        }
        fence_proxy_async_smem();
        consumers_sync();  // transposed tile complete; codes tile fully read
        if (tid == 0) {
            tma_store_2d(pick(j, &tmQT0, &tmQT1, &tmQT2), smem_addr(sT), r0, c0);
            bulk_commit_group();
        }
    }
    if (tid == 0) bulk_wait_group<0>();
}

// One launch of the TMA-fed cast kernel (with or without its transpose stage).
template <int FMT, bool RELU2, bool TRANS>
lm_status launch_cast_tma_kernel(const CUtensorMap (&tx)[kMaxSet],
                                 const CUtensorMap (&tq)[kMaxSet], const CastSet& set, int grid,
                                 unsigned int* err, cudaStream_t s) {
    static bool configured[64] = {};
    constexpr int smem = tmac::smem_bytes(TRANS);
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return LM_ERR_CUDA;
    if (!configured[dev]) {
        if (cudaFuncSetAttribute(cast_tma_kernel<FMT, RELU2, TRANS>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
            return LM_ERR_CUDA;
        configured[dev] = true;
    }
    timing_mark(s, 'c');
    cast_tma_kernel<FMT, RELU2, TRANS><<<grid, tmac::THREADS, smem, s>>>(
        tx[0], tx[1], tx[2], tq[0], tq[1], tq[2], set, err);
    return launch_status();
}

// TMA-fed cast of the items (each with rows % 16 == 0) in one launch; the
// kernel without the transpose stage when no item wants qT.
template <int FMT, bool RELU2>
lm_status launch_cast_tma(const CastItem* const* items, const float* const* amax_src, int n,
                          cudaStream_t s) {
    CUtensorMap tx[kMaxSet], tq[kMaxSet];
    CastSet set = {};
    set.n = n;
    int total = 0;
    for (int j = 0; j < n; ++j) {
        const CastItem& it = *items[j];
        const int rows = (int)it.rows, cols = (int)it.cols;
        if (!encode_tmap_bf16_plain(&tx[j], it.x, (uint64_t)rows, (uint64_t)cols,
                                    (uint64_t)it.ld * 2, tmac::TR, tmac::TC))
            return LM_ERR_CUDA;
        if (it.qT) {  // qT is [cols x rows]: tile rows become 128-byte rows of codes
            if (!encode_tmap_u8(&tq[j], it.qT, (uint64_t)cols, (uint64_t)rows, (uint64_t)rows,
                                tmac::TC, tmac::TR))
                return LM_ERR_CUDA;
            set.want_qT |= 1 << j;
        } else {
            tq[j] = tx[j];  // unused
        }
        const int tiles_c = (cols + tmac::TC - 1) / tmac::TC;
        total += ((rows + tmac::TR - 1) / tmac::TR) * tiles_c;
        set.tile_end[j] = total;
        set.rows[j] = rows;
        set.cols[j] = cols;
        set.tiles_c[j] = tiles_c;
        set.amax_src[j] = amax_src[j];
        set.amax_out[j] = it.amax_out;
        set.scale_out[j] = it.scale_out;
        set.inv_out[j] = it.inv_scale_out;
        set.q[j] = it.q;
    }
    for (int j = n; j < kMaxSet; ++j) {
        set.tile_end[j] = total;
        tx[j] = tx[0];
        tq[j] = tq[0];
    }
    set.num_tiles = total;
    unsigned int* err = device_error_word();
    if (!err) return LM_ERR_CUDA;
    int grid = 2 * sm_count();
    if (grid <= 0) return LM_ERR_CUDA;
    if (grid > total) grid = total;
    return set.want_qT ? launch_cast_tma_kernel<FMT, RELU2, true>(tx, tq, set, grid, err, s)
                       : launch_cast_tma_kernel<FMT, RELU2, false>(tx, tq, set, grid, err, s);
}

// One tensor with rows % 16 != 0 (row-major codes only): one block per tile.
template <int FMT, bool RELU2>
lm_status launch_cast_rows(const CastItem& it, const float* amax_src, cudaStream_t s) {
    const int rows = (int)it.rows, cols = (int)it.cols;
    const int tiles_c = (cols + kCastCols - 1) / kCastCols;
    const int n = ((rows + kCastRows - 1) / kCastRows) * tiles_c;
    unsigned int* err = device_error_word();
    if (!err) return LM_ERR_CUDA;
    timing_mark(s, 'c');
    cast_kernel<FMT, RELU2><<<n, kThreads, 0, s>>>(static_cast<const uint16_t*>(it.x), rows, cols,
                                                  it.ld, amax_src, it.amax_out, it.scale_out,
                                                  it.inv_scale_out, it.q, it.qT, tiles_c, n, err);
    return launch_status();
}

template <int FMT, bool RELU2>
lm_status launch_casts(const CastItem* items, const float* const* amax_src, int n,
                       cudaStream_t s) {
    const CastItem* tma[kMaxSet];
    const float* tma_src[kMaxSet];
    int nt = 0;
    for (int j = 0; j < n; ++j) {
        const CastItem& it = items[j];
        if (it.rows == 0 || it.cols == 0 || (!it.q && !it.qT)) continue;
        if (it.rows % 16 == 0) {
            tma[nt] = &it;
            tma_src[nt++] = amax_src[j];
        } else if (launch_cast_rows<FMT, RELU2>(it, amax_src[j], s) != LM_OK) {
            return LM_ERR_CUDA;
        }
    }
    return nt ? launch_cast_tma<FMT, RELU2>(tma, tma_src, nt, s) : LM_OK;
}

lm_status check_item(const CastItem& it) {
    if (it.rows < 0 || it.cols < 0 || it.ld < it.cols) return LM_ERR_INVALID_ARG;
    if (!it.amax_out || !it.scale_out || !it.inv_scale_out) return LM_ERR_INVALID_ARG;
    const bool empty = it.rows == 0 || it.cols == 0;
    if (!empty && !it.x) return LM_ERR_INVALID_ARG;
    if (it.cols % 16 != 0 || it.ld % 8 != 0) return LM_ERR_UNSUPPORTED_SHAPE;
    if (it.qT && it.rows % 16 != 0) return LM_ERR_UNSUPPORTED_SHAPE;
    if (it.rows >= (int64_t(1) << 31) || it.cols >= (int64_t(1) << 31))
        return LM_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(it.x) || !aligned16(it.q) || !aligned16(it.qT)) return LM_ERR_ALIGNMENT;
    return LM_OK;
}

}  // namespace
}  // namespace lm

lm_status lm::cast_set(const CastItem* items, int n, lm_fp8_format fmt, int relu2_input,
                       bool amax_zeroed, cudaStream_t s) {
    using namespace lm;
    if (fmt != LM_FP8_E4M3 && fmt != LM_FP8_E5M2) return LM_ERR_UNSUPPORTED_FORMAT;
    if (!items || n < 1 || n > kMaxSet) return LM_ERR_INVALID_ARG;
    for (int j = 0; j < n; ++j)
        if (lm_status st = check_item(items[j])) return st;

    // pass 1: one launch reduces every tensor whose amax is not supplied
    const float* src[kMaxSet];
    AmaxSet aset = {};
    int64_t nvec[kMaxSet], total_vec = 0;
    int need_zero = 0;
    for (int j = 0; j < n; ++j) {
        const CastItem& it = items[j];
        src[j] = it.amax_in ? it.amax_in : it.amax_out;
        if (it.amax_in) continue;
        ++need_zero;
        if (it.rows == 0 || it.cols == 0) continue;
        const int k = aset.n++;
        aset.x[k] = static_cast<const uint16_t*>(it.x);
        aset.rows[k] = it.rows;
        aset.cols[k] = it.cols;
        aset.ld[k] = it.ld;
        aset.out[k] = reinterpret_cast<unsigned int*>(it.amax_out);
        nvec[k] = it.rows * (it.cols >> 3);
        total_vec += nvec[k];
    }
    if (aset.n) timing_mark(s, 'a');
    if (!amax_zeroed && need_zero)
        for (int j = 0; j < n; ++j)
            if (!items[j].amax_in &&
                cudaMemsetAsync(items[j].amax_out, 0, sizeof(float), s) != cudaSuccess)
                return LM_ERR_CUDA;
    if (aset.n) {
        const int sms = sm_count();
        if (sms <= 0) return LM_ERR_CUDA;
        // blocks shared out in proportion to size, at least one per tensor
        const int budget = 4 * sms;
        int end = 0;
        for (int k = 0; k < aset.n; ++k) {
            int b = (int)((double)budget * (double)nvec[k] / (double)total_vec);
            end += b < 1 ? 1 : b;
            aset.block_end[k] = end;
        }
        for (int k = aset.n; k < kMaxSet; ++k) aset.block_end[k] = end;
        if (relu2_input)
            amax_kernel<true><<<end, kThreads, 0, s>>>(aset);
        else
            amax_kernel<false><<<end, kThreads, 0, s>>>(aset);
        if (launch_status() != LM_OK) return LM_ERR_CUDA;
    }

    // scales alone for tensors with nothing to cast
    const float fmax = fmt == LM_FP8_E4M3 ? 448.0f : 57344.0f;
    for (int j = 0; j < n; ++j) {
        const CastItem& it = items[j];
        if (it.rows == 0 || it.cols == 0 || (!it.q && !it.qT)) {
            if (it.amax_only) continue;
            unsigned int* err = device_error_word();
            if (!err) return LM_ERR_CUDA;
            timing_mark(s, 's');
            scales_only_kernel<<<1, 1, 0, s>>>(src[j], fmax, it.amax_out, it.scale_out,
                                               it.inv_scale_out, err);
            if (launch_status() != LM_OK) return LM_ERR_CUDA;
        }
    }
    if (fmt == LM_FP8_E4M3)
        return relu2_input ? launch_casts<LM_FP8_E4M3, true>(items, src, n, s)
                           : launch_casts<LM_FP8_E4M3, false>(items, src, n, s);
    return relu2_input ? launch_casts<LM_FP8_E5M2, true>(items, src, n, s)
                       : launch_casts<LM_FP8_E5M2, false>(items, src, n, s);
}

extern "C" lm_status lm_fp8_amax_scale_cast(const void* x, int64_t rows, int64_t cols, int64_t ld,
                                            lm_fp8_format fmt, int relu2_input,
                                            const float* amax_in, float* amax_out,
                                            float* scale_out, float* inv_scale_out, uint8_t* q,
                                            uint8_t* qT, lm_stream_t stream) {
    const lm::CastItem it = {x, rows, cols, ld, amax_in, amax_out, scale_out, inv_scale_out, q, qT};
    return lm::cast_set(&it, 1, fmt, relu2_input, false, reinterpret_cast<cudaStream_t>(stream));
}
