// lm_gemm.cu -- FP8 GEMM on sm_100a tensor cores (tcgen05), D = epi(A B^T s).
//
// The pages run all three GEMMs of each linear in FP8 with one fp32 scale
// per operand, bf16 out (decomputer.nl, "Het trainen van een 3.8B LLM tot
// 0.384 CORE voor $998", section "Doorvoer (Throughput) verhogen", FP8
// bullet; manulx.blog names the library call, torch._scaled_mm).  These are
// kernels of our own for B200 in place of that library call.
//
// Main kernel (M > 128): a CTA pair (cluster of 2, cta_group::2) computes a
// 256 x 256 output tile.  Each CTA TMA-loads its own 128 rows of A and its
// own 128 rows (N) of B into a 6-stage shared-memory ring; both loads count
// on the leader CTA's "full" mbarrier; the leader issues tcgen05.mma
// kind::f8f6f4 with M = 256, N = 256, K = 32, reading both CTAs' shared
// memory, so each SM streams half of B instead of all of it.  Accumulators
// live in TMEM (2 x 256 fp32 columns per CTA, double-buffered so the
// epilogue of one tile overlaps the main loop of the next).  The epilogue
// warps of each CTA drain their own 128 rows: tcgen05.ld -> dequant scale ->
// relu^2 / relu^2' -> bf16 -> 32 x 64 staging boxes (128-byte swizzle) -> TMA
// store, and reduce the amax of what the next cast consumes.  No TMA load uses
// cluster multicast; only the MMA-completion commits are multicast to the pair.
//
// Side casts: an instantiation with four more warps casts a bf16 tensor whose
// amax an earlier kernel reduced, beside the tiles.  Either a tensor the GEMM
// does not read (flat, no waits), or the GEMM's own A operand: then the side
// warps cast it in 256 x 128 units in the order the tiles consume them and set
// a ready bit per unit, and the TMA producer loads an A box only once its
// unit's bit is set.
//
// Thin kernel (M <= 128): one CTA per 128 x 256 tile (cta_group::1), same
// ring and TMEM double buffer, per-thread global stores.
//
// Every mbarrier wait is bounded (see lm_ptx.cuh).
#include <cuda_bf16.h>

#include "lm_cast_math.cuh"
#include "lm_internal.h"
#include "lm_ptx.cuh"

namespace lm {
namespace {

constexpr int BK = 128;     // K bytes (= FP8 elements) per pipeline stage
constexpr int UMMA_K = 32;  // K per tcgen05.mma for 8-bit inputs
constexpr int NUM_THREADS = 192;  // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
constexpr int NUM_EPI_WARPS = 4;
// With a side cast: warps 6-9 cast another tensor beside the tiles.
constexpr int SIDE_WARPS = 4;
constexpr int NUM_THREADS_SIDE = NUM_THREADS + 32 * SIDE_WARPS;

// codes recorded in the device error word when a bounded wait runs out
enum : unsigned {
    W_EMPTY = 0x101, W_TEMPTY = 0x102, W_FULL = 0x103, W_DRAIN = 0x104, W_TFULL = 0x105,
    W_LOADS = 0x106, W_AUX = 0x107, W_SPLIT = 0x108, W_SPLIT_LOAD = 0x109, W_SIDE_READY = 0x10A
};

// Split-K tail.  Tiles go round-robin to the persistent clusters, so a last
// wave of r < clusters tiles leaves the other clusters idle for a whole tile.
// Each of those r tiles can instead run as S units over S consecutive ranges
// of K.  A round of C clusters holds P = C / S such tiles, whose S parts sit
// on consecutive clusters of that round (the rest of the round's clusters get
// no unit).  Parts 0..S-2 write their fp32 partial sums to a workspace slot and
// raise a flag per (CTA, warp); part S-1, on the highest of the tile's
// clusters, waits for those flags (bounded) and adds the partials to its own
// sums before the epilogue.  With S = 2 in the grid's last round the partial
// is bulk-copied into the operand ring, idle there (the unit is its cluster's
// last); otherwise it is read from global memory.  Partial layout per (tile,
// part, CTA rank, TMEM lane quarter): [chunk 8][float4 8][lane 32], so both
// the writes and the reads are contiguous across a warp.
constexpr size_t kSplitSlotFloat4 = 8 * 8 * 32;                   // one warp's partial
constexpr size_t kSplitTileBytes = 2 * NUM_EPI_WARPS * kSplitSlotFloat4 * 16;  // 256 KB
constexpr int kSplitMaxSlots = 128;  // partial tiles the workspace holds
constexpr int kSplitMaxParts = 8;

struct WorkUnit {
    int tile;  // -1: no work (a cluster left idle in a round of split tiles)
    int kb0, kb1;
    int part;  // -1: a whole tile; else part 0..S-1 of a split tile (S-1 finishes it)
};

struct GemmArgs {
    int M, N, num_mb, num_nb, num_kb, num_tiles, group_m;
    int num_units, split_first;  // units: tiles [0, split_first), then rounds of split parts
    int split_parts;             // S (>= 2 when some tiles are split)
    int split_round;             // units per round (C, the clusters of a full grid)
    int split_per_round;         // P = C / S split tiles per round
    int split_slots;             // partial tiles in the workspace: split tiles x (S - 1)
    float4* split_ws;            // partial sums of the split tiles
    unsigned int* split_flags;   // [slot][rank][quarter], zeroed before the launch
    int a_mn, b_mn;  // 1: the operand is stored MN-major ([K x M] / [K x N], M or N contiguous)
    int stream_a;  // 1: A is the streamed operand (evict-first loads), 0: B is
    const float* inv_a;
    const float* inv_b;
    const uint16_t* aux;
    void* D;
    void* D2;
    float* amax_out;
    unsigned int* err;
    uint32_t idesc;
    // side cast (kernels instantiated with SIDE only): side_nvec 16-byte
    // vectors of bf16 at side_x -> 8-byte code vectors at side_q
    const uint4* side_x;
    uint2* side_q;
    int64_t side_nvec;
    int side_fmt;
    const float* side_amax_in;
    float *side_amax_out, *side_scale_out, *side_inv_out;
    // side cast that produces this GEMM's own A (side_ready != nullptr): the
    // side warps cast A's bf16 source [M x K] (relu^2 first if side_relu2) in
    // units of 256 rows x 128 columns, in the order the tiles consume them,
    // and set bit kb % 32 of side_ready[mb * side_ready_words + kb / 32] once
    // unit (mb, kb) is stored; the producer loads an A box only after its bit
    // is set, and the epilogue takes A's scale from side_amax_in
    unsigned int* side_ready;
    int side_ready_words;
    int side_relu2;
    int side_cols;
};

// The side cast's loop for one format: eight 16-byte loads in flight per
// thread, each 8 bf16 -> 8 codes with the cast kernels' arithmetic.
template <int FMT>
__device__ __forceinline__ void side_cast_loop(const GemmArgs& a, int64_t t, int64_t nt,
                                               float scale) {
    const uint4* x = a.side_x;
    uint2* q = a.side_q;
    const int64_t n = a.side_nvec;
    int64_t i = t;
    for (; i + 7 * nt < n; i += 8 * nt) {
        uint4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) v[u] = ld_stream_v4(x + i + u * nt);
#pragma unroll
        for (int u = 0; u < 8; ++u) q[i + u * nt] = convert8<FMT, false>(v[u], scale);
    }
    for (; i < n; i += nt) q[i] = convert8<FMT, false>(ld_stream_v4(x + i), scale);
}

// The side cast feeding A keeps num_mb * words ready words, then (8-byte
// aligned) a 64-bit counter of claimed units; all of it zeroed per launch.
__host__ __device__ __forceinline__ int64_t side_counter_word(int64_t num_mb, int64_t words) {
    return (num_mb * words + 1) & ~int64_t(1);
}
__host__ __device__ __forceinline__ size_t side_ready_bytes(int64_t num_mb, int64_t words) {
    return (size_t)(side_counter_word(num_mb, words) + 2) * sizeof(unsigned int);
}

// Unit i of a side cast that feeds A -> its row block mb and k-block kb.  With
// one tile group per row block (group_m == 1) row block mb's first tile falls
// in round (mb * num_nb) / C of the C clusters; the units go round by round,
// k-block-major within a round over that round's row blocks, and an odd
// round's k-blocks backward, as its tiles walk K.  Otherwise k-block-major
// over all row blocks.  Any order is correct (the producer waits for each
// unit); this one casts a unit shortly before its first tile needs it.
__device__ __forceinline__ void side_unit(int64_t i, const GemmArgs& a, int C, int& mb, int& kb) {
    const int nkb = a.num_kb, nmb = a.num_mb, nnb = a.num_nb;
    if (a.group_m != 1) {
        kb = (int)(i / nmb);
        mb = (int)(i - (int64_t)kb * nmb);
        return;
    }
    const int v = (int)(i / nkb);
    const int r = (int)((int64_t)v * nnb / C);
    const int first = (int)(((int64_t)r * C + nnb - 1) / nnb);
    int next = (int)(((int64_t)(r + 1) * C + nnb - 1) / nnb);
    if (next > nmb) next = nmb;
    const int64_t local = i - (int64_t)first * nkb;
    const int n = next - first;
    kb = (int)(local / n);
    mb = first + (int)(local - (int64_t)kb * n);
    if (r & 1) kb = nkb - 1 - kb;
}

// A side cast that feeds A: the side warps of a CTA (thread t of 128) claim
// the next unit from a counter after the ready words (thread 0, broadcast
// through `slot` in shared memory), so units go out in the order above to
// whichever CTAs are running: no CTA waits on another being resident.  8 rows
// x 16 vectors of a unit per step, eight steps in flight per thread.  The side
// warps meet at named barrier 1 after a unit's stores; thread 0 then fences
// and publishes the unit's bit.
template <int FMT, bool RELU2>
__device__ __forceinline__ void side_cast_units(const GemmArgs& a, int t, int C, float scale,
                                                volatile int64_t* slot) {
    const uint16_t* x = static_cast<const uint16_t*>(static_cast<const void*>(a.side_x));
    uint8_t* q = reinterpret_cast<uint8_t*>(a.side_q);
    const int64_t M = a.M, K = a.side_cols;
    const int64_t total = (int64_t)a.num_mb * a.num_kb;
    unsigned long long* next = reinterpret_cast<unsigned long long*>(
        a.side_ready + side_counter_word(a.num_mb, a.side_ready_words));
    const int rr = t >> 4, v = t & 15;
    for (;;) {
        if (t == 0) *slot = (int64_t)atomicAdd(next, 1ull);
        asm volatile("bar.sync 1, %0;" ::"n"(32 * SIDE_WARPS) : "memory");
        const int64_t i = *slot;  // read by every side thread before the next claim
        if (i >= total) break;
        int mb, kb;
        side_unit(i, a, C, mb, kb);
        const int64_t col = (int64_t)kb * 128 + v * 8;
        const int64_t row0 = (int64_t)mb * 256 + rr;
#pragma unroll 1
        for (int b = 0; b < 4; ++b) {
            uint4 val[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int64_t r = row0 + 8 * (8 * b + u);
                val[u] = (r < M && col < K) ? ld_stream_v4(x + r * K + col)
                                            : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int64_t r = row0 + 8 * (8 * b + u);
                if (r < M && col < K)
                    *reinterpret_cast<uint2*>(q + r * K + col) = convert8<FMT, RELU2>(val[u], scale);
            }
        }
        // every side thread's stores, then (thread 0) a fence and the bit
        asm volatile("bar.sync 1, %0;" ::"n"(32 * SIDE_WARPS) : "memory");
        if (t == 0) {
            __threadfence();
            atomicOr(a.side_ready + (int64_t)mb * a.side_ready_words + (kb >> 5), 1u << (kb & 31));
        }
    }
}

// Wait until bit `bit` of *word is set (acquire), for at most kWaitLimitNs;
// returns the word, or 0 after recording `where` in the error word.
__device__ __forceinline__ uint32_t ready_wait(const unsigned int* word, uint32_t bit,
                                               unsigned int* err, unsigned int where) {
    uint32_t v = ld_acquire_gpu(word);
    if (v & bit) return v;
    const uint64_t t0 = global_timer_ns();
    for (;;) {
        __nanosleep(64);
        v = ld_acquire_gpu(word);
        if (v & bit) return v;
        if (global_timer_ns() - t0 > kWaitLimitNs) {
            atomicCAS(err, 0u, where);
            return 0u;
        }
    }
}

// The side cast, run by the side warps of every CTA (thread t of nt): the
// scale from the already-reduced amax, the scale block (thread 0), the codes.
// A NaN or infinite amax records kErrNonfiniteAmax, as the cast kernels do.
__device__ __forceinline__ void side_cast_run(const GemmArgs& a, int64_t t, int64_t nt,
                                              volatile int64_t* slot) {
    const float amax = *a.side_amax_in;
    const bool e4 = a.side_fmt == LM_FP8_E4M3;
    const float scale = scale_from_amax(amax, e4 ? 448.0f : 57344.0f);
    if (t == 0) {
        *a.side_amax_out = amax;
        *a.side_scale_out = scale;
        *a.side_inv_out = __fdiv_rn(1.0f, scale);
        if (!(amax <= 3.40282347e38f)) atomicCAS(a.err, 0u, kErrNonfiniteAmax);
    }
    if (a.side_ready) {
        constexpr int kT = 32 * SIDE_WARPS;
        const int cta = (int)(t / kT), ncta = (int)(nt / kT), lt = (int)(t - (int64_t)cta * kT);
        const int C = ncta / 2;
        if (e4 && a.side_relu2)
            side_cast_units<LM_FP8_E4M3, true>(a, lt, C, scale, slot);
        else if (e4)
            side_cast_units<LM_FP8_E4M3, false>(a, lt, C, scale, slot);
        else if (a.side_relu2)
            side_cast_units<LM_FP8_E5M2, true>(a, lt, C, scale, slot);
        else
            side_cast_units<LM_FP8_E5M2, false>(a, lt, C, scale, slot);
        return;
    }
    if (e4)
        side_cast_loop<LM_FP8_E4M3>(a, t, nt, scale);
    else
        side_cast_loop<LM_FP8_E5M2>(a, t, nt, scale);
}

// MULTI = false: no split, or halves in one round (units split_first + 2t and
// split_first + 2t + 1 are the halves of tile split_first + t).  MULTI = true:
// S parts, P tiles per round of split_round units.
template <bool MULTI>
__device__ __forceinline__ WorkUnit work_unit(int u, const GemmArgs& a) {
    if (u < a.split_first) return {u, 0, a.num_kb, -1};
    if constexpr (!MULTI) {
        const int s = u - a.split_first, h = s & 1, kh = a.num_kb >> 1;
        return {a.split_first + (s >> 1), h ? kh : 0, h ? a.num_kb : kh, h};
    } else {
        const int s = u - a.split_first, S = a.split_parts;
        const int round = s / a.split_round, pos = s - round * a.split_round;
        const int t = pos / S, part = pos - t * S;
        const int tile = a.split_first + round * a.split_per_round + t;
        if (t >= a.split_per_round || tile >= a.num_tiles) return {-1, 0, 0, -1};
        return {tile, part * a.num_kb / S, (part + 1) * a.num_kb / S, part};
    }
}

// The i-th k-block a unit processes in round `round` of its cluster (the
// round-th unit that cluster takes).  Even rounds walk the unit's K range
// forward, odd rounds backward: the tiles of one round start on the K slices
// the previous round read last, which are the ones still in L2.  Every
// cluster of a round takes the same direction, so the tiles in flight at
// once still read the same slices together.
__device__ __forceinline__ int k_block(const WorkUnit& w, int i, int round) {
    return (round & 1) ? w.kb1 - 1 - i : w.kb0 + i;
}

// Tile visiting order: groups of group_m row-blocks, column-blocks within a
// group, so the tiles in flight at once share A and B panels in L2.
__device__ __forceinline__ void tile_coords(int t, int group_m, int num_mb, int num_nb, int& mb,
                                            int& nb) {
    const int per_group = group_m * num_nb;
    const int g = t / per_group;
    const int first = g * group_m;
    const int gsize = min(group_m, num_mb - first);
    const int local = t - g * per_group;
    mb = first + local % gsize;
    nb = local / gsize;
}

__device__ __forceinline__ uint32_t bf16_bits(float v) {
    return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v));
}

// One accumulator value -> bf16 output bits under the epilogue, updating the
// running amax (bf16 bits) of what the next cast consumes.
template <int EPI>
__device__ __forceinline__ uint32_t epi_value(uint32_t acc_bits, float s, uint32_t h_bits,
                                              uint32_t& amax) {
    uint32_t b = bf16_bits(__fmul_rn(__uint_as_float(acc_bits), s));
    if (EPI == LM_EPI_RELU2_BWD) {
        const float g = __uint_as_float(b << 16);
        const float h = __uint_as_float(h_bits << 16);
        const float rh = h > 0.f ? h : 0.f;
        b = bf16_bits(__fmul_rn(__fmul_rn(g, 2.0f), rh));
    }
    if (EPI == LM_EPI_RELU2_FWD)
        amax = (b & 0x8000u) ? amax : max(amax, b);  // max of relu(H)
    else
        amax = max(amax, b & 0x7FFFu);
    return b;
}

// Final per-warp amax reduction into the fp32 bits at amax_out.
template <int EPI>
__device__ __forceinline__ void reduce_amax(uint32_t amax, float* amax_out, int lane) {
    if (!amax_out) return;
    const uint32_t m = __reduce_max_sync(0xFFFFFFFFu, amax);
    if (lane == 0 && m) {
        uint32_t bits = m << 16;
        if (EPI == LM_EPI_RELU2_FWD) {
            // max h = bf16(max(relu H)^2): squaring and rounding are monotone
            const float r = __uint_as_float(bits);
            bits = bf16_bits(__fmul_rn(r, r)) << 16;
        }
        atomicMax(reinterpret_cast<unsigned int*>(amax_out), bits);
    }
}

// Two accumulator values -> two bf16 output values packed in one word (lo =
// even column), and the running packed amax (bf16 bits, two halves) of what
// the next cast consumes.  bf16x2 arithmetic: for the relu^2 backward,
// dH = g * (2 relu(H)) where 2 relu(H) is exact and the product of two bf16
// values is exact before its single rounding -- the same value as
// bf16(g * 2 * relu(H)).  relu of a NaN H gives 0, as max(h, 0) does.
template <int EPI>
__device__ __forceinline__ uint32_t epi_pair(uint32_t acc0, uint32_t acc1, float s,
                                             uint32_t h_pair, uint32_t& amax2) {
    const __nv_bfloat162 g2 = __floats2bfloat162_rn(__fmul_rn(__uint_as_float(acc0), s),
                                                    __fmul_rn(__uint_as_float(acc1), s));
    uint32_t w = *reinterpret_cast<const uint32_t*>(&g2);
    if (EPI == LM_EPI_RELU2_BWD) {
        const __nv_bfloat162 h2 = *reinterpret_cast<const __nv_bfloat162*>(&h_pair);
        __nv_bfloat162 r2 = __hmax2(h2, __float2bfloat162_rn(0.0f));
        r2 = __hadd2(r2, r2);
        const __nv_bfloat162 d2 = __hmul2(g2, r2);
        w = *reinterpret_cast<const uint32_t*>(&d2);
        amax2 = __vmaxu2(amax2, w & 0x7FFF7FFFu);
    } else if (EPI == LM_EPI_RELU2_FWD) {
        amax2 = __vmaxu2(amax2, __vmaxs2(w, 0u));  // negative halves -> 0: max of relu(H)
    } else {
        amax2 = __vmaxu2(amax2, w & 0x7FFF7FFFu);
    }
    return w;
}

// silu(x) = x / (1 + exp(-x)) in fp32 (expf, one IEEE division)
__device__ __forceinline__ float silu_f32(float x) {
    return __fdiv_rn(x, __fadd_rn(1.0f, expf(-x)));
}

// Stage one 32 x 32 bf16 box (this lane's row: 16 packed words) in a ring of
// four 2 KB boxes at `ring` (64B-swizzled, as the tensor map expects) and
// TMA-store it at (x, y).  The box reused is the one stored four stores ago.
__device__ __forceinline__ void stage_box_store(uint8_t* ring, uint32_t& n_stores,
                                                const uint32_t (&w)[16], const CUtensorMap* map,
                                                int x, int y, uint64_t policy, int lane) {
    uint8_t* dst = ring + (n_stores & 3u) * 2048;
    if (lane == 0) bulk_wait_group_read<3>();
    __syncwarp();
#pragma unroll
    for (int j = 0; j < 4; ++j)
        *reinterpret_cast<uint4*>(dst + lane * 64 + ((j ^ ((lane >> 1) & 3)) << 4)) =
            make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
        tma_store_2d_hint(map, smem_addr(dst), x, y, policy);
        bulk_commit_group();
    }
    ++n_stores;
}

// =====================================================================
// CTA-pair kernel: 256 x 256 tiles, cta_group::2
// =====================================================================
namespace pair {

constexpr int TILE_M = 256, TILE_N = 256;
constexpr int STAGES = 6;
constexpr int A_BYTES = 128 * BK;  // this CTA's 128 rows of A
constexpr int B_BYTES = 128 * BK;  // this CTA's 128 rows (N) of B
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int EPI_COLS = 32;                   // columns per epilogue chunk
constexpr int BOX_BYTES = 32 * EPI_COLS * 2;   // one warp's 32 x 32 bf16 box
constexpr int STORE_BYTES = NUM_EPI_WARPS * 2 * BOX_BYTES;
constexpr int AUX_BYTES = NUM_EPI_WARPS * 2 * BOX_BYTES;
// The plain and relu^2 epilogues stage their bf16 output in boxes of 32 rows
// x 64 columns (two 32-column chunks, 4 KB, 128-byte swizzle), two per warp in
// the store and aux areas together.  The relu^2 backward loads each saved-H
// box into the same slot and writes dH over it in place.
constexpr int WIDE_COLS = 2 * EPI_COLS;
constexpr int WIDE_BYTES = 32 * WIDE_COLS * 2;
static_assert(NUM_EPI_WARPS * 2 * WIDE_BYTES == STORE_BYTES + AUX_BYTES, "wide box layout");
// the accumulating epilogue stages 32 x 32 fp32 boxes (4 KB, two per warp) in
// the store and aux areas together (contiguous, 32 KB)
constexpr int ACC_BOX_BYTES = 32 * EPI_COLS * 4;
static_assert(NUM_EPI_WARPS * 2 * ACC_BOX_BYTES == STORE_BYTES + AUX_BYTES, "staging layout");
constexpr uint32_t TMEM_COLS = 2 * TILE_N;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + STORE_BYTES + AUX_BYTES + 1024 + 512;

// Offset of 16-byte chunk j (0..7) of row r in a 32-row x 128-byte box of a
// TMA with CU_TENSOR_MAP_SWIZZLE_128B: chunk bits [4,7) XORed with r & 7.
__device__ __forceinline__ uint32_t sw128(int r, int j) {
    return (uint32_t)(r * 128 + ((j ^ (r & 7)) << 4));
}

// MULTI: the instantiation launched when the split tail has three or more
// parts (the last part reads the others' sums from global memory).  The
// instantiations for no split or halves leave that code out, which keeps the
// epilogue loop of the common case as lean as it was measured.
// SIDE: the instantiation with four more warps that run a side cast.
template <int EPI, bool MULTI, bool SIDE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(SIDE ? NUM_THREADS_SIDE : NUM_THREADS, 1)
    gemm_fp8_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                         const __grid_constant__ CUtensorMap tmB,
                         const __grid_constant__ CUtensorMap tmD,
                         const __grid_constant__ CUtensorMap tmAux,
                         const __grid_constant__ CUtensorMap tmD2, const GemmArgs args) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
    uint8_t* sA = smem;
    uint8_t* sB = sA + STAGES * A_BYTES;
    uint8_t* sStore = sB + STAGES * B_BYTES;
    uint8_t* sAux = sStore + STORE_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sAux + AUX_BYTES);
    uint64_t* full = bars;                  // [STAGES], used in the leader only
    uint64_t* empty = full + STAGES;        // [STAGES], both CTAs
    uint64_t* tfull = empty + STAGES;       // [2], both CTAs
    uint64_t* tempty = tfull + 2;           // [2], leader only
    uint64_t* drain = tempty + 2;           // leader only
    uint64_t* auxbar = drain + 1;           // [4 warps][2 boxes]
    uint64_t* splitbar = auxbar + 2 * NUM_EPI_WARPS;  // [4 warps]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(splitbar + NUM_EPI_WARPS);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int cluster = blockIdx.x >> 1, nclusters = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 2 * NUM_EPI_WARPS);
        }
        mbar_init(drain, 1);
        for (int i = 0; i < 2 * NUM_EPI_WARPS; ++i) mbar_init(&auxbar[i], 1);
        for (int i = 0; i < NUM_EPI_WARPS; ++i) mbar_init(&splitbar[i], 1);
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        tma_prefetch_desc(&tmD);
        if (EPI == LM_EPI_RELU2_BWD) tma_prefetch_desc(&tmAux);
        if (EPI == kEpiSwigluFwd) tma_prefetch_desc(&tmD2);
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();  // barriers of both CTAs initialised, TMEM allocated
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------------------------------- TMA producer (both CTAs)
            const uint32_t full_leader = map_to_rank(smem_addr(full), 0);
            // the operand that every tile wave re-reads stays at normal L2
            // priority; the one streamed through once is evicted first
            const uint64_t pol_first = l2_policy_evict_first();
            const uint64_t pol_a = args.stream_a ? pol_first : 0ull;
            const uint64_t pol_b = args.stream_a ? 0ull : pol_first;
            int stage = 0;
            uint32_t phase = 0, issued = 0;
            bool ok = true;
            uint32_t rword = 0;  // side cast feeding A: the last ready word read
            int rkey = -1;       // and its index
            for (int u = cluster, round = 0; u < args.num_units && ok;
                 u += nclusters, ++round) {
                const WorkUnit w = work_unit<MULTI>(u, args);
                if (MULTI && w.tile < 0) continue;
                int mb, nb;
                tile_coords(w.tile, args.group_m, args.num_mb, args.num_nb, mb, nb);
                const int arow = mb * TILE_M + (int)rank * 128;
                const int brow = nb * TILE_N + (int)rank * 128;
                for (int i = 0; i < w.kb1 - w.kb0; ++i) {
                    const int kb = k_block(w, i, round);
                    // box coordinates (x innermost): K-major (k, m|n), MN-major (m|n, k)
                    const int ax = args.a_mn ? arow : kb * BK, ay = args.a_mn ? kb * BK : arow;
                    const int bx = args.b_mn ? brow : kb * BK, by = args.b_mn ? kb * BK : brow;
                    if (!mbar_wait(&empty[stage], phase ^ 1u, args.err, W_EMPTY)) {
                        ok = false;
                        break;
                    }
                    if (args.side_ready) {
                        // A's unit (mb, kb) is stored by the side warps
                        const int key = mb * args.side_ready_words + (kb >> 5);
                        const uint32_t bit = 1u << (kb & 31);
                        if (key != rkey || !(rword & bit)) {
                            rkey = key;
                            rword = ready_wait(args.side_ready + key, bit, args.err, W_SIDE_READY);
                            if (!(rword & bit)) {
                                ok = false;
                                break;
                            }
                            fence_proxy_async_global();  // the acquired codes, then the TMA read
                        }
                    }
                    if (leader) mbar_arrive_expect_tx(&full[stage], 2 * STAGE_BYTES);
                    const uint32_t bar = full_leader + (uint32_t)(stage * 8);
                    if (args.stream_a) {
                        tma_load_2d_pair_hint(smem_addr(sA + stage * A_BYTES), &tmA, bar, ax, ay,
                                              pol_a);
                        tma_load_2d_pair(smem_addr(sB + stage * B_BYTES), &tmB, bar, bx, by);
                    } else {
                        tma_load_2d_pair(smem_addr(sA + stage * A_BYTES), &tmA, bar, ax, ay);
                        tma_load_2d_pair_hint(smem_addr(sB + stage * B_BYTES), &tmB, bar, bx, by,
                                              pol_b);
                    }
                    ++issued;
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (leader) {
                // both CTAs' loads of every armed phase have landed before exit
                for (int s = 0; s < STAGES; ++s) {
                    const uint32_t n = issued / STAGES + ((uint32_t)s < issued % STAGES ? 1u : 0u);
                    if (n) mbar_wait(&full[s], (n - 1) & 1u, args.err, W_LOADS);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            // ------------------------------------------- MMA issuer (leader)
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            // descriptor advance (16-byte units) per UMMA_K: 32 bytes along a
            // K-major row, or 32 rows of an MN-major tile
            const uint64_t a_step = args.a_mn ? (UMMA_K * 128) >> 4 : UMMA_K >> 4;
            const uint64_t b_step = args.b_mn ? (UMMA_K * 128) >> 4 : UMMA_K >> 4;
            for (int u = cluster; u < args.num_units && ok; u += nclusters) {
                const WorkUnit w = work_unit<MULTI>(u, args);
                if (MULTI && w.tile < 0) continue;
                if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, args.err, W_TEMPTY)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * TILE_N);
                for (int i = 0; i < w.kb1 - w.kb0; ++i) {
                    if (!mbar_wait(&full[stage], phase, args.err, W_FULL)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t ad = smem_desc_k128(smem_addr(sA + stage * A_BYTES));
                    const uint64_t bd = smem_desc_k128(smem_addr(sB + stage * B_BYTES));
#pragma unroll
                    for (int kk = 0; kk < BK / UMMA_K; ++kk)
                        mma_fp8_pair(d_tmem, ad + (uint64_t)kk * a_step, bd + (uint64_t)kk * b_step,
                                     args.idesc, (i != 0 || kk != 0) ? 1u : 0u);
                    mma_commit_pair(&empty[stage], 0x3);  // frees the stage in both CTAs
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                mma_commit_pair(&tfull[acc], 0x3);  // accumulator ready in both CTAs
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1u;
            }
            mma_commit_pair(drain, 0x1);  // all MMAs retired before teardown
            mbar_wait(drain, 0, args.err, W_DRAIN);
        }
    } else if (SIDE && warp >= 2 + NUM_EPI_WARPS) {
        // ------------------------------------------ side cast (both CTAs)
        constexpr int kSideThreads = 32 * SIDE_WARPS;
        side_cast_run(args, (int64_t)blockIdx.x * kSideThreads + (threadIdx.x - NUM_THREADS),
                      (int64_t)gridDim.x * kSideThreads,
                      reinterpret_cast<volatile int64_t*>(tmem_slot + 2));
    } else {
        // ------------------------------------------- epilogue (both CTAs)
        const int wi = warp - 2;       // staging slot
        const int quarter = warp & 3;  // TMEM lanes this warp may access
        // this warp's two 64-column boxes (plain and relu^2 epilogues), and,
        // for the relu^2 backward, one barrier per box for its saved-H load
        uint8_t* wide = sStore + wi * 2 * WIDE_BYTES;
        uint64_t* h_bar = auxbar + wi * 2;
        uint32_t h_issued = 0, h_used = 0;  // saved-H boxes loaded / consumed by this warp
        uint32_t n_wide = 0;                // 64-column boxes stored by this warp
        const uint32_t tempty_leader = map_to_rank(smem_addr(tempty), 0);
        const uint64_t stream_policy = l2_policy_evict_first();  // D and H are touched once
        // A's scale: from its amax when the side warps are still writing the
        // scale block (side cast feeding A), with the cast's own arithmetic
        const float inv_a =
            args.side_ready
                ? __fdiv_rn(1.0f, scale_from_amax(*args.side_amax_in,
                                                  args.side_fmt == LM_FP8_E4M3 ? 448.0f : 57344.0f))
                : *args.inv_a;
        const float s = __fmul_rn(inv_a, *args.inv_b);
        uint32_t amax2 = 0;  // two bf16-bit halves of the running max
        int acc = 0;
        uint32_t acc_phase = 0;
        uint32_t n_stores = 0;
        bool ok = true;
        for (int u = cluster; u < args.num_units && ok; u += nclusters) {
            const WorkUnit w = work_unit<MULTI>(u, args);
            if (MULTI && w.tile < 0) continue;
            int mb, nb;
            tile_coords(w.tile, args.group_m, args.num_mb, args.num_nb, mb, nb);
            const int grow = mb * TILE_M + (int)rank * 128 + quarter * 32;  // row of lane 0
            const int gcol = nb * TILE_N;
            const int left = args.N - gcol;
            const int n_chunks =
                left >= TILE_N ? TILE_N / EPI_COLS : (left + EPI_COLS - 1) / EPI_COLS;
            // this warp's slot of a split tile's partial sums and flags: part p
            // of the tile (p < S-1) writes slot_of(p); the last part reads them
            const int S = MULTI ? args.split_parts : 2;
            const bool finishes = w.part < 0 || w.part == S - 1;
            auto slot_of = [&](int p) {
                return (((size_t)(w.tile - args.split_first) * (size_t)(S - 1) + (size_t)p) * 2 +
                        rank) * NUM_EPI_WARPS + quarter;
            };
            // relu^2 backward: load saved-H box j (64 columns) of this warp
            // into slot j & 1, once every store that read that slot has
            // finished reading it
            const int n_pairs = (n_chunks + 1) / 2;
            auto issue_h = [&](int pair) {
                const uint32_t slot = h_issued & 1u;
                bulk_wait_group_read<0>();
                fence_proxy_async_smem();
                mbar_arrive_expect_tx(&h_bar[slot], WIDE_BYTES);
                tma_load_2d_hint(smem_addr(wide + slot * WIDE_BYTES), &tmAux, &h_bar[slot],
                                 gcol + pair * WIDE_COLS, grow, stream_policy);
            };
            if constexpr (EPI == LM_EPI_RELU2_BWD) {
                if (finishes) {
                    // this tile's first two boxes arrive while its accumulator
                    // is still being computed
                    for (int q = 0; q < 2 && q < n_pairs; ++q) {
                        if (lane == 0) issue_h(q);
                        ++h_issued;
                    }
                }
            }
            if (!mbar_wait(&tfull[acc], acc_phase, args.err, W_TFULL)) break;
            tc_fence_after();
            const uint32_t tbase =
                tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * TILE_N);
            if (!finishes) {
                // an earlier part of a split tile: publish the raw fp32 sums
                float4* dst = args.split_ws + slot_of(w.part) * kSplitSlotFloat4;
                for (int c = 0; c < n_chunks; ++c) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(tbase + (uint32_t)(c * EPI_COLS), r);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        dst[(c * 8 + i) * 32 + lane] = make_float4(
                            __uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                            __uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3]));
                }
                __threadfence();
                __syncwarp();
                if (lane == 0) st_release_gpu(args.split_flags + slot_of(w.part), 1u);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_remote_relaxed(tempty_leader + (uint32_t)(acc * 8));
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1u;
                continue;
            }
            // the last part of a split tile: the other parts' sums.  With two
            // parts in the grid's last round, the first part's sums are copied
            // into this warp's 32 KB of the operand ring (idle: no unit follows
            // on this cluster); otherwise they are read from global memory.
            const float4* part = nullptr;   // in shared memory
            const float4* gpart = nullptr;  // in global memory, slot_of(0) .. slot_of(S-2)
            if (w.part > 0 && finishes) {
                bool ready = true;
                if (lane == 0)
                    for (int p = 0; p < S - 1 && ready; ++p)
                        ready = flag_wait(args.split_flags + slot_of(p), 1u, args.err, W_SPLIT);
                ready = __shfl_sync(0xFFFFFFFFu, ready ? 1 : 0, 0) != 0;
                if (ready && (!MULTI || (S == 2 && u + nclusters >= args.num_units))) {
                    uint8_t* buf = smem + wi * (int)(kSplitSlotFloat4 * 16);
                    if (lane == 0) {
                        const uint32_t bytes = (uint32_t)n_chunks * 8 * 32 * 16;
                        fence_proxy_async_global();  // the acquired sums, then the bulk read
                        mbar_arrive_expect_tx(&splitbar[wi], bytes);
                        bulk_load_1d(smem_addr(buf), args.split_ws + slot_of(0) * kSplitSlotFloat4,
                                     bytes, &splitbar[wi]);
                    }
                    if (mbar_wait(&splitbar[wi], 0, args.err, W_SPLIT_LOAD))
                        part = reinterpret_cast<const float4*>(buf);
                    else  // error recorded; give the copy a second bounded wait before exit
                        mbar_wait(&splitbar[wi], 0, args.err, W_SPLIT_LOAD);
                } else if (ready) {
                    if constexpr (MULTI) {
                        __syncwarp();  // lane 0's acquire of the flags, then every lane's reads
                        __threadfence();
                        gpart = args.split_ws + slot_of(0) * kSplitSlotFloat4;
                    }
                }
            }
            if constexpr (EPI == kEpiSwigluFwd) {
                // gate columns [0,128) and up columns [128,256) of the tile: store
                // G, U (bf16, interleaved as computed) and h = bf16(silu(G) U)
                for (int c = 0; c < TILE_N / 2 / EPI_COLS; ++c) {
                    uint32_t rg[32], ru[32];
                    tmem_ld_32x32b_x32(tbase + (uint32_t)(c * EPI_COLS), rg);
                    tmem_ld_32x32b_x32(tbase + (uint32_t)(TILE_N / 2 + c * EPI_COLS), ru);
                    tmem_ld_wait();
                    uint32_t pg[16], pu[16], ph[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const __nv_bfloat162 g2 =
                            __floats2bfloat162_rn(__fmul_rn(__uint_as_float(rg[2 * i]), s),
                                                  __fmul_rn(__uint_as_float(rg[2 * i + 1]), s));
                        const __nv_bfloat162 u2 =
                            __floats2bfloat162_rn(__fmul_rn(__uint_as_float(ru[2 * i]), s),
                                                  __fmul_rn(__uint_as_float(ru[2 * i + 1]), s));
                        const float2 gf = __bfloat1622float2(g2), uf = __bfloat1622float2(u2);
                        const __nv_bfloat162 h2 = __floats2bfloat162_rn(
                            __fmul_rn(silu_f32(gf.x), uf.x), __fmul_rn(silu_f32(gf.y), uf.y));
                        pg[i] = *reinterpret_cast<const uint32_t*>(&g2);
                        pu[i] = *reinterpret_cast<const uint32_t*>(&u2);
                        ph[i] = *reinterpret_cast<const uint32_t*>(&h2);
                        amax2 = __vmaxu2(amax2, ph[i] & 0x7FFF7FFFu);
                    }
                    const int hcol = nb * (TILE_N / 2) + c * EPI_COLS;
                    stage_box_store(sStore + wi * 2 * ACC_BOX_BYTES, n_stores, pg, &tmD,
                                    gcol + c * EPI_COLS, grow, stream_policy, lane);
                    stage_box_store(sStore + wi * 2 * ACC_BOX_BYTES, n_stores, pu, &tmD,
                                    gcol + TILE_N / 2 + c * EPI_COLS, grow, stream_policy, lane);
                    stage_box_store(sStore + wi * 2 * ACC_BOX_BYTES, n_stores, ph, &tmD2, hcol,
                                    grow, stream_policy, lane);
                }
            } else {
                // chunk c + 1's TMEM load is issued as soon as chunk c's values
                // are computed, so it overlaps chunk c's staging and store
                uint32_t r[32];
                tmem_ld_32x32b_x32(tbase, r);
                for (int c = 0; c < n_chunks; ++c) {
                    tmem_ld_wait(r);
                    if (part) {
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const float4 p = part[(c * 8 + i) * 32 + lane];
                            const float q[4] = {p.x, p.y, p.z, p.w};
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                r[4 * i + e] =
                                    __float_as_uint(__fadd_rn(q[e], __uint_as_float(r[4 * i + e])));
                        }
                    } else if (MULTI && gpart) {
                        // parts 0..S-2 in order; a part's slots are 2 ranks x 4 warps apart
#pragma unroll 1
                        for (int p = 0; p < S - 1; ++p) {
                            const float4* src = gpart +
                                                (size_t)p * 2 * NUM_EPI_WARPS * kSplitSlotFloat4 +
                                                (size_t)(c * 8) * 32 + lane;
                            float4 v[8];
#pragma unroll
                            for (int i = 0; i < 8; ++i) v[i] = __ldcg(src + i * 32);
#pragma unroll
                            for (int i = 0; i < 8; ++i) {
                                const float q[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
                                for (int e = 0; e < 4; ++e)
                                    r[4 * i + e] = __float_as_uint(
                                        __fadd_rn(q[e], __uint_as_float(r[4 * i + e])));
                            }
                        }
                    }
                    if constexpr (EPI == LM_EPI_RELU2_BWD) {
                        // saved H of this chunk (two bf16 per word, columns
                        // 2i and 2i+1) from its half of the pair's box; dH
                        // goes back over it (each lane rewrites only its own
                        // row) and the box is TMA-stored after its second half
                        const int half = c & 1;
                        const uint32_t slot = h_used & 1u;
                        uint8_t* box = wide + slot * WIDE_BYTES;
                        if (half == 0) {
                            if (c >= 2 && c / 2 + 1 < n_pairs) {
                                // the next pair's box goes into the slot whose
                                // store was issued last
                                if (lane == 0) issue_h(c / 2 + 1);
                                ++h_issued;
                            }
                            if (!mbar_wait(&h_bar[slot], (h_used >> 1) & 1u, args.err, W_AUX)) {
                                ok = false;
                                break;
                            }
                        }
                        uint32_t hw[16];
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const uint4 v =
                                *reinterpret_cast<const uint4*>(box + sw128(lane, 4 * half + j));
                            hw[4 * j] = v.x;
                            hw[4 * j + 1] = v.y;
                            hw[4 * j + 2] = v.z;
                            hw[4 * j + 3] = v.w;
                        }
                        uint32_t packed[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            packed[i] = epi_pair<EPI>(r[2 * i], r[2 * i + 1], s, hw[i], amax2);
                        if (c + 1 < n_chunks)
                            tmem_ld_32x32b_x32(tbase + (uint32_t)((c + 1) * EPI_COLS), r);
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            *reinterpret_cast<uint4*>(box + sw128(lane, 4 * half + j)) =
                                make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2],
                                           packed[4 * j + 3]);
                        if (half == 1 || c + 1 == n_chunks) {
                            fence_proxy_async_smem();
                            __syncwarp();
                            if (lane == 0) {
                                tma_store_2d_hint(&tmD, smem_addr(box), gcol + (c & ~1) * EPI_COLS,
                                                  grow, stream_policy);
                                bulk_commit_group();
                            }
                            ++h_used;
                        }
                    } else if constexpr (EPI == LM_EPI_ACCUM_F32) {
                        // fp32 partial -> 128B-swizzled 32 x 32 fp32 box -> TMA reduce-add
                        uint8_t* dst =
                            sStore + wi * 2 * ACC_BOX_BYTES + (n_stores & 1u) * ACC_BOX_BYTES;
                        if (lane == 0) bulk_wait_group_read<1>();
                        __syncwarp();
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            *reinterpret_cast<float4*>(dst + lane * 128 + ((j ^ (lane & 7)) << 4)) =
                                make_float4(__fmul_rn(__uint_as_float(r[4 * j]), s),
                                            __fmul_rn(__uint_as_float(r[4 * j + 1]), s),
                                            __fmul_rn(__uint_as_float(r[4 * j + 2]), s),
                                            __fmul_rn(__uint_as_float(r[4 * j + 3]), s));
                        if (c + 1 < n_chunks)
                            tmem_ld_32x32b_x32(tbase + (uint32_t)((c + 1) * EPI_COLS), r);
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            tma_reduce_add_2d(&tmD, smem_addr(dst), gcol + c * EPI_COLS, grow);
                            bulk_commit_group();
                        }
                        ++n_stores;
                    } else {
                        uint32_t packed[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            packed[i] = epi_pair<EPI>(r[2 * i], r[2 * i + 1], s, 0u, amax2);
                        if (c + 1 < n_chunks)
                            tmem_ld_32x32b_x32(tbase + (uint32_t)((c + 1) * EPI_COLS), r);
                        // box n_wide & 1: before its first half is written, the
                        // store that last used it must have finished reading
                        const int half = c & 1;
                        uint8_t* box = wide + (n_wide & 1u) * WIDE_BYTES;
                        if (half == 0) {
                            if (lane == 0) bulk_wait_group_read<1>();
                            __syncwarp();
                        }
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            *reinterpret_cast<uint4*>(box + sw128(lane, 4 * half + j)) =
                                make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2],
                                           packed[4 * j + 3]);
                        if (half == 1 || c + 1 == n_chunks) {
                            fence_proxy_async_smem();
                            __syncwarp();
                            if (lane == 0) {
                                tma_store_2d_hint(&tmD, smem_addr(box), gcol + (c & ~1) * EPI_COLS,
                                                  grow, stream_policy);
                                bulk_commit_group();
                            }
                            ++n_wide;
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote_relaxed(tempty_leader + (uint32_t)(acc * 8));
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1u;
        }
        // H boxes still in flight (only after a wait ran out): let them land
        // (bounded) before the shared memory is released
        for (uint32_t j = h_used; j < h_issued; ++j)
            mbar_wait(&h_bar[j & 1u], (j >> 1) & 1u, args.err, W_AUX);
        if (lane == 0) bulk_wait_group<0>();
        reduce_amax<EPI>(max(amax2 & 0xFFFFu, amax2 >> 16), args.amax_out, lane);
    }

    tc_fence_before();
    __syncwarp();
    cluster_sync();  // peer shared memory and TMEM no longer in use
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, TMEM_COLS);
    }
}

}  // namespace pair

// =====================================================================
// Single-CTA kernel for thin problems (M <= 128): 128 x 256 tiles
// =====================================================================
namespace one {

constexpr int BM = 128, BN = 256;
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK;
constexpr int B_BYTES = BN * BK;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int B_MN_BLOCK = 128 * BK;  // one 128-wide block of an MN-major B tile
constexpr int NUM_EPI_THREADS = 128;
constexpr uint32_t TMEM_COLS = 2 * BN;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 256;

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
            int stage = 0;
            uint32_t phase = 0, issued = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < args.num_tiles && ok; t += gridDim.x) {
                int mb, nb;
                tile_coords(t, args.group_m, args.num_mb, args.num_nb, mb, nb);
                for (int kb = 0; kb < args.num_kb; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, args.err, W_EMPTY)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[stage], STAGE_BYTES);
                    if (args.a_mn)
                        tma_load_2d(smem_addr(sA + stage * A_BYTES), &tmA, &full[stage], mb * BM,
                                    kb * BK);
                    else
                        tma_load_2d(smem_addr(sA + stage * A_BYTES), &tmA, &full[stage], kb * BK,
                                    mb * BM);
                    if (args.b_mn) {
                        // two 128-wide MN blocks, B_MN_BLOCK bytes apart
                        for (int h = 0; h < BN / 128; ++h)
                            tma_load_2d(smem_addr(sB + stage * B_BYTES + h * B_MN_BLOCK), &tmB,
                                        &full[stage], nb * BN + h * 128, kb * BK);
                    } else {
                        tma_load_2d(smem_addr(sB + stage * B_BYTES), &tmB, &full[stage], kb * BK,
                                    nb * BN);
                    }
                    ++issued;
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            for (int s = 0; s < STAGES; ++s) {
                const uint32_t n = issued / STAGES + ((uint32_t)s < issued % STAGES ? 1u : 0u);
                if (n) mbar_wait(&full[s], (n - 1) & 1u, args.err, W_LOADS);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            const uint64_t a_step = args.a_mn ? (UMMA_K * 128) >> 4 : UMMA_K >> 4;
            const uint64_t b_step = args.b_mn ? (UMMA_K * 128) >> 4 : UMMA_K >> 4;
            const uint32_t b_lbo = args.b_mn ? (uint32_t)B_MN_BLOCK : 16u;
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
                    const uint64_t bd = smem_desc_sw128(smem_addr(sB + stage * B_BYTES), b_lbo);
#pragma unroll
                    for (int kk = 0; kk < BK / UMMA_K; ++kk)
                        mma_fp8(d_tmem, ad + (uint64_t)kk * a_step, bd + (uint64_t)kk * b_step,
                                args.idesc, (kb | kk) != 0 ? 1u : 0u);
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
            mma_commit(drain);
            mbar_wait(drain, 0, args.err, W_DRAIN);
        }
    } else {
        const int quarter = warp & 3;
        const float s = __fmul_rn(*args.inv_a, *args.inv_b);
        uint32_t amax = 0;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int t = blockIdx.x; t < args.num_tiles; t += gridDim.x) {
            int mb, nb;
            tile_coords(t, args.group_m, args.num_mb, args.num_nb, mb, nb);
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
                if constexpr (EPI == LM_EPI_ACCUM_F32) {
                    // each element has one owner thread: a plain read-modify-write
                    float* Df = static_cast<float*>(args.D) + off;
#pragma unroll
                    for (int v = 0; v < 8; ++v) {
                        if (col0 + v * 4 >= args.N) break;
                        float4 d4 = *reinterpret_cast<float4*>(Df + v * 4);
                        d4.x = __fadd_rn(d4.x, __fmul_rn(__uint_as_float(r[4 * v]), s));
                        d4.y = __fadd_rn(d4.y, __fmul_rn(__uint_as_float(r[4 * v + 1]), s));
                        d4.z = __fadd_rn(d4.z, __fmul_rn(__uint_as_float(r[4 * v + 2]), s));
                        d4.w = __fadd_rn(d4.w, __fmul_rn(__uint_as_float(r[4 * v + 3]), s));
                        *reinterpret_cast<float4*>(Df + v * 4) = d4;
                    }
                } else {
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        if (col0 + v * 8 >= args.N) break;
                        uint32_t hb[8] = {0, 0, 0, 0, 0, 0, 0, 0};
                        if (EPI == LM_EPI_RELU2_BWD) {
                            const uint4 a4 =
                                *reinterpret_cast<const uint4*>(args.aux + off + v * 8);
                            const uint32_t aw[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                hb[2 * i] = aw[i] & 0xFFFFu;
                                hb[2 * i + 1] = aw[i] >> 16;
                            }
                        }
                        uint32_t ob[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            ob[i] = epi_value<EPI>(r[v * 8 + i], s, hb[i], amax);
                        *reinterpret_cast<uint4*>(static_cast<uint16_t*>(args.D) + off + v * 8) =
                            make_uint4(ob[0] | (ob[1] << 16), ob[2] | (ob[3] << 16),
                                       ob[4] | (ob[5] << 16), ob[6] | (ob[7] << 16));
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&tempty[acc]);
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1u;
        }
        reduce_amax<EPI>(amax, args.amax_out, lane);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

}  // namespace one

// cudaFuncSetAttribute once per kernel and device
template <typename F>
bool ensure_smem(F* kernel, int bytes, bool (&done)[64]) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
    if (!done[dev]) {
        if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
            cudaSuccess)
            return false;
        done[dev] = true;
    }
    return true;
}

template <int EPI, bool MULTI, bool SIDE>
lm_status launch_pair_as(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& td,
                         const CUtensorMap& tx, const CUtensorMap& td2, const GemmArgs& a,
                         cudaStream_t s) {
    static bool done[64] = {};
    if (!ensure_smem(pair::gemm_fp8_pair_kernel<EPI, MULTI, SIDE>, pair::SMEM_BYTES, done))
        return LM_ERR_CUDA;
    const int sms = sm_count();
    if (sms < 2) return LM_ERR_CUDA;
    const int clusters = a.num_units < sms / 2 ? a.num_units : sms / 2;
    timing_mark(s, 'g');
    // the split tail's flags and, right after them, a fed A's ready bits:
    // one memset
    uint8_t* zero_at = nullptr;
    size_t zero_bytes = 0;
    if (a.split_flags && a.split_slots > 0) {
        zero_at = reinterpret_cast<uint8_t*>(a.split_flags);
        zero_bytes = (size_t)a.split_slots * 2 * NUM_EPI_WARPS * sizeof(unsigned int);
    }
    if (a.side_ready) {
        uint8_t* r = reinterpret_cast<uint8_t*>(a.side_ready);
        if (!zero_at) zero_at = r;
        zero_bytes = (size_t)(r - zero_at) +
                     side_ready_bytes(a.num_mb, a.side_ready_words);
    }
    if (zero_bytes && cudaMemsetAsync(zero_at, 0, zero_bytes, s) != cudaSuccess)
        return LM_ERR_CUDA;
    pair::gemm_fp8_pair_kernel<EPI, MULTI, SIDE>
        <<<2 * clusters, SIDE ? NUM_THREADS_SIDE : NUM_THREADS, pair::SMEM_BYTES, s>>>(
            ta, tb, td, tx, td2, a);
    return launch_status();
}

// No split or halves in one round: the lean instantiation; three or more parts
// (never for the gated epilogue): the one that reads partials from global memory.
// With a side cast (a.side_nvec > 0; plain and relu^2-forward epilogues, no
// multi-part tail) the instantiation with side warps; *side_done says whether
// this launch carries it.
template <int EPI>
lm_status launch_pair(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& td,
                      const CUtensorMap& tx, const CUtensorMap& td2, const GemmArgs& a,
                      cudaStream_t s, bool* side_done) {
    *side_done = false;
    if constexpr (EPI == kEpiSwigluFwd) {
        return launch_pair_as<EPI, false, false>(ta, tb, td, tx, td2, a, s);
    } else {
        const bool halves_in_one_round =
            a.split_parts <= 2 && a.num_units - a.split_first <= a.split_round;
        if (!halves_in_one_round) return launch_pair_as<EPI, true, false>(ta, tb, td, tx, td2, a, s);
        if constexpr (EPI == LM_EPI_NONE || EPI == LM_EPI_RELU2_FWD) {
            if (a.side_nvec > 0) {
                *side_done = true;
                return launch_pair_as<EPI, false, true>(ta, tb, td, tx, td2, a, s);
            }
        }
        return launch_pair_as<EPI, false, false>(ta, tb, td, tx, td2, a, s);
    }
}

template <int EPI>
lm_status launch_one(const CUtensorMap& ta, const CUtensorMap& tb, const GemmArgs& a,
                     cudaStream_t s) {
    static bool done[64] = {};
    if (!ensure_smem(one::gemm_fp8_kernel<EPI>, one::SMEM_BYTES, done)) return LM_ERR_CUDA;
    const int sms = sm_count();
    if (sms <= 0) return LM_ERR_CUDA;
    const int grid = a.num_tiles < sms ? a.num_tiles : sms;
    timing_mark(s, 'g');
    one::gemm_fp8_kernel<EPI><<<grid, NUM_THREADS, one::SMEM_BYTES, s>>>(ta, tb, a);
    return launch_status();
}

}  // namespace
}  // namespace lm

size_t lm::gemm_split_workspace_bytes() {
    return (size_t)kSplitMaxSlots * (kSplitTileBytes + 2 * NUM_EPI_WARPS * sizeof(unsigned int));
}

namespace lm {
namespace {

// Modelled time of the last wave's rem tiles run as S parts each, in units of
// one k-block of one tile: the rounds they take, each as long as one part's
// k-blocks plus the last part's reads of the other S - 1 partial sums.  Each
// read costs about 14 k-block times (5.6 us for 128 KB per CTA, read in 4 KB
// steps per warp): measured on B200 with the 48-tile wgrad of a 1024-row
// linear, where three parts over two rounds ran 15 us slower than no split.
double split_tail_cost(int rem, int num_kb, int C, int S) {
    const int per_round = C / S;
    const int rounds = (rem + per_round - 1) / per_round;
    return rounds * ((double)num_kb / S + 14.0 * (S - 1));
}

// Parts per tile for the last wave of a CTA-pair GEMM with num_tiles tiles of
// num_kb k-blocks on C clusters (1: no split).
//  - A last wave of rem <= C / 2 tiles is halved, as long as each half gets a
//    k-block; more parts only when the model above is 25% faster than halves.
//  - A fuller last wave takes the fastest S of the model when that is at least
//    10% faster than leaving the wave unsplit.
// S is at most kSplitMaxParts, each part gets two k-blocks or more when S > 2,
// and the partials fit the workspace (rem * (S - 1) <= kSplitMaxSlots).
int split_parts_for(int num_tiles, int num_kb, int C) {
    if (C < 2) return 1;
    const int rem = num_tiles % C;
    if (rem == 0 || num_kb < 2) return 1;
    const bool halves = 2 * rem <= C && rem <= kSplitMaxSlots;
    const double bound = halves ? 0.75 * split_tail_cost(rem, num_kb, C, 2) : 0.9 * num_kb;
    int best = halves ? 2 : 1;
    double best_cost = 1e300;
    for (int S = halves ? 3 : 2; S <= kSplitMaxParts; ++S) {
        if (C / S < 1 || num_kb < 2 * S || (int64_t)rem * (S - 1) > kSplitMaxSlots) continue;
        const double c = split_tail_cost(rem, num_kb, C, S);
        if (c <= bound && c < best_cost) {
            best = S;
            best_cost = c;
        }
    }
    return best;
}

}  // namespace
}  // namespace lm

extern "C" lm_status lm_fp8_gemm_split_plan(int64_t M, int64_t N, int64_t K, int sm_count,
                                            int* parts, int* tail_tiles) {
    if (!parts || !tail_tiles || M < 0 || N < 0 || K < 0 || sm_count < 2)
        return LM_ERR_INVALID_ARG;
    *parts = 1;
    *tail_tiles = 0;
    if (M <= 128 || N == 0 || K == 0) return LM_OK;  // the single-CTA kernel: never split
    const int64_t tiles = ((M + 255) / 256) * ((N + 255) / 256);
    const int64_t num_kb = (K + lm::BK - 1) / lm::BK;
    if (tiles >= (int64_t(1) << 31) || num_kb >= (int64_t(1) << 31)) return LM_ERR_UNSUPPORTED_SHAPE;
    const int C = sm_count / 2;
    const int S = lm::split_parts_for((int)tiles, (int)num_kb, C);
    if (S > 1) {
        *parts = S;
        *tail_tiles = (int)(tiles % C);
    }
    return LM_OK;
}

namespace lm {
namespace {

// The side cast as its own launch (when the GEMM launch cannot carry it).
lm_status side_cast_alone(const SideCast& sc, cudaStream_t s) {
    const CastItem it = {sc.x, sc.rows, sc.cols, sc.cols, sc.amax_in, sc.amax_out,
                         sc.scale_out, sc.inv_scale_out, sc.q, nullptr};
    return cast_set(&it, 1, sc.fmt, sc.relu2 ? 1 : 0, true, s);
}

}  // namespace
}  // namespace lm

lm_status lm::gemm_dispatch(const uint8_t* A, lm_fp8_format fa, const uint8_t* B,
                            lm_fp8_format fb, int64_t M, int64_t N, int64_t K, uint32_t flags,
                            const float* inv_scale_a, const float* inv_scale_b, int epi,
                            const void* aux, void* D, void* D2, float* amax_out, void* workspace,
                            size_t ws_bytes, lm_stream_t stream, const SideCast* side) {
    using namespace lm;
    if (side) {
        // checked like lm_fp8_amax_scale_cast's arguments, before any launch
        if ((side->fmt != LM_FP8_E4M3 && side->fmt != LM_FP8_E5M2) || side->rows < 0 ||
            side->cols < 0 || side->cols % 16 != 0 || !side->amax_in || !side->amax_out ||
            !side->scale_out || !side->inv_scale_out ||
            ((side->rows > 0 && side->cols > 0) && (!side->x || !side->q)))
            return LM_ERR_INVALID_ARG;
        if (!aligned16(side->x) || !aligned16(side->q)) return LM_ERR_ALIGNMENT;
        if (side->feeds_a && (side->q != A || side->rows != M || side->cols != K ||
                              side->fmt != fa || (flags & LM_GEMM_A_MN_MAJOR)))
            return LM_ERR_INVALID_ARG;
    }
    if ((fa != LM_FP8_E4M3 && fa != LM_FP8_E5M2) || (fb != LM_FP8_E4M3 && fb != LM_FP8_E5M2))
        return LM_ERR_UNSUPPORTED_FORMAT;
    if (fa == LM_FP8_E5M2 && fb == LM_FP8_E5M2) return LM_ERR_UNSUPPORTED_FORMAT;
    if (epi != LM_EPI_NONE && epi != LM_EPI_RELU2_FWD && epi != LM_EPI_RELU2_BWD &&
        epi != LM_EPI_ACCUM_F32 && epi != kEpiSwigluFwd)
        return LM_ERR_UNSUPPORTED_FORMAT;
    if (M < 0 || N < 0 || K < 0) return LM_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (M == 0 || N == 0) return side ? side_cast_alone(*side, s) : LM_OK;
    if (!D || !inv_scale_a || !inv_scale_b) return LM_ERR_INVALID_ARG;
    if (K > 0 && (!A || !B)) return LM_ERR_INVALID_ARG;
    if (epi == LM_EPI_RELU2_BWD && !aux) return LM_ERR_INVALID_ARG;
    if (epi == kEpiSwigluFwd && (!D2 || N % 256 != 0 || K == 0)) return LM_ERR_INVALID_ARG;
    if (flags & ~(LM_GEMM_A_MN_MAJOR | LM_GEMM_B_MN_MAJOR)) return LM_ERR_INVALID_ARG;
    const bool a_mn = (flags & LM_GEMM_A_MN_MAJOR) != 0, b_mn = (flags & LM_GEMM_B_MN_MAJOR) != 0;
    if (K % 16 != 0 || N % 8 != 0) return LM_ERR_UNSUPPORTED_SHAPE;
    // an MN-major operand's rows (one per K) must start on 16-byte boundaries
    if ((a_mn && M % 16 != 0) || (b_mn && N % 16 != 0)) return LM_ERR_UNSUPPORTED_SHAPE;
    if (M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31) || K >= (int64_t(1) << 31))
        return LM_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(A) || !aligned16(B) || !aligned16(D) || !aligned16(aux) || !aligned16(D2))
        return LM_ERR_ALIGNMENT;

    if (K == 0) {  // empty reduction: D = epi(0) = 0 (accumulating: D += 0), amax unchanged
        if (epi != LM_EPI_ACCUM_F32 &&
            cudaMemsetAsync(D, 0, (size_t)M * (size_t)N * 2, s) != cudaSuccess)
            return LM_ERR_CUDA;
        return side ? side_cast_alone(*side, s) : LM_OK;
    }
    if (side && (side->rows == 0 || side->cols == 0)) {  // nothing to cast: its scales alone
        if (lm_status st = side_cast_alone(*side, s)) return st;
        side = nullptr;
    }
    unsigned int* err = device_error_word();
    if (!err) return LM_ERR_CUDA;

    GemmArgs a;
    a.M = (int)M;
    a.N = (int)N;
    a.num_kb = (int)((K + BK - 1) / BK);
    a.inv_a = inv_scale_a;
    a.inv_b = inv_scale_b;
    a.aux = static_cast<const uint16_t*>(aux);
    a.D = D;
    a.D2 = D2;
    a.amax_out = epi == LM_EPI_ACCUM_F32 ? nullptr : amax_out;
    a.err = err;
    a.a_mn = a_mn ? 1 : 0;
    a.b_mn = b_mn ? 1 : 0;
    a.side_x = nullptr;
    a.side_q = nullptr;
    a.side_nvec = 0;
    a.side_fmt = 0;
    a.side_amax_in = nullptr;
    a.side_amax_out = a.side_scale_out = a.side_inv_out = nullptr;
    a.side_ready = nullptr;
    a.side_ready_words = 0;
    a.side_relu2 = 0;
    a.side_cols = 0;
    if (side) {
        a.side_x = static_cast<const uint4*>(side->x);
        a.side_q = reinterpret_cast<uint2*>(side->q);
        a.side_nvec = side->rows * side->cols / 8;
        a.side_fmt = (int)side->fmt;
        a.side_amax_in = side->amax_in;
        a.side_amax_out = side->amax_out;
        a.side_scale_out = side->scale_out;
        a.side_inv_out = side->inv_scale_out;
        a.side_relu2 = side->relu2 ? 1 : 0;
        a.side_cols = (int)side->cols;
    }

    CUtensorMap ta, tb;
    if (M > 128 || epi == kEpiSwigluFwd) {
        a.num_mb = (int)((M + pair::TILE_M - 1) / pair::TILE_M);
        a.num_nb = (int)((N + pair::TILE_N - 1) / pair::TILE_N);
        a.num_tiles = a.num_mb * a.num_nb;
        // Sweep the smaller operand's dimension fastest: every wave of tiles
        // then re-reads all of the smaller operand, which stays in L2, while
        // the larger one streams through once.  N <= M: column-blocks fastest
        // (groups of one row-block); otherwise row-blocks fastest (one group
        // spanning M).
        a.stream_a = N <= M ? 1 : 0;
        a.group_m = a.stream_a ? 1 : a.num_mb;
        // split-K tail: with a workspace, the last wave's rem tiles may run as
        // S parts each over ranges of K, P = C / S tiles per round of C units
        a.num_units = a.num_tiles;
        a.split_first = a.num_tiles;
        a.split_parts = 1;
        a.split_round = 1;
        a.split_per_round = 1;
        a.split_slots = 0;
        a.split_ws = nullptr;
        a.split_flags = nullptr;
        const int sms = sm_count();
        if (sms < 2) return LM_ERR_CUDA;
        const int C = sms / 2;
        const int rem = a.num_tiles % C;
        const int S = workspace && epi != kEpiSwigluFwd && aligned16(workspace)
                          ? split_parts_for(a.num_tiles, a.num_kb, C)
                          : 1;
        const size_t slots = (size_t)rem * (size_t)(S - 1);
        if (S > 1 &&
            ws_bytes >= slots * (kSplitTileBytes + 2 * NUM_EPI_WARPS * sizeof(unsigned int))) {
            const int P = C / S;
            const int rounds = (rem + P - 1) / P;
            a.split_first = a.num_tiles - rem;
            a.split_parts = S;
            a.split_round = C;
            a.split_per_round = P;
            a.split_slots = (int)slots;
            // full rounds, then the last round's tiles (no idle units at the end)
            a.num_units = a.split_first + (rounds - 1) * C + (rem - (rounds - 1) * P) * S;
            a.split_ws = static_cast<float4*>(workspace);
            a.split_flags = reinterpret_cast<unsigned int*>(static_cast<uint8_t*>(workspace) +
                                                            slots * kSplitTileBytes);
        }
        if (side && side->feeds_a) {
            // A cast by the side warps ahead of the tiles: only where the launch
            // has side warps (no multi-part split) and the workspace holds the
            // units' ready bits after the split tail's flags; otherwise A is
            // cast by its own launch first
            const bool side_warps = (epi == LM_EPI_NONE || epi == LM_EPI_RELU2_FWD) &&
                                    a.split_parts <= 2 &&
                                    a.num_units - a.split_first <= a.split_round;
            const size_t used =
                (size_t)a.split_slots * (kSplitTileBytes + 2 * NUM_EPI_WARPS * sizeof(unsigned int));
            const int words = (a.num_kb + 31) / 32;
            const size_t need = used + side_ready_bytes(a.num_mb, words);
            if (side_warps && workspace && aligned16(workspace) && ws_bytes >= need) {
                a.side_ready =
                    reinterpret_cast<unsigned int*>(static_cast<uint8_t*>(workspace) + used);
                a.side_ready_words = words;
            } else {
                const lm_status cs = side_cast_alone(*side, s);
                if (cs != LM_OK) return cs;
                side = nullptr;
                a.side_nvec = 0;
            }
        }
        a.idesc = idesc_f8((uint32_t)fa, (uint32_t)fb, pair::TILE_M, pair::TILE_N, a.a_mn, a.b_mn);
        CUtensorMap td, tx;
        // K-major: [rows x K] boxes of 128 rows x 128 K; MN-major: [K x cols]
        // boxes of 128 K x 128 columns
        const bool mok =
            (a_mn ? encode_tmap_u8(&ta, A, (uint64_t)K, (uint64_t)M, (uint64_t)M, BK, 128)
                  : encode_tmap_u8(&ta, A, (uint64_t)M, (uint64_t)K, (uint64_t)K, 128, BK)) &&
            (b_mn ? encode_tmap_u8(&tb, B, (uint64_t)K, (uint64_t)N, (uint64_t)N, BK, 128)
                  : encode_tmap_u8(&tb, B, (uint64_t)N, (uint64_t)K, (uint64_t)K, 128, BK));
        if (!mok) return LM_ERR_CUDA;
        // D: fp32 32 x 32 boxes (accumulating), bf16 32 x 32 (gated), bf16 32 x 64
        // (plain and relu^2); the saved H like D
        const bool dok =
            epi == LM_EPI_ACCUM_F32
                ? encode_tmap_f32_sw128(&td, D, (uint64_t)M, (uint64_t)N, 32, pair::EPI_COLS)
            : epi == kEpiSwigluFwd
                ? encode_tmap_bf16_sw64(&td, D, (uint64_t)M, (uint64_t)N, 32, pair::EPI_COLS)
                : encode_tmap_bf16_sw128(&td, D, (uint64_t)M, (uint64_t)N, 32, pair::WIDE_COLS);
        if (!dok) return LM_ERR_CUDA;
        if (epi == LM_EPI_RELU2_BWD) {
            if (!encode_tmap_bf16_sw128(&tx, aux, (uint64_t)M, (uint64_t)N, 32, pair::WIDE_COLS))
                return LM_ERR_CUDA;
        } else {
            tx = td;  // unused
        }
        CUtensorMap td2 = td;  // unused unless the gated epilogue writes h
        if (epi == kEpiSwigluFwd &&
            !encode_tmap_bf16_sw64(&td2, D2, (uint64_t)M, (uint64_t)(N / 2), 32, pair::EPI_COLS))
            return LM_ERR_CUDA;
        bool side_done = false;
        lm_status st;
        switch (epi) {
            case LM_EPI_NONE:
                st = launch_pair<LM_EPI_NONE>(ta, tb, td, tx, td2, a, s, &side_done);
                break;
            case LM_EPI_RELU2_FWD:
                st = launch_pair<LM_EPI_RELU2_FWD>(ta, tb, td, tx, td2, a, s, &side_done);
                break;
            case LM_EPI_RELU2_BWD:
                st = launch_pair<LM_EPI_RELU2_BWD>(ta, tb, td, tx, td2, a, s, &side_done);
                break;
            case LM_EPI_ACCUM_F32:
                st = launch_pair<LM_EPI_ACCUM_F32>(ta, tb, td, tx, td2, a, s, &side_done);
                break;
            default: st = launch_pair<kEpiSwigluFwd>(ta, tb, td, tx, td2, a, s, &side_done);
        }
        if (st != LM_OK || side_done || !side) return st;
        return side_cast_alone(*side, s);
    }
    if (side && side->feeds_a) {  // the thin kernel has no side warps: A first
        const lm_status cs = side_cast_alone(*side, s);
        if (cs != LM_OK) return cs;
        side = nullptr;
    }
    a.num_mb = (int)((M + one::BM - 1) / one::BM);
    a.num_nb = (int)((N + one::BN - 1) / one::BN);
    a.num_tiles = a.num_mb * a.num_nb;
    a.num_units = a.num_tiles;
    a.split_first = a.num_tiles;
    a.split_parts = 1;
    a.split_round = 1;
    a.split_per_round = 1;
    a.split_slots = 0;
    a.split_ws = nullptr;
    a.split_flags = nullptr;
    a.group_m = 16;
    a.stream_a = 0;
    a.idesc = idesc_f8((uint32_t)fa, (uint32_t)fb, one::BM, one::BN, a.a_mn, a.b_mn);
    const bool mok =
        (a_mn ? encode_tmap_u8(&ta, A, (uint64_t)K, (uint64_t)M, (uint64_t)M, BK, one::BM)
              : encode_tmap_u8(&ta, A, (uint64_t)M, (uint64_t)K, (uint64_t)K, one::BM, BK)) &&
        (b_mn ? encode_tmap_u8(&tb, B, (uint64_t)K, (uint64_t)N, (uint64_t)N, BK, 128)
              : encode_tmap_u8(&tb, B, (uint64_t)N, (uint64_t)K, (uint64_t)K, one::BN, BK));
    if (!mok) return LM_ERR_CUDA;
    lm_status st;
    switch (epi) {
        case LM_EPI_NONE: st = launch_one<LM_EPI_NONE>(ta, tb, a, s); break;
        case LM_EPI_RELU2_FWD: st = launch_one<LM_EPI_RELU2_FWD>(ta, tb, a, s); break;
        case LM_EPI_RELU2_BWD: st = launch_one<LM_EPI_RELU2_BWD>(ta, tb, a, s); break;
        default: st = launch_one<LM_EPI_ACCUM_F32>(ta, tb, a, s);
    }
    if (st != LM_OK || !side) return st;
    return side_cast_alone(*side, s);
}

extern "C" size_t lm_fp8_gemm_workspace_size(void) { return lm::gemm_split_workspace_bytes(); }

extern "C" lm_status lm_fp8_gemm_ex(const uint8_t* A, lm_fp8_format fa, const uint8_t* B,
                                    lm_fp8_format fb, int64_t M, int64_t N, int64_t K,
                                    uint32_t flags, const float* inv_scale_a,
                                    const float* inv_scale_b, lm_epilogue epi, const void* aux,
                                    void* D, float* amax_out, void* workspace, size_t ws_bytes,
                                    lm_stream_t stream) {
    if (epi != LM_EPI_NONE && epi != LM_EPI_RELU2_FWD && epi != LM_EPI_RELU2_BWD &&
        epi != LM_EPI_ACCUM_F32)
        return LM_ERR_UNSUPPORTED_FORMAT;
    return lm::gemm_dispatch(A, fa, B, fb, M, N, K, flags, inv_scale_a, inv_scale_b, (int)epi,
                             aux, D, nullptr, amax_out, workspace, ws_bytes, stream);
}

extern "C" lm_status lm_fp8_gemm(const uint8_t* A, lm_fp8_format fa, const uint8_t* B,
                                 lm_fp8_format fb, int64_t M, int64_t N, int64_t K,
                                 const float* inv_scale_a, const float* inv_scale_b,
                                 lm_epilogue epi, const void* aux, void* D, float* amax_out,
                                 lm_stream_t stream) {
    return lm_fp8_gemm_ex(A, fa, B, fb, M, N, K, 0u, inv_scale_a, inv_scale_b, epi, aux, D,
                          amax_out, nullptr, 0, stream);
}
