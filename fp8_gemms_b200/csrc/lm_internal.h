// lm_internal.h -- host-side helpers shared by the translation units of
// libfp8lm.so (not part of the public ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <initializer_list>

#include "lm_fp8.h"

namespace lm {

// Device address of the current device's error word (0 = no error; else the
// code of the bounded wait that ran out).  nullptr if CUDA is unusable.
unsigned int* device_error_word();

// Device error codes: 0x1xx-0x3xx a bounded wait ran out (LM_ERR_TIMEOUT),
// 0x4xx invalid device-side data (LM_ERR_INVALID_ARG), 0x5xx a non-finite
// value where the method needs a finite one (LM_ERR_NONFINITE).
constexpr unsigned int kErrNonfiniteAmax = 0x501u;  // a cast met a NaN or infinite amax

// Multiprocessor count of the current device (cached per device).
int sm_count();

// 2-D uint8 tensor map for a row-major [rows x cols] matrix (cols
// contiguous, row pitch `pitch` bytes), box [box_rows x box_cols] with the
// 128-byte swizzle; out-of-bounds elements read as zero.
bool encode_tmap_u8(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                    uint64_t pitch, uint32_t box_rows, uint32_t box_cols);

// 2-D bf16 tensor map for a row-major [rows x cols] matrix, box
// [box_rows x box_cols] with the 64-byte swizzle (box_cols * 2 must be 64);
// used for the epilogue's TMA stores of D and loads of the saved H.
bool encode_tmap_bf16_sw64(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                           uint32_t box_rows, uint32_t box_cols);

// The same with the 128-byte swizzle (box_cols * 2 must be 128): the plain and
// relu^2 epilogues' 32 x 64 boxes.
bool encode_tmap_bf16_sw128(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                            uint32_t box_rows, uint32_t box_cols);

// 2-D fp32 tensor map for a row-major [rows x cols] matrix, box
// [box_rows x box_cols] with the 128-byte swizzle (box_cols * 4 must be 128);
// used for the accumulating epilogue's TMA reduce-adds.
bool encode_tmap_f32_sw128(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                           uint32_t box_rows, uint32_t box_cols);

// 2-D bf16 tensor map, no swizzle, row pitch `pitch` bytes (a multiple of
// 16), box [box_rows x box_cols]; out-of-bounds elements read as zero.
bool encode_tmap_bf16_plain(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                            uint64_t pitch, uint32_t box_rows, uint32_t box_cols);

// Epilogue used only inside the library (the gated MLP's up GEMM): D is the
// interleaved G|U pre-activation (plain bf16 epilogue on a GEMM whose N is
// 2f, gate and up alternating in 128-column blocks) and D2 receives
// h = bf16(silu(G) U) [M x N/2]; amax_out gets max |h|.
constexpr int kEpiSwigluFwd = 4;

// A cast that a GEMM launch runs in extra warps beside its tiles: a contiguous
// bf16 tensor whose amax has already been reduced (by an earlier kernel on
// the stream) is cast to row-major codes at the scale that amax gives, and
// its {amax, scale, inv_scale} are written.  The GEMM must neither read the
// codes nor write the input.  Where the GEMM launch cannot carry it (the
// thin kernel, a multi-part split tail, an empty GEMM), gemm_dispatch runs
// the cast as its own launch after the GEMM instead; the results are the same
// bits either way.  An empty tensor (no rows or no columns) gets its scale
// block alone, from amax_in, in a launch of its own.
struct SideCast {
    const void* x;  // bf16 [rows x cols], contiguous
    int64_t rows, cols;
    lm_fp8_format fmt;
    const float* amax_in;
    float *amax_out, *scale_out, *inv_scale_out;
    uint8_t* q;  // [rows x cols] codes
    int relu2 = 0;    // cast h = bf16(relu(x)^2) instead of x
    // The codes are the GEMM's own A ([M x K], K-major, format fa, q == A):
    // the side warps cast it unit by unit ahead of the tiles that read it,
    // and the inverse scale A is dequantised with comes from amax_in.
    // Without a workspace to hold the units' ready bits, or where the
    // launch has no side warps, the cast runs as its own launch first.
    int feeds_a = 0;
};

// lm_fp8_gemm_ex with the internal epilogues, a second output and an
// optional side cast.
lm_status gemm_dispatch(const uint8_t* A, lm_fp8_format fa, const uint8_t* B, lm_fp8_format fb,
                        int64_t M, int64_t N, int64_t K, uint32_t flags, const float* inv_scale_a,
                        const float* inv_scale_b, int epi, const void* aux, void* D, void* D2,
                        float* amax_out, void* workspace, size_t ws_bytes, lm_stream_t stream,
                        const SideCast* side = nullptr);

// Workspace bytes that let any GEMM split its last wave (lm_fp8_gemm_workspace_size).
size_t gemm_split_workspace_bytes();

// One tensor of lm::cast_set: the arguments of lm_fp8_amax_scale_cast.
struct CastItem {
    const void* x;
    int64_t rows, cols, ld;
    const float* amax_in;
    float *amax_out, *scale_out, *inv_scale_out;
    uint8_t *q, *qT;
    // with q and qT NULL: reduce the amax only and leave the scales to a
    // later side cast (no scales-only launch)
    bool amax_only = false;
};
constexpr int kMaxCastSet = 3;

// lm_fp8_amax_scale_cast of up to kMaxCastSet tensors that share the format
// and relu2_input, with one launch for all their amax reductions and one for
// all their TMA-fed casts.  amax_zeroed: the caller has already zeroed, on
// this stream, every amax_out whose amax_in is NULL, so no memset is issued.
lm_status cast_set(const CastItem* items, int n, lm_fp8_format fmt, int relu2_input,
                   bool amax_zeroed, cudaStream_t s);

// If the calling thread attached timing events, record the next one on `s`
// (call right before a kernel launch); `kind` labels the launch.
void timing_mark(cudaStream_t s, char kind);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Every pointer 16-byte aligned (a null pointer counts as aligned).  The
// composite entry points check all their tensors with it before the first
// launch, so a misaligned output is refused with nothing enqueued.
inline bool all_aligned16(std::initializer_list<const void*> ps) {
    for (const void* p : ps)
        if (!aligned16(p)) return false;
    return true;
}

inline lm_status launch_status() {
    return cudaGetLastError() == cudaSuccess ? LM_OK : LM_ERR_CUDA;
}

}  // namespace lm
