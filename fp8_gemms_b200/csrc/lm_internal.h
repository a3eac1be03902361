// lm_internal.h -- host-side helpers shared by the translation units of
// libfp8lm.so (not part of the public ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "lm_fp8.h"

namespace lm {

// Device address of the current device's error word (0 = no error; else the
// code of the bounded wait that ran out).  nullptr if CUDA is unusable.
unsigned int* device_error_word();

// Multiprocessor count of the current device (cached per device).
int sm_count();

// 2-D uint8 tensor map for a row-major [rows x cols] matrix (cols
// contiguous, row pitch `pitch` bytes), box [box_rows x box_cols] with the
// 128-byte swizzle; out-of-bounds elements read as zero.
bool encode_tmap_u8(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                    uint64_t pitch, uint32_t box_rows, uint32_t box_cols);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline lm_status launch_status() {
    return cudaGetLastError() == cudaSuccess ? LM_OK : LM_ERR_CUDA;
}

}  // namespace lm
