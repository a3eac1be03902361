// lm_api.cu -- library-wide entry points: device error word, status strings,
// version, and the host helpers (SM count, TMA descriptor encoding).
#include <cudaTypedefs.h>

#include <mutex>

#include "lm_internal.h"
#include "lm_ptx.cuh"

namespace lm {

// One per device (a __device__ variable is instantiated on every device that
// loads the module).  Kernels receive its address and atomicCAS a nonzero
// code into it when a bounded wait runs out.
__device__ unsigned int g_error_word = 0;

namespace {
constexpr int kMaxDevices = 64;
unsigned int* g_err_ptr[kMaxDevices] = {};
int g_sms[kMaxDevices] = {};
std::mutex g_mu;

int current_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
    return dev;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000,
                                             cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}
struct TimingState {
    void* const* events = nullptr;
    int capacity = 0;
    int count = 0;
    char kinds[4096];  // labels of the first 4096 recorded launches
};
thread_local TimingState t_timing;
}  // namespace

void timing_mark(cudaStream_t s, char kind) {
    TimingState& t = t_timing;
    if (!t.events || t.count >= t.capacity) return;
    cudaEventRecord(static_cast<cudaEvent_t>(t.events[t.count]), s);
    if (t.count < (int)sizeof(t.kinds)) t.kinds[t.count] = kind;
    ++t.count;
}

unsigned int* device_error_word() {
    int dev = current_device();
    if (dev < 0) return nullptr;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_err_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_error_word) != cudaSuccess) return nullptr;
        g_err_ptr[dev] = static_cast<unsigned int*>(p);
    }
    return g_err_ptr[dev];
}

int sm_count() {
    int dev = current_device();
    if (dev < 0) return 0;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_sms[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return 0;
        g_sms[dev] = n;
    }
    return g_sms[dev];
}

bool encode_tmap_u8(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                    uint64_t pitch, uint32_t box_rows, uint32_t box_cols) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {pitch};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool encode_tmap_bf16_sw64(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                           uint32_t box_rows, uint32_t box_cols) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool encode_tmap_bf16_sw128(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                            uint32_t box_rows, uint32_t box_cols) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool encode_tmap_f32_sw128(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                           uint32_t box_rows, uint32_t box_cols) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 4};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool encode_tmap_bf16_plain(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                            uint64_t pitch, uint32_t box_rows, uint32_t box_cols) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {pitch};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

namespace {
// A wait that nothing satisfies: exercises the bounded-wait expiry path.
__global__ void selftest_wait_kernel(unsigned int* err, uint64_t limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait_limit(&bar, 0, err, 0x301u, limit_ns);
}
}  // namespace

}  // namespace lm

extern "C" {

lm_status lm_selftest_bounded_wait(uint32_t limit_ms, lm_stream_t stream) {
    if (limit_ms < 1 || limit_ms > 5000) return LM_ERR_INVALID_ARG;
    unsigned int* err = lm::device_error_word();
    if (!err) return LM_ERR_CUDA;
    lm::selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        err, (uint64_t)limit_ms * 1000000ull);
    return lm::launch_status();
}

lm_status lm_get_error(lm_stream_t stream, uint32_t* where_out) {
    if (where_out) *where_out = 0;
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
        return LM_ERR_CUDA;
    unsigned int* p = lm::device_error_word();
    if (!p) return LM_ERR_CUDA;
    unsigned int v = 0, zero = 0;
    if (cudaMemcpy(&v, p, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return LM_ERR_CUDA;
    if (v != 0 && cudaMemcpy(p, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
        return LM_ERR_CUDA;
    if (where_out) *where_out = v;
    if (!v) return LM_OK;
    if ((v & 0xF00u) == 0x400u) return LM_ERR_INVALID_ARG;
    if ((v & 0xF00u) == 0x500u) return LM_ERR_NONFINITE;
    return LM_ERR_TIMEOUT;
}

const char* lm_status_string(lm_status s) {
    switch (s) {
        case LM_OK: return "LM_OK";
        case LM_ERR_INVALID_ARG: return "LM_ERR_INVALID_ARG: null pointer, negative size or workspace too small";
        case LM_ERR_ALIGNMENT: return "LM_ERR_ALIGNMENT: pointer or row pitch not 16-byte aligned";
        case LM_ERR_UNSUPPORTED_SHAPE: return "LM_ERR_UNSUPPORTED_SHAPE: dimension not a supported multiple";
        case LM_ERR_UNSUPPORTED_FORMAT: return "LM_ERR_UNSUPPORTED_FORMAT: unsupported format pair or epilogue";
        case LM_ERR_CUDA: return "LM_ERR_CUDA: CUDA call or kernel launch failed";
        case LM_ERR_TIMEOUT: return "LM_ERR_TIMEOUT: a device-side bounded wait ran out";
        case LM_ERR_NONFINITE: return "LM_ERR_NONFINITE: a cast met a NaN or infinite amax";
    }
    return "unknown lm_status";
}

int lm_version(void) { return 100; }

void lm_timing_attach(void* const* events, int capacity) {
    lm::t_timing.events = events;
    lm::t_timing.capacity = events ? capacity : 0;
    lm::t_timing.count = 0;
}

int lm_timing_detach(void) {
    lm::t_timing.events = nullptr;
    lm::t_timing.capacity = 0;
    return lm::t_timing.count;
}

int lm_timing_kinds(char* out, int cap) {
    const int n = lm::t_timing.count < (int)sizeof(lm::t_timing.kinds) ? lm::t_timing.count
                                                                        : (int)sizeof(lm::t_timing.kinds);
    const int m = n < cap ? n : cap;
    for (int i = 0; i < m; ++i) out[i] = lm::t_timing.kinds[i];
    return m;
}

}  // extern "C"
