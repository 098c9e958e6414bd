// Host-side plumbing shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdint>
#include <cstdio>

#include "../../include/moe.h"

namespace swb {

// Records a thread-local message for moe_last_error() and returns `s`.
moe_status fail(moe_status s, const char* fmt, ...);

// Wraps every CUDA runtime call the library makes: honours the test hook
// (moe_debug_fail_next_cuda_calls) and turns errors into MOE_ERR_CUDA.
bool cuda_injected_failure();
moe_status cuda_check(cudaError_t e, const char* what);

// The registers per SM a gated launch may take, as set by the test hook
// moe_debug_gated_regs_per_sm (0: the library's own limit).
int64_t gated_regs_override();

#define SWB_CUDA(call)                                                          \
    do {                                                                        \
        if (::swb::cuda_injected_failure())                                     \
            return ::swb::fail(MOE_ERR_CUDA, "%s: injected failure", #call);    \
        cudaError_t _e = (call);                                                \
        if (_e != cudaSuccess) return ::swb::cuda_check(_e, #call);             \
    } while (0)

// Counts the kernels the library has launched (process-wide).
void count_launch();

// After a launch: report launch-configuration errors, count the launch.
#define SWB_LAUNCHED(what)                                                      \
    do {                                                                        \
        cudaError_t _e = cudaGetLastError();                                    \
        if (_e != cudaSuccess) return ::swb::cuda_check(_e, what);              \
        ::swb::count_launch();                                                  \
    } while (0)

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Device address of the library's device error word on the current device.
moe_status device_error_word(int** out);

// Number of SMs of the current device (cached per device).
moe_status sm_count(int* out);

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// dependency on libcuda).
moe_status encode_tiled(CUtensorMap* map, CUtensorMapDataType dtype, uint32_t rank, void* base,
                        const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                        CUtensorMapSwizzle swizzle);

// cuStreamWriteValue32 through the runtime's driver entry point (the 32-bit
// stream memory operations need no device opt-in on CUDA 12): the write lands
// once the stream's earlier work has finished.
moe_status stream_write_u32(cudaStream_t s, uint32_t* addr, uint32_t value);

// Progress value that releases chunk `chunk` of a paced fetch of n_chunks:
// base for the first lead_chunks, the others spread evenly over the reports
// base + 1 .. base + steps + 1 (moe_pace_threshold).
uint32_t pace_threshold(int64_t chunk, int64_t n_chunks, int32_t lead_chunks, uint32_t base,
                        int32_t steps);

// Bits of the device error word.
enum : int { kDevErrTimeout = 1, kDevErrIndex = 2 };

}  // namespace swb
