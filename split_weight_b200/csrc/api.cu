// Library-wide entry points: status text, errors, the device error word,
// tensor-map encoding, expert image layout and the copy-engine prefetch.
#include <atomic>
#include <chrono>
#include <cstring>
#include <mutex>
#include <thread>

#include "device.cuh"
#include "internal.h"

namespace swb {

namespace {
thread_local char g_last_error[512] = "";
std::atomic<int> g_fail_next{0};
std::atomic<int64_t> g_gated_regs{0};   // 0: the library's limit

// One error word per device, in device memory owned by this library's
// module (a __device__ variable: the library still allocates nothing).
__device__ int g_device_error_word;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
std::mutex g_mu;
EncodeTiledFn g_encode = nullptr;
constexpr int kMaxDevices = 64;
int g_sm_count[kMaxDevices] = {0};
int* g_err_word[kMaxDevices] = {nullptr};
}  // namespace

moe_status fail(moe_status s, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
    va_end(ap);
    return s;
}

int64_t gated_regs_override() { return g_gated_regs.load(); }

bool cuda_injected_failure() {
    int n = g_fail_next.load();
    while (n > 0) {
        if (g_fail_next.compare_exchange_weak(n, n - 1)) return true;
    }
    return false;
}

moe_status cuda_check(cudaError_t e, const char* what) {
    // reported here: clear it so the next launch check does not report it again
    (void)cudaGetLastError();
    return fail(MOE_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

moe_status device_error_word(int** out) {
    int dev = 0;
    SWB_CUDA(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kMaxDevices) return fail(MOE_ERR_UNSUPPORTED, "device %d", dev);
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_err_word[dev]) {
        void* p = nullptr;
        SWB_CUDA(cudaGetSymbolAddress(&p, g_device_error_word));
        g_err_word[dev] = static_cast<int*>(p);
    }
    *out = g_err_word[dev];
    return MOE_OK;
}

moe_status sm_count(int* out) {
    int dev = 0;
    SWB_CUDA(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kMaxDevices) return fail(MOE_ERR_UNSUPPORTED, "device %d", dev);
    if (!g_sm_count[dev]) {
        int n = 0;
        SWB_CUDA(cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev));
        g_sm_count[dev] = n;
    }
    *out = g_sm_count[dev];
    return MOE_OK;
}

moe_status encode_tiled(CUtensorMap* map, CUtensorMapDataType dtype, uint32_t rank, void* base,
                        const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                        CUtensorMapSwizzle swizzle) {
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!g_encode) {
            void* fn = nullptr;
            cudaDriverEntryPointQueryResult q;
            if (cuda_injected_failure())
                return fail(MOE_ERR_CUDA, "cudaGetDriverEntryPoint: injected failure");
            cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn,
                                                    cudaEnableDefault, &q);
            if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn)
                return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
            g_encode = reinterpret_cast<EncodeTiledFn>(fn);
        }
    }
    cuuint64_t d[5], s[4];
    cuuint32_t b[5], es[5];
    for (uint32_t i = 0; i < rank; ++i) {
        d[i] = dims[i];
        b[i] = box[i];
        es[i] = 1;
        if (i + 1 < rank) s[i] = strides_bytes[i];
    }
    CUresult r = g_encode(map, dtype, rank, base, d, s, b, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return fail(MOE_ERR_INVALID_ARG, "cuTensorMapEncodeTiled failed (CUresult %d)", (int)r);
    return MOE_OK;
}

using StreamValue32Fn = CUresult (*)(CUstream, CUdeviceptr, cuuint32_t, unsigned int);
namespace {
StreamValue32Fn g_write32 = nullptr;

moe_status stream_value_fn(const char* name, StreamValue32Fn* cache, StreamValue32Fn* out) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!*cache) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cuda_injected_failure())
            return fail(MOE_ERR_CUDA, "cudaGetDriverEntryPoint: injected failure");
        const cudaError_t e = cudaGetDriverEntryPoint(name, &fn, cudaEnableDefault, &q);
        if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn)
            return fail(MOE_ERR_UNSUPPORTED, "%s entry point unavailable", name);
        *cache = reinterpret_cast<StreamValue32Fn>(fn);
    }
    *out = *cache;
    return MOE_OK;
}
}  // namespace

moe_status stream_write_u32(cudaStream_t s, uint32_t* addr, uint32_t value) {
    StreamValue32Fn fn = nullptr;
    moe_status st = stream_value_fn("cuStreamWriteValue32", &g_write32, &fn);
    if (st != MOE_OK) return st;
    if (cuda_injected_failure()) return fail(MOE_ERR_CUDA, "cuStreamWriteValue32: injected failure");
    const CUresult r = fn(reinterpret_cast<CUstream>(s), reinterpret_cast<CUdeviceptr>(addr), value,
                          CU_STREAM_WRITE_VALUE_DEFAULT);
    if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "cuStreamWriteValue32 failed (CUresult %d)", (int)r);
    return MOE_OK;
}


uint32_t pace_threshold(int64_t chunk, int64_t n_chunks, int32_t lead_chunks, uint32_t base,
                        int32_t steps) {
    if (chunk < lead_chunks) return base;
    const int64_t paced = n_chunks - lead_chunks, j = chunk - lead_chunks;
    return base + (uint32_t)(((j + 1) * ((int64_t)steps + 1)) / (paced + 1));
}

// A paced chunk's wait, one thread on the copy stream: polls the progress
// word (acquire loads at GPU scope) until it reaches the threshold, or gives
// up after kPaceWaitNs and lets the chunk go (pacing only spreads the copy;
// the readiness flags, not this wait, order it before its readers).  A
// bounded kernel rather than a stream memory wait, so that no ordering of
// streams on the hardware queues can turn it into a wait without end.
constexpr uint64_t kPaceWaitNs = 200000000ull;   // 200 ms

__global__ void k_pace_wait(const uint32_t* word, uint32_t threshold, uint64_t limit_ns) {
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        uint32_t v;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(word) : "memory");
        if ((int32_t)(v - threshold) >= 0) return;
        if (globaltimer_ns() - t0 > limit_ns) return;
        __nanosleep(2000);
    }
}

// The chunked copy of moe_prefetch_layer_flagged / _paced: per chunk an
// optional wait for the progress word, the copy, then the chunk's flag.
moe_status flagged_copy(const void* src, void* dst, size_t bytes, size_t chunk_bytes,
                        cudaStream_t copy_stream, cudaEvent_t wait_free, uint32_t* flags,
                        uint32_t epoch, const moe_progress* pace, int32_t lead_chunks,
                        cudaEvent_t ready_out) {
    if (wait_free) SWB_CUDA(cudaStreamWaitEvent(copy_stream, wait_free, 0));
    const int64_t n = (int64_t)((bytes + chunk_bytes - 1) / chunk_bytes);
    int64_t c = 0;
    for (size_t off = 0; off < bytes; off += chunk_bytes, ++c) {
        moe_status st;
        if (pace) {
            const uint32_t thr = pace_threshold(c, n, lead_chunks, pace->base, pace->steps);
            if (thr != pace->base) {   // the lead chunks go at once
                if (cuda_injected_failure()) return fail(MOE_ERR_CUDA, "k_pace_wait: injected failure");
                k_pace_wait<<<1, 1, 0, copy_stream>>>(pace->word, thr, kPaceWaitNs);
                SWB_LAUNCHED("k_pace_wait");
            }
        }
        const size_t len = bytes - off < chunk_bytes ? bytes - off : chunk_bytes;
        SWB_CUDA(cudaMemcpyAsync(static_cast<char*>(dst) + off,
                                 static_cast<const char*>(src) + off, len,
                                 cudaMemcpyDeviceToDevice, copy_stream));
        if ((st = stream_write_u32(copy_stream, flags + c, epoch)) != MOE_OK) return st;
    }
    if (ready_out) SWB_CUDA(cudaEventRecord(ready_out, copy_stream));
    return MOE_OK;
}

std::atomic<uint64_t> g_launches{0};
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

}  // namespace swb

using namespace swb;

extern "C" {

const char* moe_status_string(moe_status s) {
    switch (s) {
        case MOE_OK: return "MOE_OK";
        case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
        case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
        case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
        case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
        case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT";
        case MOE_ERR_DEVICE_CHECK: return "MOE_ERR_DEVICE_CHECK";
    }
    return "MOE_ERR_UNKNOWN";
}

const char* moe_last_error(void) { return g_last_error; }

int32_t moe_abi_version(void) { return MOE_ABI_VERSION; }

uint64_t moe_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

void moe_debug_fail_next_cuda_calls(int32_t count) { g_fail_next.store(count > 0 ? count : 0); }
void moe_debug_gated_regs_per_sm(int64_t limit) { g_gated_regs.store(limit > 0 ? limit : 0); }

moe_status moe_expert_layout_get(int32_t H, int32_t I, moe_dtype w_dtype, moe_expert_layout* out) {
    if (!out) return fail(MOE_ERR_INVALID_ARG, "moe_expert_layout_get: out is NULL");
    if (H <= 0 || I <= 0 || H % 128 || I % 128)
        return fail(MOE_ERR_INVALID_ARG, "moe_expert_layout_get: H=%d I=%d must be positive "
                    "multiples of 128", H, I);
    auto up = [](int64_t v) { return (v + 255) / 256 * 256; };
    int64_t es;
    if (w_dtype == MOE_BF16) es = 2;
    else if (w_dtype == MOE_E4M3) es = 1;
    else return fail(MOE_ERR_UNSUPPORTED, "moe_expert_layout_get: weight dtype %d", (int)w_dtype);
    const int64_t gu = 2LL * I * H * es, dn = (int64_t)H * I * es;
    out->gu_offset = 0;
    out->down_offset = up(gu);
    int64_t end = out->down_offset + up(dn);
    out->gu_scale_offset = out->down_scale_offset = -1;
    if (w_dtype == MOE_E4M3) {
        out->gu_scale_offset = end;
        end += up((2LL * I / 128) * (H / 128) * 4);
        out->down_scale_offset = end;
        end += up((int64_t)(H / 128) * (I / 128) * 4);
    }
    out->bytes = end;
    return MOE_OK;
}

moe_status moe_prefetch_layer(const void* src, void* dst, size_t bytes, size_t chunk_bytes,
                              cudaStream_t copy_stream, cudaEvent_t wait_free,
                              cudaEvent_t ready_out) {
    if (bytes > 0 && (!src || !dst))
        return fail(MOE_ERR_INVALID_ARG, "moe_prefetch_layer: NULL buffer");
    if (bytes > 0) {
        const char* s = static_cast<const char*>(src);
        char* d = static_cast<char*>(dst);
        if ((s < d + bytes) && (d < s + bytes))
            return fail(MOE_ERR_INVALID_ARG, "moe_prefetch_layer: source and destination overlap");
    }
    if (wait_free) SWB_CUDA(cudaStreamWaitEvent(copy_stream, wait_free, 0));
    size_t step = chunk_bytes ? chunk_bytes : bytes;
    for (size_t off = 0; off < bytes; off += step) {
        size_t n = bytes - off < step ? bytes - off : step;
        SWB_CUDA(cudaMemcpyAsync(static_cast<char*>(dst) + off,
                                 static_cast<const char*>(src) + off, n,
                                 cudaMemcpyDeviceToDevice, copy_stream));
    }
    if (ready_out) SWB_CUDA(cudaEventRecord(ready_out, copy_stream));
    return MOE_OK;
}

moe_status moe_prefetch_layer_flagged(const void* src, void* dst, size_t bytes, size_t chunk_bytes,
                                      cudaStream_t copy_stream, cudaEvent_t wait_free,
                                      uint32_t* flags, uint32_t epoch, cudaEvent_t ready_out) {
    if (bytes > 0 && (!src || !dst))
        return fail(MOE_ERR_INVALID_ARG, "moe_prefetch_layer_flagged: NULL buffer");
    if (chunk_bytes == 0 || !flags || !aligned(flags, 4))
        return fail(MOE_ERR_INVALID_ARG, "moe_prefetch_layer_flagged: chunk_bytes > 0 and "
                    "4-byte aligned flags needed");
    if (bytes > 0) {
        const char* s = static_cast<const char*>(src);
        char* d = static_cast<char*>(dst);
        if ((s < d + bytes) && (d < s + bytes))
            return fail(MOE_ERR_INVALID_ARG, "moe_prefetch_layer_flagged: source and destination "
                        "overlap");
    }
    return flagged_copy(src, dst, bytes, chunk_bytes, copy_stream, wait_free, flags, epoch, nullptr,
                        0, ready_out);
}

moe_status moe_prefetch_layer_paced(const void* src, void* dst, size_t bytes, size_t chunk_bytes,
                                    cudaStream_t copy_stream, cudaEvent_t wait_free, uint32_t* flags,
                                    uint32_t epoch, const moe_progress* pace, int32_t lead_chunks,
                                    cudaEvent_t ready_out) {
    if (bytes > 0 && (!src || !dst))
        return fail(MOE_ERR_INVALID_ARG, "moe_prefetch_layer_paced: NULL buffer");
    if (chunk_bytes == 0 || !flags || !aligned(flags, 4))
        return fail(MOE_ERR_INVALID_ARG, "moe_prefetch_layer_paced: chunk_bytes > 0 and "
                    "4-byte aligned flags needed");
    if (!pace || !pace->word || !aligned(pace->word, 4) || pace->steps < 1 || lead_chunks < 0)
        return fail(MOE_ERR_INVALID_ARG, "moe_prefetch_layer_paced: a progress word (4-byte "
                    "aligned), steps >= 1 and lead_chunks >= 0 needed");
    if (bytes > 0) {
        const char* s = static_cast<const char*>(src);
        char* d = static_cast<char*>(dst);
        if ((s < d + bytes) && (d < s + bytes))
            return fail(MOE_ERR_INVALID_ARG, "moe_prefetch_layer_paced: source and destination "
                        "overlap");
    }
    return flagged_copy(src, dst, bytes, chunk_bytes, copy_stream, wait_free, flags, epoch, pace,
                        lead_chunks, ready_out);
}

moe_status moe_prefetch_slots(const void* src, void* dst, size_t slot_bytes, int32_t pool_slots,
                              const int32_t* slots, int32_t n, cudaStream_t copy_stream,
                              cudaEvent_t wait_free, uint32_t* flags, uint32_t epoch,
                              cudaEvent_t ready_out) {
    if (n < 0 || pool_slots < 0 || (n > 0 && (!src || !dst || !slots || slot_bytes == 0)) ||
        !flags || !aligned(flags, 4))
        return fail(MOE_ERR_INVALID_ARG, "moe_prefetch_slots: n >= 0, pool_slots >= 0, buffers, "
                    "slots, slot_bytes > 0 and 4-byte aligned flags needed");
    for (int32_t i = 0; i < n; ++i)
        if (slots[i] < 0 || slots[i] >= pool_slots)
            return fail(MOE_ERR_INVALID_ARG, "moe_prefetch_slots: slot %d outside [0, %d)",
                        slots[i], pool_slots);
    if (n > 0) {   // the pool images of src and dst may not overlap
        const size_t span = (size_t)pool_slots * slot_bytes;
        const char* s = static_cast<const char*>(src);
        char* d = static_cast<char*>(dst);
        if ((s < d + span) && (d < s + span))
            return fail(MOE_ERR_INVALID_ARG, "moe_prefetch_slots: source and destination overlap");
    }
    if (wait_free) SWB_CUDA(cudaStreamWaitEvent(copy_stream, wait_free, 0));
    for (int32_t i = 0; i < n;) {   // runs of consecutive slots: one copy each
        int32_t j = i + 1;
        while (j < n && slots[j] == slots[j - 1] + 1) ++j;
        const size_t off = (size_t)slots[i] * slot_bytes;
        SWB_CUDA(cudaMemcpyAsync(static_cast<char*>(dst) + off, static_cast<const char*>(src) + off,
                                 (size_t)(j - i) * slot_bytes, cudaMemcpyDeviceToDevice,
                                 copy_stream));
        for (int32_t q = i; q < j; ++q) {
            const moe_status st = stream_write_u32(copy_stream, flags + slots[q], epoch);
            if (st != MOE_OK) return st;
        }
        i = j;
    }
    if (ready_out) SWB_CUDA(cudaEventRecord(ready_out, copy_stream));
    return MOE_OK;
}

uint32_t moe_pace_threshold(int64_t chunk, int64_t n_chunks, int32_t lead_chunks, uint32_t base,
                            int32_t steps) {
    return swb::pace_threshold(chunk, n_chunks, lead_chunks, base, steps);
}

moe_status moe_wait_ready(cudaEvent_t ev, int32_t timeout_ms) {
    if (!ev) return fail(MOE_ERR_INVALID_ARG, "moe_wait_ready: NULL event");
    const auto t0 = std::chrono::steady_clock::now();
    while (true) {
        if (cuda_injected_failure()) return fail(MOE_ERR_CUDA, "cudaEventQuery: injected failure");
        cudaError_t e = cudaEventQuery(ev);
        if (e == cudaSuccess) return MOE_OK;
        if (e != cudaErrorNotReady) return cuda_check(e, "cudaEventQuery");
        auto ms = std::chrono::duration_cast<std::chrono::milliseconds>(
                      std::chrono::steady_clock::now() - t0).count();
        if (ms >= timeout_ms)
            return fail(MOE_ERR_TIMEOUT, "moe_wait_ready: event not complete after %d ms",
                        (int)timeout_ms);
        std::this_thread::sleep_for(std::chrono::microseconds(100));
    }
}

moe_status moe_check_device(void) {
    int* w = nullptr;
    moe_status st = device_error_word(&w);
    if (st != MOE_OK) return st;
    SWB_CUDA(cudaDeviceSynchronize());
    int v = 0;
    SWB_CUDA(cudaMemcpy(&v, w, sizeof v, cudaMemcpyDeviceToHost));
    if (v) {
        int zero = 0;
        SWB_CUDA(cudaMemcpy(w, &zero, sizeof zero, cudaMemcpyHostToDevice));
        if (v & kDevErrTimeout) return fail(MOE_ERR_TIMEOUT, "a kernel wait ran out (word %d)", v);
        return fail(MOE_ERR_DEVICE_CHECK, "device check failed (word %d)", v);
    }
    return MOE_OK;
}

}  // extern "C"
