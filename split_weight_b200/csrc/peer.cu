// Peer fetch of a rank's missing experts in a DWDP group.
//
// The explainer "Distributed Weight Data Parallelism cuts LLM inference
// stalls" has each rank pull the expert weights it lacks straight from a
// peer's memory with cudaMemcpyAsync over NVLink, on the copy engine
// (fetch-path caption), and notes that several destinations can converge on
// one source mid-pull; time-division multiplexed slicing across destinations
// removes that (contention caption).
//
// Here every source pool is cut into pieces, and step j of rank r copies a
// piece of source (r + 1 + j mod (G-1)) mod G.  The offset j mod (G-1) + 1 is
// the same on every rank at step j, so the ranks' sources form a rotation of
// the group with no fixed point: at each step every source serves exactly one
// destination.  The copies are plain cudaMemcpyAsync calls on the caller's
// copy stream (copy engine, no SM work, no kernel ever reads a peer's memory).
//
// Peer memory reaches this process either through peer access between
// devices of one process (moe_enable_peer_access) or through CUDA IPC between
// processes (moe_pool_export / moe_pool_import).
#include <cstring>
#include <mutex>
#include <vector>

#include "internal.h"

namespace swb {
namespace {

constexpr int kMaxGroup = 64;

using GetAddressRangeFn = CUresult (*)(CUdeviceptr*, size_t*, CUdeviceptr);
std::mutex g_peer_mu;
GetAddressRangeFn g_range = nullptr;

moe_status address_range(const void* p, CUdeviceptr* base, size_t* size) {
    {
        std::lock_guard<std::mutex> lk(g_peer_mu);
        if (!g_range) {
            void* fn = nullptr;
            cudaDriverEntryPointQueryResult q;
            if (cuda_injected_failure())
                return fail(MOE_ERR_CUDA, "cudaGetDriverEntryPoint: injected failure");
            cudaError_t e = cudaGetDriverEntryPoint("cuMemGetAddressRange", &fn, cudaEnableDefault, &q);
            if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn)
                return fail(MOE_ERR_CUDA, "cuMemGetAddressRange entry point unavailable");
            g_range = reinterpret_cast<GetAddressRangeFn>(fn);
        }
    }
    const CUresult r = g_range(base, size, reinterpret_cast<CUdeviceptr>(p));
    if (r != CUDA_SUCCESS)
        return fail(MOE_ERR_INVALID_ARG, "cuMemGetAddressRange failed (CUresult %d)", (int)r);
    return MOE_OK;
}

}  // namespace
}  // namespace swb

using namespace swb;

extern "C" {

moe_status moe_peer_fetch_plan(int32_t group_size, int32_t rank, int64_t bytes_per_rank,
                               int32_t slices, moe_peer_copy* plan, int32_t plan_capacity,
                               int32_t* plan_len) {
    if (group_size < 2 || group_size > kMaxGroup || rank < 0 || rank >= group_size)
        return fail(MOE_ERR_INVALID_ARG, "moe_peer_fetch_plan: group %d, rank %d", group_size, rank);
    if (bytes_per_rank <= 0 || bytes_per_rank % 256 || slices < 1)
        return fail(MOE_ERR_INVALID_ARG, "moe_peer_fetch_plan: %lld bytes per rank (a positive "
                    "multiple of 256), %d slices", (long long)bytes_per_rank, slices);
    if (!plan_len) return fail(MOE_ERR_INVALID_ARG, "moe_peer_fetch_plan: plan_len is NULL");
    // pieces of a source pool: 256-byte multiples, the last one takes the rest
    const int64_t units = bytes_per_rank / 256;
    const int32_t pieces = (int32_t)(units < slices ? units : slices);
    const int32_t n = (group_size - 1) * pieces;
    *plan_len = n;
    if (!plan) return MOE_OK;   // size query
    if (plan_capacity < n)
        return fail(MOE_ERR_INVALID_ARG, "moe_peer_fetch_plan: capacity %d < %d entries",
                    plan_capacity, n);
    const int64_t piece = units / pieces * 256;
    for (int32_t j = 0; j < n; ++j) {
        const int32_t c = j % (group_size - 1), i = j / (group_size - 1);
        const int32_t s = (rank + 1 + c) % group_size;
        const int32_t pos = s < rank ? s : s - 1;          // place of s in the remote buffer
        const int64_t off = (int64_t)i * piece;
        moe_peer_copy& e = plan[j];
        e.step = j;
        e.src_rank = s;
        e.src_offset = off;
        e.dst_offset = (int64_t)pos * bytes_per_rank + off;
        e.bytes = (i == pieces - 1) ? bytes_per_rank - off : piece;
    }
    return MOE_OK;
}

moe_status moe_prefetch_peers(int32_t group_size, int32_t rank, const void* const* src_pools,
                              int64_t bytes_per_rank, int32_t slices, void* dst,
                              cudaStream_t copy_stream, cudaEvent_t wait_free,
                              cudaEvent_t ready_out) {
    int32_t n = 0;
    moe_status st = moe_peer_fetch_plan(group_size, rank, bytes_per_rank, slices, nullptr, 0, &n);
    if (st != MOE_OK) return st;
    if (!src_pools || !dst) return fail(MOE_ERR_INVALID_ARG, "moe_prefetch_peers: NULL pointer");
    if (!aligned(dst, 256)) return fail(MOE_ERR_INVALID_ARG, "moe_prefetch_peers: dst not 256-byte aligned");
    const char* d = static_cast<const char*>(dst);
    const int64_t dst_bytes = (int64_t)(group_size - 1) * bytes_per_rank;
    for (int32_t s = 0; s < group_size; ++s) {
        if (s == rank) continue;
        const char* p = static_cast<const char*>(src_pools[s]);
        if (!p || !aligned(p, 256))
            return fail(MOE_ERR_INVALID_ARG, "moe_prefetch_peers: pool of rank %d missing or not "
                        "256-byte aligned", s);
        if (p < d + dst_bytes && d < p + bytes_per_rank)
            return fail(MOE_ERR_INVALID_ARG, "moe_prefetch_peers: pool of rank %d overlaps dst", s);
    }
    std::vector<moe_peer_copy> plan((size_t)n);   // host memory only
    moe_peer_copy* pl = plan.data();
    st = moe_peer_fetch_plan(group_size, rank, bytes_per_rank, slices, pl, n, &n);
    if (st == MOE_OK && wait_free) {
        if (cuda_injected_failure()) st = fail(MOE_ERR_CUDA, "cudaStreamWaitEvent: injected failure");
        else if (cudaError_t e = cudaStreamWaitEvent(copy_stream, wait_free, 0); e != cudaSuccess)
            st = cuda_check(e, "cudaStreamWaitEvent");
    }
    for (int32_t j = 0; st == MOE_OK && j < n; ++j) {
        const moe_peer_copy& e = pl[j];
        const char* src = static_cast<const char*>(src_pools[e.src_rank]) + e.src_offset;
        if (cuda_injected_failure()) {
            st = fail(MOE_ERR_CUDA, "cudaMemcpyAsync: injected failure");
        } else if (cudaError_t ce = cudaMemcpyAsync(static_cast<char*>(dst) + e.dst_offset, src,
                                                    (size_t)e.bytes, cudaMemcpyDefault, copy_stream);
                   ce != cudaSuccess) {
            st = cuda_check(ce, "cudaMemcpyAsync (peer piece)");
        }
    }
    if (st != MOE_OK) return st;
    if (ready_out) SWB_CUDA(cudaEventRecord(ready_out, copy_stream));
    return MOE_OK;
}

moe_status moe_enable_peer_access(int32_t peer_device) {
    int dev = 0, can = 0;
    SWB_CUDA(cudaGetDevice(&dev));
    if (peer_device == dev) return MOE_OK;
    SWB_CUDA(cudaDeviceCanAccessPeer(&can, dev, peer_device));
    if (!can)
        return fail(MOE_ERR_UNSUPPORTED, "moe_enable_peer_access: device %d cannot access device %d",
                    dev, peer_device);
    if (cuda_injected_failure()) return fail(MOE_ERR_CUDA, "cudaDeviceEnablePeerAccess: injected failure");
    const cudaError_t e = cudaDeviceEnablePeerAccess(peer_device, 0);
    if (e == cudaErrorPeerAccessAlreadyEnabled) {
        (void)cudaGetLastError();
        return MOE_OK;
    }
    if (e != cudaSuccess) return cuda_check(e, "cudaDeviceEnablePeerAccess");
    return MOE_OK;
}

moe_status moe_pool_export(const void* base, moe_pool_handle* out) {
    if (!base || !out) return fail(MOE_ERR_INVALID_ARG, "moe_pool_export: NULL pointer");
    static_assert(sizeof(cudaIpcMemHandle_t) <= sizeof(out->ipc), "IPC handle size");
    CUdeviceptr alloc = 0;
    size_t size = 0;
    moe_status st = address_range(base, &alloc, &size);
    if (st != MOE_OK) return st;
    cudaIpcMemHandle_t h;
    SWB_CUDA(cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(alloc)));
    memset(out, 0, sizeof *out);
    memcpy(out->ipc, &h, sizeof h);
    out->offset = (int64_t)(reinterpret_cast<CUdeviceptr>(base) - alloc);
    return MOE_OK;
}

moe_status moe_pool_import(const moe_pool_handle* h, void** base_out, void** mapping_out) {
    if (!h || !base_out || !mapping_out) return fail(MOE_ERR_INVALID_ARG, "moe_pool_import: NULL pointer");
    if (h->offset < 0) return fail(MOE_ERR_INVALID_ARG, "moe_pool_import: negative offset");
    cudaIpcMemHandle_t ih;
    memcpy(&ih, h->ipc, sizeof ih);
    void* p = nullptr;
    SWB_CUDA(cudaIpcOpenMemHandle(&p, ih, cudaIpcMemLazyEnablePeerAccess));
    *mapping_out = p;
    *base_out = static_cast<char*>(p) + h->offset;
    return MOE_OK;
}

moe_status moe_pool_close(void* mapping) {
    if (!mapping) return fail(MOE_ERR_INVALID_ARG, "moe_pool_close: NULL mapping");
    SWB_CUDA(cudaIpcCloseMemHandle(mapping));
    return MOE_OK;
}

}  // extern "C"
