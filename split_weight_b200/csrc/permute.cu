// moe_permute: expert histogram, scan, stable scatter and row gather.
//
// Groups every rank's token-expert assignments by expert so that one grouped
// GEMM serves all of them (explainer "Distributed Weight Data Parallelism
// cuts LLM inference stalls", split-weight figure: one grouped GEMM over the
// local and remote experts).  The order is the stable counting sort of the
// assignments a = t*k + j by expert: one unique answer, reproduced exactly.
//
// Three small integer kernels (per-block histogram, one-block scan,
// per-block stable scatter with warp match/popc ranks) and one bandwidth
// kernel that copies x rows into expert order with 128-bit accesses.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include <mutex>

#include "device.cuh"
#include "internal.h"

namespace swb {
namespace {

constexpr int kItemsPerThread = 8;
constexpr int kThreads = 256;
constexpr int kPB = kItemsPerThread * kThreads;  // assignments per block

__device__ __forceinline__ int load_expert(const int32_t* idx, int64_t a, int64_t A, int E,
                                           int* err) {
    if (a >= A) return -1;
    const int e = idx[a];
    if (e < 0 || e >= E) {
        atomicOr(err, kDevErrIndex);
        return -1;
    }
    return e;
}

__global__ void __launch_bounds__(kThreads) k_hist(const int32_t* __restrict__ idx, int64_t A,
                                                   int E, int32_t* __restrict__ blk_counts,
                                                   int* err) {
    extern __shared__ int cnt[];
    for (int e = threadIdx.x; e < E; e += kThreads) cnt[e] = 0;
    __syncthreads();
    const int64_t base = (int64_t)blockIdx.x * kPB;
    for (int i = 0; i < kItemsPerThread; ++i) {
        const int e = load_expert(idx, base + i * kThreads + threadIdx.x, A, E, err);
        if (e >= 0) atomicAdd(&cnt[e], 1);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += kThreads)
        blk_counts[(int64_t)blockIdx.x * E + e] = cnt[e];
}

// touched[e] = 1 for every expert some assignment selects (entries outside
// [0, E) are reported and skipped, as in k_hist); the caller zeroed touched.
__global__ void k_touched(const int32_t* __restrict__ idx, int64_t A, int E,
                          uint8_t* __restrict__ touched, int* err) {
    for (int64_t a = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; a < A;
         a += (int64_t)gridDim.x * blockDim.x) {
        const int e = load_expert(idx, a, A, E, err);
        if (e >= 0) touched[e] = 1;
    }
}

// One block of 1024 threads: offsets[] and each block's first row per expert.
__global__ void __launch_bounds__(1024) k_scan(const int32_t* __restrict__ blk_counts, int nb,
                                               int E, int32_t* __restrict__ blk_base,
                                               int32_t* __restrict__ offsets) {
    __shared__ int warp_sums[32];
    const int e = threadIdx.x;
    int run = 0;
    if (e < E) {
        for (int b = 0; b < nb; ++b) {
            const int c = blk_counts[(int64_t)b * E + e];
            blk_base[(int64_t)b * E + e] = run;
            run += c;
        }
    }
    // exclusive scan of run over e (1024 threads)
    const int lane = e & 31, warp = e >> 5;
    int v = (e < E) ? run : 0, incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int s = warp_sums[lane], si = s;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, si, o);
            if (lane >= o) si += n;
        }
        warp_sums[lane] = si - s;  // exclusive
    }
    __syncthreads();
    const int excl = warp_sums[warp] + incl - v;
    if (e < E) {
        offsets[e] = excl;
        if (e == E - 1) offsets[E] = excl + v;
        for (int b = 0; b < nb; ++b) blk_base[(int64_t)b * E + e] += excl;
    }
}

// Stable scatter.  The block's assignments are taken in 8 rounds of 256, in
// order; inside a round warp w holds the 32 assignments 32w..32w+31.  A
// thread's row = (rows of its expert before this round) + (rows of its
// expert in earlier warps of the round) + (its rank among equal experts of
// its warp).
__global__ void __launch_bounds__(kThreads) k_scatter(const int32_t* __restrict__ idx, int64_t A,
                                                      int k, int E,
                                                      const int32_t* __restrict__ blk_base,
                                                      int32_t* __restrict__ perm_src,
                                                      int32_t* __restrict__ inv_pos, int* err) {
    extern __shared__ int sm[];
    int* run = sm;               // [E]
    int* wcnt = sm + E;          // [8][E]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int e = threadIdx.x; e < E; e += kThreads) {
        run[e] = blk_base[(int64_t)blockIdx.x * E + e];
        for (int w = 0; w < 8; ++w) wcnt[w * E + e] = 0;
    }
    __syncthreads();
    const int64_t base = (int64_t)blockIdx.x * kPB;
    const uint32_t lt = (1u << lane) - 1u;
    for (int r = 0; r < kItemsPerThread; ++r) {
        const int64_t a = base + r * kThreads + threadIdx.x;
        const int e = load_expert(idx, a, A, E, err);
        const uint32_t peers = __match_any_sync(0xffffffffu, e);
        const int rank = __popc(peers & lt);
        const bool leader = (peers & lt) == 0;
        if (e >= 0 && leader) wcnt[warp * E + e] = __popc(peers);
        __syncthreads();
        if (e >= 0) {
            int pos = run[e] + rank;
            for (int w = 0; w < warp; ++w) pos += wcnt[w * E + e];
            perm_src[pos] = static_cast<int32_t>(a / k);
            inv_pos[a] = pos;
        } else if (a < A) {
            inv_pos[a] = -1;  // skipped (reported): the combine sees no row
        }
        __syncthreads();
        if (e >= 0 && leader) {
            atomicAdd(&run[e], __popc(peers));
            wcnt[warp * E + e] = 0;
        }
        __syncthreads();
    }
}

// Eight consecutive fp32 values as two 16-byte loads.
__device__ __forceinline__ void load8(const float* row, int c, float (&v)[8]) {
    const float4 a = *reinterpret_cast<const float4*>(row + c);
    const float4 b = *reinterpret_cast<const float4*>(row + c + 4);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// Source token of permuted row r, or -1 when it is not a token of x.  Rows
// r < A come from perm_src; when an expert index was skipped (out of range)
// the rows past the last scattered one were never written, so the value is
// checked before it addresses x.
__device__ __forceinline__ int64_t gather_source(const int32_t* perm_src, int64_t r, int64_t A,
                                                 int64_t T, int* err) {
    if (r >= A) return r - A;
    const int64_t src = perm_src[r];
    if (src < 0 || src >= T) {
        if ((threadIdx.x & 31) == 0) atomicOr(err, kDevErrIndex);
        return -1;
    }
    return src;
}

// One warp per output row; 8 columns (one 16-byte bf16 vector) per lane step.
template <typename XT>
__global__ void __launch_bounds__(256) k_gather_bf16(const XT* __restrict__ x,
                                                     const int32_t* __restrict__ perm_src,
                                                     int64_t A, int64_t T, int64_t rows, int H,
                                                     __nv_bfloat16* __restrict__ out, int* err) {
    const int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (r >= rows) return;
    const int lane = threadIdx.x & 31;
    const int64_t src = gather_source(perm_src, r, A, T, err);
    __nv_bfloat16* o = out + r * H;
    if (src < 0) {  // reported above: the row is zero-filled
        for (int c = lane * 8; c < H; c += 256) *reinterpret_cast<uint4*>(o + c) = make_uint4(0, 0, 0, 0);
        return;
    }
    const XT* in = x + src * H;
    for (int c = lane * 8; c < H; c += 256) {
        if constexpr (sizeof(XT) == 2) {
            *reinterpret_cast<uint4*>(o + c) = *reinterpret_cast<const uint4*>(in + c);
        } else {
            float v[8];
            load8(in, c, v);
            uint4 u;
            __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
            for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
            *reinterpret_cast<uint4*>(o + c) = u;
        }
    }
}

// Eight consecutive values of a bf16 or fp32 row as fp32: one or two 16-byte loads.
__device__ __forceinline__ void load8(const __nv_bfloat16* row, int c, float (&v)[8]) {
    const uint4 u = *reinterpret_cast<const uint4*>(row + c);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(h[i]);
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
    }
}

// One warp per output row, two 128-column blocks per step: lanes 0-15 hold
// block b and lanes 16-31 block b + 1, 8 columns per lane (16-byte loads,
// 8-byte stores).  Per block: s = amax / 448, code = e4m3(v / s).
template <typename XT>
__global__ void __launch_bounds__(256) k_gather_e4m3(const XT* __restrict__ x,
                                                     const int32_t* __restrict__ perm_src,
                                                     int64_t A, int64_t T, int64_t rows, int H,
                                                     uint8_t* __restrict__ out,
                                                     float* __restrict__ scales, int* err) {
    const int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (r >= rows) return;
    const int lane = threadIdx.x & 31;
    const int64_t src = gather_source(perm_src, r, A, T, err);
    const XT* in = x + (src < 0 ? 0 : src) * H;
    const int nblk = H / 128;
    for (int b0 = 0; b0 < nblk; b0 += 2) {
        const int b = b0 + (lane >> 4);
        const bool act = b < nblk;
        const int c = b * 128 + (lane & 15) * 8;
        float v[8];
        if (act && src >= 0) {
            load8(in, c, v);
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) v[i] = 0.0f;
        }
        float m = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(v[i]));
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        const float s = (m > 0.0f) ? m / 448.0f : 1.0f;
        uint32_t packed[2] = {0u, 0u};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float q = fminf(fmaxf(v[i] / s, -448.0f), 448.0f);
            packed[i >> 2] |= (uint32_t)__nv_cvt_float_to_fp8(q, __NV_SATFINITE, __NV_E4M3) << (8 * (i & 3));
        }
        if (act) {
            *reinterpret_cast<uint2*>(out + r * H + c) = make_uint2(packed[0], packed[1]);
            if ((lane & 15) == 0) scales[(int64_t)b * rows + r] = s;  // [H/128][rows]
        }
    }
}

int64_t num_blocks(int64_t A) { return (A + kPB - 1) / kPB; }

}  // namespace
}  // namespace swb

using namespace swb;

extern "C" {

size_t moe_permute_workspace_size(int32_t T, int32_t k, int32_t E) {
    if (T < 0 || k <= 0 || E <= 0) return 0;
    const int64_t nb = num_blocks((int64_t)T * k);
    return (size_t)(2 * nb * E) * sizeof(int32_t);
}

moe_status moe_experts_touched(const int32_t* topk_idx, int64_t A, int32_t E, uint8_t* touched,
                               cudaStream_t stream) {
    if (A < 0 || E <= 0 || E > MOE_MAX_EXPERTS || !touched || (A > 0 && !topk_idx))
        return fail(MOE_ERR_INVALID_ARG, "moe_experts_touched: A=%lld E=%d, touched and topk_idx "
                    "needed", (long long)A, E);
    int* err = nullptr;
    moe_status st = device_error_word(&err);
    if (st != MOE_OK) return st;
    SWB_CUDA(cudaMemsetAsync(touched, 0, (size_t)E, stream));
    if (A == 0) return MOE_OK;
    int sms = 0;
    if ((st = sm_count(&sms)) != MOE_OK) return st;
    const int64_t want = (A + 255) / 256;
    const unsigned g = (unsigned)(want < 4 * sms ? want : 4 * sms);
    k_touched<<<g, 256, 0, stream>>>(topk_idx, A, E, touched, err);
    SWB_LAUNCHED("moe_experts_touched");
    return MOE_OK;
}

}  // extern "C"

namespace swb {
namespace {

// Host-side checks shared by moe_permute and moe_permute_noalloc: everything
// but the workspace, before anything is enqueued or any CUDA call is made.
moe_status permute_check_args(int32_t T, int32_t k, int32_t E, int32_t H, const int32_t* topk_idx,
                              const void* x, moe_dtype x_dtype, moe_dtype perm_dtype,
                              int32_t* offsets, int32_t* perm_src, int32_t* inv_pos, void* x_perm,
                              float* x_perm_scales) {
    if (T < 0 || k <= 0 || k > MOE_MAX_TOPK || E <= 0 || E > MOE_MAX_EXPERTS || H <= 0 ||
        H % 128)
        return fail(MOE_ERR_INVALID_ARG, "moe_permute: T=%d k=%d E=%d H=%d", T, k, E, H);
    if (x_dtype != MOE_F32 && x_dtype != MOE_BF16)
        return fail(MOE_ERR_UNSUPPORTED, "moe_permute: x dtype %d", (int)x_dtype);
    if (perm_dtype != MOE_BF16 && perm_dtype != MOE_E4M3)
        return fail(MOE_ERR_UNSUPPORTED, "moe_permute: x_perm dtype %d", (int)perm_dtype);
    if (!offsets) return fail(MOE_ERR_INVALID_ARG, "moe_permute: offsets is NULL");
    if ((int64_t)T * k + T > INT32_MAX) return fail(MOE_ERR_UNSUPPORTED, "moe_permute: too many rows");
    if (T > 0 && (!topk_idx || !x || !perm_src || !inv_pos))
        return fail(MOE_ERR_INVALID_ARG, "moe_permute: NULL pointer");
    if (perm_dtype == MOE_E4M3 && T > 0 && x_perm && !x_perm_scales)
        return fail(MOE_ERR_INVALID_ARG, "moe_permute: e4m3 x_perm needs x_perm_scales");
    if (!aligned(topk_idx, 16) || !aligned(x, 16) || !aligned(offsets, 16) ||
        !aligned(perm_src, 16) || !aligned(inv_pos, 16) || !aligned(x_perm, 16) ||
        !aligned(x_perm_scales, 16))
        return fail(MOE_ERR_INVALID_ARG, "moe_permute: pointers must be 16-byte aligned");
    return MOE_OK;
}

}  // namespace
}  // namespace swb

extern "C" {

moe_status moe_permute(int32_t T, int32_t k, int32_t E, int32_t H, const int32_t* topk_idx,
                       const void* x, moe_dtype x_dtype, moe_dtype perm_dtype, int32_t with_shared,
                       int32_t* offsets, int32_t* perm_src, int32_t* inv_pos, void* x_perm,
                       float* x_perm_scales, void* workspace, size_t workspace_bytes,
                       cudaStream_t stream) {
    moe_status st = permute_check_args(T, k, E, H, topk_idx, x, x_dtype, perm_dtype, offsets,
                                       perm_src, inv_pos, x_perm, x_perm_scales);
    if (st != MOE_OK) return st;
    const int64_t A = (int64_t)T * k;
    const int64_t rows = A + (with_shared ? T : 0);
    const size_t need = moe_permute_workspace_size(T, k, E);
    if (workspace_bytes < need || (need && !workspace))
        return fail(MOE_ERR_WORKSPACE, "moe_permute: workspace %zu < %zu bytes",
                    workspace_bytes, need);
    int* err = nullptr;
    st = device_error_word(&err);
    if (st != MOE_OK) return st;
    const int64_t nb = num_blocks(A);
    int32_t* blk_counts = static_cast<int32_t*>(workspace);
    int32_t* blk_base = blk_counts + nb * E;
    if (A == 0) {
        SWB_CUDA(cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (E + 1), stream));
    } else {
        k_hist<<<(unsigned)nb, kThreads, E * sizeof(int), stream>>>(topk_idx, A, E, blk_counts,
                                                                     err);
        SWB_LAUNCHED("moe_permute: histogram kernel");
        k_scan<<<1, 1024, 0, stream>>>(blk_counts, (int)nb, E, blk_base, offsets);
        SWB_LAUNCHED("moe_permute: scan kernel");
        k_scatter<<<(unsigned)nb, kThreads, 9 * E * sizeof(int), stream>>>(
            topk_idx, A, k, E, blk_base, perm_src, inv_pos, err);
        SWB_LAUNCHED("moe_permute: scatter kernel");
    }
    if (x_perm && rows > 0) {
        const unsigned g = (unsigned)((rows + 7) / 8);
        if (perm_dtype == MOE_BF16) {
            if (x_dtype == MOE_BF16)
                k_gather_bf16<<<g, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(x),
                                                     perm_src, A, T, rows, H,
                                                     static_cast<__nv_bfloat16*>(x_perm), err);
            else
                k_gather_bf16<<<g, 256, 0, stream>>>(static_cast<const float*>(x), perm_src, A,
                                                     T, rows, H,
                                                     static_cast<__nv_bfloat16*>(x_perm), err);
        } else {
            if (x_dtype == MOE_BF16)
                k_gather_e4m3<<<g, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(x),
                                                     perm_src, A, T, rows, H,
                                                     static_cast<uint8_t*>(x_perm), x_perm_scales,
                                                     err);
            else
                k_gather_e4m3<<<g, 256, 0, stream>>>(static_cast<const float*>(x), perm_src, A,
                                                     T, rows, H, static_cast<uint8_t*>(x_perm),
                                                     x_perm_scales, err);
        }
        SWB_LAUNCHED("moe_permute: gather kernel");
    }
    return MOE_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free variant of moe_permute.
//
// For callers that cannot allocate device memory at all, not even a
// workspace of their own: for example a plug-in running inside a host
// application or serving runtime that has reserved all device memory for its
// own pool and forbids any other allocation, or code on a latency-critical
// path where a cudaMalloc (which may synchronise the whole device) is not
// allowed.  The scratch that moe_permute takes as `workspace` (per-block
// expert counts and bases) lives instead in a fixed array in this library's
// device memory.  The array belongs to this file's device code module: it is
// placed on a device when that module is loaded there (with CUDA's default
// lazy loading, at the first kernel launch or symbol lookup of this file on
// that device) and stays until the process exits.
// ---------------------------------------------------------------------------
namespace swb {
namespace {

constexpr size_t kPermuteScratchBytes = size_t(1) << 20;  // 1 MiB per device
static __device__ __align__(256) unsigned char g_permute_scratch[kPermuteScratchBytes];

std::mutex g_scratch_mu;
constexpr int kMaxScratchDevices = 64;
void* g_scratch_addr[kMaxScratchDevices] = {nullptr};

// Device address of g_permute_scratch on the current device.  In host code
// the array's name is only a host-side stand-in, so the address is looked up
// once per device with cudaGetSymbolAddress (this is done by the first call
// on each device) and cached.
moe_status permute_scratch_address(void** out) {
    int dev = 0;
    SWB_CUDA(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kMaxScratchDevices)
        return fail(MOE_ERR_UNSUPPORTED, "moe_permute_noalloc: device %d", dev);
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        if (cuda_injected_failure())
            return fail(MOE_ERR_CUDA, "cudaGetSymbolAddress: injected failure");
        const cudaError_t e = cudaGetSymbolAddress(&p, g_permute_scratch);
        if (e != cudaSuccess) return cuda_check(e, "cudaGetSymbolAddress(permute scratch)");
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return MOE_OK;
}

}  // namespace
}  // namespace swb

extern "C" {

moe_status moe_permute_noalloc(int32_t T, int32_t k, int32_t E, int32_t H,
                               const int32_t* topk_idx, const void* x, moe_dtype x_dtype,
                               moe_dtype perm_dtype, int32_t with_shared, int32_t* offsets,
                               int32_t* perm_src, int32_t* inv_pos, void* x_perm,
                               float* x_perm_scales, cudaStream_t stream) {
    moe_status st = permute_check_args(T, k, E, H, topk_idx, x, x_dtype, perm_dtype, offsets,
                                       perm_src, inv_pos, x_perm, x_perm_scales);
    if (st != MOE_OK) return st;
    const size_t need = moe_permute_workspace_size(T, k, E);
    if (need > kPermuteScratchBytes)
        return fail(MOE_ERR_WORKSPACE,
                    "moe_permute_noalloc: T=%d k=%d E=%d needs %zu bytes of scratch, more than "
                    "the built-in %zu bytes (use moe_permute with a workspace)",
                    T, k, E, need, kPermuteScratchBytes);
    void* scratch = nullptr;
    st = permute_scratch_address(&scratch);
    if (st != MOE_OK) return st;
    // Every scratch word the kernels read is written earlier in the same
    // call (block counts, then bases), so nothing needs clearing first.
    return moe_permute(T, k, E, H, topk_idx, x, x_dtype, perm_dtype, with_shared, offsets,
                       perm_src, inv_pos, x_perm, x_perm_scales, scratch, kPermuteScratchBytes,
                       stream);
}

}  // extern "C"
