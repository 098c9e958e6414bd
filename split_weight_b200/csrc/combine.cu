// moe_combine: the weighted unpermute that closes the MoE block.
//
//   y[t] = sum_{j ascending} w[t,j] * y_perm[inv_pos[t,j]] + y_perm[T*k + t]
//
// Deterministic (no atomics): each 16-byte column slice of a token row is
// owned by one thread, which reads the k + 1 source rows with 128-bit loads
// and accumulates in fp32.  Bandwidth bound: (k + 1) reads, one write.
#include <cuda_bf16.h>

#include "device.cuh"
#include "internal.h"

namespace swb {
namespace {

__device__ __forceinline__ void add_row(const __nv_bfloat16* row, int c, float w, float (&acc)[8]) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(row + c));
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(h[i]);
        acc[2 * i] = fmaf(w, f.x, acc[2 * i]);
        acc[2 * i + 1] = fmaf(w, f.y, acc[2 * i + 1]);
    }
}

// grid.x = tokens, grid.y = column slices of 8 * blockDim.x columns
template <bool OUT_BF16>
__global__ void __launch_bounds__(128) k_combine(const __nv_bfloat16* __restrict__ y_perm,
                                                 const int32_t* __restrict__ inv_pos,
                                                 const float* __restrict__ topk_w, int T, int k,
                                                 int H, int with_shared, void* __restrict__ y,
                                                 int* err) {
    __shared__ int rows[MOE_MAX_TOPK];
    __shared__ float ws[MOE_MAX_TOPK];
    const int t = blockIdx.x;
    if (threadIdx.x < k) {
        int r = inv_pos[(int64_t)t * k + threadIdx.x];
        float w = topk_w[(int64_t)t * k + threadIdx.x];
        if (r < 0 || r >= T * k) {  // not a row of y_perm: report and skip
            if (blockIdx.y == 0) atomicOr(err, kDevErrIndex);
            r = 0;
            w = 0.0f;
        }
        rows[threadIdx.x] = r;
        ws[threadIdx.x] = w;
    }
    __syncthreads();
    const int c = (blockIdx.y * blockDim.x + threadIdx.x) * 8;
    if (c >= H) return;
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
    for (int j = 0; j < k; ++j) add_row(y_perm + (int64_t)rows[j] * H, c, ws[j], acc);
    if (with_shared) add_row(y_perm + ((int64_t)T * k + t) * H, c, 1.0f, acc);
    if constexpr (OUT_BF16) {
        uint4 u;
        __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
        for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
        *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(y) + (int64_t)t * H + c) = u;
    } else {
        float* o = static_cast<float*>(y) + (int64_t)t * H + c;
        *reinterpret_cast<float4*>(o) = make_float4(acc[0], acc[1], acc[2], acc[3]);
        *reinterpret_cast<float4*>(o + 4) = make_float4(acc[4], acc[5], acc[6], acc[7]);
    }
}

}  // namespace
}  // namespace swb

using namespace swb;

extern "C" {

moe_status moe_combine(int32_t T, int32_t k, int32_t H, const void* y_perm, const int32_t* inv_pos,
                       const float* topk_w, int32_t with_shared, void* y, moe_dtype y_dtype,
                       cudaStream_t stream) {
    if (T < 0 || k <= 0 || k > MOE_MAX_TOPK || H <= 0 || H % 8)
        return fail(MOE_ERR_INVALID_ARG, "moe_combine: T=%d k=%d H=%d", T, k, H);
    if (y_dtype != MOE_F32 && y_dtype != MOE_BF16)
        return fail(MOE_ERR_UNSUPPORTED, "moe_combine: y dtype %d", (int)y_dtype);
    if (T == 0) return MOE_OK;
    if (!y_perm || !inv_pos || !topk_w || !y)
        return fail(MOE_ERR_INVALID_ARG, "moe_combine: NULL pointer");
    if (!aligned(y_perm, 16) || !aligned(inv_pos, 16) || !aligned(topk_w, 16) || !aligned(y, 16))
        return fail(MOE_ERR_INVALID_ARG, "moe_combine: pointers must be 16-byte aligned");
    if ((int64_t)T * k > INT32_MAX) return fail(MOE_ERR_UNSUPPORTED, "moe_combine: too many rows");
    int* err = nullptr;
    moe_status st = device_error_word(&err);
    if (st != MOE_OK) return st;
    const int threads = 128;
    dim3 grid(T, (H / 8 + threads - 1) / threads);
    const __nv_bfloat16* yp = static_cast<const __nv_bfloat16*>(y_perm);
    if (y_dtype == MOE_BF16)
        k_combine<true><<<grid, threads, 0, stream>>>(yp, inv_pos, topk_w, T, k, H, with_shared, y, err);
    else
        k_combine<false><<<grid, threads, 0, stream>>>(yp, inv_pos, topk_w, T, k, H, with_shared, y, err);
    SWB_LAUNCHED("moe_combine");
    return MOE_OK;
}

}  // extern "C"
