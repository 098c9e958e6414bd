// Device-side seeded generator for the synthetic expert weights.
//
// Fills expert weight tensors directly in GPU memory so that the 22-45 GB of
// weights of the DeepSeek-R1-shaped workloads take milliseconds to create.
// It implements the same published definitions as philox_cpu.c, with every
// floating-point step an explicit single IEEE rounding, so both produce the
// same bits for the same (key, element index):
//
//   Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as
//   easy as 1, 2, 3", SC'11, section 3.1), counter (lo32(i), hi32(i), 0, 0);
//   the eight 16-bit halves of the output block summed, centred (262140) and
//   scaled by 1/sqrt(8*(65536^2-1)/12) in fp64, then by sigma, then rounded
//   to fp32 and on to bf16 (RNE) or quantised per 128x128 block to e4m3.
//
// Input generation only: it holds none of the MoE layer's arithmetic.
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <math.h>

namespace {

__device__ __forceinline__ void philox_10(uint32_t c[4], uint32_t k0, uint32_t k1) {
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        if (r > 0) {
            k0 += 0x9E3779B9u;
            k1 += 0xBB67AE85u;
        }
        uint32_t lo0 = 0xD2511F53u * c[0];
        uint32_t hi0 = __umulhi(0xD2511F53u, c[0]);
        uint32_t lo1 = 0xCD9E8D57u * c[2];
        uint32_t hi1 = __umulhi(0xCD9E8D57u, c[2]);
        uint32_t n0 = hi1 ^ c[1] ^ k0;
        uint32_t n2 = hi0 ^ c[3] ^ k1;
        c[0] = n0;
        c[1] = lo1;
        c[2] = n2;
        c[3] = lo0;
    }
}

__device__ __forceinline__ float value_f32(uint64_t i, uint32_t k0, uint32_t k1, double c8,
                                           double sigma) {
    uint32_t c[4] = {(uint32_t)i, (uint32_t)(i >> 32), 0u, 0u};
    philox_10(c, k0, k1);
    long long s = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) s += (long long)(c[j] & 0xFFFFu) + (long long)(c[j] >> 16);
    double z = __dmul_rn((double)(s - 262140), c8);
    return __double2float_rn(__dmul_rn(z, sigma));
}

__global__ void k_philox(const uint32_t* in, uint32_t k0, uint32_t k1, uint32_t* out) {
    uint32_t c[4] = {in[0], in[1], in[2], in[3]};
    philox_10(c, k0, k1);
    for (int j = 0; j < 4; ++j) out[j] = c[j];
}

__global__ void k_normal_f32(float* out, int64_t n, uint32_t k0, uint32_t k1, double c8,
                             double sigma) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x)
        out[i] = value_f32((uint64_t)i, k0, k1, c8, sigma);
}

__global__ void k_normal_bf16(__nv_bfloat16* out, int64_t n, uint32_t k0, uint32_t k1, double c8,
                              double sigma) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x)
        out[i] = __float2bfloat16_rn(value_f32((uint64_t)i, k0, k1, c8, sigma));
}

// One CTA (256 threads) per 128x128 block.
__global__ void k_e4m3_blocks(uint8_t* q, float* scales, int64_t rows, int64_t cols, uint32_t k0,
                              uint32_t k1, double c8, double sigma) {
    const int64_t cb = (cols + 127) / 128;
    const int64_t b = blockIdx.x;
    const int64_t r0 = (b / cb) * 128, c0 = (b % cb) * 128;
    const int tid = threadIdx.x;
    float v[64];
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < 64; ++j) {
        const int local = j * 256 + tid;
        const int64_t r = r0 + local / 128, c = c0 + local % 128;
        v[j] = 0.0f;
        if (r < rows && c < cols) {
            v[j] = value_f32((uint64_t)(r * cols + c), k0, k1, c8, sigma);
            amax = fmaxf(amax, fabsf(v[j]));
        }
    }
    __shared__ float red[8];
    __shared__ float s_sh;
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if ((tid & 31) == 0) red[tid >> 5] = amax;
    __syncthreads();
    if (tid == 0) {
        float m = red[0];
        for (int w = 1; w < 8; ++w) m = fmaxf(m, red[w]);
        float s = __fdiv_rn(m, 448.0f);
        if (m == 0.0f) s = 1.0f;
        s_sh = s;
        scales[b] = s;
    }
    __syncthreads();
    const float s = s_sh;
#pragma unroll
    for (int j = 0; j < 64; ++j) {
        const int local = j * 256 + tid;
        const int64_t r = r0 + local / 128, c = c0 + local % 128;
        if (r < rows && c < cols) {
            float x = __fdiv_rn(v[j], s);
            x = fminf(fmaxf(x, -448.0f), 448.0f);
            q[r * cols + c] = (uint8_t)__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3);
        }
    }
}

double unit_scale() { return 1.0 / sqrt(2863311530.0); }

int grid_for(int64_t n) {
    int64_t g = (n + 255) / 256;
    return (int)(g < 148 * 64 ? g : 148 * 64);
}

}  // namespace

extern "C" {

// All functions return a cudaError_t value (0 on success) and run on `stream`.

int moegen_gpu_philox4x32_10(const uint32_t* d_in, uint32_t k0, uint32_t k1, uint32_t* d_out,
                             cudaStream_t stream) {
    k_philox<<<1, 1, 0, stream>>>(d_in, k0, k1, d_out);
    return (int)cudaGetLastError();
}

int moegen_gpu_normal_f32(float* out, int64_t n, uint32_t k0, uint32_t k1, double sigma,
                          cudaStream_t stream) {
    if (n <= 0) return 0;
    k_normal_f32<<<grid_for(n), 256, 0, stream>>>(out, n, k0, k1, unit_scale(), sigma);
    return (int)cudaGetLastError();
}

int moegen_gpu_normal_bf16(void* out, int64_t n, uint32_t k0, uint32_t k1, double sigma,
                           cudaStream_t stream) {
    if (n <= 0) return 0;
    k_normal_bf16<<<grid_for(n), 256, 0, stream>>>((__nv_bfloat16*)out, n, k0, k1, unit_scale(),
                                                     sigma);
    return (int)cudaGetLastError();
}

int moegen_gpu_e4m3_blocks(void* q, float* scales, int64_t rows, int64_t cols, uint32_t k0,
                           uint32_t k1, double sigma, cudaStream_t stream) {
    const int64_t nb = ((rows + 127) / 128) * ((cols + 127) / 128);
    if (nb <= 0) return 0;
    k_e4m3_blocks<<<(unsigned)nb, 256, 0, stream>>>((uint8_t*)q, scales, rows, cols, k0, k1,
                                                     unit_scale(), sigma);
    return (int)cudaGetLastError();
}

}  // extern "C"
