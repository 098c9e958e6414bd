// moe_route: router logits (fp32 SIMT, fixed order), scores and top-k.
//
// The DWDP pages run DeepSeek-R1's MoE layer on every data-parallel rank
// (arXiv 2604.01621, abstract) and state no router arithmetic; the routing
// here is the DeepSeek-R1 layer shape read plainly (see include/moe.h).
//
// Logits are a dense [T,E] x [E,H]^T product, but they decide integers (the
// selected experts), so they are computed on the CUDA cores in one defined
// order that a CPU can reproduce bit for bit: chunks of 256 consecutive h,
// each a chain of fused multiply-adds from 0, chunk sums added in ascending
// order.  Tensor cores accumulate in an undefined order and are not used.
#include <cuda_bf16.h>

#include "device.cuh"
#include "internal.h"

namespace swb {
namespace {

constexpr int kChunk = 256;  // h per fused-multiply-add chain
constexpr int kKT = 32;      // h per shared-memory tile

// Two IEEE fused multiply-adds in one sm_100 instruction (packed fp32):
// lane i of d becomes fma(a_i, b_i, d_i), rounded to nearest like fmaf.
__device__ __forceinline__ uint64_t pack2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ float2 unpack2(uint64_t v) {
    float2 r;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
    return r;
}
__device__ __forceinline__ void fma2(uint64_t& d, uint64_t a, uint64_t b) {
    asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(d) : "l"(a), "l"(b));
}

// Eight consecutive values as fp32 (16-byte aligned source), or zeros.
__device__ __forceinline__ void load8(const __nv_bfloat16* p, bool in, float (&r)[8]) {
    const uint4 u = in ? *reinterpret_cast<const uint4*>(p) : make_uint4(0, 0, 0, 0);
    const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(b2[i]);
        r[2 * i] = f.x;
        r[2 * i + 1] = f.y;
    }
}
__device__ __forceinline__ void load8(const float* p, bool in, float (&r)[8]) {
    const float4 a = in ? *reinterpret_cast<const float4*>(p) : make_float4(0, 0, 0, 0);
    const float4 b = in ? *reinterpret_cast<const float4*>(p + 4) : make_float4(0, 0, 0, 0);
    r[0] = a.x; r[1] = a.y; r[2] = a.z; r[3] = a.w;
    r[4] = b.x; r[5] = b.y; r[6] = b.z; r[7] = b.w;
}

// Each thread owns a TM x TN block of (token, expert) pairs of a
// (16 TM) x (16 TN) block tile; 32 h per shared-memory stage, the next
// stage's global loads held in registers while the current one is consumed.
// With split != 0 the z index of the grid is the chunk and the kernel writes
// that chunk's sum P_c to part[c][t][e]; otherwise it walks all chunks and
// writes l[t][e].
template <typename XT, int TM, int TN>
__global__ void __launch_bounds__(256) k_logits(const XT* __restrict__ x,
                                                const float* __restrict__ wg, int T, int H, int E,
                                                int split, float* __restrict__ out) {
    constexpr int BT = 16 * TM, BE = 16 * TN;
    static_assert(TN % 2 == 0 && BT * kKT / 8 <= 256 && BE * kKT / 8 <= 256, "tile");
    __shared__ __align__(16) float xs[2][kKT][BT + 4];  // [buffer][h][token]
    __shared__ __align__(16) float ws[2][kKT][BE + 4];  // [buffer][h][expert]
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    const int e0 = blockIdx.x * BE, t0 = blockIdx.y * BT;
    int h_begin = 0, h_end = H;
    if (split) {
        h_begin = blockIdx.z * kChunk;
        h_end = min(H, h_begin + kChunk);
    }
    // loader: thread tid moves 8 consecutive h of tile row tid / 4
    const int lr = tid >> 2, lh = (tid & 3) * 8;
    const bool xl = tid < BT * kKT / 8, wl = tid < BE * kKT / 8;
    const bool xin = xl && t0 + lr < T, win = wl && e0 + lr < E;
    const XT* xrow = x + (int64_t)(xin ? t0 + lr : 0) * H + lh;
    const float* wrow = wg + (int64_t)(win ? e0 + lr : 0) * H + lh;
    float rx[8], rw[8];
    auto store = [&](int buf) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if (xl) xs[buf][lh + i][lr] = rx[i];
            if (wl) ws[buf][lh + i][lr] = rw[i];
        }
    };
    float l[TM][TN];
    uint64_t p[TM][TN / 2];  // chain sums of columns 2q, 2q + 1
#pragma unroll
    for (int i = 0; i < TM; ++i) {
#pragma unroll
        for (int j = 0; j < TN; ++j) l[i][j] = 0.0f;
#pragma unroll
        for (int q = 0; q < TN / 2; ++q) p[i][q] = 0;
    }
    const int nk = (h_end - h_begin) / kKT;
    load8(xrow + h_begin, xin, rx);
    load8(wrow + h_begin, win, rw);
    store(0);
    __syncthreads();
    for (int it = 0; it < nk; ++it) {
        const int buf = it & 1, h0 = h_begin + it * kKT;
        if (it + 1 < nk) {
            load8(xrow + h0 + kKT, xin, rx);
            load8(wrow + h0 + kKT, win, rw);
        }
#pragma unroll 8
        for (int kk = 0; kk < kKT; ++kk) {
            float a[TM], b[TN];
#pragma unroll
            for (int i = 0; i < TM; ++i) a[i] = xs[buf][kk][ty * TM + i];
#pragma unroll
            for (int j = 0; j < TN; ++j) b[j] = ws[buf][kk][tx * TN + j];
#pragma unroll
            for (int i = 0; i < TM; ++i) {
                const uint64_t ai = pack2(a[i], a[i]);
#pragma unroll
                for (int q = 0; q < TN / 2; ++q) fma2(p[i][q], ai, pack2(b[2 * q], b[2 * q + 1]));
            }
        }
        const int h_next = h0 + kKT;
        if (h_next % kChunk == 0 || h_next >= h_end) {  // a chunk ends here
            const bool first = split || (h_next - 1) / kChunk == 0;
#pragma unroll
            for (int i = 0; i < TM; ++i)
#pragma unroll
                for (int q = 0; q < TN / 2; ++q) {
                    const float2 v = unpack2(p[i][q]);
                    l[i][2 * q] = first ? v.x : __fadd_rn(l[i][2 * q], v.x);
                    l[i][2 * q + 1] = first ? v.y : __fadd_rn(l[i][2 * q + 1], v.y);
                    p[i][q] = 0;
                }
        }
        if (it + 1 < nk) store(buf ^ 1);
        __syncthreads();
    }
    float* o = split ? out + (int64_t)blockIdx.z * T * E : out;
#pragma unroll
    for (int i = 0; i < TM; ++i) {
        const int t = t0 + ty * TM + i;
        if (t >= T) continue;
#pragma unroll
        for (int j = 0; j < TN; ++j) {
            const int e = e0 + tx * TN + j;
            if (e < E) o[(int64_t)t * E + e] = l[i][j];
        }
    }
}

// Large batches: a 64-token x 128-expert block tile on 128 threads, 8 x 8
// (token, expert) pairs per thread in packed fp32x2 fused multiply-adds
// (four 16-byte shared loads feed 32 of them), 16 h per shared-memory stage
// with the next stage's global loads held in registers while the current one
// is consumed.  The arithmetic order is the same as k_logits: per 256-wide
// chunk a fused multiply-add chain in ascending h, chunk sums added in
// ascending order.
constexpr int kBigT = 64, kBigE = 128, kBigK = 16;

constexpr int kBigLd = kBigE + 4;  // row stride of the running sums in shared memory
constexpr size_t kBigDynSmem = (size_t)kBigT * kBigLd * sizeof(float);

//
// SPLIT: the z index of the grid is the 256-wide chunk.  The block computes
// that chunk's sums alone and writes them to plane z of out ([chunks][T][E]);
// k_reduce_parts then adds the planes in chunk order.  The same arithmetic,
// spread over H/256 times as many blocks, so that every SM holds three.
template <typename XT, bool SPLIT>
__global__ void __launch_bounds__(128, 3) k_logits_big(const XT* __restrict__ x,
                                                       const float* __restrict__ wg, int T, int H,
                                                       int E, float* __restrict__ out) {
    __shared__ __align__(16) float xs[2][kBigK][kBigT + 4];  // [buffer][h][token]
    __shared__ __align__(16) float ws[2][kBigK][kBigE + 4];
    extern __shared__ float ls[];
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;   // ty 0..7
    const int e0 = blockIdx.x * kBigE, t0 = blockIdx.y * kBigT;
    const int lt = tid >> 1, lh = (tid & 1) * 8;
    const bool odd = tid & 1;
    const bool xin = t0 + lt < T, win = e0 + tid < E;
    const XT* xrow = x + (int64_t)(xin ? t0 + lt : 0) * H + lh;
    const float* wrow = wg + (int64_t)(win ? e0 + tid : 0) * H;
    float rx[8], rw[16];
    auto load = [&](int h0) {
        if constexpr (sizeof(XT) == 2) {
            const uint4 u = xin ? *reinterpret_cast<const uint4*>(xrow + h0) : make_uint4(0, 0, 0, 0);
            const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 f = __bfloat1622float2(b2[i]);
                rx[2 * i] = f.x;
                rx[2 * i + 1] = f.y;
            }
        } else {
            const float4 a = xin ? *reinterpret_cast<const float4*>(xrow + h0) : make_float4(0, 0, 0, 0);
            const float4 b = xin ? *reinterpret_cast<const float4*>(xrow + h0 + 4) : make_float4(0, 0, 0, 0);
            rx[0] = a.x; rx[1] = a.y; rx[2] = a.z; rx[3] = a.w;
            rx[4] = b.x; rx[5] = b.y; rx[6] = b.z; rx[7] = b.w;
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float4 a = win ? *reinterpret_cast<const float4*>(wrow + h0 + 4 * q) : make_float4(0, 0, 0, 0);
            rw[4 * q] = a.x; rw[4 * q + 1] = a.y; rw[4 * q + 2] = a.z; rw[4 * q + 3] = a.w;
        }
    };
    // x is staged transposed (h-major, rows of kBigT + 4 floats); the two
    // lanes that load one token row write its column at h rows eight apart,
    // which share a bank, so odd lanes store their eight rows rotated by four
    // and a warp's stores hit 32 distinct banks
    auto store = [&](int buf) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int j = odd ? (i + 4) & 7 : i;
            const float vx = odd ? rx[(i + 4) & 7] : rx[i];
            xs[buf][lh + j][lt] = vx;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) ws[buf][i][tid] = rw[i];
    };
    auto row_of = [&](int i) { return i < 4 ? ty * 4 + i : 32 + ty * 4 + i - 4; };
    auto col_of = [&](int j) { return j < 4 ? tx * 4 + j : 64 + tx * 4 + j - 4; };
    uint64_t p[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int q = 0; q < 4; ++q) p[i][q] = 0;
    const int h_begin = SPLIT ? blockIdx.z * kChunk : 0;
    const int nk = SPLIT ? (min(H - h_begin, kChunk)) / kBigK : H / kBigK;
    load(h_begin);
    store(0);
    __syncthreads();
    for (int kt = 0; kt < nk; ++kt) {
        const int buf = kt & 1;
        if (kt + 1 < nk) load(h_begin + (kt + 1) * kBigK);
#pragma unroll
        for (int kk = 0; kk < kBigK; ++kk) {
            const float4 a0 = *reinterpret_cast<const float4*>(&xs[buf][kk][ty * 4]);
            const float4 a1 = *reinterpret_cast<const float4*>(&xs[buf][kk][32 + ty * 4]);
            const float4 b0 = *reinterpret_cast<const float4*>(&ws[buf][kk][tx * 4]);
            const float4 b1 = *reinterpret_cast<const float4*>(&ws[buf][kk][64 + tx * 4]);
            const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const uint64_t b[4] = {pack2(b0.x, b0.y), pack2(b0.z, b0.w), pack2(b1.x, b1.y),
                                   pack2(b1.z, b1.w)};
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint64_t ai = pack2(a[i], a[i]);
#pragma unroll
                for (int q = 0; q < 4; ++q) fma2(p[i][q], ai, b[q]);
            }
        }
        const int h_next = (kt + 1) * kBigK;
        if (!SPLIT && (h_next % kChunk == 0 || h_next >= H)) {
            const bool first = (h_next - 1) / kChunk == 0;
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float2 v = unpack2(p[i][q]);
                    float* l0 = &ls[row_of(i) * kBigLd + col_of(2 * q)];
                    float* l1 = &ls[row_of(i) * kBigLd + col_of(2 * q + 1)];
                    *l0 = first ? v.x : __fadd_rn(*l0, v.x);
                    *l1 = first ? v.y : __fadd_rn(*l1, v.y);
                    p[i][q] = 0;
                }
        }
        if (kt + 1 < nk) store(buf ^ 1);
        __syncthreads();
    }
    if constexpr (SPLIT) {
        float* o = out + (int64_t)blockIdx.z * T * E;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int t = t0 + row_of(i);
            if (t >= T) continue;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float2 v = unpack2(p[i][q]);
                const int e = e0 + col_of(2 * q);   // col_of(2q + 1) = e + 1
                if (e < E) o[(int64_t)t * E + e] = v.x;
                if (e + 1 < E) o[(int64_t)t * E + e + 1] = v.y;
            }
        }
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int t = t0 + row_of(i);
            if (t >= T) continue;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int e = e0 + col_of(j);
                if (e < E) out[(int64_t)t * E + e] = ls[row_of(i) * kBigLd + col_of(j)];
            }
        }
    }
}

// e^y in fp64 for |y| <= 700, every step one IEEE operation: Cody-Waite
// reduction with ln 2 = LN2_HI + LN2_LO (LN2_HI has 21 trailing zero bits),
// Taylor polynomial to degree 13 by Horner, exact scaling by 2^n.
// (W. J. Cody and W. Waite, Software Manual for the Elementary Functions.)
__device__ __forceinline__ double exp64_cw(double y) {
    const double kInvLn2 = 0x1.71547652b82fep+0;
    const double kLn2Hi = 0x1.62e42fee00000p-1;
    const double kLn2Lo = 0x1.a39ef35793c76p-33;
    const double c[14] = {0x1.0000000000000p+0, 0x1.0000000000000p+0, 0x1.0000000000000p-1,
                          0x1.5555555555555p-3, 0x1.5555555555555p-5, 0x1.1111111111111p-7,
                          0x1.6c16c16c16c17p-10, 0x1.a01a01a01a01ap-13, 0x1.a01a01a01a01ap-16,
                          0x1.71de3a556c734p-19, 0x1.27e4fb7789f5cp-22, 0x1.ae64567f544e4p-26,
                          0x1.1eed8eff8d898p-29, 0x1.6124613a86d09p-33};  // 1 / i!
    const double n = rint(__dmul_rn(y, kInvLn2));
    const double r = __dsub_rn(__dsub_rn(y, __dmul_rn(n, kLn2Hi)), __dmul_rn(n, kLn2Lo));
    double p = c[13];
#pragma unroll
    for (int i = 12; i >= 0; --i) p = __dadd_rn(__dmul_rn(p, r), c[i]);
    const long long e = static_cast<long long>(n) + 1023;
    return __dmul_rn(p, __longlong_as_double(e << 52));
}

// fp32( 1 / (1 + e^-x) ) with x clamped to [-120, 40] (no fp32 result changes).
__device__ __forceinline__ float sigmoid_f32(float l) {
    const double x = fmin(fmax(static_cast<double>(l), -120.0), 40.0);
    const double e = exp64_cw(-x);
    return __double2float_rn(__ddiv_rn(1.0, __dadd_rn(1.0, e)));
}

__device__ __forceinline__ bool better(float ka, int ia, float kb, int ib) {
    return ka > kb || (ka == kb && ia < ib);
}

// Warp-wide best (key, index) pair; every lane gets the result.
__device__ __forceinline__ void warp_best(float& k, int& i) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float k2 = __shfl_xor_sync(0xffffffffu, k, o);
        const int i2 = __shfl_xor_sync(0xffffffffu, i, o);
        if (better(k2, i2, k, i)) {
            k = k2;
            i = i2;
        }
    }
}

// Sum of the chunk partials of the split router, in chunk order:
// l[t][e] = ((P_0 + P_1) + P_2) + ...  written over P_0.  One thread per
// (token, expert); its loads are independent of each other.
__global__ void __launch_bounds__(256) k_reduce_parts(float* __restrict__ parts, int nsplit,
                                                      int64_t TE) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= TE) return;
    float v[32];
    const int n = nsplit < 32 ? nsplit : 32;
#pragma unroll
    for (int c = 0; c < 32; ++c)
        if (c < n) v[c] = parts[(int64_t)c * TE + i];
    float acc = v[0];
#pragma unroll
    for (int c = 1; c < 32; ++c)
        if (c < n) acc = __fadd_rn(acc, v[c]);
    for (int c = 32; c < nsplit; ++c) acc = __fadd_rn(acc, parts[(int64_t)c * TE + i]);
    parts[i] = acc;
}

// One warp per token.  Lane `lane` holds experts e = lane + 32 v.
template <int V>
__global__ void __launch_bounds__(256) k_select(const float* __restrict__ logits, int nsplit, int T,
                                                int E, int k, int score, int n_group,
                                                int topk_group, float routed_scale, int renorm,
                                                const float* __restrict__ bias,
                                                int32_t* __restrict__ topk_idx,
                                                float* __restrict__ topk_w) {
    __shared__ float keys_sh[8][32 * V];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x >> 5) + warp;
    if (t >= T) return;
    const float kNegInf = -__int_as_float(0x7f800000);
    float lg[V], key[V], sc[V];
    bool cand[V];
    // l = P_0 + P_1 + ... in chunk order; the loads of one chunk for all of
    // this lane's experts are independent and issued together
#pragma unroll
    for (int v = 0; v < V; ++v) {
        const int e = lane + 32 * v;
        lg[v] = (e < E) ? logits[(int64_t)t * E + e] : kNegInf;
    }
#pragma unroll 2
    for (int c = 1; c < nsplit; ++c) {
        const float* part = logits + ((int64_t)c * T + t) * E;
        float pc[V];
#pragma unroll
        for (int v = 0; v < V; ++v) pc[v] = (lane + 32 * v < E) ? part[lane + 32 * v] : 0.0f;
#pragma unroll
        for (int v = 0; v < V; ++v)
            if (lane + 32 * v < E) lg[v] = __fadd_rn(lg[v], pc[v]);
    }
#pragma unroll
    for (int v = 0; v < V; ++v) {
        const int e = lane + 32 * v;
        if (score == MOE_SCORE_SIGMOID) {
            sc[v] = (e < E) ? sigmoid_f32(lg[v]) : 0.0f;
            key[v] = (e < E) ? (bias ? __fadd_rn(sc[v], bias[e]) : sc[v]) : kNegInf;
        } else {
            sc[v] = lg[v];
            key[v] = lg[v];
        }
        cand[v] = e < E;
    }
    // group-limited candidates
    if (score == MOE_SCORE_SIGMOID && topk_group < n_group) {
#pragma unroll
        for (int v = 0; v < V; ++v) keys_sh[warp][lane + 32 * v] = key[v];
        __syncwarp();
        const int gs = E / n_group;
        float gscore = kNegInf;
        if (lane < n_group) {
            float b1 = kNegInf, b2 = kNegInf;
            for (int i = 0; i < gs; ++i) {
                const float kv = keys_sh[warp][lane * gs + i];
                if (kv > b1) {
                    b2 = b1;
                    b1 = kv;
                } else if (kv > b2) {
                    b2 = kv;
                }
            }
            gscore = (gs == 1) ? b1 : __fadd_rn(b1, b2);
        }
        uint32_t gmask = 0;
        float gk = gscore;
        for (int s = 0; s < topk_group; ++s) {
            float bk = (lane < n_group && !((gmask >> lane) & 1u)) ? gk : kNegInf;
            int bi = (lane < n_group && !((gmask >> lane) & 1u)) ? lane : 0x7fffffff;
            warp_best(bk, bi);
            gmask |= 1u << bi;
        }
#pragma unroll
        for (int v = 0; v < V; ++v) {
            const int e = lane + 32 * v;
            cand[v] = cand[v] && ((gmask >> (e / gs)) & 1u);
        }
    }
    // top-k, descending key, ties to the lower expert
    int my_e = -1;
    float my_s = 0.0f;
    for (int j = 0; j < k; ++j) {
        float bk = kNegInf;
        int bi = 0x7fffffff;
#pragma unroll
        for (int v = 0; v < V; ++v) {
            const int e = lane + 32 * v;
            if (cand[v] && better(key[v], e, bk, bi)) {
                bk = key[v];
                bi = e;
            }
        }
        warp_best(bk, bi);
        float s_sel = 0.0f;
#pragma unroll
        for (int v = 0; v < V; ++v)
            if (lane + 32 * v == bi) {
                cand[v] = false;
                s_sel = sc[v];
            }
        s_sel = __shfl_sync(0xffffffffu, s_sel, bi & 31);
        if (lane == j) {
            my_e = bi;
            my_s = s_sel;
        }
    }
    float w = 0.0f;
    if (score == MOE_SCORE_SIGMOID) {
        float d = 0.0f;
        for (int j = 0; j < k; ++j) {
            const float sj = __shfl_sync(0xffffffffu, my_s, j);
            d = (j == 0) ? sj : __fadd_rn(d, sj);
        }
        w = renorm ? __fdiv_rn(my_s, d) : my_s;
    } else {
        const float lmax = __shfl_sync(0xffffffffu, my_s, 0);
        const float num = (lane < k) ? expf(my_s - lmax) : 0.0f;
        float den = 0.0f;
        if (renorm) {
            den = num;
        } else {
#pragma unroll
            for (int v = 0; v < V; ++v)
                if (lane + 32 * v < E) den += expf(lg[v] - lmax);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
        w = num / den;
    }
    if (lane < k) {
        topk_idx[(int64_t)t * k + lane] = my_e;
        topk_w[(int64_t)t * k + lane] = __fmul_rn(w, routed_scale);
    }
}

struct RoutePlan {
    int tm;      // 2 or 4 (k_logits, TM == TN) or 8 (k_logits_big, 64 x 128 tiles)
    int nsplit;  // 1, or the number of 256-wide chunks
};

// Small batches split the h chunks over the grid (partial sums added in
// chunk order by k_reduce_parts); large ones use the 64 x 128 tile when it
// fills the GPU, with the chunks split over the grid as well (one block per
// tile and chunk: a tile per block alone leaves two of an SM's three block
// slots or fewer in use).
RoutePlan plan(const moe_route_cfg* c) {
    RoutePlan p;
    const int64_t tiles32 = (int64_t)((c->T + 31) / 32) * ((c->E + 31) / 32);
    const int64_t tiles_big = (int64_t)((c->T + kBigT - 1) / kBigT) * ((c->E + kBigE - 1) / kBigE);
    const bool small = tiles32 < 512;
    p.tm = small ? 2 : (tiles_big >= 240 ? 8 : 4);
    p.nsplit = (small || p.tm == 8) ? (c->H + kChunk - 1) / kChunk : 1;
    return p;
}

moe_status validate(const moe_route_cfg* c) {
    if (!c) return fail(MOE_ERR_INVALID_ARG, "moe_route: cfg is NULL");
    if (c->T < 0 || c->H <= 0 || c->E <= 0 || c->k <= 0)
        return fail(MOE_ERR_INVALID_ARG, "moe_route: T=%d H=%d E=%d k=%d", c->T, c->H, c->E, c->k);
    if (c->E > MOE_MAX_EXPERTS || c->k > MOE_MAX_TOPK || c->k > c->E)
        return fail(MOE_ERR_INVALID_ARG, "moe_route: E=%d (max %d), k=%d (max %d, <= E)", c->E,
                    MOE_MAX_EXPERTS, c->k, MOE_MAX_TOPK);
    if (c->H % 32) return fail(MOE_ERR_INVALID_ARG, "moe_route: H=%d not a multiple of 32", c->H);
    if (c->score == MOE_SCORE_SIGMOID) {
        if (c->n_group <= 0 || c->n_group > 32 || c->E % c->n_group)
            return fail(MOE_ERR_INVALID_ARG, "moe_route: n_group=%d must divide E=%d, <= 32",
                        c->n_group, c->E);
        if (c->topk_group <= 0 || c->topk_group > c->n_group)
            return fail(MOE_ERR_INVALID_ARG, "moe_route: topk_group=%d", c->topk_group);
        if ((int64_t)c->k > (int64_t)c->topk_group * (c->E / c->n_group))
            return fail(MOE_ERR_INVALID_ARG, "moe_route: k=%d exceeds the %d candidates", c->k,
                        c->topk_group * (c->E / c->n_group));
    } else if (c->score != MOE_SCORE_SOFTMAX) {
        return fail(MOE_ERR_INVALID_ARG, "moe_route: score=%d", c->score);
    }
    return MOE_OK;
}

template <typename XT>
void launch_logits(const moe_route_cfg* c, const RoutePlan& p, const XT* x, const float* wg,
                   float* out, cudaStream_t s) {
    const int B = 16 * p.tm;
    dim3 grid((c->E + B - 1) / B, (c->T + B - 1) / B, p.nsplit);
    if (p.tm == 8 && p.nsplit > 1) {
        dim3 g((c->E + kBigE - 1) / kBigE, (c->T + kBigT - 1) / kBigT, p.nsplit);
        k_logits_big<XT, true><<<g, 128, 0, s>>>(x, wg, c->T, c->H, c->E, out);
    } else if (p.tm == 8) {
        dim3 g((c->E + kBigE - 1) / kBigE, (c->T + kBigT - 1) / kBigT);
        cudaFuncSetAttribute(k_logits_big<XT, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kBigDynSmem);
        k_logits_big<XT, false><<<g, 128, kBigDynSmem, s>>>(x, wg, c->T, c->H, c->E, out);
    } else if (p.tm == 2) {
        k_logits<XT, 2, 2><<<grid, 256, 0, s>>>(x, wg, c->T, c->H, c->E, p.nsplit > 1, out);
    } else {
        k_logits<XT, 4, 4><<<grid, 256, 0, s>>>(x, wg, c->T, c->H, c->E, p.nsplit > 1, out);
    }
}

}  // namespace
}  // namespace swb

using namespace swb;

extern "C" {

size_t moe_route_workspace_size(const moe_route_cfg* c) {
    if (validate(c) != MOE_OK) return 0;
    const RoutePlan p = plan(c);
    return (size_t)p.nsplit * c->T * c->E * sizeof(float);
}

moe_status moe_route(const moe_route_cfg* c, const void* x, moe_dtype x_dtype, const float* w_gate,
                     const float* bias, int32_t* topk_idx, float* topk_w, void* workspace,
                     size_t workspace_bytes, cudaStream_t stream) {
    moe_status st = validate(c);
    if (st != MOE_OK) return st;
    if (x_dtype != MOE_F32 && x_dtype != MOE_BF16)
        return fail(MOE_ERR_UNSUPPORTED, "moe_route: x dtype %d", (int)x_dtype);
    if (c->T == 0) return MOE_OK;
    if (!x || !w_gate || !topk_idx || !topk_w)
        return fail(MOE_ERR_INVALID_ARG, "moe_route: NULL pointer");
    if (bias && c->score != MOE_SCORE_SIGMOID)
        return fail(MOE_ERR_INVALID_ARG, "moe_route: bias is only defined for sigmoid scores");
    if (!aligned(x, 16) || !aligned(w_gate, 16) || !aligned(topk_idx, 16) ||
        !aligned(topk_w, 16) || (bias && !aligned(bias, 16)))
        return fail(MOE_ERR_INVALID_ARG, "moe_route: pointers must be 16-byte aligned");
    const size_t need = moe_route_workspace_size(c);
    if (workspace_bytes < need || (need && !workspace))
        return fail(MOE_ERR_WORKSPACE, "moe_route: workspace %zu < %zu bytes", workspace_bytes,
                    need);
    if (cuda_injected_failure()) return fail(MOE_ERR_CUDA, "moe_route: injected failure");
    const RoutePlan p = plan(c);
    float* lg = static_cast<float*>(workspace);
    if (x_dtype == MOE_F32)
        launch_logits(c, p, static_cast<const float*>(x), w_gate, lg, stream);
    else
        launch_logits(c, p, static_cast<const __nv_bfloat16*>(x), w_gate, lg, stream);
    SWB_LAUNCHED("moe_route: logits kernel");
    int nsplit = p.nsplit;
    if (nsplit > 1) {   // chunk partials -> logits, in chunk order
        const int64_t TE = (int64_t)c->T * c->E;
        k_reduce_parts<<<(unsigned)((TE + 255) / 256), 256, 0, stream>>>(lg, nsplit, TE);
        SWB_LAUNCHED("moe_route: partial-sum kernel");
        nsplit = 1;
    }
    // one warp per token; small batches get one warp per block to use every SM
    const int warps = c->T < 8 * 148 ? 1 : 8;
    const int blocks = (c->T + warps - 1) / warps;
    const int V = (c->E + 31) / 32;
#define SWB_SELECT(VV)                                                                        \
    k_select<VV><<<blocks, 32 * warps, 0, stream>>>(lg, nsplit, c->T, c->E, c->k, c->score,   \
                                                    c->n_group, c->topk_group,               \
                                                    c->routed_scale, c->renormalize, bias,   \
                                                    topk_idx, topk_w)
    if (V <= 1) SWB_SELECT(1);
    else if (V <= 2) SWB_SELECT(2);
    else if (V <= 4) SWB_SELECT(4);
    else if (V <= 8) SWB_SELECT(8);
    else if (V <= 16) SWB_SELECT(16);
    else SWB_SELECT(32);
#undef SWB_SELECT
    SWB_LAUNCHED("moe_route: select kernel");
    return MOE_OK;
}

}  // extern "C"
