// moe_grouped_ffn: grouped SwiGLU expert GEMMs over split weight pools.
//
// The block's grouped GEMM (explainer "Distributed Weight Data Parallelism
// cuts LLM inference stalls", split-weight figure) must read each expert's
// weights wherever they sit: in this rank's local pool or in the buffer the
// remote experts were fetched into.  Instead of merging the two into one
// contiguous buffer, every pool gets a 3-D TMA tensor map {K, rows, slot};
// an expert is (pool, slot) in the per-expert table, so the producer warp
// simply picks the map and passes the slot as the third coordinate.
//
// One persistent, warp-specialised kernel per GEMM (sm_100a):
//   warp 0      TMA producer (one thread): weight tile(s) + token rows
//   warp 1      tcgen05.mma issuer (one thread); owns the TMEM allocation
//   warps 2..   epilogue (4 or 8 warps): TMEM -> registers -> (SwiGLU) -> bf16
// The MMA puts weight rows on M (128 per instruction) and the expert's tokens
// on N (16..256), so a decode-sized expert with 4 tokens costs an N=16 MMA,
// not a 128-row tile.  A CTA holds one or two weight tiles per stage:
//   GATED  gate rows and up rows of the same 128 features, two fp32
//          accumulators, SwiGLU fused in the epilogue (GEMM1);
//   PAIR   two adjacent 128-row blocks (256 output features, GEMM2);
//   SINGLE one 128-row block.
// Both weight tiles share the token tile, which halves the activation bytes
// each MMA needs.  Accumulators are double buffered in TMEM when they fit
// (two buffers of up to 256 columns) so the epilogue of one tile overlaps
// the next tile's main loop; the widest tiles (2 x 256 columns) use all 512
// TMEM columns in one buffer and 8 epilogue warps.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "device.cuh"
#include "internal.h"

namespace swb {
namespace {

constexpr int kMaxGroups = MOE_MAX_EXPERTS + 1;
constexpr int kBM = 128;                       // weight rows per tile (MMA M)
constexpr int kBK = 64;                        // K per stage: one 128-byte swizzle atom
constexpr int kBoxN = 16;                      // token rows per TMA box
constexpr uint32_t kABytes = kBM * kBK * 2;    // one weight tile, 16 KB
constexpr uint32_t kSmemBudget = 200 * 1024;   // pipeline stages

struct alignas(64) FfnArgs {
    CUtensorMap w_map[3];      // 0 local pool, 1 remote pool, 2 shared expert: {K, rows, slot}
    CUtensorMap act_map;       // activation rows {K, rows}, 16-row box
    CUtensorMap act_map64;     // the same rows, 64-row box
    const int32_t* offsets;    // [E+1] first row of each expert
    __nv_bfloat16* out;        // [rows, ld_out]
    int* err;                  // device error word
    int32_t E, T, A, has_shared;
    int32_t K;                 // reduction length (H for GEMM1, I for GEMM2)
    int32_t M;                 // output features per expert (I for GEMM1, H for GEMM2)
    int32_t up_row;            // GEMM1: first row of the "up" half of w_gu (= I)
    int32_t ld_out;
    int32_t pool_slot[kMaxGroups];  // (pool << 31) | slot per routed expert
    // e4m3 weights only: block scales of (slot, row block, k block) at
    // w_base[map] + slot * w_stride[map] + scale_off + 4 * (row_block * kblocks + k_block)
    const uint8_t* w_base[3];
    int64_t w_stride[3];
    int64_t scale_off;
    int32_t kblocks;
    // e4m3 activations (tensor-core fp8 path): activation scales [K/128][act_scale_ld]
    // (row = permuted row), and for the gate/up kernel the e4m3 output h with its
    // scales [M/128][act_scale_ld]
    const float* act_scale;
    int32_t act_scale_ld;
    uint8_t* out8;
    float* out_scale;
};

enum { kSingle = 0, kGated = 1, kPair = 2 };

constexpr uint32_t kA8Bytes = kBM * kBK;       // one e4m3 weight tile as loaded, 8 KB
constexpr int kConvThreads = 256;              // e4m3 -> bf16 converter warps (8)

// Per stage: the bf16 weight tile(s) the MMA reads (128-byte swizzled), the
// token tile, and for e4m3 weights the staging tile(s) TMA writes.
template <int BN, int MODE, bool W8>
struct Cfg {
    static constexpr int kNA = MODE == kSingle ? 1 : 2;           // weight tiles per stage
    static constexpr uint32_t kAStage = kABytes * kNA;
    static constexpr uint32_t kBStage = BN * kBK * 2;
    static constexpr uint32_t kA8Stage = W8 ? kA8Bytes * kNA : 0;
    static constexpr uint32_t kStageBytes = kAStage + kBStage + kA8Stage;
    static constexpr int kStages = (kSmemBudget / kStageBytes) > 12 ? 12 : (kSmemBudget / kStageBytes);
    static constexpr uint32_t kAccCols = kNA * BN;                // one accumulator set
    static constexpr int kAccBufs = 2 * kAccCols <= 512 ? 2 : 1;
    static constexpr uint32_t kTmemCols = kAccBufs * kAccCols;
    static constexpr int kEpiWarps = BN >= 256 ? 8 : 4;
    static constexpr int kConvWarps = W8 ? kConvThreads / 32 : 0;
    static constexpr int kConvFirstWarp = 2 + kEpiWarps;
    static constexpr int kThreads = 64 + 32 * (kEpiWarps + kConvWarps);
    static constexpr int kRowsPerTile = MODE == kPair ? 2 * kBM : kBM;  // output features
    static constexpr size_t kDynSmem = (size_t)kStages * kStageBytes + 1024;
    static_assert(kTmemCols >= 32 && kTmemCols <= 512 && (kTmemCols & (kTmemCols - 1)) == 0,
                  "TMEM allocation must be a power of two in [32, 512]");
    static_assert(kStages >= 2, "pipeline needs two stages");
};

// e4m3 weights and e4m3 activations on the tensor cores (kind::f8f6f4).
// A stage is one 128 x 128 scale block of K; its MMAs go into a fresh TMEM
// partial sum, which the epilogue warps fold into fp32 registers with the
// block's scales (weight block scale x per-token activation scale).
template <int BN, int MODE>
struct CfgF8 {
    static constexpr int kNA = 2;                                   // GATED or PAIR
    static constexpr int kBK8 = 128;                                // K (bytes) per stage
    static constexpr uint32_t kATile = kBM * kBK8;                  // 16 KB
    static constexpr uint32_t kAStage = kATile * kNA;
    static constexpr uint32_t kBStage = BN * kBK8;
    static constexpr uint32_t kStageBytes = kAStage + kBStage;
    static constexpr int kStages = (kSmemBudget / kStageBytes) > 8 ? 8 : (kSmemBudget / kStageBytes);
    static constexpr uint32_t kPartCols = kNA * BN;                 // one partial-sum set
    static constexpr int kPBufs = (512 / kPartCols) >= 8 ? 8 : (512 / kPartCols);
    static constexpr uint32_t kTmemCols = kPBufs * kPartCols;
    static constexpr int kEpiWarps = 8;                             // 2 per TMEM lane quarter
    static constexpr int kThreads = 64 + 32 * kEpiWarps;
    static constexpr int kRowsPerTile = MODE == kPair ? 2 * kBM : kBM;
    static constexpr int kCols = BN / 2;                            // columns per epilogue warp
    // per-warp combined scales [8][2][kCols] + amax exchange [2 halves][2 tiles][4][kCols]
    static constexpr size_t kScratch = (size_t)kEpiWarps * 2 * kCols * 4 + 2 * 2 * 4 * kCols * 4;
    static constexpr size_t kDynSmem = (size_t)kStages * kStageBytes + 1024 + kScratch;
    static_assert(kTmemCols >= 32 && kTmemCols <= 512 && (kTmemCols & (kTmemCols - 1)) == 0,
                  "TMEM allocation must be a power of two in [32, 512]");
    static_assert(kStages >= 2 && BN <= 64 && BN % 16 == 0, "fp8 tile shape");
};

struct Tile {
    int m0, row0, n_rows, n_mma, map, slot;
};

struct Tables {
    int tile_start[kMaxGroups + 1];
    int row0[kMaxGroups];
    int n[kMaxGroups];
    int ps[kMaxGroups];  // (map << 24) | slot   (map 0 local, 1 remote, 2 shared)
};

// An expert's n rows are cut into equal token tiles of tr rows (a multiple of
// 16, at most BN): tiles of one expert that stream the same weights then run
// at the same pace, so the second one finds the weights still in L2.
template <int BN>
__device__ __host__ __forceinline__ int tile_rows(int n) {
    const int ntn = (n + BN - 1) / BN;
    const int per = (n + ntn - 1) / ntn;
    return (per + 15) & ~15;
}

template <int BN>
__device__ __host__ __forceinline__ int token_tiles(int n) {
    if (n <= 0) return 0;
    const int tr = tile_rows<BN>(n);
    return (n + tr - 1) / tr;
}

template <int BN, int ROWS>
__device__ __forceinline__ Tile decode_tile(int tile, const Tables& tb, int G) {
    int lo = 0, hi = G - 1;
    while (lo < hi) {  // largest group whose first tile is <= tile (never an empty one)
        const int mid = (lo + hi + 1) >> 1;
        if (tb.tile_start[mid] <= tile) lo = mid;
        else hi = mid - 1;
    }
    const int g = lo, local = tile - tb.tile_start[g], n = tb.n[g];
    const int tr = tile_rows<BN>(n);
    const int ntn = (n + tr - 1) / tr;
    const int mt = local / ntn, nt = local - mt * ntn;
    Tile t;
    t.m0 = mt * ROWS;
    t.row0 = tb.row0[g] + nt * tr;
    t.n_rows = min(tr, n - nt * tr);
    t.n_mma = (t.n_rows + 15) & ~15;
    t.map = tb.ps[g] >> 24;
    t.slot = tb.ps[g] & 0xFFFFFF;
    return t;
}

// One warp: per-group first row, rows, tile count and (pool, slot), and the
// exclusive scan of tiles over the groups (routed experts, then the shared one).
template <int BN>
__device__ __forceinline__ void build_tables(const FfnArgs& p, Tables& tb, int G, int MT, int lane) {
    const int per = (G + 31) / 32, g0 = lane * per, g1 = min(G, g0 + per);
    int sum = 0;
    for (int g = g0; g < g1; ++g) {
        int n, r0, ps;
        if (g < p.E) {
            r0 = p.offsets[g];
            n = p.offsets[g + 1] - r0;
            const uint32_t v = static_cast<uint32_t>(p.pool_slot[g]);
            ps = (int)(((v >> 31) << 24) | (v & 0xFFFFFFu));
        } else {
            r0 = p.A;
            n = p.T;
            ps = 2 << 24;
        }
        tb.row0[g] = r0;
        tb.n[g] = n;
        tb.ps[g] = ps;
        sum += token_tiles<BN>(n) * MT;
    }
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    int run = incl - sum;
    for (int g = g0; g < g1; ++g) {
        tb.tile_start[g] = run;
        run += token_tiles<BN>(tb.n[g]) * MT;
    }
    if (lane == 31) tb.tile_start[G] = incl;
}

__device__ __forceinline__ float silu_mul(float g, float u) { return g / (1.0f + __expf(-g)) * u; }

// 16 e4m3 weights (one 16-byte chunk of a staged row) times their block
// scale, rounded to bf16: 32 bytes, the two 16-byte chunks that follow.
__device__ __forceinline__ void e4m3x16_to_bf16(const uint4 in, float s, uint4& lo, uint4& hi) {
    const uint32_t w[4] = {in.x, in.y, in.z, in.w};
    uint32_t o[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const __nv_fp8x2_storage_t pair = static_cast<__nv_fp8x2_storage_t>(w[i] >> (16 * h));
            const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(pair, __NV_E4M3);
            const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&hr));
            const __nv_bfloat162 b = __floats2bfloat162_rn(f.x * s, f.y * s);
            o[2 * i + h] = *reinterpret_cast<const uint32_t*>(&b);
        }
    }
    lo = make_uint4(o[0], o[1], o[2], o[3]);
    hi = make_uint4(o[4], o[5], o[6], o[7]);
}

template <int BN, int MODE, bool W8>
__global__ void __launch_bounds__(Cfg<BN, MODE, W8>::kThreads, 1)
    k_grouped_ffn(const __grid_constant__ FfnArgs p) {
    using C = Cfg<BN, MODE, W8>;
    extern __shared__ uint8_t dyn_smem[];
    __shared__ __align__(8) uint64_t full_bar[C::kStages], empty_bar[C::kStages];
    __shared__ __align__(8) uint64_t conv_bar[W8 ? C::kStages : 1];  // bf16 tiles converted
    __shared__ __align__(8) uint64_t acc_full[2], acc_empty[2];
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_sh;
    __shared__ Tables tb;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t stages = (smem_u32(dyn_smem) + 1023u) & ~1023u;
    const int G = p.E + (p.has_shared ? 1 : 0);
    const int MT = p.M / C::kRowsPerTile;
    const int KB = p.K / kBK;
    volatile int* abort_flag = &abort_sh;

    if (threadIdx.x == 0) {
        abort_sh = 0;
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(smem_u32(&full_bar[s]), 1);
            mbar_init(smem_u32(&empty_bar[s]), 1);
            if constexpr (W8) mbar_init(smem_u32(&conv_bar[s]), C::kConvWarps);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(smem_u32(&acc_full[a]), 1);
            mbar_init(smem_u32(&acc_empty[a]), C::kEpiWarps);
        }
        fence_mbar_init();
        tma_prefetch_map(&p.act_map);
        tma_prefetch_map(&p.act_map64);
        for (int m = 0; m < 3; ++m) tma_prefetch_map(&p.w_map[m]);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&tmem_base_sh), C::kTmemCols);
        tmem_relinquish();
    }
    if (warp == 2) build_tables<BN>(p, tb, G, MT, lane);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_base_sh;
    const int total = tb.tile_start[G];

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
                const Tile t = decode_tile<BN, C::kRowsPerTile>(tile, tb, G);
                const CUtensorMap* wm = &p.w_map[t.map];
                const uint32_t tx = (W8 ? C::kA8Stage : C::kAStage) + (uint32_t)t.n_mma * kBK * 2;
                const int row_a1 = MODE == kGated ? p.up_row + t.m0 : t.m0 + kBM;
                for (int kb = 0; kb < KB; ++kb) {
                    const uint32_t eb = smem_u32(&empty_bar[stage]);
                    const uint32_t fb = smem_u32(&full_bar[stage]);
                    if (!mbar_wait(eb, phase ^ 1u, abort_flag, p.err)) {
                        ok = false;
                        break;
                    }
                    const uint32_t sa = stages + stage * C::kStageBytes;
                    mbar_arrive_expect_tx(fb, tx);
                    // e4m3 weights land in the staging area, bf16 ones straight in the operand
                    const uint32_t sw = W8 ? sa + C::kAStage + C::kBStage : sa;
                    const uint32_t w_step = W8 ? kA8Bytes : kABytes;
                    tma_load_3d(sw, wm, fb, kb * kBK, t.m0, t.slot);
                    if constexpr (C::kNA == 2) tma_load_3d(sw + w_step, wm, fb, kb * kBK, row_a1, t.slot);
                    const uint32_t sb = sa + C::kAStage;
                    int r = 0;
                    for (; r + 64 <= t.n_mma; r += 64)
                        tma_load_2d(sb + r * kBK * 2, &p.act_map64, fb, kb * kBK, t.row0 + r);
                    for (; r < t.n_mma; r += kBoxN)
                        tma_load_2d(sb + r * kBK * 2, &p.act_map, fb, kb * kBK, t.row0 + r);
                    if (++stage == C::kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            int stage = 0, acc = 0;
            uint32_t phase = 0, acc_use[2] = {0u, 0u};
            bool ok = true;
            for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
                const Tile t = decode_tile<BN, C::kRowsPerTile>(tile, tb, G);
                if (!mbar_wait(smem_u32(&acc_empty[acc]), (acc_use[acc] & 1u) ^ 1u, abort_flag,
                               p.err))
                    break;
                tc_fence_after();
                const uint32_t d0 = tmem_base + acc * C::kAccCols;
                const uint32_t idesc = idesc_bf16_f32(kBM, t.n_mma);
                for (int kb = 0; kb < KB; ++kb) {
                    const uint32_t ready_bar = W8 ? smem_u32(&conv_bar[stage]) : smem_u32(&full_bar[stage]);
                    if (!mbar_wait(ready_bar, phase, abort_flag, p.err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = stages + stage * C::kStageBytes;
                    const uint32_t sb = sa + C::kAStage;
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk) {
                        const uint32_t accum = (kb | kk) != 0;
                        const uint64_t bd = sw128_desc(sb + kk * 32);
                        mma_bf16_ss(d0, sw128_desc(sa + kk * 32), bd, idesc, accum);
                        if constexpr (C::kNA == 2)
                            mma_bf16_ss(d0 + BN, sw128_desc(sa + kABytes + kk * 32), bd, idesc, accum);
                    }
                    mma_commit(smem_u32(&empty_bar[stage]));
                    if (++stage == C::kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                mma_commit(smem_u32(&acc_full[acc]));
                ++acc_use[acc];
                if (C::kAccBufs == 2) acc ^= 1;
            }
        }
    } else if (W8 && warp >= C::kConvFirstWarp) {
        // ------------------------------------------------ e4m3 -> bf16 converters
        // Each staged row is 64 e4m3 bytes (4 chunks of 16); the bf16 operand
        // row is 128 bytes in the 128-byte swizzle: 16-byte chunk j of row r
        // sits at position j ^ (r % 8).  One 128x128 block scale covers the
        // whole stage (64 columns of K, 128 rows).
        const int ct = threadIdx.x - 32 * C::kConvFirstWarp;  // 0 .. kConvThreads-1
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
            const Tile t = decode_tile<BN, C::kRowsPerTile>(tile, tb, G);
            const uint8_t* sbase = p.w_base[t.map] + (int64_t)t.slot * p.w_stride[t.map] + p.scale_off;
            const float* sc0 = reinterpret_cast<const float*>(sbase) + (int64_t)(t.m0 / kBM) * p.kblocks;
            const int rb1 = MODE == kGated ? (p.up_row + t.m0) / kBM : t.m0 / kBM + 1;
            const float* sc1 = reinterpret_cast<const float*>(sbase) + (int64_t)rb1 * p.kblocks;
            for (int kb = 0; kb < KB; ++kb) {
                const float s0 = __ldg(sc0 + (kb >> 1));
                const float s1 = C::kNA == 2 ? __ldg(sc1 + (kb >> 1)) : 0.0f;
                ok = mbar_wait(smem_u32(&full_bar[stage]), phase, abort_flag, p.err);
                if (!__all_sync(0xffffffffu, ok)) {
                    ok = false;
                    break;
                }
                const uint32_t sa = stages + stage * C::kStageBytes;
                const uint32_t s8 = sa + C::kAStage + C::kBStage;
#pragma unroll
                for (int a = 0; a < C::kNA; ++a) {
                    const float sc = a == 0 ? s0 : s1;
#pragma unroll
                    for (int i = 0; i < (kBM * kBK / 16) / kConvThreads; ++i) {
                        const int id = ct + kConvThreads * i, r = id >> 2, c = id & 3;
                        uint4 in, lo, hi;
                        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                                     : "=r"(in.x), "=r"(in.y), "=r"(in.z), "=r"(in.w)
                                     : "r"(s8 + a * kA8Bytes + r * kBK + c * 16));
                        e4m3x16_to_bf16(in, sc, lo, hi);
                        const uint32_t row = sa + a * kABytes + r * 128;
                        const uint32_t j0 = (2 * c) ^ (r & 7), j1 = (2 * c + 1) ^ (r & 7);
                        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(row + j0 * 16),
                                     "r"(lo.x), "r"(lo.y), "r"(lo.z), "r"(lo.w)
                                     : "memory");
                        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(row + j1 * 16),
                                     "r"(hi.x), "r"(hi.y), "r"(hi.z), "r"(hi.w)
                                     : "memory");
                    }
                }
                // generic-proxy stores -> visible to the tensor core's async proxy
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&conv_bar[stage]));
                if (++stage == C::kStages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
    } else {
        // ------------------------------------------------ epilogue
        const int q = warp & 3;                    // TMEM lane quarter this warp may access
        const int part = (warp - 2) >> 2;          // column half (8 epilogue warps) or 0
        constexpr int kCols = C::kEpiWarps == 8 ? BN / 2 : BN;
        int acc = 0;
        uint32_t acc_use[2] = {0u, 0u};
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
            const Tile t = decode_tile<BN, C::kRowsPerTile>(tile, tb, G);
            bool ok = mbar_wait(smem_u32(&acc_full[acc]), acc_use[acc] & 1u, abort_flag, p.err);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            const uint32_t tacc = tmem_base + ((uint32_t)(32 * q) << 16) + acc * C::kAccCols;
            const int f = t.m0 + 32 * q + lane;
            __nv_bfloat16* out = p.out + (int64_t)t.row0 * p.ld_out + f;
            const int c_begin = part * kCols, c_end = min(t.n_rows, c_begin + kCols);
            for (int c0 = c_begin; c0 < c_end; c0 += 16) {
                float g[16];
                tmem_ld_16(tacc + c0, g);
                if constexpr (C::kNA == 2) {
                    float u[16];
                    tmem_ld_16(tacc + BN + c0, u);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        if (c0 + i >= t.n_rows) continue;
                        __nv_bfloat16* o = out + (int64_t)(c0 + i) * p.ld_out;
                        if constexpr (MODE == kGated) {
                            o[0] = __float2bfloat16_rn(silu_mul(g[i], u[i]));
                        } else {
                            o[0] = __float2bfloat16_rn(g[i]);
                            o[kBM] = __float2bfloat16_rn(u[i]);
                        }
                    }
                } else {
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        if (c0 + i < t.n_rows)
                            out[(int64_t)(c0 + i) * p.ld_out] = __float2bfloat16_rn(g[i]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&acc_empty[acc]));
            ++acc_use[acc];
            if (C::kAccBufs == 2) acc ^= 1;
        }
    }

    __syncthreads();
    if (*abort_flag) {  // let copies still in flight land before TMEM is released
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 2000000ull) __nanosleep(1000);
    }
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, C::kTmemCols);
    }
}

// ---------------------------------------------------------------- fp8 tensor-core kernel
// warp 0 TMA producer, warp 1 MMA issuer, warps 2..9 epilogue.  Every stage
// (one 128-wide block of K) is multiplied into a fresh TMEM partial sum; the
// epilogue warps fold it into fp32 registers as acc += P * s_w * s_x[token],
// where s_w is the 128 x 128 weight block scale and s_x the activation
// scale of the token for that block of K.  GATED then quantises
// h = silu(gate) * up to e4m3 per (token, 128 features) for the down GEMM;
// PAIR writes bf16.
template <int BN, int MODE>
__global__ void __launch_bounds__(CfgF8<BN, MODE>::kThreads, 1)
    k_grouped_ffn_f8(const __grid_constant__ FfnArgs p) {
    using C = CfgF8<BN, MODE>;
    extern __shared__ uint8_t dyn_smem[];
    __shared__ __align__(8) uint64_t full_bar[C::kStages], empty_bar[C::kStages];
    __shared__ __align__(8) uint64_t part_full[C::kPBufs], part_empty[C::kPBufs];
    __shared__ __align__(8) uint64_t half_bar[2];   // the 4 epilogue warps of one column half
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_sh;
    __shared__ Tables tb;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t base_addr = smem_u32(dyn_smem);
    const uint32_t stages = (base_addr + 1023u) & ~1023u;
    float* scratch = reinterpret_cast<float*>(dyn_smem + (stages - base_addr) +
                                              (size_t)C::kStages * C::kStageBytes);
    const int G = p.E + (p.has_shared ? 1 : 0);
    const int MT = p.M / C::kRowsPerTile;
    const int KB = p.K / C::kBK8;
    volatile int* abort_flag = &abort_sh;

    if (threadIdx.x == 0) {
        abort_sh = 0;
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(smem_u32(&full_bar[s]), 1);
            mbar_init(smem_u32(&empty_bar[s]), 1);
        }
        for (int b = 0; b < C::kPBufs; ++b) {
            mbar_init(smem_u32(&part_full[b]), 1);
            mbar_init(smem_u32(&part_empty[b]), C::kEpiWarps);
        }
        mbar_init(smem_u32(&half_bar[0]), 4);
        mbar_init(smem_u32(&half_bar[1]), 4);
        fence_mbar_init();
        tma_prefetch_map(&p.act_map);
        tma_prefetch_map(&p.act_map64);
        for (int m = 0; m < 3; ++m) tma_prefetch_map(&p.w_map[m]);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&tmem_base_sh), C::kTmemCols);
        tmem_relinquish();
    }
    if (warp == 2) build_tables<BN>(p, tb, G, MT, lane);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_base_sh;
    const int total = tb.tile_start[G];

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
                const Tile t = decode_tile<BN, C::kRowsPerTile>(tile, tb, G);
                const CUtensorMap* wm = &p.w_map[t.map];
                const uint32_t tx = C::kAStage + (uint32_t)t.n_mma * C::kBK8;
                const int row_a1 = MODE == kGated ? p.up_row + t.m0 : t.m0 + kBM;
                for (int kb = 0; kb < KB; ++kb) {
                    const uint32_t fb = smem_u32(&full_bar[stage]);
                    if (!mbar_wait(smem_u32(&empty_bar[stage]), phase ^ 1u, abort_flag, p.err)) {
                        ok = false;
                        break;
                    }
                    const uint32_t sa = stages + stage * C::kStageBytes;
                    mbar_arrive_expect_tx(fb, tx);
                    tma_load_3d(sa, wm, fb, kb * C::kBK8, t.m0, t.slot);
                    tma_load_3d(sa + C::kATile, wm, fb, kb * C::kBK8, row_a1, t.slot);
                    const uint32_t sb = sa + C::kAStage;
                    int r = 0;
                    for (; r + 64 <= t.n_mma; r += 64)
                        tma_load_2d(sb + r * C::kBK8, &p.act_map64, fb, kb * C::kBK8, t.row0 + r);
                    for (; r < t.n_mma; r += kBoxN)
                        tma_load_2d(sb + r * C::kBK8, &p.act_map, fb, kb * C::kBK8, t.row0 + r);
                    if (++stage == C::kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            int stage = 0, pb = 0;
            uint32_t phase = 0, use[C::kPBufs];
#pragma unroll
            for (int b = 0; b < C::kPBufs; ++b) use[b] = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
                const Tile t = decode_tile<BN, C::kRowsPerTile>(tile, tb, G);
                const uint32_t idesc = idesc_e4m3_f32(kBM, t.n_mma);
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait(smem_u32(&part_empty[pb]), (use[pb] & 1u) ^ 1u, abort_flag, p.err) ||
                        !mbar_wait(smem_u32(&full_bar[stage]), phase, abort_flag, p.err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = stages + stage * C::kStageBytes;
                    const uint32_t sb = sa + C::kAStage;
                    const uint32_t d0 = tmem_base + pb * C::kPartCols;
#pragma unroll
                    for (int kk = 0; kk < C::kBK8 / 32; ++kk) {
                        const uint64_t bd = sw128_desc(sb + kk * 32);
                        mma_e4m3_ss(d0, sw128_desc(sa + kk * 32), bd, idesc, kk != 0);
                        mma_e4m3_ss(d0 + BN, sw128_desc(sa + C::kATile + kk * 32), bd, idesc, kk != 0);
                    }
                    mma_commit(smem_u32(&empty_bar[stage]));
                    mma_commit(smem_u32(&part_full[pb]));
                    ++use[pb];
                    if (++pb == C::kPBufs) pb = 0;
                    if (++stage == C::kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
        }
    } else {
        // ------------------------------------------------ epilogue (warps 2..9)
        constexpr int kC = C::kCols;
        const int q = warp & 3;              // TMEM lane quarter this warp may access
        const int part = (warp - 2) >> 2;    // which half of the token columns
        const int e = warp - 2;
        const int c_begin = part * kC;
        float* cg = scratch + e * 2 * kC;    // this warp's combined scales, gate / row block 0
        float* cu = cg + kC;                 //                              up / row block 1
        float* red_half = scratch + C::kEpiWarps * 2 * kC + part * 2 * 4 * kC;  // [2][4][kC]
        uint32_t tiles_done = 0;
        int pb = 0;
        uint32_t use[C::kPBufs];
#pragma unroll
        for (int b = 0; b < C::kPBufs; ++b) use[b] = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
            const Tile t = decode_tile<BN, C::kRowsPerTile>(tile, tb, G);
            const uint8_t* sbase = p.w_base[t.map] + (int64_t)t.slot * p.w_stride[t.map] + p.scale_off;
            const float* sw0p = reinterpret_cast<const float*>(sbase) + (int64_t)(t.m0 / kBM) * p.kblocks;
            const int rb1 = MODE == kGated ? (p.up_row + t.m0) / kBM : t.m0 / kBM + 1;
            const float* sw1p = reinterpret_cast<const float*>(sbase) + (int64_t)rb1 * p.kblocks;
            // this lane's token columns of the activation scales: c_begin + lane + 32 i
            constexpr int kSx = (kC + 31) / 32;
            auto load_sx = [&](int kb, float (&sx)[kSx]) {
#pragma unroll
                for (int i = 0; i < kSx; ++i) {
                    const int col = c_begin + lane + 32 * i;
                    const int r = t.row0 + col;
                    sx[i] = (lane + 32 * i < kC && col < t.n_rows)
                                ? __ldg(p.act_scale + (int64_t)kb * p.act_scale_ld + r) : 0.0f;
                }
            };
            float acc0[kC], acc1[kC];
#pragma unroll
            for (int j = 0; j < kC; ++j) acc0[j] = acc1[j] = 0.0f;
            float sx[kSx], sxn[kSx];
            load_sx(0, sx);
            float sw0 = __ldg(sw0p), sw1 = __ldg(sw1p);
            for (int kb = 0; kb < KB; ++kb) {
#pragma unroll
                for (int i = 0; i < kSx; ++i) {
                    if (lane + 32 * i < kC) {
                        cg[lane + 32 * i] = sx[i] * sw0;
                        cu[lane + 32 * i] = sx[i] * sw1;
                    }
                }
                __syncwarp();
                float sw0n = 0.0f, sw1n = 0.0f;
                if (kb + 1 < KB) {   // next block's scales travel while this one is folded in
                    load_sx(kb + 1, sxn);
                    sw0n = __ldg(sw0p + kb + 1);
                    sw1n = __ldg(sw1p + kb + 1);
                }
                ok = mbar_wait(smem_u32(&part_full[pb]), use[pb] & 1u, abort_flag, p.err);
                if (!__all_sync(0xffffffffu, ok)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t tp = tmem_base + ((uint32_t)(32 * q) << 16) + pb * C::kPartCols + c_begin;
                // the warp's whole slice of both partial sums, one wait, then the
                // buffer goes straight back to the MMA
                float a[kC], b[kC];
                tmem_ld_n<kC>(tp, a);
                tmem_ld_n<kC>(tp + BN, b);
                tmem_ld_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&part_empty[pb]));
#pragma unroll
                for (int c0 = 0; c0 < kC; c0 += 4) {
                    const float4 g = *reinterpret_cast<const float4*>(cg + c0);
                    const float4 u = *reinterpret_cast<const float4*>(cu + c0);
                    acc0[c0] = fmaf(a[c0], g.x, acc0[c0]);
                    acc0[c0 + 1] = fmaf(a[c0 + 1], g.y, acc0[c0 + 1]);
                    acc0[c0 + 2] = fmaf(a[c0 + 2], g.z, acc0[c0 + 2]);
                    acc0[c0 + 3] = fmaf(a[c0 + 3], g.w, acc0[c0 + 3]);
                    acc1[c0] = fmaf(b[c0], u.x, acc1[c0]);
                    acc1[c0 + 1] = fmaf(b[c0 + 1], u.y, acc1[c0 + 1]);
                    acc1[c0 + 2] = fmaf(b[c0 + 2], u.z, acc1[c0 + 2]);
                    acc1[c0 + 3] = fmaf(b[c0 + 3], u.w, acc1[c0 + 3]);
                }
                ++use[pb];
                if (++pb == C::kPBufs) pb = 0;
#pragma unroll
                for (int i = 0; i < kSx; ++i) sx[i] = sxn[i];
                sw0 = sw0n;
                sw1 = sw1n;
            }
            if (!ok) break;
            const int f = t.m0 + 32 * q + lane;
            if constexpr (MODE == kGated) {
                // h = silu(gate) * up, then e4m3 per (token, these 128 features):
                // the 128 features of a token column are the 4 warps of this half
                float* red = red_half + (tiles_done & 1u) * 4 * kC;
#pragma unroll
                for (int j = 0; j < kC; ++j) {
                    acc0[j] = silu_mul(acc0[j], acc1[j]);
                    float m = fabsf(acc0[j]);
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                    if (lane == 0) red[q * kC + j] = m;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&half_bar[part]));
                ok = mbar_wait(smem_u32(&half_bar[part]), tiles_done & 1u, abort_flag, p.err);
                if (!__all_sync(0xffffffffu, ok)) {
                    ok = false;
                    break;
                }
#pragma unroll
                for (int j = 0; j < kC; ++j) {
                    const int col = c_begin + j;
                    const float amax = fmaxf(fmaxf(red[j], red[kC + j]), fmaxf(red[2 * kC + j], red[3 * kC + j]));
                    const float sc = amax > 0.0f ? amax / 448.0f : 1.0f;
                    if (col < t.n_rows) {
                        const float v = fminf(fmaxf(acc0[j] / sc, -448.0f), 448.0f);
                        p.out8[(int64_t)(t.row0 + col) * p.ld_out + f] =
                            (uint8_t)__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3);
                        if (q == 0 && lane == 0)
                            p.out_scale[(int64_t)(t.m0 / kBM) * p.act_scale_ld + t.row0 + col] = sc;
                    }
                }
                // red is double buffered by tile parity: the next write of this
                // buffer comes after every warp of the half has passed the next
                // tile's barrier, i.e. finished reading it here
                ++tiles_done;
            } else {
#pragma unroll
                for (int j = 0; j < kC; ++j) {
                    const int col = c_begin + j;
                    if (col < t.n_rows) {
                        __nv_bfloat16* o = p.out + (int64_t)(t.row0 + col) * p.ld_out + f;
                        o[0] = __float2bfloat16_rn(acc0[j]);
                        o[kBM] = __float2bfloat16_rn(acc1[j]);
                    }
                }
            }
        }
    }

    __syncthreads();
    if (*abort_flag) {  // let copies still in flight land before TMEM is released
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 2000000ull) __nanosleep(1000);
    }
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, C::kTmemCols);
    }
}

// ---------------------------------------------------------------- host side
template <int BN, int MODE, bool W8>
moe_status launch(const FfnArgs& a, int rows, int G, cudaStream_t s) {
    using C = Cfg<BN, MODE, W8>;
    int sms = 0;
    moe_status st = sm_count(&sms);
    if (st != MOE_OK) return st;
    const int64_t mt = a.M / C::kRowsPerTile;
    const int64_t bound = mt * ((rows + 15) / 16 + G);
    const int grid = (int)(bound < sms ? bound : sms);
    if (grid <= 0) return MOE_OK;
    auto kern = k_grouped_ffn<BN, MODE, W8>;
    SWB_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)C::kDynSmem));
    kern<<<grid, C::kThreads, C::kDynSmem, s>>>(a);
    SWB_LAUNCHED(MODE == kGated ? "moe_grouped_ffn: gate/up kernel" : "moe_grouped_ffn: down kernel");
    return MOE_OK;
}

template <int MODE, bool W8>
moe_status launch_bn(int bn, const FfnArgs& a, int rows, int G, cudaStream_t s) {
    switch (bn) {
        case 16: return launch<16, MODE, W8>(a, rows, G, s);
        case 32: return launch<32, MODE, W8>(a, rows, G, s);
        case 64: return launch<64, MODE, W8>(a, rows, G, s);
        case 128: return launch<128, MODE, W8>(a, rows, G, s);
        default: return launch<256, MODE, W8>(a, rows, G, s);
    }
}

template <int BN, int MODE>
moe_status launch_f8(const FfnArgs& a, int rows, int G, cudaStream_t s) {
    using C = CfgF8<BN, MODE>;
    int sms = 0;
    moe_status st = sm_count(&sms);
    if (st != MOE_OK) return st;
    const int64_t mt = a.M / C::kRowsPerTile;
    const int64_t bound = mt * ((rows + 15) / 16 + G);
    const int grid = (int)(bound < sms ? bound : sms);
    if (grid <= 0) return MOE_OK;
    auto kern = k_grouped_ffn_f8<BN, MODE>;
    SWB_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)C::kDynSmem));
    kern<<<grid, C::kThreads, C::kDynSmem, s>>>(a);
    SWB_LAUNCHED(MODE == kGated ? "moe_grouped_ffn: fp8 gate/up kernel" : "moe_grouped_ffn: fp8 down kernel");
    return MOE_OK;
}

template <int MODE>
moe_status launch_f8_bn(int bn, const FfnArgs& a, int rows, int G, cudaStream_t s) {
    switch (bn) {
        case 16: return launch_f8<16, MODE>(a, rows, G, s);
        case 32: return launch_f8<32, MODE>(a, rows, G, s);
        default: return launch_f8<64, MODE>(a, rows, G, s);
    }
}

template <int MODE>
moe_status launch_w(bool w8, int bn, const FfnArgs& a, int rows, int G, cudaStream_t s) {
    return w8 ? launch_bn<MODE, true>(bn, a, rows, G, s) : launch_bn<MODE, false>(bn, a, rows, G, s);
}

// Token tile from the mean tokens per routed expert, 16..256.
int pick_bn(int64_t A, int E) {
    const int64_t mean = (A + E - 1) / E;
    if (mean <= 8) return 16;
    if (mean <= 16) return 32;
    if (mean <= 32) return 64;
    if (mean <= 160) return 128;
    return 256;
}

// 3-D map {K, rows, slot} over one pool of expert images.  bf16 weights are
// loaded straight into the MMA operand layout (128-byte swizzle); e4m3
// weights as plain 64-byte rows for the converter warps.
// The e4m3 map for the tensor-core fp8 path (f8mma) loads 128-byte rows
// straight into the MMA operand layout.
moe_status encode_weight_map(CUtensorMap* m, const void* base, int64_t offset, int32_t count,
                             int64_t stride, int32_t K, int32_t rows, bool w8, bool f8mma = false) {
    const uint64_t dims[3] = {(uint64_t)K, (uint64_t)rows, (uint64_t)count};
    const uint64_t strides[2] = {(uint64_t)K * (w8 ? 1 : 2), (uint64_t)stride};
    const uint32_t box[3] = {(uint32_t)(f8mma ? 128 : kBK), (uint32_t)kBM, 1u};
    return encode_tiled(m, w8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                        const_cast<char*>(static_cast<const char*>(base)) + offset, dims, strides,
                        box, (w8 && !f8mma) ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B);
}

moe_status encode_act_map8(CUtensorMap* m, const void* base, int64_t rows, int32_t K,
                           uint32_t box_rows) {
    const uint64_t dims[2] = {(uint64_t)K, (uint64_t)rows};
    const uint64_t strides[1] = {(uint64_t)K};
    const uint32_t box[2] = {128u, box_rows};
    return encode_tiled(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims,
                        strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

moe_status encode_act_map(CUtensorMap* m, const void* base, int64_t rows, int32_t K,
                          uint32_t box_rows) {
    const uint64_t dims[2] = {(uint64_t)K, (uint64_t)rows};
    const uint64_t strides[1] = {(uint64_t)K * 2};
    const uint32_t box[2] = {(uint32_t)kBK, box_rows};
    return encode_tiled(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                        strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

moe_status validate(const moe_ffn_desc* d, const moe_expert_table* tb, moe_expert_layout* lay) {
    if (!d || !tb) return fail(MOE_ERR_INVALID_ARG, "moe_grouped_ffn: NULL descriptor or table");
    if (d->T < 0 || d->k <= 0 || d->k > MOE_MAX_TOPK || d->E <= 0 || d->E > MOE_MAX_EXPERTS ||
        d->H <= 0 || d->I <= 0 || d->H % 128 || d->I % 128)
        return fail(MOE_ERR_INVALID_ARG, "moe_grouped_ffn: T=%d H=%d I=%d E=%d k=%d", d->T, d->H,
                    d->I, d->E, d->k);
    const bool ok_types = (d->w_dtype == MOE_BF16 && d->act_dtype == MOE_BF16) ||
                          (d->w_dtype == MOE_E4M3 && d->act_dtype == MOE_BF16) ||
                          (d->w_dtype == MOE_E4M3 && d->act_dtype == MOE_E4M3 && d->H % 256 == 0);
    if (!ok_types)
        return fail(MOE_ERR_UNSUPPORTED, "moe_grouped_ffn: weight dtype %d / activation dtype %d",
                    d->w_dtype, d->act_dtype);
    moe_status st = moe_expert_layout_get(d->H, d->I, (moe_dtype)d->w_dtype, lay);
    if (st != MOE_OK) return st;
    if (!tb->pool_slot) return fail(MOE_ERR_INVALID_ARG, "moe_grouped_ffn: pool_slot is NULL");
    const void* base[2] = {tb->local_base, tb->remote_base};
    const int32_t count[2] = {tb->local_count, tb->remote_count};
    const int64_t stride[2] = {tb->local_stride, tb->remote_stride};
    for (int q = 0; q < 2; ++q) {
        if (count[q] < 0 || count[q] > 0xFFFFFF)
            return fail(MOE_ERR_INVALID_ARG, "moe_grouped_ffn: pool %d count %d", q, count[q]);
        if (count[q] == 0) continue;
        if (!base[q] || !aligned(base[q], 256))
            return fail(MOE_ERR_INVALID_ARG, "moe_grouped_ffn: pool %d base must be non-NULL and "
                        "256-byte aligned", q);
        if (stride[q] < lay->bytes || stride[q] % 256)
            return fail(MOE_ERR_INVALID_ARG, "moe_grouped_ffn: pool %d stride %lld (need >= %lld, "
                        "multiple of 256)", q, (long long)stride[q], (long long)lay->bytes);
    }
    for (int e = 0; e < d->E; ++e) {
        const uint32_t v = static_cast<uint32_t>(tb->pool_slot[e]);
        const int q = (int)(v >> 31), slot = (int)(v & 0x7FFFFFFFu);
        if (slot >= count[q])
            return fail(MOE_ERR_INVALID_ARG, "moe_grouped_ffn: expert %d -> pool %d slot %d, but "
                        "the pool has %d slots", e, q, slot, count[q]);
    }
    if (d->has_shared && (!tb->shared || !aligned(tb->shared, 256)))
        return fail(MOE_ERR_INVALID_ARG, "moe_grouped_ffn: shared expert image missing or "
                    "not 256-byte aligned");
    return MOE_OK;
}

// Both GEMMs on the e4m3 tensor-core path: x_perm and h are e4m3 with
// per-(row, 128 columns) scales stored [K/128][rows].
moe_status ffn_f8(const moe_ffn_desc* d, const moe_expert_table* tbl, const moe_expert_layout& lay,
                  const void* x_perm, const float* x_scales, void* h, void* y_perm, float* h_scales,
                  int rows, int G, FfnArgs& a, cudaStream_t stream) {
    moe_status st;
    const void* base[2] = {tbl->local_base, tbl->remote_base};
    const int32_t count[2] = {tbl->local_count, tbl->remote_count};
    const int64_t stride[2] = {tbl->local_stride, tbl->remote_stride};
    // token tiles of at most 64: a warp then folds its 32 columns of both
    // partial sums with one TMEM read, and 4 partial buffers let the MMA run ahead
    int bn = pick_bn(a.A, d->E);
    if (bn > 64) bn = 64;
    // GEMM1 -> h (e4m3) and its scales
    for (int q = 0; q < 2; ++q)
        if (count[q] > 0 && (st = encode_weight_map(&a.w_map[q], base[q], lay.gu_offset, count[q],
                                                    stride[q], d->H, 2 * d->I, true, true)) != MOE_OK)
            return st;
    if (d->has_shared && (st = encode_weight_map(&a.w_map[2], tbl->shared, lay.gu_offset, 1,
                                                 lay.bytes, d->H, 2 * d->I, true, true)) != MOE_OK)
        return st;
    if ((st = encode_act_map8(&a.act_map, x_perm, rows, d->H, kBoxN)) != MOE_OK) return st;
    if ((st = encode_act_map8(&a.act_map64, x_perm, rows, d->H, 64)) != MOE_OK) return st;
    a.K = d->H;
    a.M = d->I;
    a.up_row = d->I;
    a.ld_out = d->I;
    a.scale_off = lay.gu_scale_offset;
    a.kblocks = d->H / 128;
    a.act_scale = x_scales;
    a.act_scale_ld = rows;
    a.out8 = static_cast<uint8_t*>(h);
    a.out_scale = h_scales;
    if ((st = launch_f8_bn<kGated>(bn, a, rows, G, stream)) != MOE_OK) return st;
    // GEMM2 -> y_perm (bf16)
    for (int q = 0; q < 2; ++q)
        if (count[q] > 0 && (st = encode_weight_map(&a.w_map[q], base[q], lay.down_offset,
                                                    count[q], stride[q], d->I, d->H, true, true)) != MOE_OK)
            return st;
    if (d->has_shared && (st = encode_weight_map(&a.w_map[2], tbl->shared, lay.down_offset, 1,
                                                 lay.bytes, d->I, d->H, true, true)) != MOE_OK)
        return st;
    if ((st = encode_act_map8(&a.act_map, h, rows, d->I, kBoxN)) != MOE_OK) return st;
    if ((st = encode_act_map8(&a.act_map64, h, rows, d->I, 64)) != MOE_OK) return st;
    a.K = d->I;
    a.M = d->H;
    a.up_row = 0;
    a.ld_out = d->H;
    a.scale_off = lay.down_scale_offset;
    a.kblocks = d->I / 128;
    a.act_scale = h_scales;
    a.out = static_cast<__nv_bfloat16*>(y_perm);
    a.out8 = nullptr;
    a.out_scale = nullptr;
    return launch_f8_bn<kPair>(bn, a, rows, G, stream);
}

}  // namespace
}  // namespace swb

using namespace swb;

extern "C" {

size_t moe_grouped_ffn_workspace_size(const moe_ffn_desc* d) {
    // e4m3 activations: the fp32 scales of the e4m3 intermediate h, [I/128][rows]
    if (!d || d->act_dtype != MOE_E4M3 || d->T <= 0 || d->k <= 0 || d->I <= 0) return 0;
    const int64_t rows = (int64_t)d->T * d->k + (d->has_shared ? d->T : 0);
    return (size_t)((d->I / 128) * rows * 4 + 255) / 256 * 256;
}

moe_status moe_grouped_ffn(const moe_ffn_desc* d, const moe_expert_table* tbl, const void* x_perm,
                           const float* x_perm_scales, const int32_t* offsets, void* h,
                           void* y_perm, void* workspace, size_t workspace_bytes,
                           cudaStream_t stream) {
    moe_expert_layout lay;
    moe_status st = validate(d, tbl, &lay);
    if (st != MOE_OK) return st;
    if (d->T == 0) return MOE_OK;
    if (!x_perm || !offsets || !h || !y_perm)
        return fail(MOE_ERR_INVALID_ARG, "moe_grouped_ffn: NULL pointer");
    if (!aligned(x_perm, 16) || !aligned(offsets, 16) || !aligned(h, 16) || !aligned(y_perm, 16))
        return fail(MOE_ERR_INVALID_ARG, "moe_grouped_ffn: pointers must be 16-byte aligned");
    const int64_t A = (int64_t)d->T * d->k;
    const int64_t rows = A + (d->has_shared ? d->T : 0);
    if (rows > INT32_MAX / 2) return fail(MOE_ERR_UNSUPPORTED, "moe_grouped_ffn: too many rows");
    const int G = d->E + (d->has_shared ? 1 : 0);
    const bool f8 = d->act_dtype == MOE_E4M3;
    if (f8) {
        const size_t need = moe_grouped_ffn_workspace_size(d);
        if (!x_perm_scales || !aligned(x_perm_scales, 16))
            return fail(MOE_ERR_INVALID_ARG, "moe_grouped_ffn: e4m3 activations need x_perm_scales");
        if (workspace_bytes < need || !workspace || !aligned(workspace, 16))
            return fail(MOE_ERR_WORKSPACE, "moe_grouped_ffn: workspace %zu < %zu bytes",
                        workspace_bytes, need);
    }
    int* err = nullptr;
    st = device_error_word(&err);
    if (st != MOE_OK) return st;

    static thread_local FfnArgs a;  // ~5 KB: kept off the stack
    memset(&a, 0, sizeof a);
    a.offsets = offsets;
    a.err = err;
    a.E = d->E;
    a.T = d->T;
    a.A = (int32_t)A;
    a.has_shared = d->has_shared ? 1 : 0;
    for (int e = 0; e < d->E; ++e) a.pool_slot[e] = tbl->pool_slot[e];
    const void* base[2] = {tbl->local_base, tbl->remote_base};
    const int32_t count[2] = {tbl->local_count, tbl->remote_count};
    const int64_t stride[2] = {tbl->local_stride, tbl->remote_stride};
    const int bn = pick_bn(A, d->E);
    const bool w8 = d->w_dtype == MOE_E4M3;
    a.w_base[0] = static_cast<const uint8_t*>(tbl->local_base);
    a.w_base[1] = static_cast<const uint8_t*>(tbl->remote_base);
    a.w_base[2] = static_cast<const uint8_t*>(tbl->shared);
    a.w_stride[0] = tbl->local_stride;
    a.w_stride[1] = tbl->remote_stride;
    a.w_stride[2] = lay.bytes;
    if (f8) return ffn_f8(d, tbl, lay, x_perm, x_perm_scales, h, y_perm,
                          static_cast<float*>(workspace), (int)rows, G, a, stream);

    // GEMM1: h = silu(X W_gate^T) * (X W_up^T)
    for (int q = 0; q < 2; ++q)
        if (count[q] > 0 && (st = encode_weight_map(&a.w_map[q], base[q], lay.gu_offset, count[q],
                                                    stride[q], d->H, 2 * d->I, w8)) != MOE_OK)
            return st;
    if (d->has_shared && (st = encode_weight_map(&a.w_map[2], tbl->shared, lay.gu_offset, 1,
                                                 lay.bytes, d->H, 2 * d->I, w8)) != MOE_OK)
        return st;
    a.scale_off = lay.gu_scale_offset;
    a.kblocks = d->H / 128;
    if ((st = encode_act_map(&a.act_map, x_perm, rows, d->H, kBoxN)) != MOE_OK) return st;
    if ((st = encode_act_map(&a.act_map64, x_perm, rows, d->H, 64)) != MOE_OK) return st;
    a.K = d->H;
    a.M = d->I;
    a.up_row = d->I;
    a.out = static_cast<__nv_bfloat16*>(h);
    a.ld_out = d->I;
    if ((st = launch_w<kGated>(w8, bn, a, (int)rows, G, stream)) != MOE_OK) return st;

    // GEMM2: y = h W_down^T
    for (int q = 0; q < 2; ++q)
        if (count[q] > 0 && (st = encode_weight_map(&a.w_map[q], base[q], lay.down_offset,
                                                    count[q], stride[q], d->I, d->H, w8)) != MOE_OK)
            return st;
    if (d->has_shared && (st = encode_weight_map(&a.w_map[2], tbl->shared, lay.down_offset, 1,
                                                 lay.bytes, d->I, d->H, w8)) != MOE_OK)
        return st;
    a.scale_off = lay.down_scale_offset;
    a.kblocks = d->I / 128;
    if ((st = encode_act_map(&a.act_map, h, rows, d->I, kBoxN)) != MOE_OK) return st;
    if ((st = encode_act_map(&a.act_map64, h, rows, d->I, 64)) != MOE_OK) return st;
    a.K = d->I;
    a.M = d->H;
    a.up_row = 0;
    a.out = static_cast<__nv_bfloat16*>(y_perm);
    a.ld_out = d->H;
    if (d->H % (2 * kBM) == 0) return launch_w<kPair>(w8, bn, a, (int)rows, G, stream);
    return launch_w<kSingle>(w8, bn, a, (int)rows, G, stream);
}

}  // extern "C"
