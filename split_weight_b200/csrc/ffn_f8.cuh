// The fp8 tensor-core grouped FFN kernel (kind::f8f6f4) with per-block
// scale promotion in the epilogue.
#pragma once

#include "ffn_common.cuh"

namespace swb {
namespace {

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
    static constexpr int kEpiWarps = BN >= 64 ? 16 : 8;             // 4 or 2 per TMEM lane quarter
    static constexpr int kParts = kEpiWarps / 4;                    // column slices of the tile
    static constexpr int kThreads = 64 + 32 * kEpiWarps;
    static constexpr int kRowsPerTile = MODE == kPair ? 2 * kBM : kBM;
    static constexpr int kCols = BN / kParts;                       // columns per epilogue warp
    // per-warp combined scales [kEpiWarps][2][kCols] + amax exchange [kParts][2 tiles][4][kCols]
    static constexpr size_t kScratch = (size_t)kEpiWarps * 2 * kCols * 4 + (size_t)kParts * 2 * 4 * kCols * 4;
    static constexpr size_t kDynSmem = (size_t)kStages * kStageBytes + 1024 + kScratch;
    static_assert(kTmemCols >= 32 && kTmemCols <= 512 && (kTmemCols & (kTmemCols - 1)) == 0,
                  "TMEM allocation must be a power of two in [32, 512]");
    static_assert(kStages >= 2 && BN <= 64 && BN % 16 == 0, "fp8 tile shape");
};

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
    __shared__ __align__(8) uint64_t half_bar[C::kParts];  // the 4 epilogue warps of one column slice
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
        for (int b = 0; b < C::kParts; ++b) mbar_init(smem_u32(&half_bar[b]), 4);
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
            int stage = 0, passed = -1;
            uint32_t phase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
                const Tile t = decode_tile<BN, C::kRowsPerTile>(tile, tb, G);
                if (!gate_wait(p, t.map, t.slot, passed, abort_flag, p.err)) break;
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
                if (ok) report_progress(p, total);
            }
        }
    } else {
        // ------------------------------------------------ epilogue (warps 2..9)
        constexpr int kC = C::kCols;
        const int q = warp & 3;              // TMEM lane quarter this warp may access
        const int part = (warp - 2) >> 2;    // which slice of the token columns
        const int e = warp - 2;
        const int c_begin = part * kC;
        float* cg = scratch + e * 2 * kC;    // this warp's combined scales, gate / row block 0
        float* cu = cg + kC;                 //                              up / row block 1
        float* red_half = scratch + C::kEpiWarps * 2 * kC + part * 2 * 4 * kC;  // [2][4][kC]
        uint32_t tiles_done = 0;
        int pb = 0, passed = -1;
        uint32_t use[C::kPBufs];
#pragma unroll
        for (int b = 0; b < C::kPBufs; ++b) use[b] = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
            const Tile t = decode_tile<BN, C::kRowsPerTile>(tile, tb, G);
            // the weight block scales sit in the remote buffer too: read them only once landed
            if (!__all_sync(0xffffffffu, gate_wait(p, t.map, t.slot, passed, abort_flag, p.err))) break;
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
            const bool gated = p.ready_flags != nullptr;   // a fetch may still be writing the buffer
            float sw0 = gated ? __ldcg(sw0p) : __ldg(sw0p), sw1 = gated ? __ldcg(sw1p) : __ldg(sw1p);
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
                    sw0n = gated ? __ldcg(sw0p + kb + 1) : __ldg(sw0p + kb + 1);
                    sw1n = gated ? __ldcg(sw1p + kb + 1) : __ldg(sw1p + kb + 1);
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

}  // namespace
}  // namespace swb
