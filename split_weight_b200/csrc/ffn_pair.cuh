// The grouped FFN on CTA pairs (tcgen05.mma.cta_group::2) for 256-token
// tiles with bf16 weights and activations: the large-batch shape, where the
// tensor cores bound the layer.
//
// A pair computes a 256-row x N-token tile (N <= 256) with one MMA per 16 of
// K: each CTA stages 128 weight rows and half of the tokens, the MMA reads
// both CTAs' operands, and each CTA's TMEM receives its own 128 rows x all N
// columns.  An accumulator is then 256 columns wide, so TMEM holds two and
// the epilogue of one tile overlaps the next tile's main loop, which the
// single-CTA kernel cannot do at this tile size (two 256-column
// accumulators, gate and up, fill its TMEM).
//
//   GATED (gate/up + SwiGLU): the pair covers 128 features; CTA r stages the
//     gate and up rows of features [64r, 64r + 64) interleaved (row 2i =
//     gate of feature i, row 2i + 1 = its up), loaded with one 4-D TMA box
//     {K 64, gate|up 2, feature 64}.  A TMEM lane pair then holds a feature's
//     gate and up, and the epilogue combines them with one shuffle.
//   PAIR (down): the pair covers 256 output features, 128 per CTA.
//
// Roles (both CTAs): warp 0 producer (one thread: its CTA's operands, the
// transaction bytes counted on the leader's barrier), warp 1 owns TMEM and,
// in the leader (cluster rank 0) only, issues the MMAs; warps 2..9 epilogue.
#pragma once

#include "ffn_common.cuh"

namespace swb {
namespace {

template <int MODE>
struct CfgPair {
    static constexpr int kBN = 256;                            // tokens per tile (MMA N)
    static constexpr int kAL = 32;                             // tile rows: halves of 16-row boxes
    static constexpr uint32_t kAStage = kABytes;               // 128 weight rows x 64 K, 16 KB
    static constexpr uint32_t kBStage = (kBN / 2) * kBK * 2;   // half the tokens x 64 K, 16 KB
    static constexpr uint32_t kStageBytes = kAStage + kBStage;
    static constexpr int kStages = (kSmemBudget / kStageBytes) > 8 ? 8 : (kSmemBudget / kStageBytes);
    static constexpr uint32_t kAccCols = kBN;                  // one accumulator: 256 fp32 columns
    static constexpr uint32_t kTmemCols = 2 * kAccCols;        // two, double buffered
    static constexpr int kEpiWarps = 8;                        // 2 per TMEM lane quarter
    static constexpr int kThreads = 64 + 32 * kEpiWarps;
    static constexpr int kRowsPerTile = MODE == kGated ? kBM : 2 * kBM;   // output features per tile
    static constexpr size_t kDynSmem = (size_t)kStages * kStageBytes + 1024;
    static_assert(MODE == kGated || MODE == kPair, "pair kernel modes");
    static_assert(kStages >= 4, "pipeline depth");
};

template <int MODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(CfgPair<MODE>::kThreads, 1)
    k_grouped_ffn_pair(const __grid_constant__ FfnArgs p) {
    using C = CfgPair<MODE>;
    extern __shared__ uint8_t dyn_smem[];
    __shared__ __align__(8) uint64_t full_bar[C::kStages], empty_bar[C::kStages];
    __shared__ __align__(8) uint64_t acc_full[2], acc_empty[2];
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_sh;
    __shared__ Tables tb;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();   // 0: the leader, which issues the MMAs
    const uint32_t stages = (smem_u32(dyn_smem) + 1023u) & ~1023u;   // same offset in both CTAs
    const int G = p.E + (p.has_shared ? 1 : 0);
    const int MT = p.M / C::kRowsPerTile;
    const int KB = p.K / kBK;
    volatile int* abort_flag = &abort_sh;

    if (threadIdx.x == 0) {
        abort_sh = 0;
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(smem_u32(&full_bar[s]), 1);    // the leader's: armed by the leader's producer
            mbar_init(smem_u32(&empty_bar[s]), 1);   // every CTA's: the leader's MMA commit
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(smem_u32(&acc_full[a]), 1);
            mbar_init(smem_u32(&acc_empty[a]), 2 * C::kEpiWarps);   // the leader's: both CTAs' epilogues
        }
        fence_mbar_init();
        tma_prefetch_map(&p.act_map);
        tma_prefetch_map(&p.act_map64);
        for (int m = 0; m < 3; ++m) tma_prefetch_map(MODE == kGated ? &p.w_map4[m] : &p.w_map[m]);
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_u32(&tmem_base_sh), C::kTmemCols);
        tmem_relinquish_pair();
    }
    if (warp == 2) build_tables<C::kBN, C::kAL>(p, tb, G, MT, lane);
    tc_fence_before();
    __syncthreads();
    cluster_sync();   // both CTAs' barriers initialised before any remote arrival
    tc_fence_after();
    const uint32_t tmem_base = tmem_base_sh;
    const int total = tb.tile_start[G];
    const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
    const uint32_t lead_full = mapa_shared(smem_u32(&full_bar[0]), 0);        // + 8 * stage
    const uint32_t lead_acc_empty = mapa_shared(smem_u32(&acc_empty[0]), 0);  // + 8 * buffer

    if (warp == 0) {
        // ------------------------------------------------ TMA producer (each CTA)
        if (lane == 0) {
            int stage = 0, passed = -1;
            uint32_t phase = 0;
            bool ok = true;
            for (int tile = pair; tile < total && ok; tile += n_pairs) {
                const Tile t = decode_tile<C::kBN, C::kRowsPerTile, C::kAL>(tile, tb, G);
                if (!gate_wait(p, t.map, t.slot, passed, abort_flag, p.err)) break;
                const int half = t.n_mma / 2;
                const uint32_t tx = 2u * (C::kAStage + (uint32_t)half * kBK * 2);   // both CTAs
                const int brow = t.row0 + (int)rank * half;
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait_cluster(smem_u32(&empty_bar[stage]), phase ^ 1u, abort_flag, p.err)) {
                        ok = false;
                        break;
                    }
                    const uint32_t sa = stages + stage * C::kStageBytes;
                    const uint32_t fb = lead_full + 8u * stage;
                    if (rank == 0) mbar_arrive_expect_tx(smem_u32(&full_bar[stage]), tx);
                    if constexpr (MODE == kGated) {
                        tma_load_4d_pair(sa, &p.w_map4[t.map], fb, kb * kBK, 0, t.m0 + 64 * (int)rank,
                                         t.slot);
                    } else {
                        tma_load_3d_pair(sa, &p.w_map[t.map], fb, kb * kBK, t.m0 + kBM * (int)rank,
                                         t.slot);
                    }
                    const uint32_t sb = sa + C::kAStage;
                    int r = 0;
                    for (; r + 64 <= half; r += 64)
                        tma_load_2d_pair(sb + r * kBK * 2, &p.act_map64, fb, kb * kBK, brow + r);
                    for (; r < half; r += kBoxN)
                        tma_load_2d_pair(sb + r * kBK * 2, &p.act_map, fb, kb * kBK, brow + r);
                    if (++stage == C::kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (leader only)
        if (rank == 0 && lane == 0) {
            int stage = 0, acc = 0;
            uint32_t phase = 0, acc_use[2] = {0u, 0u};
            bool ok = true;
            for (int tile = pair; tile < total && ok; tile += n_pairs) {
                const Tile t = decode_tile<C::kBN, C::kRowsPerTile, C::kAL>(tile, tb, G);
                // both CTAs' epilogues have drained this accumulator
                if (!mbar_wait_cluster(smem_u32(&acc_empty[acc]), (acc_use[acc] & 1u) ^ 1u, abort_flag,
                                       p.err))
                    break;
                tc_fence_after();
                const uint32_t d0 = tmem_base + acc * C::kAccCols;
                const uint32_t idesc = idesc_bf16_f32(2 * kBM, t.n_mma);
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait_cluster(smem_u32(&full_bar[stage]), phase, abort_flag, p.err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = stages + stage * C::kStageBytes;
                    const uint32_t sb = sa + C::kAStage;
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk)
                        mma_bf16_pair(d0, sw128_desc(sa + kk * 32), sw128_desc(sb + kk * 32), idesc,
                                      (kb | kk) != 0);
                    mma_commit_pair(smem_u32(&empty_bar[stage]), 0x3);
                    if (++stage == C::kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                mma_commit_pair(smem_u32(&acc_full[acc]), 0x3);
                ++acc_use[acc];
                acc ^= 1;
            }
        }
    } else {
        // ------------------------------------------------ epilogue (each CTA, its 128 rows)
        const int q = warp & 3;                 // TMEM lane quarter this warp may access
        const int part = (warp - 2) >> 2;       // which 128 token columns
        int acc = 0;
        uint32_t acc_use[2] = {0u, 0u};
        for (int tile = pair; tile < total; tile += n_pairs) {
            const Tile t = decode_tile<C::kBN, C::kRowsPerTile, C::kAL>(tile, tb, G);
            const bool ok = mbar_wait_cluster(smem_u32(&acc_full[acc]), acc_use[acc] & 1u, abort_flag,
                                              p.err);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            const uint32_t tacc = tmem_base + ((uint32_t)(32 * q) << 16) + acc * C::kAccCols;
            const int c_begin = part * (C::kBN / 2);
            const int c_end = min(t.n_rows, c_begin + C::kBN / 2);
            if constexpr (MODE == kGated) {
                // lane L holds row 32q + L: feature 16q + L/2 of this CTA, gate (L even) or up
                const int f = t.m0 + 64 * (int)rank + 16 * q + (lane >> 1);
                const bool up = lane & 1;
                __nv_bfloat16* out = p.out + f;
                for (int c0 = c_begin; c0 < c_end; c0 += 16) {
                    float v[16];
                    tmem_ld_16(tacc + c0, v);
                    tmem_ld_wait();
                    // even lanes finish tokens c0..c0+7, odd lanes c0+8..c0+15
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const float other = __shfl_xor_sync(0xffffffffu, up ? v[j] : v[8 + j], 1);
                        const float g = up ? other : v[j];
                        const float u = up ? v[8 + j] : other;
                        const int c = c0 + (up ? 8 : 0) + j;
                        if (c < t.n_rows)
                            out[(int64_t)(t.row0 + c) * p.ld_out] = __float2bfloat16_rn(silu_mul(g, u));
                    }
                }
            } else {
                const int f = t.m0 + kBM * (int)rank + 32 * q + lane;
                __nv_bfloat16* out = p.out + (int64_t)t.row0 * p.ld_out + f;
                for (int c0 = c_begin; c0 < c_end; c0 += 16) {
                    float v[16];
                    tmem_ld_16(tacc + c0, v);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        if (c0 + i < t.n_rows) out[(int64_t)(c0 + i) * p.ld_out] = __float2bfloat16_rn(v[i]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(lead_acc_empty + 8u * acc);
            ++acc_use[acc];
            acc ^= 1;
        }
    }

    __syncthreads();
    if (*abort_flag) {  // let copies still in flight land before TMEM is released
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 2000000ull) __nanosleep(1000);
    }
    tc_fence_before();
    cluster_sync();   // both CTAs finished with the shared TMEM and each other's barriers
    tc_fence_after();
    if (warp == 1) tmem_dealloc_pair(tmem_base, C::kTmemCols);
}

}  // namespace
}  // namespace swb
