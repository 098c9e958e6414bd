// The bf16 tensor-core grouped FFN kernel (kind::f16), with bf16 weights or
// with e4m3 weights that converter warps dequantise into bf16 operand
// buffers of their own.
#pragma once

#include "ffn_common.cuh"

namespace swb {
namespace {

constexpr int kConvThreads = 256;              // e4m3 -> bf16 converter warps (8)

// bf16 weights: one ring of stages, each the bf16 weight tile(s) the MMA
// reads (128-byte swizzled) and the token tile.  e4m3 weights: a TMA ring of
// {token tile, e4m3 staging tile(s)} and a ring of kStagesY converted bf16
// weight operands, so that the token tile of a 256-token tile and three TMA
// stages fit beside the two operand buffers the converters and the MMA
// alternate on.
template <int BN, int MODE, bool W8>
struct Cfg {
    static constexpr int kNA = MODE == kSingle ? 1 : 2;           // weight tiles per stage
    static constexpr int kBKs = kBK;                              // K per stage
    static constexpr uint32_t kATile = kBM * kBKs * 2;            // one bf16 weight tile
    static constexpr uint32_t kA8Tile = kBM * kBKs;               // one e4m3 tile as loaded
    static constexpr uint32_t kAStage = kATile * kNA;
    static constexpr uint32_t kBStage = BN * kBKs * 2;
    static constexpr uint32_t kA8Stage = W8 ? kA8Tile * kNA : 0;
    static constexpr int kStagesY = W8 ? 2 : 0;                   // converted operand buffers
    // offsets within a TMA stage: bf16 weights | tokens, or tokens | e4m3 codes
    static constexpr uint32_t kTokOff = W8 ? 0 : kAStage;
    static constexpr uint32_t kCodeOff = kBStage;
    static constexpr uint32_t kStageBytes = W8 ? kBStage + kA8Stage : kAStage + kBStage;
    static constexpr uint32_t kRingBudget = W8 ? kSmemBudgetW8 - kStagesY * kAStage : kSmemBudget;
    static constexpr int kStages = (kRingBudget / kStageBytes) > 12 ? 12 : (kRingBudget / kStageBytes);
    static constexpr uint32_t kYOff = kStages * kStageBytes;      // the operand ring, after the TMA ring
    static constexpr uint32_t kAccCols = kNA * BN;                // one accumulator set
    static constexpr int kAccBufs = 2 * kAccCols <= 512 ? 2 : 1;
    static constexpr uint32_t kTmemCols = kAccBufs * kAccCols;
    // one TMEM buffer at BN=256: its epilogue stalls the MMA, so it gets 16
    // warps (8 beside the e4m3 converters, within the threads' register room)
    static constexpr int kEpiWarps = BN >= 256 ? (W8 ? 8 : 16) : 4;
    static constexpr int kConvWarps = W8 ? kConvThreads / 32 : 0;
    static constexpr int kConvFirstWarp = 2 + kEpiWarps;
    static constexpr int kThreads = 64 + 32 * (kEpiWarps + kConvWarps);
    static constexpr int kRowsPerTile = MODE == kPair ? 2 * kBM : kBM;  // output features
    static constexpr size_t kDynSmem = (size_t)kStages * kStageBytes + kStagesY * kAStage + 1024;
    static_assert(kTmemCols >= 32 && kTmemCols <= 512 && (kTmemCols & (kTmemCols - 1)) == 0,
                  "TMEM allocation must be a power of two in [32, 512]");
    static_assert(kStages >= (W8 ? 3 : 2), "pipeline needs two stages (three beside the converters)");
    static_assert(kStageBytes % 1024 == 0 && kAStage % 1024 == 0, "operand tiles sit on 1024-byte swizzle atoms");
};
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
    __shared__ __align__(8) uint64_t conv_bar[W8 ? C::kStagesY : 1];  // operand buffer converted
    __shared__ __align__(8) uint64_t yempty_bar[W8 ? C::kStagesY : 1]; // operand buffer read by the MMAs
    __shared__ __align__(8) uint64_t acc_full[2], acc_empty[2];
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_sh;
    __shared__ Tables tb;
    __shared__ TileQueue tq;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t stages = (smem_u32(dyn_smem) + 1023u) & ~1023u;
    const int G = p.E + (p.has_shared ? 1 : 0);
    const int MT = p.M / C::kRowsPerTile;
    const int KB = p.K / C::kBKs;
    volatile int* abort_flag = &abort_sh;

    if (threadIdx.x == 0) {
        abort_sh = 0;
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(smem_u32(&full_bar[s]), 1);
            mbar_init(smem_u32(&empty_bar[s]), 1);
        }
        for (int y = 0; y < C::kStagesY; ++y) {
            mbar_init(smem_u32(&conv_bar[y]), C::kConvWarps);
            mbar_init(smem_u32(&yempty_bar[y]), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(smem_u32(&acc_full[a]), 1);
            mbar_init(smem_u32(&acc_empty[a]), C::kEpiWarps);
        }
        for (int q = 0; q < kTileRing; ++q) {   // consumers: MMA thread, epilogue and converter warps
            mbar_init(smem_u32(&tq.full[q]), 1);
            mbar_init(smem_u32(&tq.empty[q]), 1 + C::kEpiWarps + C::kConvWarps);
        }
        fence_mbar_init();
        if (p.gather) {
            tma_prefetch_map(&p.x_map);
        } else {
            tma_prefetch_map(&p.act_map);
            tma_prefetch_map(&p.act_map64);
        }
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

    if (warp == 0 && !p.gather) {
        // ------------------------------------------------ TMA producer (one thread)
        // weight tile(s) and the token tile from x_perm in 64- and 16-row boxes
        if (lane == 0) {
            int stage = 0, passed = -1;
            uint32_t phase = 0;
            bool ok = true;
            for (int it = 0; ok; ++it) {
                const int tile = tile_produce(p, tq, it, abort_flag, p.err);
                if (tile >= total) break;
                const Tile t = decode_tile<BN, C::kRowsPerTile>(tile, tb, G);
                if (!gate_wait(p, t.map, t.slot, passed, abort_flag, p.err)) break;
                const CUtensorMap* wm = &p.w_map[t.map];
                const uint32_t tx = (W8 ? C::kA8Stage : C::kAStage) + (uint32_t)t.n_mma * C::kBKs * 2;
                const int row_a1 = MODE == kGated ? p.up_row + t.m0 : t.m0 + kBM;
                for (int kb = 0; kb < KB; ++kb) {
                    const uint32_t fb = smem_u32(&full_bar[stage]);
                    if (!mbar_wait(smem_u32(&empty_bar[stage]), phase ^ 1u, abort_flag, p.err)) {
                        ok = false;
                        break;
                    }
                    const uint32_t sa = stages + stage * C::kStageBytes;
                    mbar_arrive_expect_tx(fb, tx);
                    // e4m3 weights land in the staging area, bf16 ones straight in the operand
                    const uint32_t sw = W8 ? sa + C::kCodeOff : sa;
                    const uint32_t w_step = W8 ? C::kA8Tile : C::kATile;
                    tma_load_3d(sw, wm, fb, kb * C::kBKs, t.m0, t.slot);
                    if constexpr (C::kNA == 2) tma_load_3d(sw + w_step, wm, fb, kb * C::kBKs, row_a1, t.slot);
                    const uint32_t sb = sa + C::kTokOff;
                    int r = 0;
                    for (; r + 64 <= t.n_mma; r += 64)
                        tma_load_2d(sb + r * C::kBKs * 2, &p.act_map64, fb, kb * C::kBKs, t.row0 + r);
                    for (; r < t.n_mma; r += kBoxN)
                        tma_load_2d(sb + r * C::kBKs * 2, &p.act_map, fb, kb * C::kBKs, t.row0 + r);
                    if (++stage == C::kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
        }
    } else if (warp == 0) {
        // ------------------------------------------------ TMA producer (gathered token rows)
        // Lane 0 arms each stage and loads the weight tile(s); the token tile
        // comes straight from x through perm_src: four rows per
        // tile::gather4 load, lane i loading rows 4i..4i+3 and 128+4i..131+4i.
        // Rows past the tile's tokens repeat its last token (their products
        // are never stored).
        int stage = 0, passed = -1;
        uint32_t phase = 0;
        bool ok = true;
        for (int it = 0; ok; ++it) {
            int tile = 0;
            if (lane == 0) tile = tile_produce(p, tq, it, abort_flag, p.err);
            tile = __shfl_sync(0xffffffffu, tile, 0);
            if (tile >= total) break;
            const Tile t = decode_tile<BN, C::kRowsPerTile>(tile, tb, G);
            if (!__all_sync(0xffffffffu, lane != 0 || gate_wait(p, t.map, t.slot, passed, abort_flag, p.err)))
                break;
            const CUtensorMap* wm = &p.w_map[t.map];
            const uint32_t tx = (W8 ? C::kA8Stage : C::kAStage) + (uint32_t)t.n_mma * C::kBKs * 2;
            const int row_a1 = MODE == kGated ? p.up_row + t.m0 : t.m0 + kBM;
            int tok[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int r = (j >> 2) * 128 + 4 * lane + (j & 3);
                const int rr = min(r, t.n_rows - 1);
                int v = 0;
                if (r < t.n_mma) {
                    // the shared expert's rows are the tokens in order
                    v = t.map == 2 ? t.row0 + rr - p.A : __ldg(p.perm_src + t.row0 + rr);
                    if (v < 0 || v >= p.T) {   // not a token: report, read token 0
                        atomicOr(p.err, kDevErrIndex);
                        v = 0;
                    }
                }
                tok[j] = v;
            }
            for (int kb = 0; kb < KB; ++kb) {
                const uint32_t eb = smem_u32(&empty_bar[stage]);
                const uint32_t fb = smem_u32(&full_bar[stage]);
                bool w = true;
                if (lane == 0) w = mbar_wait(eb, phase ^ 1u, abort_flag, p.err);
                if (!__shfl_sync(0xffffffffu, w, 0)) {
                    ok = false;
                    break;
                }
                const uint32_t sa = stages + stage * C::kStageBytes;
                const uint32_t sb = sa + C::kTokOff;
                if (lane == 0) {
                    mbar_arrive_expect_tx(fb, tx);
                    const uint32_t sw = W8 ? sa + C::kCodeOff : sa;
                    const uint32_t w_step = W8 ? C::kA8Tile : C::kATile;
                    tma_load_3d(sw, wm, fb, kb * C::kBKs, t.m0, t.slot);
                    if constexpr (C::kNA == 2) tma_load_3d(sw + w_step, wm, fb, kb * C::kBKs, row_a1, t.slot);
                }
                __syncwarp();
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int r0 = h * 128 + 4 * lane;
                    if (r0 < t.n_mma)
                        tma_gather4(sb + r0 * C::kBKs * 2, &p.x_map, fb, kb * C::kBKs, tok[4 * h],
                                    tok[4 * h + 1], tok[4 * h + 2], tok[4 * h + 3]);
                }
                if (++stage == C::kStages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            int stage = 0, acc = 0, ys = 0;
            uint32_t phase = 0, yphase = 0, acc_use[2] = {0u, 0u};
            bool ok = true;
            for (int it = 0; ok; ++it) {
                const int tile = tile_consume(p, tq, it, abort_flag, p.err);
                if (tile >= total) break;
                tile_release(p, tq, it);
                const Tile t = decode_tile<BN, C::kRowsPerTile>(tile, tb, G);
                if (!mbar_wait(smem_u32(&acc_empty[acc]), (acc_use[acc] & 1u) ^ 1u, abort_flag,
                               p.err))
                    break;
                tc_fence_after();
                const uint32_t d0 = tmem_base + acc * C::kAccCols;
                const uint32_t idesc = idesc_bf16_f32(kBM, t.n_mma);
                for (int kb = 0; kb < KB; ++kb) {
                    // e4m3 weights: the converters have filled operand buffer ys
                    // (after this stage's TMA landed)
                    if (W8 && !mbar_wait(smem_u32(&conv_bar[ys]), yphase, abort_flag, p.err)) {
                        ok = false;
                        break;
                    }
                    if (!mbar_wait(smem_u32(&full_bar[stage]), phase, abort_flag, p.err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sb = stages + stage * C::kStageBytes + C::kTokOff;
                    const uint32_t sa = W8 ? stages + C::kYOff + ys * C::kAStage
                                           : stages + stage * C::kStageBytes;
#pragma unroll
                    for (int kk = 0; kk < C::kBKs / 16; ++kk) {
                        const uint32_t accum = (kb | kk) != 0;
                        const uint64_t bd = sw128_desc(sb + kk * 32);
                        const uint32_t a0 = sa + kk * 32, a1 = a0 + C::kATile;
                        mma_bf16_ss(d0, sw128_desc(a0), bd, idesc, accum);
                        if constexpr (C::kNA == 2)
                            mma_bf16_ss(d0 + BN, sw128_desc(a1), bd, idesc, accum);
                    }
                    mma_commit(smem_u32(&empty_bar[stage]));
                    if constexpr (W8) {
                        mma_commit(smem_u32(&yempty_bar[ys]));
                        if (++ys == C::kStagesY) {
                            ys = 0;
                            yphase ^= 1u;
                        }
                    }
                    if (++stage == C::kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                mma_commit(smem_u32(&acc_full[acc]));
                report_progress(p, total);
                ++acc_use[acc];
                if (C::kAccBufs == 2) acc ^= 1;
            }
        }
    } else if (W8 && warp >= C::kConvFirstWarp) {
        // ------------------------------------------------ e4m3 -> bf16 converters
        // Each staged row is kBKs e4m3 bytes (chunks of 16); the bf16 operand
        // row is 2 kBKs bytes in the matching swizzle.  One 128x128 block scale
        // covers the whole stage (kBKs columns of K, 128 rows).
        const int ct = threadIdx.x - 32 * C::kConvFirstWarp;  // 0 .. kConvThreads-1
        int stage = 0, ys = 0, passed = -1;
        uint32_t phase = 0, yphase = 0;
        bool ok = true;
        for (int it = 0; ok; ++it) {
            const int tile = tile_consume(p, tq, it, abort_flag, p.err);
            if (tile >= total) break;
            __syncwarp();
            if (lane == 0) tile_release(p, tq, it);
            const Tile t = decode_tile<BN, C::kRowsPerTile>(tile, tb, G);
            // the block scales sit in the remote buffer too: read them only once
            // landed, and L2-coherently while a gated fetch may be writing other slots
            if (!__all_sync(0xffffffffu, gate_wait(p, t.map, t.slot, passed, abort_flag, p.err))) break;
            const uint8_t* sbase = p.w_base[t.map] + (int64_t)t.slot * p.w_stride[t.map] + p.scale_off;
            const float* sc0 = reinterpret_cast<const float*>(sbase) + (int64_t)(t.m0 / kBM) * p.kblocks;
            const int rb1 = MODE == kGated ? (p.up_row + t.m0) / kBM : t.m0 / kBM + 1;
            const float* sc1 = reinterpret_cast<const float*>(sbase) + (int64_t)rb1 * p.kblocks;
            // the block scale of the stage's 128-wide K block: L1-cached loads,
            // unless a gated fetch may still be writing the buffer
            auto scale = [&](const float* sc, int kb) {
                const int sblk = (kb * C::kBKs) >> 7;
                return p.ready_flags ? __ldcg(sc + sblk) : __ldg(sc + sblk);
            };
            // loaded one stage ahead, so that converting a stage never waits on them
            float s0n = scale(sc0, 0), s1n = C::kNA == 2 ? scale(sc1, 0) : 0.0f;
            for (int kb = 0; kb < KB; ++kb) {
                const float s0 = s0n, s1 = s1n;
                if (kb + 1 < KB) {
                    s0n = scale(sc0, kb + 1);
                    if constexpr (C::kNA == 2) s1n = scale(sc1, kb + 1);
                }
                // the stage's codes have landed, and the MMAs are done with the
                // operand buffer's previous contents
                ok = mbar_wait(smem_u32(&full_bar[stage]), phase, abort_flag, p.err) &&
                     mbar_wait(smem_u32(&yempty_bar[ys]), yphase ^ 1u, abort_flag, p.err);
                if (!__all_sync(0xffffffffu, ok)) {
                    ok = false;
                    break;
                }
                const uint32_t sa = stages + C::kYOff + ys * C::kAStage;
                const uint32_t s8 = stages + stage * C::kStageBytes + C::kCodeOff;
#pragma unroll
                for (int a = 0; a < C::kNA; ++a) {
                    const float sc = a == 0 ? s0 : s1;
#pragma unroll
                    for (int i = 0; i < (kBM * C::kBKs / 16) / kConvThreads; ++i) {
                        constexpr int kCh = C::kBKs / 16;   // 16-code chunks of a staged row
                        const int id = ct + kConvThreads * i, r = id / kCh, c = id % kCh;
                        uint4 in, lo, hi;
                        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                                     : "=r"(in.x), "=r"(in.y), "=r"(in.z), "=r"(in.w)
                                     : "r"(s8 + a * C::kA8Tile + r * C::kBKs + c * 16));
                        e4m3x16_to_bf16(in, sc, lo, hi);
                        // the operand row r (kBKs * 2 bytes): 16-byte chunk j at
                        // j ^ (r % 8) (128-byte swizzle)
                        const uint32_t row = sa + a * C::kATile + r * (C::kBKs * 2);
                        const uint32_t sw = r & 7;
                        const uint32_t j0 = (2 * c) ^ sw, j1 = (2 * c + 1) ^ sw;
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
                if (lane == 0) mbar_arrive(smem_u32(&conv_bar[ys]));
                if (++ys == C::kStagesY) {
                    ys = 0;
                    yphase ^= 1u;
                }
                if (++stage == C::kStages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
    } else {
        // ------------------------------------------------ epilogue
        const int q = warp & 3;                    // TMEM lane quarter this warp may access
        const int part = (warp - 2) >> 2;          // column slice of this warp's lane quarter
        constexpr int kCols = BN / (C::kEpiWarps / 4);
        int acc = 0;
        uint32_t acc_use[2] = {0u, 0u};
        for (int it = 0;; ++it) {
            const int tile = tile_consume(p, tq, it, abort_flag, p.err);
            if (tile >= total) break;
            __syncwarp();
            if (lane == 0) tile_release(p, tq, it);
            const Tile t = decode_tile<BN, C::kRowsPerTile>(tile, tb, G);
            bool ok = mbar_wait(smem_u32(&acc_full[acc]), acc_use[acc] & 1u, abort_flag, p.err);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            const uint32_t tacc = tmem_base + ((uint32_t)(32 * q) << 16) + acc * C::kAccCols;
            const int f = t.m0 + 32 * q + lane;
            __nv_bfloat16* out = p.out + (int64_t)t.row0 * p.ld_out + f;
            const int c_begin = part * kCols, c_end = min(t.n_rows, c_begin + kCols);
            constexpr int kChunks = kCols / 16;
            constexpr int kOut = (C::kNA == 2 && MODE != kGated) ? 2 : 1;
            if constexpr (C::kAccBufs == 1 && (!W8 || MODE == kGated)) {
                // One accumulator set: the next tile's MMAs wait for it.  Pull this
                // warp's columns out of TMEM into packed bf16 registers (at most 64),
                // free the accumulator, then store while the MMAs run.  With e4m3
                // weights (8 epilogue warps, 128 columns each) only the gate/up
                // launch does so: the paired down launch would hold 128.
                uint32_t pk[kChunks][kOut][8];
#pragma unroll
                for (int ch = 0; ch < kChunks; ++ch) {
                    const int c0 = c_begin + 16 * ch;
                    if (c0 >= c_end) break;   // warp-uniform
                    float g[16];
                    tmem_ld_16(tacc + c0, g);
                    if constexpr (C::kNA == 2) {
                        float u[16];
                        tmem_ld_16(tacc + BN + c0, u);
                        tmem_ld_wait();
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            if constexpr (MODE == kGated) {
                                pk[ch][0][i] = pack_bf16x2(silu_mul(g[2 * i], u[2 * i]),
                                                           silu_mul(g[2 * i + 1], u[2 * i + 1]));
                            } else {
                                pk[ch][0][i] = pack_bf16x2(g[2 * i], g[2 * i + 1]);
                                pk[ch][kOut - 1][i] = pack_bf16x2(u[2 * i], u[2 * i + 1]);
                            }
                        }
                    } else {
                        tmem_ld_wait();
#pragma unroll
                        for (int i = 0; i < 8; ++i) pk[ch][0][i] = pack_bf16x2(g[2 * i], g[2 * i + 1]);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&acc_empty[acc]));
                uint16_t* out16 = reinterpret_cast<uint16_t*>(out);
#pragma unroll
                for (int ch = 0; ch < kChunks; ++ch) {
                    const int c0 = c_begin + 16 * ch;
                    if (c0 >= c_end) break;
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        if (c0 + i >= t.n_rows) break;
                        uint16_t* o = out16 + (int64_t)(c0 + i) * p.ld_out;
                        const int sh = 16 * (i & 1);
                        o[0] = (uint16_t)(pk[ch][0][i >> 1] >> sh);
                        if constexpr (kOut == 2) o[kBM] = (uint16_t)(pk[ch][1][i >> 1] >> sh);
                    }
                }
            } else {
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
            }
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

}  // namespace
}  // namespace swb
