// Shared by the grouped FFN kernels: kernel arguments, the tile schedule
// (per-expert token tiles, balanced and 16-aligned) and the SwiGLU helper.
#pragma once

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

}  // namespace
}  // namespace swb
