// Shared by the grouped FFN kernels: kernel arguments, the tile schedule
// (per-expert token tiles, balanced and 16-aligned) and the SwiGLU helper.
#pragma once

#include <climits>

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
constexpr uint32_t kSmemBudgetW8 = 208 * 1024; // both rings, e4m3 weights on bf16 MMAs

// Registers a call gated by readiness flags may take on each SM (one CTA per
// SM).  Its CTAs wait for a fetch; between two buffers of one GPU that fetch
// (cudaMemcpyAsync) runs as a copy kernel on the SMs, so the CTA must leave
// it room.  Measured on B200: a CTA holding 55,296 of the SM's 65,536
// registers left the copy running beside it; one holding 59,904 kept it from
// starting until the CTA ended, and the gated call's bounded wait ran out.
constexpr int64_t kGatedRegsPerSm = 55296;

struct alignas(64) FfnArgs {
    CUtensorMap w_map[3];      // 0 local pool, 1 remote pool, 2 shared expert: {K, rows, slot}
    CUtensorMap act_map;       // activation rows {K, rows}, 16-row box
    CUtensorMap act_map64;     // the same rows, 64-row box
    CUtensorMap x_map;         // gathered token tiles: x [T, K] bf16, 64 x 1 box (tile::gather4)
    const int32_t* offsets;    // [E+1] first row of each expert
    const int32_t* perm_src;   // [T*k] token of each permuted row (gather != 0)
    int32_t gather;            // token tiles read from x through perm_src, not from x_perm
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
    // readiness gate of the remote pool (NULL flags: none): the chunk of
    // slots_per_flag remote slots holding slot s has landed once
    // ready_flags[s / slots_per_flag] has reached ready_epoch
    const uint32_t* ready_flags;
    uint32_t ready_epoch;
    int32_t slots_per_flag;
    uint64_t ready_timeout_ns;
    // progress reports (NULL progress_word: none): when the d-th tile of this
    // launch has its MMAs issued (d counted in *progress_tiles), the word is
    // raised to progress_base + floor(d * progress_steps / tiles)
    uint32_t* progress_word;
    uint32_t* progress_tiles;
    uint32_t progress_base;
    int32_t progress_steps;
    // dynamic tile schedule (NULL: static round-robin): the launch's next tile
    // index, zeroed by the host before the launch
    int32_t* tile_counter;
    // tile enumeration order: position i holds group order[i] (local experts
    // and the shared one first, then the remote experts in slot order, the
    // order in which a fetch fills them)
    uint16_t order[kMaxGroups];
};

// passed by value as a __grid_constant__ kernel parameter (sm_70+ limit 32764 bytes)
static_assert(sizeof(FfnArgs) <= 32764, "FfnArgs exceeds the kernel parameter limit");

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
// AL: the MMA row granule of a tile (16; 32 when a CTA pair splits it in halves).
template <int BN, int AL = 16>
__device__ __host__ __forceinline__ int tile_rows(int n) {
    const int ntn = (n + BN - 1) / BN;
    const int per = (n + ntn - 1) / ntn;
    return (per + AL - 1) & ~(AL - 1);
}

template <int BN, int AL = 16>
__device__ __host__ __forceinline__ int token_tiles(int n) {
    if (n <= 0) return 0;
    const int tr = tile_rows<BN, AL>(n);
    return (n + tr - 1) / tr;
}

template <int BN, int ROWS, int AL = 16>
__device__ __forceinline__ Tile decode_tile(int tile, const Tables& tb, int G) {
    int lo = 0, hi = G - 1;
    while (lo < hi) {  // largest group whose first tile is <= tile (never an empty one)
        const int mid = (lo + hi + 1) >> 1;
        if (tb.tile_start[mid] <= tile) lo = mid;
        else hi = mid - 1;
    }
    const int g = lo, local = tile - tb.tile_start[g], n = tb.n[g];
    const int tr = tile_rows<BN, AL>(n);
    const int ntn = (n + tr - 1) / tr;
    const int mt = local / ntn, nt = local - mt * ntn;
    Tile t;
    t.m0 = mt * ROWS;
    t.row0 = tb.row0[g] + nt * tr;
    t.n_rows = min(tr, n - nt * tr);
    t.n_mma = (t.n_rows + AL - 1) & ~(AL - 1);
    t.map = tb.ps[g] >> 24;
    t.slot = tb.ps[g] & 0xFFFFFF;
    return t;
}

// One warp: per position (group p.order[i]) the first row, rows, tile count
// and (pool, slot), and the exclusive scan of tiles over the positions.
template <int BN, int AL = 16>
__device__ __forceinline__ void build_tables(const FfnArgs& p, Tables& tb, int G, int MT, int lane) {
    const int per = (G + 31) / 32, i0 = lane * per, i1 = min(G, i0 + per);
    int sum = 0;
    for (int i = i0; i < i1; ++i) {
        const int g = p.order[i];
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
        tb.row0[i] = r0;
        tb.n[i] = n;
        tb.ps[i] = ps;
        sum += token_tiles<BN, AL>(n) * MT;
    }
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    int run = incl - sum;
    for (int i = i0; i < i1; ++i) {
        tb.tile_start[i] = run;
        run += token_tiles<BN, AL>(tb.n[i]) * MT;
    }
    if (lane == 31) tb.tile_start[G] = incl;
}

// One look at the readiness flag of a remote slot, without waiting: true if
// the tile reads no fetch in flight, or its chunk has landed (then ordered
// like gate_wait).
__device__ __forceinline__ bool gate_ready(const FfnArgs& p, int map, int slot, int& passed) {
    if (p.ready_flags == nullptr || map != 1) return true;
    const int f = slot / p.slots_per_flag;
    if (f == passed) return true;
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p.ready_flags + f) : "memory");
    if ((int32_t)(v - p.ready_epoch) < 0) return false;
    asm volatile("fence.proxy.async.global;" ::: "memory");
    passed = f;
    return true;
}

// Per-expert readiness of a fetch still in flight: waits until the chunk of
// the remote pool that holds `slot` has landed (its flag, written by the copy
// stream after the chunk, has reached the epoch).  Only remote tiles of a
// gated call wait.  Every calling thread polls (acquire, GPU scope); the wait
// gives up after ready_timeout_ns: it raises *abort, sets the timeout bit of
// the device error word and returns false.  `passed` caches the last flag
// seen ready by this thread (flags only grow during a call).  On success the
// async proxy (TMA) is ordered after the acquire.
__device__ __forceinline__ bool gate_wait(const FfnArgs& p, int map, int slot, int& passed,
                                          volatile int* abort, int* err) {
    if (p.ready_flags == nullptr || map != 1) return true;
    const int f = slot / p.slots_per_flag;
    if (f == passed) return true;
    const uint32_t* flag = p.ready_flags + f;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        uint32_t v;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
        if ((int32_t)(v - p.ready_epoch) >= 0) break;
        if (*abort) return false;
        if (globaltimer_ns() - t0 > p.ready_timeout_ns) {
            *abort = 1;
            atomicOr(err, kDevErrTimeout);
            return false;
        }
        __nanosleep(200);
    }
    asm volatile("fence.proxy.async.global;" ::: "memory");
    passed = f;
    return true;
}

// One more tile of this launch has its MMAs issued (called once per tile by
// the MMA thread): count it, and when it completes a new step raise the
// progress word to progress_base + step, a maximum in wrap-around order so
// that a CTA that reports late never lowers it.
__device__ __forceinline__ void report_progress(const FfnArgs& p, int total) {
    if (!p.progress_word) return;
    const uint64_t d = atomicAdd(p.progress_tiles, 1u) + 1ull;
    const uint64_t steps = (uint64_t)p.progress_steps;
    const uint32_t s = (uint32_t)(d * steps / (uint64_t)total);
    if (s == (uint32_t)((d - 1) * steps / (uint64_t)total)) return;
    const uint32_t v = p.progress_base + s;
    uint32_t cur = *reinterpret_cast<volatile uint32_t*>(p.progress_word);
    while ((int32_t)(v - cur) > 0) {
        const uint32_t old = atomicCAS(p.progress_word, cur, v);
        if (old == cur) break;
        cur = old;
    }
}

// The tiles of one CTA, in the order all its roles take them.  Static
// (tile_counter NULL): blockIdx.x, + gridDim.x, ...  Dynamic: the producer
// takes the launch's next tile from a global counter whenever it is ready
// for one, so a CTA that drew small tiles takes more of them, and hands each
// index to the other roles through a ring in shared memory; an index >= the
// tile count (or an abort) ends every role.
constexpr int kTileRing = 4;
// workspace bytes the bf16-activation call uses for its two tile counters
constexpr size_t kTileCounterBytes = 256;

struct TileQueue {
    int id[kTileRing];
    uint64_t full[kTileRing];    // one arrival: the producer wrote id[s]
    uint64_t empty[kTileRing];   // one arrival per consumer role (warp or thread)
};

__device__ __forceinline__ int tile_produce(const FfnArgs& p, TileQueue& q, int it,
                                            volatile int* abort, int* err) {
    if (!p.tile_counter) return (int)blockIdx.x + it * (int)gridDim.x;
    const int s = it % kTileRing;
    const uint32_t ph = (uint32_t)(it / kTileRing) & 1u;
    if (!mbar_wait(smem_u32(&q.empty[s]), ph ^ 1u, abort, err)) return INT_MAX;
    const int t = *abort ? INT_MAX : atomicAdd(p.tile_counter, 1);
    *reinterpret_cast<volatile int*>(&q.id[s]) = t;
    mbar_arrive(smem_u32(&q.full[s]));
    return t;
}

// Every thread of a consumer role reads the index; then one thread per role
// calls tile_release for the same `it`.
__device__ __forceinline__ int tile_consume(const FfnArgs& p, TileQueue& q, int it,
                                            volatile int* abort, int* err) {
    if (!p.tile_counter) return (int)blockIdx.x + it * (int)gridDim.x;
    const int s = it % kTileRing;
    const uint32_t ph = (uint32_t)(it / kTileRing) & 1u;
    if (!mbar_wait(smem_u32(&q.full[s]), ph, abort, err)) return INT_MAX;
    return *reinterpret_cast<volatile int*>(&q.id[s]);
}

__device__ __forceinline__ void tile_release(const FfnArgs& p, TileQueue& q, int it) {
    if (p.tile_counter) mbar_arrive(smem_u32(&q.empty[it % kTileRing]));
}

// Two fp32 values rounded to bf16 (round to nearest even), lo in bits 0-15.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&b);
}

// silu(g) * u = g / (1 + e^-g) * u with the fast exponential and division
// (a few ulp in fp32; h is rounded to bf16 or e4m3 right after).  For
// g < -87, 1 + e^-g exceeds 2^126 and __fdividef gives 0, which is silu(g)
// rounded to any output format.
__device__ __forceinline__ float silu_mul(float g, float u) {
    return __fdividef(g, 1.0f + __expf(-g)) * u;
}

}  // namespace
}  // namespace swb
