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
//   warps 2..   epilogue (4, 8 or 16 warps): TMEM -> registers -> (SwiGLU) -> bf16
//   then        e4m3 weights only: 8 converter warps, staged e4m3 codes x block
//               scale -> the bf16 operand buffers the MMA reads
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
// TMEM columns in one buffer and 16 epilogue warps, so the epilogue that
// holds up the next tile's MMA is short.
#include <atomic>

#include "ffn_bf16.cuh"
#include "ffn_f8.cuh"

namespace swb {
namespace {

// ---------------------------------------------------------------- host side
// A call gated by readiness flags keeps its CTAs waiting for a fetch that may
// run as a copy kernel on the same SMs: refuse a kernel whose CTA would leave
// it less room than measured to work (kGatedRegsPerSm), rather than let the
// gate's wait run out.
// regs: the kernel's register count once looked up (-1 before), one per kernel.
template <typename Kern>
moe_status check_gated_room(const FfnArgs& a, Kern kern, std::atomic<int>& regs, int threads,
                            const char* what) {
    if (!a.ready_flags) return MOE_OK;
    int r = regs.load(std::memory_order_relaxed);
    if (r < 0) {
        cudaFuncAttributes fa;
        SWB_CUDA(cudaFuncGetAttributes(&fa, kern));
        r = fa.numRegs;
        regs.store(r, std::memory_order_relaxed);
    }
    const int64_t limit = gated_regs_override() > 0 ? gated_regs_override() : kGatedRegsPerSm;
    if ((int64_t)r * threads > limit)
        return fail(MOE_ERR_CUDA, "%s: %d registers x %d threads leave a gated fetch's copy no room",
                    what, r, threads);
    return MOE_OK;
}

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
    static std::atomic<int> regs{-1};
    if ((st = check_gated_room(a, kern, regs, C::kThreads, "moe_grouped_ffn")) != MOE_OK) return st;
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
    static std::atomic<int> regs{-1};
    if ((st = check_gated_room(a, kern, regs, C::kThreads, "moe_grouped_ffn (fp8)")) != MOE_OK) return st;
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

// Token tile from the mean tokens per routed expert, 16..256.  e4m3 weights
// are converted once per token tile, so they move to 256-token tiles sooner:
// routing skew leaves the experts a token picks with more than the mean, and
// a 256-token tile converts an expert's weights once where 128-token tiles
// convert them twice.
int pick_bn(int64_t A, int E, bool w8 = false) {
    const int64_t mean = (A + E - 1) / E;
    if (mean <= 8) return 16;
    if (mean <= 16) return 32;
    if (mean <= 32) return 64;
    if (mean <= (w8 ? 96 : 160)) return 128;
    return 256;
}

// 3-D map {K, rows, slot} over one pool of expert images.  bf16 weights are
// loaded straight into the MMA operand layout (64-wide boxes: 128-byte rows
// and swizzle); e4m3 weights as plain 64-byte rows for the converter warps.
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

// bf16 rows {K, rows}: boxes of 64 (128-byte swizzle) x box_rows.
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
// Progress fields of launch `which` (0 gate/up, 1 down) of a call that
// reports to `pr` (NULL: none): the gate/up launch covers steps
// 1 .. round(2 steps / 3), about its share of the FLOPs, the down launch the rest.
void set_progress(FfnArgs& a, const moe_progress* pr, int which) {
    if (!pr) {
        a.progress_word = nullptr;
        return;
    }
    const int s1 = (2 * pr->steps + 1) / 3;
    a.progress_word = pr->word;
    a.progress_tiles = pr->tiles + which;
    a.progress_base = pr->base + (which ? (uint32_t)s1 : 0u);
    a.progress_steps = which ? pr->steps - s1 : s1;
}

moe_status ffn_f8(const moe_ffn_desc* d, const moe_expert_table* tbl, const moe_expert_layout& lay,
                  const void* x_perm, const float* x_scales, void* h, void* y_perm, float* h_scales,
                  int rows, int G, FfnArgs& a, const moe_progress* progress, cudaStream_t stream) {
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
    set_progress(a, progress, 0);
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
    set_progress(a, progress, 1);
    return launch_f8_bn<kPair>(bn, a, rows, G, stream);
}

moe_status ffn_run(const moe_ffn_desc* d, const moe_expert_table* tbl, const moe_ready_gate* gate,
                   const moe_progress* progress, const void* x_perm, const float* x_perm_scales,
                   const int32_t* perm_src, const int32_t* offsets, void* h, void* y_perm,
                   void* workspace, size_t workspace_bytes, cudaStream_t stream);

}  // namespace
}  // namespace swb

using namespace swb;

extern "C" {

size_t moe_grouped_ffn_workspace_size(const moe_ffn_desc* d) {
    if (!d) return 0;
    // bf16 activations: the two launches' tile counters (dynamic tile schedule)
    if (d->act_dtype != MOE_E4M3) return kTileCounterBytes;
    // e4m3 activations: the fp32 scales of the e4m3 intermediate h, [I/128][rows]
    if (d->T <= 0 || d->k <= 0 || d->I <= 0) return 0;
    const int64_t rows = (int64_t)d->T * d->k + (d->has_shared ? d->T : 0);
    return (size_t)((d->I / 128) * rows * 4 + 255) / 256 * 256;
}

moe_status moe_grouped_ffn(const moe_ffn_desc* d, const moe_expert_table* tbl, const void* x_perm,
                           const float* x_perm_scales, const int32_t* offsets, void* h,
                           void* y_perm, void* workspace, size_t workspace_bytes,
                           cudaStream_t stream) {
    return moe_grouped_ffn_gated(d, tbl, nullptr, x_perm, x_perm_scales, offsets, h, y_perm,
                                 workspace, workspace_bytes, stream);
}

moe_status moe_grouped_ffn_gated(const moe_ffn_desc* d, const moe_expert_table* tbl,
                                 const moe_ready_gate* gate, const void* x_perm,
                                 const float* x_perm_scales, const int32_t* offsets, void* h,
                                 void* y_perm, void* workspace, size_t workspace_bytes,
                                 cudaStream_t stream) {
    return ffn_run(d, tbl, gate, nullptr, x_perm, x_perm_scales, nullptr, offsets, h, y_perm,
                   workspace, workspace_bytes, stream);
}

moe_status moe_grouped_ffn_x(const moe_ffn_desc* d, const moe_expert_table* tbl,
                             const moe_ready_gate* gate, const void* x, const int32_t* perm_src,
                             const int32_t* offsets, void* h, void* y_perm, void* workspace,
                             size_t workspace_bytes, cudaStream_t stream) {
    if (d && d->act_dtype != MOE_BF16)
        return fail(MOE_ERR_UNSUPPORTED, "moe_grouped_ffn_x: activations must be bf16 (dtype %d)",
                    d->act_dtype);
    if (d && d->T > 0 && (!perm_src || !aligned(perm_src, 16)))
        return fail(MOE_ERR_INVALID_ARG, "moe_grouped_ffn_x: perm_src NULL or not 16-byte aligned");
    return ffn_run(d, tbl, gate, nullptr, x, nullptr, perm_src, offsets, h, y_perm, workspace,
                   workspace_bytes, stream);
}

moe_status moe_grouped_ffn_paced(const moe_ffn_desc* d, const moe_expert_table* tbl,
                                 const moe_ready_gate* gate, const moe_progress* progress,
                                 const void* x_perm, const float* x_perm_scales, const void* x,
                                 const int32_t* perm_src, const int32_t* offsets, void* h,
                                 void* y_perm, void* workspace, size_t workspace_bytes,
                                 cudaStream_t stream) {
    if (!progress || !progress->word || !progress->tiles || !aligned(progress->word, 4) ||
        !aligned(progress->tiles, 4) || progress->steps < 2)
        return fail(MOE_ERR_INVALID_ARG, "moe_grouped_ffn_paced: progress needs word and tiles "
                    "(4-byte aligned) and steps >= 2");
    const bool gather = x && perm_src;
    moe_status st;
    if (gather && d && d->act_dtype != MOE_BF16)
        st = fail(MOE_ERR_UNSUPPORTED, "moe_grouped_ffn_paced: gathered rows need bf16 "
                  "activations (dtype %d)", d->act_dtype);
    else if (gather && d && d->T > 0 && !aligned(perm_src, 16))
        st = fail(MOE_ERR_INVALID_ARG, "moe_grouped_ffn_paced: perm_src not 16-byte aligned");
    else
        st = ffn_run(d, tbl, gate, progress, gather ? x : x_perm, x_perm_scales,
                     gather ? perm_src : nullptr, offsets, h, y_perm, workspace, workspace_bytes,
                     stream);
    // the call's end, done or not: releases every chunk paced by it
    const moe_status fin = stream_write_u32(stream, progress->word,
                                            progress->base + (uint32_t)progress->steps + 1u);
    return st != MOE_OK ? st : fin;
}

}  // extern "C"

namespace swb {
namespace {

// The grouped FFN behind both entry points: the token tiles of GEMM1 come from
// `act` = x_perm (perm_src NULL) or from `act` = x through perm_src.
moe_status ffn_run(const moe_ffn_desc* d, const moe_expert_table* tbl, const moe_ready_gate* gate,
                   const moe_progress* progress, const void* x_perm, const float* x_perm_scales,
                   const int32_t* perm_src, const int32_t* offsets, void* h, void* y_perm,
                   void* workspace, size_t workspace_bytes, cudaStream_t stream) {
    moe_expert_layout lay;
    moe_status st = validate(d, tbl, &lay);
    if (st != MOE_OK) return st;
    if (gate) {
        if (!gate->flags || !aligned(gate->flags, 4) || gate->slots_per_flag <= 0 ||
            gate->timeout_ns < 0)
            return fail(MOE_ERR_INVALID_ARG, "moe_grouped_ffn_gated: gate needs flags (4-byte "
                        "aligned), slots_per_flag > 0 and timeout_ns >= 0");
        if (gate->n_flags < (tbl->remote_count + gate->slots_per_flag - 1) / gate->slots_per_flag)
            return fail(MOE_ERR_INVALID_ARG, "moe_grouped_ffn_gated: %d flags cannot cover %d "
                        "remote slots at %d per flag", gate->n_flags, tbl->remote_count,
                        gate->slots_per_flag);
    }
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
    // tile order: local experts by slot, the shared expert, remote experts by
    // slot (the order a fetch fills the remote buffer in)
    {
        static thread_local int32_t by_slot[2][kMaxGroups];
        for (int q = 0; q < 2; ++q)
            for (int i = 0; i < kMaxGroups; ++i) by_slot[q][i] = -1;
        for (int e = 0; e < d->E; ++e) {
            const uint32_t v = static_cast<uint32_t>(tbl->pool_slot[e]);
            const int q = (int)(v >> 31), slot = (int)(v & 0x7FFFFFFFu);
            if (slot < kMaxGroups) by_slot[q][slot] = e;   // slots beyond E: see below
        }
        int n = 0;
        for (int q = 0; q < 2; ++q) {
            for (int i = 0; i < kMaxGroups && n < d->E + 1; ++i)
                if (by_slot[q][i] >= 0) a.order[n++] = (uint16_t)by_slot[q][i];
            if (q == 0 && d->has_shared) a.order[n++] = (uint16_t)d->E;
        }
        if (n != G) {  // several experts share a slot, or slots lie beyond kMaxGroups: expert order
            n = 0;
            for (int g = 0; g < G; ++g) a.order[n++] = (uint16_t)g;
        }
    }
    if (gate) {
        a.ready_flags = gate->flags;
        a.ready_epoch = gate->epoch;
        a.slots_per_flag = gate->slots_per_flag;
        a.ready_timeout_ns = gate->timeout_ns > 0 ? (uint64_t)gate->timeout_ns : kWaitLimitNs;
    }
    const void* base[2] = {tbl->local_base, tbl->remote_base};
    const int32_t count[2] = {tbl->local_count, tbl->remote_count};
    const int64_t stride[2] = {tbl->local_stride, tbl->remote_stride};
    const bool w8 = d->w_dtype == MOE_E4M3;
    const int bn = pick_bn(A, d->E, w8);
    a.w_base[0] = static_cast<const uint8_t*>(tbl->local_base);
    a.w_base[1] = static_cast<const uint8_t*>(tbl->remote_base);
    a.w_base[2] = static_cast<const uint8_t*>(tbl->shared);
    a.w_stride[0] = tbl->local_stride;
    a.w_stride[1] = tbl->remote_stride;
    a.w_stride[2] = lay.bytes;
    if (progress) {   // fresh tile counters for the two launches
        if ((st = stream_write_u32(stream, progress->tiles, 0u)) != MOE_OK ||
            (st = stream_write_u32(stream, progress->tiles + 1, 0u)) != MOE_OK)
            return st;
    }
    // bf16 activations with a workspace: the two launches take their tiles
    // from counters in it (dynamic schedule); without one, round-robin
    int32_t* tile_counters = nullptr;
    if (!f8 && workspace && workspace_bytes >= kTileCounterBytes && aligned(workspace, 16)) {
        tile_counters = static_cast<int32_t*>(workspace);
        SWB_CUDA(cudaMemsetAsync(tile_counters, 0, 2 * sizeof(int32_t), stream));
    }
    if (f8) return ffn_f8(d, tbl, lay, x_perm, x_perm_scales, h, y_perm,
                          static_cast<float*>(workspace), (int)rows, G, a, progress, stream);

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
    if (perm_src) {   // token tiles gathered from x [T, H] through perm_src
        const uint64_t dims[2] = {(uint64_t)d->H, (uint64_t)d->T};
        const uint64_t strides[1] = {(uint64_t)d->H * 2};
        const uint32_t box[2] = {(uint32_t)kBK, 1u};
        if ((st = encode_tiled(&a.x_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x_perm),
                               dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) != MOE_OK)
            return st;
        a.perm_src = perm_src;
        a.gather = 1;
    } else {
        if ((st = encode_act_map(&a.act_map, x_perm, rows, d->H, kBoxN)) != MOE_OK) return st;
        if ((st = encode_act_map(&a.act_map64, x_perm, rows, d->H, 64)) != MOE_OK) return st;
    }
    a.K = d->H;
    a.M = d->I;
    a.up_row = d->I;
    a.out = static_cast<__nv_bfloat16*>(h);
    a.ld_out = d->I;
    set_progress(a, progress, 0);
    a.tile_counter = tile_counters;
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
    a.gather = 0;
    if ((st = encode_act_map(&a.act_map, h, rows, d->I, kBoxN)) != MOE_OK) return st;
    if ((st = encode_act_map(&a.act_map64, h, rows, d->I, 64)) != MOE_OK) return st;
    a.K = d->I;
    a.M = d->H;
    a.up_row = 0;
    a.out = static_cast<__nv_bfloat16*>(y_perm);
    a.ld_out = d->H;
    set_progress(a, progress, 1);
    a.tile_counter = tile_counters ? tile_counters + 1 : nullptr;
    if (d->H % (2 * kBM) == 0) return launch_w<kPair>(w8, bn, a, (int)rows, G, stream);
    return launch_w<kSingle>(w8, bn, a, (int)rows, G, stream);
}

}  // namespace
}  // namespace swb
