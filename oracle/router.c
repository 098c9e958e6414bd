/* ORACLE (test infrastructure only; never linked into the product path).
 *
 * Router logits of the MoE block in one fixed fp32 summation order, so that
 * the GPU router can be checked bit for bit:
 *
 *   l[t,e] = sum over h of x[t,h] * W_g[e,h]
 *
 * The DWDP pages (arXiv 2604.01621 abstract; explainer figures) run "the MoE
 * expert layer" of DeepSeek-R1 on each rank but state no router arithmetic.
 * The order used here is this library's definition:
 *   - split h into chunks of 256 consecutive indices (the last may be short);
 *   - within chunk c:  p = 0; for h ascending: p = fma(x[t,h], W_g[e,h], p)
 *     (one fused multiply-add, a single rounding);
 *   - l = P_0, then l = l + P_c for c = 1, 2, ... (fp32 round-to-nearest adds).
 *
 * Built with -ffp-contract=off so that no other operation is fused.
 */
#include <math.h>
#include <stdint.h>

#define CHUNK 256

void oracle_router_logits(const float *x, const float *wg, int64_t T, int64_t H, int64_t E,
                          float *logits) {
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        const float *xr = x + t * H;
        for (int64_t e = 0; e < E; ++e) {
            const float *wr = wg + e * H;
            float l = 0.0f;
            for (int64_t c0 = 0; c0 < H; c0 += CHUNK) {
                const int64_t c1 = c0 + CHUNK < H ? c0 + CHUNK : H;
                float p = 0.0f;
                for (int64_t h = c0; h < c1; ++h) p = fmaf(xr[h], wr[h], p);
                l = (c0 == 0) ? p : l + p;
            }
            logits[t * E + e] = l;
        }
    }
}
