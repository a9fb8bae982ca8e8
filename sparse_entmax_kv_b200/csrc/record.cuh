// record.cuh -- the per-page metadata record (EntmaxKV summary, section 2.A),
// shared by the metadata build, the append kernel and the fused append +
// scoring pass.
#pragma once

#include "common.cuh"
#include "internal.h"

namespace ekv {

// Thread j of a D-thread CTA: the record of coordinate j of logical page p of
// (b, kvh), whose n valid keys are col[t * D], t < n.  When t_new >= 0 the
// key of token t_new is k_new (it was just written by this thread, so it is
// not read back through the read-only path).
template <int D, int P>
__device__ __forceinline__ void page_record(const MetaArgs &a, const uint16_t *col, int n, int t_new, uint16_t k_new,
                                            int b, int kvh, int p) {
    // every load of the page is issued before the first use
    uint16_t h[P];
#pragma unroll
    for (int t = 0; t < P; ++t) h[t] = t < n && t != t_new ? __ldg(col + (size_t)t * D) : (uint16_t)0;
    if (t_new >= 0) {
#pragma unroll
        for (int t = 0; t < P; ++t)
            if (t == t_new) h[t] = k_new;
    }

    uint16_t bmin = h[0], bmax = h[0];
    float vmin = bf16f(bmin), vmax = vmin;
    double s1 = 0.0, s2 = 0.0;
#pragma unroll
    for (int t = 0; t < P; ++t) {
        if (t < n) {
            const float x = bf16f(h[t]);
            if (x < vmin) { vmin = x; bmin = h[t]; }
            if (x > vmax) { vmax = x; bmax = h[t]; }
            const double xd = (double)x;
            s1 = __dadd_rn(s1, xd);
            s2 = __fma_rn(xd, xd, s2);  // xd*xd is exact, so this is s2 + xd*xd rounded once
        }
    }
    const double dn = (double)n;
    const double m = __ddiv_rn(s1, dn);
    double v = __dsub_rn(__ddiv_rn(s2, dn), __dmul_rn(m, m));
    if (v < 0.0) v = 0.0;

    const int j = threadIdx.x;
    const int tile = p / META_TILE, sl = p % META_TILE;
    const long long T = ((long long)b * a.Hkv + kvh) * a.n_tiles + tile;
    const int c = j / 16, e = j % 16;
    uint8_t *bb = a.meta + T * 128 * D + c * 2048;
    const int ob = sl * 32 + 16 * ((e >> 3) ^ ((sl >> 2) & 1)) + 2 * (e & 7);
    *reinterpret_cast<uint16_t *>(bb + ob) = bmin;
    *reinterpret_cast<uint16_t *>(bb + 1024 + ob) = bmax;
    uint8_t *mm = a.meta + a.n_tiles_total * 128 * D + T * 256 * D + c * 4096;
    const int om = sl * 64 + 16 * ((e >> 2) ^ ((sl >> 1) & 3)) + 4 * (e & 3);
    *reinterpret_cast<float *>(mm + om) = (float)m;
    *reinterpret_cast<float *>(mm + 2048 + om) = (float)v;
}

}  // namespace ekv
