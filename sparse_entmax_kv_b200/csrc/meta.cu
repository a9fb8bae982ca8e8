// meta.cu -- per-page key metadata (EntmaxKV summary, section 2.A: coordinate-
// wise k_min / k_max for the bounding box, key mean and variance for the
// Gaussian page model), rebuilt for a range of logical pages.
//
// One CTA per (page, sequence, kv head); thread j owns coordinate j and walks
// the page's valid tokens in order.  Sums run in fp64 (every bf16 value and
// square is exact there) and are rounded once to fp32, so the record is
// defined to the bit:  mean = fp32(S1/n), var = fp32(max(0, S2/n - (S1/n)^2)).
#include "common.cuh"
#include "internal.h"

namespace ekv {

template <int D>
__global__ void __launch_bounds__(D) build_meta_kernel(MetaArgs a) {
    const int b = blockIdx.y;
    const int kvh = blockIdx.z;
    const int p = a.first_page + blockIdx.x;
    const int seq = a.seq_lens[b];
    if (p >= n_pages_of(seq, a.P)) return;
    const int blk = a.page_table[(size_t)b * a.max_pages + p];
    if (blk < 0 || blk >= a.num_blocks) {
        if (threadIdx.x == 0) atomicOr(a.status, ENTMAXKV_STATUS_BAD_PAGE);
        return;
    }
    const int n = tokens_in_page(seq, a.P, p);
    const long long rec = (long long)blk * a.Hkv + kvh;
    const int j = threadIdx.x;
    const uint16_t *col = a.k + (size_t)rec * a.P * D + j;

    uint16_t bmin = col[0], bmax = col[0];
    float vmin = bf16f(bmin), vmax = vmin;
    double s1 = 0.0, s2 = 0.0;
    int t = 0;
    for (; t + 8 <= n; t += 8) {
        uint16_t h[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) h[i] = __ldg(col + (size_t)(t + i) * D);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            float x = bf16f(h[i]);
            if (x < vmin) { vmin = x; bmin = h[i]; }
            if (x > vmax) { vmax = x; bmax = h[i]; }
            double xd = (double)x;
            s1 = __dadd_rn(s1, xd);
            s2 = __fma_rn(xd, xd, s2);  // xd*xd is exact, so this equals s2 + xd*xd rounded once
        }
    }
    for (; t < n; ++t) {
        uint16_t h = __ldg(col + (size_t)t * D);
        float x = bf16f(h);
        if (x < vmin) { vmin = x; bmin = h; }
        if (x > vmax) { vmax = x; bmax = h; }
        double xd = (double)x;
        s1 = __dadd_rn(s1, xd);
        s2 = __fma_rn(xd, xd, s2);
    }
    const double dn = (double)n;
    const double m = __ddiv_rn(s1, dn);
    double v = __dsub_rn(__ddiv_rn(s2, dn), __dmul_rn(m, m));
    if (v < 0.0) v = 0.0;

    uint16_t *bb = reinterpret_cast<uint16_t *>(a.meta + (size_t)rec * 4 * D);
    bb[j] = bmin;
    bb[D + j] = bmax;
    float *mm = reinterpret_cast<float *>(a.meta + (size_t)a.R * 4 * D + (size_t)rec * 8 * D);
    mm[j] = (float)m;
    mm[D + j] = (float)v;
}

cudaError_t launch_build_meta(const MetaArgs &a, cudaStream_t st) {
    if (a.n_pages <= 0) return cudaSuccess;
    dim3 grid(a.n_pages, a.B, a.Hkv);
    if (a.d == 64)
        build_meta_kernel<64><<<grid, 64, 0, st>>>(a);
    else
        build_meta_kernel<128><<<grid, 128, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace ekv
