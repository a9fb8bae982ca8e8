// meta.cu -- per-page key metadata (EntmaxKV summary, section 2.A: coordinate-
// wise k_min / k_max for the bounding box, key mean and variance for the
// Gaussian page model), rebuilt for a range of logical pages, or written
// together with each sequence's newest key/value row (append).
//
// One CTA per (page, sequence, kv head); thread j owns coordinate j and walks
// the page's valid tokens in order.  Sums run in fp64 (every bf16 value and
// square is exact there) and are rounded once to fp32, so the record is
// defined to the bit:  mean = fp32(S1/n), var = fp32(max(0, S2/n - (S1/n)^2)).
// The record is stored at its logical page in the tiled, swizzled layout the
// scoring pass streams (include/entmaxkv.h, entmaxkv_meta_bytes).
#include "record.cuh"

namespace ekv {

template <int D, int P>
__global__ void __launch_bounds__(D) build_meta_kernel(MetaArgs a) {
    pdl_wait();
    const int b = blockIdx.y;
    const int kvh = a.kv0 + blockIdx.z;
    const int p = a.first_page + blockIdx.x;
    const int seq = seq_len_of(a.seq_lens, b, P, a.max_pages, a.status);
    if (p >= n_pages_of(seq, P)) return;
    const int blk = a.page_table[(size_t)b * a.max_pages + p];
    if (blk < 0 || blk >= a.num_blocks) {
        if (threadIdx.x == 0) atomicOr(a.status, ENTMAXKV_STATUS_BAD_PAGE);
        return;
    }
    const long long rec = (long long)blk * a.Hkv + kvh;  // the page's keys: k_cache[blk][kvh]
    page_record<D, P>(a, a.k + (size_t)rec * P * D + threadIdx.x, tokens_in_page(seq, P, p), -1, 0, b, kvh, p);
}

// One CTA per (sequence, kv head): the new token's key and value rows land in
// slot seq_len-1 of the paged cache, then the record of that page is rebuilt;
// optionally the group's query rows are copied too (the inputs may be read
// straight from pinned host memory).
template <int D, int P>
__global__ void __launch_bounds__(D) append_kernel(AppendArgs a) {
    pdl_wait();
    const int b = blockIdx.x, kvh = a.m.kv0 + blockIdx.y;
    if (a.q_in) {  // the step's queries of this group, staged for the later calls
        // (all rows loaded before the first store: one round trip over the
        // bus when they sit in pinned host memory, not one per row)
        const int G = a.Hq / a.m.Hkv;  // 1..8
        const size_t o = ((size_t)b * a.Hq + kvh * G) * D + threadIdx.x;
        uint16_t qv[8];
#pragma unroll
        for (int g = 0; g < 8; ++g)
            if (g < G) qv[g] = a.q_in[o + (size_t)g * D];
#pragma unroll
        for (int g = 0; g < 8; ++g)
            if (g < G) a.q_out[o + (size_t)g * D] = qv[g];
    }
    const int seq = a.m.seq_lens[b];
    if (seq <= 0) return;
    const int p = (seq - 1) / P, t = (seq - 1) % P;
    if (p >= a.m.max_pages) {
        if (threadIdx.x == 0) atomicOr(a.m.status, ENTMAXKV_STATUS_BAD_LENGTH);
        return;
    }
    const int blk = a.m.page_table[(size_t)b * a.m.max_pages + p];
    if (blk < 0 || blk >= a.m.num_blocks) {
        if (threadIdx.x == 0) atomicOr(a.m.status, ENTMAXKV_STATUS_BAD_PAGE);
        return;
    }
    const int j = threadIdx.x;
    const size_t src = ((size_t)b * a.m.Hkv + kvh) * D + j;
    const size_t rec = ((size_t)blk * a.m.Hkv + kvh) * P * D;
    const uint16_t kn = a.k_new[src], vn = a.v_new[src];  // both loads before the first store
    a.k_cache[rec + (size_t)t * D + j] = kn;
    a.v_cache[rec + (size_t)t * D + j] = vn;
    page_record<D, P>(a.m, a.k_cache + rec + j, t + 1, t, kn, b, kvh, p);
}

template <int D>
cudaError_t launch_d(const MetaArgs &a, cudaStream_t st) {
    dim3 grid(a.n_pages, a.B, a.nk);
    cudaError_t e = cudaSuccess;
    switch (a.P) {
        case 16: e = launch_pdl(build_meta_kernel<D, 16>, dim3(grid), dim3(D), 0, st, a); break;
        case 32: e = launch_pdl(build_meta_kernel<D, 32>, dim3(grid), dim3(D), 0, st, a); break;
        case 64: e = launch_pdl(build_meta_kernel<D, 64>, dim3(grid), dim3(D), 0, st, a); break;
        default: return cudaErrorInvalidValue;
    }
    return e;
}

template <int D>
cudaError_t launch_append_d(const AppendArgs &a, cudaStream_t st) {
    dim3 grid(a.m.B, a.m.nk);
    switch (a.m.P) {
        case 16: return launch_pdl(append_kernel<D, 16>, dim3(grid), dim3(D), 0, st, a);
        case 32: return launch_pdl(append_kernel<D, 32>, dim3(grid), dim3(D), 0, st, a);
        case 64: return launch_pdl(append_kernel<D, 64>, dim3(grid), dim3(D), 0, st, a);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_append(const AppendArgs &a, cudaStream_t st) {
    return a.m.d == 64 ? launch_append_d<64>(a, st) : launch_append_d<128>(a, st);
}

cudaError_t launch_build_meta(const MetaArgs &a, cudaStream_t st) {
    if (a.n_pages <= 0) return cudaSuccess;
    return a.d == 64 ? launch_d<64>(a, st) : launch_d<128>(a, st);
}

}  // namespace ekv
