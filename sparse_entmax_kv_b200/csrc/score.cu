// score.cu -- query-aware page scoring (EntmaxKV summary, section 2.A).
//
// For every (sequence b, query head h, page p):
//   bbox  = (sum_j max(q_j kmin_j, q_j kmax_j)) / sqrt(d)   upper bound on s
//   mu    = (sum_j q_j mean_j) / sqrt(d)                    Gaussian mean
//   sigma = sqrt((sum_j q_j^2 var_j) / d)                   Gaussian std
//
// The bound is one fp64 chain over j in index order, so it is reproducible to
// the bit.  max(q a, q b) with a <= b is q b for q >= 0 and q a for q < 0: the
// chain takes one fused multiply-add per coordinate and head, of q (fp64) and
// the bound its sign picks.  A bf16 value widened to fp64 has an all-zero low
// word, so the pick is a select of the two high words.
// mu and sigma feed only the approximate tau_hat; they are fp32 sums kept as
// two interleaved chains (even and odd j) so that packed f32x2 FMAs do two
// coordinates per instruction.
//
// Layout of the work: the metadata sits in logical page order, in tiles of 32
// pages whose 16-coordinate chunk blocks are contiguous (see include/
// entmaxkv.h).  A warp owns one tile: lane = page.  It streams the tile chunk
// by chunk through a two-stage ring in shared memory, each stage filled by
// two 1-D bulk copies (2 KB of bounds, 4 KB of moments) completing on an
// mbarrier, so HBM sees long contiguous reads and the SM issues no per-lane
// copy instructions.  Each lane scores its page for all G query heads of the
// group, so every byte crosses HBM once per group.  q sits in shared memory
// as fp64 ([j][head]: one 16-byte load serves two heads) and fp32 ([head][j]).
// (An earlier form kept (min(q,0), max(q,0)) pairs, one 16-byte load and two
// FMAs per coordinate and head; its shared-memory loads filled 79% of the LSU
// data pipe in the bound-only scan, which then stalled on the MIO queue.)
#include "common.cuh"
#include "internal.h"

namespace ekv {

namespace {

constexpr int TP = 32;       // pages per tile (= lanes)
constexpr int CHK = 16;      // coordinates per chunk
constexpr int WARPS = 8;
constexpr int THREADS = WARPS * 32;
constexpr int BOUND_CHUNK = 128 * CHK;  // kmin + kmax block of one chunk: 2048 B
constexpr int MOM_CHUNK = 256 * CHK;    // mean + var block of one chunk:  4096 B

// A ring stage holds CPS chunks: the Gaussian policy's one chunk of bounds
// and moments (2 KB + 4 KB), or top-k's two consecutive chunks of bounds
// (one 4 KB copy: the bound-only stream measured faster with 4 KB copies in
// two stages than with 2 KB copies in four, 24 vs 31 us of loads alone for
// the 128k-token batch of 8).
template <bool GAUSS>
struct Ring {
    static constexpr int CPS = GAUSS ? 1 : 2;
    static constexpr int STAGE = GAUSS ? BOUND_CHUNK + MOM_CHUNK : CPS * BOUND_CHUNK;
    static constexpr int NST = 2;
};

template <int D, int G>
struct QBytes {
    static constexpr int VALUE = D * G * 8 + D * G * 4;
};

template <int D, int G, bool GAUSS>
constexpr size_t smem_bytes() {
    return ((QBytes<D, G>::VALUE + WARPS * Ring<GAUSS>::NST * 8 + 127) & ~size_t(127)) +
           (size_t)WARPS * Ring<GAUSS>::NST * Ring<GAUSS>::STAGE;
}

// Two CTAs per SM for the Gaussian policy (its 6 KB stages fill shared
// memory); three for top-k (4 KB stages), whose bounds-only stream does the
// same fp64 work per chunk on a third of the bytes and gains from more warps.
template <int D, int G, bool GAUSS>
__global__ void __launch_bounds__(THREADS, G <= 4 ? (GAUSS ? 2 : 3) : 1) score_kernel(ScoreArgs a) {
    pdl_wait();
    if (a.umap) {
        // decode step: clear this group's row of the selection's union marks
        // (the CTAs of the group share it; rows of other kv heads are left to
        // their own calls)
        int b0, k0;
        group_of(blockIdx.y, a.kv0, a.nk, b0, k0);
        uint4 *row = reinterpret_cast<uint4 *>(a.umap + (size_t)(b0 * a.Hkv + k0) * a.uwords);
        for (int i = blockIdx.x * THREADS + threadIdx.x; i < a.uwords / 4; i += gridDim.x * THREADS)
            row[i] = make_uint4(0u, 0u, 0u, 0u);
    }
    using RG = Ring<GAUSS>;
    constexpr int CPS = RG::CPS;
    constexpr int NCH = D / CHK / CPS;  // ring stages per tile
    constexpr int NST = RG::NST;
    extern __shared__ __align__(128) unsigned char smem[];
    double *qd = reinterpret_cast<double *>(smem);          // [D][G] q
    float *qh = reinterpret_cast<float *>(qd + D * G);       // [G][D] q
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + QBytes<D, G>::VALUE);
    unsigned char *ring = smem + ((QBytes<D, G>::VALUE + WARPS * NST * 8 + 127) & ~127);

    int b, kvh;
    group_of(blockIdx.y, a.kv0, a.nk, b, kvh);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

    __shared__ unsigned q_bad;  // bit g: head g's query has a NaN or an infinity
    if (threadIdx.x == 0) q_bad = 0u;
    __syncthreads();
    for (int i = threadIdx.x; i < G * D; i += THREADS) {
        const int g = i / D, j = i % D;
        const float v = bf16f(a.q[((size_t)b * a.Hq + kvh * G + g) * D + j]);
        if (!isfinite(v)) atomicOr(&q_bad, 1u << g);
        qd[j * G + g] = (double)v;
        qh[g * D + j] = v;
    }
    if (threadIdx.x < WARPS * NST) mbar_init(&bars[threadIdx.x], 1);
    mbar_fence_init();
    __syncthreads();
    const unsigned bad = q_bad;
    if (bad && threadIdx.x == 0 && blockIdx.x == 0) atomicOr(a.status, ENTMAXKV_STATUS_NONFINITE);

    const int np = n_pages_of(seq_len_of(a.seq_lens, b, a.P, a.max_pages, a.status), a.P);
    const int tile = blockIdx.x * WARPS + warp;
    const int page0 = tile * TP;
    if (page0 >= np) return;  // whole warp past the end

    const long long T = ((long long)b * a.Hkv + kvh) * a.n_tiles + tile;
    const unsigned char *gb = a.meta + T * 128 * D;
    const unsigned char *gm = a.meta + (size_t)a.n_tiles_total * 128 * D + T * 256 * D;
    unsigned char *wring = ring + warp * NST * RG::STAGE;
    uint64_t *wbar = bars + warp * NST;

    auto issue = [&](int c) {
        if (lane == 0) {
            unsigned char *st = wring + (c % NST) * RG::STAGE;
            uint64_t *bar = &wbar[c % NST];
            mbar_arrive_expect_tx(bar, RG::STAGE);
            bulk_g2s(st, gb + c * CPS * BOUND_CHUNK, CPS * BOUND_CHUNK, bar);
            if (GAUSS) bulk_g2s(st + BOUND_CHUNK, gm + c * MOM_CHUNK, MOM_CHUNK, bar);
        }
    };
#pragma unroll
    for (int c = 0; c < NST - 1; ++c)
        if (c < NCH) issue(c);

    double ab[G];
    float2 am[G], av[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        ab[g] = 0.0;
        am[g] = av[g] = make_float2(0.f, 0.f);
    }
    const int s = lane;
    const int xb = (s >> 2) & 1, xm = (s >> 1) & 3;  // the layout's swizzles
    bool ok = true;
    for (int ci = 0; ci < NCH; ++ci) {
        if (ci + NST - 1 < NCH) issue(ci + NST - 1);
        ok &= mbar_wait(&wbar[ci % NST], (ci / NST) & 1, a.status);
#pragma unroll
        for (int k = 0; k < CPS; ++k) {
        const unsigned char *st = wring + (ci % NST) * RG::STAGE + k * BOUND_CHUNK;  // chunk c's bounds
        const int c = ci * CPS + k;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {  // two halves of 8 coordinates
            const uint4 kn = *reinterpret_cast<const uint4 *>(st + s * 32 + 16 * (hf ^ xb));
            const uint4 kx = *reinterpret_cast<const uint4 *>(st + 1024 + s * 32 + 16 * (hf ^ xb));
            const unsigned wn[4] = {kn.x, kn.y, kn.z, kn.w};
            const unsigned wx[4] = {kx.x, kx.y, kx.z, kx.w};
            const int j0 = c * CHK + 8 * hf;
            if (GAUSS) {
#pragma unroll
                for (int qt = 0; qt < 2; ++qt) {  // quarters of 4 coordinates
                    const int pc = (2 * hf + qt) ^ xm;
                    const float4 m4 = *reinterpret_cast<const float4 *>(st + BOUND_CHUNK + s * 64 + 16 * pc);
                    const float4 v4 = *reinterpret_cast<const float4 *>(st + BOUND_CHUNK + 2048 + s * 64 + 16 * pc);
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        const float4 q4 = *reinterpret_cast<const float4 *>(qh + g * D + j0 + 4 * qt);
                        const float2 q01 = make_float2(q4.x, q4.y), q23 = make_float2(q4.z, q4.w);
                        am[g] = __ffma2_rn(q01, make_float2(m4.x, m4.y), am[g]);
                        am[g] = __ffma2_rn(q23, make_float2(m4.z, m4.w), am[g]);
                        av[g] = __ffma2_rn(__fmul2_rn(q01, q01), make_float2(v4.x, v4.y), av[g]);  // q^2 exact
                        av[g] = __ffma2_rn(__fmul2_rn(q23, q23), make_float2(v4.z, v4.w), av[g]);
                    }
                }
            }
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
                const unsigned w_n = wn[jj >> 1], w_x = wx[jj >> 1];
                // high words of kmin_j and kmax_j widened to fp64 (low words zero)
                const int lo_h = __double2hiint((double)((jj & 1) ? bf16hi(w_n) : bf16lo(w_n)));
                const int hi_h = __double2hiint((double)((jj & 1) ? bf16hi(w_x) : bf16lo(w_x)));
                const int j = j0 + jj;
                double q[G];
                if constexpr (G == 1) {
                    q[0] = qd[j];
                } else {
#pragma unroll
                    for (int g = 0; g < G; g += 2) {
                        const double2 q2 = *reinterpret_cast<const double2 *>(qd + j * G + g);
                        q[g] = q2.x;
                        q[g + 1] = q2.y;
                    }
                }
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    const double k = __hiloint2double(__double2hiint(q[g]) < 0 ? lo_h : hi_h, 0);
                    ab[g] = __fma_rn(q[g], k, ab[g]);
                }
            }
        }
        }
        __syncwarp();  // every lane is done with this stage before it is refilled
    }

    const int page = page0 + lane;
    if (!ok || page >= np) return;
    const double inv_sqrt_d = __ddiv_rn(1.0, __dsqrt_rn((double)D));
    const float inv_sqrt_df = D == 64 ? 0.125f : 0.08838834764831845f;
    const float qnan = __int_as_float(0x7fc00000);
#pragma unroll
    for (int g = 0; g < G; ++g) {
        const size_t o = ((size_t)b * a.Hq + kvh * G + g) * a.max_pages + page;
        const bool hb = (bad >> g) & 1u;
        a.bbox[o] = hb ? qnan : (float)__dmul_rn(ab[g], inv_sqrt_d);
        if (GAUSS) {
            a.mu[o] = hb ? qnan : (am[g].x + am[g].y) * inv_sqrt_df;
            a.sigma[o] = hb ? qnan : sqrtf((av[g].x + av[g].y) * (1.f / (float)D));
        }
    }
}

template <int D, int G, bool GAUSS>
cudaError_t launch_t(const ScoreArgs &a, cudaStream_t st) {
    constexpr size_t smem = smem_bytes<D, G, GAUSS>();
    auto kern = score_kernel<D, G, GAUSS>;
    cudaError_t e = ensure_smem(reinterpret_cast<const void *>(kern), smem);
    if (e != cudaSuccess) return e;
    dim3 grid(ceil_div(a.n_tiles, WARPS), a.B * a.nk);
    return launch_pdl(kern, dim3(grid), dim3(THREADS), smem, st, a);
}

template <int D, bool GAUSS>
cudaError_t launch_g(const ScoreArgs &a, cudaStream_t st) {
    switch (a.Hq / a.Hkv) {
        case 1: return launch_t<D, 1, GAUSS>(a, st);
        case 2: return launch_t<D, 2, GAUSS>(a, st);
        case 4: return launch_t<D, 4, GAUSS>(a, st);
        case 8: return launch_t<D, 8, GAUSS>(a, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_score_pages(const ScoreArgs &a, cudaStream_t st) {
    const bool gauss = a.mu != nullptr;
    if (a.d == 64) return gauss ? launch_g<64, true>(a, st) : launch_g<64, false>(a, st);
    return gauss ? launch_g<128, true>(a, st) : launch_g<128, false>(a, st);
}

}  // namespace ekv
