// score.cu -- query-aware page scoring (EntmaxKV summary, section 2.A).
//
// For every (sequence b, query head h, page p):
//   bbox  = (sum_j max(q_j kmin_j, q_j kmax_j)) / sqrt(d)   upper bound on s
//   mu    = (sum_j q_j mean_j) / sqrt(d)                    Gaussian mean
//   sigma = sqrt((sum_j q_j^2 var_j) / d)                   Gaussian std
// The bound is one fp64 chain over j in index order with exact products, so
// it is reproducible to the bit; max(q a, q b) with a <= b is q b for q >= 0
// and q a otherwise, one fused multiply-add per coordinate.  mu and sigma feed
// only the approximate tau_hat; they are fp32 chains over j in index order.
//
// Layout of the work: a CTA owns 256 consecutive logical pages of one
// (b, kv head); thread = page, and the thread scores that page for all G query
// heads of the group, so each metadata record crosses HBM once per group.
// Records are streamed through a per-warp ring of 8-coordinate chunks with
// 16-byte cp.async copies: the 32 records of a warp are fetched cooperatively
// (consecutive lanes take consecutive 16-byte pieces of a record, so whole
// 32-byte sectors move per instruction) into padded per-thread slots, and each
// thread then reads its own slot.  The slot pitch keeps the 16-byte reads of
// any 8 consecutive lanes on distinct banks.  q is kept in shared memory
// coordinate-major ([j][head]) so one vector load serves all heads of a
// coordinate.
#include "common.cuh"
#include "internal.h"

namespace ekv {

namespace {

constexpr int SC_THREADS = 256;
constexpr int SC_WARPS = SC_THREADS / 32;
constexpr int CH = 8;  // coordinates per chunk

template <bool GAUSS>
struct ScoreCfg {
    static constexpr int PIECES = GAUSS ? 6 : 2;   // 16-byte pieces per record chunk
    static constexpr int SLOT = PIECES * 16 + 16;  // padded slot pitch (bytes)
    static constexpr int NST = GAUSS ? 3 : 6;      // ring depth (chunks in flight per warp)
    static constexpr int WARP_STAGE = 32 * SLOT;
};

template <int D, int G>
struct QLayout {
    // qd: [D][G] fp64; qf: [D][G] fp32 (the same bf16 values)
    static constexpr int D_BYTES = D * G * 8;
    static constexpr int F_BYTES = D * G * 4;
    static constexpr int BYTES = D_BYTES + F_BYTES;
};

template <int D, int G, bool GAUSS>
__global__ void __launch_bounds__(SC_THREADS, 2) score_kernel(ScoreArgs a) {
    using Cfg = ScoreCfg<GAUSS>;
    using QL = QLayout<D, G>;
    constexpr int NCH = D / CH;
    extern __shared__ __align__(16) unsigned char smem[];
    double *qd = reinterpret_cast<double *>(smem);
    float *qf = reinterpret_cast<float *>(smem + QL::D_BYTES);
    unsigned char *ring = smem + QL::BYTES;

    const int bk = blockIdx.y;
    const int b = bk / a.Hkv, kvh = bk % a.Hkv;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

    for (int i = threadIdx.x; i < G * D; i += SC_THREADS) {
        const int g = i / D, j = i % D;
        const float v = bf16f(a.q[((size_t)b * a.Hq + kvh * G + g) * D + j]);
        qd[j * G + g] = (double)v;
        qf[j * G + g] = v;
    }
    __syncthreads();

    const int seq = a.seq_lens[b];
    const int np = n_pages_of(seq, a.P);
    const int page0 = blockIdx.x * SC_THREADS + warp * 32;
    if (page0 >= np) return;  // whole warp past the end
    const int page = page0 + lane;
    long long rec = -1;
    if (page < np) {
        int blk = a.page_table[(size_t)b * a.max_pages + page];
        if (blk >= 0 && blk < a.num_blocks)
            rec = (long long)blk * a.Hkv + kvh;
        else
            atomicOr(a.status, ENTMAXKV_STATUS_BAD_PAGE);
    }

    // Piece i*32+lane of a chunk belongs to record (i*32+lane)/PIECES.  Piece
    // 0 is kmin, 1 kmax (bound region: kmin at [0,2D) bytes of the record,
    // kmax at [2D,4D), chunk c adds 16c); pieces 2-3 are mean, 4-5 var
    // (moment region: mean at [0,4D), var at [4D,8D), chunk c adds 32c).
    const unsigned char *src[Cfg::PIECES];
    int dst_off[Cfg::PIECES];
#pragma unroll
    for (int i = 0; i < Cfg::PIECES; ++i) {
        const int idx = i * 32 + lane;
        const int rl = idx / Cfg::PIECES, pc = idx % Cfg::PIECES;
        const long long r = __shfl_sync(FULL, rec, rl);
        dst_off[i] = rl * Cfg::SLOT + pc * 16;
        if (r < 0) {
            src[i] = nullptr;
        } else if (pc < 2) {
            src[i] = a.meta + (size_t)r * 4 * D + pc * 2 * D;
        } else {
            src[i] = a.meta + (size_t)a.R * 4 * D + (size_t)r * 8 * D +
                     (pc < 4 ? (pc - 2) * 16 : 4 * D + (pc - 4) * 16);
        }
    }

    unsigned char *wring = ring + warp * Cfg::NST * Cfg::WARP_STAGE;
    auto issue = [&](int c) {
        unsigned char *st = wring + (c % Cfg::NST) * Cfg::WARP_STAGE;
#pragma unroll
        for (int i = 0; i < Cfg::PIECES; ++i) {
            if (src[i] == nullptr) continue;
            // bound pieces sit in the first 32 bytes of the slot
            const int cstride = dst_off[i] % Cfg::SLOT < 32 ? 16 : 32;
            cp_async16(st + dst_off[i], src[i] + c * cstride);
        }
    };

#pragma unroll
    for (int c = 0; c < Cfg::NST - 1; ++c) {
        if (c < NCH) issue(c);
        cp_async_commit();
    }

    double ab[G];
    float am[G], av[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        ab[g] = 0.0;
        am[g] = av[g] = 0.f;
    }

    const unsigned char *myslot0 = wring + lane * Cfg::SLOT;
    for (int c = 0; c < NCH; ++c) {
        if (c + Cfg::NST - 1 < NCH) issue(c + Cfg::NST - 1);
        cp_async_commit();
        cp_async_wait<Cfg::NST - 1>();
        __syncwarp();
        const unsigned char *slot = myslot0 + (c % Cfg::NST) * Cfg::WARP_STAGE;
        const uint4 kn = *reinterpret_cast<const uint4 *>(slot + 0);
        const uint4 kx = *reinterpret_cast<const uint4 *>(slot + 16);
        const unsigned wn[4] = {kn.x, kn.y, kn.z, kn.w};
        const unsigned wx[4] = {kx.x, kx.y, kx.z, kx.w};
        float mv[CH], vv[CH];
        if (GAUSS) {
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                float4 m4 = *reinterpret_cast<const float4 *>(slot + 32 + 16 * i);
                float4 v4 = *reinterpret_cast<const float4 *>(slot + 64 + 16 * i);
                mv[4 * i] = m4.x; mv[4 * i + 1] = m4.y; mv[4 * i + 2] = m4.z; mv[4 * i + 3] = m4.w;
                vv[4 * i] = v4.x; vv[4 * i + 1] = v4.y; vv[4 * i + 2] = v4.z; vv[4 * i + 3] = v4.w;
            }
        }
        const double *qdc = qd + (size_t)c * CH * G;
        const float *qfc = qf + c * CH * G;
#pragma unroll
        for (int jj = 0; jj < CH; ++jj) {
            const unsigned w_n = wn[jj >> 1], w_x = wx[jj >> 1];
            const double lo = (double)((jj & 1) ? bf16hi(w_n) : bf16lo(w_n));
            const double hi = (double)((jj & 1) ? bf16hi(w_x) : bf16lo(w_x));
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const double qv = qdc[jj * G + g];
                ab[g] = __fma_rn(qv, (__double2hiint(qv) < 0) ? lo : hi, ab[g]);
                if (GAUSS) {
                    const float qs = qfc[jj * G + g];
                    am[g] = __fmaf_rn(qs, mv[jj], am[g]);
                    av[g] = __fmaf_rn(__fmul_rn(qs, qs), vv[jj], av[g]);  // q^2 exact in fp32
                }
            }
        }
        __syncwarp();
    }
    cp_async_wait<0>();

    if (rec < 0) return;
    const double inv_sqrt_d = __ddiv_rn(1.0, __dsqrt_rn((double)D));
    const float inv_sqrt_df = D == 64 ? 0.125f : 0.08838834764831845f;
#pragma unroll
    for (int g = 0; g < G; ++g) {
        const size_t o = ((size_t)b * a.Hq + kvh * G + g) * a.max_pages + page;
        a.bbox[o] = (float)__dmul_rn(ab[g], inv_sqrt_d);
        if (GAUSS) {
            a.mu[o] = am[g] * inv_sqrt_df;
            a.sigma[o] = sqrtf(av[g] * (1.f / (float)D));
        }
    }
}

template <int D, int G, bool GAUSS>
cudaError_t launch_t(const ScoreArgs &a, cudaStream_t st) {
    using Cfg = ScoreCfg<GAUSS>;
    const size_t smem = QLayout<D, G>::BYTES + (size_t)SC_WARPS * Cfg::NST * Cfg::WARP_STAGE;
    auto kern = score_kernel<D, G, GAUSS>;
    cudaError_t e = ensure_smem(reinterpret_cast<const void *>(kern), smem);
    if (e != cudaSuccess) return e;
    dim3 grid(ceil_div(a.max_pages, SC_THREADS), a.B * a.Hkv);
    kern<<<grid, SC_THREADS, smem, st>>>(a);
    return cudaGetLastError();
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
