// decode.cu -- alpha-entmax decode attention over paged bf16 K/V (EntmaxKV
// summary: section 2.C sparse attention over the selected pages; section 4
// full-cache entmax and full-cache softmax as comparison points).
//
// Sparse path, four launches on one stream, no host round trip:
//   union_kernel   per (sequence, kv head): union of the G query heads'
//                  selected pages, ascending, each with a G-bit head mask;
//                  also resets the running maxima and the combine counters.
//   qk_kernel      split over the union: TMA 2-D loads (128-byte swizzle) of
//                  the K tiles through a 4-stage mbarrier ring fed by one
//                  producer warp; z = (alpha-1) q.k/sqrt(d) for every head of
//                  the group from one copy of each tile (tensor-core
//                  m16n8k16 with tokens as M and the G heads as N when G >= 2,
//                  CUDA cores when G == 1); z goes to a scratch row per head,
//                  and the per-head max to an atomic.
//   tau_kernel     per (sequence, query head): the exact threshold.  Every
//                  support token has z > z_max - 1 (p <= 1), so only those
//                  candidates are kept on chip; the root of
//                  sum (z - tau)_+^r = 1 is bracketed in [z_max - 1,
//                  z_max - n^(1-alpha)] and narrowed by multisection (512
//                  points per pass for small candidate sets, 32 per pass
//                  with a block reduction otherwise).
//   pv_gather_kernel  split over the union: p = (z - tau)_+^r, and only the
//                  value rows with p > 0 for some head of the group are read
//                  (their weight is exactly zero otherwise); partial sums are
//                  combined by the last CTA of the group in a fixed order.
// Full-cache entmax runs qk_kernel over every page, tau_kernel, and
// pv_stream_kernel, which streams every V tile through the same TMA ring.
// Full-cache softmax runs softmax_kernel (K and V tiles per stage, online
// max / sum per split) and combines the splits the same way.
#include "common.cuh"
#include "internal.h"

namespace ekv {

namespace {

constexpr int NWC = 4;                     // consumer warps
constexpr int DEC_THREADS = (NWC + 1) * 32;  // + one producer warp
constexpr int PPS_MAX = 8;

template <int G>
struct Tile {
    static constexpr int TPS = G == 1 ? 128 : 64;  // tokens per pipeline stage
};

struct PageInfo {
    int page;   // logical page (-1: none)
    int mask;   // heads of the group that use it
    int nval;   // valid tokens (0 if the page could not be loaded)
    int upos;   // position in the union (row offset in the z scratch / P)
};

__device__ __forceinline__ size_t zrow(const DecodeArgs &a, int b, int h) {
    return ((size_t)b * a.Hq + h) * (size_t)a.max_pages * a.P;
}

// ------------------------------------------------------------------ union

__global__ void __launch_bounds__(512) union_kernel(DecodeArgs a) {
    extern __shared__ unsigned words[];
    __shared__ int sh[72];
    const int bk = blockIdx.x;
    const int b = bk / a.Hkv, kvh = bk % a.Hkv;
    const int G = a.Hq / a.Hkv;
    const int np = n_pages_of(a.seq_lens[b], a.P);
    const int nw = ceil_div(np, 4);
    for (int i = threadIdx.x; i < nw; i += blockDim.x) words[i] = 0u;
    __syncthreads();
    for (int g = 0; g < G; ++g) {
        const int bh = b * a.Hq + kvh * G + g;
        int c = a.cnt[bh];
        if (c < 0 || c > np) {
            if (threadIdx.x == 0) atomicOr(a.status, ENTMAXKV_STATUS_BAD_SELECTION);
            c = c < 0 ? 0 : np;
        }
        const int *sl = a.sel + (size_t)bh * a.max_pages;
        for (int i = threadIdx.x; i < c; i += blockDim.x) {
            const int p = sl[i];
            if (p >= 0 && p < np)
                atomicOr(&words[p >> 2], 1u << ((p & 3) * 8 + g));
            else
                atomicOr(a.status, ENTMAXKV_STATUS_BAD_SELECTION);
        }
        if (threadIdx.x == 0) {
            a.ws.zmax[bh] = ORD_NEG_INF;
        }
    }
    __syncthreads();
    constexpr int IT = 16;
    int *ue = a.ws.union_e + (size_t)bk * a.max_pages;
    int base = 0;
    for (int t0 = 0; t0 < np; t0 += 512 * IT) {
        const int p0 = t0 + threadIdx.x * IT;
        unsigned bits = 0;
#pragma unroll
        for (int i = 0; i < IT; ++i) {
            const int p = p0 + i;
            if (p < np && ((words[p >> 2] >> ((p & 3) * 8)) & 0xffu)) bits |= 1u << i;
        }
        int tot;
        int w = base + block_excl_scan(__popc(bits), sh, &tot);
#pragma unroll
        for (int i = 0; i < IT; ++i)
            if (bits & (1u << i)) {
                const int p = p0 + i;
                ue[w++] = (p << 8) | ((words[p >> 2] >> ((p & 3) * 8)) & 0xffu);
            }
        base += tot;
    }
    if (threadIdx.x == 0) {
        a.ws.union_cnt[bk] = base;
        a.ws.counters[bk] = 0;
    }
}

__global__ void dense_init_kernel(DecodeArgs a) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < a.B * a.Hq) a.ws.zmax[i] = ORD_NEG_INF;
    if (i < a.B * a.Hkv) a.ws.counters[i] = 0;
}

// ------------------------------------------------------ shared TMA pipeline

// Shared-memory carve-up of the TMA ring kernels.
template <int D, int G, int NS, int NMAP>
struct Ring {
    static constexpr int TPS = Tile<G>::TPS;
    static constexpr int STAGE = TPS * D * 2 * NMAP;  // bytes per stage (K and/or V)
    static constexpr size_t BYTES = 1024 + (size_t)NS * STAGE + 2 * NS * 8 + NS * PPS_MAX * sizeof(PageInfo);
};

// Producer side: for local step `it`, gather the step's pages (union entries
// [step*PPS, step*PPS+PPS) of this group), publish them in `pinfo`, and issue
// the box loads of every valid page into the stage.  maps[0] / maps[1] are the
// K / V maps; a stage holds the K tile block first, then the V tile block.
template <int D, int NMAP>
__device__ __forceinline__ bool produce_step(const DecodeArgs &a, bool dense, int b, int kvh, int bk, int U,
                                             int step, int PPS, unsigned char *stage, int stage_half,
                                             uint64_t *full, PageInfo *pinfo) {
    int blk_i[PPS_MAX];
    unsigned bytes = 0;
    const int seq = a.seq_lens[b];
    for (int i = 0; i < PPS; ++i) {
        const int e = step * PPS + i;
        PageInfo pi{-1, 0, 0, e};
        blk_i[i] = -1;
        if (e < U) {
            const int entry = dense ? ((e << 8) | 0xff) : a.ws.union_e[(size_t)bk * a.max_pages + e];
            pi.page = entry >> 8;
            pi.mask = entry & 0xff;
            const int blk = a.page_table[(size_t)b * a.max_pages + pi.page];
            if (blk >= 0 && blk < a.num_blocks) {
                pi.nval = tokens_in_page(seq, a.P, pi.page);
                blk_i[i] = blk;
                bytes += (unsigned)(a.P * D * 2 * NMAP);
            } else {
                atomicOr(a.status, ENTMAXKV_STATUS_BAD_PAGE);
            }
        }
        pinfo[i] = pi;
    }
    mbar_arrive_expect_tx(full, bytes);
    for (int i = 0; i < PPS; ++i) {
        if (blk_i[i] < 0) continue;
        const int y = (blk_i[i] * a.Hkv + kvh) * a.P;
        unsigned char *dst = stage + (size_t)i * a.P * D * 2;
#pragma unroll
        for (int box = 0; box < D / 64; ++box) {
            tma_load_2d(dst + box * a.P * 128, &a.kmap, box * 64, y, full);
            if (NMAP == 2) tma_load_2d(dst + stage_half + box * a.P * 128, &a.vmap, box * 64, y, full);
        }
    }
    return true;
}

// Address of the 16-byte chunk `c16` (8 bf16) of row r in a swizzled page tile.
template <int D>
__device__ __forceinline__ const unsigned char *tile_chunk(const unsigned char *page_base, int P, int r, int c16) {
    const int box = c16 >> 3, cc = c16 & 7;
    return page_base + box * P * 128 + r * 128 + ((cc ^ (r & 7)) << 4);
}

// ----------------------------------------------------------------- q . K^T

template <int D, int G, bool DENSE>
__global__ void __launch_bounds__(DEC_THREADS) qk_kernel(const __grid_constant__ DecodeArgs a) {
    constexpr int NS = 4;
    using RG = Ring<D, G, NS, 1>;
    constexpr int TPS = RG::TPS;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *stages = reinterpret_cast<unsigned char *>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint64_t *full = reinterpret_cast<uint64_t *>(stages + (size_t)NS * RG::STAGE);
    uint64_t *empty = full + NS;
    PageInfo *pinfo = reinterpret_cast<PageInfo *>(empty + NS);
    __shared__ float qs[G == 1 ? D : 1];

    const int bk = blockIdx.y;
    const int b = bk / a.Hkv, kvh = bk % a.Hkv;
    const int P = a.P, PPS = TPS / P;
    const int seq = a.seq_lens[b];
    const int np = n_pages_of(seq, P);
    const int U = DENSE ? np : a.ws.union_cnt[bk];
    const int nsteps = ceil_div(U, PPS);
    const int S = gridDim.x;
    const int my_n = nsteps > (int)blockIdx.x ? ceil_div(nsteps - blockIdx.x, S) : 0;
    if (my_n == 0) return;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], NWC);
        }
        mbar_fence_init();
    }
    if (G == 1)
        for (int j = threadIdx.x; j < D; j += blockDim.x) qs[j] = bf16f(a.q[((size_t)b * a.Hq + kvh) * D + j]);
    __syncthreads();

    if (warp == NWC) {
        if (lane == 0) {
            prefetch_tmap(&a.kmap);
            for (int it = 0; it < my_n; ++it) {
                const int st = it % NS, ph = (it / NS) & 1;
                if (!mbar_wait(&empty[st], ph ^ 1, a.status)) break;
                produce_step<D, 1>(a, DENSE, b, kvh, bk, U, blockIdx.x + it * S, PPS, stages + (size_t)st * RG::STAGE,
                                   0, &full[st], pinfo + st * PPS_MAX);
            }
        }
        return;
    }

    // z = (alpha-1) * s, s = q.k / sqrt(d); 1/sqrt(d) as a correctly rounded constant
    const float zs = (a.alpha - 1.f) * (D == 64 ? 0.125f : 0.08838834764831845f);

    if constexpr (G >= 2) {
        // B fragments: q of head n = lane/4 (zero for n >= G), k pair 2*(lane%4)
        unsigned qb[D / 16][2];
        {
            const int n = lane >> 2, kp = 2 * (lane & 3);
            const uint16_t *qh = a.q + ((size_t)b * a.Hq + kvh * G + (n < G ? n : 0)) * D;
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                unsigned lo = n < G ? *reinterpret_cast<const unsigned *>(qh + 16 * ks + kp) : 0u;
                unsigned hi = n < G ? *reinterpret_cast<const unsigned *>(qh + 16 * ks + kp + 8) : 0u;
                qb[ks][0] = lo;
                qb[ks][1] = hi;
            }
        }
        float zmx0 = -INFINITY, zmx1 = -INFINITY;
        const int h0 = 2 * (lane & 3);
        for (int it = 0; it < my_n; ++it) {
            const int st = it % NS, ph = (it / NS) & 1;
            if (!mbar_wait(&full[st], ph, a.status)) return;
            const unsigned char *stage = stages + (size_t)st * RG::STAGE;
            const PageInfo *pis = pinfo + st * PPS_MAX;
            for (int mt = warp; mt < TPS / 16; mt += NWC) {
                const int tok0 = mt * 16, pi_i = tok0 / P, r0 = tok0 % P;
                const PageInfo pi = pis[pi_i];
                if (pi.page < 0) continue;
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
                const unsigned char *pbase = stage + (size_t)pi_i * P * D * 2;
                if (pi.nval > 0) {
                    const int mat = lane >> 3, rr = lane & 7;
                    const int row = r0 + (mat & 1) * 8 + rr;
#pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks) {
                        unsigned a0, a1, a2, a3;
                        ldsm_x4(smem_u32(tile_chunk<D>(pbase, P, row, ks * 2 + (mat >> 1))), a0, a1, a2, a3);
                        mma_bf16_16816(acc, a0, a1, a2, a3, qb[ks][0], qb[ks][1]);
                    }
                }
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    const int hh = h0 + (v & 1);
                    const int t = r0 + (lane >> 2) + (v >= 2 ? 8 : 0);
                    if (hh < G) {
                        // heads that did not select the page see -inf
                        const float z = (t < pi.nval && ((pi.mask >> hh) & 1)) ? acc[v] * zs : -INFINITY;
                        a.ws.zbuf[zrow(a, b, kvh * G + hh) + (size_t)pi.upos * P + t] = z;
                        if (v & 1) zmx1 = fmaxf(zmx1, z);
                        else zmx0 = fmaxf(zmx0, z);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);
        }
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
            zmx0 = fmaxf(zmx0, __shfl_xor_sync(FULL, zmx0, o));
            zmx1 = fmaxf(zmx1, __shfl_xor_sync(FULL, zmx1, o));
        }
        if (lane < 4) {
            if (h0 < G && zmx0 > -INFINITY) atomicMax(&a.ws.zmax[b * a.Hq + kvh * G + h0], f2ord(zmx0));
            if (h0 + 1 < G && zmx1 > -INFINITY) atomicMax(&a.ws.zmax[b * a.Hq + kvh * G + h0 + 1], f2ord(zmx1));
        }
    } else {
        // G == 1: thread per token, q broadcast from shared memory
        float zmx = -INFINITY;
        const int tau_i = threadIdx.x;  // token within the stage
        for (int it = 0; it < my_n; ++it) {
            const int st = it % NS, ph = (it / NS) & 1;
            if (!mbar_wait(&full[st], ph, a.status)) return;
            const unsigned char *stage = stages + (size_t)st * RG::STAGE;
            const PageInfo pi = pinfo[st * PPS_MAX + tau_i / P];
            const int r = tau_i % P;
            if (pi.page >= 0) {
                float acc = 0.f;
                const bool use = r < pi.nval && (pi.mask & 1);
                if (use) {
                    const unsigned char *pbase = stage + (size_t)(tau_i / P) * P * D * 2;
#pragma unroll
                    for (int c16 = 0; c16 < D / 8; ++c16) {
                        const uint4 kv = *reinterpret_cast<const uint4 *>(tile_chunk<D>(pbase, P, r, c16));
                        const float4 q0 = *reinterpret_cast<const float4 *>(qs + 8 * c16);
                        const float4 q1 = *reinterpret_cast<const float4 *>(qs + 8 * c16 + 4);
                        acc = fmaf(q0.x, bf16lo(kv.x), acc);
                        acc = fmaf(q0.y, bf16hi(kv.x), acc);
                        acc = fmaf(q0.z, bf16lo(kv.y), acc);
                        acc = fmaf(q0.w, bf16hi(kv.y), acc);
                        acc = fmaf(q1.x, bf16lo(kv.z), acc);
                        acc = fmaf(q1.y, bf16hi(kv.z), acc);
                        acc = fmaf(q1.z, bf16lo(kv.w), acc);
                        acc = fmaf(q1.w, bf16hi(kv.w), acc);
                    }
                }
                const float z = use ? acc * zs : -INFINITY;
                a.ws.zbuf[zrow(a, b, kvh) + (size_t)pi.upos * P + r] = z;
                zmx = fmaxf(zmx, z);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) zmx = fmaxf(zmx, __shfl_xor_sync(FULL, zmx, o));
        if (lane == 0 && zmx > -INFINITY) atomicMax(&a.ws.zmax[b * a.Hq + kvh], f2ord(zmx));
    }
}

// ------------------------------------------------------------------- tau

constexpr int TAU_THREADS = 512;
constexpr int ZCAP = 11008;  // on-chip candidates per head (static shared memory)

__global__ void __launch_bounds__(TAU_THREADS) tau_kernel(const __grid_constant__ DecodeArgs a, int dense) {
    __shared__ float cz[ZCAP];
    __shared__ float red[16][33];
    __shared__ int ncand;
    __shared__ float br[2];
    const int bh = blockIdx.x;
    const int b = bh / a.Hq, h = bh % a.Hq;
    const int kvh = h / (a.Hq / a.Hkv);
    const int np = n_pages_of(a.seq_lens[b], a.P);
    const int U = dense ? np : a.ws.union_cnt[b * a.Hkv + kvh];
    const int n_tok = U * a.P;
    const float zmax = ord2f(a.ws.zmax[bh]);
    const float r = 1.f / (a.alpha - 1.f);
    const int ri = a.r_int;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (!(zmax > -INFINITY)) {  // no token at all
        if (threadIdx.x == 0) {
            a.ws.tau[bh] = __int_as_float(0x7fc00000);
            if (a.tau_out) a.tau_out[bh] = __int_as_float(0x7fc00000);
        }
        return;
    }
    const float thr = zmax - 1.f;
    const float *zr = a.ws.zbuf + zrow(a, b, h);
    if (threadIdx.x == 0) ncand = 0;
    __syncthreads();
    const int nround = ceil_div(n_tok, TAU_THREADS) * TAU_THREADS;
    for (int i = threadIdx.x; i < nround; i += TAU_THREADS) {
        const float z = i < n_tok ? __ldcg(zr + i) : -INFINITY;
        const bool c = z > thr;
        const unsigned bal = __ballot_sync(FULL, c);
        int base = 0;
        if (lane == 0 && bal) base = atomicAdd(&ncand, __popc(bal));
        base = __shfl_sync(FULL, base, 0);
        if (c) {
            const int slot = base + __popc(bal & ((1u << lane) - 1u));
            if (slot < ZCAP) cz[slot] = z;
        }
    }
    __syncthreads();
    const int nc = ncand;
    const bool onchip = nc <= ZCAP;
    if (!onchip && threadIdx.x == 0) atomicOr(a.status, ENTMAXKV_STATUS_OVERFLOW);

    float lo = thr;
    float hi = zmax - powf((float)nc, 1.f - a.alpha);
    if (nc > 1 && hi > lo) {
        const float tol = 1e-7f * fmaxf(1.f, fabsf(zmax));
        if (onchip && nc <= 256) {
            // every thread evaluates one point over all candidates
            for (int pass = 0; pass < 4 && hi - lo > tol; ++pass) {
                const float w = (hi - lo) / (float)(TAU_THREADS + 1);
                const float t = lo + w * (float)(threadIdx.x + 1);
                float f = 0.f;
                for (int c = 0; c < nc; ++c) f += pos_pow(cz[c] - t, r, ri);
                const bool ge = f >= 1.f;  // still left of the root
                const unsigned bal = __ballot_sync(FULL, ge);
                __syncthreads();
                if (lane == 0) reinterpret_cast<unsigned *>(&red[0][0])[warp] = bal;
                __syncthreads();
                // points are increasing in thread order and f decreases, so the
                // "ge" flags form a prefix; count them
                int cntge = 0;
                for (int ww = 0; ww < TAU_THREADS / 32; ++ww) cntge += __popc(reinterpret_cast<unsigned *>(&red[0][0])[ww]);
                const float nlo = cntge > 0 ? lo + w * (float)cntge : lo;
                const float nhi = cntge < TAU_THREADS ? lo + w * (float)(cntge + 1) : hi;
                lo = nlo;
                hi = nhi;
                __syncthreads();
            }
        } else {
            // 32 points per pass, candidates spread over the block
            for (int pass = 0; pass < 12 && hi - lo > tol; ++pass) {
                const float w = (hi - lo) / 33.f;
                float f[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) f[j] = 0.f;
                if (onchip) {
                    for (int c = threadIdx.x; c < nc; c += TAU_THREADS) {
                        const float z = cz[c];
#pragma unroll
                        for (int j = 0; j < 32; ++j) f[j] += pos_pow(z - (lo + w * (float)(j + 1)), r, ri);
                    }
                } else {
                    for (int i = threadIdx.x; i < n_tok; i += TAU_THREADS) {
                        const float z = __ldcg(zr + i);
                        if (!(z > thr)) continue;
#pragma unroll
                        for (int j = 0; j < 32; ++j) f[j] += pos_pow(z - (lo + w * (float)(j + 1)), r, ri);
                    }
                }
                // transpose-reduce: lane l ends with the warp sum of point l
#pragma unroll
                for (int s = 16; s >= 1; s >>= 1) {
#pragma unroll
                    for (int i = 0; i < s; ++i) {
                        const bool up = lane & s;
                        const float send = up ? f[i] : f[i + s];
                        const float keep = up ? f[i + s] : f[i];
                        f[i] = keep + __shfl_xor_sync(FULL, send, s);
                    }
                }
                red[warp][lane] = f[0];
                __syncthreads();
                if (warp == 0) {
                    float tot = 0.f;
                    for (int ww = 0; ww < TAU_THREADS / 32; ++ww) tot += red[ww][lane];
                    const unsigned bal = __ballot_sync(FULL, tot >= 1.f);
                    if (lane == 0) {
                        const int cntge = __popc(bal);
                        br[0] = cntge > 0 ? lo + w * (float)cntge : lo;
                        br[1] = cntge < 32 ? lo + w * (float)(cntge + 1) : hi;
                    }
                }
                __syncthreads();
                lo = br[0];
                hi = br[1];
                __syncthreads();
            }
        }
    } else {
        hi = lo;
    }
    if (threadIdx.x == 0) {
        const float tau = 0.5f * (lo + hi);
        a.ws.tau[bh] = tau;
        if (a.tau_out) a.tau_out[bh] = tau;
    }
}

// ------------------------------------------------- partial-sum combination

// Called by all threads of a CTA after it wrote its partial for the heads of
// group bk.  The last CTA of the group to arrive sums the S partials of each
// head in slot order and writes the output.
template <int D, int G>
__device__ __forceinline__ void combine_last(const DecodeArgs &a, int bk, int b, int kvh, int S, bool softmax) {
    __shared__ int s_last;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = atomicAdd(&a.ws.counters[bk], 1) == S - 1;
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    const int BH = a.B * a.Hq;
    for (int i = threadIdx.x; i < G * D; i += blockDim.x) {
        const int g = i / D, j = i % D;
        const int bh = b * a.Hq + kvh * G + g;
        if (!softmax) {
            float s = 0.f;
            for (int sl = 0; sl < S; ++sl) s += __ldcg(&a.ws.partial[((size_t)sl * BH + bh) * (D + 2) + 2 + j]);
            a.out[(size_t)bh * D + j] = s;
        } else {
            float M = -INFINITY;
            for (int sl = 0; sl < S; ++sl) M = fmaxf(M, __ldcg(&a.ws.partial[((size_t)sl * BH + bh) * (D + 2)]));
            float num = 0.f, den = 0.f;
            for (int sl = 0; sl < S; ++sl) {
                const float *pp = &a.ws.partial[((size_t)sl * BH + bh) * (D + 2)];
                const float m = __ldcg(pp);
                if (!(m > -INFINITY)) continue;
                const float sc = expf(m - M);
                den += sc * __ldcg(pp + 1);
                num += sc * __ldcg(pp + 2 + j);
            }
            a.out[(size_t)bh * D + j] = den > 0.f ? num / den : 0.f;
            if (j == 0 && a.tau_out) a.tau_out[bh] = M;
        }
    }
    if (threadIdx.x == 0) a.ws.counters[bk] = 0;
}

// ----------------------------------------------------- p.V, sparse gather

constexpr int PV_THREADS = 128;

template <int D, int G>
__global__ void __launch_bounds__(PV_THREADS) pv_gather_kernel(const __grid_constant__ DecodeArgs a) {
    constexpr int CPL = D / 32;  // coordinates per lane
    __shared__ float red[PV_THREADS / 32][G][D];
    const int bk = blockIdx.y;
    const int b = bk / a.Hkv, kvh = bk % a.Hkv;
    const int P = a.P;
    const int seq = a.seq_lens[b];
    const int U = a.ws.union_cnt[bk];
    const int S = gridDim.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const float r = 1.f / (a.alpha - 1.f);
    const int ri = a.r_int;
    float tau[G];
#pragma unroll
    for (int g = 0; g < G; ++g) tau[g] = a.ws.tau[b * a.Hq + kvh * G + g];
    float acc[G][CPL];
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
        for (int c = 0; c < CPL; ++c) acc[g][c] = 0.f;

    const size_t lstride = (size_t)a.max_pages * P;
    for (int e = blockIdx.x * (PV_THREADS / 32) + warp; e < U; e += S * (PV_THREADS / 32)) {
        const int entry = a.ws.union_e[(size_t)bk * a.max_pages + e];
        const int page = entry >> 8, mask = entry & 0xff;
        const int blk = a.page_table[(size_t)b * a.max_pages + page];
        if (blk < 0 || blk >= a.num_blocks) continue;  // flagged by qk_kernel
        const int nval = tokens_in_page(seq, P, page);
        const uint16_t *vpage = a.v + ((size_t)blk * a.Hkv + kvh) * P * D;
        for (int t0 = 0; t0 < P; t0 += 32) {
            const int t = t0 + lane;
            float p[G];
            bool any = false;
#pragma unroll
            for (int g = 0; g < G; ++g) {
                p[g] = 0.f;
                if (t < nval && ((mask >> g) & 1)) {
                    const float z = __ldcg(a.ws.zbuf + zrow(a, b, kvh * G + g) + (size_t)e * P + t);
                    p[g] = pos_pow(z - tau[g], r, ri);
                    if (a.p_out) a.p_out[((size_t)b * a.Hq + kvh * G + g) * lstride + (size_t)page * P + t] = p[g];
                }
                any |= p[g] > 0.f;
            }
            unsigned bal = __ballot_sync(FULL, any);
            while (bal) {
                // up to 8 rows in flight at once
                int rows[8], nr = 0;
                while (bal && nr < 8) {
                    rows[nr++] = __ffs(bal) - 1;
                    bal &= bal - 1;
                }
                float vv[8][CPL];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    if (i < nr) {
                        const uint16_t *row = vpage + (size_t)(t0 + rows[i]) * D + lane * CPL;
                        if (CPL == 4) {
                            const uint2 w = __ldg(reinterpret_cast<const uint2 *>(row));
                            vv[i][0] = bf16lo(w.x);
                            vv[i][1] = bf16hi(w.x);
                            vv[i][2] = bf16lo(w.y);
                            vv[i][3] = bf16hi(w.y);
                        } else {
                            const unsigned w = __ldg(reinterpret_cast<const unsigned *>(row));
                            vv[i][0] = bf16lo(w);
                            vv[i][1] = bf16hi(w);
                        }
                    }
                }
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    if (i < nr) {
#pragma unroll
                        for (int g = 0; g < G; ++g) {
                            const float pg = __shfl_sync(FULL, p[g], rows[i]);
#pragma unroll
                            for (int c = 0; c < CPL; ++c) acc[g][c] = fmaf(pg, vv[i][c], acc[g][c]);
                        }
                    }
                }
            }
        }
    }
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
        for (int c = 0; c < CPL; ++c) red[warp][g][lane * CPL + c] = acc[g][c];
    __syncthreads();
    const int BH = a.B * a.Hq;
    for (int i = threadIdx.x; i < G * D; i += PV_THREADS) {
        const int g = i / D, j = i % D;
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < PV_THREADS / 32; ++w) s += red[w][g][j];
        a.ws.partial[((size_t)blockIdx.x * BH + b * a.Hq + kvh * G + g) * (D + 2) + 2 + j] = s;
    }
    combine_last<D, G>(a, bk, b, kvh, S, false);
}

// ------------------------------------------------- p.V, full-cache stream

template <int D, int G>
__global__ void __launch_bounds__(DEC_THREADS) pv_stream_kernel(const __grid_constant__ DecodeArgs a) {
    constexpr int NS = 4;
    using RG = Ring<D, G, NS, 1>;
    constexpr int TPS = RG::TPS;
    constexpr int CPL = D / 32;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *stages = reinterpret_cast<unsigned char *>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint64_t *full = reinterpret_cast<uint64_t *>(stages + (size_t)NS * RG::STAGE);
    uint64_t *empty = full + NS;
    PageInfo *pinfo = reinterpret_cast<PageInfo *>(empty + NS);
    __shared__ float red[NWC][G][D];

    const int bk = blockIdx.y;
    const int b = bk / a.Hkv, kvh = bk % a.Hkv;
    const int P = a.P, PPS = TPS / P;
    const int seq = a.seq_lens[b];
    const int np = n_pages_of(seq, P);
    const int nsteps = ceil_div(np, PPS);
    const int S = gridDim.x;
    const int my_n = nsteps > (int)blockIdx.x ? ceil_div(nsteps - blockIdx.x, S) : 0;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], NWC);
        }
        mbar_fence_init();
    }
    __syncthreads();

    float acc[G][CPL];
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
        for (int c = 0; c < CPL; ++c) acc[g][c] = 0.f;

    if (warp == NWC) {
        if (lane == 0) {
            prefetch_tmap(&a.kmap);
            for (int it = 0; it < my_n; ++it) {
                const int st = it % NS, ph = (it / NS) & 1;
                if (!mbar_wait(&empty[st], ph ^ 1, a.status)) break;
                // a.kmap is the V map for this kernel (set by the launcher)
                produce_step<D, 1>(a, true, b, kvh, bk, np, blockIdx.x + it * S, PPS, stages + (size_t)st * RG::STAGE,
                                   0, &full[st], pinfo + st * PPS_MAX);
            }
        }
    } else {
        const float r = 1.f / (a.alpha - 1.f);
        const int ri = a.r_int;
        float tau[G];
#pragma unroll
        for (int g = 0; g < G; ++g) tau[g] = a.ws.tau[b * a.Hq + kvh * G + g];
        const size_t lstride = (size_t)a.max_pages * P;
        bool ok = true;
        for (int it = 0; it < my_n && ok; ++it) {
            const int st = it % NS, ph = (it / NS) & 1;
            if (!mbar_wait(&full[st], ph, a.status)) {
                ok = false;
                break;
            }
            const unsigned char *stage = stages + (size_t)st * RG::STAGE;
            const PageInfo *pis = pinfo + st * PPS_MAX;
            for (int bt = warp; bt < TPS / 32; bt += NWC) {
                const int tk = bt * 32 + lane;
                const int pi_i = tk / P, rr = tk % P;
                const PageInfo pi = pis[pi_i];
                float p[G];
                bool any = false;
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    p[g] = 0.f;
                    if (pi.page >= 0 && rr < pi.nval) {
                        const float z = __ldcg(a.ws.zbuf + zrow(a, b, kvh * G + g) + (size_t)pi.page * P + rr);
                        p[g] = pos_pow(z - tau[g], r, ri);
                        if (a.p_out)
                            a.p_out[((size_t)b * a.Hq + kvh * G + g) * lstride + (size_t)pi.page * P + rr] = p[g];
                    }
                    any |= p[g] > 0.f;
                }
                unsigned bal = __ballot_sync(FULL, any);
                while (bal) {
                    const int tt = __ffs(bal) - 1;
                    bal &= bal - 1;
                    const int tk2 = bt * 32 + tt;
                    const int pj = tk2 / P, r2 = tk2 % P;
                    const unsigned char *pbase = stage + (size_t)pj * P * D * 2;
                    float vv[CPL];
                    if (CPL == 4) {
                        const uint2 w = *reinterpret_cast<const uint2 *>(tile_chunk<D>(pbase, P, r2, lane >> 1) + (lane & 1) * 8);
                        vv[0] = bf16lo(w.x);
                        vv[1] = bf16hi(w.x);
                        vv[2] = bf16lo(w.y);
                        vv[3] = bf16hi(w.y);
                    } else {
                        const unsigned w = *reinterpret_cast<const unsigned *>(tile_chunk<D>(pbase, P, r2, lane >> 2) + (lane & 3) * 4);
                        vv[0] = bf16lo(w);
                        vv[1] = bf16hi(w);
                    }
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        const float pg = __shfl_sync(FULL, p[g], tt);
#pragma unroll
                        for (int c = 0; c < CPL; ++c) acc[g][c] = fmaf(pg, vv[c], acc[g][c]);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);
        }
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int c = 0; c < CPL; ++c) red[warp][g][lane * CPL + c] = acc[g][c];
    }
    __syncthreads();
    const int BH = a.B * a.Hq;
    for (int i = threadIdx.x; i < G * D; i += blockDim.x) {
        const int g = i / D, j = i % D;
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < NWC; ++w) s += red[w][g][j];
        a.ws.partial[((size_t)blockIdx.x * BH + b * a.Hq + kvh * G + g) * (D + 2) + 2 + j] = s;
    }
    combine_last<D, G>(a, bk, b, kvh, S, false);
}

// ----------------------------------------------------- softmax split-K

template <int D, int G>
__global__ void __launch_bounds__(DEC_THREADS) softmax_kernel(const __grid_constant__ DecodeArgs a) {
    constexpr int NS = 3;
    using RG = Ring<D, G, NS, 2>;
    constexpr int TPS = RG::TPS;
    constexpr int CPL = D / 32;
    constexpr int HALF = RG::STAGE / 2;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *stages = reinterpret_cast<unsigned char *>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint64_t *full = reinterpret_cast<uint64_t *>(stages + (size_t)NS * RG::STAGE);
    uint64_t *empty = full + NS;
    PageInfo *pinfo = reinterpret_cast<PageInfo *>(empty + NS);
    __shared__ float st_s[2][TPS][G];  // scores of the stage, double-buffered
    __shared__ float qs[G == 1 ? D : 1];
    __shared__ float red[NWC][G][D];
    __shared__ float redl[NWC][G];
    __shared__ int s_abort;

    const int bk = blockIdx.y;
    const int b = bk / a.Hkv, kvh = bk % a.Hkv;
    const int P = a.P, PPS = TPS / P;
    const int seq = a.seq_lens[b];
    const int np = n_pages_of(seq, P);
    const int nsteps = ceil_div(np, PPS);
    const int S = gridDim.x;
    const int my_n = nsteps > (int)blockIdx.x ? ceil_div(nsteps - blockIdx.x, S) : 0;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float sscale = D == 64 ? 0.125f : 0.08838834764831845f;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], NWC);
        }
        mbar_fence_init();
    }
    if (G == 1)
        for (int j = threadIdx.x; j < D; j += blockDim.x) qs[j] = bf16f(a.q[((size_t)b * a.Hq + kvh) * D + j]);
    if (threadIdx.x == 0) s_abort = 0;
    __syncthreads();

    float m[G], l[G], acc[G][CPL];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        m[g] = -INFINITY;
        l[g] = 0.f;
#pragma unroll
        for (int c = 0; c < CPL; ++c) acc[g][c] = 0.f;
    }

    if (warp == NWC) {
        if (lane == 0) {
            prefetch_tmap(&a.kmap);
            prefetch_tmap(&a.vmap);
            for (int it = 0; it < my_n; ++it) {
                const int st = it % NS, ph = (it / NS) & 1;
                if (!mbar_wait(&empty[st], ph ^ 1, a.status)) break;
                produce_step<D, 2>(a, true, b, kvh, bk, np, blockIdx.x + it * S, PPS, stages + (size_t)st * RG::STAGE,
                                   HALF, &full[st], pinfo + st * PPS_MAX);
            }
        }
    } else {
        unsigned qb[G >= 2 ? D / 16 : 1][2];
        if constexpr (G >= 2) {
            const int n = lane >> 2, kp = 2 * (lane & 3);
            const uint16_t *qh = a.q + ((size_t)b * a.Hq + kvh * G + (n < G ? n : 0)) * D;
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                qb[ks][0] = n < G ? *reinterpret_cast<const unsigned *>(qh + 16 * ks + kp) : 0u;
                qb[ks][1] = n < G ? *reinterpret_cast<const unsigned *>(qh + 16 * ks + kp + 8) : 0u;
            }
        }
        for (int it = 0; it < my_n; ++it) {
            const int st = it % NS, ph = (it / NS) & 1;
            // a warp whose wait ran out still takes part in the named barrier
            // below; all consumer warps then leave together
            const bool ready = mbar_wait(&full[st], ph, a.status);
            if (!ready) s_abort = 1;
            const unsigned char *stage = stages + (size_t)st * RG::STAGE;
            const PageInfo *pis = pinfo + st * PPS_MAX;
            float(*sc)[G] = st_s[it & 1];
            // scores of the stage's tokens
            if (!ready) {
            } else if constexpr (G >= 2) {
                for (int mt = warp; mt < TPS / 16; mt += NWC) {
                    const int tok0 = mt * 16, pi_i = tok0 / P, r0 = tok0 % P;
                    const PageInfo pi = pis[pi_i];
                    float c4[4] = {0.f, 0.f, 0.f, 0.f};
                    if (pi.nval > 0) {
                        const unsigned char *pbase = stage + (size_t)pi_i * P * D * 2;
                        const int mat = lane >> 3, rr = lane & 7;
                        const int row = r0 + (mat & 1) * 8 + rr;
#pragma unroll
                        for (int ks = 0; ks < D / 16; ++ks) {
                            unsigned a0, a1, a2, a3;
                            ldsm_x4(smem_u32(tile_chunk<D>(pbase, P, row, ks * 2 + (mat >> 1))), a0, a1, a2, a3);
                            mma_bf16_16816(c4, a0, a1, a2, a3, qb[ks][0], qb[ks][1]);
                        }
                    }
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        const int hh = 2 * (lane & 3) + (v & 1);
                        const int t = r0 + (lane >> 2) + (v >= 2 ? 8 : 0);
                        if (hh < G) sc[tok0 - r0 + t][hh] = (t < pi.nval) ? c4[v] * sscale : -INFINITY;
                    }
                }
            } else {
                const int tk = threadIdx.x;  // 128 consumer threads, TPS == 128
                const int pi_i = tk / P, r = tk % P;
                const PageInfo pi = pis[pi_i];
                float s = -INFINITY;
                if (r < pi.nval) {
                    const unsigned char *pbase = stage + (size_t)pi_i * P * D * 2;
                    float accd = 0.f;
#pragma unroll
                    for (int c16 = 0; c16 < D / 8; ++c16) {
                        const uint4 kv = *reinterpret_cast<const uint4 *>(tile_chunk<D>(pbase, P, r, c16));
                        const float4 q0 = *reinterpret_cast<const float4 *>(qs + 8 * c16);
                        const float4 q1 = *reinterpret_cast<const float4 *>(qs + 8 * c16 + 4);
                        accd = fmaf(q0.x, bf16lo(kv.x), accd);
                        accd = fmaf(q0.y, bf16hi(kv.x), accd);
                        accd = fmaf(q0.z, bf16lo(kv.y), accd);
                        accd = fmaf(q0.w, bf16hi(kv.y), accd);
                        accd = fmaf(q1.x, bf16lo(kv.z), accd);
                        accd = fmaf(q1.y, bf16hi(kv.z), accd);
                        accd = fmaf(q1.z, bf16lo(kv.w), accd);
                        accd = fmaf(q1.w, bf16hi(kv.w), accd);
                    }
                    s = accd * sscale;
                }
                sc[tk][0] = s;
            }
            asm volatile("bar.sync 1, %0;" ::"n"(NWC * 32) : "memory");
            if (s_abort) break;
            // tile max per head (every warp computes it identically)
            float mn[G], scl[G];
#pragma unroll
            for (int g = 0; g < G; ++g) {
                float x = -INFINITY;
                for (int t = lane; t < TPS; t += 32) x = fmaxf(x, sc[t][g]);
#pragma unroll
                for (int o = 16; o; o >>= 1) x = fmaxf(x, __shfl_xor_sync(FULL, x, o));
                mn[g] = fmaxf(m[g], x);
                scl[g] = (mn[g] == -INFINITY) ? 1.f : expf(m[g] - mn[g]);
                m[g] = mn[g];
                l[g] *= scl[g];
#pragma unroll
                for (int c = 0; c < CPL; ++c) acc[g][c] *= scl[g];
            }
            for (int t = warp; t < TPS; t += NWC) {
                const int pj = t / P, r2 = t % P;
                const PageInfo pi = pis[pj];
                if (r2 >= pi.nval) continue;
                const unsigned char *vbase = stage + HALF + (size_t)pj * P * D * 2;
                float vv[CPL];
                if (CPL == 4) {
                    const uint2 w = *reinterpret_cast<const uint2 *>(tile_chunk<D>(vbase, P, r2, lane >> 1) + (lane & 1) * 8);
                    vv[0] = bf16lo(w.x);
                    vv[1] = bf16hi(w.x);
                    vv[2] = bf16lo(w.y);
                    vv[3] = bf16hi(w.y);
                } else {
                    const unsigned w = *reinterpret_cast<const unsigned *>(tile_chunk<D>(vbase, P, r2, lane >> 2) + (lane & 3) * 4);
                    vv[0] = bf16lo(w);
                    vv[1] = bf16hi(w);
                }
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    const float p = expf(sc[t][g] - m[g]);
                    l[g] += p;
#pragma unroll
                    for (int c = 0; c < CPL; ++c) acc[g][c] = fmaf(p, vv[c], acc[g][c]);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);
        }
#pragma unroll
        for (int g = 0; g < G; ++g) {
#pragma unroll
            for (int c = 0; c < CPL; ++c) red[warp][g][lane * CPL + c] = acc[g][c];
            if (lane == 0) redl[warp][g] = l[g];
        }
    }
    __syncthreads();
    // all consumer warps share m; sum l and acc over warps
    const int BH = a.B * a.Hq;
    for (int i = threadIdx.x; i < G * D; i += blockDim.x) {
        const int g = i / D, j = i % D;
        const size_t o = ((size_t)blockIdx.x * BH + b * a.Hq + kvh * G + g) * (D + 2);
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < NWC; ++w) s += red[w][g][j];
        a.ws.partial[o + 2 + j] = s;
        if (j == 0) {
            float ls = 0.f;
#pragma unroll
            for (int w = 0; w < NWC; ++w) ls += redl[w][g];
            a.ws.partial[o + 1] = ls;
        }
    }
    // m lives in the consumer warps' registers; warp 0 lane 0 publishes it
    if (threadIdx.x == 0) {
#pragma unroll
        for (int g = 0; g < G; ++g) a.ws.partial[((size_t)blockIdx.x * BH + b * a.Hq + kvh * G + g) * (D + 2)] = m[g];
    }
    combine_last<D, G>(a, bk, b, kvh, S, true);
}

// ---------------------------------------------------------------- launch

int pick_splits(int sms, int per_sm, int groups, int max_steps, int cap) {
    int s = ceil_div(sms * per_sm, groups > 0 ? groups : 1);
    if (s > max_steps) s = max_steps;
    if (s > cap) s = cap;
    return s < 1 ? 1 : s;
}

template <int D, int G>
cudaError_t sparse_t(const DecodeArgs &a, cudaStream_t st) {
    cudaError_t e;
    const int groups = a.B * a.Hkv;
    const size_t ub = (size_t)ceil_div(a.max_pages, 4) * 4;
    if ((e = cudaFuncSetAttribute(union_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ub)) != cudaSuccess)
        return e;
    union_kernel<<<groups, 512, ub, st>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;

    using RG = Ring<D, G, 4, 1>;
    const int PPS = RG::TPS / a.P;
    {
        auto k = qk_kernel<D, G, false>;
        if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)RG::BYTES)) != cudaSuccess)
            return e;
        const int S = pick_splits(a.sms, 3, groups, ceil_div(a.max_pages, PPS), 1 << 16);
        k<<<dim3(S, groups), DEC_THREADS, RG::BYTES, st>>>(a);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    tau_kernel<<<a.B * a.Hq, TAU_THREADS, 0, st>>>(a, 0);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    {
        const int S = pick_splits(a.sms, 4, groups, ceil_div(a.max_pages, PV_THREADS / 32), MAX_SPLITS);
        pv_gather_kernel<D, G><<<dim3(S, groups), PV_THREADS, 0, st>>>(a);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

template <int D, int G>
cudaError_t dense_entmax_t(const DecodeArgs &a, cudaStream_t st) {
    cudaError_t e;
    const int groups = a.B * a.Hkv;
    const int n = a.B * a.Hq > groups ? a.B * a.Hq : groups;
    dense_init_kernel<<<ceil_div(n, 256), 256, 0, st>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    using RG = Ring<D, G, 4, 1>;
    const int PPS = RG::TPS / a.P;
    {
        auto k = qk_kernel<D, G, true>;
        if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)RG::BYTES)) != cudaSuccess)
            return e;
        const int S = pick_splits(a.sms, 3, groups, ceil_div(a.max_pages, PPS), 1 << 16);
        k<<<dim3(S, groups), DEC_THREADS, RG::BYTES, st>>>(a);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    tau_kernel<<<a.B * a.Hq, TAU_THREADS, 0, st>>>(a, 1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    {
        DecodeArgs av = a;
        av.kmap = a.vmap;  // the stream kernel loads V through the first map slot
        auto k = pv_stream_kernel<D, G>;
        if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)RG::BYTES)) != cudaSuccess)
            return e;
        const int S = pick_splits(a.sms, 3, groups, ceil_div(a.max_pages, PPS), MAX_SPLITS);
        k<<<dim3(S, groups), DEC_THREADS, RG::BYTES, st>>>(av);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

template <int D, int G>
cudaError_t dense_softmax_t(const DecodeArgs &a, cudaStream_t st) {
    cudaError_t e;
    const int groups = a.B * a.Hkv;
    const int n = a.B * a.Hq > groups ? a.B * a.Hq : groups;
    dense_init_kernel<<<ceil_div(n, 256), 256, 0, st>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    using RG = Ring<D, G, 3, 2>;
    const int PPS = RG::TPS / a.P;
    auto k = softmax_kernel<D, G>;
    if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)RG::BYTES)) != cudaSuccess)
        return e;
    const int S = pick_splits(a.sms, 2, groups, ceil_div(a.max_pages, PPS), MAX_SPLITS);
    k<<<dim3(S, groups), DEC_THREADS, RG::BYTES, st>>>(a);
    return cudaGetLastError();
}

}  // namespace

#define EKV_DISPATCH(FN, a, st)                                        \
    do {                                                               \
        const int G_ = (a).Hq / (a).Hkv;                               \
        if ((a).d == 64) {                                             \
            switch (G_) {                                              \
                case 1: return FN<64, 1>(a, st);                       \
                case 2: return FN<64, 2>(a, st);                       \
                case 4: return FN<64, 4>(a, st);                       \
                case 8: return FN<64, 8>(a, st);                       \
            }                                                          \
        } else {                                                       \
            switch (G_) {                                              \
                case 1: return FN<128, 1>(a, st);                      \
                case 2: return FN<128, 2>(a, st);                      \
                case 4: return FN<128, 4>(a, st);                      \
                case 8: return FN<128, 8>(a, st);                      \
            }                                                          \
        }                                                              \
        return cudaErrorInvalidValue;                                  \
    } while (0)

cudaError_t launch_decode_sparse(const DecodeArgs &a, cudaStream_t st) { EKV_DISPATCH(sparse_t, a, st); }
cudaError_t launch_decode_dense_entmax(const DecodeArgs &a, cudaStream_t st) { EKV_DISPATCH(dense_entmax_t, a, st); }
cudaError_t launch_decode_dense_softmax(const DecodeArgs &a, cudaStream_t st) { EKV_DISPATCH(dense_softmax_t, a, st); }

size_t decode_ws_bytes(int B, int Hq, int Hkv, int d, int P, int max_pages, DecodeWs *carve, void *base) {
    size_t off = 0;
    auto take = [&](size_t bytes) {
        size_t o = off;
        off += (bytes + 255) & ~(size_t)255;
        return o;
    };
    const size_t o_union = take((size_t)B * Hkv * max_pages * 4);
    const size_t o_ucnt = take((size_t)B * Hkv * 4);
    const size_t o_zmax = take((size_t)B * Hq * 4);
    const size_t o_tau = take((size_t)B * Hq * 4);
    const size_t o_cnt = take((size_t)B * Hkv * 4);
    const size_t o_part = take((size_t)MAX_SPLITS * B * Hq * (d + 2) * 4);
    const size_t o_z = take((size_t)B * Hq * max_pages * P * 4);
    if (carve && base) {
        char *p = static_cast<char *>(base);
        carve->union_e = reinterpret_cast<int *>(p + o_union);
        carve->union_cnt = reinterpret_cast<int *>(p + o_ucnt);
        carve->zmax = reinterpret_cast<int *>(p + o_zmax);
        carve->tau = reinterpret_cast<float *>(p + o_tau);
        carve->counters = reinterpret_cast<int *>(p + o_cnt);
        carve->partial = reinterpret_cast<float *>(p + o_part);
        carve->zbuf = reinterpret_cast<float *>(p + o_z);
    }
    return off;
}

}  // namespace ekv
