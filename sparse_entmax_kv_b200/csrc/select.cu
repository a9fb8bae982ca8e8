// select.cu -- candidate page selection (EntmaxKV summary, section 2.B).
//
// One CTA per (sequence, query head), or for the Gaussian policies on rows of
// up to 16384 pages a cluster of four.  In the fused decode step the kernels
// also prepare each GQA group's union of selected pages (below).
//
// Top-k: radix select on the order-preserving 32-bit image of the fp32 bound
// (four 8-bit digits, most significant first; per-warp shared-memory
// histograms summed after each pass), which pins the k-th largest key T and how many keys equal to T
// are still needed; a single ordered pass then keeps keys > T plus the first
// such keys == T in page order (ties to the lower page index) and writes them
// in ascending page order.  No sort.
//
// Gaussian (and its estimated-max variant, which keeps a page when
// (alpha-1) min(bound, mu + sqrt(2 ln n) sigma) clears the cut):
// tau_hat solves F(tau) = sum_p n_p E[(X_p - tau)_+^r] = 1 with
// X_p ~ N(m_p, s_p^2), m_p = (alpha-1) mu_p, s_p = (alpha-1) sigma_p, using the
// closed-form Gaussian partial moments.  F is decreasing, F >= 1 at
// tau0 = max_p (m_p - n_p^(-1/r)) (Jensen) and F < 1 at max_p (m_p + 10 s_p)
// (every page is then 10 standard deviations into its tail).  Pages with
// m_p + 10 s_p < tau0 contribute below n_p s_p^r J_r(10) ~ 1e-25 n_p s_p^r
// anywhere in that bracket and are pruned.  Newton's method on F^(1/r),
// which is convex, climbs from tau0 to the root without overshooting.  Pages
// are then kept when (alpha-1) bbox_p > tau_hat - Delta.
#include "common.cuh"
#include "internal.h"

namespace ekv {

namespace {

constexpr int SEL_THREADS = 1024;
constexpr int ITEMS = 16;  // keys per thread per tile
constexpr int TILE = SEL_THREADS * ITEMS;

__device__ __forceinline__ unsigned key_of(float f) {
    unsigned x = __float_as_uint(f);
    return (x & 0x80000000u) ? ~x : (x | 0x80000000u);
}




// ------------------------------------------ the group union (decode step)
//
// With a.umap set (the decode step), the selection also prepares the union
// of the G heads' selections of each (sequence, kv head) group for the q.K
// pass.  With G = 1 the selection list is the union: each entry is written
// beside the selection with its page-table entry (union_e / union_blk /
// union_cnt, as the decode workspace holds them), and the q.K pass's running
// max is reset.  With G > 1 every CTA ORs head g's bit into byte p of its
// group's row of umap for each page p it keeps (the row is zero on entry);
// a separate kernel of the decode then compacts the rows.

// Page-table entries of the kept pages among p0 .. p0+N-1 (bit i: page
// p0+i), all loads issued together; -1 elsewhere.
template <int N>
__device__ __forceinline__ void blocks_run(const int *pt, int p0, unsigned bits, int (&blk)[N]) {
#pragma unroll
    for (int i = 0; i < N; ++i) blk[i] = (bits >> i) & 1u ? __ldg(pt + p0 + i) : -1;
}

// G = 1: union entry `pos` is the kept page p with physical block blk.
__device__ __forceinline__ void union_entry(const SelectArgs &a, int *ue, int *ub, int pos, int p, int blk) {
    const bool ok = blk >= 0 && blk < a.num_blocks;
    if (!ok) atomicOr(a.status, ENTMAXKV_STATUS_BAD_PAGE);
    ue[pos] = (p << 8) | 1;
    ub[pos] = ok ? blk : -1;
}

// G > 1: marks the kept pages among p0 .. p0+N-1 (p0 and N multiples of 4)
// for head g: one OR per 4-page word holding a kept page.
template <int N>
__device__ __forceinline__ void mark_run(unsigned *row, int p0, unsigned bits, int g) {
#pragma unroll
    for (int j = 0; j < N / 4; ++j) {
        const unsigned nib = (bits >> (4 * j)) & 0xfu;
        if (nib) {
            unsigned w = 0u;
#pragma unroll
            for (int i = 0; i < 4; ++i) w |= ((nib >> i) & 1u) << (8 * i + g);
            atomicOr(row + (p0 >> 2) + j, w);
        }
    }
}

// Top-k: the keys of one tile (NT * IT pages) stay in registers, IT
// consecutive pages per thread, through the four radix passes and the final
// ordered compaction; longer sequences take several tiles per pass.
template <int NT, int IT>
__global__ void __launch_bounds__(NT) topk_kernel(SelectArgs a) {
    constexpr int TILE_NT = NT * IT;
    pdl_wait();
    __shared__ int whist[NT / 32][256];  // one histogram per warp (contention stays inside a warp)
    __shared__ int hist[256];
    __shared__ int sh[72];
    __shared__ int pick[2];
    int b, h;
    head_of(blockIdx.x, a.h0, a.nh, b, h);
    const int bh = b * a.Hq + h;
    const int n = n_pages_of(seq_len_of(a.seq_lens, b, a.P, a.max_pages, a.status), a.P);
    const float *sc = a.bbox + (size_t)bh * a.max_pages;
    int *sel = a.sel + (size_t)bh * a.max_pages;
    const int k = min(a.k, n);
    // decode step: the group's union (see above)
    const int G = a.Hq / a.Hkv;
    const bool uni = a.umap != nullptr;
    const int bk = b * a.Hkv + h / G;
    const int *pt = a.page_table + (size_t)b * a.max_pages;  // (read only when uni)
    if (k >= n) {
        unsigned *urow = a.umap + (size_t)bk * a.uwords;
        int *ue = a.union_e + (size_t)bk * a.max_pages, *ub = a.union_blk + (size_t)bk * a.max_pages;
        for (int p = threadIdx.x; p < n; p += blockDim.x) sel[p] = p;
        if (threadIdx.x == 0) a.cnt[bh] = n;
        if (uni) {
            for (int p0 = threadIdx.x * IT; p0 < n; p0 += NT * IT) {
                const unsigned bits = n - p0 >= IT ? (1u << IT) - 1u : (1u << (n - p0)) - 1u;
                if (G > 1) {
                    mark_run<IT>(a.umap + (size_t)bk * a.uwords, p0, bits, h % G);
                } else {
                    int blk[IT];
                    blocks_run<IT>(pt, p0, bits, blk);
#pragma unroll
                    for (int i = 0; i < IT; ++i)
                        if ((bits >> i) & 1u)
                            union_entry(a, a.union_e + (size_t)bk * a.max_pages,
                                        a.union_blk + (size_t)bk * a.max_pages, p0 + i, p0 + i, blk[i]);
                }
            }
            if (G == 1 && threadIdx.x == 0) {
                a.union_cnt[bk] = n;
                a.zmax[bh] = ORD_NEG_INF;
            }
        }
        return;
    }
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const bool one_tile = n <= TILE_NT;
    unsigned key[IT];
    auto load_tile = [&](int t0) {
        const int p0 = t0 + threadIdx.x * IT;
#pragma unroll
        for (int i = 0; i < IT; ++i) key[i] = (p0 + i < n) ? key_of(__ldg(sc + p0 + i)) : 0u;
    };
    if (one_tile) load_tile(0);
    unsigned prefix = 0, mask = 0;
    int remaining = k;
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = threadIdx.x; i < (NT / 32) * 256; i += blockDim.x) (&whist[0][0])[i] = 0;
        __syncthreads();
        for (int t0 = 0; t0 < n; t0 += TILE_NT) {
            if (!one_tile) load_tile(t0);
            const int p0 = t0 + threadIdx.x * IT;
#pragma unroll
            for (int i = 0; i < IT; ++i)
                if (p0 + i < n && (key[i] & mask) == prefix) atomicAdd(&whist[warp][(key[i] >> shift) & 255], 1);
        }
        __syncthreads();
        if (threadIdx.x < 256) {
            int c = 0;
#pragma unroll 8
            for (int w = 0; w < NT / 32; ++w) c += whist[w][threadIdx.x];
            hist[threadIdx.x] = c;
        }
        __syncthreads();
        if (threadIdx.x < 32) {
            // lane l owns buckets [8l, 8l+8); suffix sums from the top bucket down
            int c[8], s = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                c[i] = hist[8 * lane + i];
                s += c[i];
            }
            int suf = s;  // inclusive suffix over lanes >= lane
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                int y = __shfl_down_sync(FULL, suf, o);
                if (lane + o < 32) suf += y;
            }
            const int above = suf - s;  // keys in higher lanes' buckets
            const bool here = above < remaining && remaining <= suf;
            const unsigned who = __ballot_sync(FULL, here);
            if (lane == __ffs(who) - 1) {
                int acc = above, bsel = 8 * lane;
                for (int i = 7; i >= 0; --i) {
                    if (acc + c[i] >= remaining) {
                        bsel = 8 * lane + i;
                        break;
                    }
                    acc += c[i];
                }
                pick[0] = bsel;
                pick[1] = remaining - acc;
            }
        }
        __syncthreads();
        prefix |= (unsigned)pick[0] << shift;
        mask |= 255u << shift;
        remaining = pick[1];
        __syncthreads();
    }
    const unsigned T = prefix;
    // keys == T are taken in page order up to `remaining` of them
    int eq_base = 0, base = 0;
    unsigned u_take = 0u;  // decode step (one tile): this thread's kept pages
    int u_pos = 0;         // and the list position of the first
    for (int t0 = 0; t0 < n; t0 += TILE_NT) {
        if (!one_tile) load_tile(t0);
        const int p0 = t0 + threadIdx.x * IT;
        unsigned gt = 0, eq = 0;
#pragma unroll
        for (int i = 0; i < IT; ++i) {
            if (p0 + i < n) {
                if (key[i] > T) gt |= 1u << i;
                if (key[i] == T) eq |= 1u << i;
            }
        }
        int eq_tot;
        int eq_off = eq_base + block_excl_scan(__popc(eq), sh, &eq_tot);
        unsigned take = gt;
#pragma unroll
        for (int i = 0; i < IT; ++i)
            if (eq & (1u << i)) {
                if (eq_off < remaining) take |= 1u << i;
                ++eq_off;
            }
        if (uni && G > 1) mark_run<IT>(a.umap + (size_t)bk * a.uwords, p0, take, h % G);  // complete behind the scan
        if (uni && G == 1)  // page-table entries to L2 during the scan (no registers held)
#pragma unroll
            for (int i = 0; i < IT; ++i)
                if ((take >> i) & 1u) asm volatile("prefetch.global.L2 [%0];" ::"l"(pt + p0 + i));
        int tot;
        int w = base + block_excl_scan(__popc(take), sh, &tot);
        u_take = take;
        u_pos = w;
#pragma unroll
        for (int i = 0; i < IT; ++i)
            if (take & (1u << i)) sel[w++] = p0 + i;
        base += tot;
        eq_base += eq_tot;
    }
    if (threadIdx.x == 0) a.cnt[bh] = base;
    if (uni && G == 1) {
        // one tile (the decode step's limit): this thread's kept pages and
        // their first list position are u_take and u_pos; the keys are dead
        // now, which leaves registers for the page-table entries
        const int p0 = threadIdx.x * IT;
        int blk[IT];
        blocks_run<IT>(pt, p0, u_take, blk);
        int *ue = a.union_e + (size_t)bk * a.max_pages, *ub = a.union_blk + (size_t)bk * a.max_pages;
#pragma unroll
        for (int i = 0; i < IT; ++i)
            if ((u_take >> i) & 1u) union_entry(a, ue, ub, u_pos++, p0 + i, blk[i]);
        if (threadIdx.x == 0) {
            a.union_cnt[bk] = base;
            a.zmax[bh] = ORD_NEG_INF;
        }
    }
}

// Gaussian partial moments of a standard normal: J_R(c) = E[(Z-c)_+^R] and
// J_{R-1}(c), from M_i(c) = E[Z^i 1{Z>c}] (M_0 = erfc(c/sqrt2)/2, M_1 = phi(c),
// M_i = c^{i-1} phi(c) + (i-1) M_{i-2}) and the binomial expansion of (Z-c)^R.
__host__ __device__ constexpr float binomf(int n, int k) {
    float r = 1.f;
    for (int t = 0; t < k; ++t) r = r * (float)(n - t) / (float)(t + 1);
    return r;
}

template <int R>
__device__ __forceinline__ void gauss_JJ(float c, float &jr, float &jr1) {
    float M[R + 1], pw[R + 1];
    const float phi = 0.3989422804014327f * expf(-0.5f * c * c);
    M[0] = 0.5f * erfcf(c * 0.7071067811865476f);
    if (R >= 1) M[1] = phi;
    float cp = 1.f;  // c^{i-1}
#pragma unroll
    for (int i = 2; i <= R; ++i) {
        cp *= c;
        M[i] = cp * phi + (float)(i - 1) * M[i - 2];
    }
    pw[0] = 1.f;
#pragma unroll
    for (int i = 1; i <= R; ++i) pw[i] = pw[i - 1] * (-c);
    float s = 0.f, s1 = 0.f;
#pragma unroll
    for (int i = 0; i <= R; ++i) s += binomf(R, i) * pw[R - i] * M[i];
#pragma unroll
    for (int i = 0; i <= R - 1; ++i) s1 += binomf(R - 1, i) * pw[R - 1 - i] * M[i];
    jr = fmaxf(s, 0.f);
    jr1 = fmaxf(s1, 0.f);
}

// Adds page (m, s, weight w)'s term of F(tau) = sum_p n_p E[(X_p - tau)_+^R]
// and of its derivative F'(tau) = -R sum_p n_p E[(X_p - tau)_+^(R-1)].
template <int R>
__device__ __forceinline__ void gauss_contrib(float m, float s, float w, float tau, float &F, float &Fp) {
    if (s > 1e-30f) {
        const float c = (tau - m) / s;
        if (c > 38.f) return;
        float jr, jr1;
        gauss_JJ<R>(c, jr, jr1);
        float sp = 1.f;
#pragma unroll
        for (int i = 1; i < R; ++i) sp *= s;  // s^(R-1)
        F += w * sp * s * jr;
        Fp -= (float)R * w * sp * jr1;
    } else {
        const float x = m - tau;
        if (x > 0.f) {
            float xp = 1.f;
#pragma unroll
            for (int i = 1; i < R; ++i) xp *= x;
            F += w * xp * x;
            Fp -= (float)R * w * xp;
        }
    }
}

// Estimated maximum of n standard normal draws, sqrt(2 ln n) (0 for n = 1).
__device__ __forceinline__ float zmax_of(int n) { return n >= 2 ? sqrtf(2.f * logf((float)n)) : 0.f; }

// One Newton step on g = F^(1/R) from tau towards the root, kept below hi.
// Returns false when tau has converged (F <= 1 within 2e-6, or a step below
// 1e-7 max(1, |tau|)).
template <int R>
__device__ __forceinline__ bool newton_step(float F, float Fp, float hi, float &tau) {
    if (!(F > 1.f + 2e-6f) || !(Fp < 0.f)) return false;
    const float Fr = R == 1 ? 1.f : (R == 2 ? sqrtf(F) : powf(F, 1.f - 1.f / (float)R));  // F^(1-1/R)
    const float step = (float)R * (F - Fr) / (-Fp);
    float nt = tau + step;
    if (!(nt < hi)) nt = 0.5f * (tau + hi);  // stay inside the bracket
    const bool done = !(nt - tau > 1e-7f * fmaxf(1.f, fabsf(tau)));
    tau = nt;
    return !done;
}

constexpr int GCAP = 3072;  // pruned candidate pages held on chip

// Gaussian selection.  One tile (TILE pages, ITEMS per thread) of mu, sigma
// and the bound is loaded up front; pages are interleaved across threads for
// the max / pruning pass and contiguous per thread for the ordered
// compaction.  Newton iterations reduce F and F' with one barrier each
// (double-buffered partials).
template <int R>
__global__ void __launch_bounds__(SEL_THREADS) gauss_kernel(SelectArgs a) {
    pdl_wait();
    __shared__ float cm[GCAP], cs[GCAP], cn[GCAP];
    __shared__ float shm[32], shm2[32];
    __shared__ int shi[72];
    __shared__ int ncand;
    int b, h;
    head_of(blockIdx.x, a.h0, a.nh, b, h);
    const int bh = b * a.Hq + h;
    const int seq = seq_len_of(a.seq_lens, b, a.P, a.max_pages, a.status);
    const int n = n_pages_of(seq, a.P);
    const size_t row = (size_t)bh * a.max_pages;
    const float a1 = a.alpha - 1.f;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (n == 0) {
        if (threadIdx.x == 0) {
            a.cnt[bh] = 0;
            if (a.tau_hat) a.tau_hat[bh] = __int_as_float(0x7fc00000);
        }
        return;
    }
    const bool one_tile = n <= TILE;
    // bound of this thread's contiguous pages (for the final compaction)
    float ub[ITEMS];
    if (one_tile) {
        const int p0 = threadIdx.x * ITEMS;
#pragma unroll
        for (int i = 0; i < ITEMS; ++i) ub[i] = (p0 + i < n) ? __ldg(a.bbox + row + p0 + i) : 0.f;
    }
    // interleaved pages p = t0 + tid + SEL_THREADS*i
    float mm[ITEMS], ss[ITEMS];
    auto load_ms = [&](int t0) {
#pragma unroll
        for (int i = 0; i < ITEMS; ++i) {
            const int p = t0 + threadIdx.x + SEL_THREADS * i;
            mm[i] = p < n ? a1 * __ldg(a.mu + row + p) : -INFINITY;
            ss[i] = p < n ? a1 * __ldg(a.sigma + row + p) : 0.f;
        }
    };
    // Lower end of the bracket.  Jensen: E[(X-tau)_+^R] >= (E[X]-tau)_+^R, so
    // F(tau) >= 1 wherever some page has n_p (m_p - tau)^R >= 1, i.e.
    // tau_hat >= max_p (m_p - n_p^(-1/R)).  Every page but the sequence's last
    // is full, so the root n_p^(-1/R) takes two values.
    const float inv_r = 1.f / (float)R;
    const float drop_full = powf((float)a.P, -inv_r);
    const int n_last = tokens_in_page(seq, a.P, n - 1);
    const float drop_last = powf((float)n_last, -inv_r);
    float mloc = -INFINITY;
    for (int t0 = 0; t0 < n; t0 += TILE) {
        load_ms(t0);
#pragma unroll
        for (int i = 0; i < ITEMS; ++i) {
            const int p = t0 + threadIdx.x + SEL_THREADS * i;
            mloc = fmaxf(mloc, mm[i] - (p == n - 1 ? drop_last : drop_full));
        }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) mloc = fmaxf(mloc, __shfl_xor_sync(FULL, mloc, o));
    if (lane == 0) shm[warp] = mloc;
    __syncthreads();
    float tau0 = -INFINITY;
    for (int w = 0; w < SEL_THREADS / 32; ++w) tau0 = fmaxf(tau0, shm[w]);

    // Pages with m + 10 s below tau0 add less than n_p s^R J_R(10) to F at any
    // tau >= tau0 (a relative 1e-23 of one page's worth): they are dropped.
    // The kept pages take their slots from a block scan in thread order (then
    // item order), so the list, and every sum over it, is the same each call.
    float hloc = -INFINITY;  // max over pages of m + 10 s: F < 1 there
    int nkept = 0;
    for (int t0 = 0; t0 < n; t0 += TILE) {
        if (!one_tile) load_ms(t0);
        unsigned keep = 0;
#pragma unroll
        for (int i = 0; i < ITEMS; ++i) {
            const int p = t0 + threadIdx.x + SEL_THREADS * i;
            if (p < n) hloc = fmaxf(hloc, mm[i] + 10.f * ss[i]);
            if (p < n && mm[i] + 10.f * ss[i] >= tau0) keep |= 1u << i;
        }
        int tot;
        int slot = nkept + block_excl_scan(__popc(keep), shi, &tot);
#pragma unroll
        for (int i = 0; i < ITEMS; ++i)
            if ((keep >> i) & 1u) {
                if (slot < GCAP) {
                    cm[slot] = mm[i];
                    cs[slot] = ss[i];
                    cn[slot] = (float)tokens_in_page(seq, a.P, t0 + threadIdx.x + SEL_THREADS * i);
                }
                ++slot;
            }
        nkept += tot;
    }
    if (threadIdx.x == 0) ncand = nkept;
#pragma unroll
    for (int o = 16; o; o >>= 1) hloc = fmaxf(hloc, __shfl_xor_sync(FULL, hloc, o));
    if (lane == 0) shm2[warp] = hloc;
    __syncthreads();
    const int nc = ncand;
    const bool overflow = nc > GCAP;
    float hmax = -INFINITY;
    for (int w = 0; w < SEL_THREADS / 32; ++w) hmax = fmaxf(hmax, shm2[w]);
    hmax = fmaxf(hmax, tau0 + 1.f);
    if (overflow && threadIdx.x == 0) atomicOr(a.status, ENTMAXKV_STATUS_OVERFLOW);

    auto contrib = [&](float m, float s, float w, float tau, float &F, float &Fp) {
        gauss_contrib<R>(m, s, w, tau, F, Fp);
    };

    // Newton on g = F^(1/R) from the bracket's left end.  F^(1/R) is R-norm of
    // (X - tau)_+ under the pages' mixture (times a constant), hence convex and
    // decreasing in tau: every tangent meets zero left of the root, so the
    // iterates climb monotonically to it.  Each evaluation is spread over the
    // whole block (one barrier each, double-buffered partials).
    __shared__ float nred[2][64];
    const float hi = hmax;
    float tau = tau0;
    for (int it = 0; it < 48; ++it) {
        float F = 0.f, Fp = 0.f;
        if (!overflow) {
            for (int i = threadIdx.x; i < nc; i += SEL_THREADS) contrib(cm[i], cs[i], cn[i], tau, F, Fp);
        } else {
            for (int p = threadIdx.x; p < n; p += SEL_THREADS)
                contrib(a1 * a.mu[row + p], a1 * a.sigma[row + p], (float)tokens_in_page(seq, a.P, p), tau, F,
                        Fp);
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) {
            F += __shfl_xor_sync(FULL, F, o);
            Fp += __shfl_xor_sync(FULL, Fp, o);
        }
        float *buf = nred[it & 1];
        if (lane == 0) {
            buf[2 * warp] = F;
            buf[2 * warp + 1] = Fp;
        }
        __syncthreads();
        F = 0.f;
        Fp = 0.f;
        for (int w = 0; w < SEL_THREADS / 32; ++w) {
            F += buf[2 * w];
            Fp += buf[2 * w + 1];
        }
        if (!newton_step<R>(F, Fp, hi, tau)) break;
    }
    if (threadIdx.x == 0 && a.tau_hat) a.tau_hat[bh] = tau;

    const float thr = tau - a.delta;
    const bool est = a.policy == ENTMAXKV_GAUSS_EST;
    const float z_full = zmax_of(a.P), z_last = zmax_of(tokens_in_page(seq, a.P, n - 1));
    int *sel = a.sel + row;
    int base = 0;
    for (int t0 = 0; t0 < n; t0 += TILE) {
        const int p0 = t0 + threadIdx.x * ITEMS;
        if (!one_tile) {
#pragma unroll
            for (int i = 0; i < ITEMS; ++i) ub[i] = (p0 + i < n) ? __ldg(a.bbox + row + p0 + i) : 0.f;
        }
        unsigned bits = 0;
#pragma unroll
        for (int i = 0; i < ITEMS; ++i) {
            if (!(p0 + i < n)) continue;
            float e = a1 * ub[i];
            if (est) {
                const int p = p0 + i;
                e = fminf(e, a1 * __ldg(a.mu + row + p) + (p == n - 1 ? z_last : z_full) * a1 * __ldg(a.sigma + row + p));
            }
            if (e > thr) bits |= 1u << i;
        }
        int tot;
        int w = base + block_excl_scan(__popc(bits), shi, &tot);
#pragma unroll
        for (int i = 0; i < ITEMS; ++i)
            if (bits & (1u << i)) sel[w++] = p0 + i;
        base += tot;
    }
    if (threadIdx.x == 0) a.cnt[bh] = base;
}

// ------------------------------------------- Gaussian selection, cluster form
//
// A cluster of GCL CTAs per (sequence, head) for sequences of up to
// GCL * GTH * GIT pages.  CTA r keeps pages [r Q, (r+1) Q), Q = ceil(n/GCL),
// GIT consecutive pages per thread, in registers from first load to last use.
// Exchanges are pushes into the peers' shared memory followed by one cluster
// barrier each: (1) the CTAs' maxima give the bracket, (2) each CTA pushes its
// pruned candidates to rank 0, (3) rank 0 solves for tau_hat (its whole block
// evaluates each Newton step) and pushes it back, (4) the CTAs' selected-page
// counts give each CTA its offset in the ascending list.  If a CTA has more
// candidates than rank 0 holds for it, every Newton step is instead reduced
// over the cluster (one barrier per step); the iterates are the same in every
// CTA.
constexpr int GCL = 4;
// 512 threads of 8 pages: 12.9 us at 1M tokens against 14.0 for 256 x 16
// (the per-page loops are unrolled, and a launch fetches its code cold:
// instruction fetch was the kernel's top stall); 1024 x 4 spills.
constexpr int GTH = 512;
constexpr int GIT = 8;
constexpr int GCAPR = 768;  // candidates per CTA that rank 0 holds

template <int R>
__global__ void __cluster_dims__(GCL, 1, 1) __launch_bounds__(GTH) gauss_cluster_kernel(SelectArgs a) {
    pdl_wait();
    __shared__ float rmax[GCL], rhmax[GCL];             // pushed by every CTA
    __shared__ int rcnt[GCL], rsel[GCL];                // pushed by every CTA
    __shared__ float cm[GCL * GCAPR], cs[GCL * GCAPR], cn[GCL * GCAPR];  // candidates (rank 0)
    __shared__ float s_tau;                             // pushed by rank 0
    __shared__ float rF[2][GCL], rFp[2][GCL];           // pushed Newton partials (fallback)
    __shared__ float rNw[2][2 * (GTH / 32)];            // per-warp Newton partials (rank 0)
    __shared__ float wa[GTH / 32], wb[GTH / 32];
    __shared__ int sh[72];
    const unsigned rank = cl_rank();
    int b, h;
    head_of(blockIdx.x / GCL, a.h0, a.nh, b, h);
    const int bh = b * a.Hq + h;
    const int seq = seq_len_of(a.seq_lens, b, a.P, a.max_pages, a.status);
    const int n = n_pages_of(seq, a.P);
    const size_t row = (size_t)bh * a.max_pages;
    const float a1 = a.alpha - 1.f;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    // decode step: the group's union (see above)
    const int G = a.Hq / a.Hkv;
    const bool uni = a.umap != nullptr;
    const int bk = b * a.Hkv + h / G;
    if (n == 0) {  // the same in every CTA of the cluster: no barrier is skipped by half of it
        if (rank == 0 && threadIdx.x == 0) {
            a.cnt[bh] = 0;
            if (a.tau_hat) a.tau_hat[bh] = __int_as_float(0x7fc00000);
        }
        if (uni && G == 1 && rank == 0 && threadIdx.x == 0) {
            a.union_cnt[bk] = 0;
            a.zmax[bh] = ORD_NEG_INF;
        }
        return;
    }
    const int Q = ceil_div(ceil_div(n, GCL), GIT) * GIT;  // whole GIT-page runs per thread
    const int lo_p = min(n, (int)rank * Q), hi_p = min(n, (int)(rank + 1) * Q);
    const int p0 = lo_p + threadIdx.x * GIT;
    float ub[GIT], mm[GIT], ss[GIT];
    const bool al16 = ((reinterpret_cast<uintptr_t>(a.bbox) | reinterpret_cast<uintptr_t>(a.mu) |
                        reinterpret_cast<uintptr_t>(a.sigma)) & 15) == 0;
    if (al16 && (row & 3) == 0 && p0 + GIT <= hi_p) {
        // a full run on a 16-byte boundary: 128-bit loads, all issued together
#pragma unroll
        for (int i = 0; i < GIT; i += 4) {
            const float4 u = __ldg(reinterpret_cast<const float4 *>(a.bbox + row + p0 + i));
            const float4 m = __ldg(reinterpret_cast<const float4 *>(a.mu + row + p0 + i));
            const float4 v = __ldg(reinterpret_cast<const float4 *>(a.sigma + row + p0 + i));
            ub[i] = u.x; ub[i + 1] = u.y; ub[i + 2] = u.z; ub[i + 3] = u.w;
            mm[i] = a1 * m.x; mm[i + 1] = a1 * m.y; mm[i + 2] = a1 * m.z; mm[i + 3] = a1 * m.w;
            ss[i] = a1 * v.x; ss[i + 1] = a1 * v.y; ss[i + 2] = a1 * v.z; ss[i + 3] = a1 * v.w;
        }
    } else {
#pragma unroll
        for (int i = 0; i < GIT; ++i) {
            const bool v = p0 + i < hi_p;
            ub[i] = v ? __ldg(a.bbox + row + p0 + i) : 0.f;
            mm[i] = v ? a1 * __ldg(a.mu + row + p0 + i) : -INFINITY;
            ss[i] = v ? a1 * __ldg(a.sigma + row + p0 + i) : 0.f;
        }
    }
    // (1) bracket: tau_hat >= max_p (m_p - n_p^(-1/R)) (Jensen); F < 1 at
    // max_p (m_p + 10 s_p)
    const float inv_r = 1.f / (float)R;
    const float drop_full = powf((float)a.P, -inv_r);
    const float drop_last = powf((float)tokens_in_page(seq, a.P, n - 1), -inv_r);
    float lmx = -INFINITY, lhx = -INFINITY;
#pragma unroll
    for (int i = 0; i < GIT; ++i) {
        if (p0 + i < hi_p) {
            lmx = fmaxf(lmx, mm[i] - (p0 + i == n - 1 ? drop_last : drop_full));
            lhx = fmaxf(lhx, mm[i] + 10.f * ss[i]);
        }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
        lmx = fmaxf(lmx, __shfl_xor_sync(FULL, lmx, o));
        lhx = fmaxf(lhx, __shfl_xor_sync(FULL, lhx, o));
    }
    if (lane == 0) {
        wa[warp] = lmx;
        wb[warp] = lhx;
    }
    __syncthreads();
    if (threadIdx.x < GCL) {
        float x = -INFINITY, y = -INFINITY;
        for (int w = 0; w < GTH / 32; ++w) {
            x = fmaxf(x, wa[w]);
            y = fmaxf(y, wb[w]);
        }
        cl_stf(cl_map(&rmax[rank], threadIdx.x), x);
        cl_stf(cl_map(&rhmax[rank], threadIdx.x), y);
    }
    cl_sync();
    float tau0 = -INFINITY, hmax = -INFINITY;
#pragma unroll
    for (int r = 0; r < GCL; ++r) {
        tau0 = fmaxf(tau0, rmax[r]);
        hmax = fmaxf(hmax, rhmax[r]);
    }
    hmax = fmaxf(hmax, tau0 + 1.f);

    // (2) candidates: pages with m + 10 s >= tau0 (the rest add less than
    // n_p s^R J_R(10) to F anywhere right of tau0), pushed to rank 0
    unsigned keep = 0;
#pragma unroll
    for (int i = 0; i < GIT; ++i)
        if (p0 + i < hi_p && mm[i] + 10.f * ss[i] >= tau0) keep |= 1u << i;
    int lc;
    int w = block_excl_scan(__popc(keep), sh, &lc);
#pragma unroll
    for (int i = 0; i < GIT; ++i)
        if (keep & (1u << i)) {
            if (w < GCAPR) {
                const int slot = (int)rank * GCAPR + w;
                cl_stf(cl_map(&cm[slot], 0), mm[i]);
                cl_stf(cl_map(&cs[slot], 0), ss[i]);
                cl_stf(cl_map(&cn[slot], 0), (float)tokens_in_page(seq, a.P, p0 + i));
            }
            ++w;
        }
    if (threadIdx.x < GCL) cl_sti(cl_map(&rcnt[rank], threadIdx.x), lc);
    cl_sync();
    bool spill = false;
#pragma unroll
    for (int r = 0; r < GCL; ++r) spill |= rcnt[r] > GCAPR;
    if (spill && rank == 0 && threadIdx.x == 0) atomicOr(a.status, ENTMAXKV_STATUS_OVERFLOW);

    // (3) tau_hat: Newton on g = F^(1/R) from tau0 (g is convex and
    // decreasing, so the iterates climb to the root without overshooting)
    float tau = tau0;
    if (!spill) {
        if (rank == 0) {
            // rank 0 alone: candidate c of CTA r is item (r, c) of the
            // concatenated lists; thread t takes items t, t + GTH, ...  (One
            // warp running the steps alone, with no barrier, measured slower:
            // each lane's Gaussian moments are a long dependent chain.)
            const int n0 = rcnt[0], n1 = n0 + rcnt[1], n2 = n1 + rcnt[2], n3 = n2 + rcnt[3];
            for (int it = 0; it < 48; ++it) {
                float F = 0.f, Fp = 0.f;
                for (int k = threadIdx.x; k < n3; k += GTH) {
                    const int r = k < n0 ? 0 : k < n1 ? 1 : k < n2 ? 2 : 3;
                    const int c = r * GCAPR + k - (r == 0 ? 0 : r == 1 ? n0 : r == 2 ? n1 : n2);
                    gauss_contrib<R>(cm[c], cs[c], cn[c], tau, F, Fp);
                }
#pragma unroll
                for (int o = 16; o; o >>= 1) {
                    F += __shfl_xor_sync(FULL, F, o);
                    Fp += __shfl_xor_sync(FULL, Fp, o);
                }
                float *buf = rNw[it & 1];  // double-buffered: one barrier per step
                if (lane == 0) {
                    buf[2 * warp] = F;
                    buf[2 * warp + 1] = Fp;
                }
                __syncthreads();
                F = 0.f;
                Fp = 0.f;
#pragma unroll
                for (int ww = 0; ww < GTH / 32; ++ww) {
                    F += buf[2 * ww];
                    Fp += buf[2 * ww + 1];
                }
                if (!newton_step<R>(F, Fp, hmax, tau)) break;  // the same in every thread
            }
            if (threadIdx.x < GCL) cl_stf(cl_map(&s_tau, threadIdx.x), tau);
        }
        cl_sync();
        tau = s_tau;
    } else {
        for (int it = 0; it < 48; ++it) {
            float F = 0.f, Fp = 0.f;
#pragma unroll
            for (int i = 0; i < GIT; ++i)
                if (keep & (1u << i)) gauss_contrib<R>(mm[i], ss[i], (float)tokens_in_page(seq, a.P, p0 + i), tau, F, Fp);
#pragma unroll
            for (int o = 16; o; o >>= 1) {
                F += __shfl_xor_sync(FULL, F, o);
                Fp += __shfl_xor_sync(FULL, Fp, o);
            }
            __syncthreads();  // the previous step's wa/wb are read
            if (lane == 0) {
                wa[warp] = F;
                wb[warp] = Fp;
            }
            __syncthreads();
            if (threadIdx.x < GCL) {
                float x = 0.f, y = 0.f;
                for (int ww = 0; ww < GTH / 32; ++ww) {
                    x += wa[ww];
                    y += wb[ww];
                }
                cl_stf(cl_map(&rF[it & 1][rank], threadIdx.x), x);
                cl_stf(cl_map(&rFp[it & 1][rank], threadIdx.x), y);
            }
            cl_sync();
            F = 0.f;
            Fp = 0.f;
#pragma unroll
            for (int r = 0; r < GCL; ++r) {
                F += rF[it & 1][r];
                Fp += rFp[it & 1][r];
            }
            if (!newton_step<R>(F, Fp, hmax, tau)) break;  // the same decision in every CTA
        }
    }
    if (rank == 0 && threadIdx.x == 0 && a.tau_hat) a.tau_hat[bh] = tau;

    // (4) pages with (alpha-1) x (estimated max) > tau_hat - Delta, ascending;
    // the estimate is the bound, or min(bound, mu + z(n) sigma)
    const float thr = tau - a.delta;
    const bool est = a.policy == ENTMAXKV_GAUSS_EST;
    const float z_full = zmax_of(a.P), z_last = zmax_of(tokens_in_page(seq, a.P, n - 1));
    unsigned bits = 0;
#pragma unroll
    for (int i = 0; i < GIT; ++i) {
        const float e = est ? fminf(a1 * ub[i], mm[i] + (p0 + i == n - 1 ? z_last : z_full) * ss[i]) : a1 * ub[i];
        if (p0 + i < hi_p && e > thr) bits |= 1u << i;
    }
    int blk[GIT];
    if (uni && G == 1) blocks_run<GIT>(a.page_table + (size_t)b * a.max_pages, p0, bits, blk);  // in flight during the scan
    if (uni && G > 1) mark_run<GIT>(a.umap + (size_t)bk * a.uwords, p0, bits, h % G);  // the marks complete behind the scan
    int ls;
    int o = block_excl_scan(__popc(bits), sh, &ls);
    if (threadIdx.x < GCL) cl_sti(cl_map(&rsel[rank], threadIdx.x), ls);
    cl_sync();
    int off = 0, total = 0;
#pragma unroll
    for (int r = 0; r < GCL; ++r) {
        off += r < (int)rank ? rsel[r] : 0;
        total += rsel[r];
    }
    int *sel = a.sel + row;
    o += off;
#pragma unroll
    for (int i = 0; i < GIT; ++i)
        if (bits & (1u << i)) {
            if (uni && G == 1)
                union_entry(a, a.union_e + (size_t)bk * a.max_pages, a.union_blk + (size_t)bk * a.max_pages, o,
                            p0 + i, blk[i]);
            sel[o++] = p0 + i;
        }
    if (rank == 0 && threadIdx.x == 0) a.cnt[bh] = total;
    if (uni && G == 1 && rank == 0 && threadIdx.x == 0) {
        a.union_cnt[bk] = total;
        a.zmax[bh] = ORD_NEG_INF;
    }
}

}  // namespace

bool select_marks_union(const SelectArgs &a) {
    // one top-k tile, or the cluster form of the Gaussian selection: both
    // hold up to 16384 pages
    return a.max_pages <= SEL_THREADS * ITEMS && a.max_pages <= GCL * GTH * GIT;
}

cudaError_t launch_select(const SelectArgs &a, cudaStream_t st) {
    const int grid = a.B * a.nh;
    cudaError_t e = cudaSuccess;
    if (a.policy == ENTMAXKV_TOPK) {
        // short sequences: a quarter of the threads holds every page in registers
        // rows of up to 4096 pages: 512 threads of 8 keys (less unrolled code,
        // fetched cold each launch: 9.9 vs 11.0 us for the 128k-token batch of
        // 8) while the heads fit one wave of two CTAs per SM, else 256 of 16
        // (four per SM: the 512-head batch took 19.6 us in two waves against
        // 15.1 in one)
        if (a.max_pages <= 4096 && grid <= 2 * a.sms)
            e = launch_pdl(topk_kernel<512, 8>, dim3(grid), dim3(512), 0, st, a);
        else if (a.max_pages <= 4096)
            e = launch_pdl(topk_kernel<256, ITEMS>, dim3(grid), dim3(256), 0, st, a);
        else
            e = launch_pdl(topk_kernel<SEL_THREADS, ITEMS>, dim3(grid), dim3(SEL_THREADS), 0, st, a);
    } else if (a.max_pages <= GCL * GTH * GIT) {
        switch (a.r_int) {
            case 1: e = launch_pdl(gauss_cluster_kernel<1>, dim3(grid * GCL), dim3(GTH), 0, st, a); break;
            case 2: e = launch_pdl(gauss_cluster_kernel<2>, dim3(grid * GCL), dim3(GTH), 0, st, a); break;
            case 3: e = launch_pdl(gauss_cluster_kernel<3>, dim3(grid * GCL), dim3(GTH), 0, st, a); break;
            case 4: e = launch_pdl(gauss_cluster_kernel<4>, dim3(grid * GCL), dim3(GTH), 0, st, a); break;
            case 5: e = launch_pdl(gauss_cluster_kernel<5>, dim3(grid * GCL), dim3(GTH), 0, st, a); break;
            case 6: e = launch_pdl(gauss_cluster_kernel<6>, dim3(grid * GCL), dim3(GTH), 0, st, a); break;
            case 7: e = launch_pdl(gauss_cluster_kernel<7>, dim3(grid * GCL), dim3(GTH), 0, st, a); break;
            case 8: e = launch_pdl(gauss_cluster_kernel<8>, dim3(grid * GCL), dim3(GTH), 0, st, a); break;
            default: return cudaErrorInvalidValue;
        }
    } else {
        switch (a.r_int) {
            case 1: e = launch_pdl(gauss_kernel<1>, dim3(grid), dim3(SEL_THREADS), 0, st, a); break;
            case 2: e = launch_pdl(gauss_kernel<2>, dim3(grid), dim3(SEL_THREADS), 0, st, a); break;
            case 3: e = launch_pdl(gauss_kernel<3>, dim3(grid), dim3(SEL_THREADS), 0, st, a); break;
            case 4: e = launch_pdl(gauss_kernel<4>, dim3(grid), dim3(SEL_THREADS), 0, st, a); break;
            case 5: e = launch_pdl(gauss_kernel<5>, dim3(grid), dim3(SEL_THREADS), 0, st, a); break;
            case 6: e = launch_pdl(gauss_kernel<6>, dim3(grid), dim3(SEL_THREADS), 0, st, a); break;
            case 7: e = launch_pdl(gauss_kernel<7>, dim3(grid), dim3(SEL_THREADS), 0, st, a); break;
            case 8: e = launch_pdl(gauss_kernel<8>, dim3(grid), dim3(SEL_THREADS), 0, st, a); break;
            default: return cudaErrorInvalidValue;
        }
    }
    return e;
}

}  // namespace ekv
