// decode.cu -- alpha-entmax decode attention over paged bf16 K/V (EntmaxKV
// summary: section 2.C sparse attention over the selected pages; section 4
// full-cache entmax and full-cache softmax as comparison points).
//
// Sparse path, two or three launches on one stream, no host round trip:
//   union_kernel   per (sequence, kv head), one CTA: union of the G query
//                  heads' selected pages, ascending, each with a G-bit head
//                  mask and its physical block.  Skipped when the q.K grid
//                  has at most two CTAs per group (many groups): each q.K CTA
//                  then builds its group's union itself, in its still unused
//                  ring memory (one page bitmap per head), and writes the
//                  entries of its own steps.
//   qk_kernel      split over the union: TMA 2-D loads (128-byte swizzle) of
//                  the K tiles through a 2-stage mbarrier ring fed by one
//                  producer warp, five CTAs per SM; z = (alpha-1) q.k/sqrt(d) for all G heads
//                  of the group from one copy of each tile (tensor-core
//                  m16n8k16, tokens as M and the heads as N, when G >= 2; CUDA
//                  cores when G == 1), stored in list order with the max of
//                  every 16-token tile.
//   tau_pv_kernel  per (sequence, query head): max z is the max of the tile
//                  maxima; every token that can carry weight has
//                  z > max z - 1 (no weight exceeds 1), so those candidates
//                  are compacted on chip in list order; the exact root of
//                  sum (z - tau)_+^r = 1 lies in [z_max - 1, z_max - n^(1-alpha)]
//                  and is reached by Newton's method from the end where it is
//                  monotone, and p v is summed over the support, reading only
//                  those value rows.
// In the fused decode step (entmaxkv_decode_step) the selection kernel has
// marked each group's pages, and union_map_kernel compacts the marks in place
// of union_kernel (with G = 1 the selection wrote the union itself).
// Sparse softmax (alpha = 1) builds the union with union_kernel and runs
// softmax_kernel over its pages.
// Full-cache entmax runs qk_kernel over every page, tau_pv_kernel for tau, and
// pv_stream_kernel, which streams every V tile through the TMA ring.  Full-cache softmax runs softmax_kernel (K and V
// tiles per stage, online max / sum per split); both dense paths combine
// their splits in a fixed order in the last CTA of each group.
#include "pipeline.cuh"

namespace ekv {

namespace {

// ------------------------------------------------------------------ union

// Union of the G heads' selections of a group, ascending, each entry with its
// head mask.  One CTA per (sequence, kv head): the pages are taken UCH at a
// time; every head's entries that fall in the chunk mark a shared-memory
// bitmap (one byte of head bits per page), which is then compacted in page
// order behind the entries of the earlier chunks.
constexpr int UTH = 512;
constexpr int UCH = 16384;  // pages per chunk (one byte each)

__global__ void __launch_bounds__(UTH) union_kernel(DecodeArgs a) {
    {
        // the group's page-table row, on its way to L2 while the previous
        // kernel finishes (a hint only: nothing is read before the dependency
        // wait), so the lookups below find it there
        const int b0 = blockIdx.x / a.nk;
        const char *row = reinterpret_cast<const char *>(a.page_table + (size_t)b0 * a.max_pages);
        for (int l = threadIdx.x; l * 32 < a.max_pages; l += UTH)
            asm volatile("prefetch.global.L2 [%0];" ::"l"(row + (size_t)l * 128));
    }
    pdl_wait();
    __shared__ unsigned words[UCH / 4];
    __shared__ int sh[72];
    __shared__ int cnts[8], offs[9];
    int b, kvh;
    group_of(blockIdx.x, a.kv0, a.nk, b, kvh);
    const int bk = b * a.Hkv + kvh;
    const int G = a.Hq / a.Hkv;
    const int np = n_pages_of(seq_len_of(a.seq_lens, b, a.P, a.max_pages, a.status), a.P);
    if (threadIdx.x < G) {
        const int bh = b * a.Hq + kvh * G + threadIdx.x;
        int c = a.cnt[bh];
        const int cmax = a.sharded ? a.sel_stride : np;  // sharded: counts over all shards' pages
        if (c < 0 || c > cmax) {
            atomicOr(a.status, ENTMAXKV_STATUS_BAD_SELECTION);
            c = c < 0 ? 0 : cmax;
        }
        cnts[threadIdx.x] = c;
        a.ws.zmax[bh] = ORD_NEG_INF;  // the q.K kernel's running max
    }
    if (threadIdx.x == 0) a.ws.counters[bk] = 0;  // the softmax path's last-CTA combine
    __syncthreads();
    if (threadIdx.x == 0) {
        offs[0] = 0;
        for (int g = 0; g < G; ++g) offs[g + 1] = offs[g] + cnts[g];
    }
    __syncthreads();
    const int total = offs[G];  // every head's entries as one flat range
    int *ue = a.ws.union_e + (size_t)bk * a.max_pages;
    int *ub = a.ws.union_blk + (size_t)bk * a.max_pages;
    const int *pt = a.page_table + (size_t)b * a.max_pages;
    int done = 0;
    for (int lo = 0; lo < np; lo += UCH) {
        const int hi = min(np, lo + UCH);
        const int nw = ceil_div(hi - lo, 4);
        for (int i = threadIdx.x; i < nw; i += UTH) words[i] = 0u;
        __syncthreads();
        // four loads in flight per thread
        for (int k0 = threadIdx.x; k0 < total; k0 += 4 * UTH) {
            int p[4], g[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int k = k0 + u * UTH;
                p[u] = -1;
                g[u] = 0;
                if (k < total) {
                    int gg = 0;
                    while (k >= offs[gg + 1]) ++gg;
                    g[u] = gg;
                    p[u] = __ldg(a.sel + (size_t)(b * a.Hq + kvh * G + gg) * a.sel_stride + (k - offs[gg])) -
                           a.page_begin;  // this shard's page index
                }
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                if (k0 + u * UTH >= total) continue;
                if (p[u] >= lo && p[u] < hi)
                    atomicOr(&words[(p[u] - lo) >> 2], 1u << ((p[u] & 3) * 8 + g[u]));
                else if (lo == 0 && (a.sharded ? (p[u] + a.page_begin < 0 || p[u] + a.page_begin >= a.sel_stride)
                                               : (p[u] < 0 || p[u] >= np)))
                    atomicOr(a.status, ENTMAXKV_STATUS_BAD_SELECTION);  // (sharded: other shards' pages are skipped)
            }
        }
        __syncthreads();
        // the chunk's entries in page order: thread t owns words [t*wpt, (t+1)*wpt);
        // the page-table entries of its selected pages are all loaded first
        constexpr int WPT_MAX = UCH / 4 / UTH;
        const int wpt = ceil_div(nw, UTH);
        const int w0 = threadIdx.x * wpt;
        unsigned wv[WPT_MAX];
        int blk[WPT_MAX][4];
        int mine = 0;
#pragma unroll
        for (int i = 0; i < WPT_MAX; ++i) {
            wv[i] = i < wpt && w0 + i < nw ? words[w0 + i] : 0u;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const bool sel = (wv[i] >> (8 * j)) & 0xffu;
                blk[i][j] = sel ? __ldg(pt + lo + 4 * (w0 + i) + j) : -1;
                mine += sel ? 1 : 0;
            }
        }
        int chunk_total;
        int pos = done + block_excl_scan(mine, sh, &chunk_total);
#pragma unroll
        for (int i = 0; i < WPT_MAX; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const unsigned m = (wv[i] >> (8 * j)) & 0xffu;
                if (m) {
                    // the entry and its physical block (-1 if the page-table entry is bad)
                    const bool ok = blk[i][j] >= 0 && blk[i][j] < a.num_blocks;
                    if (!ok) atomicOr(a.status, ENTMAXKV_STATUS_BAD_PAGE);
                    ue[pos] = ((lo + 4 * (w0 + i) + j) << 8) | (int)m;
                    ub[pos++] = ok ? blk[i][j] : -1;
                }
            }
        done += chunk_total;
        __syncthreads();  // the bitmap is read before the next chunk clears it
    }
    if (threadIdx.x == 0) a.ws.union_cnt[bk] = done;
}

// Union of a group's selections from the marks the selection kernel left
// (decode step, G > 1): byte p of the group's row of ws.umap holds the head
// bits of page p.  One CTA per (sequence, kv head); the page-table row is
// sent to L2 before the dependency wait.  Per pass of UM_WPT words (4 UM_WPT
// pages) a thread, all loads of a pass issued together:
//   1. its words go to shared memory and a block scan of their marked-page
//      counts gives each thread its first position;
//   2. the entries are dealt round-robin to the threads, each finding its
//      entry's page by a binary search over those positions, and the
//      page-table entries of four entries per thread are loaded together
//      before they are written.
// It also resets the q.K pass's running max of the group's heads.
constexpr int UMT = 512;
constexpr int UM_WPT = 8;

// Bit j set where byte j of w is non-zero.
__device__ __forceinline__ unsigned nz_bytes(unsigned w) {
    return (w & 0xffu ? 1u : 0u) | (w & 0xff00u ? 2u : 0u) | (w & 0xff0000u ? 4u : 0u) | (w & 0xff000000u ? 8u : 0u);
}

__global__ void __launch_bounds__(UMT) union_map_kernel(DecodeArgs a) {
    {
        const int b0 = blockIdx.x / a.nk;
        const char *prow = reinterpret_cast<const char *>(a.page_table + (size_t)b0 * a.max_pages);
        for (int l = threadIdx.x; l * 32 < a.max_pages; l += UMT)
            asm volatile("prefetch.global.L2 [%0];" ::"l"(prow + (size_t)l * 128));
    }
    pdl_wait();
    __shared__ unsigned words[UMT * UM_WPT];
    __shared__ int pre[UMT];
    __shared__ int sh[72];
    int b, kvh;
    group_of(blockIdx.x, a.kv0, a.nk, b, kvh);
    const int bk = b * a.Hkv + kvh;
    const int G = a.Hq / a.Hkv;
    if (threadIdx.x < G) a.ws.zmax[b * a.Hq + kvh * G + threadIdx.x] = ORD_NEG_INF;
    const int np = n_pages_of(seq_len_of(a.seq_lens, b, a.P, a.max_pages, a.status), a.P);
    const int nw = ceil_div(np, 4);
    const unsigned *row = a.ws.umap + (size_t)bk * a.ws.uwords;
    const int *pt = a.page_table + (size_t)b * a.max_pages;
    int *ue = a.ws.union_e + (size_t)bk * a.max_pages;
    int *ub = a.ws.union_blk + (size_t)bk * a.max_pages;
    int done = 0;
    for (int base = 0; base < nw; base += UMT * UM_WPT) {
        const int w0 = base + threadIdx.x * UM_WPT;  // a multiple of 4: 16-byte loads (rows are 16-byte aligned)
        int mine = 0;
#pragma unroll
        for (int i = 0; i < UM_WPT; i += 4) {
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (w0 + i < nw) v = __ldcg(reinterpret_cast<const uint4 *>(row + w0 + i));
            unsigned *dst = words + threadIdx.x * UM_WPT + i;
            dst[0] = v.x;
            dst[1] = v.y;
            dst[2] = v.z;
            dst[3] = v.w;
            mine += __popc(nz_bytes(v.x)) + __popc(nz_bytes(v.y)) + __popc(nz_bytes(v.z)) + __popc(nz_bytes(v.w));
        }
        int tot;
        pre[threadIdx.x] = block_excl_scan(mine, sh, &tot);
        __syncthreads();
        for (int e0 = 0; e0 < tot; e0 += 4 * UMT) {
            int page[4], mask[4], blk[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int e = e0 + u * UMT + (int)threadIdx.x;
                page[u] = -1;
                if (e >= tot) continue;
                int lo = 0, hi = UMT - 1;  // the last thread whose first position is <= e
                while (lo < hi) {
                    const int mid = (lo + hi + 1) >> 1;
                    if (pre[mid] <= e) lo = mid;
                    else hi = mid - 1;
                }
                int r = e - pre[lo];  // that thread holds more than r marked pages
                const unsigned *wsrc = words + lo * UM_WPT;
                int i = 0;
                unsigned m = nz_bytes(wsrc[0]);
                while (r >= __popc(m)) {
                    r -= __popc(m);
                    m = nz_bytes(wsrc[++i]);
                }
                while (r-- > 0) m &= m - 1u;
                const int j = __ffs(m) - 1;
                page[u] = 4 * (base + lo * UM_WPT + i) + j;
                mask[u] = (int)((wsrc[i] >> (8 * j)) & 0xffu);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) blk[u] = page[u] >= 0 ? __ldg(pt + page[u]) : -1;
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (page[u] >= 0) {
                    const bool ok = blk[u] >= 0 && blk[u] < a.num_blocks;
                    if (!ok) atomicOr(a.status, ENTMAXKV_STATUS_BAD_PAGE);
                    const int pos = done + e0 + u * UMT + (int)threadIdx.x;
                    ue[pos] = (page[u] << 8) | mask[u];
                    ub[pos] = ok ? blk[u] : -1;
                }
        }
        done += tot;
        __syncthreads();  // the words are read before the next pass overwrites them
    }
    if (threadIdx.x == 0) a.ws.union_cnt[bk] = done;
}

__global__ void dense_init_kernel(DecodeArgs a) {
    pdl_wait();
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    const int G = a.Hq / a.Hkv;
    int b, x;
    if (i < a.B * a.nk * G) {
        head_of(i, a.kv0 * G, a.nk * G, b, x);
        a.ws.zmax[b * a.Hq + x] = ORD_NEG_INF;
    }
    if (i < a.B * a.nk) {
        group_of(i, a.kv0, a.nk, b, x);
        a.ws.counters[b * a.Hkv + x] = 0;
    }
}

// ------------------------------------------------------ page producer

// Producer warp: for the CTA's local steps 0..my_n-1 (global step
// blockIdx.x + it*gridDim.x, covering entries [step*PPS, step*PPS+PPS) of the
// group's page list), resolve the pages 32 steps at a time with all lanes,
// then lane 0 waits for each stage to be free, publishes the step's pages and
// issues the box loads (map m0, and m1 into the second half when NMAP == 2).
// With ZG > 0 it also copies the z rows of the step's pages for the ZG heads
// of the group into zst ([stage][head][token], TPS tokens a row).
// Returns early (all lanes) if a wait ran out.
template <int D, int NMAP, int ZG = 0>
__device__ void produce(const DecodeArgs &a, const CUtensorMap *m0, const CUtensorMap *m1, bool dense, int b,
                        int kvh, int bk, int U, int my_n, int PPS, int NS, int stage_bytes, int stage_half,
                        unsigned char *stages, uint64_t *full, uint64_t *empty, PageInfo *pinfo, PageInfo *stash,
                        float *zst = nullptr, int TPS = 0) {
    const int lane = threadIdx.x & 31;
    const int seq = seq_len_of(a.seq_lens, b, a.P, a.max_pages, nullptr);  // (flagged by the caller kernel)
    const int S = gridDim.x;
    if (lane == 0) {
        prefetch_tmap(m0);
        if (NMAP == 2) prefetch_tmap(m1);
    }
    for (int base = 0; base < my_n; base += 32) {
        const int nb = min(32, my_n - base);
        for (int k = lane; k < nb * PPS; k += 32) {
            const int it = base + k / PPS, i = k % PPS;
            const int e = (blockIdx.x + it * S) * PPS + i;
            PageInfo r{-1, 0, 0, e, -1};
            if (e < U) {
                // sparse: the union entry and its resolved block, loaded
                // together (through L2 when the q.K CTAs wrote them
                // themselves; else through L1, where the kernel's start sent
                // the first batch); dense: page e and its page-table entry
                const int *pe = a.ws.union_e + (size_t)bk * a.max_pages + e;
                const int *pb = a.ws.union_blk + (size_t)bk * a.max_pages + e;
                const int entry = dense ? ((e << 8) | 0xff) : (a.union_in_qk ? __ldcg(pe) : *pe);
                const int blk = dense ? __ldg(a.page_table + (size_t)b * a.max_pages + e)
                                      : (a.union_in_qk ? __ldcg(pb) : *pb);
                r.page = entry >> 8;
                r.mask = entry & 0xff;
                if (blk >= 0 && blk < a.num_blocks) {
                    r.blk = blk;
                    r.nval = tokens_in_page(seq, a.P, r.page);
                } else if (dense) {
                    atomicOr(a.status, ENTMAXKV_STATUS_BAD_PAGE);
                }
            }
            stash[k] = r;
        }
        __syncwarp();
        bool ok = true;
        if (lane == 0) {
            for (int j = 0; j < nb && ok; ++j) {
                const int it = base + j;
                const int st = it % NS, ph = (it / NS) & 1;
                if (!mbar_wait(&empty[st], ph ^ 1, a.status)) {
                    ok = false;
                    break;
                }
                unsigned bytes = 0;
                for (int i = 0; i < PPS; ++i) {
                    const PageInfo r = stash[j * PPS + i];
                    pinfo[st * PPS_MAX + i] = r;
                    if (r.blk >= 0) bytes += (unsigned)(a.P * D * 2 * NMAP);
                    if (ZG > 0 && r.page >= 0) bytes += (unsigned)(ZG * a.P * 4);
                }
                mbar_arrive_expect_tx(&full[st], bytes);
                unsigned char *stage = stages + (size_t)st * stage_bytes;
                for (int i = 0; i < PPS; ++i) {
                    const PageInfo r = stash[j * PPS + i];
                    if (r.blk < 0) continue;
                    const int y = (r.blk * a.Hkv + kvh) * a.P;
                    unsigned char *dst = stage + (size_t)i * a.P * D * 2;
#pragma unroll
                    for (int box = 0; box < D / 64; ++box) {
                        tma_load_2d(dst + box * a.P * 128, m0, box * 64, y, &full[st]);
                        if (NMAP == 2) tma_load_2d(dst + stage_half + box * a.P * 128, m1, box * 64, y, &full[st]);
                    }
                }
                if (ZG > 0)
                    for (int i = 0; i < PPS; ++i) {
                        const PageInfo r = stash[j * PPS + i];
                        if (r.page < 0) continue;
#pragma unroll
                        for (int g = 0; g < ZG; ++g)
                            bulk_g2s(zst + (size_t)(st * ZG + g) * TPS + i * a.P,
                                     a.ws.zbuf + tok_row(a, b, kvh * ZG + g) + (size_t)r.upos * a.P, a.P * 4, &full[st]);
                    }
            }
        }
        ok = __shfl_sync(FULL, ok, 0);
        if (!ok) return;
        __syncwarp();
    }
}

// ------------------------------------------------------ union in the q.K CTA

// The union of the G heads' selections of group (b, kvh), built by every CTA
// of the group's q.K grid in shared memory it does not use yet (its ring,
// which holds G page bitmaps of np bits): each head's entries set bits of its
// bitmap; the union's pages are then counted in page order (a block scan
// over the bitmap words), which gives every entry its list position e.  The
// CTA writes the entries of its own steps (step e / PPS, owned by CTA
// step mod gridDim.x) to the workspace, each with its G-bit head mask and
// physical block (the page-table loads issued eight at a time), for its
// producer and for the tau kernel; CTA 0 also writes the count.  Every CTA
// reads the same lists, so all agree on U and on the positions.  A warp marks
// 32 consecutive list entries at a time: lanes whose entries fall in the same
// bitmap word (a run of neighbouring pages of one head's ascending list) OR
// their bits together first, and the first lane of each run sets them with one
// shared-memory atomic.  All threads call it; it returns U.
__device__ int union_in_cta(const DecodeArgs &a, int b, int kvh, int bk, int np, int PPS, unsigned *bm, int *s_cnt,
                            int *s_off, int *sh) {
    const int G = a.Hq / a.Hkv;
    const int nt = blockDim.x, S = gridDim.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = nt >> 5;
    const int *selg = a.sel + (size_t)(b * a.Hq + kvh * G) * a.sel_stride;  // head g's list at g * sel_stride
    const int *pt = a.page_table + (size_t)b * a.max_pages;
    int *ue = a.ws.union_e + (size_t)bk * a.max_pages;
    int *ub = a.ws.union_blk + (size_t)bk * a.max_pages;
    const bool report = blockIdx.x == 0;  // argument errors are flagged by one CTA
    const int W = ceil_div(np, 32);
    for (int i = threadIdx.x; i < G * W; i += nt) bm[i] = 0u;
    if (threadIdx.x < G) {
        int c = a.cnt[b * a.Hq + kvh * G + threadIdx.x];
        const int cmax = a.sharded ? a.sel_stride : np;  // sharded: counts over all shards' pages
        if (c < 0 || c > cmax) {
            if (report) atomicOr(a.status, ENTMAXKV_STATUS_BAD_SELECTION);
            c = c < 0 ? 0 : cmax;
        }
        s_cnt[threadIdx.x] = c;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        s_off[0] = 0;
        for (int g = 0; g < G; ++g) s_off[g + 1] = s_off[g] + s_cnt[g];
    }
    __syncthreads();
    const int total = s_off[G];  // every head's entries as one flat range
    // each warp takes 32 consecutive entries per round, two rounds' loads in flight
    for (int k0 = warp * 32; k0 < total; k0 += 2 * nwarps * 32) {
        int wd[2];
        unsigned bit[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int k = k0 + u * nwarps * 32 + lane;
            wd[u] = -1 - lane;  // unique: merges with no other lane
            bit[u] = 0u;
            if (k < total) {
                int gg = 0;
                while (k >= s_off[gg + 1]) ++gg;
                const int p = __ldg(selg + (size_t)gg * a.sel_stride + (k - s_off[gg])) - a.page_begin;
                if (p >= 0 && p < np) {
                    wd[u] = gg * W + (p >> 5);
                    bit[u] = 1u << (p & 31);
                } else if (report && (!a.sharded || p + a.page_begin < 0 || p + a.page_begin >= a.sel_stride)) {
                    atomicOr(a.status, ENTMAXKV_STATUS_BAD_SELECTION);  // (sharded: other shards' pages are skipped)
                }
            }
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            // OR over the lane's run of equal words (suffix scan within runs)
            unsigned acc = bit[u];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const unsigned y = __shfl_down_sync(FULL, acc, o);
                const int wy = __shfl_down_sync(FULL, wd[u], o);
                if (lane + o < 32 && wy == wd[u]) acc |= y;
            }
            const int wprev = __shfl_up_sync(FULL, wd[u], 1);
            if (acc && (lane == 0 || wprev != wd[u])) atomicOr(&bm[wd[u]], acc);
        }
    }
    __syncthreads();
    // thread t counts the union pages of words [t*wpt, (t+1)*wpt)
    const int wpt = ceil_div(W, nt);
    const int w0 = threadIdx.x * wpt;
    int mine = 0;
    for (int i = 0; i < wpt && w0 + i < W; ++i) {
        unsigned u = 0u;
        for (int g = 0; g < G; ++g) u |= bm[g * W + w0 + i];
        mine += __popc(u);
    }
    int U;
    int pos = block_excl_scan(mine, sh, &U);
    int q_page[8], q_e[8], q_mask[8];
    int nq = 0;
    auto resolve = [&]() {
        int blk[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) blk[j] = j < nq ? __ldg(pt + q_page[j]) : -1;
#pragma unroll
        for (int j = 0; j < 8; ++j)
            if (j < nq) {
                const bool ok = blk[j] >= 0 && blk[j] < a.num_blocks;
                if (!ok) atomicOr(a.status, ENTMAXKV_STATUS_BAD_PAGE);
                ue[q_e[j]] = (q_page[j] << 8) | q_mask[j];
                ub[q_e[j]] = ok ? blk[j] : -1;
            }
        nq = 0;
    };
    for (int i = 0; i < wpt && w0 + i < W; ++i) {
        const int w = w0 + i;
        unsigned u = 0u;
        for (int g = 0; g < G; ++g) u |= bm[g * W + w];
        while (u) {
            const int bit = __ffs(u) - 1;
            u &= u - 1;
            const int e = pos++;
            if ((e / PPS) % S != (int)blockIdx.x) continue;  // another CTA's step
            int mask = 0;
            for (int g = 0; g < G; ++g) mask |= (int)((bm[g * W + w] >> bit) & 1u) << g;
            q_page[nq] = 32 * w + bit;
            q_e[nq] = e;
            q_mask[nq] = mask;
            if (++nq == 8) resolve();
        }
    }
    resolve();
    if (report && threadIdx.x == 0) a.ws.union_cnt[bk] = U;
    return U;
}

// ----------------------------------------------------------------- q . K^T

// q.K ring: two stages per CTA and five CTAs per SM.  Measured on the gathered
// pass (device timeline, 1M-token Gaussian / 128k-token top-k steps): 5 x 2
// stages 20.6 / 20.9 us, 4 x 3 22.0 / 21.3, 6 x 2 23.9 / 25.2; earlier, 4 x 3
// beat 3 x 4 (42 vs 46.5 us for the whole 128k-token decode).  More CTAs with
// a shallower ring gather random pages faster, up to the point where the
// launch's CTAs no longer hide each other's ramp.
constexpr int QK_NS = 2;
constexpr int QK_PER_SM = 5;

template <int D, int G, bool DENSE>
__global__ void __launch_bounds__(DEC_THREADS) qk_kernel(const __grid_constant__ DecodeArgs a) {
    pdl_wait();
    constexpr int NS = QK_NS;
    using RG = Ring<D, G, NS, 1>;
    constexpr int TPS = RG::TPS;
    if (!DENSE && !a.union_in_qk && (threadIdx.x >> 5) == NWC) {
        // the producer's first 32 steps of union entries head for L1 together
        // with the union size below (their addresses do not depend on it), so
        // the first copies issue one round trip sooner
        const int pps = TPS / a.P, bk0 = (a.kv0 + (int)blockIdx.y % a.nk) + ((int)blockIdx.y / a.nk) * a.Hkv;
        for (int k = threadIdx.x & 31; k < 32 * pps; k += 32) {
            const int e = ((int)blockIdx.x + (k / pps) * (int)gridDim.x) * pps + k % pps;
            if (e < a.max_pages) {
                asm volatile("prefetch.global.L1 [%0];" ::"l"(a.ws.union_e + (size_t)bk0 * a.max_pages + e));
                asm volatile("prefetch.global.L1 [%0];" ::"l"(a.ws.union_blk + (size_t)bk0 * a.max_pages + e));
            }
        }
    }
    extern __shared__ unsigned char smem_raw[];
    RingView<D, G, NS, 1> R(smem_raw);
    __shared__ float qs[G == 1 ? D : 1];
    __shared__ int s_cnt[8], s_off[9], s_sh[72];

    int b, kvh;
    group_of(blockIdx.y, a.kv0, a.nk, b, kvh);
    const int bk = b * a.Hkv + kvh;
    const int P = a.P, PPS = TPS / P;
    const int seq = seq_len_of(a.seq_lens, b, P, a.max_pages, a.status);
    const int np = n_pages_of(seq, P);
    int U = np;
    if constexpr (!DENSE) {
        if (a.union_in_qk) {
            // the union of the group's selections, in the ring's memory
            U = union_in_cta(a, b, kvh, bk, np, PPS, reinterpret_cast<unsigned *>(R.stages), s_cnt, s_off, s_sh);
            // the ring's bytes were written through the generic proxy; the TMA
            // copies that refill them come through the async proxy
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncthreads();
        } else {
            U = a.ws.union_cnt[bk];  // from union_kernel
        }
    }
    const int nsteps = ceil_div(U, PPS);
    const int S = gridDim.x;
    const int my_n = nsteps > (int)blockIdx.x ? ceil_div(nsteps - blockIdx.x, S) : 0;
    if (my_n == 0) return;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&R.full[s], 1);
            mbar_init(&R.empty[s], NWC);
        }
        mbar_fence_init();
    }
    if (G == 1)
        for (int j = threadIdx.x; j < D; j += blockDim.x) qs[j] = bf16f(a.q[((size_t)b * a.Hq + kvh) * D + j]);
    __syncthreads();

    if (warp == NWC) {
        produce<D, 1>(a, &a.kmap, &a.kmap, DENSE, b, kvh, bk, U, my_n, PPS, NS, RG::STAGE, 0, R.stages, R.full,
                      R.empty, R.pinfo, R.stash);
        return;
    }

    // z = (alpha-1) * q.k / sqrt(d); 1/sqrt(d) as a correctly rounded constant
    const float zs = (a.alpha - 1.f) * (D == 64 ? 0.125f : 0.08838834764831845f);

    if constexpr (G >= 2) {
        // B fragments: q of head n = lane/4 (zero for n >= G), k pair 2*(lane%4)
        unsigned qb[D / 16][2];
        const int n = lane >> 2, kp = 2 * (lane & 3);
        {
            const uint16_t *qh = a.q + ((size_t)b * a.Hq + kvh * G + (n < G ? n : 0)) * D;
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                qb[ks][0] = n < G ? *reinterpret_cast<const unsigned *>(qh + 16 * ks + kp) : 0u;
                qb[ks][1] = n < G ? *reinterpret_cast<const unsigned *>(qh + 16 * ks + kp + 8) : 0u;
            }
        }
        const int h0 = 2 * (lane & 3);  // this lane's two heads: h0, h0+1
        float run0 = -INFINITY, run1 = -INFINITY;  // this lane's max of z for heads h0, h0+1
        for (int it = 0; it < my_n; ++it) {
            const int st = it % NS, ph = (it / NS) & 1;
            if (!mbar_wait(&R.full[st], ph, a.status)) return;
            const unsigned char *stage = R.stages + (size_t)st * RG::STAGE;
            const PageInfo *pis = R.pinfo + st * PPS_MAX;
            for (int mt = warp; mt < TPS / 16; mt += NWC) {
                const int tok0 = mt * 16, pi_i = tok0 / P, r0 = tok0 % P;
                const PageInfo pi = pis[pi_i];
                if (pi.page < 0) continue;
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
                if (pi.nval > 0) {
                    const unsigned char *pbase = stage + (size_t)pi_i * P * D * 2;
                    const int mat = lane >> 3, rr = lane & 7;
                    const int row = r0 + (mat & 1) * 8 + rr;
#pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks) {
                        unsigned a0, a1, a2, a3;
                        ldsm_x4(smem_u32(tile_chunk(pbase, P, row, ks * 2 + (mat >> 1))), a0, a1, a2, a3);
                        mma_bf16_16816(acc, a0, a1, a2, a3, qb[ks][0], qb[ks][1]);
                    }
                }
                // acc[v]: token r0 + lane/4 + 8*(v>>1), head h0 + (v&1)
                float z[4];
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    const int hh = h0 + (v & 1);
                    const int t = r0 + (lane >> 2) + 8 * (v >> 1);
                    const bool use = hh < G && t < pi.nval && ((pi.mask >> hh) & 1);
                    z[v] = use ? acc[v] * zs : -INFINITY;
                    if (hh < G) a.ws.zbuf[tok_row(a, b, kvh * G + hh) + (size_t)pi.upos * P + t] = z[v];
                    if (a.p_out && use) a.p_out[tok_row(a, b, kvh * G + hh) + (size_t)pi.page * P + t] = 0.f;
                }
                // max over the m-tile's 16 tokens, per head (lanes with equal lane%4
                // hold the same two heads)
                float m0 = fmaxf(z[0], z[2]), m1 = fmaxf(z[1], z[3]);
#pragma unroll
                for (int o = 4; o < 32; o <<= 1) {
                    m0 = fmaxf(m0, __shfl_xor_sync(FULL, m0, o));
                    m1 = fmaxf(m1, __shfl_xor_sync(FULL, m1, o));
                }
                run0 = fmaxf(run0, m0);
                run1 = fmaxf(run1, m1);
                if (lane < 4) {
                    const size_t ti = ((size_t)pi.upos * P + r0) / 16;
                    if (h0 < G) a.ws.tmax[tile_row(a, b, kvh * G + h0) + ti] = m0;
                    if (h0 + 1 < G) a.ws.tmax[tile_row(a, b, kvh * G + h0 + 1) + ti] = m1;
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&R.empty[st]);
        }
        // the running max of z per head (reset by the kernel before this one;
        // with the union built here the tau kernel takes it from the tile maxima)
        if (lane < 4 && !a.union_in_qk) {
            const int bh0 = b * a.Hq + kvh * G + h0;
            if (h0 < G && run0 > -INFINITY) atomicMax(&a.ws.zmax[bh0], f2ord(run0));
            if (h0 + 1 < G && run1 > -INFINITY) atomicMax(&a.ws.zmax[bh0 + 1], f2ord(run1));
        }
    } else {
        // G == 1: thread per token, q broadcast from shared memory
        float run = -INFINITY;
        const int ti = threadIdx.x;  // token within the stage
        for (int it = 0; it < my_n; ++it) {
            const int st = it % NS, ph = (it / NS) & 1;
            if (!mbar_wait(&R.full[st], ph, a.status)) return;
            const unsigned char *stage = R.stages + (size_t)st * RG::STAGE;
            const PageInfo pi = R.pinfo[st * PPS_MAX + ti / P];
            const int r = ti % P;
            const bool use = pi.page >= 0 && r < pi.nval && (pi.mask & 1);
            float z = -INFINITY;
            if (use) {
                const unsigned char *pbase = stage + (size_t)(ti / P) * P * D * 2;
                float acc = 0.f;
#pragma unroll
                for (int c16 = 0; c16 < D / 8; ++c16) {
                    const uint4 kv = *reinterpret_cast<const uint4 *>(tile_chunk(pbase, P, r, c16));
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
                z = acc * zs;
                if (a.p_out) a.p_out[tok_row(a, b, kvh) + (size_t)pi.page * P + r] = 0.f;
            }
            if (pi.page >= 0) a.ws.zbuf[tok_row(a, b, kvh) + (size_t)pi.upos * P + r] = z;
            // max of each 16-token tile (a half warp; tiles never straddle pages)
            float tm = z;
#pragma unroll
            for (int o = 1; o < 16; o <<= 1) tm = fmaxf(tm, __shfl_xor_sync(FULL, tm, o));
            if ((lane & 15) == 0 && pi.page >= 0)
                a.ws.tmax[tile_row(a, b, kvh) + ((size_t)pi.upos * P + r) / 16] = tm;
            run = fmaxf(run, z);
            __syncwarp();
            if (lane == 0) mbar_arrive(&R.empty[st]);
        }
        if (!a.union_in_qk) {
#pragma unroll
            for (int o = 16; o; o >>= 1) run = fmaxf(run, __shfl_xor_sync(FULL, run, o));
            if (lane == 0 && run > -INFINITY) atomicMax(&a.ws.zmax[b * a.Hq + kvh], f2ord(run));
        }
    }
}

// -------------------------------------------------------- tau and p . V

constexpr int TAU_NT = 256;  // threads per head
constexpr int TAU_NW = TAU_NT / 32;
constexpr int TAU_TB = 16;   // tile maxima per thread and round
constexpr int ZCAP_MAX = 8192;

// Candidate buffers for zcap candidates: z, list position and value row
// (zcap each), and up to zcap / 2 candidate 16-token tiles.
inline size_t tau_smem(int zcap) { return (size_t)zcap * 14; }

// The largest candidate capacity (a power of two in [1024, ZCAP_MAX]) that
// still lets the grid's CTAs share each SM in one wave.
inline int tau_zcap(int ctas, int sms) {
    const int per_sm = ctas > sms && sms > 0 ? ceil_div(ctas, sms) : 1;
    const size_t budget = (size_t)(220 << 10) / per_sm - (4 << 10);
    int z = ZCAP_MAX;
    while (z > 1024 && tau_smem(z) > budget) z >>= 1;
    return z;
}

// The entmax threshold: the root t of sum_c [z_c - t]_+^r = 1 over the
// candidates (every token with weight has z > z_max - 1), which lies in
// [lo, hi] = [z_max - 1, z_max - n^(1-alpha)] where F(t) = sum - 1 decreases.
// Newton's method, for r >= 1 (alpha <= 2) on g(t) = (sum_c [z_c - t]_+^r)^(1/r),
// a norm of (z - t)_+ and so convex (one step when the support's z are equal),
// from the left end; for r < 1 on F, which is then concave, from the right
// end: either way the iterates move to the root monotonically.
// for_each(add, first, stride) calls add(z) on candidates first, first +
// stride, ...  With n candidates, n <= TAU_WARP_MAX, warp 0 runs every pass
// by itself (lane-strided sums, a shuffle butterfly) and hands t to the other
// warps with one barrier at the end.  Otherwise each thread takes a
// TAU_NT-strided share and the warps' sums are added in warp order
// (reproducible), one barrier per pass (red is double-buffered).  All TAU_NT
// threads call it and return the same t.
constexpr int TAU_WARP_MAX = 256;
template <class ForEach>
__device__ float entmax_tau(ForEach for_each, int n, float lo, float hi, float zmax, float r, int ri,
                            float (*red)[TAU_NW][2]) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const bool per_warp = n <= TAU_WARP_MAX;
    const int first = per_warp ? lane : (int)threadIdx.x, stride = per_warp ? 32 : TAU_NT;
    const float tol = 1e-7f * fmaxf(1.f, fabsf(zmax));
    const int rim1 = ri >= 2 ? ri - 1 : 0;
    float t = r >= 1.f ? lo : hi;
    for (int it = 0; it < 40 && (!per_warp || warp == 0); ++it) {
        float s0 = 0.f, s1 = 0.f;  // sum x^r, sum x^(r-1) over x = z - t > 0
        auto add = [&](float z) {
            const float x = z - t;
            if (ri == 2) {  // alpha = 3/2: branch-free
                const float y = fmaxf(x, 0.f);
                s0 = fmaf(y, y, s0);
                s1 += y;
            } else if (x > 0.f) {
                const float y = ri == 1 ? 1.f : pos_pow(x, r - 1.f, rim1);
                s0 = fmaf(x, y, s0);
                s1 += y;
            }
        };
        for_each(add, first, stride);
#pragma unroll
        for (int o = 16; o; o >>= 1) {
            s0 += __shfl_xor_sync(FULL, s0, o);
            s1 += __shfl_xor_sync(FULL, s1, o);
        }
        float S0 = s0, S1 = s1;
        if (!per_warp) {
            if (lane == 0) {
                red[it & 1][warp][0] = s0;
                red[it & 1][warp][1] = s1;
            }
            __syncthreads();
            S0 = 0.f;
            S1 = 0.f;
#pragma unroll
            for (int ww = 0; ww < TAU_NW; ++ww) {
                S0 += red[it & 1][ww][0];
                S1 += red[it & 1][ww][1];
            }
        }
        if (!(S1 > 0.f)) break;  // no weight right of t (t at the top already)
        // r >= 1: t' = t + (S0 - S0^(1-1/r)) / S1;  r < 1: t' = t + (S0 - 1) / (r S1)
        float step;
        if (ri == 2) step = (S0 - sqrtf(S0)) / S1;
        else if (ri == 1) step = (S0 - 1.f) / S1;
        else if (r >= 1.f) step = (S0 - powf(S0, 1.f - 1.f / r)) / S1;
        else step = (S0 - 1.f) / (r * S1);
        const float tn = fminf(hi, fmaxf(lo, t + step));
        const bool done = !(fabsf(tn - t) > tol);
        t = tn;
        if (done) break;
    }
    if (per_warp) {
        __syncthreads();  // every warp is past the caller's earlier use of red
        if (threadIdx.x == 0) red[0][0][0] = t;
        __syncthreads();
        t = red[0][0][0];
    }
    return t;
}

// Exact threshold and (GATHER) the weighted sum of the support's value rows.
template <int D, bool GATHER>
__global__ void __launch_bounds__(TAU_NT, D == 64 ? 4 : 3) tau_pv_kernel(const __grid_constant__ DecodeArgs a, int dense, int zcap) {
    pdl_wait();
    constexpr int CPL = D / 32;
    // candidates in list order: z, list position and value row; once the
    // gather has read them, the same bytes hold the per-warp output partials
    extern __shared__ __align__(16) unsigned char tsm[];
    float *cz = reinterpret_cast<float *>(tsm);
    int *cpos = reinterpret_cast<int *>(tsm + (size_t)zcap * 4);
    int *crow = reinterpret_cast<int *>(tsm + (size_t)zcap * 8);
    int *ctile = reinterpret_cast<int *>(tsm + (size_t)zcap * 12);  // candidate 16-token tiles
    const int tcap = zcap / 2;
    double(*accs)[D] = reinterpret_cast<double(*)[D]>(tsm);
    __shared__ int wcnt[72];  // block scan scratch
    __shared__ float red[2][TAU_NW][2];  // double-buffered pass sums
    const int G = a.Hq / a.Hkv;
    int b, h;
    head_of(blockIdx.x, a.kv0 * G, a.nk * G, b, h);
    const int bh = b * a.Hq + h, kvh = h / G;
    const int bk = b * a.Hkv + kvh;
    const int P = a.P;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const bool given_tau = a.tau_in != nullptr;
    const bool export_cand = a.cand_z != nullptr;
    // the loads that depend on nothing are issued together: the query row (its
    // finite check), the running max of z and the union size
    const uint16_t qbits = threadIdx.x < D ? a.q[(size_t)bh * D + threadIdx.x] : (uint16_t)0;
    // max z of the head: the q.K kernel's running max, or, when the q.K CTAs
    // built the union themselves (nothing reset the running max), the max of
    // the tile maxima; in the sequence-sharded phases the global max z comes
    // in (and the candidates phase writes out this shard's candidate z values)
    const bool zmax_from_tiles = !a.zmax_in && a.union_in_qk;
    const int zord = a.zmax_in || zmax_from_tiles ? 0 : a.ws.zmax[bh];
    const int np = n_pages_of(seq_len_of(a.seq_lens, b, P, a.max_pages, a.status), P);
    const int U = dense ? np : a.ws.union_cnt[bk];
    // a query with a NaN or an infinity: NaN output and threshold, no candidates
    if (!__syncthreads_and(threadIdx.x >= D || (qbits & 0x7f80u) != 0x7f80u)) {
        if (threadIdx.x == 0) atomicOr(a.status, ENTMAXKV_STATUS_NONFINITE);
        if (export_cand) {
            if (threadIdx.x == 0) a.cand_n[bh] = 0;
            return;
        }
        if (GATHER)
            for (int j = threadIdx.x; j < D; j += TAU_NT) a.out[(size_t)bh * D + j] = __int_as_float(0x7fc00000);
        if (threadIdx.x == 0 && !given_tau) {
            a.ws.tau[bh] = __int_as_float(0x7fc00000);
            if (a.tau_out) a.tau_out[bh] = __int_as_float(0x7fc00000);
        }
        return;
    }
    const int n_tok = U * P;  // a multiple of 16
    const size_t trow = tile_row(a, b, h);
    const float *tr = a.ws.tmax + trow;
    const int n_tiles = n_tok / 16;
    const bool tvec = (trow & 3) == 0;
    // this thread's TAU_TB tile maxima of the round starting at tile t0
    auto load_tiles = [&](int t0, float(&v)[TAU_TB]) {
        const int p0 = t0 + threadIdx.x * TAU_TB;
        if (tvec && p0 + TAU_TB <= n_tiles) {
#pragma unroll
            for (int i = 0; i < TAU_TB / 4; ++i) {
                const float4 f = __ldcg(reinterpret_cast<const float4 *>(tr + p0) + i);
                v[4 * i] = f.x;
                v[4 * i + 1] = f.y;
                v[4 * i + 2] = f.z;
                v[4 * i + 3] = f.w;
            }
        } else {
#pragma unroll
            for (int i = 0; i < TAU_TB; ++i) v[i] = p0 + i < n_tiles ? __ldcg(tr + p0 + i) : -INFINITY;
        }
    };
    float v0[TAU_TB];  // the first round's tile maxima, kept for the candidate pass
    load_tiles(0, v0);
    float zmax;
    if (a.zmax_in) {
        zmax = a.zmax_in[bh];
    } else if (!zmax_from_tiles) {
        zmax = ord2f(zord);
    } else {
        __shared__ float s_wmax[TAU_NW];
        float m = -INFINITY;
#pragma unroll
        for (int i = 0; i < TAU_TB; ++i) m = fmaxf(m, v0[i]);
        for (int t0 = TAU_NT * TAU_TB; t0 < n_tiles; t0 += TAU_NT * TAU_TB) {
            float v[TAU_TB];
            load_tiles(t0, v);
#pragma unroll
            for (int i = 0; i < TAU_TB; ++i) m = fmaxf(m, v[i]);
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(FULL, m, o));
        if (lane == 0) s_wmax[warp] = m;
        __syncthreads();
        zmax = s_wmax[0];
#pragma unroll
        for (int w = 1; w < TAU_NW; ++w) zmax = fmaxf(zmax, s_wmax[w]);
    }
    const float r = 1.f / (a.alpha - 1.f);
    const int ri = a.r_int;
    if (!(zmax > -INFINITY) || (given_tau && !(a.tau_in[bh] == a.tau_in[bh]))) {  // no token at all
        if (export_cand) {
            if (threadIdx.x == 0) a.cand_n[bh] = 0;
            return;
        }
        if (GATHER)
            for (int j = threadIdx.x; j < D; j += TAU_NT) a.out[(size_t)bh * D + j] = 0.f;
        if (threadIdx.x == 0 && !given_tau) {
            a.ws.tau[bh] = __int_as_float(0x7fc00000);
            if (a.tau_out) a.tau_out[bh] = __int_as_float(0x7fc00000);
        }
        return;
    }
    // tokens that can carry weight: z > z_max - 1 (no weight exceeds 1), or,
    // with tau known, z > tau
    const float thr = given_tau ? a.tau_in[bh] : zmax - 1.f;
    const float *zr = a.ws.zbuf + tok_row(a, b, h);
    auto row_of_pos = [&](int pos) -> int {
        const int up = pos / P, t = pos - up * P;
        const int blk = dense ? __ldg(a.page_table + (size_t)b * a.max_pages + up)
                              : __ldcg(a.ws.union_blk + (size_t)bk * a.max_pages + up);
        return (blk * a.Hkv + kvh) * P + t;
    };

    // Candidates (z > z_max - 1) in list order, in two ordered block-wide
    // compactions: the 16-token tiles whose max clears the bar (TAU_TB tile
    // maxima per thread, loaded together), then their tokens (one tile per
    // thread: its 16 z and, for the gather, its page's value row, loaded
    // together).
    int ntc = 0;
    for (int t0 = 0; t0 < n_tiles; t0 += TAU_NT * TAU_TB) {
        const int p0 = t0 + threadIdx.x * TAU_TB;
        float v[TAU_TB];
        if (t0 == 0) {
#pragma unroll
            for (int i = 0; i < TAU_TB; ++i) v[i] = v0[i];
        } else {
            load_tiles(t0, v);
        }
        unsigned bits = 0;
#pragma unroll
        for (int i = 0; i < TAU_TB; ++i)
            if (v[i] > thr) bits |= 1u << i;
        int tot;
        int w = ntc + block_excl_scan(__popc(bits), wcnt, &tot);
#pragma unroll
        for (int i = 0; i < TAU_TB; ++i)
            if ((bits >> i) & 1u) {
                if (w < tcap) ctile[w] = p0 + i;
                ++w;
            }
        ntc += tot;
    }
    __syncthreads();
    int nc = 0;
    if (ntc <= tcap) {
        for (int r0 = 0; r0 < ntc && nc <= zcap; r0 += TAU_NT) {
            const int i = r0 + threadIdx.x;
            float zz[16];
            int pos0 = 0, row0 = 0;
            unsigned bits = 0;
            if (i < ntc) {
                pos0 = ctile[i] * 16;
                const float4 *zp = reinterpret_cast<const float4 *>(zr + pos0);
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const float4 f = __ldcg(zp + q4);
                    zz[4 * q4] = f.x;
                    zz[4 * q4 + 1] = f.y;
                    zz[4 * q4 + 2] = f.z;
                    zz[4 * q4 + 3] = f.w;
                }
                if (GATHER) row0 = row_of_pos(pos0);  // tiles never straddle pages
#pragma unroll
                for (int k = 0; k < 16; ++k)
                    if (zz[k] > thr) bits |= 1u << k;
                // the value rows of the candidates travel to L2 while tau is solved
                if (GATHER)
#pragma unroll
                    for (int k = 0; k < 16; ++k)
                        if ((bits >> k) & 1u) prefetch_l2_row<D>(a.v + (size_t)(row0 + k) * D);
            }
            int tot;
            int w = nc + block_excl_scan(__popc(bits), wcnt, &tot);
#pragma unroll
            for (int k = 0; k < 16; ++k)
                if ((bits >> k) & 1u) {
                    if (w < zcap) {
                        cz[w] = zz[k];
                        cpos[w] = pos0 + k;
                        if (GATHER) crow[w] = row0 + k;
                    }
                    ++w;
                }
            nc += tot;
        }
    } else {
        nc = zcap + 1;  // too many candidate tiles to list: the whole-row path below
    }
    __syncthreads();
    const bool onchip = nc <= zcap;
    if (export_cand) {
        // this shard's candidates, in list order, at most cap of them (the
        // count is exact either way)
        float *cz_out = a.cand_z + (size_t)bh * a.cap;
        int total = 0;
        if (onchip) {
            for (int i = threadIdx.x; i < min(nc, a.cap); i += TAU_NT) cz_out[i] = cz[i];
            total = nc;
        } else {
            for (int t0 = 0; t0 < n_tok; t0 += TAU_NT * 16) {
                const int e0 = t0 + threadIdx.x * 16;
                float zz[16];
                unsigned bits = 0;
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    zz[k] = e0 + k < n_tok ? __ldcg(zr + e0 + k) : -INFINITY;
                    if (zz[k] > thr) bits |= 1u << k;
                }
                int tot;
                int w = total + block_excl_scan(__popc(bits), wcnt, &tot);
#pragma unroll
                for (int k = 0; k < 16; ++k)
                    if ((bits >> k) & 1u) {
                        if (w < a.cap) cz_out[w] = zz[k];
                        ++w;
                    }
                total += tot;
            }
        }
        if (threadIdx.x == 0) {
            a.cand_n[bh] = total;
            if (total > a.cap) atomicOr(a.status, ENTMAXKV_STATUS_OVERFLOW);
        }
        return;
    }
    if (!onchip && threadIdx.x == 0) atomicOr(a.status, ENTMAXKV_STATUS_OVERFLOW);
    const int nloop = onchip ? nc : n_tok;
    auto cz_at = [&](int i) -> float { return onchip ? cz[i] : __ldcg(zr + i); };

    // the exact threshold (on chip nc is the exact candidate count; off chip
    // only a lower bound on it, so the bracket uses every token of the list);
    // the finish phase of a sharded decode takes it as given
    float tau = thr;
    if (!given_tau) {
        const float lo = thr;
        const float hi = zmax - powf((float)(onchip ? nc : n_tok), 1.f - a.alpha);
        if (nc > 1 && hi > lo) {
            if (onchip) {
                tau = entmax_tau([&](auto add, int f, int st) { for (int c = f; c < nc; c += st) add(cz[c]); }, nc,
                                 lo, hi, zmax, r, ri, red);
            } else {
                // too many candidates to hold: stream the z row through shared
                // memory in coalesced chunks of zcap
                // (n_tok > zcap >= 1024 here: the block-wide form)
                tau = entmax_tau(
                    [&](auto add, int f, int st) {
                        for (int c0 = 0; c0 < n_tok; c0 += zcap) {
                            const int m = min(zcap, n_tok - c0);
                            __syncthreads();  // the previous chunk has been read
                            for (int i = threadIdx.x; i < m; i += TAU_NT) cz[i] = __ldcg(zr + c0 + i);
                            __syncthreads();
                            for (int c = f; c < m; c += st) add(cz[c]);
                        }
                    },
                    n_tok, lo, hi, zmax, r, ri, red);
            }
        }
    }
    if (threadIdx.x == 0 && !given_tau) {
        a.ws.tau[bh] = tau;
        if (a.tau_out) a.tau_out[bh] = tau;
    }
    if constexpr (GATHER) {
        // p v over the support: every warp takes a strided share of the
        // candidates, moves the lanes with weight to the front eight at a time and
        // sums p v of their value rows in fp64 (exact products).
        double acc[CPL];
    #pragma unroll
        for (int c = 0; c < CPL; ++c) acc[c] = 0.0;
        const size_t lstride = (size_t)a.max_pages * P;
        auto put_p = [&](int pos, float p) {
            if (!a.p_out) return;
            const int up = pos / P, t = pos - up * P;
            const int page = dense ? up : (__ldcg(a.ws.union_e + (size_t)bk * a.max_pages + up) >> 8);
            a.p_out[(size_t)bh * lstride + (size_t)page * P + t] = p;
        };
        auto gather8 = [&](int nr, int row, float p) {
            // lanes 0..nr-1 hold (row, p) of up to eight support tokens; the
            // rows' bf16 words are all loaded before the first product
            unsigned vw[8][CPL / 2];
            float pp[8];
    #pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int rw = __shfl_sync(FULL, row, i);
                pp[i] = i < nr ? __shfl_sync(FULL, p, i) : 0.f;
                const uint16_t *vr = a.v + (size_t)rw * D + lane * CPL;
                if (CPL == 4) {
                    uint2 w = make_uint2(0u, 0u);
                    if (i < nr) w = __ldg(reinterpret_cast<const uint2 *>(vr));
                    vw[i][0] = w.x;
                    vw[i][CPL / 2 - 1] = w.y;
                } else {
                    vw[i][0] = i < nr ? __ldg(reinterpret_cast<const unsigned *>(vr)) : 0u;
                }
            }
    #pragma unroll
            for (int i = 0; i < 8; ++i)
    #pragma unroll
                for (int cc = 0; cc < CPL; ++cc) {
                    const unsigned w = vw[i][cc >> 1];
                    acc[cc] = fma((double)pp[i], (double)((cc & 1) ? bf16hi(w) : bf16lo(w)), acc[cc]);
                }
        };
        // candidate c belongs to warp c % TAU_NW (lane (c / TAU_NW) % 32), so a
        // small support spreads over all warps
        for (int k0 = 0; k0 < nloop; k0 += TAU_NT) {
            const int c = k0 + lane * TAU_NW + warp;
            const float z = c < nloop ? cz_at(c) : -INFINITY;
            const float p = pos_pow(z - tau, r, ri);
            unsigned bal = __ballot_sync(FULL, p > 0.f);
            while (bal) {
                int src = 0, nr = 0;
    #pragma unroll
                for (int i = 0; i < 8; ++i)
                    if (bal) {
                        const int l = __ffs(bal) - 1;
                        bal &= bal - 1;
                        if (lane == i) src = l;
                        nr = i + 1;
                    }
                const int cs = k0 + __shfl_sync(FULL, lane, src) * TAU_NW + warp;
                const float pl = __shfl_sync(FULL, p, src);
                int row = 0;
                if (lane < nr) {
                    const int pos = onchip ? cpos[cs] : cs;
                    row = onchip ? crow[cs] : row_of_pos(pos);
                    put_p(pos, pl);
                }
                gather8(nr, row, lane < nr ? pl : 0.f);
            }
        }
        __syncthreads();  // every warp is done with the candidates
    #pragma unroll
        for (int cc = 0; cc < CPL; ++cc) accs[warp][lane * CPL + cc] = acc[cc];
        __syncthreads();
        for (int j = threadIdx.x; j < D; j += TAU_NT) {
            double sum = 0.0;
    #pragma unroll
            for (int w = 0; w < TAU_NW; ++w) sum += accs[w][j];
            a.out[(size_t)bh * D + j] = (float)sum;
        }
    }
}

// ------------------------------------------- sequence-sharded decode pieces

// Per head: the shard's max z (after q.K): the q.K kernel's running max, or,
// when the q.K CTAs built the union themselves, the max of the 16-token tile
// maxima; -inf when it has none.  One CTA per head.
constexpr int ZX_NT = 128;
__global__ void __launch_bounds__(ZX_NT) zmax_export_kernel(DecodeArgs a) {
    pdl_wait();
    __shared__ float s_wmax[ZX_NT / 32];
    const int G = a.Hq / a.Hkv;
    int b, h;
    head_of(blockIdx.x, a.kv0 * G, a.nk * G, b, h);
    if (!a.union_in_qk) {
        if (threadIdx.x == 0) a.zmax_out[b * a.Hq + h] = ord2f(a.ws.zmax[b * a.Hq + h]);
        return;
    }
    const int n_tiles = a.ws.union_cnt[b * a.Hkv + h / G] * a.P / 16;
    const float *tr = a.ws.tmax + tile_row(a, b, h);
    float m = -INFINITY;
    for (int i = threadIdx.x; i < n_tiles; i += ZX_NT) m = fmaxf(m, __ldcg(tr + i));
#pragma unroll
    for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(FULL, m, o));
    if ((threadIdx.x & 31) == 0) s_wmax[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < ZX_NT / 32; ++w) m = fmaxf(m, s_wmax[w]);
        a.zmax_out[b * a.Hq + h] = fmaxf(m, s_wmax[0]);
    }
}

// Per head: the exact threshold over the candidates of all S shards (each
// shard's list in list order, the shards in order: the single-device list
// order when shards hold consecutive page ranges).
__global__ void __launch_bounds__(TAU_NT) threshold_kernel(const __grid_constant__ ThresholdArgs a) {
    pdl_wait();
    extern __shared__ float tz[];  // up to S * cap candidates
    __shared__ float red[2][TAU_NW][2];
    __shared__ int s_over;
    const int G = a.Hq / a.Hkv;
    int b, h;
    head_of(blockIdx.x, a.kv0 * G, a.nk * G, b, h);
    const int bh = b * a.Hq + h;
    const size_t BH = (size_t)a.B * a.Hq;
    const float zmax = a.zmax[bh];
    if (!(zmax > -INFINITY)) {
        if (threadIdx.x == 0) a.tau[bh] = __int_as_float(0x7fc00000);
        return;
    }
    if (threadIdx.x == 0) {
        int over = 0;
        for (int sh = 0; sh < a.S; ++sh) {
            const int c = a.cand_n[sh * BH + bh];
            over |= c > a.cap || c < 0;
        }
        s_over = over;
    }
    __syncthreads();
    int n = 0;
    for (int sh = 0; sh < a.S; ++sh) {
        const int c = min(max(a.cand_n[sh * BH + bh], 0), a.cap);
        const float *src = a.cand_z + (sh * BH + bh) * a.cap;
        for (int i = threadIdx.x; i < c; i += TAU_NT) tz[n + i] = __ldcg(src + i);
        n += c;
    }
    __syncthreads();
    if (s_over && threadIdx.x == 0) atomicOr(a.status, ENTMAXKV_STATUS_OVERFLOW);
    const float r = 1.f / (a.alpha - 1.f);
    const float lo = zmax - 1.f, hi = zmax - powf((float)n, 1.f - a.alpha);
    float tau = lo;
    if (n > 1 && hi > lo)
        tau = entmax_tau([&](auto add, int f, int st) { for (int c = f; c < n; c += st) add(tz[c]); }, n, lo, hi,
                         zmax, r, a.r_int, red);
    if (threadIdx.x == 0) a.tau[bh] = tau;
}

// ------------------------------------------------- partial-sum combination

// Called by all threads of a CTA after it wrote its partial for the heads of
// group bk.  The last CTA of the group to arrive sums the S partials of each
// head in slot order and writes the output.
template <int D, int G>
__device__ __forceinline__ void combine_last(const DecodeArgs &a, int bk, int b, int kvh, int S, bool softmax) {
    __shared__ int s_last;
    __shared__ unsigned s_qbad;  // bit g: head g's query is not finite (its output is NaN)
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = atomicAdd(&a.ws.counters[bk], 1) == S - 1;
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    if (threadIdx.x == 0) {
        unsigned m = 0u;
        for (int g = 0; g < G; ++g)
            if (!q_row_finite(a.q + ((size_t)b * a.Hq + kvh * G + g) * D, D)) m |= 1u << g;
        s_qbad = m;
        if (m) atomicOr(a.status, ENTMAXKV_STATUS_NONFINITE);
    }
    __syncthreads();
    const int BH = a.B * a.Hq;
    for (int i = threadIdx.x; i < G * D; i += blockDim.x) {
        const int g = i / D, j = i % D;
        const int bh = b * a.Hq + kvh * G + g;
        if ((s_qbad >> g) & 1u) {
            a.out[(size_t)bh * D + j] = __int_as_float(0x7fc00000);
            if (j == 0 && softmax && a.tau_out) a.tau_out[bh] = __int_as_float(0x7fc00000);
            continue;
        }
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
            if (j == 0 && a.tau_out) a.tau_out[bh] = den > 0.f ? M + logf(den) : __int_as_float(0x7fc00000);
        }
    }
    if (threadIdx.x == 0) a.ws.counters[bk] = 0;
}

// ------------------------------------------------- p.V, full-cache stream

// Every V tile of the cache passes through a TMA ring; the producer also
// copies the tiles' z rows for the G heads, so p = [z - tau]_+^r is formed in
// registers straight in the B-operand layout (lane: head lane / 4, tokens
// 2 (lane % 4) + {0, 1, 8, 9}).  A warp takes whole 16-token steps and skips
// the MMAs of a step whose p are all zero (most of them: entmax is sparse).
constexpr int PVS_NS = 3;

template <int D, int G>
constexpr size_t pvs_smem() {
    return ((Ring<D, G, PVS_NS, 1>::BYTES + 127) & ~(size_t)127) + (size_t)PVS_NS * G * Tile<G>::TPS * 4;
}

template <int D, int G>
__global__ void __launch_bounds__(DEC_THREADS) pv_stream_kernel(const __grid_constant__ DecodeArgs a) {
    pdl_wait();
    constexpr int NS = PVS_NS;
    using RG = Ring<D, G, NS, 1>;
    constexpr int TPS = RG::TPS;
    extern __shared__ unsigned char smem_raw[];
    RingView<D, G, NS, 1> R(smem_raw);
    float *zst = reinterpret_cast<float *>(smem_raw + ((RG::BYTES + 127) & ~(size_t)127));
    __shared__ float red[NWC][G][D];

    int b, kvh;
    group_of(blockIdx.y, a.kv0, a.nk, b, kvh);
    const int bk = b * a.Hkv + kvh;
    const int P = a.P, PPS = TPS / P;
    const int seq = seq_len_of(a.seq_lens, b, P, a.max_pages, a.status);
    const int np = n_pages_of(seq, P);
    const int nsteps = ceil_div(np, PPS);
    const int S = gridDim.x;
    const int my_n = nsteps > (int)blockIdx.x ? ceil_div(nsteps - blockIdx.x, S) : 0;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&R.full[s], 1);
            mbar_init(&R.empty[s], NWC);
        }
        mbar_fence_init();
    }
    __syncthreads();

    if (warp == NWC) {
        produce<D, 1, G>(a, &a.vmap, &a.vmap, true, b, kvh, bk, np, my_n, PPS, NS, RG::STAGE, 0, R.stages, R.full,
                         R.empty, R.pinfo, R.stash, zst, TPS);
    } else {
        const float r = 1.f / (a.alpha - 1.f);
        const int ri = a.r_int;
        const int n = lane >> 2, kp = 2 * (lane & 3);  // B operand: head n, tokens kp, kp+1, kp+8, kp+9
        const float tau = n < G ? a.ws.tau[b * a.Hq + kvh * G + n] : __int_as_float(0x7fc00000);
        float acc[D / 16][4];
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
        for (int it = 0; it < my_n; ++it) {
            const int st = it % NS, ph = (it / NS) & 1;
            if (!mbar_wait(&R.full[st], ph, a.status)) break;
            const unsigned char *stage = R.stages + (size_t)st * RG::STAGE;
            const PageInfo *pis = R.pinfo + st * PPS_MAX;
            for (int kt = warp; kt < TPS / 16; kt += NWC) {
                const int tok0 = kt * 16, pi_i = tok0 / P, r0 = tok0 % P;
                const PageInfo pi = pis[pi_i];
                if (pi.nval <= r0) continue;  // no page, or no valid token in this step
                float p[4] = {0.f, 0.f, 0.f, 0.f};
                if (n < G) {
                    const float *zr = zst + (size_t)(st * G + n) * TPS + tok0 + kp;
                    const float2 za = *reinterpret_cast<const float2 *>(zr);
                    const float2 zb = *reinterpret_cast<const float2 *>(zr + 8);
                    p[0] = pos_pow(za.x - tau, r, ri);
                    p[1] = pos_pow(za.y - tau, r, ri);
                    p[2] = pos_pow(zb.x - tau, r, ri);
                    p[3] = pos_pow(zb.y - tau, r, ri);
                    if (a.p_out) {
                        float *po = a.p_out + tok_row(a, b, kvh * G + n) + (size_t)pi.page * P + r0 + kp;
#pragma unroll
                        for (int v = 0; v < 4; ++v)
                            if (r0 + kp + (v & 1) + 8 * (v >> 1) < pi.nval) po[(v & 1) + 8 * (v >> 1)] = p[v];
                    }
                }
                if (!__any_sync(FULL, p[0] > 0.f || p[1] > 0.f || p[2] > 0.f || p[3] > 0.f)) continue;
                unsigned bh0, bh1, bl0, bl1;
                split_pair(p[0], p[1], bh0, bl0);
                split_pair(p[2], p[3], bh1, bl1);
                pv_mma<D>(acc, stage + (size_t)pi_i * P * D * 2, P, r0, pi.nval, bh0, bh1, bl0, bl1);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&R.empty[st]);
        }
        // acc[mt][v]: coordinate 16 mt + lane/4 + 8 (v >> 1), head 2 (lane % 4) + (v & 1)
        const int h0 = 2 * (lane & 3);
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt)
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                const int hh = h0 + (v & 1);
                if (hh < G) red[warp][hh][16 * mt + (lane >> 2) + 8 * (v >> 1)] = acc[mt][v];
            }
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

// K and V tiles of each step through one TMA ring.  A warp owns whole
// 16-token steps: scores on the tensor cores (tokens as M, the group's heads
// as N), its own running max and sum per head (the lane's two heads), p
// through a small per-warp scratch into the B-operand layout, then P.V on the
// tensor cores.  The warps' states are merged at the end of the CTA, and the
// CTAs' in a fixed order by the last one of the group.
template <int D, int G, bool SPARSE>
__global__ void __launch_bounds__(DEC_THREADS) softmax_kernel(const __grid_constant__ DecodeArgs a) {
    pdl_wait();
    constexpr int NS = 3;
    using RG = Ring<D, G, NS, 2>;
    constexpr int TPS = RG::TPS;
    constexpr int HALF = RG::STAGE / 2;
    extern __shared__ unsigned char smem_raw[];
    RingView<D, G, NS, 2> R(smem_raw);
    __shared__ __align__(16) uint16_t pw[NWC][2][8][16];  // per warp: p as [hi/lo][head][token]
    __shared__ float red[NWC][G][D];
    __shared__ float redm[NWC][G], redl[NWC][G];

    int b, kvh;
    group_of(blockIdx.y, a.kv0, a.nk, b, kvh);
    const int bk = b * a.Hkv + kvh;
    const int P = a.P, PPS = TPS / P;
    const int seq = seq_len_of(a.seq_lens, b, P, a.max_pages, a.status);
    const int np = n_pages_of(seq, P);
    const int U = SPARSE ? a.ws.union_cnt[bk] : np;  // pages to read: the group's union, or all
    const int nsteps = ceil_div(U, PPS);
    const int S = gridDim.x;
    const int my_n = nsteps > (int)blockIdx.x ? ceil_div(nsteps - blockIdx.x, S) : 0;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float sscale = D == 64 ? 0.125f : 0.08838834764831845f;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&R.full[s], 1);
            mbar_init(&R.empty[s], NWC);
        }
        mbar_fence_init();
    }
    __syncthreads();

    if (warp == NWC) {
        produce<D, 2>(a, &a.kmap, &a.vmap, !SPARSE, b, kvh, bk, U, my_n, PPS, NS, RG::STAGE, HALF, R.stages, R.full,
                      R.empty, R.pinfo, R.stash);
    } else {
        // B fragments of q: head n = lane/4 (zero for n >= G), coordinate pair 2 (lane % 4)
        unsigned qb[D / 16][2];
        const int n = lane >> 2, kp = 2 * (lane & 3);
        {
            const uint16_t *qh = a.q + ((size_t)b * a.Hq + kvh * G + (n < G ? n : 0)) * D;
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                qb[ks][0] = n < G ? *reinterpret_cast<const unsigned *>(qh + 16 * ks + kp) : 0u;
                qb[ks][1] = n < G ? *reinterpret_cast<const unsigned *>(qh + 16 * ks + kp + 8) : 0u;
            }
        }
        const int h0 = kp;  // this lane's heads in the score and output fragments: h0, h0 + 1
        float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
        float acc[D / 16][4];
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
        uint16_t(*pwh)[16] = pw[warp][0];
        uint16_t(*pwl)[16] = pw[warp][1];
        for (int it = 0; it < my_n; ++it) {
            const int st = it % NS, ph = (it / NS) & 1;
            if (!mbar_wait(&R.full[st], ph, a.status)) break;
            const unsigned char *stage = R.stages + (size_t)st * RG::STAGE;
            const PageInfo *pis = R.pinfo + st * PPS_MAX;
            for (int kt = warp; kt < TPS / 16; kt += NWC) {
                const int tok0 = kt * 16, pi_i = tok0 / P, r0 = tok0 % P;
                const PageInfo pi = pis[pi_i];
                if (pi.nval <= r0) continue;  // no page, or no valid token in this step
                const unsigned char *kbase = stage + (size_t)pi_i * P * D * 2;
                float c4[4] = {0.f, 0.f, 0.f, 0.f};
                {
                    const int mat = lane >> 3, rr = lane & 7;
                    const int row = r0 + (mat & 1) * 8 + rr;
#pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks) {
                        unsigned a0, a1, a2, a3;
                        ldsm_x4(smem_u32(tile_chunk(kbase, P, row, ks * 2 + (mat >> 1))), a0, a1, a2, a3);
                        mma_bf16_16816(c4, a0, a1, a2, a3, qb[ks][0], qb[ks][1]);
                    }
                }
                // c4[v]: token r0 + lane/4 + 8 (v >> 1), head h0 + (v & 1); a head
                // scores only the pages it selected (all of them when dense)
                float sv[4];
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    const int hh = h0 + (v & 1);
                    const int t = r0 + (lane >> 2) + 8 * (v >> 1);
                    sv[v] = (hh < G && t < pi.nval && ((pi.mask >> hh) & 1)) ? c4[v] * sscale : -INFINITY;
                }
                float x0 = fmaxf(sv[0], sv[2]), x1 = fmaxf(sv[1], sv[3]);
#pragma unroll
                for (int o = 4; o < 32; o <<= 1) {
                    x0 = fmaxf(x0, __shfl_xor_sync(FULL, x0, o));
                    x1 = fmaxf(x1, __shfl_xor_sync(FULL, x1, o));
                }
                const float n0 = fmaxf(m0, x0), n1 = fmaxf(m1, x1);
                const float c0 = n0 == -INFINITY ? 1.f : expf(m0 - n0);
                const float c1 = n1 == -INFINITY ? 1.f : expf(m1 - n1);
                if (__any_sync(FULL, c0 != 1.f || c1 != 1.f)) {
#pragma unroll
                    for (int mt = 0; mt < D / 16; ++mt) {
                        acc[mt][0] *= c0;
                        acc[mt][2] *= c0;
                        acc[mt][1] *= c1;
                        acc[mt][3] *= c1;
                    }
                }
                m0 = n0;
                m1 = n1;
                float p[4];
#pragma unroll
                for (int v = 0; v < 4; ++v) p[v] = sv[v] > -INFINITY ? expf(sv[v] - ((v & 1) ? n1 : n0)) : 0.f;
                l0 = l0 * c0 + (p[0] + p[2]);
                l1 = l1 * c1 + (p[1] + p[3]);
                // p^T into the B-operand layout through the warp's scratch
                __syncwarp();
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    const int hh = h0 + (v & 1), t = (lane >> 2) + 8 * (v >> 1);
                    const uint16_t hi = f2bf(p[v]);
                    pwh[hh][t] = hi;
                    pwl[hh][t] = f2bf(p[v] - bf16f(hi));
                }
                __syncwarp();
                const unsigned bh0 = *reinterpret_cast<const unsigned *>(&pwh[n][kp]);
                const unsigned bh1 = *reinterpret_cast<const unsigned *>(&pwh[n][kp + 8]);
                const unsigned bl0 = *reinterpret_cast<const unsigned *>(&pwl[n][kp]);
                const unsigned bl1 = *reinterpret_cast<const unsigned *>(&pwl[n][kp + 8]);
                pv_mma<D>(acc, stage + HALF + (size_t)pi_i * P * D * 2, P, r0, pi.nval, bh0, bh1, bl0, bl1);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&R.empty[st]);
        }
        // sums over the lanes that hold the same heads; then the warp's state
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
            l0 += __shfl_xor_sync(FULL, l0, o);
            l1 += __shfl_xor_sync(FULL, l1, o);
        }
        if (lane < 4) {
            if (h0 < G) {
                redm[warp][h0] = m0;
                redl[warp][h0] = l0;
            }
            if (h0 + 1 < G) {
                redm[warp][h0 + 1] = m1;
                redl[warp][h0 + 1] = l1;
            }
        }
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt)
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                const int hh = h0 + (v & 1);
                if (hh < G) red[warp][hh][16 * mt + (lane >> 2) + 8 * (v >> 1)] = acc[mt][v];
            }
    }
    __syncthreads();
    // the CTA's partial per head: max, sum and numerator, the warps merged in order
    const int BH = a.B * a.Hq;
    for (int i = threadIdx.x; i < G * D; i += blockDim.x) {
        const int g = i / D, j = i % D;
        const size_t o = ((size_t)blockIdx.x * BH + b * a.Hq + kvh * G + g) * (D + 2);
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < NWC; ++w) M = fmaxf(M, redm[w][g]);
        float num = 0.f, den = 0.f;
#pragma unroll
        for (int w = 0; w < NWC; ++w) {
            const float mw = redm[w][g];
            if (!(mw > -INFINITY)) continue;
            const float sc = expf(mw - M);
            num = fmaf(sc, red[w][g][j], num);
            den = fmaf(sc, redl[w][g], den);
        }
        a.ws.partial[o + 2 + j] = num;
        if (j == 0) {
            a.ws.partial[o] = M;
            a.ws.partial[o + 1] = den;
        }
    }
    combine_last<D, G>(a, bk, b, kvh, S, true);
}

// ---------------------------------------------------------------- launch

// Splits per (sequence, kv head) so that the whole grid fits one wave of
// per_sm resident CTAs on every SM.
int pick_splits(int sms, int per_sm, int groups, int max_steps, int cap) {
    int s = (sms * per_sm) / (groups > 0 ? groups : 1);
    if (s > max_steps) s = max_steps;
    if (s > cap) s = cap;
    return s < 1 ? 1 : s;
}

template <class K>
cudaError_t set_smem(K kern, size_t bytes) {
    return ensure_smem(reinterpret_cast<const void *>(kern), bytes);
}

template <int D, int G, bool DENSE>
cudaError_t launch_qk(const DecodeArgs &a, cudaStream_t st) {
    using RG = Ring<D, G, QK_NS, 1>;
    auto k = qk_kernel<D, G, DENSE>;
    cudaError_t e = set_smem(k, RG::BYTES);
    if (e != cudaSuccess) return e;
    const int groups = a.B * a.nk;
    const int S = pick_splits(a.sms, QK_PER_SM, groups, ceil_div(a.max_pages, RG::TPS / a.P), 1 << 16);
    return launch_pdl(k, dim3(S, groups), dim3(DEC_THREADS), RG::BYTES, st, a);
}

// The union of each group's selections for the sparse q.K pass.  With at
// most UNION_IN_QK_SPLITS q.K CTAs per group (many groups) each CTA builds its
// group's union itself (union_in_cta) when the G page bitmaps fit in its ring;
// otherwise union_kernel builds it first, once per group, rather than every
// CTA of a wide split repeating it.  Returns the arguments for q.K and the
// kernels after it, with the choice recorded.
constexpr int UNION_IN_QK_SPLITS = 2;

template <int D, int G>
bool union_in_qk_for(const DecodeArgs &a) {
    using RG = Ring<D, G, QK_NS, 1>;
    const int S = pick_splits(a.sms, QK_PER_SM, a.B * a.nk, ceil_div(a.max_pages, RG::TPS / a.P), 1 << 16);
    const bool fits = (size_t)G * ceil_div(a.max_pages, 32) * 4 <= (size_t)QK_NS * RG::STAGE;
    return S <= UNION_IN_QK_SPLITS && fits;
}

template <int D, int G>
cudaError_t launch_union(const DecodeArgs &a, cudaStream_t st, DecodeArgs &out) {
    out = a;
    out.union_in_qk = union_in_qk_for<D, G>(a);
    if (out.union_in_qk) return cudaSuccess;
    return launch_pdl(union_kernel, dim3(a.B * a.nk), dim3(UTH), 0, st, out);
}

// Kernels one sparse decode launches: softmax (union, softmax_kernel), or
// entmax ([union,] q.K, tau with p.V).
template <int D, int G>
int sparse_kernels_t(const DecodeArgs &a) {
    if (a.alpha == 1.f) return 2;
    return union_in_qk_for<D, G>(a) ? 2 : 3;
}

template <int D, int G>
cudaError_t sparse_t(const DecodeArgs &a, cudaStream_t st) {
    cudaError_t e;
    const int groups = a.B * a.nk;
    if (a.alpha == 1.f) {
        // softmax over the selected pages: the union, then K and V of its
        // pages, split over pages
        if ((e = launch_pdl(union_kernel, dim3(groups), dim3(UTH), 0, st, a)) != cudaSuccess) return e;
        using RG = Ring<D, G, 3, 2>;
        auto k = softmax_kernel<D, G, true>;
        if ((e = set_smem(k, RG::BYTES)) != cudaSuccess) return e;
        const int S = pick_splits(a.sms, 2, groups, ceil_div(a.max_pages, RG::TPS / a.P), MAX_SPLITS);
        return launch_pdl(k, dim3(S, groups), dim3(DEC_THREADS), RG::BYTES, st, a);
    }
    DecodeArgs u;
    if ((e = launch_union<D, G>(a, st, u)) != cudaSuccess) return e;
    if ((e = launch_qk<D, G, false>(u, st)) != cudaSuccess) return e;
    const int nheads = a.B * a.nk * (a.Hq / a.Hkv);
    const int zcap = tau_zcap(nheads, a.sms);
    if ((e = set_smem(tau_pv_kernel<D, true>, tau_smem(ZCAP_MAX))) != cudaSuccess) return e;
    return launch_pdl(tau_pv_kernel<D, true>, dim3(nheads), dim3(TAU_NT), tau_smem(zcap), st, u, 0, zcap);
}

// The decode of a step whose selection kernel marked each group's union in
// ws.umap (G > 1: union_map_kernel compacts it) or wrote it (G = 1), then
// q.K and tau with p.V.
template <int D, int G>
cudaError_t step_tail_t(const DecodeArgs &a, cudaStream_t st) {
    cudaError_t e;
    DecodeArgs u = a;
    u.union_in_qk = 0;
    if (G > 1 && (e = launch_pdl(union_map_kernel, dim3(a.B * a.nk), dim3(UMT), 0, st, u)) != cudaSuccess) return e;
    if ((e = launch_qk<D, G, false>(u, st)) != cudaSuccess) return e;
    const int nheads = a.B * a.nk * G;
    const int zcap = tau_zcap(nheads, a.sms);
    if ((e = set_smem(tau_pv_kernel<D, true>, tau_smem(ZCAP_MAX))) != cudaSuccess) return e;
    return launch_pdl(tau_pv_kernel<D, true>, dim3(nheads), dim3(TAU_NT), tau_smem(zcap), st, u, 0, zcap);
}

template <int D, int G>
cudaError_t begin_t(const DecodeArgs &a, cudaStream_t st) {
    cudaError_t e;
    DecodeArgs u;
    if ((e = launch_union<D, G>(a, st, u)) != cudaSuccess) return e;
    if ((e = launch_qk<D, G, false>(u, st)) != cudaSuccess) return e;
    return launch_pdl(zmax_export_kernel, dim3(a.B * a.nk * G), dim3(ZX_NT), 0, st, u);
}

template <int D, int G>
cudaError_t candidates_t(const DecodeArgs &a, cudaStream_t st) {
    cudaError_t e;
    const int nheads = a.B * a.nk * G;
    const int zcap = tau_zcap(nheads, a.sms);
    if ((e = set_smem(tau_pv_kernel<D, false>, tau_smem(ZCAP_MAX))) != cudaSuccess) return e;
    return launch_pdl(tau_pv_kernel<D, false>, dim3(nheads), dim3(TAU_NT), tau_smem(zcap), st, a, 0, zcap);
}

template <int D, int G>
cudaError_t finish_t(const DecodeArgs &a, cudaStream_t st) {
    cudaError_t e;
    const int nheads = a.B * a.nk * G;
    const int zcap = tau_zcap(nheads, a.sms);
    if ((e = set_smem(tau_pv_kernel<D, true>, tau_smem(ZCAP_MAX))) != cudaSuccess) return e;
    return launch_pdl(tau_pv_kernel<D, true>, dim3(nheads), dim3(TAU_NT), tau_smem(zcap), st, a, 0, zcap);
}

template <int D, int G>
cudaError_t dense_entmax_t(const DecodeArgs &a, cudaStream_t st) {
    cudaError_t e;
    const int groups = a.B * a.nk;
    const int n = a.B * a.nk * (a.Hq / a.Hkv);
    if ((e = launch_pdl(dense_init_kernel, dim3(ceil_div(n, 256)), dim3(256), 0, st, a)) != cudaSuccess) return e;
    if ((e = launch_qk<D, G, true>(a, st)) != cudaSuccess) return e;
    const int nheads = a.B * a.nk * (a.Hq / a.Hkv);
    const int zcap = tau_zcap(nheads, a.sms);
    if ((e = set_smem(tau_pv_kernel<D, false>, tau_smem(ZCAP_MAX))) != cudaSuccess) return e;
    if ((e = launch_pdl(tau_pv_kernel<D, false>, dim3(nheads), dim3(TAU_NT), tau_smem(zcap), st, a, 1, zcap)) !=
        cudaSuccess)
        return e;
    auto k = pv_stream_kernel<D, G>;
    constexpr size_t smem = pvs_smem<D, G>();
    if ((e = set_smem(k, smem)) != cudaSuccess) return e;
    const int S = pick_splits(a.sms, 3, groups, ceil_div(a.max_pages, Tile<G>::TPS / a.P), MAX_SPLITS);
    return launch_pdl(k, dim3(S, groups), dim3(DEC_THREADS), smem, st, a);
}

template <int D, int G>
cudaError_t dense_softmax_t(const DecodeArgs &a, cudaStream_t st) {
    cudaError_t e;
    const int groups = a.B * a.nk;
    const int n = a.B * a.nk * (a.Hq / a.Hkv);
    if ((e = launch_pdl(dense_init_kernel, dim3(ceil_div(n, 256)), dim3(256), 0, st, a)) != cudaSuccess) return e;
    using RG = Ring<D, G, 3, 2>;
    auto k = softmax_kernel<D, G, false>;
    if ((e = set_smem(k, RG::BYTES)) != cudaSuccess) return e;
    const int S = pick_splits(a.sms, 2, groups, ceil_div(a.max_pages, RG::TPS / a.P), MAX_SPLITS);
    return launch_pdl(k, dim3(S, groups), dim3(DEC_THREADS), RG::BYTES, st, a);
}

}  // namespace

#define EKV_DISPATCH(FN, a, st)                   \
    do {                                          \
        const int G_ = (a).Hq / (a).Hkv;          \
        if ((a).d == 64) {                        \
            switch (G_) {                         \
                case 1: return FN<64, 1>(a, st);  \
                case 2: return FN<64, 2>(a, st);  \
                case 4: return FN<64, 4>(a, st);  \
                case 8: return FN<64, 8>(a, st);  \
            }                                     \
        } else {                                  \
            switch (G_) {                         \
                case 1: return FN<128, 1>(a, st); \
                case 2: return FN<128, 2>(a, st); \
                case 4: return FN<128, 4>(a, st); \
                case 8: return FN<128, 8>(a, st); \
            }                                     \
        }                                         \
        return cudaErrorInvalidValue;             \
    } while (0)

cudaError_t launch_decode_sparse(const DecodeArgs &a, cudaStream_t st) { EKV_DISPATCH(sparse_t, a, st); }

int decode_sparse_kernels(const DecodeArgs &a) {
    const int G = a.Hq / a.Hkv;
    if (a.d == 64) {
        switch (G) {
            case 1: return sparse_kernels_t<64, 1>(a);
            case 2: return sparse_kernels_t<64, 2>(a);
            case 4: return sparse_kernels_t<64, 4>(a);
            case 8: return sparse_kernels_t<64, 8>(a);
        }
    } else {
        switch (G) {
            case 1: return sparse_kernels_t<128, 1>(a);
            case 2: return sparse_kernels_t<128, 2>(a);
            case 4: return sparse_kernels_t<128, 4>(a);
            case 8: return sparse_kernels_t<128, 8>(a);
        }
    }
    return -1;
}
cudaError_t launch_decode_step_tail(const DecodeArgs &a, cudaStream_t st) { EKV_DISPATCH(step_tail_t, a, st); }
int decode_step_tail_kernels(const DecodeArgs &a) { return a.Hq / a.Hkv > 1 ? 3 : 2; }
cudaError_t launch_decode_sparse_begin(const DecodeArgs &a, cudaStream_t st) { EKV_DISPATCH(begin_t, a, st); }
cudaError_t launch_decode_sparse_candidates(const DecodeArgs &a, cudaStream_t st) {
    EKV_DISPATCH(candidates_t, a, st);
}
cudaError_t launch_decode_sparse_finish(const DecodeArgs &a, cudaStream_t st) { EKV_DISPATCH(finish_t, a, st); }

cudaError_t launch_entmax_threshold(const ThresholdArgs &a, cudaStream_t st) {
    const size_t smem = (size_t)a.S * a.cap * 4;
    cudaError_t e = set_smem(threshold_kernel, smem);
    if (e != cudaSuccess) return e;
    const int nheads = a.B * a.nk * (a.Hq / a.Hkv);
    return launch_pdl(threshold_kernel, dim3(nheads), dim3(TAU_NT), smem, st, a);
}
cudaError_t launch_decode_dense_entmax(const DecodeArgs &a, cudaStream_t st) { EKV_DISPATCH(dense_entmax_t, a, st); }
cudaError_t launch_decode_dense_softmax(const DecodeArgs &a, cudaStream_t st) {
    EKV_DISPATCH(dense_softmax_t, a, st);
}

size_t decode_ws_bytes(bool dense, int B, int Hq, int Hkv, int d, int P, int max_pages, DecodeWs *carve,
                       void *base, bool step) {
    size_t off = 0;
    auto take = [&](size_t bytes) {
        size_t o = off;
        off += (bytes + 255) & ~(size_t)255;
        return o;
    };
    const size_t tokens = (size_t)B * Hq * max_pages * P;
    const int uwords = (ceil_div(max_pages, 4) + 3) & ~3;
    const size_t o_union = take(dense ? 0 : (size_t)B * Hkv * max_pages * 4);
    const size_t o_ublk = take(dense ? 0 : (size_t)B * Hkv * max_pages * 4);
    const size_t o_ucnt = take((size_t)B * Hkv * 4);
    const size_t o_zmax = take((size_t)B * Hq * 4);
    const size_t o_tau = take((size_t)B * Hq * 4);
    const size_t o_cnt = take((size_t)B * Hkv * 4);
    const size_t o_part = take((size_t)MAX_SPLITS * B * Hq * (d + 2) * 4);  // split-K softmax partials
    const size_t o_z = take(tokens * 4);
    const size_t o_t = take(tokens / 16 * 4);
    // decode step: the union marks, one row per group
    const size_t o_umap = take(step ? (size_t)B * Hkv * uwords * 4 : 0);
    if (carve && base) {
        char *p = static_cast<char *>(base);
        carve->union_e = reinterpret_cast<int *>(p + o_union);
        carve->union_blk = reinterpret_cast<int *>(p + o_ublk);
        carve->union_cnt = reinterpret_cast<int *>(p + o_ucnt);
        carve->zmax = reinterpret_cast<int *>(p + o_zmax);
        carve->tau = reinterpret_cast<float *>(p + o_tau);
        carve->counters = reinterpret_cast<int *>(p + o_cnt);
        carve->partial = reinterpret_cast<float *>(p + o_part);
        carve->zbuf = reinterpret_cast<float *>(p + o_z);
        carve->tmax = reinterpret_cast<float *>(p + o_t);
        carve->umap = step ? reinterpret_cast<unsigned *>(p + o_umap) : nullptr;
        carve->uwords = uwords;
    }
    return off;
}

}  // namespace ekv
