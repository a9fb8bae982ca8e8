/*
 * entmaxkv.h -- C ABI of libentmaxkv.so: paged, support-aware alpha-entmax
 * decode attention for NVIDIA B200 (sm_100a).
 *
 * The operations follow "EntmaxKV - Support-aware decoding for entmax
 * attention" (technical summary, gist.science paper 2605.21649; the same text
 * exists in Spanish, Japanese, Korean and Arabic).  One decode step, for
 * every (sequence b, query head h), against a paged bf16 K/V cache:
 *
 *   entmaxkv_build_meta     per-page metadata (section 2.A)
 *   entmaxkv_append         write each sequence's new key/value row and
 *                           refresh the metadata of its page (section 2.A)
 *   entmaxkv_score_pages    query-aware page scores (section 2.A)
 *   entmaxkv_select         candidate pages: top-k or Gaussian tau_hat - Delta
 *                           (section 2.B)
 *   entmaxkv_decode_sparse  exact alpha-entmax attention over the selected
 *                           pages only (section 2.C)
 *   entmaxkv_decode_dense   full-cache entmax, or full-cache softmax split-K,
 *                           the comparison points of section 4 "Efficiency"
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Pointers named *_cache, q, meta, page_table, seq_lens, scores, sel, cnt,
 *   out, workspace are DEVICE pointers owned by the caller; the library never
 *   allocates, frees or keeps them.  `stream` is a cudaStream_t passed as
 *   void* (NULL = legacy default stream).  Every call only enqueues work on
 *   that stream and returns; it never synchronises the host (except
 *   entmaxkv_get_status, which is a query).
 * - Return value: ENTMAXKV_OK (0) or a negative ENTMAXKV_ERR_* code.  All
 *   argument checks run on the host before anything is launched, so an error
 *   return means nothing was enqueued.  ENTMAXKV_ERR_CUDA reports a failed
 *   launch (cudaGetLastError).
 * - Errors the host cannot see (a page-table entry outside [0, num_blocks), a
 *   selected page index outside the sequence, a sequence length above
 *   max_pages * P, a non-finite query, a wait that ran out) are recorded in a
 *   per-device status word (ENTMAXKV_STATUS_* bits, OR-ed) read with
 *   entmaxkv_get_status.  Kernels never trap; the offending page is skipped,
 *   an over-long sequence is clamped to max_pages * P tokens.
 * - Non-finite queries: a query row (b, h) holding a NaN or +-Inf gets NaN
 *   scores from entmaxkv_score_pages (bbox, mu and sigma of every page), and
 *   out[b][h][*] = NaN, tau_out[b][h] = NaN from every decode call; the call
 *   sets ENTMAXKV_STATUS_NONFINITE.  Other heads are computed as usual.
 * - Layouts (row-major, all contiguous):
 *     k_cache, v_cache  bf16  [num_blocks][Hkv][P][d]   16-byte aligned
 *     q                 bf16  [B][Hq][d]                 16-byte aligned
 *     page_table        int32 [B][max_pages]  logical page -> physical block
 *     seq_lens          int32 [B]             tokens per sequence (<= max_pages*P;
 *                                             longer: ENTMAXKV_STATUS_BAD_LENGTH)
 *   Query head h reads kv head h / G, G = Hq / Hkv.  Sequence b has
 *   N_b = ceil(seq_lens[b] / P) pages; page p holds min(P, seq_lens[b] - p*P)
 *   valid tokens.  Scores are s = q.k / sqrt(d); entmax uses z = (alpha-1) s
 *   and p = [z - tau]_+^(1/(alpha-1)) with tau such that sum p = 1.
 * - Supported: d in {64, 128}; P in {16, 32, 64}; G in {1, 2, 4, 8};
 *   max_pages * P < 2^31; max_pages <= 196608 for entmaxkv_select and
 *   entmaxkv_decode_sparse.
 */
#ifndef ENTMAXKV_H
#define ENTMAXKV_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ENTMAXKV_API __attribute__((visibility("default")))
#else
#define ENTMAXKV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct entmaxkv_shape {
    int32_t B;          /* sequences in the batch */
    int32_t Hq;         /* query heads per sequence */
    int32_t Hkv;        /* key/value heads; Hq % Hkv == 0 */
    int32_t d;          /* head dimension */
    int32_t page_size;  /* P, tokens per page */
    int32_t max_pages;  /* row length of page_table (pages per sequence at most) */
    int32_t num_blocks; /* physical blocks held by k_cache / v_cache */
    /* kv-head range a call works on: kv heads [kv_begin, kv_begin + n) of
     * every sequence, and their query heads, with n = kv_count, or
     * Hkv - kv_begin when kv_count is 0 (a zero-filled struct means all
     * heads).  Every buffer keeps its full-size layout; entries of heads
     * outside the range are neither read nor written, so calls on disjoint
     * ranges may run concurrently, and may share one workspace. */
    int32_t kv_begin;
    int32_t kv_count;
} entmaxkv_shape;

enum {
    ENTMAXKV_OK = 0,
    ENTMAXKV_ERR_NULL = -1,        /* a required pointer is NULL */
    ENTMAXKV_ERR_SHAPE = -2,       /* shape field out of range or inconsistent */
    ENTMAXKV_ERR_ALPHA = -3,       /* alpha out of range for the call */
    ENTMAXKV_ERR_POLICY = -4,      /* unknown policy, k < 1, or Delta not finite */
    ENTMAXKV_ERR_WORKSPACE = -5,   /* workspace missing or smaller than required */
    ENTMAXKV_ERR_CUDA = -6,        /* CUDA runtime/driver error */
    ENTMAXKV_ERR_UNSUPPORTED = -7, /* valid but not implemented (e.g. non-integer r) */
    ENTMAXKV_ERR_ALIGN = -8,       /* pointer not 16-byte aligned */
    ENTMAXKV_ERR_TOO_LARGE = -9    /* problem needs more than the fixed scratch of
                                      entmaxkv_decode_sparse_static */
};

/* Size of the fixed on-device scratch used by entmaxkv_decode_sparse_static. */
#define ENTMAXKV_STATIC_SCRATCH_BYTES ((size_t)16 << 20)

enum { ENTMAXKV_TOPK = 0, ENTMAXKV_GAUSS = 1, ENTMAXKV_GAUSS_EST = 2 };

/* `call` argument of entmaxkv_workspace_size */
enum {
    ENTMAXKV_CALL_SELECT = 2,
    ENTMAXKV_CALL_DECODE_SPARSE = 3,
    ENTMAXKV_CALL_DECODE_DENSE = 4,
    ENTMAXKV_CALL_DECODE_STEP = 5
};

/* bits of the device status word */
enum {
    ENTMAXKV_STATUS_BAD_PAGE = 1,      /* page_table entry outside [0, num_blocks) */
    ENTMAXKV_STATUS_BAD_SELECTION = 2, /* sel entry outside [0, N_b) or cnt > N_b */
    ENTMAXKV_STATUS_TIMEOUT = 4,       /* an on-device wait hit its limit */
    ENTMAXKV_STATUS_OVERFLOW = 8,      /* a candidate list overflowed on-chip storage
                                          (handled by a slower exact path) */
    ENTMAXKV_STATUS_BAD_LENGTH = 16,   /* seq_lens[b] > max_pages * P: the sequence was
                                          treated as max_pages * P tokens long
                                          (entmaxkv_append skips it instead) */
    ENTMAXKV_STATUS_NONFINITE = 32     /* a query row held a NaN or an infinity: that
                                          head's scores and output are NaN */
};

/* Text for an ENTMAXKV_* return code. Static storage; never NULL. */
ENTMAXKV_API const char *entmaxkv_strerror(int code);

/* Library version as 10000*major + 100*minor + patch. */
ENTMAXKV_API int entmaxkv_version(void);

/*
 * Bytes of the metadata buffer written by entmaxkv_build_meta and read by
 * entmaxkv_score_pages: B * Hkv * n_tiles * 384 * d, n_tiles =
 * ceil(max_pages / 32).  Records are kept in logical page order, so a score
 * pass streams contiguous memory however the page table scatters the blocks.
 * Pages are grouped in tiles of 32 consecutive logical pages of one
 * (sequence b, kv head): tile T = (b * Hkv + kv_head) * n_tiles + p / 32,
 * page slot s = p % 32.  Coordinates are grouped in chunks of 16: chunk
 * c = j / 16, e = j % 16.
 *   bound region, bytes [0, NT*128d) with NT = B*Hkv*n_tiles:
 *     tile T at T*128d, chunk c at +2048c, kmin block at +0, kmax block at
 *     +1024; in a block, slot s holds its 16 bf16 values in two 16-byte
 *     halves h = e/8 stored at 32s + 16*(h ^ ((s>>2)&1)), element at +2(e%8).
 *   moment region, bytes [NT*128d, NT*384d):
 *     tile T at NT*128d + T*256d, chunk c at +4096c, mean block at +0, var
 *     block at +2048; in a block, slot s holds its 16 fp32 values in four
 *     16-byte quarters h = e/4 stored at 64s + 16*(h ^ ((s>>1)&3)),
 *     element at +4(e%4).
 * (The XOR places the pieces eight neighbouring pages read at one time on
 * distinct shared-memory banks once a chunk block is copied on chip.)
 * d must be a multiple of 16.  Returns 0 for an invalid shape.
 */
ENTMAXKV_API size_t entmaxkv_meta_bytes(const entmaxkv_shape *shape);

/*
 * Workspace bytes needed by `call` (ENTMAXKV_CALL_*) for this shape on the
 * current device; 0 means the call needs none.  Returns (size_t)-1 for an
 * invalid shape or call.  The caller allocates it (any device memory, 256-byte
 * aligned) and passes it with its size; contents need not be initialised and
 * are scratch after the call.  Calls that may overlap on the GPU need separate
 * workspaces, unless their kv-head ranges are disjoint.
 */
ENTMAXKV_API size_t entmaxkv_workspace_size(const entmaxkv_shape *shape, int call);

/*
 * Read the device status word of the current device into *status_out
 * (ENTMAXKV_STATUS_* bits) after synchronising `stream`; clear it when
 * `clear` != 0.  The word is shared by all calls on the device.
 */
ENTMAXKV_API int entmaxkv_get_status(int32_t *status_out, int clear, void *stream);

/*
 * Diagnostic with no counterpart in the EntmaxKV summary: launch one kernel
 * whose single thread waits on an mbarrier that nothing ever arrives at,
 * through the same bounded wait that every pipelined kernel of the library
 * uses, with the limit limit_ns (1 .. 2e9 nanoseconds of the GPU's global
 * timer, else ENTMAXKV_ERR_SHAPE).  When the limit passes the kernel sets
 * ENTMAXKV_STATUS_TIMEOUT and returns, so the stream and the context stay
 * usable: a caller can check that an on-device wait that runs out is
 * reported instead of hanging.  No copy is in flight during the wait.
 */
ENTMAXKV_API int entmaxkv_selftest_wait(uint64_t limit_ns, void *stream);

/*
 * Section 2.A (bounding box and Gaussian statistics, "maintained on append"):
 * for each sequence b, each logical page p in [first_page, first_page+n_pages)
 * with p < N_b (n_pages = -1: to the end), and each kv head, recompute the
 * metadata record of logical page p (its keys are in block page_table[b][p])
 * from its n = min(P, seq_len - pP) valid tokens, per coordinate j:
 *   kmin_j, kmax_j : the bf16 extreme (first token wins exact ties)
 *   mean_j = fp32(S1/n),  var_j = fp32(max(0, S2/n - (S1/n)^2))
 * with S1 = sum k_tj, S2 = sum k_tj^2 accumulated in fp64 in token order (the
 * result is defined to the bit).  Calling it on the page a new token was
 * appended to keeps the metadata current.  Records of pages outside the
 * range are not touched.
 */
ENTMAXKV_API int entmaxkv_build_meta(const entmaxkv_shape *shape, const void *k_cache,
                        const int32_t *page_table, const int32_t *seq_lens,
                        int32_t first_page, int32_t n_pages, void *meta,
                        void *stream);

/*
 * Section 2.A, the append step of decoding: each sequence b with
 * seq_lens[b] = L > 0 has just grown by one token, at position L-1.  For every
 * kv head, write that token's key row k_new[b][kvh][0..d) and value row
 * v_new[b][kvh][0..d) (bf16, device, [B][Hkv][d] contiguous) into slot
 * (L-1) mod P of block page_table[b][(L-1)/P] of k_cache / v_cache, then
 * rebuild the metadata record of logical page (L-1)/P exactly as
 * entmaxkv_build_meta does (same bits).  Sequences with L <= 0 are skipped.  A
 * page-table entry outside [0, num_blocks) sets ENTMAXKV_STATUS_BAD_PAGE, and
 * L > max_pages * P sets ENTMAXKV_STATUS_BAD_LENGTH; either skips that
 * sequence.  If q_in and q_out are
 * both given (bf16 [B][Hq][d]), the step's queries of the kv heads in range
 * are copied from q_in to q_out as well (one of them NULL without the other:
 * ENTMAXKV_ERR_NULL).  k_new, v_new and q_in may be pinned host memory
 * (cudaHostAlloc; unified addressing maps it into the device's address
 * space): the kernel then reads the step's inputs over the bus itself, so no
 * separate host-to-device copy is needed.  One kernel launch on `stream`; no
 * allocation.  k_cache, v_cache and meta must be 16-byte aligned
 * (ENTMAXKV_ERR_ALIGN).
 */
ENTMAXKV_API int entmaxkv_append(const entmaxkv_shape *shape, const void *k_new,
                    const void *v_new, const int32_t *page_table,
                    const int32_t *seq_lens, void *k_cache, void *v_cache,
                    void *meta, const void *q_in, void *q_out, void *stream);

/*
 * Section 2.A (query-aware page scoring): for every (b, h) and page p < N_b,
 *   bbox[b][h][p]  = fp32( (sum_j max(q_j kmin_j, q_j kmax_j)) / sqrt(d) )
 *   mu[b][h][p]    = fp32( (sum_j q_j mean_j) / sqrt(d) )
 *   sigma[b][h][p] = fp32( sqrt( (sum_j q_j^2 var_j) / d ) )
 * bbox bounds every token score s of the page from above.  Its sum runs in
 * fp64 over j in index order (every product is exact there) and is rounded
 * once, so the bound is defined to the bit.  mu and sigma feed only the
 * approximate threshold tau_hat of the Gaussian policies; their sums are
 * fp32, accurate to the forward error bound of a d-term fp32 dot product
 * (|error| <= 2 d 2^-24 sum_j |term_j|, plus the final rounding), not to the
 * bit.  Outputs are fp32 [B][Hq][max_pages]; entries for p >= N_b are not
 * written.  mu and sigma may both be NULL (bound only, reads 4d bytes per
 * page and kv head instead of 12d); if one is non-NULL both must be.  The
 * metadata is addressed by logical page, so no page table is needed; pages
 * whose keys are not all finite have unspecified scores.
 */
ENTMAXKV_API int entmaxkv_score_pages(const entmaxkv_shape *shape, const void *q,
                         const void *meta, const int32_t *seq_lens, float *bbox,
                         float *mu, float *sigma, void *stream);

/*
 * Section 2.B (candidate selection), per (b, h), written to
 * sel[b][h][0..cnt[b][h]) in ascending page order:
 *  ENTMAXKV_TOPK:  the k pages of largest bbox (k clipped to N_b; ties go to
 *                  the lower page index).  mu, sigma, delta, tau_hat unused.
 *  ENTMAXKV_GAUSS: tau_hat solves the approximate normalisation equation
 *                    sum_p n_p E[(X_p - tau)_+^r] = 1,
 *                    X_p ~ N((alpha-1) mu_p, (alpha-1)^2 sigma_p^2),
 *                    r = 1/(alpha-1) (must be an integer 1..8, else
 *                    ENTMAXKV_ERR_UNSUPPORTED),
 *                  and the pages kept are those with (alpha-1) bbox_p >
 *                  tau_hat - delta (the bound is the estimated max score).
 *                  tau_hat (nullable, fp32 [B][Hq]) receives the solution.
 *  ENTMAXKV_GAUSS_EST: as ENTMAXKV_GAUSS, but the estimated max score of a
 *                  page comes from its Gaussian model, capped by the bound:
 *                  keep p if (alpha-1) min(bbox_p, mu_p + z(n_p) sigma_p) >
 *                  tau_hat - delta, z(n) = sqrt(2 ln n) (z(1) = 0).  Keeps a
 *                  subset of ENTMAXKV_GAUSS's pages; unlike it, it can drop a
 *                  page holding a support token.
 * sel is int32 [B][Hq][max_pages], cnt int32 [B][Hq].  Needs alpha > 1 for
 * the Gaussian policies.  Non-finite scores (a non-finite query): top-k ranks
 * NaN above every number (ties to the lower page index); the Gaussian
 * policies keep no page when tau_hat is NaN.  workspace may be NULL when entmaxkv_workspace_size
 * reports 0.
 */
ENTMAXKV_API int entmaxkv_select(const entmaxkv_shape *shape, const int32_t *seq_lens,
                    const float *bbox, const float *mu, const float *sigma,
                    int32_t policy, int32_t k, float alpha, float delta,
                    int32_t *sel, int32_t *cnt, float *tau_hat,
                    void *workspace, size_t ws_bytes, void *stream);

/*
 * Section 2.C (sparse entmax attention): for each (b, h), over the tokens T of
 * the pages sel[b][h][0..cnt[b][h]) (ascending, as written by
 * entmaxkv_select), compute s_t, z_t = (alpha-1) s_t, the exact threshold
 * tau with sum_{t in T} [z_t - tau]_+^(1/(alpha-1)) = 1, p_t and
 *   out[b][h] = sum_t p_t v_t      (fp32 [B][Hq][d]).
 * If T contains the full-cache support, out equals the full-cache result.
 * Each page selected by any head of a GQA group is read once for the whole
 * group; value rows whose weight is zero for every head of the group are not
 * read.  tau_out (nullable) fp32 [B][Hq].  p_out (nullable, for checking)
 * fp32 [B][Hq][max_pages*P] in logical token order: for every selected page,
 * p of its valid tokens is written (0 off the support); other entries are
 * left untouched.  A head with no selected page gets out = 0 and tau = NaN.
 * out may be pinned host memory (allocated with cudaHostAlloc, which unified
 * addressing maps into the device's address space): the kernels then write
 * the result straight to the host, so no separate device-to-host copy is
 * needed after the call.
 * alpha == 1 gives softmax over the same tokens T (for comparing entmax and
 * softmax at one kept set): out = sum_T softmax(s)_t v_t, every selected
 * token carries weight, so K and V of the group's selected pages are read;
 * tau_out receives log sum_T exp(s_t); p_out must be NULL.
 */
ENTMAXKV_API int entmaxkv_decode_sparse(const entmaxkv_shape *shape, const void *q,
                           const void *k_cache, const void *v_cache,
                           const int32_t *page_table, const int32_t *seq_lens,
                           const int32_t *sel, const int32_t *cnt, float alpha,
                           float *out, float *tau_out, float *p_out,
                           void *workspace, size_t ws_bytes, void *stream);

/*
 * The number of kernels one entmaxkv_decode_sparse call with this shape and
 * alpha launches on the current device (2 or 3: the union of each GQA group's
 * selections is built by its own kernel, or inside the q.K kernel when that
 * kernel has at most two CTAs per group), for callers that count launches or
 * size CUDA graphs.  Negative ENTMAXKV_ERR_* on a bad shape or alpha < 1.
 * Launches nothing.
 */
ENTMAXKV_API int entmaxkv_decode_sparse_kernels(const entmaxkv_shape *shape, float alpha);

/*
 * One sparse decode step in one call: sections 2.A, 2.B and 2.C of the
 * summary in sequence -- page scores (as entmaxkv_score_pages), selection (as
 * entmaxkv_select) and sparse entmax attention over the selected pages (as
 * entmaxkv_decode_sparse) -- with the same arguments, outputs and errors as
 * those three calls made one after the other, and bit-identical results.
 * What differs is the work between them: the selection kernel also prepares
 * each GQA group's union of selected pages -- it marks its kept pages in a
 * per-group page map in the workspace, which one small kernel per group then
 * compacts (one read of the map, no pass over the selection lists); with one
 * query head per group the selection list is the union and is written as
 * such, with its physical blocks.  The step is five kernels (scoring,
 * selection, union, q.K, tau with p.V), four with one query head per group;
 * entmaxkv_decode_step_kernels gives the count.  Rows of more than 16384
 * pages fall back to the separate union pass of entmaxkv_decode_sparse.
 * - alpha must be > 1 (entmax; ENTMAXKV_ERR_ALPHA otherwise).  mu and sigma
 *   are required by the Gaussian policies; with top-k they may both be NULL
 *   (the bound alone is scored).
 * - workspace: entmaxkv_workspace_size(shape, ENTMAXKV_CALL_DECODE_STEP)
 *   bytes, 256-byte aligned; its contents need no initialisation (the scoring
 *   kernel clears the page-map rows of the call's groups every call).  As
 *   with every call, calls on disjoint kv-head ranges may share it and run
 *   concurrently.
 * - bbox/mu/sigma, sel/cnt/tau_hat, out/tau_out/p_out: as in the three calls.
 */
ENTMAXKV_API int entmaxkv_decode_step(const entmaxkv_shape *shape, const void *q, const void *meta,
                         const void *k_cache, const void *v_cache,
                         const int32_t *page_table, const int32_t *seq_lens,
                         int32_t policy, int32_t k, float alpha, float delta,
                         float *bbox, float *mu, float *sigma,
                         int32_t *sel, int32_t *cnt, float *tau_hat,
                         float *out, float *tau_out, float *p_out,
                         void *workspace, size_t ws_bytes, void *stream);

/*
 * The number of kernels one entmaxkv_decode_step call with this shape, policy
 * and alpha launches (5, 4 with one query head per group, more for rows of
 * more than 16384 pages).  Negative
 * ENTMAXKV_ERR_* on a bad shape, policy or alpha.  Launches nothing.
 */
ENTMAXKV_API int entmaxkv_decode_step_kernels(const entmaxkv_shape *shape, int32_t policy, float alpha);

/*
 * Allocation-free form of entmaxkv_decode_sparse (the EntmaxKV summary has no
 * counterpart; this is a library convenience).  Same arguments, results and
 * errors, minus the workspace: the scratch lives in a fixed array of
 * ENTMAXKV_STATIC_SCRATCH_BYTES (16 MiB) of device memory that the library
 * declares at file scope, so every GPU that loads the library holds it until
 * the process exits.  Meant for callers that cannot call cudaMalloc at decode
 * time -- for instance code that runs inside a memory pool or graph-building
 * framework that forbids allocation, or an embedding host whose allocator
 * owns all device memory.  The call itself allocates nothing.
 * - Problems whose entmaxkv_workspace_size(.., ENTMAXKV_CALL_DECODE_SPARSE)
 *   exceeds ENTMAXKV_STATIC_SCRATCH_BYTES return ENTMAXKV_ERR_TOO_LARGE (about
 *   four million (query head, context token) pairs fit).
 * - The first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call
 *   before any stream capture.
 * - All calls on a device share the one array, which keeps the last call's
 *   contents (every kernel initialises what it reads, so nothing needs to be
 *   cleared between calls).  Calls that may overlap on the GPU -- different
 *   streams without ordering, or two host threads -- race on it; serialise
 *   them.
 */
ENTMAXKV_API int entmaxkv_decode_sparse_static(const entmaxkv_shape *shape, const void *q,
                                  const void *k_cache, const void *v_cache,
                                  const int32_t *page_table, const int32_t *seq_lens,
                                  const int32_t *sel, const int32_t *cnt, float alpha,
                                  float *out, float *tau_out, float *p_out,
                                  void *stream);

/*
 * Sequence-sharded sparse decode: one context split across S devices, each
 * holding a consecutive range of its logical pages (the summary's section 2.C
 * computation, done in pieces with three small exchanges).  Shard r holds
 * global pages [page_begin, page_begin + max_pages) in its own paged cache,
 * page table and seq_lens (its tokens only); sel/cnt are the GLOBAL selection
 * (every shard runs entmaxkv_select on the all-gathered page scores, so all
 * hold the same lists, rows of sel_max_pages global page ids).  Per step:
 *   1. entmaxkv_decode_sparse_begin       this shard's pages of sel: union,
 *      z of their tokens (kept in the workspace) and the shard's max z per
 *      head, zmax_out fp32 [B][Hq] (-inf if the shard has none);
 *   2. the caller all-reduces zmax with max;
 *   3. entmaxkv_decode_sparse_candidates  the shard's tokens with
 *      z > zmax_in - 1 (every token that can carry weight), in list order:
 *      cand_z fp32 [B][Hq][cap], cand_n int32 [B][Hq] (the exact count; if it
 *      exceeds cap only cap values are written and ENTMAXKV_STATUS_OVERFLOW is
 *      set: call again with a larger cap);
 *   4. the caller all-gathers cand_z / cand_n into [S][B][Hq][cap] / [S][B][Hq]
 *      (shards in page order);
 *   5. entmaxkv_entmax_threshold          the exact tau of each head from all
 *      shards' candidates (the same Newton solve as entmaxkv_decode_sparse, on
 *      the same list in the same order, so the same tau), tau_out fp32 [B][Hq];
 *   6. entmaxkv_decode_sparse_finish      out[b][h] = sum over the shard's
 *      support of p_t v_t (a partial sum: entmax weights are absolute, so the
 *      shards' partials add up to the output);
 *   7. the caller all-reduces out with sum.
 * The workspace carries state from step 1 to step 6 (one workspace per shard
 * and step in flight).  alpha must be > 1.  n_shards * cap * 4 bytes must fit
 * in 200 KiB (ENTMAXKV_ERR_SHAPE).  kv-head ranges apply as in every call.
 */
ENTMAXKV_API int entmaxkv_decode_sparse_begin(const entmaxkv_shape *shape, const void *q,
                    const void *k_cache, const void *v_cache, const int32_t *page_table,
                    const int32_t *seq_lens, const int32_t *sel, const int32_t *cnt,
                    int32_t sel_max_pages, int32_t page_begin, float alpha,
                    float *zmax_out, void *workspace, size_t ws_bytes, void *stream);
ENTMAXKV_API int entmaxkv_decode_sparse_candidates(const entmaxkv_shape *shape, const void *q,
                    const void *k_cache, const void *v_cache, const int32_t *page_table,
                    const int32_t *seq_lens, float alpha, const float *zmax_in, int32_t cap,
                    float *cand_z, int32_t *cand_n, void *workspace, size_t ws_bytes,
                    void *stream);
ENTMAXKV_API int entmaxkv_entmax_threshold(const entmaxkv_shape *shape, int32_t n_shards,
                    int32_t cap, const float *cand_z, const int32_t *cand_n,
                    const float *zmax_in, float alpha, float *tau_out, void *stream);
ENTMAXKV_API int entmaxkv_decode_sparse_finish(const entmaxkv_shape *shape, const void *q,
                    const void *k_cache, const void *v_cache, const int32_t *page_table,
                    const int32_t *seq_lens, float alpha, const float *zmax_in,
                    const float *tau_in, float *out, float *p_out, void *workspace,
                    size_t ws_bytes, void *stream);

/*
 * Section 4 comparison paths, over every token of every sequence:
 *  alpha > 1:  full-cache alpha-entmax (all of K and all of V are read):
 *              out = sum_t p_t v_t; tau_out (nullable) gets tau.
 *  alpha == 1: full-cache softmax, split over pages with a combine step:
 *              out = sum_t softmax(s)_t v_t; tau_out (nullable) gets the
 *              log-sum-exp log sum_t exp(s_t).
 * out fp32 [B][Hq][d].  p_out as in entmaxkv_decode_sparse (alpha > 1 only;
 * must be NULL for alpha == 1).
 */
ENTMAXKV_API int entmaxkv_decode_dense(const entmaxkv_shape *shape, const void *q,
                          const void *k_cache, const void *v_cache,
                          const int32_t *page_table, const int32_t *seq_lens,
                          float alpha, float *out, float *tau_out, float *p_out,
                          void *workspace, size_t ws_bytes, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* ENTMAXKV_H */
