// internal.h -- host-side launch interface between the C ABI (api.cu) and the
// kernel translation units.  Not part of the public header.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace ekv {

// Most split-K slots a decode call may use per (sequence, head).
constexpr int MAX_SPLITS = 64;

struct DevInfo {
    int sms;
    int *status;  // device address of the status word
};

// Grid index -> (sequence, kv head) of a kv-head range [kv0, kv0 + nk), and
// -> (sequence, query head) of a query-head range [h0, h0 + nh).
__host__ __device__ inline void group_of(int idx, int kv0, int nk, int &b, int &kvh) {
    b = idx / nk;
    kvh = kv0 + idx % nk;
}
__host__ __device__ inline void head_of(int idx, int h0, int nh, int &b, int &h) {
    b = idx / nh;
    h = h0 + idx % nh;
}

// Pages per metadata tile and the tile count of one (sequence, kv head).
constexpr int META_TILE = 32;
inline int meta_tiles(int max_pages) { return (max_pages + META_TILE - 1) / META_TILE; }

struct MetaArgs {
    const uint16_t *k;
    const int *page_table;
    const int *seq_lens;
    uint8_t *meta;
    int n_tiles;              // tiles per (sequence, kv head)
    long long n_tiles_total;  // B * Hkv * n_tiles
    int B, Hkv, d, P, max_pages, num_blocks;
    int first_page, n_pages;  // n_pages >= 0 here (resolved by the caller)
    int kv0, nk;              // kv-head range [kv0, kv0 + nk)
    int *status;
};
cudaError_t launch_build_meta(const MetaArgs &a, cudaStream_t st);

// One new token per sequence: its k/v rows go to slot seq_len-1 and the
// metadata record of its page is rebuilt (the MetaArgs fields first_page and
// n_pages are unused).
struct AppendArgs {
    MetaArgs m;
    uint16_t *k_cache, *v_cache;
    const uint16_t *k_new, *v_new;  // [B][Hkv][d]
    const uint16_t *q_in;           // [B][Hq][d] or null: copied to q_out
    uint16_t *q_out;
    int Hq;
};
cudaError_t launch_append(const AppendArgs &a, cudaStream_t st);

struct ScoreArgs {
    const uint16_t *q;
    const uint8_t *meta;
    const int *seq_lens;
    float *bbox, *mu, *sigma;
    int n_tiles;
    long long n_tiles_total;
    int B, Hq, Hkv, d, P, max_pages;
    int kv0, nk;  // kv-head range [kv0, kv0 + nk)
    int *status;
    // decode step: the rows of umap (uwords words each, a multiple of 4) of
    // the call's groups are cleared for the selection of the same step
    unsigned *umap;
    int uwords;
};
cudaError_t launch_score_pages(const ScoreArgs &a, cudaStream_t st);

struct SelectArgs {
    const int *seq_lens;
    const float *bbox, *mu, *sigma;
    int *sel, *cnt;
    float *tau_hat;
    int B, Hq, P, max_pages;
    int policy, k;
    float alpha, delta;
    int r_int;  // 1/(alpha-1) for the Gaussian policy
    int h0, nh;  // query-head range [h0, h0 + nh)
    int sms;     // SMs of the device (grid shape choice)
    int *status;
    // decode step (umap non-null): the union of each group's selections for
    // the q.K pass.  G > 1: each CTA ORs the head bit of every page it keeps
    // into that page's byte of the group's row of umap (zero on entry, uwords
    // words a row), which the decode's union_map_kernel compacts.  G = 1: the
    // selection list is written as the union (union_e / union_blk / union_cnt,
    // the decode workspace's layout, with page_table looked up) and zmax is
    // reset.
    unsigned *umap;
    int uwords;
    int *union_e, *union_blk, *union_cnt, *zmax;
    const int *page_table;
    int Hkv, num_blocks;
};
cudaError_t launch_select(const SelectArgs &a, cudaStream_t st);
bool select_marks_union(const SelectArgs &a);  // whether launch_select can prepare the union for this shape

// Workspace carve-up shared by the decode paths.
struct DecodeWs {
    int *union_e;    // [B*Hkv][max_pages]   (page << 8) | head mask (sparse)
    int *union_blk;  // [B*Hkv][max_pages]   physical block of each union entry (sparse)
    int *union_cnt;  // [B*Hkv]
    int *zmax;       // [B*Hq] order-mapped max z (when union_kernel or the dense init resets it)
    float *tau;      // [B*Hq]
    int *counters;   // [B*Hkv] last-CTA combine counters
    float *partial;  // [MAX_SPLITS][B*Hq][d+2]  (dense paths)
    float *zbuf;     // [B*Hq][max_pages*P]  z of every token of the page list, in list order
    float *tmax;     // [B*Hq][max_pages*P/16]  max z of each 16-token tile of zbuf
    unsigned *umap;  // [B*Hkv][uwords]  decode step: head bits per page, a byte each (4 pages a word)
    int uwords;      // words per umap row: ceil(max_pages / 4) rounded up to a multiple of 4
};

struct DecodeArgs {
    const uint16_t *q;
    const uint16_t *k, *v;
    const int *page_table, *seq_lens;
    const int *sel, *cnt;  // sparse only
    float *out, *tau_out, *p_out;
    CUtensorMap kmap, vmap;  // 2-D maps over [num_blocks*Hkv*P rows][d] bf16
    DecodeWs ws;
    int B, Hq, Hkv, d, P, max_pages, num_blocks;
    float alpha;
    int r_int;  // 1/(alpha-1) if an integer 1..8, else 0
    int sms;
    int kv0, nk;  // kv-head range [kv0, kv0 + nk); query heads [kv0 G, (kv0 + nk) G)
    // sequence-sharded phases: sel rows of sel_stride global page ids, this
    // shard's page i being global page page_begin + i (entries of other shards
    // are skipped); the global max z / tau per head come in, the shard's max z
    // and candidate z values go out
    int sharded, page_begin, sel_stride;
    int union_in_qk;  // sparse q.K: each CTA builds the group's union itself (set by the launcher)
    const float *zmax_in, *tau_in;
    float *zmax_out;
    float *cand_z;
    int *cand_n;
    int cap;
    int *status;
};
cudaError_t launch_decode_sparse(const DecodeArgs &a, cudaStream_t st);
int decode_sparse_kernels(const DecodeArgs &a);  // launches of one launch_decode_sparse
cudaError_t launch_decode_sparse_begin(const DecodeArgs &a, cudaStream_t st);
cudaError_t launch_decode_sparse_candidates(const DecodeArgs &a, cudaStream_t st);
cudaError_t launch_decode_sparse_finish(const DecodeArgs &a, cudaStream_t st);
// The decode of a step whose selection marked the union (G > 1: union_map_kernel
// compacts the marks) or wrote it (G = 1): then q.K and tau with p.V
cudaError_t launch_decode_step_tail(const DecodeArgs &a, cudaStream_t st);
int decode_step_tail_kernels(const DecodeArgs &a);

struct ThresholdArgs {
    const float *cand_z;  // [S][B*Hq][cap]
    const int *cand_n;    // [S][B*Hq]
    const float *zmax;    // [B*Hq]
    float *tau;           // [B*Hq]
    int S, cap, B, Hq, Hkv, kv0, nk;
    float alpha;
    int r_int;
    int *status;
};
cudaError_t launch_entmax_threshold(const ThresholdArgs &a, cudaStream_t st);
cudaError_t launch_decode_dense_entmax(const DecodeArgs &a, cudaStream_t st);
cudaError_t launch_decode_dense_softmax(const DecodeArgs &a, cudaStream_t st);

// Workspace of a decode call; step adds the union marks of
// entmaxkv_decode_step (one row per group, each call clearing its groups' rows).
size_t decode_ws_bytes(bool dense, int B, int Hq, int Hkv, int d, int P, int max_pages, DecodeWs *carve,
                      void *base, bool step = false);

}  // namespace ekv
