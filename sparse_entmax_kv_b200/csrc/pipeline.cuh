// pipeline.cuh -- pieces shared by the decode kernels: the per-page record a
// producer warp publishes for each ring stage, the stage ring of TMA page
// tiles (K and/or V of a few pages per stage, 128-byte swizzled boxes, full and
// empty mbarriers), and row addressing of the per-head z buffers.
#pragma once

#include "common.cuh"
#include "internal.h"

namespace ekv {

constexpr int NWC = 4;                       // consumer warps
constexpr int DEC_THREADS = (NWC + 1) * 32;  // + one producer warp
constexpr int PPS_MAX = 8;

template <int G>
struct Tile {
    static constexpr int TPS = G == 1 ? 128 : 64;  // tokens per pipeline stage
};

struct PageInfo {
    int page;  // logical page (-1: none)
    int mask;  // heads of the group that use it
    int nval;  // valid tokens (0 if the page could not be loaded)
    int upos;  // position in the union (page index on the dense paths)
    int blk;   // physical block (-1: none)
};

__device__ __forceinline__ size_t tok_row(const DecodeArgs &a, int b, int h) {
    return ((size_t)b * a.Hq + h) * (size_t)a.max_pages * a.P;
}
__device__ __forceinline__ size_t tile_row(const DecodeArgs &a, int b, int h) {
    return ((size_t)b * a.Hq + h) * (size_t)a.max_pages * a.P / 16;
}

template <int D, int G, int NS, int NMAP>
struct Ring {
    static constexpr int TPS = Tile<G>::TPS;
    static constexpr int STAGE = TPS * D * 2 * NMAP;  // bytes per stage (K and/or V)
    static constexpr size_t BYTES = 1024 + (size_t)NS * STAGE + 2 * NS * 8 + NS * PPS_MAX * sizeof(PageInfo) +
                                    32 * PPS_MAX * sizeof(PageInfo);
};

template <int D, int G, int NS, int NMAP>
struct RingView {
    unsigned char *stages;
    uint64_t *full, *empty;
    PageInfo *pinfo;  // [NS][PPS_MAX]
    PageInfo *stash;  // [32 * PPS_MAX], producer scratch
    __device__ RingView(unsigned char *raw) {
        using RG = Ring<D, G, NS, NMAP>;
        stages = reinterpret_cast<unsigned char *>(((uintptr_t)raw + 1023) & ~(uintptr_t)1023);
        full = reinterpret_cast<uint64_t *>(stages + (size_t)NS * RG::STAGE);
        empty = full + NS;
        pinfo = reinterpret_cast<PageInfo *>(empty + NS);
        stash = pinfo + NS * PPS_MAX;
    }
};

// Address of the 16-byte chunk `c16` (8 bf16) of row r in a swizzled page tile.
__device__ __forceinline__ const unsigned char *tile_chunk(const unsigned char *page_base, int P, int r, int c16) {
    const int box = c16 >> 3, cc = c16 & 7;
    return page_base + box * P * 128 + r * 128 + ((cc ^ (r & 7)) << 4);
}

// P.V on the tensor cores for one 16-token step of one warp.
//   acc[mt] (m16n8 fragment): rows = value coordinates 16 mt .. 16 mt + 15,
//   columns = the group's heads (lane holds heads 2 (lane % 4) and + 1).
// A = V^T of rows r0 .. r0 + 15 of a swizzled page tile, read with transposing
// ldmatrix; B = P^T of those tokens as bf16 hi and lo parts (p = hi + lo to
// about 2^-17 relative), two MMAs per tile.  Value halves of tokens at or past
// nval are zeroed (those rows of the tile may hold anything, and 0 * NaN is
// NaN).
template <int D>
__device__ __forceinline__ void pv_mma(float (&acc)[D / 16][4], const unsigned char *vpage, int P, int r0, int nval,
                                       unsigned bh0, unsigned bh1, unsigned bl0, unsigned bl1) {
    const int lane = threadIdx.x & 31;
    const int row = r0 + ((lane >> 4) << 3) + (lane & 7);
    const int csel = (lane >> 3) & 1;
    unsigned m01 = 0xffffffffu, m23 = 0xffffffffu;
    if (r0 + 16 > nval) {
        const int t = r0 + 2 * (lane & 3);
        m01 = (t < nval ? 0x0000ffffu : 0u) | (t + 1 < nval ? 0xffff0000u : 0u);
        m23 = (t + 8 < nval ? 0x0000ffffu : 0u) | (t + 9 < nval ? 0xffff0000u : 0u);
    }
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) {
        unsigned a0, a1, a2, a3;
        ldsm_x4_t(smem_u32(tile_chunk(vpage, P, row, 2 * mt + csel)), a0, a1, a2, a3);
        a0 &= m01;
        a1 &= m01;
        a2 &= m23;
        a3 &= m23;
        mma_bf16_16816(acc[mt], a0, a1, a2, a3, bh0, bh1);
        mma_bf16_16816(acc[mt], a0, a1, a2, a3, bl0, bl1);
    }
}

// p0, p1 (two consecutive tokens of one head) as the hi and lo bf16 pairs of
// a B fragment register (first token in the low half).
__device__ __forceinline__ void split_pair(float p0, float p1, unsigned &hi, unsigned &lo) {
    const uint16_t h0 = f2bf(p0), h1 = f2bf(p1);
    const uint16_t l0 = f2bf(p0 - bf16f(h0)), l1 = f2bf(p1 - bf16f(h1));
    hi = (unsigned)h0 | ((unsigned)h1 << 16);
    lo = (unsigned)l0 | ((unsigned)l1 << 16);
}

}  // namespace ekv
