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

}  // namespace ekv
