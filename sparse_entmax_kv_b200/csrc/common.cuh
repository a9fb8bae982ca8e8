// common.cuh -- device helpers shared by the EntmaxKV kernels (sm_100a).
//
// PTX wrappers for mbarriers, 1-D bulk copies and 2-D tiled TMA loads (no
// cluster multicast anywhere), warp-level mma.sync for the bf16 q.K^T tiles,
// bf16 unpacking and the order-preserving float <-> int32 map used for
// atomic max.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "../../include/entmaxkv.h"

namespace ekv {

constexpr unsigned FULL = 0xffffffffu;
// Longest an mbarrier wait may spin before it reports ENTMAXKV_STATUS_TIMEOUT
// and gives up (nanoseconds of %globaltimer).
constexpr unsigned long long WAIT_LIMIT_NS = 2000000000ull;

__device__ __forceinline__ unsigned smem_u32(const void *p) {
    return static_cast<unsigned>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long globaltimer() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// ------------------------------------------------------------- mbarrier

__device__ __forceinline__ void mbar_init(uint64_t *bar, unsigned count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void mbar_fence_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, unsigned bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// One potentially blocking probe: the thread is suspended until the phase
// completes or a hardware time limit passes (so a waiting warp does not take
// issue slots from the warps that compute).
__device__ __forceinline__ bool mbar_try(uint64_t *bar, unsigned parity) {
    unsigned ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait for the phase with the given parity.  Returns false (and sets
// the TIMEOUT status bit) if it did not complete within limit_ns nanoseconds
// of %globaltimer (or 2^30 probes, whichever comes first).
__device__ __forceinline__ bool mbar_wait_for(uint64_t *bar, unsigned parity, int *status,
                                              unsigned long long limit_ns) {
    if (mbar_try(bar, parity)) return true;
    const unsigned long long t0 = globaltimer();
    for (unsigned it = 0; it < (1u << 30); ++it) {
        if (mbar_try(bar, parity)) return true;
        if (globaltimer() - t0 > limit_ns) break;
    }
    if (status) atomicOr(status, ENTMAXKV_STATUS_TIMEOUT);
    return false;
}

// The kernels' waits: bounded by WAIT_LIMIT_NS.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, unsigned parity, int *status) {
    return mbar_wait_for(bar, parity, status, WAIT_LIMIT_NS);
}

// -------------------------------------------------------- bulk / TMA copies

// 1-D bulk copy global -> shared, completion counted on `bar` (bytes).
// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, unsigned bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// 2-D tiled TMA load of one box at element coordinates (x, y) (x = innermost).
// x * sizeof(element) must be a multiple of 16 bytes.
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Ampere-style 16-byte async copy (bypasses L1), grouped with commit/wait.
// Ask for the 128-byte lines of one row of D bf16 values to be brought into L2.
template <int D>
__device__ __forceinline__ void prefetch_l2_row(const uint16_t *row) {
#pragma unroll
    for (int o = 0; o < D * 2; o += 128) asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<const char *>(row) + o));
}

__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ------------------------------------------------ programmatic dependent launch
//
// Every kernel of the library is launched with programmatic stream
// serialisation and starts with pdl_wait(), which blocks until the previous
// kernel of the stream has completed and its writes are visible.  The launch
// of a kernel is thereby processed while its predecessor still runs.  No
// kernel triggers its dependants early: CTAs of the next kernel parked on
// the SMs slowed the running one down.  Because every CTA waits before doing
// anything else, a kernel completes only after its predecessor, so completion
// stays ordered along the stream.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<Args &&>(args)...);
}

// ------------------------------------------------------- thread-block clusters

__device__ __forceinline__ unsigned cl_rank() {
    unsigned r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// Barrier over every thread of every CTA of the cluster; shared-memory
// writes (local or pushed into a peer) before it are visible after it.
__device__ __forceinline__ void cl_sync() {
    __syncwarp();
    asm volatile(
        "barrier.cluster.arrive.release.aligned;\n\t"
        "barrier.cluster.wait.acquire.aligned;" ::
            : "memory");
}
// Address of `p` (a shared variable of this CTA) in the CTA of rank `rank`.
__device__ __forceinline__ unsigned cl_map(const void *p, unsigned rank) {
    unsigned r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
    return r;
}
// Stores into a peer CTA's shared memory (visible there after the next
// cluster barrier).  Exchanges push data to the CTAs that read it, so every
// read after a barrier is local.
__device__ __forceinline__ void cl_stf(unsigned addr, float v) {
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}
__device__ __forceinline__ void cl_sti(unsigned addr, int v) {
    asm volatile("st.shared::cluster.s32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// ------------------------------------------------------------ tensor cores

// ldmatrix x4 (four 8x8 b16 matrices), one row address per lane.
__device__ __forceinline__ void ldsm_x4(unsigned addr, unsigned &r0, unsigned &r1, unsigned &r2, unsigned &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

// The same with each 8x8 matrix transposed on the way into registers.
__device__ __forceinline__ void ldsm_x4_t(unsigned addr, unsigned &r0, unsigned &r1, unsigned &r2, unsigned &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

// D = A(16x16 bf16, row) * B(16x8 bf16, col) + C, fp32 accumulate.
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], unsigned a0, unsigned a1, unsigned a2, unsigned a3,
                                               unsigned b0, unsigned b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// --------------------------------------------------------------- numbers

__device__ __forceinline__ float bf16lo(unsigned w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(unsigned w) { return __uint_as_float(w & 0xffff0000u); }
__device__ __forceinline__ float bf16f(uint16_t h) { return __uint_as_float(((unsigned)h) << 16); }
// float -> bf16, round to nearest even.
__device__ __forceinline__ uint16_t f2bf(float x) {
    uint16_t r;
    asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(r) : "f"(x));
    return r;
}

// Order-preserving map float -> int32 (for atomicMax) and back.
__device__ __forceinline__ int f2ord(float f) {
    int i = __float_as_int(f);
    return i >= 0 ? i : i ^ 0x7fffffff;
}
__device__ __forceinline__ float ord2f(int i) { return __int_as_float(i >= 0 ? i : i ^ 0x7fffffff); }
constexpr int ORD_NEG_INF = (int)(0xff800000u ^ 0x7fffffffu);  // f2ord(-inf)

__host__ __device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

__device__ __forceinline__ int n_pages_of(int seq_len, int P) { return seq_len > 0 ? (seq_len + P - 1) / P : 0; }

// Tokens of sequence b as every kernel uses them: seq_lens[b] clamped to
// [0, max_pages * P].  A longer length is a caller error the host cannot see
// (the lengths live on the device); thread 0 of each CTA that meets one sets
// ENTMAXKV_STATUS_BAD_LENGTH, and the sequence is treated as max_pages * P
// tokens long, so no kernel indexes past a row of max_pages pages.
__device__ __forceinline__ int seq_len_of(const int *seq_lens, int b, int P, int max_pages, int *status) {
    const int s = seq_lens[b];
    const int cap = max_pages * P;
    if (s > cap) {
        if (threadIdx.x == 0 && status) atomicOr(status, ENTMAXKV_STATUS_BAD_LENGTH);
        return cap;
    }
    return s < 0 ? 0 : s;
}

// True when every bf16 value of the d-element query row is finite (a bf16 is
// NaN or +-Inf exactly when its eight exponent bits are all ones).
__device__ __forceinline__ bool q_row_finite(const uint16_t *q, int d) {
    bool ok = true;
    for (int j = 0; j < d; ++j) ok &= (q[j] & 0x7f80u) != 0x7f80u;
    return ok;
}

__device__ __forceinline__ int tokens_in_page(int seq_len, int P, int p) {
    int n = seq_len - p * P;
    return n > P ? P : (n < 0 ? 0 : n);
}

// [x]_+^r.  ri = r when r is an integer in 1..8 (repeated products), ri = 0
// for any other exponent (powf).
__device__ __forceinline__ float pos_pow(float x, float r, int ri) {
    if (!(x > 0.f)) return 0.f;
    switch (ri) {
        case 1: return x;
        case 2: return x * x;
        case 3: return x * x * x;
        case 4: { float y = x * x; return y * y; }
        case 5: { float y = x * x; return y * y * x; }
        case 6: { float y = x * x * x; return y * y; }
        case 7: { float y = x * x * x; return y * y * x; }
        case 8: { float y = x * x; y = y * y; return y * y; }
        default: return powf(x, r);
    }
}

// Block-wide exclusive scan of one int per thread, in thread order.  `sh`
// needs 65 ints of shared memory; *total receives the block total.
__device__ __forceinline__ int block_excl_scan(int v, int *sh, int *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(FULL, x, o);
        if (lane >= o) x += y;
    }
    __syncthreads();
    if (lane == 31) sh[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = lane < nw ? sh[lane] : 0;
        int ws = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(FULL, ws, o);
            if (lane >= o) ws += y;
        }
        if (lane < nw) sh[32 + lane] = ws - w;
        if (lane == nw - 1) sh[64] = ws;
    }
    __syncthreads();
    *total = sh[64];
    return sh[32 + warp] + x - v;
}


// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) once per (kernel, device,
// size): the setting persists, and repeating the driver call on every launch
// costs host time on the decode path.
inline cudaError_t ensure_smem(const void *func, size_t bytes) {
    struct Entry {
        const void *f;
        int dev;
        size_t bytes;
    };
    static std::mutex mu;
    static Entry cache[256];
    static int n = 0;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lk(mu);
    for (int i = 0; i < n; ++i)
        if (cache[i].f == func && cache[i].dev == dev && cache[i].bytes >= bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess && n < 256) cache[n++] = Entry{func, dev, bytes};
    return e;
}

}  // namespace ekv
