// Token-to-expert bucketing for the forward pass.
//
// PagedWeight, "Dynamic Paging": the router decides which experts a pass
// needs; their pages serve all of their tokens at once. Assignment a = t*k + j
// (token t's j-th routed expert ids[a]):
//   perm    = the assignments ordered by expert id, stable in a;
//   offsets = exclusive prefix sums of the per-expert counts (E+1 entries);
//   inv[a]  = position of a in perm, -1 for ids outside [0, E) (dropped, with
//             MPE_STATUS_BAD_EXPERT_ID set);
// plus the decode work groups: each expert's tokens cut into runs of at most
// `group` positions, listed as (expert, first position, count).
//
// Stable ranks come from warp matching: inside a warp, lanes holding the same
// id rank by lane; across warps, by the per-warp counts of earlier warps;
// across 1024-assignment chunks, by the per-chunk histograms.
#include <cstdio>

#include "internal.h"

namespace mpe {
namespace {

constexpr int kChunk = 1024;

// offsets_and_groups packs the work-group counts of the three width classes
// into 21-bit fields of one 64-bit scan: a class holds at most
// MPE_MAX_ASSIGNMENTS / group + E groups (group >= kDecodeGroup), which must
// stay below 2^21. The entry points reject T*k above MPE_MAX_ASSIGNMENTS.
static_assert((long long)MPE_MAX_ASSIGNMENTS / kDecodeGroup + MPE_MAX_EXPERTS < (1ll << 21),
              "work-group counts overflow their 21-bit scan fields");

// Exclusive block scan of one uint64 per thread over 1024 threads.
__device__ uint64_t block_exclusive_scan(uint64_t v, uint64_t* s_warp, uint64_t* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint64_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint64_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) s_warp[warp] = x;
    __syncthreads();
    if (warp == 0) {
        uint64_t w = s_warp[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint64_t y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        s_warp[lane] = w;  // inclusive over warps
    }
    __syncthreads();
    const uint64_t before = (warp > 0 ? s_warp[warp - 1] : 0) + x - v;
    *total = s_warp[31];
    __syncthreads();
    return before;
}

// Offsets and work groups from per-expert counts (thread e holds count[e]).
// Work groups are listed by width class of their expert -- 8-bit, then 4-bit,
// then 3-bit -- so each decode loop runs one specialised code path;
// n_wg = {total, class 8, class 4, class 3}.
__device__ void offsets_and_groups(int E, int cnt, int group, const Pte* pte, int32_t* offsets,
                                   int32_t* wg, int32_t* n_wg, int32_t* s_off) {
    __shared__ uint64_t s_warp[32];
    const int e = threadIdx.x;
    const int c = (e < E) ? cnt : 0;
    uint64_t total;
    const int off = (int)block_exclusive_scan((uint64_t)c, s_warp, &total);
    const int n_assign = (int)total;
    int cls = -1;
    if (e < E) {
        const int b = pte[e].bits;
        cls = b == 8 ? 0 : (b == 4 ? 1 : (b == 3 ? 2 : -1));
    }
    const int ng = (cls >= 0) ? (c + group - 1) / group : 0;
    const uint64_t packed = cls < 0 ? 0ull : ((uint64_t)ng << (21 * cls));
    uint64_t gtot;
    const uint64_t gex = block_exclusive_scan(packed, s_warp, &gtot);
    const int t8 = (int)(gtot & 0x1FFFFF), t4 = (int)((gtot >> 21) & 0x1FFFFF),
              t3 = (int)((gtot >> 42) & 0x1FFFFF);
    if (e < E) {
        offsets[e] = off;
        s_off[e] = off;
        if (cls >= 0) {
            const int start = cls == 0 ? 0 : (cls == 1 ? t8 : t8 + t4);
            const int goff = start + (int)((gex >> (21 * cls)) & 0x1FFFFF);
            for (int i = 0; i < ng; ++i) {
                wg[3 * (goff + i) + 0] = e;
                wg[3 * (goff + i) + 1] = off + i * group;
                wg[3 * (goff + i) + 2] = min(group, c - i * group);
            }
        }
    }
    if (e == 0) {
        offsets[E] = n_assign;
        n_wg[0] = t8 + t4 + t3;
        n_wg[1] = t8;
        n_wg[2] = t4;
        n_wg[3] = t3;
    }
}

// Stable scatter of one chunk: base[e] = first position of this chunk's
// assignments with id e.
__device__ void scatter_chunk(const int32_t* ids, int a0, int n, int E, const int32_t* base,
                              uint16_t* wcnt, int32_t* perm, int32_t* inv, uint32_t* status) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int a = a0 + threadIdx.x;
    int e = -1;
    bool valid = false;
    if (threadIdx.x < n) {
        e = ids[a];
        valid = (e >= 0 && e < E);
        if (!valid) set_status(status, MPE_STATUS_BAD_EXPERT_ID);
    }
    const int key = valid ? e : -1;
    const unsigned peers = __match_any_sync(0xffffffffu, key);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    if (valid && rank == 0) wcnt[warp * E + e] = (uint16_t)__popc(peers);
    __syncthreads();
    if (valid) {
        int pre = 0;
        for (int w = 0; w < warp; ++w) pre += wcnt[w * E + e];
        const int pos = base[e] + pre + rank;
        perm[pos] = a;
        inv[a] = pos;
    } else if (threadIdx.x < n) {
        inv[a] = -1;
    }
}

// T*k <= 1024: everything in one CTA.
__global__ void __launch_bounds__(kChunk)
k_route_small(const int32_t* ids, int Tk, int E, int group, const Pte* pte, int32_t* perm,
              int32_t* offsets, int32_t* inv, int32_t* wg, int32_t* n_wg, uint32_t* status,
              int32_t* zero6) {
    // launched programmatically: the previous pass's kernels still read these
    // buffers until they finish
    griddep_wait();
    griddep_launch_dependents();
    if (threadIdx.x < 6 && zero6) zero6[threadIdx.x] = 0;
    extern __shared__ __align__(16) uint8_t sm[];
    int32_t* s_cnt = reinterpret_cast<int32_t*>(sm);       // [E]
    int32_t* s_off = s_cnt + MPE_MAX_EXPERTS;               // [E]
    uint16_t* wcnt = reinterpret_cast<uint16_t*>(s_off + MPE_MAX_EXPERTS);  // [32][E]
    for (int i = threadIdx.x; i < 32 * E; i += kChunk) wcnt[i] = 0;
    for (int i = threadIdx.x; i < E; i += kChunk) s_cnt[i] = 0;
    __syncthreads();
    if (threadIdx.x < Tk) {
        const int e = ids[threadIdx.x];
        if (e >= 0 && e < E) atomicAdd(&s_cnt[e], 1);
    }
    __syncthreads();
    const int cnt = threadIdx.x < E ? s_cnt[threadIdx.x] : 0;
    offsets_and_groups(E, cnt, group, pte, offsets, wg, n_wg, s_off);
    __syncthreads();
    scatter_chunk(ids, 0, Tk, E, s_off, wcnt, perm, inv, status);
}

// T*k > 1024, step 1: per-chunk histograms hist[c][e].
__global__ void __launch_bounds__(kChunk)
k_route_hist(const int32_t* ids, int Tk, int E, int32_t* hist) {
    griddep_wait();
    griddep_launch_dependents();
    __shared__ int32_t s_cnt[MPE_MAX_EXPERTS];
    for (int i = threadIdx.x; i < E; i += kChunk) s_cnt[i] = 0;
    __syncthreads();
    const int a = blockIdx.x * kChunk + threadIdx.x;
    if (a < Tk) {
        const int e = ids[a];
        if (e >= 0 && e < E) atomicAdd(&s_cnt[e], 1);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < E; i += kChunk) hist[(size_t)blockIdx.x * E + i] = s_cnt[i];
}

// Step 2 (one CTA): hist[c][e] <- first position of chunk c's id-e assignments.
__global__ void __launch_bounds__(kChunk)
k_route_scan(int32_t* hist, int n_chunks, int E, int group, const Pte* pte, int32_t* offsets,
             int32_t* wg, int32_t* n_wg, int32_t* zero6) {
    griddep_wait();
    griddep_launch_dependents();
    if (threadIdx.x < 6 && zero6) zero6[threadIdx.x] = 0;
    __shared__ int32_t s_off[MPE_MAX_EXPERTS];
    // small tables (chunks x experts <= kScanSmem) go through shared memory:
    // one coalesced read, the per-expert sums on chip, one coalesced write
    constexpr int kScanSmem = 10240;
    __shared__ int32_t s_h[kScanSmem];
    const int e = threadIdx.x;
    const int n_h = n_chunks * E;
    const bool on_chip = n_h <= kScanSmem;
    int run = 0;
    if (on_chip) {
        for (int i = threadIdx.x; i < n_h; i += kChunk) s_h[i] = hist[i];
        __syncthreads();
        if (e < E)
            for (int c = 0; c < n_chunks; ++c) {
                const int h = s_h[c * E + e];
                s_h[c * E + e] = run;
                run += h;
            }
    } else if (e < E) {
        // eight chunks' counts loaded before their exclusive sums are written
        for (int c0 = 0; c0 < n_chunks; c0 += 8) {
            int h[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) h[u] = c0 + u < n_chunks ? hist[(size_t)(c0 + u) * E + e] : 0;
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                if (c0 + u < n_chunks) hist[(size_t)(c0 + u) * E + e] = run;
                run += h[u];
            }
        }
    }
    offsets_and_groups(E, run, group, pte, offsets, wg, n_wg, s_off);
    __syncthreads();
    if (on_chip) {
        for (int i = threadIdx.x; i < n_h; i += kChunk) hist[i] = s_h[i] + s_off[i % E];
    } else if (e < E) {
        const int off = s_off[e];
#pragma unroll 8
        for (int c = 0; c < n_chunks; ++c) hist[(size_t)c * E + e] += off;
    }
}

// Step 3: stable scatter of each chunk.
__global__ void __launch_bounds__(kChunk)
k_route_scatter(const int32_t* ids, int Tk, int E, const int32_t* hist, int32_t* perm,
                int32_t* inv, uint32_t* status) {
    griddep_wait();
    griddep_launch_dependents();
    extern __shared__ __align__(16) uint8_t sm[];
    uint16_t* wcnt = reinterpret_cast<uint16_t*>(sm);  // [32][E]
    for (int i = threadIdx.x; i < 32 * E; i += kChunk) wcnt[i] = 0;
    __syncthreads();
    const int a0 = blockIdx.x * kChunk;
    scatter_chunk(ids, a0, min(kChunk, Tk - a0), E, hist + (size_t)blockIdx.x * E, wcnt, perm,
                  inv, status);
}

}  // namespace

void launch_route(mpe_ctx* c, const int32_t* ids, int Tk, int k, int32_t* perm,
                  int32_t* offsets, int32_t* inv, int group) {
    (void)k;
    const int E = c->E;
    if (Tk <= kChunk) {
        const size_t sm = 2 * MPE_MAX_EXPERTS * sizeof(int32_t) + 32 * E * sizeof(uint16_t);
        launch_pdl(k_route_small, dim3(1), dim3(kChunk), sm, c->stream, ids, Tk, E, group,
                   (const Pte*)c->d_pte, perm, offsets, inv, c->s.wg, c->s.n_wg, c->d_status,
                   c->s.task_ctr);
        c->launches++;
        return;
    }
    const int nch = (Tk + kChunk - 1) / kChunk;
    launch_pdl(k_route_hist, dim3(nch), dim3(kChunk), 0, c->stream, ids, Tk, E, c->s.hist);
    launch_pdl(k_route_scan, dim3(1), dim3(kChunk), 0, c->stream, c->s.hist, nch, E, group,
               (const Pte*)c->d_pte, offsets, c->s.wg, c->s.n_wg, c->s.task_ctr);
    const size_t sm = 32 * E * sizeof(uint16_t);
    launch_pdl(k_route_scatter, dim3(nch), dim3(kChunk), sm, c->stream, ids, Tk, E,
               (const int32_t*)c->s.hist, perm, inv, c->d_status);
    c->launches += 3;
}

void route_set_smem_limits() {
    const int maxsm = 2 * MPE_MAX_EXPERTS * 4 + 32 * MPE_MAX_EXPERTS * 2;
    cudaFuncSetAttribute(k_route_small, cudaFuncAttributeMaxDynamicSharedMemorySize, maxsm);
    cudaFuncSetAttribute(k_route_scatter, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         32 * MPE_MAX_EXPERTS * 2);
}

}  // namespace mpe

// ---------------------------------------------------------------------------
// No-allocation variant of the bucketing step (mpe_route_noalloc).
//
// Some callers cannot allocate device memory at the point where they route
// tokens: a serving engine that hands the GPU a fixed memory plan up front, or
// code recorded while another component owns the allocator. For them the
// multi-chunk histograms live in one file-scope device array instead of
// context scratch. The array holds up to kNoAllocMaxAssign assignments
// (64 chunks of 1024) for up to MPE_MAX_EXPERTS experts; every GPU that loads
// the library keeps it until the process exits.
// ---------------------------------------------------------------------------
namespace mpe {
int report_global_error(int code, const char* msg);

namespace {

constexpr int kNoAllocMaxAssign = 65536;
constexpr int kNoAllocChunks = kNoAllocMaxAssign / kChunk;
constexpr size_t kNaHistBytes = sizeof(int32_t) * (size_t)kNoAllocChunks * MPE_MAX_EXPERTS;
constexpr size_t kNaWgBytes =
    sizeof(int32_t) * 3 * ((size_t)MPE_MAX_EXPERTS + kNoAllocMaxAssign / kDecodeGroup + 1);
constexpr size_t kNaSmallBytes = 256;  // work-group counts and a status word
constexpr size_t kNaPteBytes = sizeof(Pte) * MPE_MAX_EXPERTS;
constexpr size_t kNaBytes = kNaHistBytes + kNaWgBytes + kNaSmallBytes + kNaPteBytes;

// Shared by every call on a device; the histograms are fully rewritten by each
// call before they are read, and the page-table region is never written (all
// widths 0, so no decode work groups are formed).
static __device__ __align__(256) unsigned char g_route_scratch[kNaBytes];

int noalloc_cuda_error(const char* what, cudaError_t e) {
    char buf[256];
    snprintf(buf, sizeof(buf), "mpe_route_noalloc: %s: %s", what, cudaGetErrorString(e));
    return report_global_error(MPE_ERR_CUDA, buf);
}

// Device address of the array on the current device. Host code may use the
// symbol only through cudaGetSymbolAddress; it is looked up on every call
// (it allocates nothing), so nothing cached can outlive a device reset. The
// kernels' shared-memory limit is set on every call for the same reason.
int noalloc_scratch(unsigned char** out) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_route_scratch);
    if (e != cudaSuccess) return noalloc_cuda_error("cudaGetSymbolAddress failed", e);
    route_set_smem_limits();
    if ((e = cudaGetLastError()) != cudaSuccess)
        return noalloc_cuda_error("setting the shared-memory limit failed", e);
    *out = static_cast<unsigned char*>(p);
    return MPE_OK;
}

}  // namespace
}  // namespace mpe

extern "C" int mpe_route_noalloc(const int32_t* ids, int32_t T, int32_t k, int32_t E,
                                 int32_t* perm, int32_t* offsets, int32_t* inv, void* stream) {
    using namespace mpe;
    if (E < 1 || E > MPE_MAX_EXPERTS || T < 0 || k < 1 || k > 32)
        return report_global_error(MPE_ERR_INVALID, "mpe_route_noalloc: bad E, T or k");
    const long long Tk = (long long)T * k;
    if (!offsets || (Tk > 0 && (!ids || !perm || !inv)))
        return report_global_error(MPE_ERR_INVALID, "mpe_route_noalloc: null pointer");
    if (Tk > kNoAllocMaxAssign) {
        char buf[160];
        snprintf(buf, sizeof(buf),
                 "mpe_route_noalloc: T*k = %lld exceeds the no-allocation maximum of %d",
                 Tk, kNoAllocMaxAssign);
        return report_global_error(MPE_ERR_INVALID, buf);
    }
    // an error left by earlier work on this thread is reported as such (and
    // left pending), not taken for a failure of this call's launches
    const cudaError_t before = cudaPeekAtLastError();
    if (before != cudaSuccess)
        return noalloc_cuda_error("a CUDA error from earlier work is pending", before);
    unsigned char* base = nullptr;
    int rc = noalloc_scratch(&base);
    if (rc != MPE_OK) return rc;
    int32_t* hist = reinterpret_cast<int32_t*>(base);
    int32_t* wg = reinterpret_cast<int32_t*>(base + kNaHistBytes);
    int32_t* n_wg = reinterpret_cast<int32_t*>(base + kNaHistBytes + kNaWgBytes);
    uint32_t* status = reinterpret_cast<uint32_t*>(n_wg + 8);
    const Pte* pte = reinterpret_cast<const Pte*>(base + kNaHistBytes + kNaWgBytes + kNaSmallBytes);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int n = (int)Tk;
    if (n == 0) {
        if (cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (E + 1), st) != cudaSuccess)
            return report_global_error(MPE_ERR_CUDA, "mpe_route_noalloc: memset failed");
        return MPE_OK;
    }
    cudaError_t e;
    if (n <= kChunk) {
        const size_t sm = 2 * MPE_MAX_EXPERTS * sizeof(int32_t) + 32 * E * sizeof(uint16_t);
        k_route_small<<<1, kChunk, sm, st>>>(ids, n, E, kDecodeGroup, pte, perm, offsets, inv, wg,
                                             n_wg, status, nullptr);
        if ((e = cudaGetLastError()) != cudaSuccess)
            return noalloc_cuda_error("launch of k_route_small failed", e);
    } else {
        const int nch = (n + kChunk - 1) / kChunk;
        k_route_hist<<<nch, kChunk, 0, st>>>(ids, n, E, hist);
        if ((e = cudaGetLastError()) != cudaSuccess)
            return noalloc_cuda_error("launch of k_route_hist failed", e);
        k_route_scan<<<1, kChunk, 0, st>>>(hist, nch, E, kDecodeGroup, pte, offsets, wg, n_wg,
                                           nullptr);
        if ((e = cudaGetLastError()) != cudaSuccess)
            return noalloc_cuda_error("launch of k_route_scan failed", e);
        k_route_scatter<<<nch, kChunk, 32 * E * sizeof(uint16_t), st>>>(ids, n, E, hist, perm,
                                                                         inv, status);
        if ((e = cudaGetLastError()) != cudaSuccess)
            return noalloc_cuda_error("launch of k_route_scatter failed", e);
    }
    return MPE_OK;
}
